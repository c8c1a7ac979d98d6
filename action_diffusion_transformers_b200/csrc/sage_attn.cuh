// sage_attn.cuh - quantized attention forward on sm_100a tensor cores.
//
// One CTA computes one 128-row query tile of one (b, h).  Warp roles:
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r).  Per tile it
//              reads its 128 scores from TMEM, reduces their max and min, forms
//              the E4M3 codes of P~ * 448 16 keys at a time (scores re-read from
//              TMEM, the next 16 loaded while the current 16 are processed, so
//              only 32 are live next to the exp2 state), writes them
//              into a 128B-swizzled shared P tile, rescales its row of the O
//              accumulator in TMEM when its row max moves, and runs the
//              epilogue.  Two CTAs share an SM.
// S is accumulated onto the integer 0x4B400000 (the bits of 1.5 * 2^23) that
// the softmax warps write into the S columns before each QK^T MMA: read as a
// float, a loaded S word is then exactly 1.5 * 2^23 + S (|S| <= 127^2 * D <
// 2^22), and the exponent is formed from it directly: u = fma(S + 1.5 * 2^23,
// c, e') with the offset e' = fma(-1.5 * 2^23, c, e) formed once per row and
// 64-key half.
//   warp 4     producer: one thread issues TMA tile loads (Q once; K and V
//              tiles into 2-stage rings).
//   warp 5     MMA: allocates TMEM; one thread issues
//              S  = Qc Kc^T  tcgen05.mma kind::i8      (INT32 accumulate)
//              O += P8 V8    tcgen05.mma kind::f8f6f4  (FP32 accumulate).
// TMEM (256 columns): S at columns [0, 128), O at [128, 128 + D).
// Shared memory: Q (128 x D), K[2] (128 x D), V[2] (D x 128), P (128 x 128),
// all 8-bit, in the tensor-core K-major swizzled layouts (128 B swizzle; the
// D = 64 Q/K tiles use 64 B).
//
// Pipeline per KV tile j: the MMA warp issues S_j as soon as K_j has landed and
// the softmax warps have read S_{j-1} out of TMEM, then issues PV_{j-1} once
// P_{j-1} is in shared memory, so the tensor core computes S_j while the
// softmax of tile j-1 runs.
//
// Every wait is bounded (see mbar_wait_bounded).  On a timeout the CTA raises a
// shared abort flag, every role leaves its loop, the producer waits (bounded)
// for its TMA loads in flight, the MMA thread waits for its tensor-core work,
// TMEM is freed, a device error word is set, and the kernel returns.
#pragma once
#include "sage_ptx.cuh"

namespace sage {

constexpr int kBM = 128;   // query rows per tile
constexpr int kBN = 128;   // keys per tile
constexpr int kAttnThreads = 192;      // 4 softmax warps + producer + MMA
constexpr int kSoftmaxThreads = 128;   // one thread per query row
constexpr int kWarpProducer = 4;
constexpr int kWarpMma = 5;
constexpr int kNumBars = 14;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kSBiasBits = 0x4B400000u;   // S accumulates onto these bits
constexpr float kSBias = 12582912.0f;          // their float value, 1.5 * 2^23
constexpr float kLog2P8 = 8.8073549220576041f; // log2(448): the P scale, folded into the exponent

template <int D>
struct AttnSmem {
  static constexpr int kQBytes = kBM * D;
  static constexpr int kKBytes = kBN * D;
  static constexpr int kVBytes = D * kBN;
  static constexpr int kPBytes = kBM * kBN;
  static constexpr int kQ = 0;
  static constexpr int kK0 = kQ + kQBytes;
  static constexpr int kK1 = kK0 + kKBytes;
  static constexpr int kV0 = kK1 + kKBytes;
  static constexpr int kV1 = kV0 + kVBytes;
  static constexpr int kP = kV1 + kVBytes;
  static constexpr int kVf = kP + kPBytes;     // D floats: v_scale
  static constexpr int kVm = kVf + 4 * D;      // D floats: v_mean
  static constexpr int kBar = kVm + 4 * D;
  static constexpr int kMisc = kBar + kNumBars * 8;  // tmem slot, abort flag
  static constexpr int kTotal = kMisc + 16;
  static constexpr int kAlloc = kTotal + 1024; // slack for 1024-byte alignment
};

struct AttnParams {
  const float* q_scale;   // [B*H, Npad/64] (64-token blocks) or [B*H, Npad] (q_tok)
  const float* k_scale;   // [B*H, Npad/64], or [B*H, Npad] in the kKTok kernel
  const float* v_scale;   // [B*H, D]
  const float* v_mean;    // [B*H, D]
  void* out;              // [B, N, H, D] bf16 or f32
  float* lse;             // [B, H, N] or null
  int* err;               // device error word
  int N, H, Npad, nkv;
  float sl2e;             // sm_scale * log2(e)
  int out_fp32;
  int q_tok;              // q_scale holds one scale per token
  int64_t timeout_ns;
  uint8_t* p_codes;       // [B*H, N, Npad] E4M3 codes of P (sage_attn_p_codes_kernel only)
};

enum : int { kBarQ = 0, kBarKFull = 1, kBarKEmpty = 3, kBarVFull = 5, kBarVEmpty = 7, kBarSFull = 9,
             kBarSEmpty = 10, kBarPFull = 11, kBarPVDone = 12, kBarDrain = 13 };

// Bounded wait whose outcome is the same in every lane of the warp, so that a
// warp never splits in front of a warp-collective tcgen05 instruction.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int64_t timeout_ns) {
  const bool ok = mbar_wait_bounded(bar, parity, abort_flag, timeout_ns);
  return __all_sync(0xFFFFFFFFu, ok);
}

__device__ __forceinline__ float int_to_float(uint32_t s) {
  return __int2float_rn(static_cast<int>(s));
}

// Max over the valid keys and min over all keys of 32 biased scores.
template <bool kMasked>
__device__ __forceinline__ void chunk_minmax(const uint32_t (&a)[32], int valid, float& mx, float& mn) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(a[i]);
  float w[11];
#pragma unroll
  for (int i = 0; i < 10; ++i) w[i] = fmin3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
  w[10] = fminf(v[30], v[31]);
  mn = fminf(fmin3(fmin3(w[0], w[1], w[2]), fmin3(w[3], w[4], w[5]), fmin3(w[6], w[7], w[8])),
             fminf(w[9], w[10]));
  if (kMasked) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i >= valid) v[i] = 0.f;                        // below every biased score
  }
#pragma unroll
  for (int i = 0; i < 10; ++i) w[i] = fmax3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
  w[10] = fmaxf(v[30], v[31]);
  mx = fmaxf(fmax3(fmax3(w[0], w[1], w[2]), fmax3(w[3], w[4], w[5]), fmax3(w[6], w[7], w[8])),
             fmaxf(w[9], w[10]));
}

// Multipliers c and exponent offsets e' = RN(e - 1.5 * 2^23 * c) of a key pair.
struct MulOff {
  f32x2_t c, off;
};

// One multiplier and offset for every key of a quarter (its 64-key half shares
// one K scale).
struct UniformMul {
  MulOff mo;
  __device__ __forceinline__ MulOff operator()(int) const { return mo; }
};

// Per-key multipliers c = RN(RN(qs * ks_j) * sl2e) and their offsets: lane L
// holds ks of key 32 * quarter + L in kq, and a shuffle brings it to every row.
struct KeyMul {
  f32x2_t qs2, sl2e2, e2;
  float kq;
  __device__ __forceinline__ MulOff operator()(int p) const {
    const float k0 = __shfl_sync(0xFFFFFFFFu, kq, 2 * p);
    const float k1 = __shfl_sync(0xFFFFFFFFu, kq, 2 * p + 1);
    const f32x2_t c = x2_mul(x2_mul(x2_pack(__float_as_uint(k0), __float_as_uint(k1)), qs2), sl2e2);
    return MulOff{c, x2_fma(x2_splat(-kSBias), c, e2)};
  }
};

struct HalfMuls {      // keys 0-63 use (c0, off0), keys 64-127 (c1, off1)
  float c0, c1, off0, off1;
  __device__ __forceinline__ UniformMul operator()(int qq) const {
    return UniformMul{MulOff{x2_splat(qq < 2 ? c0 : c1), x2_splat(qq < 2 ? off0 : off1)}};
  }
};

struct KeyMuls {       // per-key scales of the tile's four 32-key quarters
  float qs, sl2e, e;
  const float (&kq)[4];
  __device__ __forceinline__ KeyMul operator()(int qq) const {
    return KeyMul{x2_splat(qs), x2_splat(sl2e), x2_splat(e), kq[qq]};
  }
};

// The contract's exponentials for 16 of this thread's keys, pairs 8 h8 .. 8 h8 + 7
// of a 32-key quarter (biased scores Sb = S + 1.5 * 2^23 as loaded from TMEM;
// `valid` counts from the quarter's first key): u = RN(Sb * c + e') with
// e' = RN(e - 1.5 * 2^23 * c) and e = RN(log2 448 - m_new) (one fused
// multiply-add per key), y = exp2_fixed_x2(u) -> E4M3 code; the row sum
// accumulates y.  Every step is a binary32 operation with fixed rounding, so y
// and its code equal the oracle's bit for bit.  kClamp: some u of this warp's
// tile may be below -126.  pk[w] holds the codes of the chunk's keys 4w .. 4w+3.
// cmul(p) gives the multipliers c and offsets e' of the quarter's keys 2p and
// 2p+1.  Stage-major over the 8 pairs: every step is issued for all 8 before
// the next, so consecutive instructions do not depend on each other.
template <bool kMasked, bool kClamp, class CMul>
__device__ __forceinline__ void softmax_eighth(const uint32_t (&s)[16], const CMul& cmul, int h8, int valid,
                                               const Exp2Consts& k, f32x2_t (&lsum)[4], uint32_t (&pk)[4]) {
  f32x2_t u[8], xr[8], f[8], p[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const auto mo = cmul(8 * h8 + i);
    u[i] = x2_fma(x2_pack(s[2 * i], s[2 * i + 1]), mo.c, mo.off);
  }
  if (kClamp) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      u[i] = x2_pack(__float_as_uint(fmaxf(x2_lo(u[i]), kExp2Min)), __float_as_uint(fmaxf(x2_hi(u[i]), kExp2Min)));
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) xr[i] = x2_add(u[i], k.round);
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = x2_sub(xr[i], k.round);
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] = x2_sub(u[i], f[i]);
#pragma unroll
  for (int i = 0; i < 8; ++i) p[i] = x2_fma(k.c2, f[i], k.c1);
#pragma unroll
  for (int i = 0; i < 8; ++i) p[i] = x2_fma(p[i], f[i], k.c0);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f32x2_t y = x2_add_exponent(p[i], xr[i]);
    if (kMasked) {
      const int j = 8 * h8 + i;
      const uint32_t lo = 2 * j < valid ? static_cast<uint32_t>(y) : 0u;
      const uint32_t hi = 2 * j + 1 < valid ? static_cast<uint32_t>(y >> 32) : 0u;
      y = (static_cast<f32x2_t>(hi) << 32) | lo;
    }
    p[i] = y;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) lsum[i & 3] = x2_add(lsum[i & 3], p[i]);
#pragma unroll
  for (int i = 0; i < 4; ++i) pk[i] = x2_e4m3x4(p[2 * i], p[2 * i + 1]);
}

// The exponential pass over a row's 128 scores in TMEM (taddr), 16 at a time,
// the next 16 columns loaded while the current 16 are processed (two 16-word
// buffers: the same registers as one 32-word chunk); each chunk's 16 codes go
// straight to the row's 128B-swizzled P line (16-byte chunk q of row r lives at
// q ^ (r & 7)).
// kSlow: masked keys or clamped exponents.  muls(qq) gives quarter qq's multipliers.
template <bool kSlow, class Muls>
__device__ __forceinline__ void exp_pass(uint32_t taddr, const Muls& muls, int valid,
                                         const Exp2Consts& ek, f32x2_t (&lsum)[4], uint8_t* prow, int row) {
  uint32_t ra[16], rb[16];
  tmem_ld16(taddr, ra);
  tmem_wait_ld();
  reg_fence16(ra);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t (&cur)[16] = (c & 1) ? rb : ra;
    uint32_t (&nxt)[16] = (c & 1) ? ra : rb;
    if (c < 7) tmem_ld16(taddr + 16 * (c + 1), nxt);
    const int qq = c >> 1;
    uint32_t pk[4];
    softmax_eighth<kSlow, kSlow>(cur, muls(qq), c & 1, valid - 32 * qq, ek, lsum, pk);
    *reinterpret_cast<uint4*>(prow + (c ^ (row & 7)) * 16) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    if (c < 7) {
      tmem_wait_ld();
      reg_fence16(nxt);
    }
  }
}

// Tiles whose K scales differ inside a 64-key half (per-key multipliers; see
// KeyMul); ks points at the tile's 128 per-key scales.
//
// Row max of t = RN(S_j * c_j) over the tile's valid keys.
__device__ __forceinline__ float keywise_tile_max(uint32_t taddr, float qs, float sl2e, const float* ks, int valid) {
  const int lane = threadIdx.x & 31;
  float kq[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) kq[i] = ks[32 * i + lane];
  float tmax = -__int_as_float(0x7F800000);
#pragma unroll
  for (int qq = 0; qq < 4; ++qq) {
    uint32_t cur[32];
    tmem_ld32(taddr + 32 * qq, cur);
    tmem_wait_ld();
    reg_fence(cur);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float c = __fmul_rn(__fmul_rn(qs, __shfl_sync(0xFFFFFFFFu, kq[qq], i)), sl2e);
      const float tv = __fmul_rn(__fsub_rn(__uint_as_float(cur[i]), kSBias), c);
      if (32 * qq + i < valid) tmax = fmaxf(tmax, tv);
    }
  }
  return tmax;
}

// The exponential pass of such a tile (always masked and clamped); returns the
// tile's row sum of y = P~ * 448 as a pair (low + high is the sum).
__device__ __forceinline__ f32x2_t keywise_exp_pass(uint32_t taddr, float qs, float sl2e, const float* ks, float e,
                                                 int valid, uint8_t* prow, int row) {
  const int lane = threadIdx.x & 31;
  float kq[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) kq[i] = ks[32 * i + lane];
  const Exp2Consts ek;
  f32x2_t lsum[4] = {0, 0, 0, 0};
  exp_pass<true>(taddr, KeyMuls{qs, sl2e, e, kq}, valid, ek, lsum, prow, row);
  return x2_add(x2_add(lsum[0], lsum[1]), x2_add(lsum[2], lsum[3]));
}

// One KV tile of a softmax thread's loop (thread = query row).  kKeywise: the
// tile's K scales differ inside a 64-key half, so every key gets its own
// multiplier (and the exponent is always clamped); the two instantiations are
// separate code paths, so the rare per-key tiles leave the register allocation
// of the common tiles alone.  kDumpP: also copy the row's finished P line to
// pdump (the diagnostic kernel).
template <int D, bool kDumpP>
struct SoftmaxTile {
  uint64_t* bars;
  volatile int* abort_flag;
  int64_t tmo;
  uint32_t ts, to;       // this warp's S and O columns in TMEM
  float qs, sl2e;
  const float* ks;       // per-key K scales of the head (per-key tiles only)
  uint8_t* prow;         // this row of the shared P tile
  uint8_t* pdump;        // kDumpP: this row's line of the P-code output (null past N)
  int row;
  float& m;              // running row max of t
  float& l;              // running row sum of P~ * 448

  // Returns false when a bounded wait gave up.
  template <bool kKeywise>
  __device__ __forceinline__ bool step(int j, int valid, float c0, float c1) {
    const Exp2Consts ek;
    if (!warp_wait(&bars[kBarSFull], static_cast<uint32_t>(j) & 1, abort_flag, tmo)) return false;
    tc_fence_after();
    // Row max of t = RN(S * c) (c > 0, so per block it is the max S scaled) and
    // the per-block min S, which bounds every u from below.
    float tmax, smin0 = 0.f, smin1 = 0.f;
    if constexpr (kKeywise) {
      tmax = keywise_tile_max(ts, qs, sl2e, ks + j * kBN, valid);
    } else {
      // Four 32-column loads, each issued while the previous chunk is reduced.
      uint32_t ra[32], rb[32];
      float mx[4], mn[4];
      tmem_ld32(ts, ra);
      tmem_wait_ld();
      reg_fence(ra);
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        uint32_t (&cur)[32] = (qq & 1) ? rb : ra;
        uint32_t (&nxt)[32] = (qq & 1) ? ra : rb;
        if (qq < 3) tmem_ld32(ts + 32 * (qq + 1), nxt);
        if (valid >= kBN)
          chunk_minmax<false>(cur, 32, mx[qq], mn[qq]);
        else
          chunk_minmax<true>(cur, valid - 32 * qq, mx[qq], mn[qq]);
        if (qq < 3) {
          tmem_wait_ld();
          reg_fence(nxt);
        }
      }
      tmax = __fmul_rn(__fsub_rn(fmaxf(mx[0], mx[1]), kSBias), c0);
      if (valid > 64) tmax = fmaxf(tmax, __fmul_rn(__fsub_rn(fmaxf(mx[2], mx[3]), kSBias), c1));
      smin0 = fminf(mn[0], mn[1]);       // biased
      smin1 = fminf(mn[2], mn[3]);
    }
    // Running row max (alpha is exactly 1 while it stays).
    const float m_new = fmaxf(m, tmax);
    const float alpha = exp2_fixed5(__fsub_rn(m, m_new));
    const float e = __fsub_rn(kLog2P8, m_new);
    const float off0 = __fmaf_rn(-kSBias, c0, e);
    const float off1 = __fmaf_rn(-kSBias, c1, e);
    // u is monotone in S (c > 0), so the smallest u of a block is its min S's;
    // clamping is the identity unless that is below -126.
    const bool clamp = kKeywise ||
                       __any_sync(0xFFFFFFFFu, fminf(__fmaf_rn(smin0, c0, off0), __fmaf_rn(smin1, c1, off1)) < kExp2Min);
    // P is single-buffered in shared memory: PV_{j-1} (issued right after QK_j)
    // must have read it before this tile's codes are written.
    if (j > 0 && !warp_wait(&bars[kBarPVDone], static_cast<uint32_t>(j - 1) & 1, abort_flag, tmo)) return false;
    f32x2_t lsum[4] = {0, 0, 0, 0};
    if constexpr (kKeywise)
      lsum[0] = keywise_exp_pass(ts, qs, sl2e, ks + j * kBN, e, valid, prow, row);
    else if (valid >= kBN && !clamp)
      exp_pass<false>(ts, HalfMuls{c0, c1, off0, off1}, kBN, ek, lsum, prow, row);
    else
      exp_pass<true>(ts, HalfMuls{c0, c1, off0, off1}, valid, ek, lsum, prow, row);
    if constexpr (kDumpP) {
      // The thread's own P line, unswizzled: keys j * 128 + 16 c .. + 15 in chunk c.
      if (pdump != nullptr) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          reinterpret_cast<uint4*>(pdump + j * kBN)[c] = *reinterpret_cast<const uint4*>(prow + (c ^ (row & 7)) * 16);
      }
    }
    // Re-seed S with the bias for the next tile's MMA, then release the buffer.
    tmem_fill64(ts, kSBiasBits);
    tmem_fill64(ts + 64, kSBiasBits);
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&bars[kBarSEmpty]);
    const f32x2_t ls2 = x2_add(x2_add(lsum[0], lsum[1]), x2_add(lsum[2], lsum[3]));
    l = __fadd_rn(__fmul_rn(l, alpha), __fadd_rn(x2_lo(ls2), x2_hi(ls2)));

    if (j > 0 && __any_sync(0xFFFFFFFFu, alpha != 1.f)) {
      tc_fence_after();
      const f32x2_t a2 = x2_splat(alpha);
#pragma unroll
      for (int cb = 0; cb < D; cb += 32) {
        f32x2_t o[16];
        tmem_ld32_pairs(to + cb, o);
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] = x2_mul(o[i], a2);
        tmem_st32_pairs(to + cb, o);
      }
      tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(&bars[kBarPFull]);
    m = m_new;
    return true;
  }
};

// kKTok: k_scale holds one scale per key (per-token or segment-local K
// scales).  A tile whose K scales are equal within each 64-key half (the usual
// case) runs exactly as with 64-token blocks; any other tile takes per-key
// multipliers and always clamps.
// kDumpP: the diagnostic form, which also writes every E4M3 code of P to
// prm.p_codes; the product kernel is the kDumpP = false instantiation.
template <int D, bool kKTok, bool kDumpP>
__device__ __forceinline__ void attn_cta(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                         const AttnParams& prm) {
  using L = AttnSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  float* s_vf = reinterpret_cast<float*>(smem + L::kVf);
  float* s_vm = reinterpret_cast<float*>(smem + L::kVm);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int qt = blockIdx.x;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int bh = b * prm.H + h;
  const int nkv = prm.nkv;
  const int64_t tmo = prm.timeout_ns;

  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      uint32_t count = 1u;
      if (i == kBarSEmpty || i == kBarPFull) count = kSoftmaxThreads;
      mbar_init(&bars[i], count);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < D; i += kAttnThreads) {
    s_vf[i] = prm.v_scale[static_cast<int64_t>(bh) * D + i];
    s_vm[i] = prm.v_mean[static_cast<int64_t>(bh) * D + i];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_s = tmem;
  const uint32_t tmem_o = tmem + 128;

  if (warp == kWarpProducer) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int issued = 0;  // KV tiles whose loads were issued
      mbar_arrive_expect_tx(&bars[kBarQ], L::kQBytes);
      tma_load_2d(smem + L::kQ, &tm_q, 0, bh * prm.Npad + qt * kBM, &bars[kBarQ]);
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        const uint32_t use = static_cast<uint32_t>(j >> 1);
        if (j >= 2 && !mbar_wait_bounded(&bars[kBarKEmpty + st], (use - 1) & 1, abort_flag, tmo)) break;
        mbar_arrive_expect_tx(&bars[kBarKFull + st], L::kKBytes);
        tma_load_2d(smem + (st ? L::kK1 : L::kK0), &tm_k, 0, bh * prm.Npad + j * kBN, &bars[kBarKFull + st]);
        if (j >= 2 && !mbar_wait_bounded(&bars[kBarVEmpty + st], (use - 1) & 1, abort_flag, tmo)) {
          issued = -(j + 1);  // K_j issued, V_j not
          break;
        }
        mbar_arrive_expect_tx(&bars[kBarVFull + st], L::kVBytes);
        tma_load_2d(smem + (st ? L::kV1 : L::kV0), &tm_v, j * kBN, bh * D, &bars[kBarVFull + st]);
        issued = j + 1;
      }
      if (*abort_flag) {
        // Drain: wait (bounded) for Q and for the last load issued into each
        // ring slot; a slot's full barrier only moves when its load lands.
        const int64_t drain = 200000000;  // 200 ms
        int no_abort = 0;
        volatile int* nf = reinterpret_cast<volatile int*>(&no_abort);
        mbar_wait_bounded(&bars[kBarQ], 0, nf, drain);
        const int nk = issued >= 0 ? issued : -issued;      // K loads issued
        const int nv = issued >= 0 ? issued : -issued - 1;  // V loads issued
        for (int st = 0; st < 2; ++st) {
          if (nk > st) {
            const int last = ((nk - 1 - st) / 2) * 2 + st;
            mbar_wait_bounded(&bars[kBarKFull + st], static_cast<uint32_t>(last >> 1) & 1, nf, drain);
          }
          if (nv > st) {
            const int last = ((nv - 1 - st) / 2) * 2 + st;
            mbar_wait_bounded(&bars[kBarVFull + st], static_cast<uint32_t>(last >> 1) & 1, nf, drain);
          }
        }
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescQK = make_idesc(2u, 1u, 128u, 128u);          // S32 <- S8 x S8
      constexpr uint32_t kIdescPV = make_idesc(1u, 0u, 128u, static_cast<uint32_t>(D));  // F32 <- E4M3
      constexpr uint32_t kQKSbo = D == 128 ? 1024u : 512u;
      constexpr uint32_t kQKSwz = D == 128 ? 2u : 4u;
      const uint64_t qdesc = make_sdesc(smem_u32(smem + L::kQ), kQKSbo, kQKSwz);
      const uint64_t kdesc0 = make_sdesc(smem_u32(smem + L::kK0), kQKSbo, kQKSwz);
      const uint64_t kdesc1 = make_sdesc(smem_u32(smem + L::kK1), kQKSbo, kQKSwz);
      const uint64_t pdesc = make_sdesc(smem_u32(smem + L::kP), 1024u, 2u);
      const uint64_t vdesc0 = make_sdesc(smem_u32(smem + L::kV0), 1024u, 2u);
      const uint64_t vdesc1 = make_sdesc(smem_u32(smem + L::kV1), 1024u, 2u);
      bool ok = mbar_wait_bounded(&bars[kBarQ], 0, abort_flag, tmo);
      for (int j = 0; ok && j <= nkv; ++j) {
        if (j < nkv) {
          const int st = j & 1;
          if (!mbar_wait_bounded(&bars[kBarKFull + st], static_cast<uint32_t>(j >> 1) & 1, abort_flag, tmo)) break;
          // Completion j of S-empty: the softmax warps have re-seeded S with the bias.
          if (!mbar_wait_bounded(&bars[kBarSEmpty], static_cast<uint32_t>(j) & 1, abort_flag, tmo)) break;
          tc_fence_after();
          const uint64_t kd = st ? kdesc1 : kdesc0;
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            mma_i8_ss(tmem_s, qdesc + 2u * kk, kd + 2u * kk, kIdescQK, 1u);
          tc_commit(&bars[kBarKEmpty + st]);
          tc_commit(&bars[kBarSFull]);
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int st = jj & 1;
          if (!mbar_wait_bounded(&bars[kBarPFull], static_cast<uint32_t>(jj) & 1, abort_flag, tmo)) break;
          if (!mbar_wait_bounded(&bars[kBarVFull + st], static_cast<uint32_t>(jj >> 1) & 1, abort_flag, tmo))
            break;
          tc_fence_after();
          const uint64_t vd = st ? vdesc1 : vdesc0;
#pragma unroll
          for (int kk = 0; kk < kBN / 32; ++kk)
            mma_f8_ss(tmem_o, pdesc + 2u * kk, vd + 2u * kk, kIdescPV, (jj > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&bars[kBarVEmpty + st]);
          tc_commit(&bars[kBarPVDone]);
        }
      }
      // Wait for every tensor-core operation issued above before TMEM is freed.
      tc_commit(&bars[kBarDrain]);
      int dummy = 0;
      mbar_wait_bounded(&bars[kBarDrain], 0, reinterpret_cast<volatile int*>(&dummy), 200000000);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int row = tid;                          // TMEM lane == query row in tile
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t ts = tmem_s + lane_base;
    const uint32_t to = tmem_o + lane_base;
    const int nqb = prm.Npad / 64;
    const float qs = prm.q_tok ? prm.q_scale[static_cast<int64_t>(bh) * prm.Npad + qt * kBM + row]
                               : prm.q_scale[static_cast<int64_t>(bh) * nqb + qt * 2 + (row >> 6)];
    const float* ks = prm.k_scale + static_cast<int64_t>(bh) * (kKTok ? prm.Npad : nqb);
    const float sl2e = prm.sl2e;
    uint8_t* sP = smem + L::kP;
    const float kNegInf = -__int_as_float(0x7F800000);
    float m = kNegInf;
    float l = 0.f;                                // sum of P~ * 448
    bool ok = true;
    static_assert(kSBias == kExp2Round, "the S bias doubles as the exp2 rounding constant");
    // Seed S with the bias and release it for the first QK^T MMA.
    tmem_fill64(ts, kSBiasBits);
    tmem_fill64(ts + 64, kSBiasBits);
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&bars[kBarSEmpty]);
    uint8_t* pdump = nullptr;
    if constexpr (kDumpP) {
      if (qt * kBM + row < prm.N) pdump = prm.p_codes + (static_cast<int64_t>(bh) * prm.N + qt * kBM + row) * prm.Npad;
    }
    SoftmaxTile<D, kDumpP> tile{bars, abort_flag, tmo, ts, to, qs, sl2e, ks, sP + row * 128, pdump, row, m, l};
    for (int j = 0; j < nkv; ++j) {
      const int valid = min(kBN, prm.N - j * kBN);   // valid keys in this tile
      float c0, c1;
      bool keywise = false;      // kKTok: a 64-key half mixes K scales
      if constexpr (kKTok) {
        float kq[4];             // lane L: the scale of key 32 * i + L in kq[i]
#pragma unroll
        for (int i = 0; i < 4; ++i) kq[i] = ks[j * kBN + 32 * i + lane];
        const float f0 = __shfl_sync(0xFFFFFFFFu, kq[0], 0);    // key 0 (always valid)
        const float f1 = __shfl_sync(0xFFFFFFFFu, kq[2], 0);    // key 64
        bool same = true;
#pragma unroll
        for (int i = 0; i < 4; ++i) same = same && (32 * i + lane >= valid || kq[i] == (i < 2 ? f0 : f1));
        keywise = !__all_sync(0xFFFFFFFFu, same);
        c0 = __fmul_rn(__fmul_rn(qs, f0), sl2e);
        c1 = __fmul_rn(__fmul_rn(qs, f1), sl2e);
      } else {
        // Keys 0-63 and 64-127 of the tile are two scale blocks.
        c0 = __fmul_rn(__fmul_rn(qs, ks[2 * j]), sl2e);
        c1 = __fmul_rn(__fmul_rn(qs, ks[2 * j + 1]), sl2e);
      }
      if (kKTok && keywise) {
        if (!tile.template step<true>(j, valid, c0, c1)) {
          ok = false;
          break;
        }
      } else if (!tile.template step<false>(j, valid, c0, c1)) {
        ok = false;
        break;
      }
    }
    if (ok && warp_wait(&bars[kBarPVDone], static_cast<uint32_t>(nkv - 1) & 1, abort_flag, tmo)) {
      tc_fence_after();
      const int qrow = qt * kBM + row;
      // O_acc ~ sum_k P8_k * code_k with P8 ~ 448 P~ and l = sum 448 P~:
      // O = RN(O_acc * v_scale) * RN(1 / l) + v_mean (one fused multiply-add).
      const float rl = __fdiv_rn(1.f, l);
      const int64_t obase = ((static_cast<int64_t>(b) * prm.N + qrow) * prm.H + h) * D;
#pragma unroll
      for (int cb = 0; cb < D; cb += 32) {
        uint32_t o[32];
        tmem_ld32(to + cb, o);
        tmem_wait_ld();
        reg_fence(o);
        float r[32];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 t = fmul2(make_float2(__uint_as_float(o[i]), __uint_as_float(o[i + 1])),
                                 make_float2(s_vf[cb + i], s_vf[cb + i + 1]));
          const float2 u = ffma2(t, make_float2(rl, rl), make_float2(s_vm[cb + i], s_vm[cb + i + 1]));
          r[i] = u.x;
          r[i + 1] = u.y;
        }
        if (qrow < prm.N) {
          if (prm.out_fp32) {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(prm.out) + obase + cb);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(prm.out) + obase + cb);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint32_t w[4];
#pragma unroll
              for (int k2 = 0; k2 < 4; ++k2)
                w[k2] = float_to_bf16_bits(r[8 * i + 2 * k2]) | (float_to_bf16_bits(r[8 * i + 2 * k2 + 1]) << 16);
              dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
      if (prm.lse && qrow < prm.N)
        prm.lse[static_cast<int64_t>(bh) * prm.N + qrow] = (m + log2f(l) - kLog2P8) * 0.69314718055994531f;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && tid == 0) atomicExch(prm.err, 1);
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool kKTok>
__global__ void __launch_bounds__(kAttnThreads, 2)
    sage_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const AttnParams prm) {
  pdl_enter();
  attn_cta<D, kKTok, false>(tm_q, tm_k, tm_v, prm);
}

// The same attention, plus the E4M3 code of every P~ * 448 at
// prm.p_codes[(bh * N + row) * Npad + key] (keys past N: 0).  For tests.
template <int D, bool kKTok>
__global__ void __launch_bounds__(kAttnThreads, 2)
    sage_attn_p_codes_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const AttnParams prm) {
  pdl_enter();
  attn_cta<D, kKTok, true>(tm_q, tm_k, tm_v, prm);
}

}  // namespace sage
