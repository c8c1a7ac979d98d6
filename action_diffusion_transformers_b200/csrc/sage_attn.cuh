// sage_attn.cuh - quantized attention forward on sm_100a tensor cores.
//
// One CTA computes one 128-row query tile of one (b, h).  Warp roles:
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r); reads S from
//              TMEM, runs the FP32 online softmax, writes P as E4M3 into a
//              128B-swizzled shared tile, rescales the O accumulator in TMEM
//              when its row max moves, and runs the epilogue.
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
constexpr int kAttnThreads = 192;
constexpr uint32_t kTmemCols = 256;

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
  static constexpr int kVf = kP + kPBytes;     // D floats: v_scale / 448
  static constexpr int kVm = kVf + 4 * D;      // D floats: v_mean
  static constexpr int kBar = kVm + 4 * D;     // 16 mbarriers
  static constexpr int kMisc = kBar + 16 * 8;  // tmem slot, abort flag
  static constexpr int kTotal = kMisc + 16;
  static constexpr int kAlloc = kTotal + 1024; // slack for 1024-byte alignment
};

struct AttnParams {
  const float* q_scale;   // [B*H, Npad/64]
  const float* k_scale;   // [B*H, Npad/64]
  const float* v_scale;   // [B*H, D]
  const float* v_mean;    // [B*H, D]
  void* out;              // [B, N, H, D] bf16 or f32
  float* lse;             // [B, H, N] or null
  int* err;               // device error word
  int N, H, Npad, nkv;
  float sl2e;             // sm_scale * log2(e)
  int out_fp32;
  int64_t timeout_ns;
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

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    sage_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const AttnParams prm) {
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

  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < 16; ++i) mbar_init(&bars[i], (i == kBarSEmpty || i == kBarPFull) ? 128u : 1u);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < D; i += kAttnThreads) {
    s_vf[i] = __fdiv_rn(prm.v_scale[static_cast<int64_t>(bh) * D + i], 448.f);
    s_vm[i] = prm.v_mean[static_cast<int64_t>(bh) * D + i];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_s = tmem;
  const uint32_t tmem_o = tmem + 128;

  if (warp == 4) {
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
  } else if (warp == 5) {
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
          if (j >= 1 && !mbar_wait_bounded(&bars[kBarSEmpty], static_cast<uint32_t>(j - 1) & 1, abort_flag, tmo))
            break;
          tc_fence_after();
          const uint64_t kd = st ? kdesc1 : kdesc0;
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            mma_i8_ss(tmem_s, qdesc + 2u * kk, kd + 2u * kk, kIdescQK, kk > 0 ? 1u : 0u);
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
    const int nqb = prm.Npad / 64;
    const float qs = prm.q_scale[static_cast<int64_t>(bh) * nqb + qt * 2 + (row >> 6)];
    const float* ks = prm.k_scale + static_cast<int64_t>(bh) * nqb;
    const float sl2e = prm.sl2e;
    uint8_t* sP = smem + L::kP;
    float m = -__int_as_float(0x7F800000);
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const float c0 = __fmul_rn(__fmul_rn(qs, ks[2 * j]), sl2e);
      const float c1 = __fmul_rn(__fmul_rn(qs, ks[2 * j + 1]), sl2e);
      if (!warp_wait(&bars[kBarSFull], static_cast<uint32_t>(j) & 1, abort_flag, tmo)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sa[32], sb[32], sc[32], sd[32];
      tmem_ld32(tmem_s + lane_base + 0, sa);
      tmem_ld32(tmem_s + lane_base + 32, sb);
      tmem_ld32(tmem_s + lane_base + 64, sc);
      tmem_ld32(tmem_s + lane_base + 96, sd);
      tmem_wait_ld();
      reg_fence(sa);
      reg_fence(sb);
      reg_fence(sc);
      reg_fence(sd);
      tc_fence_before();
      mbar_arrive(&bars[kBarSEmpty]);

      const int valid = min(kBN, prm.N - j * kBN);
      int ia = INT_MIN, ib = INT_MIN;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        if (k < valid) ia = max(ia, static_cast<int>(sa[k]));
        if (k + 32 < valid) ia = max(ia, static_cast<int>(sb[k]));
        if (k + 64 < valid) ib = max(ib, static_cast<int>(sc[k]));
        if (k + 96 < valid) ib = max(ib, static_cast<int>(sd[k]));
      }
      float tmax = -__int_as_float(0x7F800000);
      if (valid > 0) tmax = __fmul_rn(__int2float_rn(ia), c0);
      if (valid > 64) tmax = fmaxf(tmax, __fmul_rn(__int2float_rn(ib), c1));
      const float m_new = fmaxf(m, tmax);
      const float alpha = ex2_approx(__fsub_rn(m, m_new));
      const float neg = -m_new;
      float sum = 0.f;
      uint32_t pk[32];  // 128 E4M3 codes, 4 per word, key order
#pragma unroll
      for (int w = 0; w < 32; ++w) {
        const uint32_t* src = w < 8 ? sa : (w < 16 ? sb : (w < 24 ? sc : sd));
        const float c = w < 16 ? c0 : c1;
        float p[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int key = 4 * w + i;
          const float pv = ex2_approx(__fmaf_rn(int_to_float(src[(4 * w + i) & 31]), c, neg));
          p[i] = key < valid ? pv : 0.f;
          sum = __fadd_rn(sum, p[i]);
        }
        pk[w] = cvt_e4m3x2(__fmul_rn(p[0], 448.f), __fmul_rn(p[1], 448.f)) |
                (cvt_e4m3x2(__fmul_rn(p[2], 448.f), __fmul_rn(p[3], 448.f)) << 16);
      }
      l = __fadd_rn(__fmul_rn(l, alpha), sum);

      if (j > 0 && !warp_wait(&bars[kBarPVDone], static_cast<uint32_t>(j - 1) & 1, abort_flag, tmo)) {
        ok = false;
        break;
      }
      // P row -> shared tile, 128B swizzle: 16-byte chunk c of row r lives at c ^ (r & 7).
      uint8_t* prow = sP + row * 128;
#pragma unroll
      for (int cch = 0; cch < 8; ++cch) {
        const int pc = cch ^ (row & 7);
        *reinterpret_cast<uint4*>(prow + pc * 16) =
            make_uint4(pk[4 * cch], pk[4 * cch + 1], pk[4 * cch + 2], pk[4 * cch + 3]);
      }
      if (j > 0 && __any_sync(0xFFFFFFFFu, alpha != 1.f)) {
        tc_fence_after();
#pragma unroll
        for (int cb = 0; cb < D; cb += 32) {
          uint32_t o[32];
          tmem_ld32(tmem_o + lane_base + cb, o);
          tmem_wait_ld();
          reg_fence(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__fmul_rn(__uint_as_float(o[i]), alpha));
          tmem_st32(tmem_o + lane_base + cb, o);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[kBarPFull]);
      m = m_new;
    }
    if (ok && warp_wait(&bars[kBarPVDone], static_cast<uint32_t>(nkv - 1) & 1, abort_flag, tmo)) {
      tc_fence_after();
      const int qrow = qt * kBM + row;
      const float rl = __fdiv_rn(1.f, l);
      const int64_t obase = ((static_cast<int64_t>(b) * prm.N + qrow) * prm.H + h) * D;
#pragma unroll
      for (int cb = 0; cb < D; cb += 32) {
        uint32_t o[32];
        tmem_ld32(tmem_o + lane_base + cb, o);
        tmem_wait_ld();
        reg_fence(o);
        float r[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
          r[i] = __fadd_rn(__fmul_rn(__fmul_rn(__uint_as_float(o[i]), s_vf[cb + i]), rl), s_vm[cb + i]);
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
        prm.lse[static_cast<int64_t>(bh) * prm.N + qrow] = (m + log2f(l)) * 0.69314718055994531f;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && tid == 0) atomicExch(prm.err, 1);
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace sage
