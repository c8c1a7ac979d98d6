// fp8_linear.cuh - the row-wise FP8 projection on sm_100a tensor cores:
//   y[m, n] = RN(RN(acc[m, n] * sx[m]) * sw[n]),  acc = sum_k xq[m, k] * wq[n, k]
// with E4M3 activations quantized per token (row of X) and E4M3 weights with
// one scale per output row (row of W), FP32 accumulation in tensor memory.
//
//  fp8_quant_rows_kernel  one CTA per row: absmax, scale = RN(amax/448),
//                         inv = RN(448/amax), codes = E4M3(RN(x * inv)).
//  fp8_gemm_kernel        persistent, one CTA per SM over 128 x 256 output
//                         (or 128 x 192) tiles; when the last wave would be
//                         mostly empty, its tiles are split into 2 or 4
//                         narrower column blocks, so that more SMs share it.  Warp 0 issues TMA loads of
//                         128 x 128 A and BN x 128 B tiles into a 4- or 5-stage
//                         ring; warp 1 issues tcgen05.mma kind::f8f6f4 (M 128,
//                         N BN, K 32) into one of two BN-column TMEM
//                         accumulators; warps
//                         2-5 (one per TMEM lane quadrant) read the other
//                         accumulator, apply the two scales and store BF16 or
//                         FP32, so a tile's epilogue overlaps the next tile's
//                         products.  Every wait is bounded as in the attention
//                         kernel.
#pragma once
#include "sage_ptx.cuh"
#include "sage_quant.cuh"

namespace sage {

// ----------------------------------------------------------------------------
// Per-row E4M3 quantization.  K % 8 == 0; row stride ld (elements, % 8 == 0).
// kChunks 16-byte pieces per thread cover K <= kChunks * 8 * 128.
// ----------------------------------------------------------------------------
constexpr int kFqThreads = 128;

template <int kChunks>
__global__ void __launch_bounds__(kFqThreads) fp8_quant_rows_kernel(const uint16_t* __restrict__ x, int K,
                                                                    int64_t ld, uint8_t* __restrict__ codes,
                                                                    float* __restrict__ scale) {
  pdl_enter();
  __shared__ float red[kFqThreads / 32];
  const int r = blockIdx.x;
  const uint16_t* row = x + static_cast<int64_t>(r) * ld;
  const int nch = K / 8;
  uint4 raw[kChunks];
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    const int j = threadIdx.x + c * kFqThreads;
    raw[c] = j < nch ? ld_nc_16(row + 8 * j) : make_uint4(0u, 0u, 0u, 0u);
  }
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    float f[8];
    unpack8(raw[c], f);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  float a = red[0];
#pragma unroll
  for (int w = 1; w < kFqThreads / 32; ++w) a = fmaxf(a, red[w]);
  float inv = 0.f;
  if (a > 0.f) inv = __fdiv_rn(448.f, a);
  uint8_t* out = codes + static_cast<int64_t>(r) * K;
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    const int j = threadIdx.x + c * kFqThreads;
    if (j < nch) {
      float f[8];
      unpack8(raw[c], f);
      uint32_t w[2];
#pragma unroll
      for (int h = 0; h < 2; ++h)
        w[h] = cvt_e4m3x2(__fmul_rn(f[4 * h], inv), __fmul_rn(f[4 * h + 1], inv)) |
               (cvt_e4m3x2(__fmul_rn(f[4 * h + 2], inv), __fmul_rn(f[4 * h + 3], inv)) << 16);
      *reinterpret_cast<uint2*>(out + 8 * j) = make_uint2(w[0], w[1]);
    }
  }
  if (threadIdx.x == 0) scale[r] = a > 0.f ? __fdiv_rn(a, 448.f) : 0.f;
}

// ----------------------------------------------------------------------------
// Persistent FP8 GEMM with row-wise scales.
// ----------------------------------------------------------------------------
constexpr int kGemmBM = 128;        // rows of X per tile (TMEM lanes)
constexpr int kGemmBK = 128;        // K bytes (= E4M3 elements) per stage: one 128 B swizzle row
constexpr int kGemmThreads = 192;   // producer, MMA, 4 epilogue warps

// BN rows of W per tile (TMEM columns per accumulator): 256, or 192 where it
// fills the last wave of the persistent grid better.  Stages: as many 16 KB +
// BN * 128 B ring slots as fit next to the barriers.
template <int BN>
struct GemmSmem {
  static constexpr int kStages = BN == 256 ? 4 : 5;
  static constexpr int kABytes = kGemmBM * kGemmBK;
  static constexpr int kBBytes = BN * kGemmBK;
  static constexpr int kA = 0;
  static constexpr int kB = kA + kStages * kABytes;
  static constexpr int kBar = kB + kStages * kBBytes;
  // full[S], empty[S], acc_full[2], acc_empty[2], drain
  static constexpr int kFull = 0, kEmpty = kStages, kAccFull = 2 * kStages, kAccEmpty = 2 * kStages + 2,
                       kDrain = 2 * kStages + 4;
  static constexpr int kNumBars = 2 * kStages + 5;
  static constexpr int kMisc = kBar + kNumBars * 8;   // tmem slot, abort flag
  static constexpr int kTotal = kMisc + 16;
  static constexpr int kAlloc = kTotal + 1024;        // slack for 1024-byte alignment
};

struct GemmParams {
  const float* sx;     // [M] per-token activation scales
  const float* sw;     // [N] per-output-row weight scales
  void* out;           // [M, N] BF16 or FP32, row-major
  int M, N, K;
  int out_fp32;
  int* err;            // device error word
  int64_t timeout_ns;
  int tail_start;      // work units below this are whole tiles (unit = tile)
  int tail_split;      // each tile from tail_start on is this many column blocks (1, 2 or 4)
};

// Work unit -> output block (row tile tm, first column n0, width nw): units
// below tail_start are whole tiles; unit tail_start + q is column block
// q % tail_split of tile tail_start + q / tail_split (kTail only).
template <int BN, bool kTail>
__device__ __forceinline__ void gemm_unit(const GemmParams& prm, int ntn, int unit, int& tm, int& n0, int& nw) {
  int tile = unit, sub = 0;
  nw = BN;
  if (kTail && unit >= prm.tail_start) {
    const int q = unit - prm.tail_start;
    tile = prm.tail_start + q / prm.tail_split;
    sub = q % prm.tail_split;
    nw = BN / prm.tail_split;
  }
  tm = tile / ntn;
  n0 = (tile % ntn) * BN + sub * nw;
}

// tm_b_tail: the W map with a box of BN / tail_split rows (the column blocks).
// kTail: the last wave is split (prm.tail_split > 1); without it the kernel
// runs whole tiles only and never reads tm_b_tail.
template <int BN, bool kTail>
__global__ void __launch_bounds__(kGemmThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_b_tail, const GemmParams prm) {
  pdl_enter();
  using L = GemmSmem<BN>;
  constexpr int kGemmBN = BN;
  constexpr int kGemmStages = L::kStages;
  constexpr uint32_t kTmemCols = 2 * BN <= 256 ? 256u : 512u;   // power of two
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int ntm = (prm.M + kGemmBM - 1) / kGemmBM;
  const int ntn = (prm.N + kGemmBN - 1) / kGemmBN;
  const int ntiles = ntm * ntn;
  const int nunits = kTail ? prm.tail_start + (ntiles - prm.tail_start) * prm.tail_split : ntiles;
  const int nk = (prm.K + kGemmBK - 1) / kGemmBK;
  const int64_t tmo = prm.timeout_ns;

  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < L::kNumBars; ++i)
      mbar_init(&bars[i], (i >= L::kAccEmpty && i < L::kAccEmpty + 2) ? 4 * 32 : 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      if (kTail) tma_prefetch_desc(&tm_b_tail);
      uint32_t it = 0;          // stage uses issued, over all units
      for (int unit = blockIdx.x; unit < nunits && !*abort_flag; unit += gridDim.x) {
        int tm, n0, nw;
        gemm_unit<kGemmBN, kTail>(prm, ntn, unit, tm, n0, nw);
        const CUtensorMap* mb = (!kTail || nw == kGemmBN) ? &tm_b : &tm_b_tail;
        const uint32_t bytes = static_cast<uint32_t>(L::kABytes + nw * kGemmBK);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = static_cast<int>(it % kGemmStages);
          const uint32_t use = it / kGemmStages;
          if (use > 0 && !mbar_wait_bounded(&bars[L::kEmpty + s], (use - 1) & 1, abort_flag, tmo)) break;
          mbar_arrive_expect_tx(&bars[L::kFull + s], bytes);
          tma_load_2d(smem + L::kA + s * L::kABytes, &tm_a, kb * kGemmBK, tm * kGemmBM, &bars[L::kFull + s]);
          tma_load_2d(smem + L::kB + s * L::kBBytes, mb, kb * kGemmBK, n0, &bars[L::kFull + s]);
        }
      }
      if (*abort_flag) {
        // Drain: wait (bounded) for the last load issued into each ring slot.
        int no_abort = 0;
        volatile int* nf = reinterpret_cast<volatile int*>(&no_abort);
        for (uint32_t s = 0; s < kGemmStages; ++s) {
          if (it > s) {
            const uint32_t last = ((it - 1 - s) / kGemmStages) * kGemmStages + s;
            mbar_wait_bounded(&bars[L::kFull + s], (last / kGemmStages) & 1, nf, 200000000);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdesc = make_idesc(1u, 0u, kGemmBM, kGemmBN);   // F32 <- E4M3 x E4M3
      const uint32_t idesc_tail = kTail ? make_idesc(1u, 0u, kGemmBM, static_cast<uint32_t>(kGemmBN / prm.tail_split))
                                        : kIdesc;
      uint32_t it = 0;
      uint32_t acc_it = 0;
      bool ok = true;
      for (int unit = blockIdx.x; ok && unit < nunits; unit += gridDim.x, ++acc_it) {
        const uint32_t idesc = (kTail && unit >= prm.tail_start) ? idesc_tail : kIdesc;
        const uint32_t buf = acc_it & 1;
        const uint32_t use = acc_it >> 1;
        if (use > 0 && !mbar_wait_bounded(&bars[L::kAccEmpty + buf], (use - 1) & 1, abort_flag, tmo)) break;
        tc_fence_after();
        const uint32_t d = tmem + buf * kGemmBN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = static_cast<int>(it % kGemmStages);
          if (!mbar_wait_bounded(&bars[L::kFull + s], (it / kGemmStages) & 1, abort_flag, tmo)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = make_sdesc(smem_u32(smem + L::kA + s * L::kABytes), 1024u, 2u);
          const uint64_t bd = make_sdesc(smem_u32(smem + L::kB + s * L::kBBytes), 1024u, 2u);
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 32; ++kk)
            mma_f8_ss(d, ad + 2u * kk, bd + 2u * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&bars[L::kEmpty + s]);
        }
        if (ok) tc_commit(&bars[L::kAccFull + buf]);
      }
      // Wait for every tensor-core operation issued above before TMEM is freed.
      tc_commit(&bars[L::kDrain]);
      int dummy = 0;
      mbar_wait_bounded(&bars[L::kDrain], 0, reinterpret_cast<volatile int*>(&dummy), 200000000);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;                         // TMEM lanes 32*quad .. +31
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    uint32_t acc_it = 0;
    for (int unit = blockIdx.x; unit < nunits; unit += gridDim.x, ++acc_it) {
      const uint32_t buf = acc_it & 1;
      // the outcome is made the same in every lane before the warp-collective TMEM loads
      const bool ok = mbar_wait_bounded(&bars[L::kAccFull + buf], (acc_it >> 1) & 1, abort_flag, tmo);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      tc_fence_after();
      int tm, nb, nw;
      gemm_unit<kGemmBN, kTail>(prm, ntn, unit, tm, nb, nw);
      const int m = tm * kGemmBM + quad * 32 + lane;
      const float sxm = m < prm.M ? prm.sx[m] : 0.f;
#pragma unroll 1
      for (int cb = 0; cb < (kTail ? nw : kGemmBN); cb += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + buf * kGemmBN + cb + lane_base, r);
        tmem_wait_ld();
        reg_fence(r);
        const int n0 = nb + cb;
        if (n0 >= prm.N) continue;                     // the same for the whole warp
        float y[32];
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          const float4 s4 = n0 + i < prm.N ? *reinterpret_cast<const float4*>(prm.sw + n0 + i)
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
          y[i] = __fmul_rn(__fmul_rn(__uint_as_float(r[i]), sxm), s4.x);
          y[i + 1] = __fmul_rn(__fmul_rn(__uint_as_float(r[i + 1]), sxm), s4.y);
          y[i + 2] = __fmul_rn(__fmul_rn(__uint_as_float(r[i + 2]), sxm), s4.z);
          y[i + 3] = __fmul_rn(__fmul_rn(__uint_as_float(r[i + 3]), sxm), s4.w);
        }
        if (m < prm.M) {
          const int64_t o = static_cast<int64_t>(m) * prm.N + n0;
          if (prm.out_fp32) {
            float* dst = reinterpret_cast<float*>(prm.out) + o;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              if (n0 + i < prm.N) *reinterpret_cast<float4*>(dst + i) = make_float4(y[i], y[i + 1], y[i + 2], y[i + 3]);
          } else {
            uint16_t* dst = reinterpret_cast<uint16_t*>(prm.out) + o;
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              if (n0 + i < prm.N) {
                uint32_t w[4];
#pragma unroll
                for (int k2 = 0; k2 < 4; ++k2)
                  w[k2] = float_to_bf16_bits(y[i + 2 * k2]) | (float_to_bf16_bits(y[i + 2 * k2 + 1]) << 16);
                *reinterpret_cast<uint4*>(dst + i) = make_uint4(w[0], w[1], w[2], w[3]);
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[L::kAccEmpty + buf]);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && tid == 0) atomicExch(prm.err, 1);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace sage
