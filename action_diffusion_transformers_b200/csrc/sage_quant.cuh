// sage_quant.cuh - bandwidth-bound kernels of sage_quant_qk / sage_quant_v.
//
//  colstats_partial  per 64-token block, per channel: FP64 sum in token order
//                    (and, for V, min / max) -> workspace partials.
//  k_mean_finalize   FP64 block partials -> K mean, BF16 (one rounding).
//  v_stats_finalize  FP64 block partials -> V mean, per-channel FP8 scales.
//  qk_block_quant    Q and K (centred, BF16-rounded) -> INT8 codes with one
//                    FP32 scale per 64-token block of one head.
//  v_quant_t         centred V -> E4M3 codes, transposed through shared memory
//                    to [B, H, D, Npad].
//
// All inputs are BF16 [B, N, H, D] with a token stride; every global access is
// a 16-byte vector for the inputs.  Reductions use a fixed order, so repeated
// calls give identical bytes.
#pragma once
#include <type_traits>
#include "sage_ptx.cuh"

namespace sage {

constexpr int kQKBlock = 64;     // tokens per INT8 scale block
constexpr int kSumBlock = 64;    // tokens per first-level FP64 partial
constexpr int kSumLanes = 32;    // interleaved second-level partials
constexpr int kTile = 128;       // padding granularity of the token axis

__device__ __forceinline__ uint4 ld_nc_16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void unpack8(const uint4& raw, float (&f)[8]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = bf16_bits_to_float(w[i] & 0xFFFFu);
    f[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
  }
}

// ----------------------------------------------------------------------------
// QK RMSNorm + RoPE in BF16 rounding, applied to a token row as it is loaded
// (sage_quant_qk_normrope).  The D channels of one (token, head) row are held
// by L = D/8 consecutive lanes, 8 channels each.
//   ss = sum of x^2: each lane adds its 8 squares in order from +0 (x^2 of a
//        BF16 value is exact, so fma(x, x, ss) is one rounding of ss + x^2),
//        then ss <- ss + ss[lane ^ o] for o = L/2 .. 1 (every lane ends equal);
//   r  = RN(1 / RN(sqrt(RN(RN(ss / D) + eps))))   (correctly rounded sqrt, div);
//   y  = RN_bf16(RN(x * r));  z = RN_bf16(y * w);
//   pair (z[2i], z[2i+1]) = (a, b) of table pair p = (d0 + 2i) / 2:
//   o0 = RN_bf16(RN(RN(c * a) - RN(s * b))), o1 = RN_bf16(RN(RN(s * a) + RN(c * b))).
// ----------------------------------------------------------------------------
struct NormRopeArgs {
  const uint16_t* q_w;    // BF16 [D] RMSNorm weight of Q
  const uint16_t* k_w;    // BF16 [D] RMSNorm weight of K
  const float* cos;       // [N, D/2] per token and channel pair
  const float* sin;       // [N, D/2]
  float eps;
};

__device__ __forceinline__ f32x2_t x2_of(float lo, float hi) {
  return x2_pack(__float_as_uint(lo), __float_as_uint(hi));
}

// Both halves RN_bf16, packed (low half = lo).
__device__ __forceinline__ uint32_t bf16x2_round(f32x2_t v) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(x2_hi(v)), "f"(x2_lo(v)));
  return d;
}

// RN_bf16(a * b) per half of two packed BF16 pairs (the product of two BF16
// values is exact, so this is the binary32 product rounded once to BF16).
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// kRows token rows of this lane (8 channels d0 .. d0+7 each), in place.  The
// kL = D/8 lanes of a row are consecutive lanes of the warp, and every lane of
// the warp executes this call.  Rows past the data hold zeros and stay zero.
// The root and reciprocal of row t are formed once, by lane t of the row's
// lanes, and shuffled out.  cs[t], sn[t]: cos / sin of row t's pairs
// d0/2 .. d0/2+3.  The rotation takes two neighbouring pairs p, p+1 at a time,
// so that each f32x2 product has as halves the same step of the two pairs:
// with a = (a_p, a_p+1), b = (b_p, b_p+1), c = (c_p, c_p+1), s = (s_p, s_p+1)
// (c and s are adjacent words of the tables' float4s) the products are c*a,
// s*b, s*a and c*b, each rounded, then a' = RN(RN(c*a) - RN(s*b)) and
// b' = RN(RN(s*a) + RN(c*b)) per pair.
template <int kRows, int kL>
__device__ __forceinline__ void norm_rope_rows(float (&x)[kRows][8], const float (&w)[8], float eps,
                                               const float4 (&cs)[kRows], const float4 (&sn)[kRows]) {
  static_assert(kRows <= kL, "one lane per row for the root");
  constexpr float kInvD = 1.f / static_cast<float>(8 * kL);
  float ss[kRows];
#pragma unroll
  for (int t = 0; t < kRows; ++t) {
    ss[t] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) ss[t] = __fmaf_rn(x[t][i], x[t][i], ss[t]);
  }
#pragma unroll
  for (int o = kL / 2; o >= 1; o >>= 1) {
#pragma unroll
    for (int t = 0; t < kRows; ++t) ss[t] = __fadd_rn(ss[t], __shfl_xor_sync(0xFFFFFFFFu, ss[t], o));
  }
  const int lane = threadIdx.x & 31;
  const int g = (lane % kL) % kRows;
  float mine = ss[0];
#pragma unroll
  for (int t = 1; t < kRows; ++t) mine = g == t ? ss[t] : mine;
  const float rl = __fdiv_rn(1.f, __fsqrt_rn(__fadd_rn(__fmul_rn(mine, kInvD), eps)));
  const int base = lane & ~(kL - 1);
  uint32_t w2[4];                         // the weight pairs as packed BF16 (exact: w is BF16)
#pragma unroll
  for (int p = 0; p < 4; ++p) w2[p] = bf16x2_round(x2_of(w[2 * p], w[2 * p + 1]));
#pragma unroll
  for (int t = 0; t < kRows; ++t) {
    const f32x2_t r2 = x2_splat(__shfl_sync(0xFFFFFFFFu, rl, base + t));
    uint32_t zb[4];                       // z of pair p as packed BF16 (low half = even channel)
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t y = bf16x2_round(x2_mul(x2_of(x[t][2 * p], x[t][2 * p + 1]), r2));
      zb[p] = bf16x2_mul(y, w2[p]);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t z0 = zb[2 * h], z1 = zb[2 * h + 1];
      const f32x2_t a = x2_pack(z0 << 16, z1 << 16);
      const f32x2_t b = x2_pack(z0 & 0xFFFF0000u, z1 & 0xFFFF0000u);
      const f32x2_t c = h == 0 ? x2_of(cs[t].x, cs[t].y) : x2_of(cs[t].z, cs[t].w);
      const f32x2_t s = h == 0 ? x2_of(sn[t].x, sn[t].y) : x2_of(sn[t].z, sn[t].w);
      const f32x2_t ca = x2_mul(c, a), sb = x2_mul(s, b), sa = x2_mul(s, a), cb = x2_mul(c, b);
      // Scalar adds: the compiler fuses an f32x2 multiply into a following
      // f32x2 add (one rounding fewer), but never a product into __fadd_rn.
      const uint32_t o0 = bf16x2_round(x2_of(__fsub_rn(x2_lo(ca), x2_lo(sb)), __fadd_rn(x2_lo(sa), x2_lo(cb))));
      const uint32_t o1 = bf16x2_round(x2_of(__fsub_rn(x2_hi(ca), x2_hi(sb)), __fadd_rn(x2_hi(sa), x2_hi(cb))));
      x[t][4 * h] = __uint_as_float(o0 << 16);
      x[t][4 * h + 1] = __uint_as_float(o0 & 0xFFFF0000u);
      x[t][4 * h + 2] = __uint_as_float(o1 << 16);
      x[t][4 * h + 3] = __uint_as_float(o1 & 0xFFFF0000u);
    }
  }
}

__device__ __forceinline__ float4 ld_nc_f4(const float* p) {
  const uint4 r = ld_nc_16(p);
  return make_float4(__uint_as_float(r.x), __uint_as_float(r.y), __uint_as_float(r.z), __uint_as_float(r.w));
}

// ----------------------------------------------------------------------------
// Per (b, 64-token block c, channel): s = ((0 + x_{64c}) + x_{64c+1}) + ... in
// token order, in FP64.  Grid (nsb, B, ceil(HD / (8*blockDim))).
// ----------------------------------------------------------------------------
// tx: the thread's index in its group of 128 (threadIdx.x for a 128-thread CTA).
template <bool kMinMax>
__device__ __forceinline__ void colstats_body(int bx, int by, int bz, const uint16_t* __restrict__ x, int N,
                                              int HD, int64_t tok_stride, int nsb, double* __restrict__ psum,
                                              float* __restrict__ pmin, float* __restrict__ pmax,
                                              int tx = static_cast<int>(threadIdx.x)) {
  const int c = bx;
  const int b = by;
  const int ch0 = (bz * 128 + tx) * 8;
  if (ch0 >= HD) return;
  const int n0 = c * kSumBlock;
  const int n1 = min(N, n0 + kSumBlock);
  const uint16_t* p = x + (static_cast<int64_t>(b) * N + n0) * tok_stride + ch0;
  double s[8];
  // min / max kept as packed BF16 pairs (exact: the inputs are BF16)
  __nv_bfloat162 mn[4], mx[4];
#pragma unroll
  for (int i = 0; i < 8; ++i) s[i] = 0.0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    mn[i] = __floats2bfloat162_rn(__int_as_float(0x7F800000), __int_as_float(0x7F800000));
    mx[i] = __floats2bfloat162_rn(-__int_as_float(0x7F800000), -__int_as_float(0x7F800000));
  }
  auto accumulate = [&](const uint4& raw) {
    float f[8];
    unpack8(raw, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i] = __dadd_rn(s[i], static_cast<double>(f[i]));
    if (kMinMax) {
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
        mn[i] = __hmin2(mn[i], v);
        mx[i] = __hmax2(mx[i], v);
      }
    }
  };
  int n = n0;
  for (; n + 16 <= n1; n += 16) {         // 16 loads in flight
    uint4 raw[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) raw[t] = ld_nc_16(p + static_cast<int64_t>(n - n0 + t) * tok_stride);
#pragma unroll
    for (int t = 0; t < 16; ++t) accumulate(raw[t]);
  }
  for (; n < n1; ++n) accumulate(ld_nc_16(p + static_cast<int64_t>(n - n0) * tok_stride));
  const int64_t o = (static_cast<int64_t>(b) * nsb + c) * HD + ch0;
  double2* ps = reinterpret_cast<double2*>(psum + o);
#pragma unroll
  for (int i = 0; i < 4; ++i) ps[i] = make_double2(s[2 * i], s[2 * i + 1]);
  if (kMinMax) {
    float4* pn = reinterpret_cast<float4*>(pmin + o);
    float4* px = reinterpret_cast<float4*>(pmax + o);
    pn[0] = make_float4(__low2float(mn[0]), __high2float(mn[0]), __low2float(mn[1]), __high2float(mn[1]));
    pn[1] = make_float4(__low2float(mn[2]), __high2float(mn[2]), __low2float(mn[3]), __high2float(mn[3]));
    px[0] = make_float4(__low2float(mx[0]), __high2float(mx[0]), __low2float(mx[1]), __high2float(mx[1]));
    px[1] = make_float4(__low2float(mx[2]), __high2float(mx[2]), __low2float(mx[3]), __high2float(mx[3]));
  }
}

template <bool kMinMax>
__global__ void __launch_bounds__(128) colstats_partial(const uint16_t* __restrict__ x, int N, int HD,
                                                        int64_t tok_stride, int nsb,
                                                        double* __restrict__ psum,
                                                        float* __restrict__ pmin, float* __restrict__ pmax) {
  pdl_enter();
  colstats_body<kMinMax>(blockIdx.x, blockIdx.y, blockIdx.z, x, N, HD, tok_stride, nsb, psum, pmin, pmax);
}

// K column sums (as colstats_partial<false>: same grid, order and output) of
// the rows after QK RMSNorm + RoPE, for the K mean of sage_quant_qk_normrope.
// Lanes past H*D run the loop on zeros (their whole head is past it) so that
// every lane takes part in the row shuffles.
template <int D>
__global__ void __launch_bounds__(128) colstats_normrope(const uint16_t* __restrict__ x, int N, int HD,
                                                         int64_t tok_stride, int nsb, double* __restrict__ psum,
                                                         const NormRopeArgs nr) {
  pdl_enter();
  const int c = blockIdx.x;
  const int b = blockIdx.y;
  const int ch0 = (blockIdx.z * blockDim.x + threadIdx.x) * 8;
  const bool active = ch0 < HD;
  const int d0 = ch0 % D;
  float w[8];
  unpack8(active ? ld_nc_16(nr.k_w + d0) : make_uint4(0u, 0u, 0u, 0u), w);
  const int n0 = c * kSumBlock;
  const int n1 = min(N, n0 + kSumBlock);
  const uint16_t* p = x + (static_cast<int64_t>(b) * N + n0) * tok_stride + (active ? ch0 : 0);
  double s[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) s[i] = 0.0;
  constexpr int kRows = 4;                 // rows (and their table entries) in flight
  // A full 64-row block of an active lane loads without guards and zero fills.
  const bool full = active && n1 - n0 == kSumBlock;
  for (int n = n0; n < n1; n += kRows) {
    uint4 raw[kRows];
    float4 cs[kRows], sn[kRows];
    auto load_rows = [&](auto guarded) {
#pragma unroll
      for (int t = 0; t < kRows; ++t) {
        const bool ok = !decltype(guarded)::value || (active && n + t < n1);
        const int64_t tab = static_cast<int64_t>(n + t) * (D / 2) + d0 / 2;
        raw[t] = ok ? ld_nc_16(p + static_cast<int64_t>(n + t - n0) * tok_stride) : make_uint4(0u, 0u, 0u, 0u);
        cs[t] = ok ? ld_nc_f4(nr.cos + tab) : make_float4(0.f, 0.f, 0.f, 0.f);
        sn[t] = ok ? ld_nc_f4(nr.sin + tab) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    };
    if (full)
      load_rows(std::false_type{});
    else
      load_rows(std::true_type{});
    float f[kRows][8];
#pragma unroll
    for (int t = 0; t < kRows; ++t) unpack8(raw[t], f[t]);
    norm_rope_rows<kRows, D / 8>(f, w, nr.eps, cs, sn);
#pragma unroll
    for (int t = 0; t < kRows; ++t) {
      if (n + t < n1) {
#pragma unroll
        for (int i = 0; i < 8; ++i) s[i] = __dadd_rn(s[i], static_cast<double>(f[t][i]));
      }
    }
  }
  if (!active) return;
  const int64_t o = (static_cast<int64_t>(b) * nsb + c) * HD + ch0;
  double2* ps = reinterpret_cast<double2*>(psum + o);
#pragma unroll
  for (int i = 0; i < 4; ++i) ps[i] = make_double2(s[2 * i], s[2 * i + 1]);
}

// Second level of the fixed summation order for one channel: lane g sums
// blocks g, g+32, g+64, ... in increasing order from +0; then the butterfly
// u_g <- u_g + u_{g^o} for o = 16, 8, 4, 2, 1; the result is lane 0's value.
// Block of 1024 threads = 32 lanes (warps) x 32 channels (lanes of a warp, so
// every load is one coalesced 256-byte row of partials); one transpose through
// shared memory then gives warp g channel g's 32 partials, and the butterfly
// runs on shuffles.  The channel index runs over B*HD.  For V the same pass
// also reduces min / max (order-free).
template <bool kMinMax>
__device__ __forceinline__ void finalize_channel(const double* __restrict__ psum,
                                                 const float* __restrict__ pmin,
                                                 const float* __restrict__ pmax, int nsb, int HD, int b,
                                                 int ch, bool valid, double (*sh)[33], float (*shn)[33],
                                                 float (*shx)[33], double& sum, float& vmin, float& vmax) {
  const int g = threadIdx.x >> 5;
  const int cl = threadIdx.x & 31;
  double u = 0.0;
  float mn = __int_as_float(0x7F800000), mx = -__int_as_float(0x7F800000);
  if (valid) {
    const int64_t base = static_cast<int64_t>(b) * nsb * HD + ch;
#pragma unroll 4
    for (int c = g; c < nsb; c += kSumLanes) {
      u = __dadd_rn(u, psum[base + static_cast<int64_t>(c) * HD]);
      if (kMinMax) {
        mn = fminf(mn, pmin[base + static_cast<int64_t>(c) * HD]);
        mx = fmaxf(mx, pmax[base + static_cast<int64_t>(c) * HD]);
      }
    }
  }
  sh[g][cl] = u;
  if (kMinMax) {
    shn[g][cl] = mn;
    shx[g][cl] = mx;
  }
  __syncthreads();
  // Transposed: warp g now holds channel g's 32 lane partials (lane j: lane
  // j's partial), and the butterfly runs on shuffles; each lane adds its own
  // value and its partner's in that order, the pairing of the fixed order.
  double v = sh[cl][g];
  float vn = 0.f, vx = 0.f;
  if (kMinMax) {
    vn = shn[cl][g];
    vx = shx[cl][g];
  }
#pragma unroll
  for (int o = kSumLanes / 2; o >= 1; o >>= 1) {
    v = __dadd_rn(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    if (kMinMax) {
      vn = fminf(vn, __shfl_xor_sync(0xFFFFFFFFu, vn, o));
      vx = fmaxf(vx, __shfl_xor_sync(0xFFFFFFFFu, vx, o));
    }
  }
  sum = v;                 // the result for channel g of the block (every lane of warp g)
  if (kMinMax) {
    vmin = vn;
    vmax = vx;
  }
}

__device__ __forceinline__ void k_mean_body(int bx, const double* __restrict__ psum, int B, int N, int HD, int nsb,
                                            uint16_t* __restrict__ mean_ws, uint16_t* __restrict__ mean_out,
                                            double (&sh)[kSumLanes][33]) {
  const int gch = bx * 32 + (threadIdx.x & 31);
  const bool valid = gch < B * HD;
  const int b = valid ? gch / HD : 0;
  const int ch = valid ? gch % HD : 0;
  double s = 0.0;
  float dummy0, dummy1;
  finalize_channel<false>(psum, nullptr, nullptr, nsb, HD, b, ch, valid, sh, nullptr, nullptr, s, dummy0,
                          dummy1);
  const int och = bx * 32 + (threadIdx.x >> 5);   // warp g finished channel g of the block
  if (och < B * HD && (threadIdx.x & 31) == 0) {
    const uint16_t m = static_cast<uint16_t>(double_to_bf16_bits(__ddiv_rn(s, static_cast<double>(N))));
    mean_ws[och] = m;
    if (mean_out) mean_out[och] = m;
  }
}

__global__ void __launch_bounds__(1024) k_mean_finalize(const double* __restrict__ psum, int B, int N, int HD,
                                                        int nsb, uint16_t* __restrict__ mean_ws,
                                                        uint16_t* __restrict__ mean_out) {
  pdl_enter();
  __shared__ double sh[kSumLanes][33];
  k_mean_body(blockIdx.x, psum, B, N, HD, nsb, mean_ws, mean_out, sh);
}

// V: mean = RN_f32(sum / N); amax = max(RN(vmax - mean), RN(mean - vmin));
// scale = RN(amax / 448), inv = RN(448 / amax) (0, 0 for amax == 0).
__device__ __forceinline__ void v_stats_body(int bx, const double* __restrict__ psum, const float* __restrict__ pmin,
                                             const float* __restrict__ pmax, int B, int N, int HD, int nsb,
                                             float* __restrict__ v_mean, float* __restrict__ v_scale,
                                             float* __restrict__ v_inv, double (&sh)[kSumLanes][33],
                                             float (&shn)[kSumLanes][33], float (&shx)[kSumLanes][33]) {
  const int gch = bx * 32 + (threadIdx.x & 31);
  const bool valid = gch < B * HD;
  const int b = valid ? gch / HD : 0;
  const int ch = valid ? gch % HD : 0;
  double s = 0.0;
  float vmin = 0.f, vmax = 0.f;
  finalize_channel<true>(psum, pmin, pmax, nsb, HD, b, ch, valid, sh, shn, shx, s, vmin, vmax);
  const int och = bx * 32 + (threadIdx.x >> 5);   // warp g finished channel g of the block
  if (och < B * HD && (threadIdx.x & 31) == 0) {
    const float mean = __double2float_rn(__ddiv_rn(s, static_cast<double>(N)));
    const float amax = fmaxf(__fsub_rn(vmax, mean), __fsub_rn(mean, vmin));
    float scale = 0.f, inv = 0.f;
    if (amax > 0.f) {
      scale = __fdiv_rn(amax, 448.f);
      inv = __fdiv_rn(448.f, amax);
    }
    v_mean[och] = mean;
    v_scale[och] = scale;
    v_inv[och] = inv;
  }
}

__global__ void __launch_bounds__(1024) v_stats_finalize(const double* __restrict__ psum,
                                                         const float* __restrict__ pmin,
                                                         const float* __restrict__ pmax, int B, int N, int HD,
                                                         int nsb, float* __restrict__ v_mean,
                                                         float* __restrict__ v_scale, float* __restrict__ v_inv) {
  pdl_enter();
  __shared__ double sh[kSumLanes][33];
  __shared__ float shn[kSumLanes][33];
  __shared__ float shx[kSumLanes][33];
  v_stats_body(blockIdx.x, psum, pmin, pmax, B, N, HD, nsb, v_mean, v_scale, v_inv, sh, shn, shx);
}

// ----------------------------------------------------------------------------
// INT8 block quantization.  CTA = one (b, h, 128-token tile = two 64-token
// scale blocks) of K (z < B: centred by mean_k and rounded to BF16 first) or Q
// (z >= B).  K runs first so that its second read follows the column-sum pass
// while K is still in L2.  256 threads: D/8 threads cover one token row (8
// channels each); each thread holds 128 / (256 / (D/8)) tokens, so 8 16-byte
// loads are in flight per thread at D = 128.  Grid (Npad/128, H, 2*B).
// Rounding: RNE(RN(x * inv)) is formed by adding 1.5 * 2^23 (exact here:
// |x * inv| <= 127 * (1 + 2^-23)), which keeps the conversion on the FMA pipe.
// ----------------------------------------------------------------------------
__device__ __forceinline__ int rne_small(float y) {
  return __float_as_int(__fadd_rn(y, 12582912.0f)) - 0x4B400000;
}

// kNR: Q and K rows first go through QK RMSNorm + RoPE (norm_rope_rows); that
// variant takes one 64-token block per CTA (4 rows per thread), so that
// several CTAs share an SM and one's loads overlap the others' reductions and
// stores.  Both variants run three CTAs per SM (80 registers; the kNR one
// spills a few bytes there and was measured faster than two CTAs at 99).
template <int D, bool kNR>
__device__ __forceinline__ void qk_block_body(int bx, int by, int bz, const uint16_t* __restrict__ q,
                                              const uint16_t* __restrict__ k, int N, int B, int H, int Npad,
                                              int64_t tok_stride, const uint16_t* __restrict__ k_mean,
                                              int8_t* __restrict__ q_codes, float* __restrict__ q_scale,
                                              int8_t* __restrict__ k_codes, float* __restrict__ k_scale,
                                              const NormRopeArgs& nr) {
  constexpr int kWarps = 256 / 32;
  constexpr int kSlots = kNR ? 1 : 2;     // 64-token blocks per CTA
  constexpr int kTokens = kSlots * kQKBlock;
  constexpr int kLPR = D / 8;             // threads per token row
  constexpr int kRPP = 256 / kLPR;        // token rows per pass
  constexpr int kTPT = kTokens / kRPP;    // tokens per thread (kHalf in each block)
  constexpr int kHalf = kTPT / kSlots;
  __shared__ float red[kWarps][2];
  const int tile = bx;
  const bool is_k = static_cast<int>(bz) < B;
  // K heads are visited last-to-first: the column-sum pass just streamed K in
  // head order, so the most recently read heads (still in L2) come first.
  const int h = is_k ? H - 1 - static_cast<int>(by) : static_cast<int>(by);
  const int b = is_k ? bz : bz - B;
  const uint16_t* src = is_k ? k : q;
  const int cg = threadIdx.x % kLPR;
  const int r0 = threadIdx.x / kLPR;
  const int d0 = cg * 8;

  float mean[8];
  if (is_k) {
    const uint4 mraw = *reinterpret_cast<const uint4*>(k_mean + (static_cast<int64_t>(b) * H + h) * D + d0);
    unpack8(mraw, mean);
  }
  uint4 raw[kTPT];
  float4 cs[kNR ? kTPT : 1], sn[kNR ? kTPT : 1];
  // Rows past N read as zeros; a CTA whose rows are all below N (every one but
  // a ragged last tile) loads without the guards and their zero fills.
  auto load_rows = [&](auto guarded) {
#pragma unroll
    for (int t = 0; t < kTPT; ++t) {
      const int n = tile * kTokens + r0 + t * kRPP;
      const bool ok = !decltype(guarded)::value || n < N;
      raw[t] = ok ? ld_nc_16(src + (static_cast<int64_t>(b) * N + n) * tok_stride + h * D + d0)
                  : make_uint4(0u, 0u, 0u, 0u);
      if constexpr (kNR) {
        const int64_t tab = static_cast<int64_t>(n) * (D / 2) + d0 / 2;
        cs[t] = ok ? ld_nc_f4(nr.cos + tab) : make_float4(0.f, 0.f, 0.f, 0.f);
        sn[t] = ok ? ld_nc_f4(nr.sin + tab) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  };
  if ((tile + 1) * kTokens <= N)
    load_rows(std::false_type{});
  else
    load_rows(std::true_type{});
  float x[kTPT][8];
  float amax[2] = {0.f, 0.f};
#pragma unroll
  for (int t = 0; t < kTPT; ++t) unpack8(raw[t], x[t]);
  if constexpr (kNR) {
    float nw[8];
    unpack8(ld_nc_16((is_k ? nr.k_w : nr.q_w) + d0), nw);
    norm_rope_rows<kTPT, kLPR>(x, nw, nr.eps, cs, sn);   // rows past N stay zero
  }
#pragma unroll
  for (int t = 0; t < kTPT; ++t) {
    const int n = tile * kTokens + r0 + t * kRPP;
    if (is_k) {
      if (n < N) {
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          const f32x2_t dv = x2_sub(x2_pack(__float_as_uint(x[t][i]), __float_as_uint(x[t][i + 1])),
                                    x2_pack(__float_as_uint(mean[i]), __float_as_uint(mean[i + 1])));
          const __nv_bfloat162 c2 = __floats2bfloat162_rn(x2_lo(dv), x2_hi(dv));
          const uint32_t cb = *reinterpret_cast<const uint32_t*>(&c2);
          x[t][i] = __uint_as_float(cb << 16);
          x[t][i + 1] = __uint_as_float(cb & 0xFFFF0000u);
        }
      }  // padded rows stay 0
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) amax[t / kHalf] = fmaxf(amax[t / kHalf], fabsf(x[t][i]));
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    amax[0] = fmaxf(amax[0], __shfl_xor_sync(0xFFFFFFFFu, amax[0], o));
    amax[1] = fmaxf(amax[1], __shfl_xor_sync(0xFFFFFFFFu, amax[1], o));
  }
  if ((threadIdx.x & 31) == 0) {
    red[threadIdx.x >> 5][0] = amax[0];
    red[threadIdx.x >> 5][1] = amax[1];
  }
  __syncthreads();
  float scale[2], inv[2];
#pragma unroll
  for (int blk = 0; blk < 2; ++blk) {
    float a = red[0][blk];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) a = fmaxf(a, red[w][blk]);
    scale[blk] = 0.f;
    inv[blk] = 0.f;
    if (a > 0.f) {
      scale[blk] = __fdiv_rn(a, 127.f);
      inv[blk] = __fdiv_rn(127.f, a);
    }
  }
  const int64_t bh = static_cast<int64_t>(b) * H + h;
  int8_t* dst = is_k ? k_codes : q_codes;
  // code = RNE(RN(x * inv)) in [-127, 127] without a clamp: |x| <= amax gives
  // |x * inv| <= 127 * (1 + 2^-24), which rounds to at most 127.  After the
  // 1.5 * 2^23 addition the integer sits in the low bits of the float, so the
  // low byte of each word is the code's two's-complement byte; three byte
  // permutes gather four of them.  The product and the addition are the
  // scalar rounding intrinsics, which the compiler never fuses into one FMA
  // (a fused RN(x * inv + 1.5 * 2^23) would skip the rounding of the product).
#pragma unroll
  for (int t = 0; t < kTPT; ++t) {
    const int n = tile * kTokens + r0 + t * kRPP;
    const float iv = inv[t / kHalf];
    uint32_t cw[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) cw[i] = __float_as_uint(__fadd_rn(__fmul_rn(x[t][i], iv), 12582912.0f));
    const uint32_t w0 = __byte_perm(__byte_perm(cw[0], cw[1], 0x0040), __byte_perm(cw[2], cw[3], 0x0040), 0x5410);
    const uint32_t w1 = __byte_perm(__byte_perm(cw[4], cw[5], 0x0040), __byte_perm(cw[6], cw[7], 0x0040), 0x5410);
    *reinterpret_cast<uint2*>(dst + (bh * Npad + n) * D + d0) = make_uint2(w0, w1);
  }
  if (threadIdx.x < kSlots)
    (is_k ? k_scale : q_scale)[bh * (Npad / kQKBlock) + tile * kSlots + threadIdx.x] = threadIdx.x == 0 ? scale[0] : scale[1];
}

template <int D, bool kNR = false>
__global__ void __launch_bounds__(256, 3) qk_block_quant(const uint16_t* __restrict__ q,
                                                      const uint16_t* __restrict__ k, int N, int B, int H,
                                                      int Npad, int64_t tok_stride,
                                                      const uint16_t* __restrict__ k_mean,
                                                      int8_t* __restrict__ q_codes, float* __restrict__ q_scale,
                                                      int8_t* __restrict__ k_codes,
                                                      float* __restrict__ k_scale, const NormRopeArgs nr = {}) {
  pdl_enter();
  qk_block_body<D, kNR>(blockIdx.x, blockIdx.y, blockIdx.z, q, k, N, B, H, Npad, tok_stride, k_mean, q_codes,
                        q_scale, k_codes, k_scale, nr);
}

// ----------------------------------------------------------------------------
// Q / K quantization at any scale granularity (64-token blocks, one scale per
// token, 64-token blocks restarting at every segment start).  A CTA holds two
// "slots" of up to 64 consecutive tokens of one (b, h): the two halves of a
// 128-token tile for the block and token granularities, or two consecutive
// segment-local blocks.  Thread mapping as in qk_block_quant.  The absmax is
// reduced over the kLPR lanes of a token row (per token) or over the whole slot
// (per block).  Block scales go to [B*H, Npad/64]; per-token and segment-local
// scales to [B*H, Npad], every token holding its group's scale.
// ----------------------------------------------------------------------------
constexpr int kGranBlock64 = 0;
constexpr int kGranToken = 1;
constexpr int kGranSegment64 = 2;
constexpr int kMaxSegments = 256;

// The segments of a packed sequence, then the padding [N, Npad) as one more
// segment; gbase[s] = number of 64-token blocks before segment s.  Passed by
// value as a kernel parameter (2 KB).
struct SegTable {
  int n;                              // segments, the padding included
  int start[kMaxSegments + 2];        // segment s is [start[s], start[s + 1])
  int gbase[kMaxSegments + 2];        // gbase[n] = all blocks
};

// First token and length of segment-local block g (g < seg.gbase[seg.n]).
__device__ __forceinline__ void seg_block(const SegTable& seg, int g, int& start, int& len) {
  int lo = 0, hi = seg.n;               // largest s with gbase[s] <= g (empty segments skipped)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (seg.gbase[mid] <= g) lo = mid; else hi = mid;
  }
  start = seg.start[lo] + kQKBlock * (g - seg.gbase[lo]);
  len = min(kQKBlock, seg.start[lo + 1] - start);
}

// One CTA of qk_group_quant: tensor K (is_k) or Q at granularity kGran.
template <int D, int kGran, bool kNR>
__device__ __forceinline__ void group_quant_cta(bool is_k, const uint16_t* __restrict__ q,
                                                const uint16_t* __restrict__ k, int N, int B, int H, int Npad,
                                                int64_t tok_stride, const uint16_t* __restrict__ k_mean,
                                                int8_t* __restrict__ q_codes, float* __restrict__ q_scale,
                                                int8_t* __restrict__ k_codes, float* __restrict__ k_scale,
                                                const SegTable& seg, const NormRopeArgs& nr) {
  constexpr int gran = kGran;
  constexpr int kLPR = D / 8;             // threads per token row
  constexpr int kRPP = 256 / kLPR;        // token rows per pass
  constexpr int kTPT = kTile / kRPP;      // token rows per thread (half in each slot)
  constexpr int kHalf = kTPT / 2;
  __shared__ float red[8][2];
  const int h = is_k ? H - 1 - static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.y);
  const int b = static_cast<int>(blockIdx.z) % B;
  const uint16_t* src = is_k ? k : q;
  const int cg = threadIdx.x % kLPR;
  const int r0 = threadIdx.x / kLPR;
  const int d0 = cg * 8;

  int gstart[2], glen[2];
  if constexpr (gran == kGranSegment64) {
    const int G = seg.gbase[seg.n];
    if (2 * static_cast<int>(blockIdx.x) >= G) return;   // the whole CTA leaves
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int g = 2 * blockIdx.x + s;
      gstart[s] = 0;
      glen[s] = 0;
      if (g < G) seg_block(seg, g, gstart[s], glen[s]);
    }
  } else {
    if (static_cast<int>(blockIdx.x) >= Npad / kTile) return;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      gstart[s] = blockIdx.x * kTile + s * kQKBlock;
      glen[s] = kQKBlock;
    }
  }

  float mean[8];
  if (is_k) {
    const uint4 mraw = *reinterpret_cast<const uint4*>(k_mean + (static_cast<int64_t>(b) * H + h) * D + d0);
    unpack8(mraw, mean);
  }
  uint4 raw[kTPT];
  float4 cs[kNR ? kTPT : 1], sn[kNR ? kTPT : 1];
#pragma unroll
  for (int t = 0; t < kTPT; ++t) {
    const int o = r0 + (t % kHalf) * kRPP;
    const int n = gstart[t / kHalf] + o;
    const bool ok = o < glen[t / kHalf] && n < N;
    raw[t] = ok ? ld_nc_16(src + (static_cast<int64_t>(b) * N + n) * tok_stride + h * D + d0)
                : make_uint4(0u, 0u, 0u, 0u);
    if constexpr (kNR) {
      const int64_t tab = static_cast<int64_t>(n) * (D / 2) + d0 / 2;
      cs[t] = ok ? ld_nc_f4(nr.cos + tab) : make_float4(0.f, 0.f, 0.f, 0.f);
      sn[t] = ok ? ld_nc_f4(nr.sin + tab) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  float x[kTPT][8];
  float rmax[kTPT];
#pragma unroll
  for (int t = 0; t < kTPT; ++t) unpack8(raw[t], x[t]);
  if constexpr (kNR) {
    float nw[8];
    unpack8(ld_nc_16((is_k ? nr.k_w : nr.q_w) + d0), nw);
    norm_rope_rows<kTPT, kLPR>(x, nw, nr.eps, cs, sn);   // rows not loaded stay zero
  }
#pragma unroll
  for (int t = 0; t < kTPT; ++t) {
    const int o = r0 + (t % kHalf) * kRPP;
    const int n = gstart[t / kHalf] + o;
    if (is_k && o < glen[t / kHalf] && n < N) {
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const __nv_bfloat162 c2 =
            __floats2bfloat162_rn(__fsub_rn(x[t][i], mean[i]), __fsub_rn(x[t][i + 1], mean[i + 1]));
        x[t][i] = __low2float(c2);
        x[t][i + 1] = __high2float(c2);
      }
    }
    rmax[t] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) rmax[t] = fmaxf(rmax[t], fabsf(x[t][i]));
  }
  const int64_t bh = static_cast<int64_t>(b) * H + h;
  int8_t* dst = is_k ? k_codes : q_codes;
  float* sdst = is_k ? k_scale : q_scale;
  float inv[kTPT];
  if constexpr (gran == kGranToken) {
    // The kLPR lanes of one token row are consecutive lanes of one warp; after
    // the butterfly every one of them holds the absmax of all kTPT rows.  Lane
    // cg < kTPT then forms the scale of row cg (and stores it), lane kTPT + t
    // the inverse of row t: one division per lane, the inverses shuffled out.
    static_assert(2 * kTPT == kLPR, "one division per lane");
#pragma unroll
    for (int t = 0; t < kTPT; ++t) {
#pragma unroll
      for (int o = kLPR / 2; o >= 1; o >>= 1) rmax[t] = fmaxf(rmax[t], __shfl_xor_sync(0xFFFFFFFFu, rmax[t], o));
    }
    const int mine = cg % kTPT;
    float a = rmax[0];
#pragma unroll
    for (int t = 1; t < kTPT; ++t) a = mine == t ? rmax[t] : a;
    const bool is_scale = cg < kTPT;
    const float val = a > 0.f ? __fdiv_rn(is_scale ? a : 127.f, is_scale ? 127.f : a) : 0.f;
    const int base = (threadIdx.x & 31) & ~(kLPR - 1);
#pragma unroll
    for (int t = 0; t < kTPT; ++t) inv[t] = __shfl_sync(0xFFFFFFFFu, val, base + kTPT + t);
    if (is_scale) {
      const int o = r0 + (mine % kHalf) * kRPP;
      const int s = mine / kHalf;
      const int gs = s == 0 ? gstart[0] : gstart[1];
      const int gl = s == 0 ? glen[0] : glen[1];
      if (o < gl) sdst[bh * Npad + gs + o] = val;
    }
  } else {
    float amax[2] = {0.f, 0.f};
#pragma unroll
    for (int t = 0; t < kTPT; ++t) amax[t / kHalf] = fmaxf(amax[t / kHalf], rmax[t]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      amax[0] = fmaxf(amax[0], __shfl_xor_sync(0xFFFFFFFFu, amax[0], o));
      amax[1] = fmaxf(amax[1], __shfl_xor_sync(0xFFFFFFFFu, amax[1], o));
    }
    if ((threadIdx.x & 31) == 0) {
      red[threadIdx.x >> 5][0] = amax[0];
      red[threadIdx.x >> 5][1] = amax[1];
    }
    __syncthreads();
    float scale[2], sinv[2];
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      float a = red[0][s];
#pragma unroll
      for (int w = 1; w < 8; ++w) a = fmaxf(a, red[w][s]);
      scale[s] = 0.f;
      sinv[s] = 0.f;
      if (a > 0.f) {
        scale[s] = __fdiv_rn(a, 127.f);
        sinv[s] = __fdiv_rn(127.f, a);
      }
    }
#pragma unroll
    for (int t = 0; t < kTPT; ++t) inv[t] = sinv[t / kHalf];
    if constexpr (gran == kGranBlock64) {
      if (threadIdx.x < 2)
        sdst[bh * (Npad / kQKBlock) + blockIdx.x * 2 + threadIdx.x] = threadIdx.x == 0 ? scale[0] : scale[1];
    } else if (cg == 0) {
#pragma unroll
      for (int t = 0; t < kTPT; ++t) {
        const int o = r0 + (t % kHalf) * kRPP;
        if (o < glen[t / kHalf]) sdst[bh * Npad + gstart[t / kHalf] + o] = scale[t / kHalf];
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kTPT; ++t) {
    const int o = r0 + (t % kHalf) * kRPP;
    if (o >= glen[t / kHalf]) continue;
    const int n = gstart[t / kHalf] + o;
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int c = rne_small(__fmul_rn(x[t][i], inv[t]));
      c = max(-127, min(127, c));
      w[i >> 2] |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * (i & 3));
    }
    *reinterpret_cast<uint2*>(dst + (bh * Npad + n) * D + d0) = make_uint2(w[0], w[1]);
  }
}

// Grid (max CTAs of the two tensors, H, 2B): z < B quantizes K at kGranK, the
// rest Q at kGranQ.  A CTA past its tensor's tiles or blocks leaves at once.
template <int D, int kGranQ, int kGranK, bool kNR = false>
__global__ void __launch_bounds__(256, kNR ? 1 : ((kGranQ == kGranSegment64 || kGranK == kGranSegment64) ? 2 : 3))
    qk_group_quant(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, int N, int B, int H, int Npad,
                   int64_t tok_stride, const uint16_t* __restrict__ k_mean, int8_t* __restrict__ q_codes,
                   float* __restrict__ q_scale, int8_t* __restrict__ k_codes, float* __restrict__ k_scale,
                   const __grid_constant__ SegTable seg, const NormRopeArgs nr = {}) {
  pdl_enter();
  if (static_cast<int>(blockIdx.z) < B)
    group_quant_cta<D, kGranK, kNR>(true, q, k, N, B, H, Npad, tok_stride, k_mean, q_codes, q_scale, k_codes,
                                    k_scale, seg, nr);
  else
    group_quant_cta<D, kGranQ, kNR>(false, q, k, N, B, H, Npad, tok_stride, k_mean, q_codes, q_scale, k_codes,
                                    k_scale, seg, nr);
}

// ----------------------------------------------------------------------------
// V centre + E4M3 quantization + transpose.  CTA = one (b, h, 128-token tile).
// Phase 1: threads read 16-byte pieces of token rows, quantize 8 channels and
// store the 8 code bytes into a [128][D] shared tile.  Phase 2: each thread
// gathers 16 consecutive tokens of one channel and writes them as one 16-byte
// piece of the transposed output row.  Grid (Npad/128, H, B).
// ----------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void v_quant_body(int bx, int by, int bz, const uint16_t* __restrict__ v, int N, int H,
                                             int Npad, int64_t tok_stride, const float* __restrict__ v_mean,
                                             const float* __restrict__ v_inv, uint8_t* __restrict__ out) {
  constexpr int kLPR = D / 8;
  constexpr int kRPP = 256 / kLPR;
  constexpr int kTPT = kTile / kRPP;
  constexpr int kPitch = D + 16;          // bytes per token row of the shared tile
  __shared__ __align__(16) uint8_t tile[kTile * kPitch];
  const int n0 = bx * kTile;
  // Heads last-to-first: the statistics pass just streamed V in head order.
  const int h = H - 1 - static_cast<int>(by);
  const int b = bz;
  const int cg = threadIdx.x % kLPR;
  const int r0 = threadIdx.x / kLPR;
  const int d0 = cg * 8;
  const int64_t bhd = (static_cast<int64_t>(b) * H + h) * D;
  float mean[8], inv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    mean[i] = v_mean[bhd + d0 + i];
    inv[i] = v_inv[bhd + d0 + i];
  }
  uint4 raw[kTPT];                        // every row's load in flight before any is used
#pragma unroll
  for (int t = 0; t < kTPT; ++t) {
    const int n = n0 + r0 + t * kRPP;
    raw[t] = n < N ? ld_nc_16(v + (static_cast<int64_t>(b) * N + n) * tok_stride + h * D + d0)
                   : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int t = 0; t < kTPT; ++t) {
    const int nl = r0 + t * kRPP;
    const int n = n0 + nl;
    uint32_t w0 = 0u, w1 = 0u;
    if (n < N) {
      float f[8];
      unpack8(raw[t], f);
      float y[8];
#pragma unroll
      for (int i = 0; i < 8; i += 2) {     // RN(RN(v - mean) * inv) on pairs
        const f32x2_t c = x2_mul(x2_sub(x2_of(f[i], f[i + 1]), x2_of(mean[i], mean[i + 1])), x2_of(inv[i], inv[i + 1]));
        y[i] = x2_lo(c);
        y[i + 1] = x2_hi(c);
      }
      w0 = cvt_e4m3x2(y[0], y[1]) | (cvt_e4m3x2(y[2], y[3]) << 16);
      w1 = cvt_e4m3x2(y[4], y[5]) | (cvt_e4m3x2(y[6], y[7]) << 16);
    }
    *reinterpret_cast<uint2*>(tile + nl * kPitch + d0) = make_uint2(w0, w1);
  }
  __syncthreads();
  // Phase 2: a thread owns 4 channels x 16 tokens.  It reads 16 words (4
  // channels of one token each), transposes each 4x4 byte block with prmt, and
  // writes 4 transposed 16-byte pieces (16 tokens of one channel each).
  constexpr int kUnits = (D / 4) * (kTile / 16);
  for (int u = threadIdx.x; u < kUnits; u += 256) {
    const int d4 = u % (D / 4);
    const int qc = u / (D / 4);
    uint32_t col[4][4];  // col[c][j]: channel 4*d4+c, tokens qc*16 + 4j .. +3
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        r[i] = *reinterpret_cast<const uint32_t*>(tile + (qc * 16 + 4 * j + i) * kPitch + 4 * d4);
      // r[i] holds channels 0..3 of token i; gather byte c of every token.
      const uint32_t lo01 = __byte_perm(r[0], r[1], 0x5140);   // t0c0 t1c0 t0c1 t1c1
      const uint32_t lo23 = __byte_perm(r[2], r[3], 0x5140);   // t2c0 t3c0 t2c1 t3c1
      const uint32_t hi01 = __byte_perm(r[0], r[1], 0x7362);   // t0c2 t1c2 t0c3 t1c3
      const uint32_t hi23 = __byte_perm(r[2], r[3], 0x7362);   // t2c2 t3c2 t2c3 t3c3
      col[0][j] = __byte_perm(lo01, lo23, 0x5410);
      col[1][j] = __byte_perm(lo01, lo23, 0x7632);
      col[2][j] = __byte_perm(hi01, hi23, 0x5410);
      col[3][j] = __byte_perm(hi01, hi23, 0x7632);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
      *reinterpret_cast<uint4*>(out + (bhd + 4 * d4 + c) * Npad + n0 + qc * 16) =
          make_uint4(col[c][0], col[c][1], col[c][2], col[c][3]);
  }
}

template <int D>
__global__ void __launch_bounds__(256) v_quant_t(const uint16_t* __restrict__ v, int N, int H, int Npad,
                                                 int64_t tok_stride, const float* __restrict__ v_mean,
                                                 const float* __restrict__ v_inv, uint8_t* __restrict__ out) {
  pdl_enter();
  v_quant_body<D>(blockIdx.x, blockIdx.y, blockIdx.z, v, N, H, Npad, tok_stride, v_mean, v_inv, out);
}

// ----------------------------------------------------------------------------
// Persistent V code pass with TMA staging: the same arithmetic and bytes as
// v_quant_t, but one producer thread copies each 128-token tile (a 2-D TMA box
// of 128 token rows x D channels of V seen as [B*N, tok_stride], completion
// counted on an mbarrier) into a 2-stage ring while 8 consumer warps quantize
// the other stage and write it transposed.  Work items (b, h, 128-token tile)
// go round robin over the grid (two CTAs per SM).  Every wait is bounded; a
// timeout raises the error word.
// ----------------------------------------------------------------------------
constexpr int kVbStages = 2;
constexpr int kVbConsumers = 256;
constexpr int kVbThreads = kVbConsumers + 32;

__device__ __forceinline__ void consumer_bar_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kVbConsumers) : "memory");
}

template <int D>
struct VbSmem {
  static constexpr int kRowBytes = 2 * D;
  static constexpr int kStageBytes = kTile * kRowBytes;
  static constexpr int kPitch = D + 16;
  static constexpr int kTileT = kVbStages * kStageBytes;       // transposed code tile
  static constexpr int kBar = kTileT + kTile * kPitch;          // full[S], empty[S]
  static constexpr int kMisc = kBar + 2 * kVbStages * 8;        // abort flag
  static constexpr int kTotal = kMisc + 16;
  static constexpr int kAlloc = kTotal + 128;                   // slack for 128-byte alignment
};

template <int D>
__global__ void __launch_bounds__(kVbThreads, 2)
    v_codes_tma(const __grid_constant__ CUtensorMap tm_v, const uint16_t* __restrict__ v, int N, int H, int B,
                 int Npad, int64_t tok_stride, const float* __restrict__ v_mean, const float* __restrict__ v_inv,
                 uint8_t* __restrict__ out, int* err, int64_t timeout_ns) {
  pdl_enter();
  using L = VbSmem<D>;
  constexpr int kLPR = D / 8;
  constexpr int kRPP = kVbConsumers / kLPR;
  constexpr int kTPT = kTile / kRPP;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* empty = full + kVbStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc);
  uint8_t* tile = smem + L::kTileT;
  const int ntiles = Npad / kTile;
  const int total = ntiles * H * B;
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int s = 0; s < kVbStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kVbConsumers);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (tid >= kVbConsumers) {
    // ------------------------------------------------------------ producer warp
    const int lane = tid - kVbConsumers;
    uint32_t it = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x, ++it) {
      const int s = static_cast<int>(it % kVbStages);
      const uint32_t use = it / kVbStages;
      bool ok = true;
      if (lane == 0 && use > 0) ok = mbar_wait_bounded(&empty[s], (use - 1) & 1, abort_flag, timeout_ns);
      if (!__shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0)) break;
      const int tl = item % ntiles;
      const int h = H - 1 - (item / ntiles) % H;   // heads last-to-first, as v_quant_t
      const int b = item / (ntiles * H);
      const int n0 = tl * kTile;
      // One 2-D copy: rows b*N + n0 .. +127 of V seen as [B*N, tok_stride] BF16, columns
      // h*D .. +D-1.  Rows past this batch (or past B*N, zero-filled) are never read.
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(L::kStageBytes));
        tma_load_2d(smem + s * L::kStageBytes, &tm_v, h * D, b * N + n0, &full[s]);
      }
    }
    if (*abort_flag && lane == 0) {
      // Drain: wait (bounded) for the last copy issued into each ring slot.
      int no_abort = 0;
      volatile int* nf = reinterpret_cast<volatile int*>(&no_abort);
      for (uint32_t s = 0; s < kVbStages; ++s)
        if (it > s) {
          const uint32_t last = ((it - 1 - s) / kVbStages) * kVbStages + s;
          mbar_wait_bounded(&full[s], (last / kVbStages) & 1, nf, 200000000);
        }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int cg = tid % kLPR;
    const int r0 = tid / kLPR;
    const int d0 = cg * 8;
    uint32_t it = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x, ++it) {
      const int s = static_cast<int>(it % kVbStages);
      const int tl = item % ntiles;
      const int h = H - 1 - (item / ntiles) % H;
      const int b = item / (ntiles * H);
      const int n0 = tl * kTile;
      const int64_t bhd = (static_cast<int64_t>(b) * H + h) * D;
      float mean[8], inv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        mean[i] = v_mean[bhd + d0 + i];
        inv[i] = v_inv[bhd + d0 + i];
      }
      // Every consumer leaves its bounded wait; a timeout has raised the abort flag,
      // which all 256 read after the barrier and leave the loop together.
      mbar_wait_bounded(&full[s], (it / kVbStages) & 1, abort_flag, timeout_ns);
      consumer_bar_sync();
      if (*abort_flag) break;
      const uint8_t* st = smem + s * L::kStageBytes;
#pragma unroll
      for (int t = 0; t < kTPT; ++t) {
        const int nl = r0 + t * kRPP;
        const int n = n0 + nl;
        uint32_t w0 = 0u, w1 = 0u;
        if (n < N) {
          float f[8];
          unpack8(*reinterpret_cast<const uint4*>(st + nl * L::kRowBytes + 2 * d0), f);
          float y[8];
#pragma unroll
          for (int i = 0; i < 8; i += 2) {   // RN(RN(v - mean) * inv) on pairs
            const f32x2_t c = x2_mul(x2_sub(x2_of(f[i], f[i + 1]), x2_of(mean[i], mean[i + 1])), x2_of(inv[i], inv[i + 1]));
            y[i] = x2_lo(c);
            y[i + 1] = x2_hi(c);
          }
          w0 = cvt_e4m3x2(y[0], y[1]) | (cvt_e4m3x2(y[2], y[3]) << 16);
          w1 = cvt_e4m3x2(y[4], y[5]) | (cvt_e4m3x2(y[6], y[7]) << 16);
        }
        *reinterpret_cast<uint2*>(tile + nl * L::kPitch + d0) = make_uint2(w0, w1);
      }
      mbar_arrive(&empty[s]);              // this stage's rows are consumed
      consumer_bar_sync();                 // the code tile is complete
      constexpr int kUnits = (D / 4) * (kTile / 16);
      for (int u = tid; u < kUnits; u += kVbConsumers) {
        const int d4 = u % (D / 4);
        const int qc = u / (D / 4);
        uint32_t col[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t r[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            r[i] = *reinterpret_cast<const uint32_t*>(tile + (qc * 16 + 4 * j + i) * L::kPitch + 4 * d4);
          const uint32_t lo01 = __byte_perm(r[0], r[1], 0x5140);
          const uint32_t lo23 = __byte_perm(r[2], r[3], 0x5140);
          const uint32_t hi01 = __byte_perm(r[0], r[1], 0x7362);
          const uint32_t hi23 = __byte_perm(r[2], r[3], 0x7362);
          col[0][j] = __byte_perm(lo01, lo23, 0x5410);
          col[1][j] = __byte_perm(lo01, lo23, 0x7632);
          col[2][j] = __byte_perm(hi01, hi23, 0x5410);
          col[3][j] = __byte_perm(hi01, hi23, 0x7632);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(out + (bhd + 4 * d4 + c) * Npad + n0 + qc * 16) =
              make_uint4(col[c][0], col[c][1], col[c][2], col[c][3]);
      }
      consumer_bar_sync();                 // the code tile is free for the next item
    }
  }
  __syncthreads();
  if (*abort_flag && tid == 0) atomicExch(err, 1);
}

// ----------------------------------------------------------------------------
// sage_quant_qkv: the statistics passes of sage_quant_qk and sage_quant_v in
// one launch and both finalizes in another (the code passes follow as their
// own two launches), so that each launch has enough CTAs to fill the GPU on
// small shapes.  The CTA bodies are the same functions, so the bytes are
// identical.
// ----------------------------------------------------------------------------
// Grid (nsb, B, 2 * zc), zc channel chunks per tensor: z < zc the V sums,
// minima and maxima (psum_v, pmin, pmax), the rest the K column sums (psum_k).  K goes last so that it is the
// part still in L2 when the K code pass (the first after the finalize) reads it
// again; measured 5% faster on the mid-video shape than K first.
__global__ void __launch_bounds__(128) colstats_kv(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                                                   int N, int HD, int64_t k_stride, int64_t v_stride, int nsb,
                                                   int zc, double* __restrict__ psum_k, double* __restrict__ psum_v,
                                                   float* __restrict__ pmin, float* __restrict__ pmax) {
  pdl_enter();
  const int z = static_cast<int>(blockIdx.z);
  if (z >= zc)
    colstats_body<false>(blockIdx.x, blockIdx.y, z - zc, k, N, HD, k_stride, nsb, psum_k, nullptr, nullptr);
  else
    colstats_body<true>(blockIdx.x, blockIdx.y, z, v, N, HD, v_stride, nsb, psum_v, pmin, pmax);
}

// Grid (nk + nv) of 1024 threads: blocks < nk the K mean, the rest the V
// statistics (32 channels per block each).
__global__ void __launch_bounds__(1024) finalize_kv(const double* __restrict__ psum_k,
                                                    const double* __restrict__ psum_v,
                                                    const float* __restrict__ pmin, const float* __restrict__ pmax,
                                                    int B, int N, int HD, int nsb, int nk,
                                                    uint16_t* __restrict__ mean_ws, uint16_t* __restrict__ mean_out,
                                                    float* __restrict__ v_mean, float* __restrict__ v_scale,
                                                    float* __restrict__ v_inv) {
  pdl_enter();
  __shared__ double sh[kSumLanes][33];
  __shared__ float shn[kSumLanes][33];
  __shared__ float shx[kSumLanes][33];
  const int bx = static_cast<int>(blockIdx.x);
  if (bx < nk)
    k_mean_body(bx, psum_k, B, N, HD, nsb, mean_ws, mean_out, sh);
  else
    v_stats_body(bx - nk, psum_v, pmin, pmax, B, N, HD, nsb, v_mean, v_scale, v_inv, sh, shn, shx);
}

}  // namespace sage
