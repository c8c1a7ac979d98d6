// sage_api.cu - host side of the C ABI declared in include/sage.h.
//
// Validates every argument before launching, lays out the caller's workspace,
// encodes the TMA tensor maps of the attention operands, launches the kernels
// of sage_quant.cuh / sage_attn.cuh on the caller's stream and reports errors
// as status codes with a thread-local message.  Nothing here allocates device
// memory or synchronises, except sage_check().
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <type_traits>

#include "sage.h"
#include "fp8_linear.cuh"
#include "sage_attn.cuh"
#include "sage_quant.cuh"

namespace {

__device__ int g_sage_err;  // set to 1 by a kernel that gave up a bounded wait

thread_local std::string g_last_error;
std::atomic<int64_t> g_timeout_ns{2000000000LL};

sage_status fail(sage_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

sage_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SAGE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  sage_status status = SAGE_OK;
  std::string message;
  int* err_ptr = nullptr;
  int sm_count = 0;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Once per device: check for sm_100, look up the error word, raise the shared
// memory limit of the attention kernels, and find cuTensorMapEncodeTiled.
sage_status device_setup(int* dev_out, int** err_out, int* sm_count_out = nullptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SAGE_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceState& ds = g_dev[dev];
  if (!ds.ready) {
    ds.ready = true;
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) {
      ds.status = SAGE_ERR_CUDA;
      ds.message = std::string("cudaGetDeviceProperties: ") + cudaGetErrorString(e);
    } else if (prop.major != 10 || prop.minor != 0) {
      ds.status = SAGE_ERR_UNSUPPORTED;
      ds.message = "this library is built for sm_100a (B200); device is sm_" + std::to_string(prop.major) +
                   std::to_string(prop.minor);
    } else {
      ds.sm_count = prop.multiProcessorCount;
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_sage_err);
      if (e == cudaSuccess) {
        ds.err_ptr = static_cast<int*>(p);
        e = cudaFuncSetAttribute(sage::sage_attn_kernel<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 sage::AttnSmem<128>::kAlloc);
      }
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(sage::sage_attn_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 sage::AttnSmem<64>::kAlloc);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(sage::sage_attn_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 sage::AttnSmem<128>::kAlloc);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(sage::sage_attn_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 sage::AttnSmem<64>::kAlloc);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(sage::sage_attn_p_codes_kernel<128, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, sage::AttnSmem<128>::kAlloc);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(sage::sage_attn_p_codes_kernel<64, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, sage::AttnSmem<64>::kAlloc);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(sage::sage_attn_p_codes_kernel<128, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, sage::AttnSmem<128>::kAlloc);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(sage::sage_attn_p_codes_kernel<64, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, sage::AttnSmem<64>::kAlloc);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(sage::v_codes_tma<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 sage::VbSmem<128>::kAlloc);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(sage::v_codes_tma<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 sage::VbSmem<64>::kAlloc);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(sage::fp8_gemm_kernel<256, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 sage::GemmSmem<256>::kAlloc);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(sage::fp8_gemm_kernel<256, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 sage::GemmSmem<256>::kAlloc);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(sage::fp8_gemm_kernel<192, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 sage::GemmSmem<192>::kAlloc);
      if (e == cudaSuccess && !g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e == cudaSuccess && (q != cudaDriverEntryPointSuccess || !fn)) e = cudaErrorSymbolNotFound;
        if (e == cudaSuccess) g_encode = reinterpret_cast<EncodeTiledFn>(fn);
      }
      if (e != cudaSuccess) {
        ds.status = SAGE_ERR_CUDA;
        ds.message = std::string("device setup: ") + cudaGetErrorString(e);
      }
    }
  }
  if (ds.status != SAGE_OK) return fail(ds.status, "%s", ds.message.c_str());
  *dev_out = dev;
  *err_out = ds.err_ptr;
  if (sm_count_out) *sm_count_out = ds.sm_count;
  return SAGE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t npad_of(int N) { return (static_cast<int64_t>(N) + 127) / 128 * 128; }

// Shape checks shared by every call.  Host-only: runs without a GPU.
sage_status check_shape(const sage_shape& s, int64_t* tok_stride) {
  if (s.B < 1 || s.N < 1 || s.H < 1) return fail(SAGE_ERR_INVALID_ARG, "B, N, H must be >= 1 (got %d, %d, %d)", s.B, s.N, s.H);
  if (s.D != 64 && s.D != 128) return fail(SAGE_ERR_UNSUPPORTED, "D must be 64 or 128 (got %d)", s.D);
  const int64_t hd = static_cast<int64_t>(s.H) * s.D;
  const int64_t ts = s.tok_stride == 0 ? hd : s.tok_stride;
  if (ts < hd) return fail(SAGE_ERR_INVALID_ARG, "tok_stride %lld < H*D %lld", (long long)ts, (long long)hd);
  if (ts % 8 != 0) return fail(SAGE_ERR_ALIGNMENT, "tok_stride %lld is not a multiple of 8", (long long)ts);
  const int64_t np = npad_of(s.N);
  if (static_cast<int64_t>(s.B) * s.H * np >= (int64_t(1) << 31) ||
      static_cast<int64_t>(s.B) * s.H * s.D >= (int64_t(1) << 31) || s.H > 65535 || 2LL * s.B > 65535)
    return fail(SAGE_ERR_INVALID_ARG, "shape too large (B*H*Npad must stay below 2^31)");
  if (s.cu_seqlens) {
    if (s.n_seg < 1) return fail(SAGE_ERR_INVALID_ARG, "n_seg must be >= 1 with cu_seqlens");
    if (s.cu_seqlens[0] != 0) return fail(SAGE_ERR_INVALID_ARG, "cu_seqlens[0] must be 0");
    for (int i = 0; i < s.n_seg; ++i)
      if (s.cu_seqlens[i + 1] < s.cu_seqlens[i])
        return fail(SAGE_ERR_INVALID_ARG, "cu_seqlens must be non-decreasing (index %d)", i + 1);
    if (s.cu_seqlens[s.n_seg] != s.N)
      return fail(SAGE_ERR_INVALID_ARG, "cu_seqlens[n_seg] = %d != N = %d", s.cu_seqlens[s.n_seg], s.N);
  } else if (s.n_seg != 0) {
    return fail(SAGE_ERR_INVALID_ARG, "n_seg = %d without cu_seqlens", s.n_seg);
  }
  for (const int g : {s.q_gran, s.k_gran})
    if (g != SAGE_GRAN_BLOCK64 && g != SAGE_GRAN_TOKEN && g != SAGE_GRAN_SEGMENT64)
      return fail(SAGE_ERR_INVALID_ARG, "q_gran / k_gran must be a sage_gran value (got %d)", g);
  if ((s.q_gran == SAGE_GRAN_SEGMENT64 || s.k_gran == SAGE_GRAN_SEGMENT64) && s.n_seg > SAGE_MAX_SEGMENTS)
    return fail(SAGE_ERR_UNSUPPORTED, "segment-local scale blocks take at most %d segments (got %d)",
                SAGE_MAX_SEGMENTS, s.n_seg);
  *tok_stride = ts;
  return SAGE_OK;
}

struct WsLayout {
  size_t psum, pmin, pmax, kmean, vinv, psum_v, single, total;
};
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
WsLayout ws_layout(const sage_shape& s) {
  const size_t nsb = (static_cast<size_t>(s.N) + sage::kSumBlock - 1) / sage::kSumBlock;
  const size_t part = static_cast<size_t>(s.B) * nsb * s.H * s.D;
  const size_t chans = static_cast<size_t>(s.B) * s.H * s.D;
  WsLayout w;
  w.psum = 0;
  w.pmin = align256(w.psum + part * 8);
  w.pmax = align256(w.pmin + part * 4);
  w.kmean = align256(w.pmax + part * 4);
  w.vinv = align256(w.kmean + chans * 2);
  w.single = align256(w.vinv + chans * 4);      // what sage_quant_qk or sage_quant_v alone needs
  w.psum_v = w.single;                          // sage_quant_qkv: V partials beside K's
  w.total = align256(w.psum_v + part * 8);
  return w;
}

sage_status check_ws(const sage_shape& s, const void* ws, size_t ws_bytes, WsLayout* lay, bool fused = false) {
  *lay = ws_layout(s);
  const size_t need = fused ? lay->total : lay->single;
  if (!ws) return fail(SAGE_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(SAGE_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  if (ws_bytes < need)
    return fail(SAGE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  return SAGE_OK;
}

#define SAGE_NEED(p, name) \
  do { if (!(p)) return fail(SAGE_ERR_INVALID_ARG, "%s is NULL", name); \
       if (!aligned16(p)) return fail(SAGE_ERR_ALIGNMENT, "%s is not 16-byte aligned", name); } while (0)

// Launches with programmatic stream serialization allowed: the kernel may be
// scheduled while the previous kernel in the stream is still running; every
// kernel of this library begins with pdl_enter(), which waits for that kernel
// to complete (and its writes to be visible) before anything is read.
// kEarly = false: an ordinary launch (after the previous kernel has finished),
// used for the attention kernel: with its blocks scheduled early beside the
// last quantization pass it measured 0.35% slower on one B200 and the same on
// another, for a gain of a few microseconds per step at most.
template <bool kEarly = true, typename... KArgs, typename... Args>
void pdl_launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = kEarly ? 1 : 0;
  // A failed launch is also recorded as this thread's last CUDA error, which
  // launch_check() reads after the call's launches.
  (void)cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

sage_status launch_check(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return SAGE_OK;
}

sage_status encode_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                      uint32_t box_outer, CUtensorMapSwizzle swz) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SAGE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return SAGE_OK;
}

static_assert(sage::kMaxSegments == SAGE_MAX_SEGMENTS, "segment table size");
static_assert(sage::kGranBlock64 == SAGE_GRAN_BLOCK64 && sage::kGranToken == SAGE_GRAN_TOKEN &&
                  sage::kGranSegment64 == SAGE_GRAN_SEGMENT64,
              "granularity codes");

// Segments of the shape (one segment [0, N) without cu_seqlens), then the
// padding [N, Npad) as one more, with the number of 64-token blocks before each.
void build_seg_table(const sage_shape& s, sage::SegTable* tab) {
  std::memset(tab, 0, sizeof(*tab));
  int n = 0, blocks = 0;
  auto add = [&](int a, int e) {
    tab->start[n] = a;
    tab->gbase[n] = blocks;
    blocks += (e - a + sage::kQKBlock - 1) / sage::kQKBlock;
    ++n;
    tab->start[n] = e;
  };
  if (s.cu_seqlens) {
    for (int i = 0; i < s.n_seg; ++i) add(s.cu_seqlens[i], s.cu_seqlens[i + 1]);
  } else {
    add(0, s.N);
  }
  add(s.N, static_cast<int>(npad_of(s.N)));
  tab->gbase[n] = blocks;
  tab->n = n;
}

// The INT8 code pass of sage_quant_qk: the 64-token block kernel when both
// tensors use blocks, the group kernel otherwise.  kNR: rows first go through
// QK RMSNorm + RoPE (sage_quant_qk_normrope).
template <bool kNR>
void launch_qk_codes(const sage_shape& s, int64_t ts, const uint16_t* qb, const uint16_t* kb,
                     const uint16_t* kmean, int8_t* q_codes, float* q_scale, int8_t* k_codes, float* k_scale,
                     const sage::NormRopeArgs& nr, cudaStream_t cs) {
  const int Npad = static_cast<int>(npad_of(s.N));
  if (s.q_gran == SAGE_GRAN_BLOCK64 && s.k_gran == SAGE_GRAN_BLOCK64) {
    // one 128-token tile per CTA, or one 64-token block with the norm / RoPE
    const dim3 g(Npad / (kNR ? sage::kQKBlock : sage::kTile), s.H, 2 * s.B);
    if (s.D == 128)
      pdl_launch(sage::qk_block_quant<128, kNR>, g, 256, 0, cs, qb, kb, s.N, s.B, s.H, Npad, ts, kmean, q_codes,
                 q_scale, k_codes, k_scale, nr);
    else
      pdl_launch(sage::qk_block_quant<64, kNR>, g, 256, 0, cs, qb, kb, s.N, s.B, s.H, Npad, ts, kmean, q_codes,
                 q_scale, k_codes, k_scale, nr);
    return;
  }
  sage::SegTable tab;
  build_seg_table(s, &tab);
  const int tiles = Npad / sage::kTile;
  const int seg_ctas = (tab.gbase[tab.n] + 1) / 2;
  int gx = 0;
  for (const int g : {s.q_gran, s.k_gran}) gx = std::max(gx, g == SAGE_GRAN_SEGMENT64 ? seg_ctas : tiles);
  const dim3 grid(gx, s.H, 2 * s.B);
  // The eight (Q, K) granularity pairs other than (block, block), each for
  // D = 64 and 128.
  auto launch = [&](auto dq, auto dk) {
    constexpr int GQ = decltype(dq)::value;
    constexpr int GK = decltype(dk)::value;
    if constexpr (GQ != sage::kGranBlock64 || GK != sage::kGranBlock64) {
      if (s.D == 128)
        pdl_launch(sage::qk_group_quant<128, GQ, GK, kNR>, grid, 256, 0, cs, qb, kb, s.N, s.B, s.H, Npad, ts, kmean,
                   q_codes, q_scale, k_codes, k_scale, tab, nr);
      else
        pdl_launch(sage::qk_group_quant<64, GQ, GK, kNR>, grid, 256, 0, cs, qb, kb, s.N, s.B, s.H, Npad, ts, kmean,
                   q_codes, q_scale, k_codes, k_scale, tab, nr);
    }
  };
  using G0 = std::integral_constant<int, sage::kGranBlock64>;
  using G1 = std::integral_constant<int, sage::kGranToken>;
  using G2 = std::integral_constant<int, sage::kGranSegment64>;
  auto with_k = [&](auto dq) {
    if (s.k_gran == SAGE_GRAN_BLOCK64) launch(dq, G0{});
    else if (s.k_gran == SAGE_GRAN_TOKEN) launch(dq, G1{});
    else launch(dq, G2{});
  };
  if (s.q_gran == SAGE_GRAN_BLOCK64) with_k(G0{});
  else if (s.q_gran == SAGE_GRAN_TOKEN) with_k(G1{});
  else with_k(G2{});
}

// The V code pass of sage_quant_qkv: persistent, TMA staged (v_codes_tma), two
// CTAs per SM.
template <int D>
sage_status launch_v_codes(const sage_shape& s, int Npad, int64_t vts, const uint16_t* vb, const float* v_mean,
                           const float* vinv, uint8_t* v_codes_t, int* err, int sm_count, cudaStream_t cs) {
  // V as a [B*N, tok_stride] BF16 matrix; one box = 128 token rows x D channels.
  CUtensorMap tv;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(vts), static_cast<cuuint64_t>(s.B) * s.N};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(vts) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(D), static_cast<cuuint32_t>(sage::kTile)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<uint16_t*>(vb), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SAGE_ERR_CUDA, "cuTensorMapEncodeTiled (V rows) failed (%d)", static_cast<int>(r));
  const int total = (Npad / sage::kTile) * s.H * s.B;
  const int grid = std::min(total, 2 * (sm_count > 0 ? sm_count : 148));
  pdl_launch(sage::v_codes_tma<D>, grid, sage::kVbThreads, sage::VbSmem<D>::kAlloc, cs, tv, vb, s.N, s.H, s.B, Npad,
             vts, v_mean, vinv, v_codes_t, err, g_timeout_ns.load());
  return SAGE_OK;
}

template <int D>
__global__ void selftest_wait_kernel(int64_t timeout_ns, int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sage::mbar_init(&bar, 1);
    abort_flag = 0;
    sage::fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the bounded wait must give up.
  const bool ok = sage::mbar_wait_bounded(&bar, 0, reinterpret_cast<volatile int*>(&abort_flag), timeout_ns);
  __syncthreads();
  if (threadIdx.x == 0 && (!ok || abort_flag)) atomicExch(err, 1);
  // Complete the barrier's phase so that no wait on it stays pending.
  if (threadIdx.x == 0) sage::mbar_arrive(&bar);
}

}  // namespace

// Scratch of sage_quant_qk_static: one array per GPU that loads the library.
static __device__ __align__(256) unsigned char g_qk_static_scratch[SAGE_QK_STATIC_SCRATCH_BYTES];

namespace {

unsigned char* g_qk_static_ptr[kMaxDevices];
std::mutex g_qk_static_mu;

// Device address of g_qk_static_scratch on the current device (looked up once
// per device; host code only holds a stand-in for the array's name).  The
// address is kept for the life of the process, so it is only valid while the
// device's primary context is the one it was looked up in (no device reset).
sage_status qk_static_scratch(int dev, unsigned char** out) {
  std::lock_guard<std::mutex> lock(g_qk_static_mu);
  if (!g_qk_static_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_qk_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    g_qk_static_ptr[dev] = static_cast<unsigned char*>(p);
  }
  *out = g_qk_static_ptr[dev];
  return SAGE_OK;
}

}  // namespace

extern "C" {

size_t sage_npad(int N) { return N < 1 ? 0 : static_cast<size_t>(npad_of(N)); }

size_t sage_workspace_bytes(sage_shape s) {
  int64_t ts = 0;
  if (check_shape(s, &ts) != SAGE_OK) return 0;
  return ws_layout(s).total;
}

const char* sage_last_error(void) { return g_last_error.c_str(); }

void sage_set_wait_timeout_ns(int64_t ns) { g_timeout_ns.store(ns > 0 ? ns : 2000000000LL); }

sage_status sage_quant_qk(const void* q, const void* k, sage_shape s, int8_t* q_codes, float* q_scale,
                          int8_t* k_codes, float* k_scale, void* k_mean, void* workspace, size_t ws_bytes,
                          sage_stream_t stream) {
  int64_t ts = 0;
  sage_status st = check_shape(s, &ts);
  if (st != SAGE_OK) return st;
  SAGE_NEED(q, "q");
  SAGE_NEED(k, "k");
  SAGE_NEED(q_codes, "q_codes");
  SAGE_NEED(q_scale, "q_scale");
  SAGE_NEED(k_codes, "k_codes");
  SAGE_NEED(k_scale, "k_scale");
  if (k_mean && !aligned16(k_mean)) return fail(SAGE_ERR_ALIGNMENT, "k_mean is not 16-byte aligned");
  WsLayout lay;
  if ((st = check_ws(s, workspace, ws_bytes, &lay)) != SAGE_OK) return st;
  int dev;
  int* err;
  if ((st = device_setup(&dev, &err)) != SAGE_OK) return st;

  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  double* psum = reinterpret_cast<double*>(ws + lay.psum);
  uint16_t* kmean = reinterpret_cast<uint16_t*>(ws + lay.kmean);
  const int HD = s.H * s.D;
  const int nsb = (s.N + sage::kSumBlock - 1) / sage::kSumBlock;
  const uint16_t* qb = static_cast<const uint16_t*>(q);
  const uint16_t* kb = static_cast<const uint16_t*>(k);

  pdl_launch(sage::colstats_partial<false>, dim3(nsb, s.B, (HD + 1023) / 1024), 128, 0, cs, kb, s.N, HD, ts, nsb,
             psum, nullptr, nullptr);
  pdl_launch(sage::k_mean_finalize, (s.B * HD + 31) / 32, 1024, 0, cs, psum, s.B, s.N, HD, nsb, kmean,
             static_cast<uint16_t*>(k_mean));
  launch_qk_codes<false>(s, ts, qb, kb, kmean, q_codes, q_scale, k_codes, k_scale, sage::NormRopeArgs{}, cs);
  return launch_check("sage_quant_qk launch");
}

sage_status sage_quant_qkv(const void* q, const void* k, const void* v, sage_shape s, int64_t v_tok_stride,
                           int8_t* q_codes, float* q_scale, int8_t* k_codes, float* k_scale, void* k_mean,
                           uint8_t* v_codes_t, float* v_scale, float* v_mean, void* workspace, size_t ws_bytes,
                           sage_stream_t stream) {
  if (s.q_gran != SAGE_GRAN_BLOCK64 || s.k_gran != SAGE_GRAN_BLOCK64) {
    // finer scale groups: the two calls one after the other
    sage_status st = sage_quant_qk(q, k, s, q_codes, q_scale, k_codes, k_scale, k_mean, workspace, ws_bytes,
                                   stream);
    if (st != SAGE_OK) return st;
    sage_shape sv = s;
    sv.tok_stride = v_tok_stride;
    return sage_quant_v(v, sv, v_codes_t, v_scale, v_mean, workspace, ws_bytes, stream);
  }
  int64_t ts = 0, vts = 0;
  sage_status st = check_shape(s, &ts);
  if (st != SAGE_OK) return st;
  sage_shape sv = s;
  sv.tok_stride = v_tok_stride;
  if ((st = check_shape(sv, &vts)) != SAGE_OK) return st;
  SAGE_NEED(q, "q");
  SAGE_NEED(k, "k");
  SAGE_NEED(v, "v");
  SAGE_NEED(q_codes, "q_codes");
  SAGE_NEED(q_scale, "q_scale");
  SAGE_NEED(k_codes, "k_codes");
  SAGE_NEED(k_scale, "k_scale");
  SAGE_NEED(v_codes_t, "v_codes_t");
  SAGE_NEED(v_scale, "v_scale");
  SAGE_NEED(v_mean, "v_mean");
  if (k_mean && !aligned16(k_mean)) return fail(SAGE_ERR_ALIGNMENT, "k_mean is not 16-byte aligned");
  WsLayout lay;
  if ((st = check_ws(s, workspace, ws_bytes, &lay, true)) != SAGE_OK) return st;
  int dev;
  int* err;
  int sm_count = 0;
  if ((st = device_setup(&dev, &err, &sm_count)) != SAGE_OK) return st;

  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  double* psum_k = reinterpret_cast<double*>(ws + lay.psum);
  double* psum_v = reinterpret_cast<double*>(ws + lay.psum_v);
  float* pmin = reinterpret_cast<float*>(ws + lay.pmin);
  float* pmax = reinterpret_cast<float*>(ws + lay.pmax);
  uint16_t* kmean = reinterpret_cast<uint16_t*>(ws + lay.kmean);
  float* vinv = reinterpret_cast<float*>(ws + lay.vinv);
  const int HD = s.H * s.D;
  const int nsb = (s.N + sage::kSumBlock - 1) / sage::kSumBlock;
  const int Npad = static_cast<int>(npad_of(s.N));
  const int zc = (HD + 1023) / 1024;
  const uint16_t* qb = static_cast<const uint16_t*>(q);
  const uint16_t* kb = static_cast<const uint16_t*>(k);
  const uint16_t* vb = static_cast<const uint16_t*>(v);

  pdl_launch(sage::colstats_kv, dim3(nsb, s.B, 2 * zc), 128, 0, cs, kb, vb, s.N, HD, ts, vts, nsb, zc, psum_k, psum_v,
             pmin, pmax);
  const int nf = (s.B * HD + 31) / 32;
  pdl_launch(sage::finalize_kv, 2 * nf, 1024, 0, cs, psum_k, psum_v, pmin, pmax, s.B, s.N, HD, nsb, nf, kmean,
             static_cast<uint16_t*>(k_mean), v_mean, v_scale, vinv);
  // The code passes stay two launches: merged, the V blocks would take the Q/K
  // blocks' register allocation and fit fewer per SM (measured slower).
  const dim3 g(Npad / sage::kTile, s.H, 2 * s.B);
  if (s.D == 128) {
    pdl_launch(sage::qk_block_quant<128>, g, 256, 0, cs, qb, kb, s.N, s.B, s.H, Npad, ts, kmean, q_codes, q_scale,
               k_codes, k_scale, sage::NormRopeArgs{});
    if ((st = launch_v_codes<128>(s, Npad, vts, vb, v_mean, vinv, v_codes_t, err, sm_count, cs)) != SAGE_OK)
      return st;
  } else {
    pdl_launch(sage::qk_block_quant<64>, g, 256, 0, cs, qb, kb, s.N, s.B, s.H, Npad, ts, kmean, q_codes, q_scale,
               k_codes, k_scale, sage::NormRopeArgs{});
    if ((st = launch_v_codes<64>(s, Npad, vts, vb, v_mean, vinv, v_codes_t, err, sm_count, cs)) != SAGE_OK)
      return st;
  }
  return launch_check("sage_quant_qkv launch");
}

sage_status sage_quant_qk_normrope(const void* q, const void* k, sage_shape s, const sage_normrope* nr,
                                   int8_t* q_codes, float* q_scale, int8_t* k_codes, float* k_scale, void* k_mean,
                                   void* workspace, size_t ws_bytes, sage_stream_t stream) {
  int64_t ts = 0;
  sage_status st = check_shape(s, &ts);
  if (st != SAGE_OK) return st;
  SAGE_NEED(q, "q");
  SAGE_NEED(k, "k");
  SAGE_NEED(q_codes, "q_codes");
  SAGE_NEED(q_scale, "q_scale");
  SAGE_NEED(k_codes, "k_codes");
  SAGE_NEED(k_scale, "k_scale");
  if (!nr) return fail(SAGE_ERR_INVALID_ARG, "nr is NULL");
  SAGE_NEED(nr->q_weight, "nr->q_weight");
  SAGE_NEED(nr->k_weight, "nr->k_weight");
  SAGE_NEED(nr->rope_cos, "nr->rope_cos");
  SAGE_NEED(nr->rope_sin, "nr->rope_sin");
  if (!(nr->eps > 0.f) || !(nr->eps < 3.0e38f)) return fail(SAGE_ERR_INVALID_ARG, "nr->eps must be finite and > 0");
  if (k_mean && !aligned16(k_mean)) return fail(SAGE_ERR_ALIGNMENT, "k_mean is not 16-byte aligned");
  WsLayout lay;
  if ((st = check_ws(s, workspace, ws_bytes, &lay)) != SAGE_OK) return st;
  int dev;
  int* err;
  if ((st = device_setup(&dev, &err)) != SAGE_OK) return st;

  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  double* psum = reinterpret_cast<double*>(ws + lay.psum);
  uint16_t* kmean = reinterpret_cast<uint16_t*>(ws + lay.kmean);
  const int HD = s.H * s.D;
  const int nsb = (s.N + sage::kSumBlock - 1) / sage::kSumBlock;
  const uint16_t* qb = static_cast<const uint16_t*>(q);
  const uint16_t* kb = static_cast<const uint16_t*>(k);
  sage::NormRopeArgs a;
  a.q_w = static_cast<const uint16_t*>(nr->q_weight);
  a.k_w = static_cast<const uint16_t*>(nr->k_weight);
  a.cos = nr->rope_cos;
  a.sin = nr->rope_sin;
  a.eps = nr->eps;

  const dim3 sg(nsb, s.B, (HD + 1023) / 1024);
  if (s.D == 128)
    pdl_launch(sage::colstats_normrope<128>, sg, 128, 0, cs, kb, s.N, HD, ts, nsb, psum, a);
  else
    pdl_launch(sage::colstats_normrope<64>, sg, 128, 0, cs, kb, s.N, HD, ts, nsb, psum, a);
  pdl_launch(sage::k_mean_finalize, (s.B * HD + 31) / 32, 1024, 0, cs, psum, s.B, s.N, HD, nsb, kmean,
             static_cast<uint16_t*>(k_mean));
  launch_qk_codes<true>(s, ts, qb, kb, kmean, q_codes, q_scale, k_codes, k_scale, a, cs);
  return launch_check("sage_quant_qk_normrope launch");
}

sage_status sage_quant_v(const void* v, sage_shape s, uint8_t* v_codes_t, float* v_scale, float* v_mean,
                         void* workspace, size_t ws_bytes, sage_stream_t stream) {
  int64_t ts = 0;
  sage_status st = check_shape(s, &ts);
  if (st != SAGE_OK) return st;
  SAGE_NEED(v, "v");
  SAGE_NEED(v_codes_t, "v_codes_t");
  SAGE_NEED(v_scale, "v_scale");
  SAGE_NEED(v_mean, "v_mean");
  WsLayout lay;
  if ((st = check_ws(s, workspace, ws_bytes, &lay)) != SAGE_OK) return st;
  int dev;
  int* err;
  if ((st = device_setup(&dev, &err)) != SAGE_OK) return st;

  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  double* psum = reinterpret_cast<double*>(ws + lay.psum);
  float* pmin = reinterpret_cast<float*>(ws + lay.pmin);
  float* pmax = reinterpret_cast<float*>(ws + lay.pmax);
  float* vinv = reinterpret_cast<float*>(ws + lay.vinv);
  const int HD = s.H * s.D;
  const int nsb = (s.N + sage::kSumBlock - 1) / sage::kSumBlock;
  const int Npad = static_cast<int>(npad_of(s.N));
  const uint16_t* vb = static_cast<const uint16_t*>(v);

  pdl_launch(sage::colstats_partial<true>, dim3(nsb, s.B, (HD + 1023) / 1024), 128, 0, cs, vb, s.N, HD, ts, nsb, psum,
             pmin, pmax);
  pdl_launch(sage::v_stats_finalize, (s.B * HD + 31) / 32, 1024, 0, cs, psum, pmin, pmax, s.B, s.N, HD, nsb, v_mean,
             v_scale, vinv);
  const dim3 g(Npad / sage::kTile, s.H, s.B);
  if (s.D == 128)
    pdl_launch(sage::v_quant_t<128>, g, 256, 0, cs, vb, s.N, s.H, Npad, ts, v_mean, vinv, v_codes_t);
  else
    pdl_launch(sage::v_quant_t<64>, g, 256, 0, cs, vb, s.N, s.H, Npad, ts, v_mean, vinv, v_codes_t);
  return launch_check("sage_quant_v launch");
}

// sage_attn_fwd, and with p_codes set its diagnostic form sage_attn_fwd_p_codes.
static sage_status attn_launch(const int8_t* q_codes, const float* q_scale, const int8_t* k_codes,
                               const float* k_scale, const uint8_t* v_codes_t, const float* v_scale,
                               const float* v_mean, sage_shape s, float sm_scale, void* out, int out_fp32,
                               float* lse, uint8_t* p_codes, sage_stream_t stream) {
  int64_t ts = 0;
  sage_status st = check_shape(s, &ts);
  if (st != SAGE_OK) return st;
  SAGE_NEED(q_codes, "q_codes");
  SAGE_NEED(q_scale, "q_scale");
  SAGE_NEED(k_codes, "k_codes");
  SAGE_NEED(k_scale, "k_scale");
  SAGE_NEED(v_codes_t, "v_codes_t");
  SAGE_NEED(v_scale, "v_scale");
  SAGE_NEED(v_mean, "v_mean");
  SAGE_NEED(out, "out");
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return fail(SAGE_ERR_ALIGNMENT, "lse is not 4-byte aligned");
  if (!(sm_scale == sm_scale)) return fail(SAGE_ERR_INVALID_ARG, "sm_scale is NaN");
  int dev;
  int* err;
  int sm_count = 0;
  if ((st = device_setup(&dev, &err, &sm_count)) != SAGE_OK) return st;

  const int64_t Npad = npad_of(s.N);
  const uint64_t rows = static_cast<uint64_t>(s.B) * s.H * Npad;
  CUtensorMap tq, tk, tv;
  const CUtensorMapSwizzle qk_swz = s.D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if ((st = encode_2d(&tq, q_codes, s.D, rows, s.D, sage::kBM, qk_swz)) != SAGE_OK) return st;
  if ((st = encode_2d(&tk, k_codes, s.D, rows, s.D, sage::kBN, qk_swz)) != SAGE_OK) return st;
  if ((st = encode_2d(&tv, v_codes_t, Npad, static_cast<uint64_t>(s.B) * s.H * s.D, sage::kBN, s.D,
                      CU_TENSOR_MAP_SWIZZLE_128B)) != SAGE_OK)
    return st;

    // sm_scale <= 0: 1/sqrt(D) formed in double and rounded once to float.
  const float scale_f = sm_scale > 0.f ? sm_scale : static_cast<float>(1.0 / sqrt(static_cast<double>(s.D)));
  const double scale = static_cast<double>(scale_f);
  sage::AttnParams prm;
  prm.q_scale = q_scale;
  prm.k_scale = k_scale;
  prm.v_scale = v_scale;
  prm.v_mean = v_mean;
  prm.out = out;
  prm.lse = lse;
  prm.err = err;
  prm.N = s.N;
  prm.H = s.H;
  prm.Npad = static_cast<int>(Npad);
  prm.nkv = static_cast<int>(Npad / sage::kBN);
  prm.sl2e = static_cast<float>(scale * 1.4426950408889634);
  prm.out_fp32 = out_fp32 ? 1 : 0;
  prm.q_tok = s.q_gran != SAGE_GRAN_BLOCK64;
  prm.timeout_ns = g_timeout_ns.load();
  prm.p_codes = p_codes;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid(static_cast<unsigned>(Npad / sage::kBM), s.H, s.B);
  (void)sm_count;
  const bool k_tok = s.k_gran != SAGE_GRAN_BLOCK64;
  if (p_codes) {
    if (s.D == 128 && !k_tok)
      pdl_launch<false>(sage::sage_attn_p_codes_kernel<128, false>, grid, sage::kAttnThreads,
                        sage::AttnSmem<128>::kAlloc, cs, tq, tk, tv, prm);
    else if (s.D == 128)
      pdl_launch<false>(sage::sage_attn_p_codes_kernel<128, true>, grid, sage::kAttnThreads,
                        sage::AttnSmem<128>::kAlloc, cs, tq, tk, tv, prm);
    else if (!k_tok)
      pdl_launch<false>(sage::sage_attn_p_codes_kernel<64, false>, grid, sage::kAttnThreads,
                        sage::AttnSmem<64>::kAlloc, cs, tq, tk, tv, prm);
    else
      pdl_launch<false>(sage::sage_attn_p_codes_kernel<64, true>, grid, sage::kAttnThreads,
                        sage::AttnSmem<64>::kAlloc, cs, tq, tk, tv, prm);
    return launch_check("sage_attn_fwd_p_codes launch");
  }
  if (s.D == 128 && !k_tok)
    pdl_launch<false>(sage::sage_attn_kernel<128, false>, grid, sage::kAttnThreads, sage::AttnSmem<128>::kAlloc, cs,
                      tq, tk, tv, prm);
  else if (s.D == 128)
    pdl_launch<false>(sage::sage_attn_kernel<128, true>, grid, sage::kAttnThreads, sage::AttnSmem<128>::kAlloc, cs,
                      tq, tk, tv, prm);
  else if (!k_tok)
    pdl_launch<false>(sage::sage_attn_kernel<64, false>, grid, sage::kAttnThreads, sage::AttnSmem<64>::kAlloc, cs, tq,
                      tk, tv, prm);
  else
    pdl_launch<false>(sage::sage_attn_kernel<64, true>, grid, sage::kAttnThreads, sage::AttnSmem<64>::kAlloc, cs, tq,
                      tk, tv, prm);
  return launch_check("sage_attn_fwd launch");
}

sage_status sage_attn_fwd(const int8_t* q_codes, const float* q_scale, const int8_t* k_codes,
                          const float* k_scale, const uint8_t* v_codes_t, const float* v_scale,
                          const float* v_mean, sage_shape s, float sm_scale, void* out, int out_fp32, float* lse,
                          sage_stream_t stream) {
  return attn_launch(q_codes, q_scale, k_codes, k_scale, v_codes_t, v_scale, v_mean, s, sm_scale, out, out_fp32,
                     lse, nullptr, stream);
}

sage_status sage_attn_fwd_p_codes(const int8_t* q_codes, const float* q_scale, const int8_t* k_codes,
                                  const float* k_scale, const uint8_t* v_codes_t, const float* v_scale,
                                  const float* v_mean, sage_shape s, float sm_scale, void* out, int out_fp32,
                                  float* lse, uint8_t* p_codes, sage_stream_t stream) {
  SAGE_NEED(p_codes, "p_codes");
  return attn_launch(q_codes, q_scale, k_codes, k_scale, v_codes_t, v_scale, v_mean, s, sm_scale, out, out_fp32,
                     lse, p_codes, stream);
}

sage_status sage_fp8_quant_rows(const void* x, int R, int K, int64_t ld, uint8_t* codes, float* scale,
                                sage_stream_t stream) {
  if (R < 1 || K < 8) return fail(SAGE_ERR_INVALID_ARG, "R >= 1 and K >= 8 required (got %d, %d)", R, K);
  if (K % 8 != 0) return fail(SAGE_ERR_ALIGNMENT, "K = %d is not a multiple of 8", K);
  if (K > 16384) return fail(SAGE_ERR_UNSUPPORTED, "K = %d above 16384", K);
  const int64_t lds = ld == 0 ? K : ld;
  if (lds < K || lds % 8 != 0) return fail(SAGE_ERR_ALIGNMENT, "ld = %lld must be >= K and a multiple of 8", (long long)lds);
  SAGE_NEED(x, "x");
  SAGE_NEED(codes, "codes");
  if (!scale) return fail(SAGE_ERR_INVALID_ARG, "scale is NULL");
  if (reinterpret_cast<uintptr_t>(scale) & 3u) return fail(SAGE_ERR_ALIGNMENT, "scale is not 4-byte aligned");
  int dev;
  int* err;
  sage_status st;
  if ((st = device_setup(&dev, &err)) != SAGE_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  const int per = K / 8;
  if (per <= 4 * sage::kFqThreads)
    pdl_launch(sage::fp8_quant_rows_kernel<4>, R, sage::kFqThreads, 0, cs, xb, K, lds, codes, scale);
  else if (per <= 8 * sage::kFqThreads)
    pdl_launch(sage::fp8_quant_rows_kernel<8>, R, sage::kFqThreads, 0, cs, xb, K, lds, codes, scale);
  else
    pdl_launch(sage::fp8_quant_rows_kernel<16>, R, sage::kFqThreads, 0, cs, xb, K, lds, codes, scale);
  return launch_check("sage_fp8_quant_rows launch");
}

sage_status sage_fp8_linear(const uint8_t* xq, const float* sx, const uint8_t* wq, const float* sw, int M, int N,
                            int K, void* out, int out_fp32, sage_stream_t stream) {
  if (M < 1 || N < 1 || K < 16) return fail(SAGE_ERR_INVALID_ARG, "M, N >= 1 and K >= 16 required");
  if (K % 16 != 0) return fail(SAGE_ERR_ALIGNMENT, "K = %d is not a multiple of 16", K);
  if (N % 8 != 0) return fail(SAGE_ERR_ALIGNMENT, "N = %d is not a multiple of 8", N);
  SAGE_NEED(xq, "xq");
  SAGE_NEED(wq, "wq");
  SAGE_NEED(sx, "sx");
  SAGE_NEED(sw, "sw");
  SAGE_NEED(out, "out");
  int dev;
  int* err;
  int sm_count = 0;
  sage_status st;
  if ((st = device_setup(&dev, &err, &sm_count)) != SAGE_OK) return st;
  // Tile width: 256, unless 192-wide tiles fill the persistent grid's waves
  // enough better to pay for their ~11% more operand bytes per flop.  Measured
  // on 8192-token projections: 192 wins at K = 3072 (72.1 vs 76.8 us for
  // 3072 x 3072), 256 at K = 12288 (237.6 vs 241.7 us), so 192 is taken only
  // for K <= 4096.
  const int sms = sm_count > 0 ? sm_count : 148;
  auto fill = [&](int bn) {
    const int64_t tiles = static_cast<int64_t>((M + sage::kGemmBM - 1) / sage::kGemmBM) * ((N + bn - 1) / bn);
    const int64_t waves = (tiles + sms - 1) / sms;
    return static_cast<double>(tiles) / static_cast<double>(waves * sms);
  };
  const int BN = (K <= 4096 && fill(192) * 0.95 > fill(256)) ? 192 : 256;
  const int64_t tiles = static_cast<int64_t>((M + sage::kGemmBM - 1) / sage::kGemmBM) * ((N + BN - 1) / BN);
  const int grid = static_cast<int>(std::min<int64_t>(tiles, sms));
  // Last wave: when its R tiles would leave most SMs idle, each becomes
  // `split` column blocks (4 or 2, so that split * R <= the SMs), which the
  // whole grid shares.  A column block reads the same A tile for a fraction of
  // the products, so it takes more than 1 / split of a tile's time; the split
  // is taken only for 256-wide tiles, where the wave is at most half full and
  // N is a whole number of tiles.
  const int64_t rem = tiles % grid;
  int split = 1;
  if (BN == 256 && tiles > grid && rem > 0 && 2 * rem <= grid && N % BN == 0) split = 4 * rem <= grid ? 4 : 2;
  CUtensorMap ta, tb, tb_tail;
  if ((st = encode_2d(&ta, xq, K, M, sage::kGemmBK, sage::kGemmBM, CU_TENSOR_MAP_SWIZZLE_128B)) != SAGE_OK) return st;
  if ((st = encode_2d(&tb, wq, K, N, sage::kGemmBK, BN, CU_TENSOR_MAP_SWIZZLE_128B)) != SAGE_OK) return st;
  if (split == 1)
    tb_tail = tb;   // not read
  else if ((st = encode_2d(&tb_tail, wq, K, N, sage::kGemmBK, BN / split, CU_TENSOR_MAP_SWIZZLE_128B)) != SAGE_OK)
    return st;
  sage::GemmParams prm;
  prm.sx = sx;
  prm.sw = sw;
  prm.out = out;
  prm.M = M;
  prm.N = N;
  prm.K = K;
  prm.out_fp32 = out_fp32 ? 1 : 0;
  prm.err = err;
  prm.timeout_ns = g_timeout_ns.load();
  prm.tail_split = split;
  prm.tail_start = static_cast<int>(split > 1 ? tiles - rem : tiles);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (BN == 256 && split > 1)
    pdl_launch(sage::fp8_gemm_kernel<256, true>, grid, sage::kGemmThreads, sage::GemmSmem<256>::kAlloc, cs, ta, tb,
               tb_tail, prm);
  else if (BN == 256)
    pdl_launch(sage::fp8_gemm_kernel<256, false>, grid, sage::kGemmThreads, sage::GemmSmem<256>::kAlloc, cs, ta, tb,
               tb_tail, prm);
  else
    pdl_launch(sage::fp8_gemm_kernel<192, false>, grid, sage::kGemmThreads, sage::GemmSmem<192>::kAlloc, cs, ta, tb,
               tb_tail, prm);
  return launch_check("sage_fp8_linear launch");
}

sage_status sage_check(sage_stream_t stream) {
  int dev;
  int* err;
  sage_status st = device_setup(&dev, &err);
  if (st != SAGE_OK) return st;
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int flag = 0;
  e = cudaMemcpy(&flag, err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (flag) {
    const int zero = 0;
    e = cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
    return fail(SAGE_ERR_DEVICE_TIMEOUT, "a kernel gave up a bounded wait (timeout %lld ns)",
                (long long)g_timeout_ns.load());
  }
  return SAGE_OK;
}

sage_status sage_selftest_wait_timeout(int64_t timeout_ns, sage_stream_t stream) {
  if (timeout_ns <= 0 || timeout_ns > 10000000000LL)
    return fail(SAGE_ERR_INVALID_ARG, "timeout_ns must be in (0, 1e10]");
  int dev;
  int* err;
  sage_status st = device_setup(&dev, &err);
  if (st != SAGE_OK) return st;
  pdl_launch(selftest_wait_kernel<0>, 1, 32, 0, reinterpret_cast<cudaStream_t>(stream), timeout_ns, err);
  return launch_check("selftest launch");
}


sage_status sage_quant_qk_static(const void* q, const void* k, sage_shape s, int8_t* q_codes, float* q_scale,
                                 int8_t* k_codes, float* k_scale, void* k_mean, sage_stream_t stream) {
  int64_t ts = 0;
  sage_status st = check_shape(s, &ts);
  if (st != SAGE_OK) return st;
  SAGE_NEED(q, "q");
  SAGE_NEED(k, "k");
  SAGE_NEED(q_codes, "q_codes");
  SAGE_NEED(q_scale, "q_scale");
  SAGE_NEED(k_codes, "k_codes");
  SAGE_NEED(k_scale, "k_scale");
  if (k_mean && !aligned16(k_mean)) return fail(SAGE_ERR_ALIGNMENT, "k_mean is not 16-byte aligned");
  const size_t nsb_sz = (static_cast<size_t>(s.N) + sage::kSumBlock - 1) / sage::kSumBlock;
  const size_t chans = static_cast<size_t>(s.B) * s.H * s.D;
  const size_t psum_bytes = align256(chans * nsb_sz * 8);
  const size_t need = psum_bytes + align256(chans * 2);
  if (need > SAGE_QK_STATIC_SCRATCH_BYTES)
    return fail(SAGE_ERR_WORKSPACE,
                "sage_quant_qk_static: shape needs %zu bytes of scratch, the built-in array holds %u; "
                "use sage_quant_qk with a workspace",
                need, SAGE_QK_STATIC_SCRATCH_BYTES);
  int dev;
  int* err;
  if ((st = device_setup(&dev, &err)) != SAGE_OK) return st;
  unsigned char* scratch = nullptr;
  if ((st = qk_static_scratch(dev, &scratch)) != SAGE_OK) return st;

  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  double* psum = reinterpret_cast<double*>(scratch);
  uint16_t* kmean = reinterpret_cast<uint16_t*>(scratch + psum_bytes);
  const int HD = s.H * s.D;
  const int nsb = static_cast<int>(nsb_sz);
  const uint16_t* qb = static_cast<const uint16_t*>(q);
  const uint16_t* kb = static_cast<const uint16_t*>(k);
  // Every scratch byte read below is written earlier in the same call.
  pdl_launch(sage::colstats_partial<false>, dim3(nsb, s.B, (HD + 1023) / 1024), 128, 0, cs, kb, s.N, HD, ts, nsb,
             psum, nullptr, nullptr);
  pdl_launch(sage::k_mean_finalize, (s.B * HD + 31) / 32, 1024, 0, cs, psum, s.B, s.N, HD, nsb, kmean,
             static_cast<uint16_t*>(k_mean));
  launch_qk_codes<false>(s, ts, qb, kb, kmean, q_codes, q_scale, k_codes, k_scale, sage::NormRopeArgs{}, cs);
  return launch_check("sage_quant_qk_static launch");
}

}  // extern "C"
