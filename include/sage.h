/*
 * sage.h - C ABI of the B200 (sm_100a) quantized-attention library.
 *
 * The method (SageAttention2-style attention inside FLUX.3-Action and MiniMax-H3
 * DiT blocks) is described on these pages:
 *  - "FLUX.3 Action RTX 5090 report", 02 ENGINEERING, card 03 "SageAttention2":
 *    INT8 QK, FP8 PV, FP32 accumulation, K smooth and V smooth kept, NHD layout;
 *    and the last-round cards A (K centring fused into the INT8 quantization,
 *    keeping the BF16 rounding of the centred K; Q quantized with the same
 *    scale and INT8 rule) and C (V mean / scale / quant with V smoothing, V
 *    read in place from a wider projection output and written transposed and
 *    padded).
 *  - "MiniMax H3 on DGX Spark", 01 Precision map: Sage2++ = QK INT8 / PV FP8.
 *  - "为什么A10也能跑得动FLUX.1", 1.1: FP8 E4M3 = 4 exponent + 3 mantissa bits.
 * The pages give no formulas; the contract fixed here (64-token Q/K scale
 * blocks, per-channel V scales, 128-key tiles, rounding rules) is stated with
 * each call.
 *
 * Conventions for every call:
 *  - Tensors are device pointers owned by the caller.  The library never
 *    allocates or frees memory; scratch space is the caller's workspace.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and never synchronise.  Device-side wait timeouts are
 *    reported by sage_check().  The quantization and projection kernels are
 *    launched with programmatic dependent launch: their blocks may be
 *    scheduled while the previous kernel on the stream is still running, and
 *    each waits for that kernel to complete before it reads anything, so
 *    stream order is kept for every input, including the caller's own
 *    kernels and copies.
 *  - Arguments are validated on the host before any launch.  On an invalid
 *    argument nothing is launched, the call returns a non-zero sage_status,
 *    and sage_last_error() describes the problem (thread-local string).
 *  - Device pointers must be 16-byte aligned; padded rows/columns of every
 *    output are written (zero codes, zero scales) so outputs are fully defined.
 *  - Results are deterministic: fixed launch configurations, fixed reduction
 *    order, no atomics on values.
 *
 * Shapes: B batch, N tokens, H heads, D head dim (64 or 128).
 * Npad = sage_npad(N) = N rounded up to a multiple of 128.
 * BF16 inputs are [B, N, H, D] ("NHD"): element (b, n, h, d) sits at
 * b*N*tok_stride + n*tok_stride + h*D + d, tok_stride >= H*D (0 means H*D),
 * tok_stride a multiple of 8.
 */
#ifndef SAGE_H_
#define SAGE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SAGE_API __attribute__((visibility("default")))
#else
#define SAGE_API
#endif

struct CUstream_st;
typedef struct CUstream_st* sage_stream_t; /* same type as cudaStream_t */

typedef enum {
  SAGE_OK = 0,
  SAGE_ERR_INVALID_ARG = 1,    /* null pointer, bad shape, bad cu_seqlens   */
  SAGE_ERR_UNSUPPORTED = 2,    /* D not 64/128, or no sm_100 device          */
  SAGE_ERR_ALIGNMENT = 3,      /* pointer or stride alignment                */
  SAGE_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed          */
  SAGE_ERR_DEVICE_TIMEOUT = 5, /* a kernel gave up a bounded wait            */
  SAGE_ERR_WORKSPACE = 6       /* workspace missing or smaller than needed   */
} sage_status;

/* INT8 scale granularity of Q or K (the groups of tokens that share one
 * scale; every group spans all D channels of one (b, h)).
 *  SAGE_GRAN_BLOCK64    64-token blocks on one grid over the whole sequence
 *                       (the configurations' "Q/K INT8 blocks 64 tokens").
 *                       Scales: f32 [B, H, Npad/64], one per block.
 *  SAGE_GRAN_TOKEN      one scale per token.  On these tensor cores one thread
 *                       owns one query row, so this is the counterpart of the
 *                       per-thread granularity named in "FLUX.3 Action RTX
 *                       5090 report", card 03.  Scales: f32 [B, H, Npad].
 *  SAGE_GRAN_SEGMENT64  64-token blocks restarting at every segment start of
 *                       cu_seqlens (a block never mixes two streams of a
 *                       packed joint sequence; a segment's last block may be
 *                       short); the padding [N, Npad) continues the 64-token
 *                       grid from N.  Scales: f32 [B, H, Npad], every token
 *                       holding its block's scale.  At most SAGE_MAX_SEGMENTS
 *                       segments; without cu_seqlens the one segment is [0, N).
 * Padded tokens always get scale 0 and zero codes.  sage_quant_qk writes and
 * sage_attn_fwd reads the layouts that the shape's q_gran / k_gran select, so
 * both calls must be given the same values. */
typedef enum {
  SAGE_GRAN_BLOCK64 = 0,
  SAGE_GRAN_TOKEN = 1,
  SAGE_GRAN_SEGMENT64 = 2
} sage_gran;
#define SAGE_MAX_SEGMENTS 256

typedef struct {
  int B, N, H, D;
  int64_t tok_stride;         /* elements between consecutive tokens of the
                                 call's BF16 input(s); 0 means H*D           */
  const int32_t* cu_seqlens;  /* HOST pointer to n_seg+1 segment offsets of a
                                 packed joint sequence, or NULL.  Validated
                                 (starts at 0, non-decreasing, ends at N).
                                 Attention is full over the concatenation and
                                 the K/V means run over all N tokens; the
                                 offsets only place SAGE_GRAN_SEGMENT64 blocks. */
  int n_seg;
  int q_gran;                 /* sage_gran of the Q scales (0: 64-token blocks) */
  int k_gran;                 /* sage_gran of the K scales (0: 64-token blocks) */
} sage_shape;

/* N rounded up to a whole 128-row tile. */
SAGE_API size_t sage_npad(int N);

/* Bytes of device workspace needed by sage_quant_qk, sage_quant_v and
 * sage_quant_qkv for this shape (one buffer serves all; calls on one stream
 * may share it). */
SAGE_API size_t sage_workspace_bytes(sage_shape s);

/*
 * sage_quant_qk - K smoothing and INT8 block quantization of Q and K.
 * ("FLUX.3 Action RTX 5090 report", last-round card A; card 03.)
 *
 * in : q, k        BF16 [B, N, H, D] with s.tok_stride (both tensors).
 * out: q_codes     int8 [B, H, Npad, D]; rows >= N are 0.
 *      q_scale     f32  [B, H, Npad/64] (s.q_gran 64-token blocks) or
 *                  [B, H, Npad] (per token, segment-local blocks); 0 past N.
 *      k_codes     int8 [B, H, Npad, D]; k_scale f32 as q_scale, by s.k_gran.
 *      k_mean      BF16 [B, H, D] or NULL.
 * Rule: mean_k[b,h,d] = RN_bf16(sum_n k / N), the FP64 sum taken in a fixed
 * order (64-token blocks in token order; 32 interleaved lanes over blocks;
 * butterfly 16,8,4,2,1 over lanes) and the quotient rounded once to BF16;
 * kc = RN_bf16(RN_f32(k - mean_k)).  For each scale group (sage_gran) of one
 * (b,h) over all D: amax = max|x|, scale = RN(amax/127), inv = RN(127/amax),
 * code = clamp(RNE(RN(x*inv)), -127, 127); amax == 0 gives 0 scale and codes.
 * Q is quantized as is, K after centring.  Codes are bit-exact with that rule.
 * workspace: >= sage_workspace_bytes(s) bytes of device memory, 256-B aligned.
 */
SAGE_API sage_status sage_quant_qk(const void* q, const void* k, sage_shape s,
                          int8_t* q_codes, float* q_scale,
                          int8_t* k_codes, float* k_scale, void* k_mean,
                          void* workspace, size_t ws_bytes, sage_stream_t stream);

/*
 * sage_quant_qkv - sage_quant_qk and sage_quant_v of one attention call
 * together: the same outputs, bit for bit, in four kernel launches instead of
 * six (the K and V statistics in one, both finalizes in one, then the Q/K and
 * the V codes), so that the short statistics passes fill the GPU on small
 * shapes.
 *
 * in : q, k with s.tok_stride; v with v_tok_stride (0 means H*D).
 * out: as sage_quant_qk and sage_quant_v.
 * workspace: >= sage_workspace_bytes(s) bytes (the K and V partial sums are
 * kept apart here).  With finer scale groups (s.q_gran or s.k_gran not
 * SAGE_GRAN_BLOCK64) it runs the two calls one after the other.
 */
SAGE_API sage_status sage_quant_qkv(const void* q, const void* k, const void* v, sage_shape s,
                                    int64_t v_tok_stride, int8_t* q_codes, float* q_scale,
                                    int8_t* k_codes, float* k_scale, void* k_mean,
                                    uint8_t* v_codes_t, float* v_scale, float* v_mean,
                                    void* workspace, size_t ws_bytes, sage_stream_t stream);

/*
 * sage_quant_qk_normrope - sage_quant_qk on Q and K straight from the
 * projection: each (token, head) row first goes through RMSNorm and the rotary
 * position embedding, in BF16 rounding, inside the same kernels (the separate
 * BF16 write and re-read of the normed Q and K are gone).  ("FLUX 3 Action",
 * 1 Model Introduction: 4-axis (t, h, w, l) RoPE in the joint blocks; its
 * serving notes: QK RMSNorm + RoPE as one fused kernel at BF16 rounding level;
 * "FLUX.3 Action RTX 5090 report", last-round card B.)
 *
 * in : q, k        BF16 [B, N, H, D] projection outputs, s.tok_stride.
 *      nr          weights, eps and rotation tables (below); all device
 *                  pointers 16-byte aligned; eps finite and > 0.
 * out: as sage_quant_qk (any q_gran / k_gran).
 * Rule for one row x of D channels (L = D/8 lanes of 8 channels):
 *   ss = FP32 sum of x^2: lane g adds channels 8g .. 8g+7 in order from +0,
 *        then ss_g <- ss_g + ss_{g xor o} for o = L/2 .. 1;
 *   r  = RN(1 / RN(sqrt(RN(RN(ss / D) + eps))))  (correctly rounded);
 *   z  = RN_bf16(RN_bf16(RN(x * r)) * w);
 *   pair i = (z[2i], z[2i+1]) = (a, b), c = rope_cos[n, i], s = rope_sin[n, i]:
 *   out[2i] = RN_bf16(RN(RN(c*a) - RN(s*b))), out[2i+1] = RN_bf16(RN(RN(s*a) + RN(c*b))).
 * The K mean, K centring and INT8 rule of sage_quant_qk then apply to the
 * rows so produced.  Codes are bit-exact with that rule.
 */
typedef struct {
  const void* q_weight;    /* BF16 [D] RMSNorm weight of Q                    */
  const void* k_weight;    /* BF16 [D] RMSNorm weight of K                    */
  const float* rope_cos;   /* f32 [N, D/2]: cos of token n's angle for pair i  */
  const float* rope_sin;   /* f32 [N, D/2]: its sine                           */
  float eps;               /* added to the mean square, > 0                    */
} sage_normrope;

SAGE_API sage_status sage_quant_qk_normrope(const void* q, const void* k, sage_shape s,
                                            const sage_normrope* nr,
                                            int8_t* q_codes, float* q_scale,
                                            int8_t* k_codes, float* k_scale, void* k_mean,
                                            void* workspace, size_t ws_bytes, sage_stream_t stream);

/*
 * sage_quant_v - V smoothing and per-channel FP8 E4M3 quantization, written
 * transposed.  ("FLUX.3 Action RTX 5090 report", last-round card C; card 03.)
 *
 * in : v           BF16 [B, N, H, D] with s.tok_stride (may be a strided
 *                  slice of a wider projection output).
 * out: v_codes_t   E4M3 bytes [B, H, D, Npad]; tokens >= N are 0.
 *      v_scale     f32 [B, H, D]; v_mean f32 [B, H, D].
 * Rule: mean = RN_f32(sum/N) (FP64 sum, same order as sage_quant_qk);
 * amax = max(RN(vmax - mean), RN(mean - vmin)); scale = RN(amax/448),
 * inv = RN(448/amax) (0, 0 when amax == 0);
 * code = E4M3_RNE_satfinite(RN(RN(v - mean) * inv)).  Bit-exact with that rule.
 */
SAGE_API sage_status sage_quant_v(const void* v, sage_shape s, uint8_t* v_codes_t,
                         float* v_scale, float* v_mean,
                         void* workspace, size_t ws_bytes, sage_stream_t stream);

/*
 * sage_attn_fwd - O = softmax(Q K^T * sm_scale) V on the quantized operands.
 * ("FLUX.3 Action RTX 5090 report", card 03: INT8 QK, FP8 PV, FP32
 * accumulation, V mean added back; "MiniMax H3 on DGX Spark", 01.)
 *
 * in : the outputs of sage_quant_qk / sage_quant_v for the same shape
 *      (s.tok_stride is ignored here; s.q_gran and s.k_gran give the layouts
 *      of q_scale and k_scale).
 *      sm_scale <= 0 selects 1/sqrt(D).
 * out: out   [B, N, H, D], BF16 (out_fp32 == 0) or FP32 (out_fp32 != 0).
 *      lse   f32 [B, H, N] natural-log softmax denominator, or NULL.
 * Per 128-row query tile and 128-key tile: S = Qc Kc^T exactly in INT32 on the
 * tensor cores; t = RN(S * c) with c = RN(RN(qs_i * ks_j) * RN(sm_scale *
 * log2 e)), qs_i / ks_j the scales of the groups holding query i / key j;
 * running row max m = max(m, max t);
 * y = exp2(RN((S + B) * c + e')) with B = 1.5 * 2^23, e = RN(log2 448 - m)
 * and e' = RN(e - B * c), exp2 a fixed binary32 algorithm (Cody-Waite split,
 * quadratic, exponent-field add); l accumulates y; P8 = E4M3(y) (<= 448);
 * O_acc = O_acc * exp2(m_old - m_new) + P8 V8 (FP8 MMA, FP32 accumulation);
 * O = RN(O_acc * v_scale) * RN(1 / l) + v_mean.  Keys >= N are masked.  The
 * E4M3 codes of P are the contract's bit for bit; O matches the contract
 * within the tensor core's FP32 summation order and the row-sum order.
 */
SAGE_API sage_status sage_attn_fwd(const int8_t* q_codes, const float* q_scale,
                          const int8_t* k_codes, const float* k_scale,
                          const uint8_t* v_codes_t, const float* v_scale,
                          const float* v_mean, sage_shape s, float sm_scale,
                          void* out, int out_fp32, float* lse,
                          sage_stream_t stream);

/*
 * sage_attn_fwd_p_codes - sage_attn_fwd that also writes out the E4M3 codes of
 * P, so that a test can compare them with a reference one by one.  A
 * diagnostic: the same attention (out and lse as sage_attn_fwd's, bit for
 * bit), slower by the extra stores.
 *
 * out: p_codes  uint8 [B*H, N, sage_npad(N)], caller-owned, 16-byte aligned:
 *      the code of y = P~ * 448 for key j of query row i of head b*H + h is at
 *      ((b*H + h) * N + i) * sage_npad(N) + j, formed in key j's 128-key tile
 *      against that tile's running max; keys j >= N hold 0.
 * Errors: those of sage_attn_fwd; SAGE_ERR_INVALID_ARG for a NULL p_codes,
 * SAGE_ERR_ALIGNMENT when it is not 16-byte aligned.
 */
SAGE_API sage_status sage_attn_fwd_p_codes(const int8_t* q_codes, const float* q_scale,
                          const int8_t* k_codes, const float* k_scale,
                          const uint8_t* v_codes_t, const float* v_scale,
                          const float* v_mean, sage_shape s, float sm_scale,
                          void* out, int out_fp32, float* lse, uint8_t* p_codes,
                          sage_stream_t stream);

/*
 * sage_fp8_quant_rows - per-row E4M3 quantization of a BF16 matrix, for the
 * activations (one scale per token) and, offline, the weights (one scale per
 * output row) of sage_fp8_linear.  ("FLUX.3 Action RTX 5090 report", 02
 * ENGINEERING card 02: E4M3 projections with one scale per output row; "FLUX 3
 * Action" serving notes: per-token activation scales.)
 *
 * in : x       BF16 [R, K], row stride ld elements (0 means K; ld % 8 == 0).
 * out: codes   E4M3 bytes [R, K] (contiguous); scale f32 [R].
 * Rule per row: amax = max|x|, scale = RN(amax/448), inv = RN(448/amax),
 * code = E4M3_RNE_satfinite(RN(x * inv)); amax == 0 gives 0 scale and codes.
 * K % 8 == 0, 8 <= K <= 16384.  Bit-exact with that rule.
 */
SAGE_API sage_status sage_fp8_quant_rows(const void* x, int R, int K, int64_t ld, uint8_t* codes,
                                         float* scale, sage_stream_t stream);

/*
 * sage_fp8_linear - y = X W^T with row-wise FP8 operands on the tensor cores.
 *
 * in : xq E4M3 [M, K], sx f32 [M] (sage_fp8_quant_rows of the activations);
 *      wq E4M3 [N, K], sw f32 [N] (the weights' per-row codes and scales).
 * out: out [M, N] BF16 (out_fp32 == 0) or FP32, row-major.
 * acc[m, n] = sum_k xq[m,k] * wq[n,k] accumulated in FP32 by the tensor core;
 * y = RN(RN(acc * sx[m]) * sw[n]); the BF16 output is RN_bf16 of y.
 * K % 16 == 0, N % 8 == 0; all pointers 16-byte aligned.  The FP32 summation
 * order is the tensor core's, so results match an exact accumulation within
 * FP32 rounding, not bit for bit.
 */
SAGE_API sage_status sage_fp8_linear(const uint8_t* xq, const float* sx, const uint8_t* wq, const float* sw,
                                     int M, int N, int K, void* out, int out_fp32, sage_stream_t stream);

/* Synchronises `stream`, then reports and clears a device-side wait timeout
 * raised by any kernel of this library (SAGE_ERR_DEVICE_TIMEOUT), or a CUDA
 * error (SAGE_ERR_CUDA); SAGE_OK otherwise. */
SAGE_API sage_status sage_check(sage_stream_t stream);

/* Bound, in nanoseconds, on every wait inside the library's kernels (default
 * 2e9).  After it the kernel stops its work, drains its own copies and tensor
 * operations, releases tensor memory, records a timeout for sage_check() and
 * returns.  Values <= 0 restore the default. */
SAGE_API void sage_set_wait_timeout_ns(int64_t ns);

/* Failure-detection self-test: launches one CTA that waits on a barrier that
 * nothing completes, bounded by timeout_ns; afterwards sage_check() returns
 * SAGE_ERR_DEVICE_TIMEOUT and the context stays usable. */
SAGE_API sage_status sage_selftest_wait_timeout(int64_t timeout_ns, sage_stream_t stream);

/*
 * sage_quant_qk_static - sage_quant_qk without a workspace argument, for
 * callers that cannot allocate device memory: a plugin whose host framework
 * owns all device memory and offers no scratch hook, a runtime whose memory
 * budget is fixed at start-up, or code that must not call cudaMalloc /
 * cudaFree because those calls synchronise the device.  (The pages have no
 * counterpart; this is an interface variant, not a step of the method.)
 *
 * Same inputs, outputs and rule as sage_quant_qk, bit-identical results.  The
 * scratch (FP64 partial sums and the K mean) lives in one array inside the
 * library, SAGE_QK_STATIC_SCRATCH_BYTES (8 MiB) per GPU that loads the
 * library, held until the process exits.  Shapes whose scratch,
 * B*ceil(N/64)*H*D*8 + B*H*D*2 bytes (each part rounded up to 256), exceeds
 * it are rejected with SAGE_ERR_WORKSPACE before any launch.
 * The call allocates nothing.  Its first call on a device looks up the
 * array's device address (with that device current); make that first call
 * before any stream capture.  Every call on a device shares the one array and
 * it keeps the last call's contents (nothing in it needs to start at zero):
 * calls that overlap on the GPU (concurrent streams) race on it, so order
 * them on one stream or with events.  The looked-up address is kept for the
 * life of the process: do not call this entry point on a device after
 * cudaDeviceReset() (or anything else that re-creates its primary context),
 * because the kept address then belongs to the old context.
 */
#define SAGE_QK_STATIC_SCRATCH_BYTES (8u << 20)
SAGE_API sage_status sage_quant_qk_static(const void* q, const void* k, sage_shape s,
                                          int8_t* q_codes, float* q_scale,
                                          int8_t* k_codes, float* k_scale, void* k_mean,
                                          sage_stream_t stream);

/* Message describing the last non-OK status of this thread. */
SAGE_API const char* sage_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_H_ */
