/*
 * moeq — routed Mixture-of-Experts expert layer with quantized weights, for NVIDIA B200 (sm_100a).
 *
 * C ABI of libmoeq.so. Plain pointers and sizes only.
 *
 * Conventions for every entry point below:
 *  - Pointers to tensors are caller-owned DEVICE memory (cudaMalloc, a torch CUDA tensor, ...).
 *    The library never allocates, frees or keeps a pointer past the call. Scratch memory comes
 *    from the caller through `ws` / `ws_bytes`, sized by the matching *_workspace_size().
 *  - All tensors are dense, row-major, contiguous. bf16 values are passed as uint16_t bit
 *    patterns, E4M3 ("fn" variant: max 448, no infinities) values as uint8_t bit patterns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). Every call only
 *    enqueues work on that stream and returns; no call synchronizes with the host or reads
 *    device data back, so a sequence of calls can be captured in a CUDA graph.
 *  - Some kernels are launched as programmatic dependents of the kernel before them in the
 *    stream, which may be the caller's. Such a kernel may start early. Each of its CTAs waits
 *    for that kernel to complete, with its writes visible, before reading anything that kernel
 *    could have written, and before exiting. Stream order toward the caller's work is
 *    therefore unchanged: a call sees everything written before it on the stream, and its
 *    outputs are complete before the caller's next launch (ordinary, or waiting in the same
 *    way), copy or event on the stream.
 *  - Status: 0 on success, else one of the MOEQ_ERR_* codes; the calling thread's last error
 *    message is available from moe_last_error(). Arguments are validated on the host before
 *    anything is enqueued; a rejected call enqueues nothing. No C++ exception crosses the ABI.
 *  - Device data must satisfy the documented value ranges (e.g. expert ids in [0, E)); kernels
 *    skip out-of-range ids instead of writing out of bounds.
 *
 * Sources, cited by page title and section:
 *  [CHORD] "vLLM x Novita AI: Chord W4A16 INT4 MoE Kernel for Kimi K2.x" (Novita blog).
 *  [SGL]   "SGLang W8A8 Block FP8 quantized kernel config files: analysis and tuning guide"
 *          (xdnf.cn article on SGLang's fp8_kernel.py).
 */
#ifndef MOEQ_H
#define MOEQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOEQ_API __attribute__((visibility("default")))
#else
#define MOEQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MOEQ_OK 0
#define MOEQ_ERR_INVALID_ARG 1    /* null pointer, negative or inconsistent size */
#define MOEQ_ERR_UNSUPPORTED 2    /* shape, alignment or quantization scheme this library does not run */
#define MOEQ_ERR_WORKSPACE 3      /* ws_bytes smaller than the matching *_workspace_size() */
#define MOEQ_ERR_CUDA 4           /* a CUDA launch or API call failed (message has the CUDA error) */
#define MOEQ_ERR_DEVICE_TIMEOUT 5 /* a kernel gave up a bounded wait (reported by moe_device_status) */

/* Message of the calling thread's last failed call ("" if none). Valid until the next call. */
MOEQ_API const char *moe_last_error(void);

/* Library version string. */
MOEQ_API const char *moe_version(void);

/*
 * Top-k softmax routing, renormalised over the selected experts ([CHORD], "vLLM integration":
 * the layer consumes routing produced upstream; the definition taken is softmax over the E
 * logits, keep the k largest, divide by their sum).
 *   logits   f32 [T, E], finite values
 *   topk_ids i32 [T, k] out: expert of slot (t, j), in (logit descending, index ascending) order
 *   topk_w   f32 [T, k] out: exp(l - l_max) / sum over the k selected, computed in double
 * Limits: 1 <= k <= 32, k <= E <= 1024, T >= 0.
 */
MOEQ_API int moe_route_topk(const float *logits, int T, int E, int k, int32_t *topk_ids, float *topk_w,
                   void *stream);

/*
 * Token-to-expert alignment ([CHORD], "Two kernel families": the indexed kernels consume
 * sorted_ids / expert_ids / num_tokens_padded; figure 3: padding guards live in the indices,
 * activations are not padded; "vLLM integration": buffers are over-allocated so that no host
 * read of the routed count is needed).
 *   topk_ids  i32 [T, k], values in [0, E)
 *   sorted_ids i32 [T*k + E*(block_m-1)] out: for experts in ascending order, the flat slots
 *              f = t*k + j routed to it in ascending f, padded with the value T*k to a multiple
 *              of block_m; entries past num_tokens_padded also hold T*k
 *   expert_ids i32 [ceil((T*k + E*(block_m-1)) / block_m)] out: expert of each block of
 *              block_m entries, -1 past num_tokens_padded
 *   num_tokens_padded i32 [1] out: sum over experts of ceil(count / block_m) * block_m
 *   ws, ws_bytes: caller-owned device scratch (256-byte aligned) of moe_align_workspace_size()
 *              bytes; with it, more than 8192 slots are aligned by many CTAs (per-chunk counts,
 *              one scan, per-chunk stable scatter), without it (NULL / too small) by one CTA.
 *              Same result either way.
 * Bit-exact (integer). Limits: 1 <= block_m <= 256, E <= 1024, T*k <= 2^24.
 */
MOEQ_API int moe_align(const int32_t *topk_ids, int T, int k, int E, int block_m, int32_t *sorted_ids,
              int32_t *expert_ids, int32_t *num_tokens_padded, void *ws, size_t ws_bytes, void *stream);

/* Scratch bytes moe_align uses for T*k slots over E experts (0: none needed; 0 also for invalid
 * arguments, which moe_align itself rejects). */
MOEQ_API size_t moe_align_workspace_size(int T, int k, int E);

/*
 * Per-token, per-128-column-group FP8 quantization of activations ([SGL], "Background": As is
 * the per token-group quantization scale matrix of the activations):
 *   s = max(max|x_group|, 1e-10) / 448 (IEEE f32 division), q = E4M3(x / s) rounded to nearest
 *   even with saturation to +-448.
 *   x bf16 [rows, cols]; q e4m3 [rows, cols] out; s f32 [rows, cols/128] out. cols % 128 == 0.
 */
MOEQ_API int moe_fp8_act_quant(const uint16_t *x, int rows, int cols, uint8_t *q, float *s, void *stream);

/*
 * W4A16 routed expert layer ([CHORD], "vLLM integration": uint4 codes, group 32, BF16 scales,
 * the pack-quantized INT4 group-32 checkpoint shape; "SM90 grouped kernels": codes [G, N, K],
 * scales [G, N, K/32]):
 *   out[t] = sum_j topk_w[t, j] * W2[e_j] . bf16( silu(W13_gate[e_j] . x[t]) * (W13_up[e_j] . x[t]) )
 *   x      bf16 [T, H]
 *   logits f32 [T, E] (routing is computed inside, as moe_route_topk)
 *   w13_q  i32 [E, 2I, H/8]  codes of the fused gate (rows [0, I)) and up (rows [I, 2I))
 *          projections; nibble j of word w holds input column 8w + j in bits [4j, 4j+4); the
 *          value of code q is (q - 8) * scale
 *   w13_s  bf16 [E, 2I, H/32] one scale per 32 consecutive input columns
 *   w2_q   i32 [E, H, I/8], w2_s bf16 [E, H, I/32]  down projection, same format
 *   out    bf16 [T, H] out
 *   topk_ids_out i32 [T, k], topk_w_out f32 [T, k]: optional (may be NULL) copies of the routing
 *   ws     scratch of at least moe_w4a16_workspace_size(T, H, I, E, k) bytes, 256-byte aligned
 * Limits: H % 128 == 0, I % 128 == 0, 1 <= k <= 32, k <= E <= 1024, T >= 0.
 */
MOEQ_API size_t moe_w4a16_workspace_size(int T, int H, int I, int E, int k);
MOEQ_API int moe_w4a16_forward(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                      const int32_t *w13_q, const uint16_t *w13_s, const int32_t *w2_q,
                      const uint16_t *w2_s, uint16_t *out, int32_t *topk_ids_out,
                      float *topk_w_out, void *ws, size_t ws_bytes, void *stream);

/*
 * The same routed layer with MXFP4 weights (lk_moe page, "Supported models & quant formats": MXFP4;
 * its launch example runs a 4-bit-weight, bf16-activation checkpoint on the weight-only MoE
 * runner). A weight is E2M1(q) * 2^(s - 127): q an E2M1 code (1 sign, 2 exponent bits with bias 1,
 * 1 mantissa bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) packed 8 per int32 in the INT4 nibble
 * order above, s the UE8M0 scale byte of its 32-input group. Activations and the intermediate
 * stay bf16 as in moe_w4a16_forward.
 *   moe_mxfp4_prepack_scales: the n UE8M0 bytes -> n bf16 group factors 2^(s - 1), the form the
 *     kernels multiply by (run once per weight tensor; codes s <= 128, i.e. group scales up to 2,
 *     are exact; larger codes give +inf factors). Device memory, asynchronous on the stream.
 *   moe_mxfp4_forward: w13_q i32 [E, 2I, H/8], w13_f bf16 [E, 2I, H/32] (prepacked factors),
 *     w2_q i32 [E, H, I/8], w2_f bf16 [E, H, I/32]; everything else, the workspace
 *     (moe_mxfp4_workspace_size, equal to the W4A16 one), limits and errors as moe_w4a16_forward.
 */
MOEQ_API int moe_mxfp4_prepack_scales(const uint8_t *ue8m0, long long n, uint16_t *factors, void *stream);
MOEQ_API size_t moe_mxfp4_workspace_size(int T, int H, int I, int E, int k);
MOEQ_API int moe_mxfp4_forward(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                               const int32_t *w13_q, const uint16_t *w13_f, const int32_t *w2_q, const uint16_t *w2_f,
                               uint16_t *out, int32_t *topk_ids_out, float *topk_w_out, void *ws, size_t ws_bytes,
                               void *stream);

/*
 * The same routed layer with NVFP4 weights (lk_moe page, "Supported models & quant formats": NVFP4,
 * compressed-tensors / modelopt). A weight is E2M1(q) * E4M3(s) * g: q an E2M1 code (INT4 nibble
 * order), s the E4M3 scale byte of its 16-input group, g one f32 tensor scale per expert and matrix.
 *   moe_nvfp4_prepack_scales: the n E4M3 bytes -> n bf16 factors E4M3(s) * 2^118 (exact for every
 *     E4M3 value; NaN stays NaN), run once per weight tensor.
 *   moe_nvfp4_forward: w13_q i32 [E, 2I, H/8], w13_f bf16 [E, 2I, H/16] (prepacked factors),
 *     w13_g f32 [E] (one tensor scale for the fused gate/up matrix), w2_q i32 [E, H, I/8],
 *     w2_f bf16 [E, H, I/16], w2_g f32 [E]; workspace moe_nvfp4_workspace_size (equal to the W4A16
 *     one); everything else, limits and errors as moe_w4a16_forward (NULL w13_g / w2_g:
 *     INVALID_ARG).
 */
MOEQ_API int moe_nvfp4_prepack_scales(const uint8_t *e4m3, long long n, uint16_t *factors, void *stream);
MOEQ_API size_t moe_nvfp4_workspace_size(int T, int H, int I, int E, int k);
MOEQ_API int moe_nvfp4_forward(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                               const int32_t *w13_q, const uint16_t *w13_f, const float *w13_g, const int32_t *w2_q,
                               const uint16_t *w2_f, const float *w2_g, uint16_t *out, int32_t *topk_ids_out,
                               float *topk_w_out, void *ws, size_t ws_bytes, void *stream);

/*
 * Expert-parallel forms of the layers ([CHORD], "Other deployment details" and the measured
 * results: EP8, EP16 and EP32 deployments, where each GPU holds E / N of the experts). One call
 * computes one rank's share of the layer:
 *   out_r[t] = sum over the slots j of token t whose expert e_j lies in [ep_base, ep_base + ep_local)
 *              of topk_w[t, j] * y_j           (y_j as in the single-GPU layer)
 * so the layer's output is the sum of out_r over ranks whose ranges tile [0, E); the caller sums
 * them (an all-reduce across GPUs). Routing still picks the top k of all E logits. Tokens with no
 * slot on this rank get a zero row.
 *   E          experts the routing picks from (logits are [T, E])
 *   ep_base    first expert this call holds, ep_local how many (ep_local >= 1,
 *              ep_base + ep_local <= E; else INVALID_ARG)
 *   weights    only this rank's experts: w13 [ep_local, ...], w2 [ep_local, ...] (and w13_g / w2_g
 *              [ep_local] for NVFP4), in the formats of the single-GPU entry points
 *   topk_ids_out (nullable) receives the global expert ids
 *   ws         moe_w4a16_ep_workspace_size (the three 4-bit formats) or
 *              moe_w8a8_block_fp8_ep_workspace_size bytes
 * The schedule follows the mean load of one expert, T * k / E, as on a single GPU.
 * Tensor parallelism needs no entry point of its own: a rank that holds the intermediate features
 * [r * I / N, (r + 1) * I / N) of every expert (those gate rows, those up rows, those down columns
 * and their scales; I / N a multiple of 128) calls the single-GPU forward with I / N, and the
 * ranks' outputs sum to the layer's.
 */
MOEQ_API size_t moe_w4a16_ep_workspace_size(int T, int H, int I, int E, int k, int ep_local);
MOEQ_API int moe_w4a16_forward_ep(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                                  int ep_base, int ep_local, const int32_t *w13_q, const uint16_t *w13_s,
                                  const int32_t *w2_q, const uint16_t *w2_s, uint16_t *out, int32_t *topk_ids_out,
                                  float *topk_w_out, void *ws, size_t ws_bytes, void *stream);
MOEQ_API int moe_mxfp4_forward_ep(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                                  int ep_base, int ep_local, const int32_t *w13_q, const uint16_t *w13_f,
                                  const int32_t *w2_q, const uint16_t *w2_f, uint16_t *out, int32_t *topk_ids_out,
                                  float *topk_w_out, void *ws, size_t ws_bytes, void *stream);
MOEQ_API int moe_nvfp4_forward_ep(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                                  int ep_base, int ep_local, const int32_t *w13_q, const uint16_t *w13_f,
                                  const float *w13_g, const int32_t *w2_q, const uint16_t *w2_f, const float *w2_g,
                                  uint16_t *out, int32_t *topk_ids_out, float *topk_w_out, void *ws,
                                  size_t ws_bytes, void *stream);

/*
 * Scratch-free W4A16 layer forward. The pages have no counterpart of this entry point: it exists
 * for callers that cannot allocate device memory where they run the layer, such as a plugin or
 * custom-op host that only hands over its input and output buffers, or a serving runtime that
 * plans all device memory at start-up and forbids allocation afterwards. It computes what
 * moe_w4a16_forward computes, with the same arguments minus ws / ws_bytes; the caller still
 * passes (and owns) the inputs and outputs.
 *  - Its scratch is one static device array of MOEQ_NOALLOC_SCRATCH_BYTES (16 MiB) inside this
 *    library; every GPU that loads the library holds it until the process exits.
 *  - Shapes whose moe_w4a16_workspace_size() exceeds that size are rejected with
 *    MOEQ_ERR_WORKSPACE before anything is enqueued (at H=7168, I=2048, E=384, k=8 the limit is
 *    T <= 103 tokens).
 *  - The call allocates nothing: no cudaMalloc, cudaFree or other allocating routine.
 *  - The first call on each device does a one-time set-up, the lookup of the array's device
 *    address (cudaGetSymbolAddress, with that device current); make that first call before any
 *    stream capture.
 *  - Every call shares the one array, which keeps the last call's contents; nothing in it needs to
 *    start at zero. Calls that can overlap on the GPU (other streams, other host threads) race on
 *    the array: serialize them.
 */
#define MOEQ_NOALLOC_SCRATCH_BYTES (16u << 20)
MOEQ_API int moe_w4a16_forward_noalloc(const uint16_t *x, const float *logits, int T, int H, int I, int E,
                                       int k, const int32_t *w13_q, const uint16_t *w13_s,
                                       const int32_t *w2_q, const uint16_t *w2_s, uint16_t *out,
                                       int32_t *topk_ids_out, float *topk_w_out, void *stream);

/*
 * W8A8 block-FP8 routed expert layer ([SGL], "Background": E4M3 weights with one f32 scale per
 * [128, 128] block, activations E4M3 with one f32 scale per token and 128-column group):
 *   the input is quantized as moe_fp8_act_quant; g, u = block-scaled products with W13[e];
 *   a = silu(g) * u is quantized the same way per slot and 128-column group; y = block-scaled
 *   product with W2[e]; out[t] = sum_j topk_w[t, j] * y_j.
 *   w13 e4m3 [E, 2I, H], w13_s f32 [E, 2I/128, H/128]; w2 e4m3 [E, H, I], w2_s f32 [E, H/128, I/128]
 *   other arguments as moe_w4a16_forward.
 * Limits: H % 128 == 0, I % 128 == 0, 1 <= k <= 32, k <= E <= 1024.
 */
MOEQ_API size_t moe_w8a8_block_fp8_workspace_size(int T, int H, int I, int E, int k);
MOEQ_API int moe_w8a8_block_fp8_forward(const uint16_t *x, const float *logits, int T, int H, int I, int E,
                               int k, const uint8_t *w13, const float *w13_s, const uint8_t *w2,
                               const float *w2_s, uint16_t *out, int32_t *topk_ids_out,
                               float *topk_w_out, void *ws, size_t ws_bytes, void *stream);
/* Expert-parallel form of the block-FP8 layer: as moe_w4a16_forward_ep above, with the weights
 * w13 [ep_local, 2I, H], w13_s [ep_local, 2I/128, H/128], w2 [ep_local, H, I],
 * w2_s [ep_local, H/128, I/128]. */
MOEQ_API size_t moe_w8a8_block_fp8_ep_workspace_size(int T, int H, int I, int E, int k, int ep_local);
MOEQ_API int moe_w8a8_block_fp8_forward_ep(const uint16_t *x, const float *logits, int T, int H, int I, int E,
                                           int k, int ep_base, int ep_local, const uint8_t *w13,
                                           const float *w13_s, const uint8_t *w2, const float *w2_s,
                                           uint16_t *out, int32_t *topk_ids_out, float *topk_w_out, void *ws,
                                           size_t ws_bytes, void *stream);

/*
 * Grouped W4A16 GEMM on the layer's kernels, for callers that route themselves ([CHORD], "SM90
 * grouped kernels": the contiguous prefill layout concatenates each expert's rows, padded to
 * 128-row boundaries, with m_indices holding each row's expert and -1 on padding; the masked
 * decode layout gives every expert a fixed budget of max_m rows, masked_m of them real, and
 * consumers ignore the rest; expected_m is the host-side rows-per-expert hint that picks the
 * launch). For every real row m with expert e:
 *   C[m, n] = bf16( sum_c A[m, c] * (q[e, n, c] - 8) * s[e, n, c / 32] )   (f32 accumulation)
 *   A    bf16 [M, K] (contiguous) or [G * max_m, K] (masked, expert e's rows at e * max_m)
 *   w_q  i32 [G, N, K/8], w_s bf16 [G, N, K/32]: the layer's INT4 group-32 format
 *   m_indices i32 [M] (contiguous): expert of each row in [0, G), -1 = padding (any order works;
 *        the 128-row padding of the pages' layout is not required)
 *   masked_m i32 [G] (masked, device): real rows per expert (values above max_m count as max_m)
 *   C    bf16 [M, N] / [G * max_m, N] out; padding / masked-out rows are not written
 *   ws, ws_bytes: device scratch (256-byte aligned) of the matching *_workspace_size() bytes
 * Limits: K % 128 == 0, N % 128 == 0 (both >= 128), 1 <= G <= 1024, rows <= 2^24. Schedule as the
 * layer's down GEMM: at >= 16 rows per expert (M / G, or expected_m) tcgen05 over 256-row blocks
 * with blocks of <= 8 rows on the register-fed kernel, below that the register-fed kernel.
 */
MOEQ_API size_t moe_w4a16_grouped_contiguous_workspace_size(int M, int K, int N, int G);
MOEQ_API int moe_w4a16_grouped_contiguous(const uint16_t *A, int M, int K, const int32_t *w_q, const uint16_t *w_s,
                                          int G, int N, const int32_t *m_indices, uint16_t *C, void *ws,
                                          size_t ws_bytes, void *stream);
MOEQ_API size_t moe_w4a16_grouped_masked_workspace_size(int G, int max_m, int K, int N, int expected_m);
MOEQ_API int moe_w4a16_grouped_masked(const uint16_t *A, int G, int max_m, int K, const int32_t *w_q,
                                      const uint16_t *w_s, int N, const int32_t *masked_m, int expected_m, uint16_t *C,
                                      void *ws, size_t ws_bytes, void *stream);

/*
 * Dense block-FP8 matmul ([SGL], "Background": w8a8_block_fp8_matmul(A, B, As, Bs, block_size,
 * output_dtype)):  C[m, n] = sum_kb As[m, kb] * Bs[n/128, kb] * sum_{k in block kb} A[m,k] B[n,k]
 *   A e4m3 [M, K], As f32 [M, K/128], B e4m3 [N, K], Bs f32 [ceil(N/128), ceil(K/128)],
 *   C bf16 [M, N] out. block_n and block_k must both be 128 ([SGL], "Config directory & naming":
 *   almost every entry uses block_shape [128, 128]); K % 128 == 0, N % 128 == 0
 *   (the page's shape check: ceil(N/block_n) == rows of Bs, ceil(K/block_k) == columns of Bs);
 *   A, B and C 16-byte aligned (else UNSUPPORTED).
 */
MOEQ_API int w8a8_block_fp8_matmul(const uint8_t *A, const float *As, const uint8_t *B, const float *Bs,
                          int M, int N, int K, int block_n, int block_k, uint16_t *C, void *stream);

/*
 * Dense channelwise FP8 matmul ([SGL], "JSON format": the channelwise variant is the W8A8 FP8 GEMM
 * with per-token activation scales and per-channel weight scales):
 *   C[m, n] = bf16( As[m] * Bs[n] * sum_k A[m, k] * B[n, k] )   (f32 accumulation over all of K)
 *   A e4m3 [M, K], As f32 [M], B e4m3 [N, K], Bs f32 [N], C bf16 [M, N] out; all device memory,
 *   row-major, caller-owned; nothing allocated.
 * Limits: K % 128 == 0, N % 128 == 0 (both >= 128), M >= 0 (0 is a no-op). Errors: INVALID_ARG for
 * null pointers or negative sizes, UNSUPPORTED for other shapes or when A, B or C is not 16-byte
 * aligned, CUDA_LAUNCH for a failed launch.
 */
MOEQ_API int w8a8_channel_fp8_matmul(const uint8_t *A, const float *As, const uint8_t *B, const float *Bs, int M, int N,
                                     int K, uint16_t *C, void *stream);

/*
 * Stage tracing, a diagnostic that is off by default. While enabled, every forward / matmul call
 * brackets each of its kernel stages with a pair of CUDA events recorded on the call's stream
 * (the library creates the events on first use, on the current device; do not enable tracing
 * during stream capture). moe_trace_read() waits for the recorded events, adds their durations
 * to per-stage totals and writes the first min(n_stages, 9) totals (milliseconds) and call
 * counts (either pointer may be NULL); it returns 9, the number of stages, or MOEQ_ERR_CUDA.
 * `reset` != 0 clears the totals after reading. Stage indices: 0 route_topk, 1 align,
 * 2 fp8_act_quant, 3 gate_up (with SiLU*up), 4 down (with the routing weight), 5 combine,
 * 6 dense block-FP8 matmul, 7 gather (routed activation rows copied into aligned order for the
 * tensor-core GEMMs), 8 few_rows (gate/up and down of the expert blocks with at most 8 routed
 * rows on the 4-bit layers' tensor-core schedule, run by the register-fed kernel).
 */
MOEQ_API int moe_trace_enable(int enable);
MOEQ_API int moe_trace_read(double *stage_ms, long long *stage_calls, int n_stages, int reset);

/*
 * Host-side cost of the entry points ("vLLM x Novita AI: Chord W4A16 INT4 MoE Kernel for Kimi
 * K2.x", section "SM90 grouped kernels": per-launch host lookup, memoized there). Every layer
 * forward, grouped GEMM and dense matmul adds its host wall time (validation, workspace carving,
 * schedule choice, tensor maps, kernel launches; not the device time) to a process-wide total.
 * The tensor maps the tensor-core kernels need are memoized on their parameters (address, type,
 * extents, box, swizzle; a ring of 64), so a repeated call on the same buffers encodes none.
 * Writes (each pointer may be NULL): the summed host time in microseconds, the number of calls,
 * tensor maps encoded through the driver and reused from the memo since load. `reset` != 0 clears
 * the time and call totals. Returns MOEQ_OK.
 */
MOEQ_API int moe_host_stats(double *host_us, long long *calls, long long *tmap_encoded, long long *tmap_reused,
                            int reset);

/*
 * Sticky device status of the library's kernels on the current device: 0 if no kernel has
 * reported a problem, else MOEQ_ERR_DEVICE_TIMEOUT. This call synchronizes with the device (it
 * is a diagnostic, not part of the forward path); `clear` != 0 resets the status.
 */
MOEQ_API int moe_device_status(int clear);

/*
 * Failure-detection self-test (diagnostic; the pages have no counterpart). Every wait inside the
 * tensor-core kernels is bounded: a wait that gives up sets the device status word and its CTA
 * drains and exits, so a stuck pipeline surfaces as MOEQ_ERR_DEVICE_TIMEOUT from
 * moe_device_status() instead of a hung GPU. This call enqueues a one-CTA kernel that runs the
 * same bounded wait on a barrier nothing ever arrives at, with a short poll limit; afterwards
 * moe_device_status() reports MOEQ_ERR_DEVICE_TIMEOUT (clear it with moe_device_status(1)).
 * No fault, trap or hang is involved; the context stays usable.
 */
MOEQ_API int moe_selftest_bounded_wait(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MOEQ_H */
