// Kernel launchers of the moeq library (internal; the public surface is include/moeq.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moeq {

enum { MODE_GATEUP = 0, MODE_DOWN = 1 };

// 4-bit weight formats: INT4 codes with zero point 8 times bf16 group-32 scales; E2M1 codes times
// bf16 group-32 factors 2^(s - 1) (MXFP4 after moe_mxfp4_prepack_scales); E2M1 codes times bf16
// group-16 factors E4M3(s) * 2^118 (NVFP4 after moe_nvfp4_prepack_scales), the accumulators then
// scaled by the expert's f32 tensor scale * 2^8 (wglobal)
enum { W4_INT4 = 0, W4_FP4 = 1, W4_NV = 2 };

struct W4GroupedArgs {
    int fmt;                 // W4_INT4 / W4_FP4 / W4_NV
    const float *wglobal;    // W4_NV: f32 tensor scale per expert [E]
    const uint16_t *act;     // gate/up: x [T, K]; down: h [T*k, K] (INT4: f16 values unless act_bf16)
    int act_row_div;         // activation row of a slot = slot / act_row_div (k for x, 1 for h)
    const int32_t *wq;       // [E, n_rows, K/8]
    const uint16_t *ws;      // [E, n_rows, K/32] bf16
    int K;
    int n_out;               // gate/up: I (weights hold 2I rows); down: H
    int n_rows;              // weight rows per expert
    int E;
    const int32_t *sorted_ids;
    const int32_t *expert_ids;
    const int32_t *num_tokens_padded;
    int n_slots;             // T*k; sorted_ids entries >= n_slots are padding
    const float *topk_w;     // [T*k] (down); null: weight 1 (plain grouped GEMM)
    uint16_t *h_out;         // [T*k, I] bf16(a) values (gate/up; f16 bits for INT4)
    uint16_t *y_out;         // [T*k, H] bf16, routing weight applied (down)
    // 0: align blocks of BM rows. Otherwise the alignment has blocks of blk_stride rows and the
    // kernel takes only those with at most BM real rows (the rest belong to the tensor-core path)
    int blk_stride;
    // down, blk_stride 0: the kernel directly before this one is the gate/up kernel of the same
    // alignment (which waits for the alignment before it lets this kernel start), so the routing
    // buffers may be read, and the weights prefetched, before waiting for h
    int after_gateup;
    // INT4: 1 = act holds bf16 values, converted to f16 in registers; 0 = act is already f16 (the
    // INT4 GEMMs compute in f16, where the dequantized weights are exact)
    int act_bf16;
};

struct F8GroupedArgs {
    const uint8_t *act;      // gate/up: xq [T, K]; down: hq [T*k, K]; dense: A [M, K]
    const float *act_s;      // [rows, K/128]
    int act_row_div;
    const uint8_t *w;        // [E, n_rows, K]
    const float *w_s;        // [E, n_rows/128, K/128]
    int K;
    int n_out;
    int n_rows;
    int E;
    const int32_t *sorted_ids;
    const int32_t *expert_ids;
    const int32_t *num_tokens_padded;
    int n_slots;             // T*k
    const float *topk_w;
    uint8_t *hq_out;         // [T*k, I]
    float *hs_out;           // [T*k, I/128]
    uint16_t *y_out;         // [T*k, H] bf16, routing weight applied (down)
};

// TC_DENSE_CW: dense channelwise FP8 (a_scale [M] per token, b_scale [N] per channel): the whole
// K accumulates in one tensor-memory buffer and the scales are applied once, in the epilogue.
enum { TC_DENSE = 0, TC_GATEUP = 1, TC_DOWN = 2, TC_DENSE_CW = 3 };

struct Fp8TcArgs {
    const float *a_scale;   // [M, K/128]: As (dense) or the gathered / intermediate row scales
    const float *b_scale;   // dense: Bs [N/128, K/128]; grouped: weight scales [E, rows/128, K/128]
    int M, N, K;            // A rows; output columns (dense N, gate/up I, down H); inputs
    int *status;            // kernel status word (bounded waits that gave up)
    uint16_t *C;            // dense: [M, N] bf16
    // grouped
    int E;
    int rows_per_expert;    // weight rows per expert (2I or H)
    const int32_t *sorted_ids;
    const int32_t *expert_ids;
    const int32_t *ntp;
    int n_slots;
    const float *topk_w;
    uint8_t *hq;            // gate/up out: [M, N] E4M3
    float *hs;              // gate/up out: [M, N/128]
    uint16_t *ys;           // down out: [n_slots, N] bf16, routing weight applied
    int tiles_per_cta;      // grouped down: output tiles per CTA (set by the launcher)
};

struct W4TcArgs {
    int fmt;                // W4_INT4 / W4_FP4 / W4_NV
    const float *wglobal;   // W4_NV: f32 tensor scale per expert [E]
    int M, N, K;            // activation rows (aligned capacity); output features / rows; inputs
    int *status;
    int E;
    int rows_per_expert;    // 2I (gate/up) or H (down)
    const int32_t *wq;      // [E * rows_per_expert, K/8]
    const uint16_t *ws;     // [E * rows_per_expert, K/32] bf16
    const int32_t *sorted_ids;
    const int32_t *expert_ids;
    const int32_t *ntp;
    int n_slots;
    const float *topk_w;
    uint16_t *h_out;        // gate/up: [M, N], bf16 values (stored as f16 for the INT4 format)
    uint16_t *ys;           // down: [n_slots, N] bf16, routing weight applied
    int small_rows;         // blocks with at most this many real rows are left to the register-fed path
    int tiles_per_cta;      // down: output tiles of 128 rows per CTA (set by the launcher)
};

// local_ids (nullable): the picks relative to the expert range [ep_base, ep_base + ep_local), -1
// outside it; ids may be null when local_ids is given.
// xh (nullable): also copies x [T, H] (bf16) into xh [T, H], each 8-input group in nibble-pair
// order, converted to f16 when xh_f16.
void launch_route_topk(const float *logits, int T, int E, int k, int32_t *ids, float *w, cudaStream_t s,
                       int32_t *local_ids = nullptr, int ep_base = 0, int ep_local = 0, const uint16_t *x = nullptr,
                       int H = 0, uint16_t *xh = nullptr, bool xh_f16 = true);
// Scratch (bytes) the alignment of n slots over E experts uses; 0 = the one-CTA kernel, which
// also runs when launch_align gets no scratch.
size_t align_scratch_bytes(int n, int E);
void launch_masked_rows(const int32_t *masked_m, int G, int max_m, int32_t *ids, int num_sms, cudaStream_t s);
void launch_align(const int32_t *topk_ids, int n, int E, int B, int32_t *sorted_ids, int32_t *expert_ids,
                  int32_t *ntp, int32_t *scratch, cudaStream_t s);
// local_ids (nullable): slots with a negative id are left out of the sum.
void launch_combine(const uint16_t *ys, int T, int k, int H, uint16_t *out, int num_sms, cudaStream_t s,
                    const int32_t *local_ids = nullptr);
// UE8M0 group scales s -> the bf16 factors 2^(s - 1) the FP4 dequantization multiplies by (s > 128
// overflows to +inf: group scales above 2 are outside the supported range)
void launch_mxfp4_scale_factors(const uint8_t *s, long long n, uint16_t *f, int num_sms, cudaStream_t st);
// E4M3 group scales -> the bf16 factors E4M3(s) * 2^118 (exact: 4 significant bits, range 2^109 ..
// 1.75 * 2^126) the NVFP4 dequantization multiplies by; E4M3 NaN stays NaN
void launch_nvfp4_scale_factors(const uint8_t *s, long long n, uint16_t *f, int num_sms, cudaStream_t st);
void launch_fp8_act_quant(const uint16_t *x, int rows, int cols, uint8_t *q, float *s, cudaStream_t st);
void launch_w4a16_grouped_mma(const W4GroupedArgs &a, int mode, int block_m, int max_blocks, cudaStream_t s);
void launch_fp8_grouped_mma(const F8GroupedArgs &a, int mode, int block_m, int max_blocks, cudaStream_t s);
// tcgen05 block-FP8 GEMM: A [M, K] and B [N, K] E4M3, K % 128 == 0, N % 128 == 0. Returns a status.
int launch_fp8_tc_gemm(const Fp8TcArgs &a, const uint8_t *A, const uint8_t *B, cudaStream_t s);
// Dense channelwise FP8 GEMM (a_scale [M], b_scale [N]) for M > fp8_skinny_max_rows(true).
int launch_fp8_tc_channel(const Fp8TcArgs &a, const uint8_t *A, const uint8_t *B, cudaStream_t s);
// Dense FP8 GEMM for M <= fp8_skinny_max_rows(channelwise) rows (swap-AB tcgen05 tiles of 128
// weight rows, K split over a cluster of `split` CTAs reduced through distributed shared memory).
int fp8_skinny_max_rows(bool channelwise);
// channelwise: a_scale [M] per token and b_scale [N] per channel, the whole K accumulated in one
// tensor-memory buffer.
int launch_fp8_tc_skinny(const Fp8TcArgs &a, const uint8_t *A, const uint8_t *B, int split, bool channelwise,
                         cudaStream_t s);
// tcgen05 grouped block-FP8 GEMM over expert-contiguous rows A [M, K] (128-row blocks, one expert
// each, per expert_ids / ntp) and weights W [E * rows_per_expert, K]; mode TC_GATEUP or TC_DOWN.
int launch_fp8_tc_grouped(const Fp8TcArgs &a, int mode, const uint8_t *A, const uint8_t *W, int E, int max_blocks,
                          cudaStream_t s);
// tcgen05 W4A16 grouped GEMM over aligned bf16 activation rows act [M, K]; mode TC_GATEUP (h =
// silu(gate) * up in aligned order) or TC_DOWN (weighted slot rows).
int launch_w4a16_tc(const W4TcArgs &a, int mode, const uint16_t *act, int max_blocks, cudaStream_t s);
// Copies the routed rows of x into aligned order (row r takes x[sorted_ids[r] / k]); only the rows
// the tensor-core MMAs read (see the kernel). to_f16: the copies are converted to f16 (the INT4
// tensor-core GEMMs compute in f16).
void launch_gather_bf16(const uint16_t *x, int H, int k, const int32_t *sorted_ids, const int32_t *ntp, int n_slots,
                        int cap_rows, int small_rows, uint16_t *xg, int num_sms, cudaStream_t s, bool to_f16);
// Copies E4M3 rows (and their scales) of the routed slots into aligned order: row r takes token
// sorted_ids[r] / k; padding rows become zero.
void launch_gather_fp8_rows(const uint8_t *xq, const float *xs, int H, int k, const int32_t *sorted_ids,
                            const int32_t *ntp, int n_slots, int cap_rows, uint8_t *xg, float *xsg, int num_sms,
                            cudaStream_t s);

}  // namespace moeq
