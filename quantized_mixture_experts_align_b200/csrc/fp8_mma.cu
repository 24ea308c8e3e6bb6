// W8A8 block-FP8: per-token group-128 activation quantizer and block-scaled GEMMs with the
// weights in the MMA M dimension (e4m3 m16n8k32 tensor-core MMA, f32 accumulate).
//
// "SGLang W8A8 Block FP8 quantized kernel config files", section "Background": E4M3 values
// (max 448), one f32 scale per [128, 128] weight block, one per token and 128-column group of
// the activations; C = sum over 128-wide K blocks of As * Bs * (A_q . B_q). Each K block is
// accumulated by its own MMAs and promoted into the f32 accumulator with its two scales, so the
// scale is stepped exactly once per 128 inputs (the constraint that page's config lookup
// enforces on BLOCK_SIZE_K).
#include "common.cuh"
#include "kernels.cuh"

namespace moeq {

// ------------------------------------------------------------------------------------------
// Activation quantizer: one warp per (row, 128-column group); lane holds 4 columns.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) fp8_act_quant_kernel(const uint16_t *__restrict__ x, int rows, int cols,
                                                            uint8_t *__restrict__ q, float *__restrict__ s)
{
    const int G = cols / 128;
    const long item = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (item >= (long)rows * G) return;
    const int lane = threadIdx.x & 31;
    const long r = item / G;
    const int grp = (int)(item - r * G);
    const size_t base = (size_t)r * cols + grp * 128 + lane * 4;
    const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(x + base));
    float v[4] = {bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y)};
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    const float sc = __fdiv_rn(fmaxf(amax, 1e-10f), 448.0f);
    const uint32_t lo = pack_e4m3x2(__fdiv_rn(v[0], sc), __fdiv_rn(v[1], sc));
    const uint32_t hi = pack_e4m3x2(__fdiv_rn(v[2], sc), __fdiv_rn(v[3], sc));
    *reinterpret_cast<uint32_t *>(q + base) = lo | (hi << 16);
    if (lane == 0) s[(size_t)r * G + grp] = sc;
}

void launch_fp8_act_quant(const uint16_t *x, int rows, int cols, uint8_t *q, float *s, cudaStream_t st)
{
    const long items = (long)rows * (cols / 128);
    if (items <= 0) return;
    fp8_act_quant_kernel<<<(unsigned)((items + 7) / 8), 256, 0, st>>>(x, rows, cols, q, s);
}

// ------------------------------------------------------------------------------------------
// Gather of quantized rows into aligned (expert-contiguous) order: one warp per row, 16-byte
// copies; padding rows (pad slot, or past the padded count) are written as zeros.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gather_fp8_rows_kernel(const uint8_t *__restrict__ xq,
                                                              const float *__restrict__ xs, int H, int k,
                                                              const int32_t *__restrict__ sorted_ids,
                                                              const int32_t *__restrict__ ntp, int n_slots,
                                                              int cap_rows, uint8_t *__restrict__ xg,
                                                              float *__restrict__ xsg)
{
    const int lane = threadIdx.x & 31;
    const int rows = min(__ldg(ntp), cap_rows);
    const int G = H / 128;
    for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += gridDim.x * (blockDim.x >> 5)) {
        const int slot = __ldg(sorted_ids + r);
        const bool real = slot < n_slots;
        const uint4 *src = reinterpret_cast<const uint4 *>(xq + (size_t)(real ? slot / k : 0) * H);
        uint4 *dst = reinterpret_cast<uint4 *>(xg + (size_t)r * H);
        for (int i = lane; i < H / 16; i += 32) dst[i] = real ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
        for (int i = lane; i < G; i += 32) xsg[(size_t)r * G + i] = real ? __ldg(xs + (size_t)(slot / k) * G + i) : 0.f;
    }
}

void launch_gather_fp8_rows(const uint8_t *xq, const float *xs, int H, int k, const int32_t *sorted_ids,
                            const int32_t *ntp, int n_slots, int cap_rows, uint8_t *xg, float *xsg, int num_sms,
                            cudaStream_t s)
{
    if (cap_rows <= 0) return;
    const int blocks = min(cdiv(cap_rows, 8), num_sms * 8);
    gather_fp8_rows_kernel<<<blocks, 256, 0, s>>>(xq, xs, H, k, sorted_ids, ntp, n_slots, cap_rows, xg, xsg);
}

// ------------------------------------------------------------------------------------------
// Block-scaled FP8 GEMM, weights as MMA A (16 rows per tile), tokens as MMA B (8 per sub-tile).
// Lane t of a quad reads 16 contiguous bytes per 64 inputs; its 4 words feed two k-steps as the
// A (and, for the token column, B) fragments directly - both operands use the same permutation
// of K inside each 64-wide chunk, which stays inside one 128-wide scale block.
//
// MODE_GATEUP: rows [f0, f0+16) gate and [I+f0, ...) up; WARPS = 8 so a CTA covers the 128
//              features of one intermediate quantization group; epilogue quantizes silu(g)*u
//              per slot and 128-group to E4M3 + f32 scale.
// MODE_DOWN:   rows [r0, r0+32); epilogue writes ys[slot, r] = topk_w[slot] * y (bf16).
// ------------------------------------------------------------------------------------------
template <int BM, int WARPS, int MODE>
__global__ void __launch_bounds__(WARPS * 32) fp8_grouped_mma_kernel(F8GroupedArgs a)
{
    constexpr int MS = BM / 8;
    __shared__ float red[WARPS][BM];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int blk = blockIdx.x;
    if (blk * BM >= __ldg(a.num_tokens_padded)) return;
    const int e = __ldg(a.expert_ids + blk);
    if (e < 0 || e >= a.E) return;
    const int tile = blockIdx.y * WARPS + warp;
    int rowA, rowB;
    bool active;
    if (MODE == MODE_GATEUP) {
        rowA = tile * 16;
        rowB = a.n_out + rowA;
        active = rowA < a.n_out;  // n_out % 128 == 0: whole CTA active or not
    } else {
        rowA = tile * 32;
        rowB = rowA + 16;
        active = rowA < a.n_out;
    }
    if (MODE != MODE_GATEUP && !active) return;

    const int K = a.K, KB = K / 128;
    // B-operand rows (column g of each sub-tile) and the scale rows of this lane's accumulator
    // columns (2t, 2t+1); padding columns read nothing and get scale 0
    const uint8_t *act_row[MS];
    const float *col_scale[MS][2];
#pragma unroll
    for (int s = 0; s < MS; ++s) {
        act_row[s] = nullptr;
#pragma unroll
        for (int c = -1; c < 2; ++c) {
            const int j = blk * BM + 8 * s + (c < 0 ? g : 2 * t + c);
            const int slot = __ldg(a.sorted_ids + j);
            const bool ok = slot < a.n_slots;
            const size_t arow = ok ? (size_t)(slot / a.act_row_div) : 0;
            if (c < 0) act_row[s] = ok ? a.act + arow * K : nullptr;
            else col_scale[s][c] = ok ? a.act_s + arow * KB : nullptr;
        }
    }

    const uint8_t *w = a.w + (size_t)e * a.n_rows * K;
    const float *wsc = a.w_s + (size_t)e * (a.n_rows / 128) * KB;
    const uint8_t *wr[4] = {w + (size_t)(rowA + g) * K, w + (size_t)(rowA + g + 8) * K,
                            w + (size_t)(rowB + g) * K, w + (size_t)(rowB + g + 8) * K};
    const float *srA = wsc + (size_t)(rowA / 128) * KB;
    const float *srB = wsc + (size_t)(rowB / 128) * KB;

    float accA[MS][4], accB[MS][4];
#pragma unroll
    for (int s = 0; s < MS; ++s)
#pragma unroll
        for (int i = 0; i < 4; ++i) { accA[s][i] = 0.f; accB[s][i] = 0.f; }

    if (active) {
        for (int kb = 0; kb < KB; ++kb) {
            uint4 wv[2][4];
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int r = 0; r < 4; ++r) wv[c][r] = ld_stream_v4(wr[r] + kb * 128 + c * 64 + 16 * t);
            const float sA = __ldg(srA + kb), sB = __ldg(srB + kb);
#pragma unroll
            for (int s = 0; s < MS; ++s) {
                float tA[4] = {0.f, 0.f, 0.f, 0.f}, tB[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint4 xv = make_uint4(0u, 0u, 0u, 0u);
                    if (act_row[s]) xv = ld_v4(act_row[s] + kb * 128 + c * 64 + 16 * t);
                    // k-step 2c: words x,y; k-step 2c+1: words z,w
                    mma_e4m3_16832(tA, wv[c][0].x, wv[c][1].x, wv[c][0].y, wv[c][1].y, xv.x, xv.y);
                    mma_e4m3_16832(tB, wv[c][2].x, wv[c][3].x, wv[c][2].y, wv[c][3].y, xv.x, xv.y);
                    mma_e4m3_16832(tA, wv[c][0].z, wv[c][1].z, wv[c][0].w, wv[c][1].w, xv.z, xv.w);
                    mma_e4m3_16832(tB, wv[c][2].z, wv[c][3].z, wv[c][2].w, wv[c][3].w, xv.z, xv.w);
                }
                // promote: columns 2t, 2t+1 carry their token's activation scale
                const float xs[2] = {col_scale[s][0] ? __ldg(col_scale[s][0] + kb) : 0.f,
                                     col_scale[s][1] ? __ldg(col_scale[s][1] + kb) : 0.f};
                accA[s][0] += tA[0] * (sA * xs[0]);
                accA[s][1] += tA[1] * (sA * xs[1]);
                accA[s][2] += tA[2] * (sA * xs[0]);
                accA[s][3] += tA[3] * (sA * xs[1]);
                accB[s][0] += tB[0] * (sB * xs[0]);
                accB[s][1] += tB[1] * (sB * xs[1]);
                accB[s][2] += tB[2] * (sB * xs[0]);
                accB[s][3] += tB[3] * (sB * xs[1]);
            }
        }
    }

    if (MODE == MODE_GATEUP) {
        // a = silu(g) * u for features (rowA + g, rowA + g + 8) x columns (2t, 2t+1)
        float av[MS][4];
        float cmax[MS][2];
#pragma unroll
        for (int s = 0; s < MS; ++s) {
#pragma unroll
            for (int i = 0; i < 4; ++i) av[s][i] = silu_f32(accA[s][i]) * accB[s][i];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                float m = fmaxf(fabsf(av[s][c]), fabsf(av[s][2 + c]));
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 8));
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 16));
                cmax[s][c] = m;
            }
            if (g == 0) {
                red[warp][8 * s + 2 * t] = cmax[s][0];
                red[warp][8 * s + 2 * t + 1] = cmax[s][1];
            }
        }
        __syncthreads();
        if (!active) return;
        const int grp = rowA / 128;
#pragma unroll
        for (int s = 0; s < MS; ++s) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int col = 8 * s + 2 * t + c;
                const int slot = __ldg(a.sorted_ids + blk * BM + col);
                if (slot >= a.n_slots) continue;
                float amax = 0.f;
#pragma unroll
                for (int ww = 0; ww < WARPS; ++ww) amax = fmaxf(amax, red[ww][col]);
                const float sc = __fdiv_rn(fmaxf(amax, 1e-10f), 448.0f);
                const uint16_t q2 = pack_e4m3x2(__fdiv_rn(av[s][c], sc), __fdiv_rn(av[s][2 + c], sc));
                uint8_t *hq = a.hq_out + (size_t)slot * a.n_out;
                hq[rowA + g] = (uint8_t)(q2 & 0xFF);
                hq[rowA + g + 8] = (uint8_t)(q2 >> 8);
                if (warp == 0 && g == 0) a.hs_out[(size_t)slot * (a.n_out / 128) + grp] = sc;
            }
        }
    } else {
#pragma unroll
        for (int s = 0; s < MS; ++s) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int j = blk * BM + 8 * s + 2 * t + c;
                const int slot = __ldg(a.sorted_ids + j);
                if (slot >= a.n_slots) continue;
                const float wt = __ldg(a.topk_w + slot);
                uint16_t *y = a.y_out + (size_t)slot * a.n_out;
                y[rowA + g] = f32_to_bf16(wt * accA[s][c]);
                y[rowA + g + 8] = f32_to_bf16(wt * accA[s][2 + c]);
                y[rowB + g] = f32_to_bf16(wt * accB[s][c]);
                y[rowB + g + 8] = f32_to_bf16(wt * accB[s][2 + c]);
            }
        }
    }
}

template <int BM, int MODE>
static void launch_f8(const F8GroupedArgs &a, int max_blocks, cudaStream_t s)
{
    constexpr int WARPS = (MODE == MODE_GATEUP) ? 8 : 4;
    const int rows_per_cta = (MODE == MODE_GATEUP ? 16 : 32) * WARPS;
    dim3 grid(max_blocks, cdiv(a.n_out, rows_per_cta));
    fp8_grouped_mma_kernel<BM, WARPS, MODE><<<grid, WARPS * 32, 0, s>>>(a);
}

void launch_fp8_grouped_mma(const F8GroupedArgs &a, int mode, int block_m, int max_blocks, cudaStream_t s)
{
    if (max_blocks <= 0) return;
#define MOEQ_F8_CASE(BMV)                                                          \
    case BMV:                                                                      \
        if (mode == MODE_GATEUP) launch_f8<BMV, MODE_GATEUP>(a, max_blocks, s);    \
        else launch_f8<BMV, MODE_DOWN>(a, max_blocks, s);                          \
        break;
    switch (block_m) {
        MOEQ_F8_CASE(8)
        MOEQ_F8_CASE(16)
        MOEQ_F8_CASE(32)
        MOEQ_F8_CASE(64)
        default: break;
    }
#undef MOEQ_F8_CASE
}

}  // namespace moeq
