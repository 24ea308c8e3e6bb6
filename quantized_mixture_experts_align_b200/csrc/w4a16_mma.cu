// W4A16 grouped GEMMs over the aligned routing, weights in the MMA M dimension ("swap-AB").
//
// "vLLM x Novita AI: Chord W4A16 INT4 MoE Kernel for Kimi K2.x", section "H200 and Blackwell
// indexed decode": at a few routed rows per expert the dequantized weights take the MMA-M
// operand and the tokens the narrow N side (block-M 8); dequantization subtracts the zero point
// and then scales, fused into the nibble extraction, which keeps the unfused BF16 rounding order.
//
// Work split: one CTA per (align block of BM slots = grid x, tile of output features = grid y);
// consecutive CTAs take consecutive blocks, so the blocks of one expert share its weights in L2.
// Each warp owns 16 (gate/up) or 32 (down) output rows for the whole K range and streams its
// packed weights straight from HBM into registers (16 B per lane per 128 inputs, no shared-memory round trip:
// the decode shapes are HBM-bound and every weight byte is used by exactly one warp). A
// dequantized 32-bit word feeds two m16n8k16 k-steps directly as A fragments.
//
// Input permutation. The sum over K does not care about order, so inside a 128-input
// "quad-group" lane t (of a 4-lane quad) takes the 32 inputs of group t = 16 contiguous bytes of
// the row, which keeps each element with its own group scale. Word m of that group feeds
// k-steps 2m and 2m+1; its nibble pairs (0,4), (1,5), (2,6), (3,7) are extracted with one shift
// and one LOP3 each (magic 0x4300 = bf16 128.0, nibble in the low mantissa bits), so the
// activation fragments take the same pairs, rebuilt with PRMT from a 16-byte load.
#include "common.cuh"
#include "kernels.cuh"

namespace moeq {

namespace {

struct DeqWord {
    uint32_t p[4];  // bf16x2 pairs: (n0,n4) (n1,n5) (n2,n6) (n3,n7), already (q-8)*scale
};

__device__ __forceinline__ DeqWord dequant_word(uint32_t w, uint32_t scale2)
{
    const uint32_t magic = 0x43004300u;  // bf16 128.0 in both halves
    const uint32_t bias = 0x43084308u;   // bf16 136.0 = 128 + 8 (zero point) in both halves
    DeqWord d;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t v = lop3_and_or(w >> (4 * i), 0x000F000Fu, magic);  // 128 + q, exact
        d.p[i] = bf16x2_mul(bf16x2_sub(v, bias), scale2);                 // (q - 8) exact, then * s
    }
    return d;
}

// activation pairs matching DeqWord's nibble pairing, from 8 consecutive bf16 (x0..x7)
__device__ __forceinline__ void act_pairs(const uint4 &v, uint32_t (&b)[4])
{
    b[0] = prmt(v.x, v.z, 0x5410u);  // (x0, x4)
    b[1] = prmt(v.x, v.z, 0x7632u);  // (x1, x5)
    b[2] = prmt(v.y, v.w, 0x5410u);  // (x2, x6)
    b[3] = prmt(v.y, v.w, 0x7632u);  // (x3, x7)
}

}  // namespace

// MODE_GATEUP: rows [f0, f0+16) (gate) and [I + f0, I + f0 + 16) (up) of W13; epilogue writes
//              h[slot, f] = bf16(silu(gate) * up).
// MODE_DOWN:   rows [r0, r0+32) of W2; epilogue writes ys[slot, r] = topk_w[slot] * y (f32).
template <int BM, int WARPS, int MODE>
__global__ void __launch_bounds__(WARPS * 32) w4a16_grouped_mma_kernel(W4GroupedArgs a)
{
    constexpr int MS = BM / 8;  // token sub-tiles of 8 columns
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int blk = blockIdx.x;
    if (blk * BM >= __ldg(a.num_tokens_padded)) return;
    const int e = __ldg(a.expert_ids + blk);
    if (e < 0 || e >= a.E) return;

    const int tile = blockIdx.y * WARPS + warp;
    int rowA, rowB;
    if (MODE == MODE_GATEUP) {
        rowA = tile * 16;
        if (rowA >= a.n_out) return;
        rowB = a.n_out + rowA;
    } else {
        rowA = tile * 32;
        if (rowA >= a.n_out) return;
        rowB = rowA + 16;
    }

    // token columns this lane feeds as MMA B (column g of each sub-tile)
    const int K = a.K;
    const int KW = K / 8;    // int32 words per weight row
    const int KG = K / 32;   // scale groups per weight row
    const uint16_t *act_row[MS];
#pragma unroll
    for (int s = 0; s < MS; ++s) {
        const int slot = __ldg(a.sorted_ids + blk * BM + 8 * s + g);
        act_row[s] = (slot < a.n_slots) ? a.act + (size_t)(slot / a.act_row_div) * K : nullptr;
    }

    const int32_t *wq = a.wq + (size_t)e * a.n_rows * KW;
    const uint16_t *wsc = a.ws + (size_t)e * a.n_rows * KG;
    const int32_t *wr[4] = {wq + (size_t)(rowA + g) * KW, wq + (size_t)(rowA + g + 8) * KW,
                            wq + (size_t)(rowB + g) * KW, wq + (size_t)(rowB + g + 8) * KW};
    const uint16_t *sr[4] = {wsc + (size_t)(rowA + g) * KG, wsc + (size_t)(rowA + g + 8) * KG,
                             wsc + (size_t)(rowB + g) * KG, wsc + (size_t)(rowB + g + 8) * KG};

    float accA[MS][4], accB[MS][4];
#pragma unroll
    for (int s = 0; s < MS; ++s)
#pragma unroll
        for (int i = 0; i < 4; ++i) { accA[s][i] = 0.f; accB[s][i] = 0.f; }

    const int NQ = K / 128;
    uint4 wcur[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) wcur[r] = ld_stream_v4(wr[r] + 4 * t);

    for (int q = 0; q < NQ; ++q) {
        // prefetch the next quad-group's words while this one is consumed
        uint4 wnext[4];
        const int qn = (q + 1 < NQ) ? q + 1 : q;
#pragma unroll
        for (int r = 0; r < 4; ++r) wnext[r] = ld_stream_v4(wr[r] + 16 * qn + 4 * t);
        uint32_t sc[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const uint32_t s16 = __ldg(sr[r] + 4 * q + t);
            sc[r] = s16 | (s16 << 16);
        }
        const int kofs = 128 * q + 32 * t;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const uint32_t words[4] = {(&wcur[0].x)[m], (&wcur[1].x)[m], (&wcur[2].x)[m], (&wcur[3].x)[m]};
            DeqWord d[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) d[r] = dequant_word(words[r], sc[r]);
#pragma unroll
            for (int s = 0; s < MS; ++s) {
                uint4 xv = make_uint4(0u, 0u, 0u, 0u);
                if (act_row[s]) xv = ld_v4(act_row[s] + kofs + 8 * m);
                uint32_t b[4];
                act_pairs(xv, b);
                // k-step 2m: pairs 0/1; k-step 2m+1: pairs 2/3
                mma_bf16_16816(accA[s], d[0].p[0], d[1].p[0], d[0].p[1], d[1].p[1], b[0], b[1]);
                mma_bf16_16816(accB[s], d[2].p[0], d[3].p[0], d[2].p[1], d[3].p[1], b[0], b[1]);
                mma_bf16_16816(accA[s], d[0].p[2], d[1].p[2], d[0].p[3], d[1].p[3], b[2], b[3]);
                mma_bf16_16816(accB[s], d[2].p[2], d[3].p[2], d[2].p[3], d[3].p[3], b[2], b[3]);
            }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) wcur[r] = wnext[r];
    }

    // epilogue: lane holds rows (g, g+8) x columns (2t, 2t+1) of each sub-tile
#pragma unroll
    for (int s = 0; s < MS; ++s) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int slot = __ldg(a.sorted_ids + blk * BM + 8 * s + 2 * t + c);
            if (slot >= a.n_slots) continue;
            if (MODE == MODE_GATEUP) {
                uint16_t *h = a.h_out + (size_t)slot * a.n_out;
                h[rowA + g] = f32_to_bf16(silu_f32(accA[s][c]) * accB[s][c]);
                h[rowA + g + 8] = f32_to_bf16(silu_f32(accA[s][2 + c]) * accB[s][2 + c]);
            } else {
                const float wt = __ldg(a.topk_w + slot);
                float *y = a.y_out + (size_t)slot * a.n_out;
                y[rowA + g] = wt * accA[s][c];
                y[rowA + g + 8] = wt * accA[s][2 + c];
                y[rowB + g] = wt * accB[s][c];
                y[rowB + g + 8] = wt * accB[s][2 + c];
            }
        }
    }
}

template <int BM, int WARPS, int MODE>
static void launch_bm(const W4GroupedArgs &a, int max_blocks, cudaStream_t s)
{
    const int rows_per_cta = (MODE == MODE_GATEUP ? 16 : 32) * WARPS;
    dim3 grid(max_blocks, cdiv(a.n_out, rows_per_cta));
    w4a16_grouped_mma_kernel<BM, WARPS, MODE><<<grid, WARPS * 32, 0, s>>>(a);
}

void launch_w4a16_grouped_mma(const W4GroupedArgs &a, int mode, int block_m, int max_blocks, cudaStream_t s)
{
    if (max_blocks <= 0) return;
#define MOEQ_W4_CASE(BMV)                                                   \
    case BMV:                                                               \
        if (mode == MODE_GATEUP) launch_bm<BMV, 4, MODE_GATEUP>(a, max_blocks, s); \
        else launch_bm<BMV, 4, MODE_DOWN>(a, max_blocks, s);                \
        break;
    switch (block_m) {
        MOEQ_W4_CASE(8)
        MOEQ_W4_CASE(16)
        MOEQ_W4_CASE(32)
        MOEQ_W4_CASE(64)
        default: break;
    }
#undef MOEQ_W4_CASE
}

}  // namespace moeq
