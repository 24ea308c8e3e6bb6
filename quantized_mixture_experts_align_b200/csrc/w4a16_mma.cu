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
// packed weights from HBM through its own multi-stage cp.async ring in shared memory (16 B per
// lane per 128 inputs per row set; three stages in flight hide the HBM latency without holding
// registers). Every weight byte is used by exactly one warp, so the dequantized weights never go
// back to shared memory: a dequantized 32-bit word feeds two m16n8k16 k-steps directly as A
// fragments.
//
// Input permutation. The sum over K does not care about order, so inside a 128-input
// "quad-group" lane t (of a 4-lane quad) takes the 32 inputs of group t = 16 contiguous bytes of
// the row, which keeps each element with its own group scale. Word m of that group feeds
// k-steps 2m and 2m+1; its nibble pairs (0,4), (1,5), (2,6), (3,7) are extracted with one LOP3
// each (INT4: the nibble ORed into the mantissa of f16 1024, one shift by 8 per word; E2M1: see
// e2m1_pair_pre), so the activation fragments take the same pairs, rebuilt with PRMT from a
// 16-byte load.
#include "common.cuh"
#include "kernels.cuh"

namespace moeq {

namespace {

struct DeqWord {
    uint32_t p[4];  // bf16x2 pairs: (n0,n4) (n1,n5) (n2,n6) (n3,n7), already (q-8)*scale
};

// INT4 in f16: (q - 8) * s has up to 11 significant bits, exact in f16 (not in bf16), so the
// INT4 instantiations compute in f16 with f16 activations; MXFP4 / NVFP4 weights are exact in bf16.
template <int FMT>
__device__ __forceinline__ DeqWord dequant_word(uint32_t w, uint32_t scale2)
{
    DeqWord d;
    if (FMT == W4_FP4 || FMT == W4_NV) {
        // E2M1 code times the group factor 2^(s - 1) (see e2m1_pair_pre)
        d.p[0] = bf16x2_mul(e2m1_pair_pre<0>(w), scale2);
        d.p[1] = bf16x2_mul(e2m1_pair_pre<1>(w), scale2);
        d.p[2] = bf16x2_mul(e2m1_pair_pre<2>(w), scale2);
        d.p[3] = bf16x2_mul(e2m1_pair_pre<3>(w), scale2);
    } else {
        uint32_t q8[4];
        int4_pairs_minus8(w, q8);  // q - 8, exact
#pragma unroll
        for (int i = 0; i < 4; ++i) d.p[i] = f16x2_mul(q8[i], scale2);  // (q - 8) * s, exact
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

// Per-warp weight ring: each stage holds one 128-input quad-group of the warp's 4 row sets
// (16 B per lane per row set, lane-private slots) and their 4 bf16 scales per row (8 B per row,
// copied by lane (g, t) for row set t, row g and shared across the warp). Four stages measured
// best: a deeper ring takes shared memory from the L1 share of the unified L1/shared storage,
// which the activation and scale loads use.
constexpr int kW4Stages = 4;
// 2048 B codes + the scales of 4 row sets x 8 rows: 4 group-32 or 8 group-16 bf16 scales each
__host__ __device__ constexpr int w4_scale_slot_bytes(int fmt) { return fmt == W4_NV ? 16 : 8; }
__host__ __device__ constexpr int w4_stage_bytes(int fmt) { return 4 * 32 * 16 + 4 * 8 * w4_scale_slot_bytes(fmt); }

// MODE_GATEUP: rows [f0, f0+16) (gate) and [I + f0, I + f0 + 16) (up) of W13; epilogue writes
//              h[slot, f] = bf16(silu(gate) * up).
// MODE_DOWN:   rows [r0, r0+32) of W2; epilogue writes ys[slot, r] = bf16(topk_w[slot] * y) (weight 1
//              without routing weights: the plain grouped GEMM).
// CVT (INT4 only): the activations are bf16 and are converted to f16 in registers; otherwise they
// are already f16 (INT4) or bf16 (MXFP4 / NVFP4).
// Paired activations: the library's own activation rows (the routing kernel's copy of x for the
// decode schedule and every h this file writes) hold each 8-input group in the nibble-pair order
// (x0 x4) (x1 x5) (x2 x6) (x3 x7), so a 16-byte load is the four MMA B registers as they are; rows
// the caller passes (bf16 x in the few-row blocks (STRIDED) of the tensor-core schedule, the
// grouped GEMM's A, both with CVT for INT4) are paired in registers.
template <int MODE, bool STRIDED, bool CVT>
__host__ __device__ constexpr bool act_paired() { return !CVT && (MODE == MODE_DOWN || !STRIDED); }
template <int BM, int WARPS, int MODE, bool STRIDED, int FMT, bool CVT>
__global__ void __launch_bounds__(WARPS * 32) w4a16_grouped_mma_kernel(W4GroupedArgs a)
{
    constexpr int MS = BM / 8;  // token sub-tiles of 8 columns
    constexpr int S = kW4Stages;
    constexpr bool kActPrefetch = MS <= 2;
    extern __shared__ __align__(16) unsigned char smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    // Launched by launch_pdl (blk_stride 0), this kernel may start before the previous one ends.
    // A down kernel right after its gate/up kernel may read the routing buffers at once (the
    // gate/up kernel lets it start only after waiting for the alignment) and prefetches its
    // weights before waiting for h; otherwise every read waits. Every CTA waits before it exits,
    // so this grid completes after the previous one.
    const bool early = MODE == MODE_DOWN && !STRIDED && a.after_gateup;
    if (!early) pdl_wait();
    pdl_trigger();
    const int blk = blockIdx.x;
    const int base = blk * (STRIDED ? a.blk_stride : BM);  // first aligned row of the block
    // Data earlier kernels of the chain write (the alignment, the routing weights, h) is read with
    // ordinary loads, never __ldg: a read-only (non-coherent) load may be scheduled ahead of the
    // programmatic-launch wait, and these kernels can start while their predecessor still runs.
    const int e = a.expert_ids[blk];
    const int tile = blockIdx.y * WARPS + warp;
    const int rowA = tile * (MODE == MODE_GATEUP ? 16 : 32);
    const int rowB = MODE == MODE_GATEUP ? a.n_out + rowA : rowA + 16;
    // strided: blocks with more than BM real rows are the tensor-core path's (real rows come first)
    if (base >= *a.num_tokens_padded || (STRIDED && a.sorted_ids[base + BM] < a.n_slots) || e < 0 ||
        e >= a.E || rowA >= a.n_out) {
        if (early) pdl_wait();
        return;
    }

    // token columns this lane feeds as MMA B (column g of each sub-tile)
    const int K = a.K;
    const int KW = K / 8;    // int32 words per weight row
    constexpr int GS = FMT == W4_NV ? 16 : 32;   // inputs per scale
    constexpr int SB = w4_stage_bytes(FMT), SS = w4_scale_slot_bytes(FMT);
    const int KG = K / GS;   // scale groups per weight row
    const uint16_t *act_row[MS];
#pragma unroll
    for (int s = 0; s < MS; ++s) {
        const int slot = a.sorted_ids[base + 8 * s + g];
        act_row[s] = (slot < a.n_slots) ? a.act + (size_t)(slot / a.act_row_div) * K : nullptr;
    }

    const int32_t *wq = a.wq + (size_t)e * a.n_rows * KW;
    const uint16_t *wsc = a.ws + (size_t)e * a.n_rows * KG;
    const int row_of_set[4] = {rowA + g, rowA + g + 8, rowB + g, rowB + g + 8};
    const int32_t *wr[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) wr[r] = wq + (size_t)row_of_set[r] * KW + 4 * t;
    const uint16_t *my_scale_row = wsc + (size_t)row_of_set[t] * KG;  // copied by this lane

    unsigned char *ring = smem + (size_t)warp * S * SB;
    auto code_slot = [&](int st, int r) { return ring + st * SB + r * 512 + lane * 16; };
    auto scale_slot = [&](int st, int r, int gg) { return ring + st * SB + 2048 + (r * 8 + gg) * SS; };

    const int NQ = K / 128;
    auto issue = [&](int q) {
        if (q < NQ) {
            const int st = q % S;
#pragma unroll
            for (int r = 0; r < 4; ++r) cp_async16_stream(code_slot(st, r), wr[r] + 16 * q);
            if (FMT == W4_NV) cp_async16_stream(scale_slot(st, t, g), my_scale_row + 8 * q);
            else cp_async8(scale_slot(st, t, g), my_scale_row + 4 * q);
        }
        cp_async_commit();  // possibly empty: keeps the group count uniform
    };

    float accA[MS][4], accB[MS][4];
#pragma unroll
    for (int s = 0; s < MS; ++s)
#pragma unroll
        for (int i = 0; i < 4; ++i) { accA[s][i] = 0.f; accB[s][i] = 0.f; }

#pragma unroll
    for (int q = 0; q < S - 1; ++q) issue(q);
    if (early) pdl_wait();  // h comes from the gate/up kernel

    uint4 xcur[kActPrefetch ? MS : 1][4];
    if (kActPrefetch) {
#pragma unroll
        for (int s = 0; s < MS; ++s)
#pragma unroll
            for (int m = 0; m < 4; ++m)
                xcur[s][m] = act_row[s] ? ld_v4_coherent(act_row[s] + 32 * t + 8 * m) : make_uint4(0u, 0u, 0u, 0u);
    }

    for (int q = 0; q < NQ; ++q) {
        cp_async_wait<S - 2>();
        __syncwarp();
        const int st = q % S;
        uint4 wcur[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) wcur[r] = *reinterpret_cast<const uint4 *>(code_slot(st, r));
        // this lane's 32 inputs: one group-32 scale, or (group 16) one for words 0-1 and one for
        // words 2-3 (sc holds both halves then)
        uint32_t sc[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            if (FMT == W4_NV) {
                sc[r] = reinterpret_cast<const uint32_t *>(scale_slot(st, r, g))[t];  // (lo, hi)
            } else {
                const uint32_t s16 = reinterpret_cast<const uint16_t *>(scale_slot(st, r, g))[t];
                if (FMT == W4_INT4) {
                    const float sf = __uint_as_float(s16 << 16);
                    sc[r] = pack_f16x2(sf, sf);  // the bf16 scale in f16, both halves (exact in range)
                } else {
                    sc[r] = s16 | (s16 << 16);
                }
            }
        }
        issue(q + S - 1);  // refills the slot every lane finished reading in iteration q - 1

        uint4 xnext[kActPrefetch ? MS : 1][4];
        const int kofs = 128 * q + 32 * t;
        if (kActPrefetch) {
            const int kn = (q + 1 < NQ) ? kofs + 128 : kofs;
#pragma unroll
            for (int s = 0; s < MS; ++s)
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    xnext[s][m] = act_row[s] ? ld_v4_coherent(act_row[s] + kn + 8 * m) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const uint32_t words[4] = {(&wcur[0].x)[m], (&wcur[1].x)[m], (&wcur[2].x)[m], (&wcur[3].x)[m]};
            DeqWord d[4];
#pragma unroll
            for (int r = 0; r < 4; ++r)
                d[r] = dequant_word<FMT>(words[r], FMT != W4_NV ? sc[r] : prmt(sc[r], sc[r], m < 2 ? 0x1010u : 0x3232u));
#pragma unroll
            for (int s = 0; s < MS; ++s) {
                uint4 xv;
                if (kActPrefetch) xv = xcur[s][m];
                else xv = act_row[s] ? ld_v4_coherent(act_row[s] + kofs + 8 * m) : make_uint4(0u, 0u, 0u, 0u);
                if (FMT == W4_INT4 && CVT) {
                    xv.x = bf16x2_to_f16x2(xv.x);
                    xv.y = bf16x2_to_f16x2(xv.y);
                    xv.z = bf16x2_to_f16x2(xv.z);
                    xv.w = bf16x2_to_f16x2(xv.w);
                }
                uint32_t b[4];
                if (act_paired<MODE, STRIDED, CVT>()) {
                    b[0] = xv.x;
                    b[1] = xv.y;
                    b[2] = xv.z;
                    b[3] = xv.w;
                } else {
                    act_pairs(xv, b);
                }
                // k-step 2m: pairs 0/1; k-step 2m+1: pairs 2/3
                if (FMT == W4_INT4) {
                    mma_f16_16816(accA[s], d[0].p[0], d[1].p[0], d[0].p[1], d[1].p[1], b[0], b[1]);
                    mma_f16_16816(accB[s], d[2].p[0], d[3].p[0], d[2].p[1], d[3].p[1], b[0], b[1]);
                    mma_f16_16816(accA[s], d[0].p[2], d[1].p[2], d[0].p[3], d[1].p[3], b[2], b[3]);
                    mma_f16_16816(accB[s], d[2].p[2], d[3].p[2], d[2].p[3], d[3].p[3], b[2], b[3]);
                } else {
                    mma_bf16_16816(accA[s], d[0].p[0], d[1].p[0], d[0].p[1], d[1].p[1], b[0], b[1]);
                    mma_bf16_16816(accB[s], d[2].p[0], d[3].p[0], d[2].p[1], d[3].p[1], b[0], b[1]);
                    mma_bf16_16816(accA[s], d[0].p[2], d[1].p[2], d[0].p[3], d[1].p[3], b[2], b[3]);
                    mma_bf16_16816(accB[s], d[2].p[2], d[3].p[2], d[2].p[3], d[3].p[3], b[2], b[3]);
                }
            }
        }
        if (kActPrefetch) {
#pragma unroll
            for (int s = 0; s < MS; ++s)
#pragma unroll
                for (int m = 0; m < 4; ++m) xcur[s][m] = xnext[s][m];
        }
    }
    cp_async_wait<0>();

    // epilogue: lane holds rows (g, g+8) x columns (2t, 2t+1) of each sub-tile; NVFP4 accumulators
    // carry 2^-8 / (tensor scale) of the true product
    if (FMT == W4_NV) {
        const float gsc = __ldg(a.wglobal + e) * 256.f;
#pragma unroll
        for (int s = 0; s < MS; ++s)
#pragma unroll
            for (int i = 0; i < 4; ++i) { accA[s][i] *= gsc; accB[s][i] *= gsc; }
    }
#pragma unroll
    for (int s = 0; s < MS; ++s) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int slot = a.sorted_ids[base + 8 * s + 2 * t + c];
            if (slot >= a.n_slots) continue;
            if (MODE == MODE_GATEUP) {
                uint16_t *h = a.h_out + (size_t)slot * a.n_out;
                // h = bf16(silu(g) * u), stored as f16 for the INT4 down GEMM (the same value)
                const float h0 = silu_f32(accA[s][c]) * accB[s][c];
                const float h1 = silu_f32(accA[s][2 + c]) * accB[s][2 + c];
                // features rowA + g and rowA + 8 + g at their paired columns (the down GEMM reads h
                // paired): position 2j of an 8-group holds input j < 4, position 2(j - 4) + 1 input j
                const int pg = g < 4 ? 2 * g : 2 * g - 7;
                h[rowA + pg] = FMT == W4_INT4 ? f32_to_bf16_as_f16(h0) : f32_to_bf16(h0);
                h[rowA + 8 + pg] = FMT == W4_INT4 ? f32_to_bf16_as_f16(h1) : f32_to_bf16(h1);
            } else {
                const float wt = a.topk_w ? a.topk_w[slot] : 1.f;
                uint16_t *y = a.y_out + (size_t)slot * a.n_out;
                y[rowA + g] = f32_to_bf16(wt * accA[s][c]);
                y[rowA + g + 8] = f32_to_bf16(wt * accA[s][2 + c]);
                y[rowB + g] = f32_to_bf16(wt * accB[s][c]);
                y[rowB + g + 8] = f32_to_bf16(wt * accB[s][2 + c]);
            }
        }
    }
}

template <int BM, int WARPS, int MODE, bool STRIDED, int FMT, bool CVT>
static void launch_bm_fmt(const W4GroupedArgs &a, int max_blocks, cudaStream_t s)
{
    const int rows_per_cta = (MODE == MODE_GATEUP ? 16 : 32) * WARPS;
    const size_t smem = (size_t)WARPS * kW4Stages * w4_stage_bytes(FMT);
    static std::atomic<int> smem_enabled[kMaxDevices];
    enable_smem(w4a16_grouped_mma_kernel<BM, WARPS, MODE, STRIDED, FMT, CVT>, (int)smem, smem_enabled);
    dim3 grid(max_blocks, cdiv(a.n_out, rows_per_cta));
    if (STRIDED)  // after the tensor-core kernels of the same stage: an ordinary launch
        w4a16_grouped_mma_kernel<BM, WARPS, MODE, STRIDED, FMT, CVT><<<grid, WARPS * 32, smem, s>>>(a);
    else
        launch_pdl(w4a16_grouped_mma_kernel<BM, WARPS, MODE, STRIDED, FMT, CVT>, grid, dim3(WARPS * 32), smem, s, a);
}

template <int BM, int WARPS, int MODE, bool STRIDED>
static void launch_bm(const W4GroupedArgs &a, int max_blocks, cudaStream_t s)
{
    if (a.fmt == W4_FP4) launch_bm_fmt<BM, WARPS, MODE, STRIDED, W4_FP4, false>(a, max_blocks, s);
    else if (a.fmt == W4_NV) launch_bm_fmt<BM, WARPS, MODE, STRIDED, W4_NV, false>(a, max_blocks, s);
    else if (a.act_bf16) launch_bm_fmt<BM, WARPS, MODE, STRIDED, W4_INT4, true>(a, max_blocks, s);
    else launch_bm_fmt<BM, WARPS, MODE, STRIDED, W4_INT4, false>(a, max_blocks, s);
}

// UE8M0 -> bf16 2^(s - 1): exponent field s + 126 (s <= 128); larger codes give +inf
__global__ void mxfp4_scale_factor_kernel(const uint8_t *__restrict__ sc, long long n, uint16_t *__restrict__ f)
{
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const uint32_t e = sc[i];
        f[i] = e <= 128u ? (uint16_t)((e + 126u) << 7) : (uint16_t)0x7F80u;
    }
}

void launch_w4a16_grouped_mma(const W4GroupedArgs &a, int mode, int block_m, int max_blocks, cudaStream_t s)
{
    if (max_blocks <= 0) return;
    if (a.blk_stride) {  // small blocks of the tensor-core schedule
        if (block_m != 8) return;
        if (mode == MODE_GATEUP) launch_bm<8, 4, MODE_GATEUP, true>(a, max_blocks, s);
        else launch_bm<8, 4, MODE_DOWN, true>(a, max_blocks, s);
        return;
    }
#define MOEQ_W4_CASE(BMV)                                                          \
    case BMV:                                                                      \
        if (mode == MODE_GATEUP) launch_bm<BMV, 4, MODE_GATEUP, false>(a, max_blocks, s); \
        else launch_bm<BMV, 4, MODE_DOWN, false>(a, max_blocks, s);                \
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

// E4M3 -> bf16 of E4M3 * 2^118: sign, exponent e (bias 7) and 3 mantissa bits m; e = 0 is the
// subnormal range m * 2^-9. The f32 product is exact and its upper half is the bf16 value.
__global__ void nvfp4_scale_factor_kernel(const uint8_t *__restrict__ sc, long long n, uint16_t *__restrict__ f)
{
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const uint32_t b = sc[i], e = (b >> 3) & 15u, m = b & 7u;
        uint32_t bits;
        if (e == 15u && m == 7u) {
            bits = 0x7FC0u;                                          // NaN
        } else {
            const float v = e ? __uint_as_float(((e + 120u) << 23) | (m << 20))  // 2^(e-7) (1+m/8)
                              : (float)m * 0x1p-9f;
            bits = __float_as_uint(v * 0x1p118f) >> 16;
        }
        f[i] = (uint16_t)(bits | ((b & 0x80u) << 8));
    }
}

void launch_nvfp4_scale_factors(const uint8_t *s, long long n, uint16_t *f, int num_sms, cudaStream_t st)
{
    const long long want = (n + 255) / 256;
    const int blocks = (int)(want < 8LL * num_sms ? want : 8LL * num_sms);
    nvfp4_scale_factor_kernel<<<blocks, 256, 0, st>>>(s, n, f);
}

void launch_mxfp4_scale_factors(const uint8_t *s, long long n, uint16_t *f, int num_sms, cudaStream_t st)
{
    const long long want = (n + 255) / 256;
    const int blocks = (int)(want < 8LL * num_sms ? want : 8LL * num_sms);
    mxfp4_scale_factor_kernel<<<blocks, 256, 0, st>>>(s, n, f);
}

}  // namespace moeq
