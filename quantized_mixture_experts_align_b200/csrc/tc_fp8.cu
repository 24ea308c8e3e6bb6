// Block-FP8 GEMM on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// "SGLang W8A8 Block FP8 quantized kernel config files", section "Background":
//   C[m, n] = sum over 128-wide K blocks kb of As[m, kb] * Bs[n/128, kb] * (A_q[m, kb] . B_q[n, kb]).
// The per-block scales are arbitrary f32 values, so the tensor core's block-scaled MMA (power-of-
// two UE8M0 scale factors per 32 inputs) does not apply. Instead every 128-wide K block is
// accumulated by the tensor core into its own tensor-memory buffer and promoted by the CUDA cores:
// acc += As * Bs * partial, with two partial buffers so the MMAs of block kb+1 run while block kb
// is promoted.
//
// CTA = one 128 x BN output tile, 18 warps:
//   warp 0      TMA producer: A [128 x 128 B] and B [BN x 128 B] tiles per K block, 128-byte
//               swizzle, into a 4-stage shared-memory ring (mbarrier transaction counts);
//   warp 1      allocates tensor memory; one elected lane issues 4 tcgen05.mma (K = 32 each) per
//               K block into partial buffer kb % 2 and commits to the stage's "empty" and the
//               buffer's "full" barriers (warps 0 and 1 run their loops warp-wide, one elected
//               lane issuing, so the operands stay warp-uniform);
//   warps 2-17  promotion and epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. +31
//               (= tile rows) and one quarter of the columns, keeps the running f32 sums in
//               registers (the next block's scales are loaded while the partial is awaited),
//               and finally writes bf16 C.
// Every wait is bounded; a wait that gives up flags the kernel status word and the CTA drains.
//
// The same kernel runs the grouped expert GEMMs of the block-FP8 MoE layer over expert-contiguous
// rows (the routed slots gathered in aligned order, every 128-row block owned by one expert):
//   TC_GATEUP  B stage = 128 gate rows + 128 up rows of the block's expert; the epilogue forms
//              a = silu(g) * u and quantizes it per row and 128-feature group to E4M3 + f32 scale
//              (the two column halves of a row meet through shared memory for the group max);
//   TC_DOWN    B = 256 rows of W2[e]; the epilogue multiplies by the slot's routing weight and
//              writes the bf16 slot row for the combine.
#include "kernels.cuh"
#include "tc_common.cuh"

namespace moeq {

namespace {

constexpr int kBM = 128;
constexpr int kFp8DownTilesPerCta = 4;  // grouped down GEMM: output tiles run by one CTA
constexpr int kBK = 128;  // one scale block; bytes = elements for E4M3
// promotion warps: 4 per tensor-memory lane quarter (each a quarter of the columns) for gate/up,
// whose epilogue is the heaviest; 2 per quarter (each half of the columns) otherwise, which
// leaves the MMA thread's SM sub-partition less crowded (both chosen from measured A/B runs)
__host__ __device__ constexpr int epi_warps(int mode) { return mode == TC_GATEUP ? 16 : 8; }
__host__ __device__ constexpr int fp8_threads(int mode) { return (2 + epi_warps(mode)) * 32; }

// PAIR: a cluster of 2 CTAs runs one 256 x BN tile with cta_group::2 MMAs; each CTA loads its 128
// rows of A and half of the BN weight rows, so a CTA moves 32 KB instead of 48 KB from L2 per K
// block for the same MMA work, and the smaller stages make a 6-deep ring.
template <int BN, bool PAIR, int MODE>
struct Fp8TcShape {
    static constexpr int kStages = PAIR ? 6 : 4;
    static constexpr int kABytes = kBM * kBK;
    static constexpr int kBBytes = (PAIR ? BN / 2 : BN) * kBK;
    static constexpr int kStageBytes = kABytes + kBBytes;
    // partial buffers: all 512 tensor-memory columns (4 of 128 or 2 of 256), so the MMAs run up to
    // kNBuf - 1 K blocks ahead of the promotion; channelwise: one accumulator over all of K
    static constexpr int kNBuf = MODE == TC_DENSE_CW ? 1 : (BN <= 128 ? 4 : 2);
    static constexpr int kTmemCols = kNBuf * BN;
    static constexpr int kSlices = epi_warps(MODE) / 4;  // column slices per lane quarter
    static constexpr int kColsPerWarp = BN / kSlices;
    static constexpr size_t kSmemBytes = (size_t)kStages * kStageBytes + 1024 + 256 + kSlices * 128 * 4;
};

// partial-tile row pitch in floats for the K-split sum: BN + 4 keeps the float4 stores of 8
// consecutive rows (one quarter warp) on distinct banks
template <int BN>
__host__ __device__ constexpr int kRedStride() { return BN + 4; }

__device__ __forceinline__ float4 ld_cluster_f32x4(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

template <int BN, int MODE, bool PAIR>
__global__ void __launch_bounds__(fp8_threads(MODE), 1)
    fp8_tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       Fp8TcArgs a)
{
    using Sh = Fp8TcShape<BN, PAIR, MODE>;
    constexpr int kStages = Sh::kStages;
    constexpr int kEpiWarps = epi_warps(MODE);
    constexpr bool kDense = MODE == TC_DENSE || MODE == TC_DENSE_CW;
    static_assert(!PAIR || BN == 256, "pair tiles are 256 x 256");
    static_assert(PAIR || (size_t)kBM * kRedStride<BN>() * 4 <= (size_t)kStages * Sh::kStageBytes,
                  "the K-split partial tile must fit in the stage ring");
    static_assert(MODE != TC_GATEUP || BN == 256, "gate/up tiles hold 128 gate + 128 up columns");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * Sh::kStageBytes);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;
    constexpr int NB = Sh::kNBuf;
    static_assert((2 * kStages + 2 * NB + 1) * 8 + 16 <= 256, "barriers, tensor-memory slot and flag fit their region");
    uint64_t *tempty = tfull + NB;
    uint64_t *mma_done = tempty + NB;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // dense: grid x = row tiles, so consecutive CTAs share a B (weight) tile in L2; grouped: grid
    // x = output tiles, so the tiles of one expert block run back to back and its activation rows
    // come from DRAM once
    // pair: rank 0 holds rows [0, 128) of the 256-row tile, rank 1 rows [128, 256); x counts CTAs
    const uint32_t rank = PAIR ? tc::cluster_rank() : 0u;
    const int tile_x = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int m0 = PAIR ? (kDense ? tile_x : (int)blockIdx.y) * 2 * kBM + (int)rank * kBM
                        : (kDense ? tile_x : (int)blockIdx.y) * kBM;
    const int KB = a.K / kBK;
    // K split (dense, no pair): the gridDim.z CTAs of a cluster take contiguous K-block ranges of
    // the same tile and sum their partial tiles through distributed shared memory at the end
    const int nsplit = (kDense && !PAIR) ? (int)gridDim.z : 1;
    const int kb0 = (kDense && !PAIR) ? (int)blockIdx.z * KB / nsplit : 0;
    const int nkb = (kDense && !PAIR) ? ((int)blockIdx.z + 1) * KB / nsplit - kb0 : KB;
    // output columns of this tile and the weight rows (in the [E * rows, K] weight matrix) loaded
    // into the B stage: dense and down take BN consecutive rows; gate/up takes 128 gate + 128 up
    int n0, brow0, brow1 = 0;
    const float *bscale0, *bscale1 = nullptr;
    if (kDense) {
        n0 = blockIdx.y * BN;
        brow0 = n0;
        bscale0 = MODE == TC_DENSE_CW ? a.b_scale + n0 : a.b_scale + (size_t)(n0 / 128) * KB;
    } else {
        // uniform over the CTA (and the pair: both test the pair's first row), before any barrier
        if ((PAIR ? (int)blockIdx.y * 2 * kBM : m0) >= __ldg(a.ntp)) return;
        const int e = __ldg(a.expert_ids + blockIdx.y);
        if (e < 0 || e >= a.E) return;
        const float *ws = a.b_scale + (size_t)e * (a.rows_per_expert / 128) * KB;
        if (MODE == TC_GATEUP) {
            n0 = tile_x * 128;                          // feature tile
            brow0 = e * a.rows_per_expert + n0;         // gate rows
            brow1 = e * a.rows_per_expert + a.N + n0;   // up rows
            bscale0 = ws + (size_t)(n0 / 128) * KB;
            bscale1 = ws + (size_t)((a.N + n0) / 128) * KB;
        } else {
            n0 = tile_x * a.tiles_per_cta * BN;  // the first of this CTA's output tiles
            brow0 = e * a.rows_per_expert + n0;
            bscale0 = ws + (size_t)(n0 / 128) * KB;
        }
    }
    // weight rows this CTA loads: all BN, or (pair) its half: gate/up rank 0 the gate rows, rank 1
    // the up rows; dense / down rank r the rows [128 r, 128 r + 128) of the tile
    const int brow_own = !PAIR ? brow0 : (MODE == TC_GATEUP ? (rank ? brow1 : brow0) : brow0 + (int)rank * 128);
    // grouped down: ntl consecutive BN-column output tiles of the block run through one pipeline;
    // the promotion warps hold the accumulator in registers, so the next tile's MMAs overlap this
    // tile's epilogue
    const int ntl = MODE == TC_DOWN ? min(a.tiles_per_cta, a.N / BN - tile_x * a.tiles_per_cta) : 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < NB; ++b) {
            tc::mbar_init(&tfull[b], 1);
            tc::mbar_init(&tempty[b], kEpiWarps * (PAIR ? 2 : 1));  // pair: both CTAs' promotion warps
        }
        tc::mbar_init(mma_done, 1);
        *abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        if (PAIR) tc::tmem_alloc_pair(tmem_slot, Sh::kTmemCols);
        else tc::tmem_alloc(tmem_slot, Sh::kTmemCols);
    }
    tc::fence_before_sync();
    if (PAIR) tc::cluster_sync();  // both CTAs' barriers exist before any copy or arrival crosses over
    else __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // the whole warp runs the producer loop (warp-uniform operands); one elected lane issues
        // each stage's copies
        if (lane == 0) {
            tc::prefetch_tmap(&tmA);
            tc::prefetch_tmap(&tmB);
        }
        const uint32_t empty0 = smem_addr(empty);
        uint32_t s = 0, ph = 0;  // ring stage of the next K block, its parity
        int issued = 0;
        bool live = true;
        for (int tt = 0, gs = 0; tt < ntl && live; ++tt)
        for (int kb = 0; kb < nkb; ++kb, ++gs) {  // local K index, x = (kb0 + kb) * kBK; gs over tiles
            if (gs >= kStages && !__all_sync(0xFFFFFFFFu, tc::mbar_try_wait_addr(empty0 + 8u * s, ph ^ 1u)) &&
                !tc::mbar_wait_warp(&empty[s], ph ^ 1u, abort_flag, a.status)) {
                live = false;
                break;
            }
            uint8_t *sa = smem + s * Sh::kStageBytes;
            if (tc::elect_one()) {
                if (PAIR) {
                    // both CTAs' bytes complete on rank 0's barrier, which alone expects them
                    const uint32_t fb = tc::cluster_addr(&full[s], 0);
                    if (rank == 0) tc::mbar_arrive_expect_tx(&full[s], 2 * Sh::kStageBytes);
                    tc::tma_load_2d_pair(sa, &tmA, fb, kb * kBK, m0);
                    tc::tma_load_2d_pair(sa + Sh::kABytes, &tmB, fb, kb * kBK, brow_own);
                } else {
                    tc::mbar_arrive_expect_tx(&full[s], Sh::kStageBytes);
                    const int x = (kb0 + kb) * kBK;
                    tc::tma_load_2d(sa, &tmA, &full[s], x, m0);
                    if (MODE == TC_GATEUP) {
                        tc::tma_load_2d(sa + Sh::kABytes, &tmB, &full[s], x, brow0);
                        tc::tma_load_2d(sa + Sh::kABytes + 128 * kBK, &tmB, &full[s], x, brow1);
                    } else {
                        tc::tma_load_2d(sa + Sh::kABytes, &tmB, &full[s], x, brow0 + tt * BN);
                    }
                }
            }
            __syncwarp();
            issued = gs + 1;
            if (++s == (uint32_t)kStages) {
                s = 0;
                ph ^= 1u;
            }
        }
        // no copy may still be landing in shared memory when the CTA exits (pair: rank 0's
        // barrier counts both CTAs' bytes; rank 1 is held by the final cluster barrier)
        if (lane == 0 && (!PAIR || rank == 0))
            for (int gs = issued - kStages > 0 ? issued - kStages : 0; gs < issued; ++gs)
                tc::mbar_drain(&full[gs % kStages], (gs / kStages) & 1, a.status);
    } else if (warp == 1) {
        if (PAIR && rank != 0) {
            // the peer issues nothing; it waits (bounded) until the pair's MMAs, which write its
            // tensor memory and read its shared memory, are done
            if (lane == 0) tc::mbar_drain(mma_done, 0, a.status);
        } else {
            // The whole warp runs the issue loop, so its operands stay warp-uniform; one elected
            // lane issues each K block's MMAs and commits (a lane-0 loop inside a divergent branch
            // competes for issue slots with the promotion warps of its sub-partition).
            constexpr uint32_t idesc = tc::idesc_f32(tc::kFmtE4M3, tc::kFmtE4M3, PAIR ? 2 * kBM : kBM, BN);
            const uint64_t a_base = tc::smem_desc_sw128(smem);
            const uint32_t full0 = smem_addr(full), tempty0 = smem_addr(tempty);
            uint32_t s = 0, ph = 0;      // ring stage of the next K block, its parity
            uint32_t buf = 0, pbuf = 0;  // partial buffer of the next K block, its parity
            bool live = true;
            for (int tt = 0, gs = 0; tt < ntl && live; ++tt)
            for (int kb = 0; kb < nkb; ++kb, ++gs) {
                if ((!__all_sync(0xFFFFFFFFu, tc::mbar_try_wait_addr(full0 + 8u * s, ph)) &&
                     !tc::mbar_wait_warp(&full[s], ph, abort_flag, a.status)) ||
                    (MODE != TC_DENSE_CW && gs >= NB &&
                     !__all_sync(0xFFFFFFFFu, tc::mbar_try_wait_addr(tempty0 + 8u * buf, pbuf ^ 1u)) &&
                     !tc::mbar_wait_warp(&tempty[buf], pbuf ^ 1u, abort_flag, a.status))) {
                    live = false;
                    break;
                }
                tc::fence_after_sync();
                // lean issue path: descriptors from a precomputed base; the first MMA of each K block
                // starts the partial, the other three always accumulate
                const uint64_t adesc = a_base + (uint64_t)((s * Sh::kStageBytes) >> 4);
                const uint64_t bdesc = adesc + (uint64_t)(Sh::kABytes >> 4);
                const uint32_t d = tmem + buf * BN;
                // channelwise: only the very first MMA starts the accumulator
                const uint32_t first_acc = (MODE == TC_DENSE_CW && kb > 0) ? 1u : 0u;
                if (tc::elect_one()) {
                    if (PAIR) {
                        tc::mma_f8f6f4_ss_pair(d, adesc, bdesc, idesc, first_acc);
#pragma unroll
                        for (int kk = 1; kk < kBK / 32; ++kk)
                            tc::mma_f8f6f4_ss_pair_acc(d, adesc + 2 * kk, bdesc + 2 * kk, idesc);
                        tc::mma_commit_pair(&empty[s], 0x3);
                        if (MODE != TC_DENSE_CW) tc::mma_commit_pair(&tfull[buf], 0x3);
                    } else {
                        tc::mma_f8f6f4_ss(d, adesc, bdesc, idesc, first_acc);
#pragma unroll
                        for (int kk = 1; kk < kBK / 32; ++kk)
                            tc::mma_f8f6f4_ss_acc(d, adesc + 2 * kk, bdesc + 2 * kk, idesc);
                        tc::mma_commit(&empty[s]);
                        if (MODE != TC_DENSE_CW) tc::mma_commit(&tfull[buf]);
                    }
                }
                __syncwarp();
                if (++s == (uint32_t)kStages) {
                    s = 0;
                    ph ^= 1u;
                }
                if (++buf == (uint32_t)NB) {
                    buf = 0;
                    pbuf ^= 1u;
                }
            }
            // (the commits below come from the lane that issued the MMAs: elect.sync picks the
            // same lane of the converged warp)
            // channelwise: the accumulator is complete once every MMA issued so far has finished
            if (MODE == TC_DENSE_CW && tc::elect_one()) {
                if (PAIR) tc::mma_commit_pair(&tfull[0], 0x3);
                else tc::mma_commit(&tfull[0]);
            }
            __syncwarp();
            // every MMA issued must finish before tensor memory is released
            if (tc::elect_one()) {
                if (PAIR) tc::mma_commit_pair(mma_done, 0x3);
                else tc::mma_commit(mma_done);
            }
            __syncwarp();
            if (lane == 0) tc::mbar_drain(mma_done, 0, a.status);
        }
    } else if (MODE == TC_DENSE_CW) {
        // warp w: tensor-memory lanes 32 (w % 4) .. +31 (= tile rows) and column slice cq; one
        // wait for the finished accumulator, then C = acc * As[m] * Bs[n] in bf16
        constexpr int COLS = Sh::kColsPerWarp;
        const int quarter = warp & 3, cq = (warp - 2) >> 2;
        const int m = m0 + quarter * 32 + lane;
        if (tc::mbar_wait_warp(&tfull[0], 0, abort_flag, a.status)) {
            tc::fence_after_sync();
            const float sa = __ldg(a.a_scale + (m < a.M ? m : a.M - 1));
            const float *bs = bscale0 + cq * COLS;
            const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + cq * COLS;
            uint16_t *crow = a.C + (size_t)m * a.N + n0 + cq * COLS;
            float *red = reinterpret_cast<float *>(smem) + (size_t)(quarter * 32 + lane) * kRedStride<BN>() + cq * COLS;
#pragma unroll 1
            for (int c = 0; c < COLS / 16; ++c) {
                uint32_t r[16];
                tc::tmem_ld16(taddr + c * 16, r);
                tc::tmem_wait_ld();
                if (nsplit > 1) {
                    // K split: the scaled partial tile goes to shared memory for the cluster sum
#pragma unroll
                    for (int j = 0; j < 16; j += 4)
                        *reinterpret_cast<float4 *>(red + c * 16 + j) = make_float4(
                            __uint_as_float(r[j]) * sa * __ldg(bs + c * 16 + j),
                            __uint_as_float(r[j + 1]) * sa * __ldg(bs + c * 16 + j + 1),
                            __uint_as_float(r[j + 2]) * sa * __ldg(bs + c * 16 + j + 2),
                            __uint_as_float(r[j + 3]) * sa * __ldg(bs + c * 16 + j + 3));
                } else if (m < a.M) {
                    uint32_t o[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        o[j] = pack_bf16x2(__uint_as_float(r[2 * j]) * sa * __ldg(bs + c * 16 + 2 * j),
                                           __uint_as_float(r[2 * j + 1]) * sa * __ldg(bs + c * 16 + 2 * j + 1));
                    *reinterpret_cast<uint4 *>(crow + c * 16) = make_uint4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<uint4 *>(crow + c * 16 + 8) = make_uint4(o[4], o[5], o[6], o[7]);
                }
            }
        }
    } else {
        // warp w: tensor-memory lanes 32 (w % 4) .. +31 (= tile rows) and column slice cq
        constexpr int COLS = Sh::kColsPerWarp;
        constexpr int GF = 128 / Sh::kSlices;  // gate/up: gate features per warp
        const int ew = warp - 2, quarter = warp & 3, cq = ew >> 2;
        const int row = quarter * 32 + lane;
        const int m = m0 + row;
        // TMEM columns of this warp: one contiguous slice of the tile, or (gate/up) GF gate
        // columns and the GF matching up columns
        const int c_first = (MODE == TC_GATEUP) ? GF * cq : cq * COLS;
        const int c_second = (MODE == TC_GATEUP) ? 128 + GF * cq : 0;
        const float *as_row = a.a_scale + (size_t)(m < a.M ? m : a.M - 1) * KB + kb0;
        bool ok = true;
        for (int tt = 0, gs = 0; tt < ntl && ok; ++tt) {
        const int n0t = n0 + tt * BN;  // this tile's first output column
        const float *bs_first =
            ((MODE == TC_GATEUP) ? bscale0 : bscale0 + (size_t)((tt * BN + cq * COLS) / 128) * KB) + kb0;
        const float *bs_second = (MODE == TC_GATEUP) ? bscale1 + kb0 : bs_first;
        float acc[COLS];
#pragma unroll
        for (int j = 0; j < COLS; ++j) acc[j] = 0.f;
        // the scales of block kb + 1 are loaded while block kb's partial is awaited
        float n_sa = __ldg(as_row), n_b0 = __ldg(bs_first), n_b1 = __ldg(bs_second);
        for (int kb = 0; kb < nkb && ok; ++kb, ++gs) {
            const int buf = gs % NB;
            const float sc0 = n_sa * n_b0, sc1 = n_sa * n_b1;
            if (kb + 1 < nkb) {
                n_sa = __ldg(as_row + kb + 1);
                n_b0 = __ldg(bs_first + kb + 1);
                n_b1 = __ldg(bs_second + kb + 1);
            }
            // lane 0 waits, the warp agrees: the tensor-memory loads below are warp-wide
            ok = tc::mbar_wait_warp(&tfull[buf], (gs / NB) & 1, abort_flag, a.status);
            if (!ok) break;
            tc::fence_after_sync();
            const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + buf * BN;
            // 16-column loads keep the registers to acc[] + 16
#pragma unroll
            for (int c = 0; c < COLS / 16; ++c) {
                // gate/up: the first GF / 16 chunks gate, the rest up; otherwise one contiguous run
                const bool second = (MODE == TC_GATEUP) && c >= GF / 16;
                const int col = (MODE == TC_GATEUP) ? (second ? c_second + (c - GF / 16) * 16 : c_first + c * 16)
                                                    : c_first + c * 16;
                const float sc = second ? sc1 : sc0;
                uint32_t r[16];
                tc::tmem_ld16(taddr + col, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[c * 16 + j] = fmaf(__uint_as_float(r[j]), sc, acc[c * 16 + j]);
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                if (PAIR && rank != 0) tc::mbar_arrive_cluster(tc::cluster_addr(&tempty[buf], 0));  // the issuer's
                else tc::mbar_arrive(&tempty[buf]);
            }
        }
        if (MODE == TC_DENSE && nsplit > 1) {
            // every MMA has completed (the last partial was awaited) and every copy landed: the
            // ring holds this CTA's partial tile, rows padded to kRedStride floats
            float *red = reinterpret_cast<float *>(smem) + (size_t)row * kRedStride<BN>() + cq * COLS;
#pragma unroll
            for (int j = 0; j < COLS; j += 4)
                *reinterpret_cast<float4 *>(red + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
        } else if (MODE == TC_DENSE) {
            if (ok && m < a.M) {
                uint16_t *crow = a.C + (size_t)m * a.N + n0 + cq * COLS;
#pragma unroll
                for (int j = 0; j < COLS; j += 8) {
                    uint4 v;
                    v.x = pack_bf16x2(acc[j], acc[j + 1]);
                    v.y = pack_bf16x2(acc[j + 2], acc[j + 3]);
                    v.z = pack_bf16x2(acc[j + 4], acc[j + 5]);
                    v.w = pack_bf16x2(acc[j + 6], acc[j + 7]);
                    *reinterpret_cast<uint4 *>(crow + j) = v;
                }
            }
        } else if (MODE == TC_GATEUP) {
            // a = silu(g) * u for features n0 + GF cq + j; E4M3 per row and 128-feature group
            float amax = 0.f;
#pragma unroll
            for (int j = 0; j < GF; ++j) {
                acc[j] = silu_f32(acc[j]) * acc[GF + j];
                amax = fmaxf(amax, fabsf(acc[j]));
            }
            float *red = reinterpret_cast<float *>(tmem_slot + 4);  // [slices][128] slice maxima
            red[cq * 128 + row] = amax;
            asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
            amax = red[row];
#pragma unroll
            for (int q = 1; q < Sh::kSlices; ++q) amax = fmaxf(amax, red[q * 128 + row]);
            const float sc = __fdiv_rn(fmaxf(amax, 1e-10f), 448.0f);
            if (ok) {
                uint8_t *hrow = a.hq + (size_t)m * a.N + n0 + GF * cq;
#pragma unroll
                for (int j = 0; j < GF; j += 16) {
                    uint4 v;
                    uint32_t *w = &v.x;
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const uint32_t lo = pack_e4m3x2(__fdiv_rn(acc[j + 4 * p], sc), __fdiv_rn(acc[j + 4 * p + 1], sc));
                        const uint32_t hi = pack_e4m3x2(__fdiv_rn(acc[j + 4 * p + 2], sc), __fdiv_rn(acc[j + 4 * p + 3], sc));
                        w[p] = lo | (hi << 16);
                    }
                    *reinterpret_cast<uint4 *>(hrow + j) = v;
                }
                if (cq == 0) a.hs[(size_t)m * (a.N / 128) + n0 / 128] = sc;
            }
        } else {
            const int slot = __ldg(a.sorted_ids + m);
            if (ok && slot < a.n_slots) {
                const float wt = __ldg(a.topk_w + slot);
                uint16_t *yrow = a.ys + (size_t)slot * a.N + n0t + cq * COLS;
#pragma unroll
                for (int j = 0; j < COLS; j += 8) {
                    uint4 v;
                    v.x = pack_bf16x2(wt * acc[j], wt * acc[j + 1]);
                    v.y = pack_bf16x2(wt * acc[j + 2], wt * acc[j + 3]);
                    v.z = pack_bf16x2(wt * acc[j + 4], wt * acc[j + 5]);
                    v.w = pack_bf16x2(wt * acc[j + 6], wt * acc[j + 7]);
                    *reinterpret_cast<uint4 *>(yrow + j) = v;
                }
            }
        }
        }  // output tiles
    }
    tc::fence_before_sync();
    if (kDense && !PAIR && nsplit > 1) {
        // K split: rank r sums rows [128 r / S, 128 (r + 1) / S) of the S partial tiles in rank
        // order (deterministic) and writes bf16 C; a second barrier keeps every CTA's partial tile
        // alive until all ranks have read it
        tc::cluster_sync();
        const int r = (int)blockIdx.z;
        const int row_lo = r * kBM / nsplit, row_hi = (r + 1) * kBM / nsplit;
        constexpr int kUnits = BN / 4;
        const float *red = reinterpret_cast<const float *>(smem);
        for (int u = threadIdx.x; u < (row_hi - row_lo) * kUnits; u += fp8_threads(MODE)) {
            const int row = row_lo + u / kUnits, col = (u % kUnits) * 4;
            const int m = m0 + row;
            if (m >= a.M) continue;
            const float *src = red + (size_t)row * kRedStride<BN>() + col;
            float4 t = ld_cluster_f32x4(tc::cluster_addr(src, 0));
            for (int q = 1; q < nsplit; ++q) {
                const float4 v = ld_cluster_f32x4(tc::cluster_addr(src, (uint32_t)q));
                t.x += v.x;
                t.y += v.y;
                t.z += v.z;
                t.w += v.w;
            }
            uint2 o;
            o.x = pack_bf16x2(t.x, t.y);
            o.y = pack_bf16x2(t.z, t.w);
            *reinterpret_cast<uint2 *>(a.C + (size_t)m * a.N + n0 + col) = o;
        }
        tc::cluster_sync();
    } else if (PAIR) {
        tc::cluster_sync();  // neither CTA leaves while the pair's copies or MMAs use it
    } else {
        __syncthreads();
    }
    tc::fence_after_sync();
    if (warp == 1) {
        if (PAIR) tc::tmem_dealloc_pair(tmem, Sh::kTmemCols);
        else tc::tmem_dealloc(tmem, Sh::kTmemCols);
    }
}

template <int BN, int MODE, bool PAIR = false>
int launch_tc(const Fp8TcArgs &a, const CUtensorMap &tmA, const CUtensorMap &tmB, int grid_x, int grid_y,
              cudaStream_t s, int split = 1)
{
    using Sh = Fp8TcShape<BN, PAIR, MODE>;
    constexpr int kThreads = fp8_threads(MODE);
    static std::atomic<int> smem_enabled[kMaxDevices];
    {
        const cudaError_t e = enable_smem(fp8_tc_gemm_kernel<BN, MODE, PAIR>, (int)Sh::kSmemBytes, smem_enabled);
        if (e != cudaSuccess)
            return set_error(MOEQ_ERR_CUDA, "tcgen05 FP8 GEMM: shared-memory attribute: %s", cudaGetErrorString(e));
    }
    if (grid_x <= 0 || grid_y <= 0) return MOEQ_OK;
    if (!PAIR && split <= 1) {
        fp8_tc_gemm_kernel<BN, MODE, PAIR><<<dim3(grid_x, grid_y), kThreads, Sh::kSmemBytes, s>>>(tmA, tmB, a);
        return MOEQ_OK;
    }
    // clusters of 2 CTAs along x (grid_x even): the pair of one 256-row tile; or (K split)
    // clusters of `split` CTAs along z: the K ranges of one tile
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid_x, grid_y, PAIR ? 1 : split);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = Sh::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr_c[1];
    attr_c[0].id = cudaLaunchAttributeClusterDimension;
    attr_c[0].val.clusterDim.x = PAIR ? 2 : 1;
    attr_c[0].val.clusterDim.y = 1;
    attr_c[0].val.clusterDim.z = PAIR ? 1 : split;
    cfg.attrs = attr_c;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, fp8_tc_gemm_kernel<BN, MODE, PAIR>, tmA, tmB, a);
    if (e != cudaSuccess) return set_error(MOEQ_ERR_CUDA, "tcgen05 FP8 clustered GEMM launch: %s", cudaGetErrorString(e));
    return MOEQ_OK;
}

}  // namespace

// Dense schedule, from measured sweeps (clean L2): single CTAs (128 x BN tiles) beat CTA pairs by
// 3-5 % on the block-scaled GEMM at 512-4096 rows of 24576 x 7168 (437 vs 451 us at 2048 rows,
// 824 vs 863 at 4096); on the channelwise GEMM the two tie, and pairs (half the B bytes per CTA)
// are kept there once the tiles fill two waves. The K range is split over a cluster only when the
// tiles fill less than half of the SMs (4096 x 4096 channelwise, 128-256 rows: 24.6 -> 20.5 us
// with a split of 4); with more tiles every split measured slower.
struct DenseSchedule {
    bool pair;
    int split;
};
static DenseSchedule pick_dense_schedule(int M, int N, int K, int bn, bool channelwise)
{
    const int KB = K / kBK, sms = 148;
    const long tiles = (long)cdiv(M, kBM) * (N / bn);
    if (channelwise && bn == 256 && M >= 256 && tiles >= 2 * sms) return {true, 1};
    if (2 * tiles < sms) {
        long sp = sms / tiles;
        if (sp > 4) sp = 4;
        if (sp > KB / 2) sp = KB / 2;
        return {false, sp < 1 ? 1 : (int)sp};
    }
    // a second wave under half full: two CTAs per tile shorten the tail (256 x 24576 x 7168: 86 ->
    // 81 us); from 1.5 waves on, every split measured slower
    if (!channelwise && tiles > sms && 2 * tiles < 3 * sms && KB >= 8) return {false, 2};
    return {false, 1};
}

int launch_fp8_tc_gemm(const Fp8TcArgs &a, const uint8_t *A, const uint8_t *B, cudaStream_t s)
{
    // Rows past 32 (fewer go to the swap-AB kernel): 256-column tiles (more weight bytes in flight
    // per SM, fewer activation re-reads; tensor bound for many rows), chosen from measured M sweeps.
    const int bn = (a.N % 256 == 0) ? 256 : 128;
    const DenseSchedule sch = pick_dense_schedule(a.M, a.N, a.K, bn, false);
    CUtensorMap tmA, tmB;
    int rc = make_tmap_2d(&tmA, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.M, (uint64_t)a.K, kBM, kBK);
    if (rc) return rc;
    rc = make_tmap_2d(&tmB, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.N, (uint64_t)a.K, bn, kBK);
    if (rc) return rc;
    if (bn == 256) return launch_tc<256, TC_DENSE>(a, tmA, tmB, cdiv(a.M, kBM), a.N / 256, s, sch.split);
    return launch_tc<128, TC_DENSE>(a, tmA, tmB, cdiv(a.M, kBM), a.N / 128, s, sch.split);
}

int launch_fp8_tc_channel(const Fp8TcArgs &a, const uint8_t *A, const uint8_t *B, cudaStream_t s)
{
    // the block-scaled GEMM's tiles and schedule: 256 columns where N allows, CTA pairs or a K split
    const int bn = (a.N % 256 == 0) ? 256 : 128;
    const DenseSchedule sch = pick_dense_schedule(a.M, a.N, a.K, bn, true);
    CUtensorMap tmA, tmB;
    int rc = make_tmap_2d(&tmA, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.M, (uint64_t)a.K, kBM, kBK);
    if (rc) return rc;
    rc = make_tmap_2d(&tmB, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.N, (uint64_t)a.K, sch.pair ? 128 : bn,
                      kBK);
    if (rc) return rc;
    if (sch.pair) return launch_tc<256, TC_DENSE_CW, true>(a, tmA, tmB, 2 * cdiv(a.M, 2 * kBM), a.N / 256, s);
    if (bn == 256) return launch_tc<256, TC_DENSE_CW>(a, tmA, tmB, cdiv(a.M, kBM), a.N / 256, s, sch.split);
    return launch_tc<128, TC_DENSE_CW>(a, tmA, tmB, cdiv(a.M, kBM), a.N / 128, s, sch.split);
}

int launch_fp8_tc_grouped(const Fp8TcArgs &a_in, int mode, const uint8_t *A, const uint8_t *W, int E, int max_blocks,
                          cudaStream_t s)
{
    // down: kFp8DownTilesPerCta output tiles per CTA (the K range is short, I = 2048: the fixed
    // per-CTA cost is shared and the next tile's MMAs overlap the epilogue)
    Fp8TcArgs a = a_in;
    a.tiles_per_cta = mode == TC_DOWN ? kFp8DownTilesPerCta : 1;
    CUtensorMap tmA, tmB;
    int rc = make_tmap_2d(&tmA, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.M, (uint64_t)a.K, kBM, kBK);
    if (rc) return rc;
    const uint32_t box = (mode == TC_GATEUP || a.N % 256 != 0) ? 128 : 256;
    rc = make_tmap_2d(&tmB, W, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)E * a.rows_per_expert, (uint64_t)a.K, box,
                      kBK);
    if (rc) return rc;
    if (mode == TC_GATEUP) return launch_tc<256, TC_GATEUP>(a, tmA, tmB, a.N / 128, max_blocks, s);
    if (a.N % 256 == 0)
        return launch_tc<256, TC_DOWN>(a, tmA, tmB, cdiv(a.N / 256, a.tiles_per_cta), max_blocks, s);
    return launch_tc<128, TC_DOWN>(a, tmA, tmB, cdiv(a.N / 128, a.tiles_per_cta), max_blocks, s);
}

}  // namespace moeq
