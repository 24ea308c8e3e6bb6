// W4A16 grouped expert GEMMs on the 5th-generation tensor cores (tcgen05, sm_100a), for expert
// blocks with many routed rows (prefill).
//
// "vLLM x Novita AI: Chord W4A16 INT4 MoE Kernel for Kimi K2.x": INT4 group-32 codes with bf16
// scales ("vLLM integration"), dequantized by subtracting the zero point and then scaling in
// bf16 ("H200 and Blackwell indexed decode"), the dequantization of the next stage overlapped
// with the pending MMAs ("H200 prefill and TP8"), a TMA producer feeding MMA consumers ("SM90
// grouped kernels"). Re-derived for tcgen05:
//
// Weights take the MMA's A side and live in TENSOR memory: dequantization warps turn the packed
// codes into f16 (INT4, exact) or bf16 (MXFP4 / NVFP4) in registers and store them with
// tcgen05.st, so dequantized weights never pass through shared memory (a 16-bit B-side tile would
// cost its shared-memory bandwidth twice, on write and on every MMA read). The activations (routed rows gathered in aligned order, one
// expert per 256-row block) are the B side, loaded by TMA with the 128-byte swizzle.
//   D[weight rows, tokens] += A_tmem[128 weight rows, K] * B_smem[tokens, K]^T   (M = 128, K = 16)
// A tile serves up to 256 tokens, so each dequantized weight feeds 256 rows of MMA work: the
// dequantization, not the MMA, bounds this kernel, and the wide tile halves it per FLOP. The
// MMA's N is the block's real row count rounded up to 16, so padding rows cost no MMA work.
// LOP3s (one shift per word) extract the nibble pairs (q0,q4) (q1,q5) (q2,q6) (q3,q7) of a 32-bit
// code word, and the weights enter tensor memory in that order: within every 8 inputs the K order is
// 0 4 1 5 2 6 3 7. The activations take the same order (the gather permutes each 8-input group of
// the routed rows it copies, the gate/up epilogue writes h that way), so the sum over K is
// unchanged and the dequantization needs no byte permutes.
//
// CTA = one 256-row activation block of one expert x consecutive output tiles, run back to back
// through one pipeline (gate/up: tiles of 64 features, each tensor-memory lane quarter holding the
// gate rows of 16 features in lanes 0-15 and their up rows in lanes 16-31; down: tiles of 128
// output rows):
//   warp 0      TMA producer of the activation tiles [256 tokens x 128 inputs] (3 stages, two
//               128-byte-swizzled halves of 64 inputs each; the warp runs the loop, one elected
//               lane issues the copies); a tile's bytes complete on the same "stage ready" barrier
//               the dequantization warps arrive on, and one commit per step frees both the weight
//               stage and the tile;
//   warp 1      tensor-memory allocation; the whole warp runs the issue loop and one elected lane
//               issues 8 MMAs (K = 16) per 128-input step into the one accumulator and commits.
//               A pipeline step costs several hundred cycles of synchronization whatever work it
//               carries (an MMA issue ~50-65 cycles, a barrier wait ~47 even when the phase is
//               complete, more under load), so the steps are long and the issuing warp waits on
//               one barrier and commits once per step;
//   warps 2-17  dequantization: a thread owns one weight row (tensor lane) and a 32-input slice
//               of each 128-input step (16 bytes of codes, 1 group scale), fetches them into
//               registers two steps ahead, and writes the dequantized slice to one of 3
//               tensor-memory stages; then the epilogue of each tile: gate/up pairs every gate
//               lane with its up lane by shuffles and writes h = bf16(silu(g) * u); down writes
//               the routing-weighted bf16 slot rows.
#include "kernels.cuh"
#include "tc_common.cuh"

namespace moeq {

namespace {

constexpr int kTok = 256;     // tokens per tile = aligned block size
constexpr int kKs = 128;      // inputs per pipeline step (8 MMAs per barrier round trip)
constexpr int kStages = 3;    // dequantized weight stages (tensor memory)
constexpr int kDownTilesPerCta = 4;    // down GEMM: 128-row output tiles run by one CTA
constexpr int kGateUpTilesPerCta = 2;  // gate/up GEMM: 64-feature output tiles run by one CTA
constexpr int kBStages = 3;   // activation tiles (shared memory)
// Per-thread packed-code prefetch depth (registers), in steps. The code loads go through L1: the
// four warps of a lane quarter read the four 16-byte quarters of each row's 64-byte step chunk, so
// the first warp's miss serves the other three (no-allocate loads ran 35 % slower). In-flight loads
// therefore hold L1 lines, and L1 is what shared memory leaves of the SM's 256 KB: measured, 2
// steps ran 2 % faster than 4 and 6 much slower, and 30 KB more shared memory made gate/up 47 %
// slower.
constexpr int kPf = 2;
constexpr int kDeqWarps = 16;  // 4 per tensor-memory lane quarter, each a quarter of every step
constexpr int kSplit = kDeqWarps / 4;           // K slices of a step (one per warp of a lane quarter)
constexpr int kThrK = kKs / kSplit;             // 32 inputs per thread per step: 4 code words, 1 group
static_assert(kThrK == 32, "one scale group per thread and step");
constexpr int kThreads = (2 + kDeqWarps) * 32;
constexpr int kAccCols = kTok;                  // one accumulator [128 lanes x 256 tokens]
constexpr int kAStageCols = kKs / 2;            // 128 bf16 inputs = 64 columns
constexpr int kTmemCols = 512;                  // 256 + 3 x 64 used, power of two allocated
constexpr int kBTile = kTok * kKs * 2;          // 64 KB: two 128-byte-swizzled halves of 64 inputs
constexpr int kBHalf = kBTile / 2;
constexpr size_t kSmemBytes = 1024 + (size_t)kBStages * kBTile + 256;
static_assert(kAccCols + kStages * kAStageCols <= kTmemCols, "tensor memory budget");
static_assert(kBStages == kStages, "one stage-free barrier serves the activation and weight stages");

// (q - 8) * scale (INT4) or E2M1(q) * 2^(s - 1) (FP4, see e2m1_pair_pre) in bf16 for the pairs
// (q0,q4) (q1,q5) (q2,q6) (q3,q7) of one code word
// INT4 runs in f16: (q - 8) * s has up to 11 significant bits (a 3-bit integer times the 8-bit
// significand of a bf16 scale), which f16 holds exactly and bf16 does not; the f16 MMA then sees
// the exact weights, and the bf16 activations, converted to f16, exactly too (within the f16 range).
// MXFP4 / NVFP4 weights are exact in bf16 and stay there.
template <int FMT>
__device__ __forceinline__ void dequant4(uint32_t w, uint32_t scale2, uint32_t *out)
{
    uint32_t p[4];  // the nibble pairs (q0,q4) (q1,q5) (q2,q6) (q3,q7)
    if (FMT == W4_FP4 || FMT == W4_NV) {
        p[0] = bf16x2_mul(e2m1_pair_pre<0>(w), scale2);
        p[1] = bf16x2_mul(e2m1_pair_pre<1>(w), scale2);
        p[2] = bf16x2_mul(e2m1_pair_pre<2>(w), scale2);
        p[3] = bf16x2_mul(e2m1_pair_pre<3>(w), scale2);
    } else {
        int4_pairs_minus8(w, p);  // q - 8, exact
#pragma unroll
        for (int i = 0; i < 4; ++i) p[i] = f16x2_mul(p[i], scale2);  // (q - 8) * s, exact
    }
    // K order 0 4 1 5 2 6 3 7 (the activations are permuted alike)
    out[0] = p[0];
    out[1] = p[1];
    out[2] = p[2];
    out[3] = p[3];
}

template <int MODE, int FMT>
__global__ void __launch_bounds__(kThreads, 1) w4a16_tc_kernel(const __grid_constant__ CUtensorMap tmX, W4TcArgs a)
{
    constexpr bool GU = MODE == TC_GATEUP;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *btiles = smem;
    uint64_t *a_full = reinterpret_cast<uint64_t *>(btiles + kBStages * kBTile);
    uint64_t *empty = a_full + kStages;
    uint64_t *acc_full = empty + kStages;
    uint64_t *mma_done = acc_full + 1;
    uint64_t *acc_empty = mma_done + 1;  // several output tiles: the accumulator has been read
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // grid x = output tiles, grid y = token blocks: the tiles of one block run back to back, so
    // the block's activation rows come from DRAM once and from L2 for the other tiles, and
    // consecutive blocks of one expert find its weights in L2
    const int r0 = blockIdx.y * kTok;
    if (r0 >= __ldg(a.ntp)) return;  // uniform over the CTA, before any barrier or allocation
    const int e = __ldg(a.expert_ids + blockIdx.y);
    if (e < 0 || e >= a.E) return;
    // nt consecutive output tiles of the block, run back to back through one pipeline (the setup,
    // the ring fill and the prefetch of the next tile's weights are shared; only the accumulator
    // drains between tiles)
    constexpr int kTileW = GU ? 64 : 128;  // output features (gate/up) or rows (down) of a tile
    const int tpc = a.tiles_per_cta;
    const int tile0 = blockIdx.x * tpc;
    const int nt = min(tpc, a.N / kTileW - tile0);
    const int n0 = tile0 * kTileW;  // first output feature (gate/up) or row (down)
    const int K = a.K, NS = K / kKs;  // K steps per tile
    // real rows of this block: the expert's slots come first, padding after
    const int valid = __syncthreads_count(threadIdx.x < kTok && __ldg(a.sorted_ids + r0 + threadIdx.x) < a.n_slots);
    const int n_mma = (valid + 15) & ~15;  // MMA N: multiple of 16 in [16, 256]
    if (valid <= a.small_rows) return;      // left to the register-fed kernel (uniform, before any barrier)

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(&a_full[s], kDeqWarps + 1);
            tc::mbar_init(&empty[s], 1);
        }
        tc::mbar_init(acc_full, 1);
        tc::mbar_init(mma_done, 1);
        tc::mbar_init(acc_empty, kDeqWarps);
        *abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // the whole warp runs the producer loop (warp-uniform operands); one elected lane issues
        // each tile's copies
        if (lane == 0) tc::prefetch_tmap(&tmX);
        const uint32_t empty0 = smem_addr(empty);
        uint32_t s = 0, ph = 0;  // stage of the next step, its parity
        int issued = 0;
        bool live = true;
        for (int tt = 0, gs = 0; tt < nt && live; ++tt) {
            for (int ks = 0; ks < NS; ++ks, ++gs) {  // gs: global step over the tiles
                if (gs >= kBStages && !__all_sync(0xFFFFFFFFu, tc::mbar_try_wait_addr(empty0 + 8u * s, ph ^ 1u)) &&
                    !tc::mbar_wait_warp(&empty[s], ph ^ 1u, abort_flag, a.status)) {
                    live = false;
                    break;
                }
                // the tile's bytes complete on the stage's a_full barrier (dequantization warps +
                // this arrival): the MMA warp waits on one barrier per step
                if (tc::elect_one()) {
                    tc::mbar_arrive_expect_tx(&a_full[s], kBTile);
                    tc::tma_load_2d(btiles + s * kBTile, &tmX, &a_full[s], ks * kKs, r0);
                    tc::tma_load_2d(btiles + s * kBTile + kBHalf, &tmX, &a_full[s], ks * kKs + kKs / 2, r0);
                }
                __syncwarp();
                issued = gs + 1;
                if (++s == kBStages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        if (lane == 0)
            for (int gs = issued - kBStages > 0 ? issued - kBStages : 0; gs < issued; ++gs)
                tc::mbar_drain(&a_full[gs % kBStages], (gs / kBStages) & 1, a.status);
    } else if (warp == 1) {
        // The whole warp runs the issue loop, so its operands stay warp-uniform; one elected lane
        // issues each step's MMAs and its commit. (Issued by lane 0 alone inside a divergent
        // branch, the loop took ~1100 cycles per step for 8 MMAs whatever their N: its operand
        // set-up competed for issue slots with the dequantization warps of its sub-partition.)
        constexpr uint32_t kFmt = FMT == W4_INT4 ? tc::kFmtF16 : tc::kFmtBF16;
        const uint32_t idesc = tc::idesc_f32(kFmt, kFmt, 128, n_mma);
        const uint32_t a_base = tmem + kAccCols;
        const uint64_t b_base = tc::smem_desc_sw128(btiles);
        const uint32_t a_full0 = smem_addr(a_full), empty0 = smem_addr(empty);
        uint32_t s = 0, ph = 0;  // stage of the next step (weights and activation tile), its parity
        bool live = true;
        for (int tt = 0; tt < nt && live; ++tt) {
            // a new tile overwrites the accumulator: the previous tile's epilogue has read it
            if (tt > 0 && !tc::mbar_wait_warp(acc_empty, (tt - 1) & 1, abort_flag, a.status)) break;
            for (int ks = 0; ks < NS; ++ks) {
                // one wait per step: a_full completes when the weight stage and the activation tile
                // are both in place
                if (!__all_sync(0xFFFFFFFFu, tc::mbar_try_wait_addr(a_full0 + 8u * s, ph)) &&
                    !tc::mbar_wait_warp(&a_full[s], ph, abort_flag, a.status)) {
                    live = false;
                    break;
                }
                tc::fence_after_sync();
                const uint64_t bdesc = b_base + (uint64_t)(s * (kBTile >> 4));
                const uint32_t astage = a_base + s * kAStageCols;
                if (tc::elect_one()) {
                    if (ks == 0) {
#pragma unroll
                        for (int kk = 0; kk < kKs / 16; ++kk)
                            tc::mma_f16_ts(tmem, astage + kk * 8, bdesc + (kk >> 2) * (kBHalf >> 4) + 2 * (kk & 3), idesc,
                                           kk > 0 ? 1u : 0u);
                    } else {
#pragma unroll
                        for (int kk = 0; kk < kKs / 16; ++kk)
                            tc::mma_f16_ts_acc(tmem, astage + kk * 8, bdesc + (kk >> 2) * (kBHalf >> 4) + 2 * (kk & 3),
                                               idesc);
                    }
                    tc::mma_commit_addr(empty0 + 8u * s);  // frees the weight stage and the activation tile
                }
                __syncwarp();
                if (++s == kStages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            if (live && tc::elect_one()) tc::mma_commit(acc_full);  // this tile's accumulator is complete
            __syncwarp();
        }
        // every MMA issued must finish before tensor memory is released (the commit comes from
        // the lane that issued them: elect.sync picks the same lane of the converged warp)
        if (tc::elect_one()) tc::mma_commit(mma_done);
        __syncwarp();
        if (lane == 0) tc::mbar_drain(mma_done, 0, a.status);
    } else {
        // ---- dequantization ----
        const int dw = warp - 2, quarter = warp & 3, kq = dw >> 2;  // lane quarter, K slice
        const int row = quarter * 32 + lane;                     // tensor-memory lane = weight row
        // gate/up: lanes 0-15 of each lane quarter hold the gate rows of 16 features, lanes 16-31
        // the up rows of the same features (the epilogue pairs them with one shuffle)
        const int grow = GU ? e * a.rows_per_expert + ((lane & 16) ? a.N : 0) + n0 + 16 * quarter + (lane & 15)
                            : e * a.rows_per_expert + n0 + row;
        const int32_t *wrow = a.wq + (size_t)grow * (K / 8) + kq * 4;  // 4 words = 32 inputs
        const size_t wtile = (size_t)kTileW * (K / 8);                  // next output tile
        // the group-32 scale of this thread's 32 inputs comes with its neighbour's in one aligned
        // 4-byte copy (rows are K/16 bytes apart, K a multiple of 128); group 16: its own two
        // scales, the same aligned 4 bytes
        constexpr int GS = FMT == W4_NV ? 16 : 32;
        const uint16_t *srow = a.ws + (size_t)grow * (K / GS) + (FMT == W4_NV ? 2 * kq : (kq & ~1));
        const size_t stile = (size_t)kTileW * (K / GS);
        // Codes and scales run kPf steps ahead in registers. A tile's steps are counted over NSP =
        // NS rounded up to kPf (the steps past NS do nothing), so the register slot of a step is its
        // index mod kPf: a constant in the loop unrolled by kPf, where slot j is consumed and refilled
        // in place. Every access is aligned: a row holds K / 2 bytes (K a multiple of 128) and a
        // thread's slice starts at 16 kq bytes.
        const int NSP = (NS + kPf - 1) / kPf * kPf;
        uint4 cq[kPf];
        uint32_t sq[kPf];
#pragma unroll
        for (int j = 0; j < kPf; ++j) {
            cq[j] = make_uint4(0u, 0u, 0u, 0u);
            sq[j] = 0u;
            if (j < NS) {
                cq[j] = __ldg(reinterpret_cast<const uint4 *>(wrow + j * (kKs / 8)));
                sq[j] = __ldg(reinterpret_cast<const uint32_t *>(srow + j * (kKs / GS)));
            }
        }
        const uint32_t a_full0 = smem_addr(a_full), empty0 = smem_addr(empty);
        // this thread's slot of weight stage 0 (tensor-memory lane quarter, K slice); stage s adds
        // s * kAStageCols columns
        const uint32_t tst0 = tmem + ((uint32_t)(quarter * 32) << 16) + kAccCols + kq * (kThrK / 2);
        // the stores of a step are waited for (tcgen05.wait::st) only after the dequantization of
        // the next step, so the tensor-memory write latency hides behind that work
        auto stage_ready = [&](uint32_t st) {
            tc::tmem_wait_st();
            tc::fence_before_sync();
            __syncwarp();
            tc::mbar_arrive_lane0(a_full0 + 8u * st, lane);
        };
        bool ok = true;
        int gs = 0;                        // steps stored so far (all tiles)
        uint32_t s = 0, ph = 0;            // stage of the next step, parity of its use count
        int pending = -1;                  // stage stored by the previous step, not yet published
        for (int tt = 0; tt < nt && ok; ++tt) {
        for (int ks0 = 0; ks0 < NSP && ok; ks0 += kPf) {
            // the slots refilled in this round: steps ks0 + kPf .. of this tile, or the next
            // tile's first kPf steps
            const bool wrap = ks0 + kPf == NSP;
            const int ft = wrap ? tt + 1 : tt, fp0 = wrap ? 0 : ks0 + kPf;
            const int32_t *fw = wrow + (size_t)ft * wtile + fp0 * (kKs / 8);
            const uint16_t *fsc = srow + (size_t)ft * stile + fp0 * (kKs / GS);
#pragma unroll
            for (int j = 0; j < kPf; ++j) {
                const uint4 c = cq[j];
                const uint32_t sc = sq[j];
                if (ft < nt && fp0 + j < NS) {
                    cq[j] = __ldg(reinterpret_cast<const uint4 *>(fw + j * (kKs / 8)));
                    sq[j] = __ldg(reinterpret_cast<const uint32_t *>(fsc + j * (kKs / GS)));
                }
                if (ks0 + j >= NS || !ok) continue;  // padding step (uniform over the warp)
                uint32_t s2, s2h;
                if (FMT == W4_INT4) {
                    // this slice's group scale, bf16 -> f32 -> f16 (exact in range), twice
                    const float sf = __uint_as_float(prmt(sc, 0u, (kq & 1) ? 0x3244u : 0x1044u));
                    s2 = s2h = pack_f16x2(sf, sf);
                } else {
                    // group 32: this slice's scale twice; group 16: words 0-1 the first, 2-3 the second
                    s2 = prmt(sc, sc, (FMT != W4_NV && (kq & 1)) ? 0x3232u : 0x1010u);
                    s2h = FMT == W4_NV ? prmt(sc, sc, 0x3232u) : s2;
                }
                uint32_t pairs[16];
                dequant4<FMT>(c.x, s2, pairs + 0);
                dequant4<FMT>(c.y, s2, pairs + 4);
                dequant4<FMT>(c.z, s2h, pairs + 8);
                dequant4<FMT>(c.w, s2h, pairs + 12);
                if (pending >= 0) stage_ready((uint32_t)pending);
                pending = -1;
                // the stage's previous contents have been read by the MMAs (all lanes poll once;
                // a bounded warp-wide wait only when the phase is not complete yet)
                if (gs >= kStages && !__all_sync(0xFFFFFFFFu, tc::mbar_try_wait_addr(empty0 + 8u * s, ph ^ 1u)))
                    ok = tc::mbar_wait_warp(&empty[s], ph ^ 1u, abort_flag, a.status);
                if (!ok) continue;
                tc::fence_after_sync();
                tc::tmem_st16(tst0 + s * kAStageCols, pairs);
                pending = (int)s;
                ++gs;
                if (++s == kStages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        if (pending >= 0 && ok) stage_ready((uint32_t)pending);
        pending = -1;

        // ---- epilogue of tile tt: tokens [64 kq, 64 kq + 64), chunks of 32 ----
        ok = ok && tc::mbar_wait_warp(acc_full, tt & 1, abort_flag, a.status);
        const int nrow0 = n0 + tt * 128;  // down: this tile's first output row
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        // NVFP4: the accumulator carries 2^-8 / (tensor scale) of the product
        const float gsc = FMT == W4_NV ? __ldg(a.wglobal + e) * 256.f : 1.f;
        if (GU) {
            // lane l < 16 holds gate row f, lane l + 16 the up row of the same feature: per token
            // pair one shuffle gives each its partner's value; the gate lane finishes tokens
            // 0-15 of a 32-token chunk, the up lane tokens 16-31
            if (ok) {
                tc::fence_after_sync();
                const bool is_gate = lane < 16;
                // feature f goes to column f of h with the 8-group K order 0 4 1 5 2 6 3 7
                const int j8 = lane & 7;
                uint16_t *hcol = a.h_out + n0 + tt * 64 + 16 * quarter + (lane & 8) + (j8 < 4 ? 2 * j8 : 2 * j8 - 7);
                for (int c = 0; c < kTok / kSplit / 32; ++c) {
                    const int tok0 = kq * (kTok / kSplit) + c * 32;
                    if (tok0 >= n_mma) break;
                    uint32_t v[32];
                    tc::tmem_ld32(lane_base + tok0, v);
                    tc::tmem_wait_ld();
                    uint16_t *hrow = hcol + (size_t)(r0 + tok0 + (is_gate ? 0 : 16)) * a.N;
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const uint32_t mine = is_gate ? v[m] : v[16 + m];
                        const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, is_gate ? v[16 + m] : v[m], 16);
                        const float g = gsc * __uint_as_float(is_gate ? mine : other);
                        const float u = gsc * __uint_as_float(is_gate ? other : mine);
                        // h = bf16(a); the INT4 down GEMM reads it as f16 (the same value)
                        const uint16_t hb = f32_to_bf16(silu_fast_f32(g) * u);
                        hrow[(size_t)m * a.N] =
                            FMT == W4_INT4 ? (uint16_t)(pack_f16x2(__uint_as_float((uint32_t)hb << 16), 0.f) & 0xFFFFu) : hb;
                    }
                }
            }
        } else {
            if (ok) {
                tc::fence_after_sync();
                for (int c = 0; c < kTok / kSplit / 32; ++c) {
                    const int tok0 = kq * (kTok / kSplit) + c * 32;
                    if (tok0 >= n_mma) break;
                    uint32_t y[32];
                    tc::tmem_ld32(lane_base + tok0, y);
                    tc::tmem_wait_ld();
                    const int my_slot = __ldg(a.sorted_ids + r0 + tok0 + lane);
                    // no routing weights (plain grouped GEMM): weight 1
                    const float my_w =
                        (my_slot < a.n_slots) ? (a.topk_w ? __ldg(a.topk_w + my_slot) : 1.f) * gsc : 0.f;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int slot = __shfl_sync(0xFFFFFFFFu, my_slot, j);
                        const float wt = __shfl_sync(0xFFFFFFFFu, my_w, j);
                        if (slot < a.n_slots)
                            a.ys[(size_t)slot * a.N + nrow0 + row] = f32_to_bf16(wt * __uint_as_float(y[j]));
                    }
                }
            }
        }
        // this warp has read its accumulator lanes: the next tile's MMAs may overwrite them
        tc::fence_before_sync();
        __syncwarp();
        tc::mbar_arrive_lane0(smem_addr(acc_empty), lane);
        }  // output tiles
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, kTmemCols);
}

// L2 policy for the gather's reads of x: each token's row is read once per routed slot, so keep it
// resident (the gathered rows written meanwhile are streamed out, evict-first).
__device__ __forceinline__ uint64_t l2_evict_last_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ uint4 ld_keep_v4(const uint4 *p, uint64_t pol)
{
    uint4 v;
    asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}

__device__ __forceinline__ void st_stream_v4(uint4 *p, const uint4 &v)
{
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// Gather of bf16 activation rows into aligned order (row r takes row sorted_ids[r] / k of x), each
// 8-input group in the K order of the dequantized weights (0 4 1 5 2 6 3 7), converted to f16 for
// the INT4 GEMMs (TO_F16); one warp per row, 16-byte copies. Only the rows the MMAs read are written: the real rows and the zero
// padding up to the block's real count rounded up to 16 (the MMA's N); blocks with at most
// small_rows real rows belong to the register-fed kernel, which reads x itself.
template <bool TO_F16>
__global__ void __launch_bounds__(256) gather_bf16_kernel(const uint16_t *__restrict__ x, int H, int k,
                                                          const int32_t *__restrict__ sorted_ids,
                                                          const int32_t *__restrict__ ntp, int n_slots, int cap_rows,
                                                          int small_rows, uint16_t *__restrict__ xg)
{
    const int lane = threadIdx.x & 31;
    const int rows = min(__ldg(ntp), cap_rows);
    const uint64_t keep = l2_evict_last_policy();
    for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += gridDim.x * (blockDim.x >> 5)) {
        const int slot = __ldg(sorted_ids + r);
        const bool real = slot < n_slots;
        // real rows come first in a block: a 16-row group is read iff its first row is real, and
        // the block is the register-fed kernel's iff its row small_rows is padding
        const int blk0 = r & ~(kTok - 1);
        if (!real && __ldg(sorted_ids + (r & ~15)) >= n_slots) continue;
        if (small_rows > 0 && __ldg(sorted_ids + blk0 + small_rows) >= n_slots) continue;
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)(real ? slot / k : 0) * H);
        uint4 *dst = reinterpret_cast<uint4 *>(xg + (size_t)r * H);
        // four 16-byte chunks in flight per lane (H / 8 is a multiple of 16)
        for (int i0 = lane; i0 < H / 8; i0 += 4 * 32) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + 32 * u;
                v[u] = (real && i < H / 8) ? ld_keep_v4(src + i, keep) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + 32 * u;
                // (x0 x1) (x2 x3) (x4 x5) (x6 x7) -> (x0 x4) (x1 x5) (x2 x6) (x3 x7)
                const uint4 w = v[u];
                v[u].x = prmt(w.x, w.z, 0x5410u);
                v[u].y = prmt(w.x, w.z, 0x7632u);
                v[u].z = prmt(w.y, w.w, 0x5410u);
                v[u].w = prmt(w.y, w.w, 0x7632u);
                if (TO_F16) {
                    v[u].x = bf16x2_to_f16x2(v[u].x);
                    v[u].y = bf16x2_to_f16x2(v[u].y);
                    v[u].z = bf16x2_to_f16x2(v[u].z);
                    v[u].w = bf16x2_to_f16x2(v[u].w);
                }
                if (i < H / 8) st_stream_v4(dst + i, v[u]);
            }
        }
    }
}

template <int MODE, int FMT>
int launch_mode(const W4TcArgs &a, const CUtensorMap &tm, int grid_x, int grid_y, cudaStream_t s)
{
    static std::atomic<int> smem_enabled[kMaxDevices];
    {
        const cudaError_t e = enable_smem(w4a16_tc_kernel<MODE, FMT>, (int)kSmemBytes, smem_enabled);
        if (e != cudaSuccess)
            return set_error(MOEQ_ERR_CUDA, "tcgen05 W4A16 GEMM: shared-memory attribute: %s", cudaGetErrorString(e));
    }
    if (grid_x <= 0 || grid_y <= 0) return MOEQ_OK;
    w4a16_tc_kernel<MODE, FMT><<<dim3(grid_x, grid_y), kThreads, kSmemBytes, s>>>(tm, a);
    return MOEQ_OK;
}

}  // namespace

int launch_w4a16_tc(const W4TcArgs &a_in, int mode, const uint16_t *act, int max_blocks, cudaStream_t s)
{
    CUtensorMap tm;
    const int rc = make_tmap_2d(&tm, act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a_in.M, (uint64_t)a_in.K,
                                kTok, kKs / 2);
    if (rc) return rc;
    // several output tiles per CTA share one pipeline (set-up, ring fill, weight prefetch across
    // the tile boundary)
    W4TcArgs a = a_in;
    a.tiles_per_cta = mode == TC_GATEUP ? kGateUpTilesPerCta : kDownTilesPerCta;
    const int gx = cdiv(a.N / (mode == TC_GATEUP ? 64 : 128), a.tiles_per_cta);
    if (a.fmt == W4_FP4) {
        if (mode == TC_GATEUP) return launch_mode<TC_GATEUP, W4_FP4>(a, tm, gx, max_blocks, s);
        return launch_mode<TC_DOWN, W4_FP4>(a, tm, gx, max_blocks, s);
    }
    if (a.fmt == W4_NV) {
        if (mode == TC_GATEUP) return launch_mode<TC_GATEUP, W4_NV>(a, tm, gx, max_blocks, s);
        return launch_mode<TC_DOWN, W4_NV>(a, tm, gx, max_blocks, s);
    }
    if (mode == TC_GATEUP) return launch_mode<TC_GATEUP, W4_INT4>(a, tm, gx, max_blocks, s);
    return launch_mode<TC_DOWN, W4_INT4>(a, tm, gx, max_blocks, s);
}

void launch_gather_bf16(const uint16_t *x, int H, int k, const int32_t *sorted_ids, const int32_t *ntp, int n_slots,
                        int cap_rows, int small_rows, uint16_t *xg, int num_sms, cudaStream_t s, bool to_f16)
{
    if (cap_rows <= 0) return;
    const int blocks = min(cdiv(cap_rows, 8), num_sms * 8);
    if (to_f16)
        gather_bf16_kernel<true><<<blocks, 256, 0, s>>>(x, H, k, sorted_ids, ntp, n_slots, cap_rows, small_rows, xg);
    else
        gather_bf16_kernel<false><<<blocks, 256, 0, s>>>(x, H, k, sorted_ids, ntp, n_slots, cap_rows, small_rows, xg);
}

}  // namespace moeq
