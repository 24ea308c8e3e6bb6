// Dense FP8 GEMM for few activation rows (block scales: M <= 32; channelwise: M <= 64) on the
// 5th-generation tensor cores.
//
// "SGLang W8A8 Block FP8 quantized kernel config files", section "Background", defines
//   C[m, n] = sum over 128-wide K blocks kb of As[m, kb] * Bs[n/128, kb] * (A_q[m, kb] . B_q[n, kb]).
// With few rows the weight matrix B [N, K] is streamed from HBM once and dominates the bytes, so
// the layout is turned around (swap-AB): 128 weight rows (one scale block) are the MMA's M side
// and the M activation rows, padded to MP in {16, 32, 64}, are its N side. A tile is then
// 128 output columns for all rows, and one K block is 16 KB of weights and 4 small MMAs.
// 24576 / 128 = 192 tiles do not fill 148 SMs evenly, so K is split over a thread-block cluster
// of S CTAs; each CTA promotes its K blocks into registers and the S partial tiles are summed
// through distributed shared memory (no workspace, no second launch).
//
// CTA = 128 weight rows x MP rows x K/S, 2 + EW warps (NC CTAs per SM). The pipeline moves G
// K blocks per step:
//   warp 0        TMA producer: per K block a weight tile [128 x 128 B] and an activation tile
//                 [MP x 128 B], 128-byte swizzle, into a shared-memory ring of steps;
//   warp 1        allocates tensor memory; lane 0 issues 4 tcgen05.mma (K = 32) per K block into
//                 its MP columns of partial buffer step % 2 and commits once per step to the
//                 stage's "empty" and the buffer's "full" barriers;
//   warps 2..     promotion: warp w reads tensor-memory lanes 32 (w % 4) .. +31 (weight rows)
//                 and a slice of the MP columns; acc += partial * As[m, kb] * Bs[n/128, kb],
//                 with the products of the two scales staged in shared memory per K block.
// Then every CTA stores its partial tile in shared memory, the cluster synchronizes, and rank r
// sums columns [128 r / S, 128 (r + 1) / S) of all S tiles in rank order and writes bf16 C.
// Every wait is bounded; a wait that gives up flags the kernel status word and the CTA drains.
#include "kernels.cuh"
#include "tc_common.cuh"

namespace moeq {

namespace {

constexpr int kRows = 128;     // weight rows per tile = one weight scale block
constexpr int kBK = 128;       // K block (E4M3: bytes = elements)
constexpr int kWBytes = kRows * kBK;

// MP padded rows; G K blocks per pipeline step (one wait, one MMA batch, one commit and one
// promotion pass per step: the hand-offs between the roles, not the bytes, set the time of a
// step); NC CTAs share an SM (1, 2 or 3: the ring is sized so that their shared memory fits);
// CW: channelwise scales (per token, per channel), the CTA's whole K range accumulated in one
// buffer and scaled once.
template <int MP, int G, int NC, bool CW>
struct SkinnyShape {
    static constexpr int kEpiWarps = MP <= 64 ? 4 : 8;        // <= 64 accumulators per thread
    static constexpr int kThreads = (2 + kEpiWarps) * 32;
    static constexpr int kCols = MP / (kEpiWarps / 4);        // columns per promotion warp
    static constexpr int kKbBytes = kWBytes + MP * kBK;       // one K block: weights + activations
    static constexpr int kStageBytes = G * kKbBytes;          // multiple of 1024 (MP >= 16)
    static constexpr int kRing = NC == 1 ? 200 * 1024 : NC == 2 ? 104 * 1024 : 64 * 1024;
    static constexpr int kStages = kRing / kStageBytes;
    static constexpr int kBufCols = CW ? MP : G * MP;         // one partial buffer: G blocks
    static constexpr int kTmemCols = 2 * kBufCols < 32 ? 32 : 2 * kBufCols;
    static_assert(kStages >= 2, "at least two pipeline stages");
    static_assert(NC >= 1 && NC <= 3, "one to three CTAs per SM");
    static_assert(kTmemCols * NC <= 512, "tensor memory of the CTAs on one SM");
    static_assert(kStages * kStageBytes >= MP * kRows * 4, "partial tile must fit in the ring");
    static_assert(kKbBytes % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
    // shared memory one CTA may take when NC of them share the SM's 228 KB (1 KB each reserved)
    static constexpr size_t kSmemCap = (NC == 1 ? 227 : 228 / NC - 1) * 1024;
    static constexpr size_t smem_bytes(int nkb_max)
    {
        return 1024 + (size_t)kStages * kStageBytes + (size_t)nkb_max * MP * 4 + (2 * kStages + 5) * 8 + 16;
    }
};

__device__ __forceinline__ float4 ld_cluster_f32x4(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

template <int MP, int G, int NC, bool CW>
__global__ void __launch_bounds__(SkinnyShape<MP, G, NC, CW>::kThreads, NC)
    fp8_tc_skinny_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                         Fp8TcArgs a, int split)
{
    using Sh = SkinnyShape<MP, G, NC, CW>;
    constexpr int kStages = Sh::kStages, kEpiWarps = Sh::kEpiWarps, COLS = Sh::kCols;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int KB = a.K / kBK;
    const int rank = (int)tc::cluster_rank();
    const int kb0 = rank * KB / split, kb1 = (rank + 1) * KB / split, nkb = kb1 - kb0;
    const int nkb_max = (KB + split - 1) / split;
    const int nstep = (nkb + G - 1) / G;  // the last step may hold fewer than G blocks
    const int n0 = blockIdx.y * kRows;

    float *sct = reinterpret_cast<float *>(smem + kStages * Sh::kStageBytes);  // [nkb][MP]: As * Bs
    uint64_t *full = reinterpret_cast<uint64_t *>(sct + (size_t)nkb_max * MP);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *mma_done = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&tfull[b], 1);
            tc::mbar_init(&tempty[b], kEpiWarps);
        }
        tc::mbar_init(mma_done, 1);
        *abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) tc::tmem_alloc(tmem_slot, Sh::kTmemCols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    float acc[COLS];
#pragma unroll
    for (int j = 0; j < COLS; ++j) acc[j] = 0.f;
    const int quarter = warp & 3, cq = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;  // weight row within the tile (promotion warps)

    if (warp == 0) {
        if (lane == 0) {
            tc::prefetch_tmap(&tmW);
            tc::prefetch_tmap(&tmX);
            int issued = 0;
            for (int i = 0; i < nstep; ++i) {
                const int s = i % kStages, ng = min(G, nkb - i * G);
                if (i >= kStages && !tc::mbar_wait(&empty[s], ((i / kStages) & 1) ^ 1, abort_flag, a.status)) break;
                uint8_t *st = smem + s * Sh::kStageBytes;
                tc::mbar_arrive_expect_tx(&full[s], ng * Sh::kKbBytes);
                for (int g = 0; g < ng; ++g) {
                    const int x = (kb0 + i * G + g) * kBK;
                    tc::tma_load_2d(st + g * Sh::kKbBytes, &tmW, &full[s], x, n0);
                    tc::tma_load_2d(st + g * Sh::kKbBytes + kWBytes, &tmX, &full[s], x, 0);
                }
                issued = i + 1;
            }
            for (int i = issued - kStages > 0 ? issued - kStages : 0; i < issued; ++i)
                tc::mbar_drain(&full[i % kStages], (i / kStages) & 1, a.status);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_f32(tc::kFmtE4M3, tc::kFmtE4M3, kRows, MP);
            const uint64_t base = tc::smem_desc_sw128(smem);
            for (int i = 0; i < nstep; ++i) {
                const int s = i % kStages, buf = i & 1, ng = min(G, nkb - i * G);
                if (!tc::mbar_wait(&full[s], (i / kStages) & 1, abort_flag, a.status)) break;
                if (!CW && i >= 2 && !tc::mbar_wait(&tempty[buf], ((i >> 1) & 1) ^ 1, abort_flag, a.status)) break;
                tc::fence_after_sync();
                for (int g = 0; g < ng; ++g) {
                    // block g of the step: its own MP columns of the partial buffer (channelwise:
                    // all blocks into one accumulator, started by the very first MMA)
                    const uint64_t wdesc = base + (uint64_t)((s * Sh::kStageBytes + g * Sh::kKbBytes) >> 4);
                    const uint64_t xdesc = wdesc + (uint64_t)(kWBytes >> 4);
                    const uint32_t d = CW ? tmem : tmem + buf * Sh::kBufCols + g * MP;
                    tc::mma_f8f6f4_ss(d, wdesc, xdesc, idesc, (CW && (i > 0 || g > 0)) ? 1u : 0u);
#pragma unroll
                    for (int kk = 1; kk < kBK / 32; ++kk)
                        tc::mma_f8f6f4_ss_acc(d, wdesc + 2 * kk, xdesc + 2 * kk, idesc);
                }
                tc::mma_commit(&empty[s]);
                if (!CW) tc::mma_commit(&tfull[buf]);
            }
            if (CW) tc::mma_commit(&tfull[0]);
            tc::mma_commit(mma_done);
            tc::mbar_drain(mma_done, 0, a.status);
        }
    } else if (CW) {
        // one wait for the accumulated K range; acc = partial * As[m] * Bs[n0 + row] (padding
        // rows m >= M get 0)
        if (tc::mbar_wait_warp(&tfull[0], 0, abort_flag, a.status)) {
            tc::fence_after_sync();
            const float sb = __ldg(a.b_scale + n0 + row);
            const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + cq * COLS;
#pragma unroll
            for (int c = 0; c < COLS / 16; ++c) {
                uint32_t r[16];
                tc::tmem_ld16(taddr + c * 16, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int m = cq * COLS + c * 16 + j;
                    acc[c * 16 + j] = m < a.M ? __uint_as_float(r[j]) * __ldg(a.a_scale + m) * sb : 0.f;
                }
            }
        }
    } else {
        // scale products of this CTA's K blocks: sct[i][m] = As[m, kb0 + i] * Bs[n0 / 128, kb0 + i]
        // (0 for padding rows m >= M)
        const float *bs = a.b_scale + (size_t)(n0 / kRows) * KB + kb0;
        for (int idx = threadIdx.x - 64; idx < nkb * MP; idx += kEpiWarps * 32) {
            const int i = idx / MP, m = idx - i * MP;
            sct[idx] = m < a.M ? __ldg(a.a_scale + (size_t)m * KB + kb0 + i) * __ldg(bs + i) : 0.f;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
        for (int i = 0; i < nstep; ++i) {
            const int buf = i & 1, ng = min(G, nkb - i * G);
            if (!tc::mbar_wait_warp(&tfull[buf], (i >> 1) & 1, abort_flag, a.status)) break;
            tc::fence_after_sync();
            for (int g = 0; g < ng; ++g) {
                const uint32_t taddr =
                    tmem + ((uint32_t)(quarter * 32) << 16) + buf * Sh::kBufCols + g * MP + cq * COLS;
                const float *sc = sct + (i * G + g) * MP + cq * COLS;
#pragma unroll
                for (int c = 0; c < COLS / 16; ++c) {
                    uint32_t r[16];
                    tc::tmem_ld16(taddr + c * 16, r);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; j += 4) {
                        const float4 s4 = *reinterpret_cast<const float4 *>(sc + c * 16 + j);
                        acc[c * 16 + j] = fmaf(__uint_as_float(r[j]), s4.x, acc[c * 16 + j]);
                        acc[c * 16 + j + 1] = fmaf(__uint_as_float(r[j + 1]), s4.y, acc[c * 16 + j + 1]);
                        acc[c * 16 + j + 2] = fmaf(__uint_as_float(r[j + 2]), s4.z, acc[c * 16 + j + 2]);
                        acc[c * 16 + j + 3] = fmaf(__uint_as_float(r[j + 3]), s4.w, acc[c * 16 + j + 3]);
                    }
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&tempty[buf]);
        }
    }
    // copies and MMAs are drained: the ring is free for the partial tile red[m][row]
    tc::fence_before_sync();
    __syncwarp();
    __syncthreads();
    float *red = reinterpret_cast<float *>(smem);
    if (warp >= 2) {
#pragma unroll
        for (int j = 0; j < COLS; ++j)
            if (cq * COLS + j < a.M) red[(cq * COLS + j) * kRows + row] = acc[j];
    }
    tc::cluster_sync();
    // rank r: output columns [n_lo, n_hi) of the tile (multiples of 4), rows m < M
    {
        const int n_lo = (rank * (kRows / 4) / split) * 4, n_hi = ((rank + 1) * (kRows / 4) / split) * 4;
        const int per_row = (n_hi - n_lo) / 4;
        const int m_end = a.M < MP ? a.M : MP;
        for (int u = threadIdx.x; u < m_end * per_row; u += Sh::kThreads) {
            const int m = u / per_row, n = n_lo + (u - m * per_row) * 4;
            const float *src = red + m * kRows + n;
            float4 t = ld_cluster_f32x4(tc::cluster_addr(src, 0));
            for (int q = 1; q < split; ++q) {
                const float4 v = ld_cluster_f32x4(tc::cluster_addr(src, (uint32_t)q));
                t.x += v.x;
                t.y += v.y;
                t.z += v.z;
                t.w += v.w;
            }
            uint2 o;
            o.x = pack_bf16x2(t.x, t.y);
            o.y = pack_bf16x2(t.z, t.w);
            *reinterpret_cast<uint2 *>(a.C + (size_t)m * a.N + n0 + n) = o;
        }
    }
    tc::fence_before_sync();
    tc::cluster_sync();  // no CTA leaves while another still reads its partial tile
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, Sh::kTmemCols);
}

template <int MP, int G, int NC, bool CW>
int launch_skinny(const Fp8TcArgs &a, const uint8_t *A, const uint8_t *B, int split, cudaStream_t s)
{
    using Sh = SkinnyShape<MP, G, NC, CW>;
    const int KB = a.K / kBK;
    // the per-block scale table grows with K / split: more CTAs per tile for very deep K
    while (Sh::smem_bytes((KB + split - 1) / split) > Sh::kSmemCap && split < 8 && split < KB) ++split;
    const size_t smem = Sh::smem_bytes((KB + split - 1) / split);
    if (smem > 227 * 1024)
        return set_error(MOEQ_ERR_UNSUPPORTED, "tcgen05 FP8 skinny GEMM: K = %d needs %zu bytes of shared memory",
                         a.K, smem);
    static std::atomic<int> smem_enabled[kMaxDevices];
    {
        const cudaError_t e = enable_smem(fp8_tc_skinny_kernel<MP, G, NC, CW>, (int)smem, smem_enabled);
        if (e != cudaSuccess)
            return set_error(MOEQ_ERR_CUDA, "tcgen05 FP8 skinny GEMM: shared-memory attribute: %s",
                             cudaGetErrorString(e));
    }
    CUtensorMap tmW, tmX;
    int rc = make_tmap_2d(&tmW, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.N, (uint64_t)a.K, kRows, kBK);
    if (rc) return rc;
    rc = make_tmap_2d(&tmX, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.M, (uint64_t)a.K, MP, kBK);
    if (rc) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(split, a.N / kRows);
    cfg.blockDim = dim3(Sh::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = split;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, fp8_tc_skinny_kernel<MP, G, NC, CW>, tmW, tmX, a, split);
    if (e != cudaSuccess) return set_error(MOEQ_ERR_CUDA, "tcgen05 FP8 skinny GEMM launch: %s", cudaGetErrorString(e));
    return MOEQ_OK;
}

}  // namespace

// Up to 32 rows the block-scaled GEMM streams the weights faster through this kernel; from 33 rows
// the 128-row tile kernel (one wave of 128 x 256 tiles for N = 24576) is as fast or faster:
// 24576 x 7168 weights at 33-64 rows 41.0 us there against 46.6 us here (L2 flushed, alternating
// runs). The channelwise GEMM keeps this kernel up to 64 rows.
int fp8_skinny_max_rows(bool channelwise) { return channelwise ? 64 : 32; }

int launch_fp8_tc_skinny(const Fp8TcArgs &a, const uint8_t *A, const uint8_t *B, int split, bool channelwise,
                         cudaStream_t s)
{
    const int KB = a.K / kBK;
    if (a.M < 1 || a.M > fp8_skinny_max_rows(channelwise) || a.N % kRows || a.K % kBK)
        return set_error(MOEQ_ERR_UNSUPPORTED, "tcgen05 FP8 skinny GEMM: M = %d, N = %d, K = %d", a.M, a.N, a.K);
    if (split < 1) split = 1;
    if (split > 8) split = 8;  // portable cluster size
    if (split > KB) split = KB;
    // two K blocks per step and two CTAs per SM, except block scales at 17-32 rows: one K block per
    // step and three CTAs per SM (with a K split of 2 every CTA of 24576 / 128 tiles is resident:
    // 38.2-38.9 us against 41.0 at 32 rows; at 16 rows both forms measured 36.9 us; the
    // channelwise GEMM keeps the two-block form it was measured with)
    if (channelwise) {
        if (a.M <= 16) return launch_skinny<16, 2, 2, true>(a, A, B, split, s);
        if (a.M <= 32) return launch_skinny<32, 2, 2, true>(a, A, B, split, s);
        return launch_skinny<64, 2, 2, true>(a, A, B, split, s);
    }
    if (a.M <= 16) return launch_skinny<16, 2, 2, false>(a, A, B, split, s);
    return launch_skinny<32, 1, 3, false>(a, A, B, split, s);
}

}  // namespace moeq
