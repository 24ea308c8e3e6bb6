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
// CTA = one 128 x BN output tile, 10 warps:
//   warp 0      TMA producer: A [128 x 128 B] and B [BN x 128 B] tiles per K block, 128-byte
//               swizzle, into a 4-stage shared-memory ring (mbarrier transaction counts);
//   warp 1      allocates tensor memory; lane 0 issues 4 tcgen05.mma (K = 32 each) per K block
//               into partial buffer kb % 2 and commits to the stage's "empty" and the buffer's
//               "full" barriers;
//   warps 2-9   promotion and epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. +31
//               (= tile rows) and one half of the columns, keeps the running f32 sums in
//               registers, and finally writes bf16 C.
// Every wait is bounded; a wait that gives up flags the kernel status word and the CTA drains.
#include "kernels.cuh"
#include "tc_common.cuh"

namespace moeq {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 128;  // one scale block; bytes = elements for E4M3
constexpr int kStages = 4;
constexpr int kEpiWarps = 8;
constexpr int kThreads = (2 + kEpiWarps) * 32;

template <int BN>
struct Fp8TcShape {
    static constexpr int kABytes = kBM * kBK;
    static constexpr int kBBytes = BN * kBK;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kTmemCols = 2 * BN;  // two partial buffers (256 or 512 columns)
    static constexpr int kColsPerWarp = BN / 2;
    static constexpr size_t kSmemBytes = (size_t)kStages * kStageBytes + 1024 + 256;
};

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    fp8_tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       Fp8TcArgs a)
{
    using Sh = Fp8TcShape<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * Sh::kStageBytes);
    uint64_t *empty = full + kStages;
    uint64_t *tfull = empty + kStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *mma_done = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * kBM;  // consecutive CTAs share a B (weight) tile in L2
    const int n0 = blockIdx.y * BN;
    const int KB = a.K / kBK;

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

    if (warp == 0) {
        if (lane == 0) {
            tc::prefetch_tmap(&tmA);
            tc::prefetch_tmap(&tmB);
            int issued = 0;
            for (int kb = 0; kb < KB; ++kb) {
                const int s = kb % kStages;
                if (kb >= kStages && !tc::mbar_wait(&empty[s], ((kb / kStages) & 1) ^ 1, abort_flag, a.status)) break;
                uint8_t *sa = smem + s * Sh::kStageBytes;
                tc::mbar_arrive_expect_tx(&full[s], Sh::kStageBytes);
                tc::tma_load_2d(sa, &tmA, &full[s], kb * kBK, m0);
                tc::tma_load_2d(sa + Sh::kABytes, &tmB, &full[s], kb * kBK, n0);
                issued = kb + 1;
            }
            // no copy may still be landing in shared memory when the CTA exits
            for (int kb = issued - kStages > 0 ? issued - kStages : 0; kb < issued; ++kb)
                tc::mbar_drain(&full[kb % kStages], (kb / kStages) & 1, a.status);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_f32(tc::kFmtE4M3, tc::kFmtE4M3, kBM, BN);
            for (int kb = 0; kb < KB; ++kb) {
                const int s = kb % kStages, buf = kb & 1;
                if (!tc::mbar_wait(&full[s], (kb / kStages) & 1, abort_flag, a.status)) break;
                if (kb >= 2 && !tc::mbar_wait(&tempty[buf], ((kb >> 1) & 1) ^ 1, abort_flag, a.status)) break;
                tc::fence_after_sync();
                const uint8_t *sa = smem + s * Sh::kStageBytes;
                const uint64_t adesc = tc::smem_desc_sw128(sa);
                const uint64_t bdesc = tc::smem_desc_sw128(sa + Sh::kABytes);
#pragma unroll
                for (int kk = 0; kk < kBK / 32; ++kk)
                    tc::mma_f8f6f4_ss(tmem + buf * BN, adesc + 2 * kk, bdesc + 2 * kk, idesc, kk > 0 ? 1u : 0u);
                tc::mma_commit(&empty[s]);
                tc::mma_commit(&tfull[buf]);
            }
            // every MMA issued must finish before tensor memory is released
            tc::mma_commit(mma_done);
            tc::mbar_drain(mma_done, 0, a.status);
        }
    } else {
        constexpr int COLS = Sh::kColsPerWarp;
        const int ew = warp - 2, quarter = warp & 3, half = ew >> 2;
        const int row = quarter * 32 + lane;
        const int m = m0 + row;
        const int col0 = half * COLS;
        const float *as_row = a.As + (size_t)(m < a.M ? m : a.M - 1) * KB;
        const float *bs_row = a.Bs + (size_t)((n0 + col0) / 128) * KB;
        float acc[COLS];
#pragma unroll
        for (int j = 0; j < COLS; ++j) acc[j] = 0.f;
        bool ok = true;
        for (int kb = 0; kb < KB && ok; ++kb) {
            const int buf = kb & 1;
            const float sc = __ldg(as_row + kb) * __ldg(bs_row + kb);
            // every lane waits, then the warp agrees: the tensor-memory loads below are warp-wide
            ok = __all_sync(0xFFFFFFFFu, tc::mbar_wait(&tfull[buf], (kb >> 1) & 1, abort_flag, a.status));
            if (!ok) break;
            tc::fence_after_sync();
            const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + buf * BN + col0;
#pragma unroll
            for (int c = 0; c < COLS / 32; ++c) {
                uint32_t r[32];
                tc::tmem_ld32(taddr + c * 32, r);
                tc::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) acc[c * 32 + j] = fmaf(__uint_as_float(r[j]), sc, acc[c * 32 + j]);
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&tempty[buf]);
        }
        if (ok && m < a.M) {
            uint16_t *crow = a.C + (size_t)m * a.N + n0 + col0;
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
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, Sh::kTmemCols);
}

template <int BN>
int launch_bn(const Fp8TcArgs &a, const uint8_t *A, const uint8_t *B, cudaStream_t s)
{
    using Sh = Fp8TcShape<BN>;
    CUtensorMap tmA, tmB;
    int rc = make_tmap_2d(&tmA, A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.M, (uint64_t)a.K, kBM, kBK);
    if (rc) return rc;
    rc = make_tmap_2d(&tmB, B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.N, (uint64_t)a.K, BN, kBK);
    if (rc) return rc;
    static bool attr = false;
    if (!attr) {
        cudaFuncSetAttribute(fp8_tc_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Sh::kSmemBytes);
        attr = true;
    }
    dim3 grid(cdiv(a.M, kBM), a.N / BN);
    fp8_tc_gemm_kernel<BN><<<grid, kThreads, Sh::kSmemBytes, s>>>(tmA, tmB, a);
    return MOEQ_OK;
}

}  // namespace

int launch_fp8_tc_gemm(const Fp8TcArgs &a, const uint8_t *A, const uint8_t *B, cudaStream_t s)
{
    if (a.N % 256 == 0) return launch_bn<256>(a, A, B, s);
    return launch_bn<128>(a, A, B, s);
}

}  // namespace moeq
