// Shared device helpers of the moeq CUDA library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "moeq.h"

namespace moeq {

constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 32;

__host__ __device__ inline int cdiv(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ inline size_t cdivz(size_t a, size_t b) { return (a + b - 1) / b; }
__host__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ---- error reporting (host) -------------------------------------------------------------
int set_error(int code, const char *fmt, ...);
int check_launch(const char *what);

// ---- dynamic shared memory above the default limit (host) ----------------------------------
// Enabled per kernel and per device (each device's context holds its own copy of the kernel).
// `enabled` remembers, per device, the largest size set so far; the entries are atomics because
// the launchers' tables are shared by every host thread, and setting the attribute twice from
// two threads is harmless.
constexpr int kMaxDevices = 64;
template <typename F>
inline cudaError_t enable_smem(F kernel, int bytes, std::atomic<int> (&enabled)[kMaxDevices])
{
    int dev = 0;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool tracked = dev >= 0 && dev < kMaxDevices;
    if (tracked && enabled[dev].load(std::memory_order_relaxed) >= bytes) return cudaSuccess;
    const cudaError_t r = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (r == cudaSuccess && tracked) enabled[dev].store(bytes, std::memory_order_relaxed);
    return r;
}

// ---- programmatic dependent launch ----------------------------------------------------------
// A kernel launched by launch_pdl may start while the previous kernel in its stream still runs.
// pdl_wait() blocks until that kernel has completed and its writes are visible (it returns at
// once in a kernel launched the ordinary way); every read of data the previous kernels wrote
// must come after it. pdl_trigger() lets the next kernel, if launched by launch_pdl, start once
// every CTA of this grid has triggered or exited (all of them resident, so none can starve).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---- bf16 / fp32 bit helpers ----------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// f32 -> bf16 bits, round to nearest even (finite inputs).
__device__ __forceinline__ uint16_t f32_to_bf16(float f)
{
    uint32_t u;
    asm("{ .reg .b16 h; cvt.rn.bf16.f32 h, %1; mov.b32 %0, {h, h}; }" : "=r"(u) : "f"(f));
    return (uint16_t)(u & 0xFFFFu);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t u;
    asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(u) : "f"(lo), "f"(hi));
    return u;
}

// Two f32 -> two E4M3 codes (nearest even, saturating to +-448), lo in bits [0,8).
__device__ __forceinline__ uint16_t pack_e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t orv)
{
    // (a & mask) | orv in one LOP3
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(orv));
    return r;
}

// E2M1 codes of nibbles P and P + 4 of a code word as bf16x2 holding 2^-126 times their values:
// the sign goes to bit 15 (31) and the 2 exponent + 1 mantissa bits to bits [8:6] ([24:22]), so the
// E2M1 exponent lands in the low bits of the bf16 exponent field and its subnormal (exponent 0,
// value 0.5) on the bf16 subnormal 2^-127. One bf16 multiply by a group factor 2^(s - 1) then
// gives value * 2^(s - 127) exactly.
template <int P>
__device__ __forceinline__ uint32_t e2m1_pair_pre(uint32_t w)
{
    const uint32_t mag = (P < 2 ? (w << (6 - 4 * P)) : (w >> (4 * P - 6))) & 0x01C001C0u;
    return lop3_and_or(w << (12 - 4 * P), 0x80008000u, mag);
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t f16x2_sub(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t f16x2_fma(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

// Unsigned INT4 nibble pairs of a code word minus the zero point 8, as exact f16x2 values
// (q - 8 in [-8, 7]): pair i holds nibbles i and i + 4. Nibbles 0 and 4 (2, 6 after a shift by 8)
// are ORed into the mantissa of 1024 (f16 1024 + q) and take 1032 off; nibbles 1 and 5 (3, 7)
// are masked in place, giving 1024 + 16 q, and one FMA by 1/16 minus 72 yields q - 8, saving their
// shift. Every intermediate is an integer or a power-of-two fraction that f16 holds exactly.
__device__ __forceinline__ void int4_pairs_minus8(uint32_t w, uint32_t (&p)[4])
{
    const uint32_t w8 = w >> 8;
    p[0] = f16x2_sub(lop3_and_or(w, 0x000F000Fu, 0x64006400u), 0x64086408u);
    p[1] = f16x2_fma(lop3_and_or(w, 0x00F000F0u, 0x64006400u), 0x2C002C00u, 0xD480D480u);  // x/16 - 72
    p[2] = f16x2_sub(lop3_and_or(w8, 0x000F000Fu, 0x64006400u), 0x64086408u);
    p[3] = f16x2_fma(lop3_and_or(w8, 0x00F000F0u, 0x64006400u), 0x2C002C00u, 0xD480D480u);
}

__device__ __forceinline__ uint32_t f16x2_mul(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Two f32 -> f16x2 (nearest even), lo in bits [0,16).
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi)
{
    uint32_t u;
    asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(u) : "f"(lo), "f"(hi));
    return u;
}

// bf16x2 -> f16x2: exact for magnitudes in [2^-14, 65504] (8 significant bits fit the f16
// significand); smaller ones round into the f16 subnormals (absolute error at most 2^-25).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) { return pack_f16x2(bf16_lo(v), bf16_hi(v)); }

// h = bf16(v) (nearest even), returned as the f16 bits of that value (exact in the f16 range).
__device__ __forceinline__ uint16_t f32_to_bf16_as_f16(float v)
{
    return (uint16_t)(pack_f16x2(__uint_as_float((uint32_t)f32_to_bf16(v) << 16), 0.f) & 0xFFFFu);
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// ---- loads ---------------------------------------------------------------------------------
// Streamed once per CTA: read-only path, no L1 allocation.
__device__ __forceinline__ uint4 ld_stream_v4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ld_v4(const void *p)
{
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// An ordinary (coherent) 16-byte load: for data an earlier kernel of a programmatic-launch chain
// writes, which must not be read ahead of the wait for that kernel (as __ldg may be scheduled).
__device__ __forceinline__ uint4 ld_v4_coherent(const void *p) { return *reinterpret_cast<const uint4 *>(p); }

// ---- tensor-core MMA (warp-level, register operands) ----------------------------------------
// D[16x8] += A[16x16] (bf16, row) * B[16x8] (bf16, col), f32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D[16x8] += A[16x16] (f16, row) * B[16x8] (f16, col), f32 accumulate.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D[16x8] = A[16x32] (e4m3, row) * B[32x8] (e4m3, col) + C, f32.
__device__ __forceinline__ void mma_e4m3_16832(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float silu_f32(float g) { return g / (1.0f + expf(-g)); }
// The same with the fast exponential and division (relative error a few f32 ulp, far below the
// bf16 rounding of h = bf16(silu(g) * u) in the 4-bit tensor-core GEMM); e^-g overflowing to +inf
// gives -0.
__device__ __forceinline__ float silu_fast_f32(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

}  // namespace moeq

namespace moeq {

// ---- asynchronous global -> shared copies (per-thread, 16 / 8 bytes) -----------------------
__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16 bytes, bypassing L1, with a 256-byte L2 prefetch of the source line
__device__ __forceinline__ void cp_async16_stream(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async8(void *dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}

// 4 bytes (4-byte aligned source and destination)
__device__ __forceinline__ void cp_async4_ca(void *dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

}  // namespace moeq
