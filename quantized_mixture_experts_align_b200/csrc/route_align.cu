// Routing (top-k softmax, renormalised) and token-to-expert alignment kernels.
//
// Alignment follows "vLLM x Novita AI: Chord W4A16 INT4 MoE Kernel for Kimi K2.x", sections
// "Two kernel families" (sorted_ids / expert_ids / num_tokens_padded) and figure 3 (padding
// guards live in the indices, activations are not padded). The stable within-expert order and
// the pad value T*k are this library's reading; they make the outputs bit-reproducible.
#include "common.cuh"
#include "kernels.cuh"

namespace moeq {

// ------------------------------------------------------------------------------------------
// Routing: one warp per token. Lane l holds logits l, l+32, ... in registers; k rounds of a
// warp arg-max (value descending, index ascending) pick the experts, then lane j < k turns its
// pick into exp(l_j - l_max) in double and every lane sums them in slot order.
// With local_ids (expert parallelism) the picks are also written relative to this rank's expert
// range [ep_base, ep_base + ep_local), -1 for experts held elsewhere; ids may then be null.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) route_topk_kernel(const float *__restrict__ logits, int T, int E,
                                                         int k, int32_t *__restrict__ ids,
                                                         float *__restrict__ w,
                                                         int32_t *__restrict__ local_ids, int ep_base,
                                                         int ep_local, const uint16_t *__restrict__ x, int H,
                                                         uint16_t *__restrict__ xh, int xh_f16)
{
    pdl_trigger();  // the alignment after this kernel may launch (it waits for these ids)
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    if (xh) {
        // the token's activation row for the register-fed GEMMs, each 8-input group in the
        // nibble-pair order of their weight words: (x0 x4) (x1 x5) (x2 x6) (x3 x7); in f16 for the
        // INT4 GEMMs (xh_f16; exact for magnitudes in [2^-14, 65504]), else bf16 as it is
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * H);
        uint4 *dst = reinterpret_cast<uint4 *>(xh + (size_t)t * H);
        for (int i = lane; i < H / 8; i += 32) {
            const uint4 v = __ldg(src + i);
            const uint32_t a0 = xh_f16 ? bf16x2_to_f16x2(v.x) : v.x, a1 = xh_f16 ? bf16x2_to_f16x2(v.y) : v.y;
            const uint32_t a2 = xh_f16 ? bf16x2_to_f16x2(v.z) : v.z, a3 = xh_f16 ? bf16x2_to_f16x2(v.w) : v.w;
            dst[i] = make_uint4(prmt(a0, a2, 0x5410u), prmt(a0, a2, 0x7632u), prmt(a1, a3, 0x5410u),
                                prmt(a1, a3, 0x7632u));
        }
    }
    const float *row = logits + (size_t)t * E;
    float v[kMaxExperts / 32];
#pragma unroll
    for (int i = 0; i < kMaxExperts / 32; ++i) {
        const int e = lane + 32 * i;
        v[i] = (e < E) ? __ldg(row + e) : 0.0f;
    }
    uint32_t taken = 0;
    float my_v = 0.0f;
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
        float bv = 0.0f;
        int be = 0x7FFFFFFF;
#pragma unroll
        for (int i = 0; i < kMaxExperts / 32; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((taken >> i) & 1u)) {
                if (be == 0x7FFFFFFF || v[i] > bv) { bv = v[i]; be = e; }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
            const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, off);
            const bool better = (oe != 0x7FFFFFFF) &&
                                (be == 0x7FFFFFFF || ov > bv || (ov == bv && oe < be));
            if (better) { bv = ov; be = oe; }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == j) { my_v = bv; my_e = be; }
    }
    const float vmax = __shfl_sync(0xFFFFFFFFu, my_v, 0);
    const double d = (lane < k) ? exp((double)my_v - (double)vmax) : 0.0;
    double den = 0.0;
    for (int j = 0; j < k; ++j) den += __shfl_sync(0xFFFFFFFFu, d, j);
    if (lane < k) {
        if (ids) ids[(size_t)t * k + lane] = my_e;
        if (local_ids) {
            const int le = my_e - ep_base;
            local_ids[(size_t)t * k + lane] = (le >= 0 && le < ep_local) ? le : -1;
        }
        w[(size_t)t * k + lane] = (float)(d / den);
    }
}

void launch_route_topk(const float *logits, int T, int E, int k, int32_t *ids, float *w, cudaStream_t s,
                       int32_t *local_ids, int ep_base, int ep_local, const uint16_t *x, int H, uint16_t *xh,
                       bool xh_f16)
{
    if (T <= 0) return;
    const int warps = 8;
    route_topk_kernel<<<cdiv(T, warps), warps * 32, 0, s>>>(logits, T, E, k, ids, w, local_ids, ep_base, ep_local,
                                                            x, H, xh, xh_f16 ? 1 : 0);
}

// ------------------------------------------------------------------------------------------
// Alignment: one CTA of 1024 threads.
//  1. per-expert counts (shared-memory atomics; order-free);
//  2. exclusive scan of the padded counts -> each expert's offset; expert_ids and pads written;
//  3. stable scatter in tiles of 1024 slots: a slot's position is its expert's offset + slots of
//     that expert in earlier tiles + those in earlier warps of this tile + its rank in its warp
//     (__match_any_sync peers below its lane).
// ------------------------------------------------------------------------------------------
constexpr int kAlignThreads = 1024;
constexpr int kAlignWarps = kAlignThreads / 32;

__global__ void __launch_bounds__(kAlignThreads) align_kernel(const int32_t *__restrict__ topk_ids, int n,
                                                              int E, int B, int32_t *__restrict__ sorted_ids,
                                                              int32_t *__restrict__ expert_ids,
                                                              int32_t *__restrict__ num_tokens_padded)
{
    __shared__ int cnt[kMaxExperts];
    __shared__ int off[kMaxExperts + 1];
    __shared__ int cursor[kMaxExperts];
    __shared__ uint8_t hist[kMaxExperts][kAlignWarps];  // per tile: count of expert e in warp w
    __shared__ int warp_sums[kAlignWarps];

    pdl_wait();     // launched by launch_pdl: the routing ids come from the previous kernel
    pdl_trigger();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int e = tid; e < E; e += kAlignThreads) { cnt[e] = 0; cursor[e] = 0; }
    for (int i = tid; i < kMaxExperts * kAlignWarps / 4; i += kAlignThreads)
        reinterpret_cast<uint32_t *>(&hist[0][0])[i] = 0u;
    __syncthreads();

    for (int f = tid; f < n; f += kAlignThreads) {
        const int e = topk_ids[f];
        if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
    }
    __syncthreads();

    // exclusive scan of padded counts, one expert per thread (E <= 1024)
    const int padded = (tid < E) ? (cnt[tid] + B - 1) / B * B : 0;
    int incl = padded;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int ws = warp_sums[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, ws, o);
            if (lane >= o) ws += y;
        }
        warp_sums[lane] = ws;  // inclusive over warps
    }
    __syncthreads();
    const int excl = incl - padded + (warp > 0 ? warp_sums[warp - 1] : 0);
    if (tid < E) off[tid] = excl;
    const int total = warp_sums[kAlignWarps - 1];
    if (tid == 0) { off[E] = total; *num_tokens_padded = total; }
    __syncthreads();

    // block ids and pad entries of each expert's range, then the tail past the total
    const long cap = (long)n + (long)E * (B - 1);
    const long nblk = (cap + B - 1) / B;
    if (tid < E) {
        const int c = cnt[tid];
        for (int i = excl + c; i < excl + padded; ++i) sorted_ids[i] = n;
        for (int b = excl / B; b < (excl + padded) / B; ++b) expert_ids[b] = tid;
    }
    for (long i = total + tid; i < cap; i += kAlignThreads) sorted_ids[i] = n;
    for (long b = total / B + tid; b < nblk; b += kAlignThreads) expert_ids[b] = -1;

    // stable scatter
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int base = 0; base < n; base += kAlignThreads) {
        const int f = base + tid;
        int e = (f < n) ? topk_ids[f] : -1;
        if (e < 0 || e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
        const int rank = __popc(peers & lt_mask);
        const bool leader = (peers & lt_mask) == 0u;
        if (e >= 0 && leader) hist[e][warp] = (uint8_t)__popc(peers);
        __syncthreads();
        if (e >= 0) {
            int before = 0;
            for (int w = 0; w < warp; ++w) before += hist[e][w];
            sorted_ids[off[e] + cursor[e] + before + rank] = f;
        }
        __syncthreads();
        if (e >= 0 && leader) {
            atomicAdd(&cursor[e], __popc(peers));
            hist[e][warp] = 0;
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------------------------------
// Alignment over many CTAs (large T*k), same result as align_kernel:
//  1. align_count_kernel: chunk c of kChunk slots -> its per-expert counts hist[c][e]
//     (warp-aggregated shared-memory atomics: one atomic per expert and warp);
//  2. align_scan_kernel (one CTA): per expert, the totals and the exclusive prefix over chunks;
//     the padded scan gives each expert's offset; hist[c][e] becomes the position of chunk c's
//     first slot of expert e; expert_ids, pads, tail and num_tokens_padded are written;
//  3. align_scatter_kernel: chunk c places its slots at hist[c][e] + their stable rank within
//     the chunk (tiles of 256 slots as in align_kernel).
// ------------------------------------------------------------------------------------------
constexpr int kChunkThreads = 256;
constexpr int kChunkWarps = kChunkThreads / 32;
constexpr int kChunk = 2048;  // slots per chunk (8 tiles of 256)
constexpr int kAlignOneCtaMax = 8192;  // up to this many slots the one-CTA kernel is faster

__global__ void __launch_bounds__(kChunkThreads) align_count_kernel(const int32_t *__restrict__ topk_ids, int n,
                                                                   int E, int32_t *__restrict__ hist)
{
    __shared__ int cnt[kMaxExperts];
    const int tid = threadIdx.x, lane = tid & 31;
    for (int e = tid; e < E; e += kChunkThreads) cnt[e] = 0;
    __syncthreads();
    const int f0 = blockIdx.x * kChunk;
    for (int i = tid; i < kChunk; i += kChunkThreads) {
        const int f = f0 + i;
        int e = (f < n) ? __ldg(topk_ids + f) : -1;
        if (e < 0 || e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
        if (e >= 0 && (peers & ((1u << lane) - 1u)) == 0u) atomicAdd(&cnt[e], __popc(peers));
    }
    __syncthreads();
    for (int e = tid; e < E; e += kChunkThreads) hist[(size_t)blockIdx.x * E + e] = cnt[e];
}

__global__ void __launch_bounds__(kAlignThreads) align_scan_kernel(int n, int E, int B, int n_chunks,
                                                                  int32_t *__restrict__ hist,
                                                                  int32_t *__restrict__ sorted_ids,
                                                                  int32_t *__restrict__ expert_ids,
                                                                  int32_t *__restrict__ num_tokens_padded)
{
    __shared__ int warp_sums[kAlignWarps];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int cnt = 0;
    if (tid < E)
        for (int c = 0; c < n_chunks; ++c) cnt += hist[(size_t)c * E + tid];
    const int padded = (tid < E) ? (cnt + B - 1) / B * B : 0;
    int incl = padded;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int ws = warp_sums[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, ws, o);
            if (lane >= o) ws += y;
        }
        warp_sums[lane] = ws;
    }
    __syncthreads();
    const int excl = incl - padded + (warp > 0 ? warp_sums[warp - 1] : 0);
    const int total = warp_sums[kAlignWarps - 1];
    if (tid == 0) *num_tokens_padded = total;
    const long cap = (long)n + (long)E * (B - 1);
    const long nblk = (cap + B - 1) / B;
    if (tid < E) {
        int pos = excl;  // chunk c's first slot of this expert
        for (int c = 0; c < n_chunks; ++c) {
            const int h = hist[(size_t)c * E + tid];
            hist[(size_t)c * E + tid] = pos;
            pos += h;
        }
        for (int i = excl + cnt; i < excl + padded; ++i) sorted_ids[i] = n;
        for (int b = excl / B; b < (excl + padded) / B; ++b) expert_ids[b] = tid;
    }
    for (long i = total + tid; i < cap; i += kAlignThreads) sorted_ids[i] = n;
    for (long b = total / B + tid; b < nblk; b += kAlignThreads) expert_ids[b] = -1;
}

__global__ void __launch_bounds__(kChunkThreads) align_scatter_kernel(const int32_t *__restrict__ topk_ids, int n,
                                                                     int E, const int32_t *__restrict__ base,
                                                                     int32_t *__restrict__ sorted_ids)
{
    __shared__ int cursor[kMaxExperts];
    __shared__ uint8_t hist[kMaxExperts][kChunkWarps];  // per tile: count of expert e in warp w
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int32_t *my_base = base + (size_t)blockIdx.x * E;
    for (int e = tid; e < E; e += kChunkThreads) {
        cursor[e] = __ldg(my_base + e);
#pragma unroll
        for (int w = 0; w < kChunkWarps; ++w) hist[e][w] = 0;
    }
    __syncthreads();
    const unsigned lt_mask = (1u << lane) - 1u;
    const int f0 = blockIdx.x * kChunk;
    for (int t0 = 0; t0 < kChunk; t0 += kChunkThreads) {
        const int f = f0 + t0 + tid;
        int e = (f < n) ? __ldg(topk_ids + f) : -1;
        if (e < 0 || e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
        const int rank = __popc(peers & lt_mask);
        const bool leader = (peers & lt_mask) == 0u;
        if (e >= 0 && leader) hist[e][warp] = (uint8_t)__popc(peers);
        __syncthreads();
        if (e >= 0) {
            int before = 0;
#pragma unroll
            for (int w = 0; w < kChunkWarps; ++w) before += (w < warp) ? hist[e][w] : 0;
            sorted_ids[cursor[e] + before + rank] = f;
        }
        __syncthreads();
        if (e >= 0 && leader) {
            atomicAdd(&cursor[e], __popc(peers));
            hist[e][warp] = 0;
        }
        __syncthreads();
    }
}

// Masked grouped layout: row e * max_m + r belongs to expert e when r < masked_m[e], else to none
// (-1), which the alignment skips.
__global__ void __launch_bounds__(256) masked_rows_kernel(const int32_t *__restrict__ masked_m, int G, int max_m,
                                                          int32_t *__restrict__ ids)
{
    const long total = (long)G * max_m;
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
        const int e = (int)(i / max_m);
        const int r = (int)(i - (long)e * max_m);
        ids[i] = (r < __ldg(masked_m + e)) ? e : -1;
    }
}

void launch_masked_rows(const int32_t *masked_m, int G, int max_m, int32_t *ids, int num_sms, cudaStream_t s)
{
    const long total = (long)G * max_m;
    if (total <= 0) return;
    const int blocks = (int)((total + 255) / 256 < (long)num_sms * 4 ? (total + 255) / 256 : (long)num_sms * 4);
    masked_rows_kernel<<<blocks, 256, 0, s>>>(masked_m, G, max_m, ids);
}

size_t align_scratch_bytes(int n, int E)
{
    return n > kAlignOneCtaMax ? (size_t)cdiv(n, kChunk) * E * sizeof(int32_t) : 0;
}

void launch_align(const int32_t *topk_ids, int n, int E, int B, int32_t *sorted_ids, int32_t *expert_ids,
                  int32_t *ntp, int32_t *scratch, cudaStream_t s)
{
    if (n > kAlignOneCtaMax && scratch) {
        const int chunks = cdiv(n, kChunk);
        align_count_kernel<<<chunks, kChunkThreads, 0, s>>>(topk_ids, n, E, scratch);
        align_scan_kernel<<<1, kAlignThreads, 0, s>>>(n, E, B, chunks, scratch, sorted_ids, expert_ids, ntp);
        align_scatter_kernel<<<chunks, kChunkThreads, 0, s>>>(topk_ids, n, E, scratch, sorted_ids);
        return;
    }
    launch_pdl(align_kernel, dim3(1), dim3(kAlignThreads), 0, s, topk_ids, n, E, B, sorted_ids, expert_ids, ntp);
}

// ------------------------------------------------------------------------------------------
// Top-k weighted combine: out[t, :] = bf16( sum_j ys[t*k + j, :] ), the slot rows (bf16) already
// carrying their routing weight. f32 sums in slot order. With local_ids (expert parallelism) the
// slots routed to experts of other ranks (-1) are left out: their rows of ys are never written.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t *__restrict__ ys, int T, int k, int H,
                                                      const int32_t *__restrict__ local_ids,
                                                      uint16_t *__restrict__ out)
{
    pdl_wait();     // launched by launch_pdl: ys comes from the previous kernel
    const int H8 = H / 8;
    const long total = (long)T * H8;
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
        const long t = i / H8;
        const int c = (int)(i - t * H8);
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const uint16_t *row0 = ys + (size_t)t * k * H;
        // up to 8 slot rows in flight per thread (the rows are read once: no L1 allocation), then
        // summed in slot order
        for (int j0 = 0; j0 < k; j0 += 8) {
            uint4 v[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int j = j0 + jj;
                const bool use = j < k && !(local_ids && __ldg(local_ids + (size_t)t * k + j) < 0);
                v[jj] = use ? ld_stream_v4(reinterpret_cast<const uint4 *>(row0 + (size_t)j * H) + c)
                            : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const uint32_t w[4] = {v[jj].x, v[jj].y, v[jj].z, v[jj].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc[2 * q] += __uint_as_float(w[q] << 16);
                    acc[2 * q + 1] += __uint_as_float(w[q] & 0xFFFF0000u);
                }
            }
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        reinterpret_cast<uint4 *>(out + (size_t)t * H)[c] = o;
    }
}

void launch_combine(const uint16_t *ys, int T, int k, int H, uint16_t *out, int num_sms, cudaStream_t s,
                    const int32_t *local_ids)
{
    if (T <= 0) return;
    const long total = (long)T * (H / 8);
    const int blocks = (int)((total + 255) / 256 < (long)num_sms * 8 ? (total + 255) / 256 : (long)num_sms * 8);
    launch_pdl(combine_kernel, dim3(blocks), dim3(256), 0, s, ys, T, k, H, local_ids, out);
}

}  // namespace moeq
