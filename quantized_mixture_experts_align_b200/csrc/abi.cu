// C ABI of libmoeq.so: argument validation, workspace layout, schedule choice and the launch
// sequence of each entry point. Declarations and contracts are in include/moeq.h.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <chrono>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.cuh"
#include "tc_common.cuh"

#define MOEQ_VERSION "moeq 0.1 (sm_100a)"

namespace moeq {

static thread_local char g_err[512] = "";

int set_error(int code, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

int check_launch(const char *what)
{
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(MOEQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return MOEQ_OK;
}

// SM count of the current device, looked up once per device.
static int num_sms()
{
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cache[dev] = n > 0 ? n : 148;
    }
    return cache[dev];
}

// ---- stage tracing (diagnostic, off by default) ---------------------------------------------
// When enabled, each kernel stage of a call is bracketed by a CUDA event pair recorded on the
// call's stream; moe_trace_read() waits for the recorded pairs and accumulates their durations.
namespace trace {
enum { ROUTE = 0, ALIGN, ACT_QUANT, GATE_UP, DOWN, COMBINE, DENSE, GATHER, FEW_ROWS, NSTAGE };
struct Rec {
    cudaEvent_t a, b;
    int stage;
};
static std::mutex mu;
static bool enabled = false;
static std::vector<Rec> pending;
static std::vector<cudaEvent_t> spare;
static double sum_ms[NSTAGE];
static long long calls[NSTAGE];
constexpr size_t kMaxPending = 1 << 16;

static cudaEvent_t take_event()
{
    if (!spare.empty()) {
        cudaEvent_t e = spare.back();
        spare.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

struct Scope {
    Rec r{nullptr, nullptr, 0};
    cudaStream_t s;
    bool on = false;
    Scope(int stage, cudaStream_t st) : s(st)
    {
        std::lock_guard<std::mutex> g(mu);
        if (!enabled || pending.size() >= kMaxPending) return;
        r.a = take_event();
        r.b = take_event();
        r.stage = stage;
        on = r.a && r.b && cudaEventRecord(r.a, s) == cudaSuccess;
    }
    ~Scope()
    {
        if (!on) return;
        std::lock_guard<std::mutex> g(mu);
        if (cudaEventRecord(r.b, s) == cudaSuccess) pending.push_back(r);
    }
};
}  // namespace trace

// ---- host submit time ------------------------------------------------------------------------
// Wall time each entry point spends on the host (validation, workspace carving, schedule choice,
// tensor maps, launches), summed per library; read with moe_host_stats.
namespace host_time {
static std::atomic<long long> ns{0}, calls{0};
struct Scope {
    std::chrono::steady_clock::time_point t0 = std::chrono::steady_clock::now();
    ~Scope()
    {
        const auto d = std::chrono::steady_clock::now() - t0;
        ns.fetch_add((long long)std::chrono::duration_cast<std::chrono::nanoseconds>(d).count(), std::memory_order_relaxed);
        calls.fetch_add(1, std::memory_order_relaxed);
    }
};
}  // namespace host_time

// ---- schedule --------------------------------------------------------------------------------
// The routed rows per expert (tok_e = T*k/E), not the token count, decides the tile ("vLLM x
// Novita AI: Chord W4A16 INT4 MoE Kernel for Kimi K2.x", sections "Summary" and "H200 prefill
// and TP8": block-M chosen from tokens per expert). Without a host read of the routing, the
// mean tok_e picks block_m: decode shapes get block-M 8 (the page's decode profile).
static int pick_block_m(long T, int k, int E)
{
    const double tok_e = (double)T * k / (double)E;
    if (tok_e <= 2.0) return 8;
    if (tok_e <= 8.0) return 16;
    if (tok_e <= 24.0) return 32;
    return 64;
}

// K split of the few-row dense FP8 GEMM (swap-AB tcgen05 tiles, used up to
// fp8_skinny_max_rows(channelwise) rows; cluster size): the smallest power of two that gives every
// SM one CTA, or two where the CTAs are light enough to share an SM (16 padded rows; 32 with
// block scales, whose CTAs there run three to an SM), at most 8. Measured on 24576 x 7168
// weights: 16 rows 36.9 us with split 2 vs 38.9 with 1; block scales at 32 rows 38.2-38.9 us with
// split 2 (three CTAs per SM) vs 41.0 with 1. The two-CTA form that the channelwise GEMM keeps
// took 41.0 / 46.6 us at 32 / 64 rows with split 1 vs 45.1 / 55.3 with 2 (block scales).
static int pick_skinny_split(int M, int N, int K, bool channelwise)
{
    (void)K;
    const int tiles = N / 128;
    const int want = (M <= 16 || (!channelwise && M <= 32) ? 2 : 1) * 148;
    int split = 1;
    while (split < 8 && tiles * split < want) split *= 2;
    return split;
}

// ---- workspace ---------------------------------------------------------------------------------
struct Carve {
    char *base;
    size_t used = 0;
    explicit Carve(void *p) : base(static_cast<char *>(p)) {}
    template <class Tp>
    Tp *take(size_t count)
    {
        Tp *p = base ? reinterpret_cast<Tp *>(base + used) : nullptr;
        used += align256(count * sizeof(Tp));
        return p;
    }
};

struct RouteBufs {
    int32_t *ids;
    float *w;
    int32_t *sorted;
    int32_t *eids;
    int32_t *ntp;
    int32_t *scratch;  // per-chunk expert counts of the many-CTA alignment (null: one-CTA kernel)
    int block_m;
    int max_blocks;
};

static RouteBufs carve_route(Carve &c, long T, int k, int E, int block_m)
{
    RouteBufs r;
    const size_t n = (size_t)T * k;
    const size_t cap = n + (size_t)E * (block_m - 1);
    r.block_m = block_m;
    r.max_blocks = (int)cdivz(cap, block_m);
    r.ids = c.take<int32_t>(n);
    r.w = c.take<float>(n);
    r.sorted = c.take<int32_t>(cap);
    r.eids = c.take<int32_t>((size_t)r.max_blocks);
    r.ntp = c.take<int32_t>(1);
    const size_t sb = align_scratch_bytes((int)n, E);
    r.scratch = sb ? c.take<int32_t>(sb / sizeof(int32_t)) : nullptr;
    return r;
}

// W4A16 layer schedule: from this many routed rows per expert on (mean T*k/E), the grouped GEMMs
// run on the tensor-core kernels over 256-row expert blocks (weights dequantized into tensor
// memory); below, the register-fed swap-AB kernels stream the weights for the few rows each
// expert has (HBM bound).
static bool w4_use_tc(long T, int k, int E) { return (double)T * k / (double)E >= 16.0; }

// Within the tensor-core schedule, expert blocks with at most this many real rows (the tail of a
// skewed routing) run on the register-fed kernel: a tcgen05 block dequantizes its whole weight
// tile whatever its row count, while the register-fed kernel streams the weights once at HBM rate.
// Measured on the Zipf prefill (T=8192, E=384): 8 rows beat 16, 32 and 64 (at 64 rows per block
// the legacy mma.sync rate, not the weight stream, bounds the register-fed kernel).
constexpr int kW4SmallRows = 8;
static_assert(kW4SmallRows == 8, "the strided register-fed instantiation is built for 8-row tiles");

// E: experts whose weights the call holds (the alignment's capacity); E_sched (0: E): experts the
// routing picks from, whose mean load T*k/E_sched picks the schedule (under expert parallelism a
// rank holds E of the E_sched experts, and each of them still sees T*k/E_sched rows on average).
// The register-fed (decode) schedule also holds a copy of x in nibble-pair order (xh: f16 for
// INT4, whose GEMMs compute in f16; bf16 for MXFP4 / NVFP4), written by the routing kernel.
// (fmt is kept for callers; the layout is the same for every 4-bit format.)
static size_t w4a16_layout(Carve &c, long T, int H, int I, int E, int k, RouteBufs *rb, uint16_t **h, uint16_t **ys,
                           uint16_t **xg = nullptr, uint16_t **h_small = nullptr, int E_sched = 0, int fmt = W4_INT4,
                           uint16_t **xh = nullptr)
{
    const int Es = E_sched > 0 ? E_sched : E;
    const bool tcp = w4_use_tc(T, k, Es);
    RouteBufs r = carve_route(c, T, k, E, tcp ? 256 : pick_block_m(T, k, Es));  // tensor-core tiles: 256 rows
    const size_t cap = (size_t)r.max_blocks * r.block_m;
    uint16_t *hp = c.take<uint16_t>((tcp ? cap : (size_t)T * k) * I);
    uint16_t *yp = c.take<uint16_t>((size_t)T * k * H);  // weighted slot rows (bf16) for the combine
    uint16_t *xgp = tcp ? c.take<uint16_t>(cap * H) : nullptr;  // routed rows of x in aligned order
    // small blocks of the tensor-core schedule: h in slot order
    uint16_t *hsp = tcp ? c.take<uint16_t>((size_t)T * k * I) : nullptr;
    // the decode schedule's copy of x in nibble-pair order (f16 for INT4), written by the routing kernel
    uint16_t *xhp = !tcp ? c.take<uint16_t>((size_t)T * H) : nullptr;
    if (rb) *rb = r;
    if (h) *h = hp;
    if (ys) *ys = yp;
    if (xg) *xg = xgp;
    if (h_small) *h_small = hsp;
    if (xh) *xh = xhp;
    return c.used;
}

// Block-FP8 layer schedule: from this many routed rows per expert on (mean T*k/E), the grouped
// GEMMs run on the tensor-core kernel over 128-row expert blocks; below, the register-fed swap-AB
// kernel streams the weights for the few rows each expert has.
static bool fp8_use_tc(long T, int k, int E) { return (double)T * k / (double)E >= 16.0; }

// E, E_sched: as w4a16_layout.
static size_t fp8_layout(Carve &c, long T, int H, int I, int E, int k, RouteBufs *rb, uint8_t **xq, float **xs,
                         uint8_t **hq, float **hs, uint16_t **ys, uint8_t **xg = nullptr, float **xsg = nullptr,
                         int E_sched = 0)
{
    const int Es = E_sched > 0 ? E_sched : E;
    const bool tcp = fp8_use_tc(T, k, Es);
    RouteBufs r = carve_route(c, T, k, E, tcp ? 128 : pick_block_m(T, k, Es));
    // aligned rows: every block the alignment can form (the tensor-core kernels index the
    // group-major scale arrays [groups, cap] with this row count)
    const size_t cap = (size_t)r.max_blocks * r.block_m;
    const size_t hrows = tcp ? cap : (size_t)T * k;                     // h rows: aligned or by slot
    uint8_t *xqp = c.take<uint8_t>((size_t)T * H);
    float *xsp = c.take<float>((size_t)T * (H / 128));
    uint8_t *hqp = c.take<uint8_t>(hrows * I);
    float *hsp = c.take<float>(hrows * (I / 128));
    uint16_t *yp = c.take<uint16_t>((size_t)T * k * H);  // weighted slot rows (bf16) for the combine
    uint8_t *xgp = tcp ? c.take<uint8_t>(cap * H) : nullptr;
    float *xsgp = tcp ? c.take<float>(cap * (H / 128)) : nullptr;
    if (rb) *rb = r;
    if (xq) *xq = xqp;
    if (xs) *xs = xsp;
    if (hq) *hq = hqp;
    if (hs) *hs = hsp;
    if (ys) *ys = yp;
    if (xg) *xg = xgp;
    if (xsg) *xsg = xsgp;
    return c.used;
}

// ---- validation ----------------------------------------------------------------------------------
static int check_routing_shape(long T, int E, int k)
{
    if (T < 0) return set_error(MOEQ_ERR_INVALID_ARG, "T must be >= 0 (got %ld)", T);
    if (E < 1 || E > kMaxExperts)
        return set_error(MOEQ_ERR_UNSUPPORTED, "E must be in [1, %d] (got %d)", kMaxExperts, E);
    if (k < 1 || k > kMaxTopK || k > E)
        return set_error(MOEQ_ERR_UNSUPPORTED, "k must be in [1, min(%d, E)] (got k=%d, E=%d)", kMaxTopK, k, E);
    if (T * (long)k > (1L << 24)) return set_error(MOEQ_ERR_UNSUPPORTED, "T*k must be <= 2^24 (got %ld)", T * k);
    return MOEQ_OK;
}

static int check_layer_shape(long T, int H, int I, int E, int k)
{
    int rc = check_routing_shape(T, E, k);
    if (rc) return rc;
    if (H < 128 || H % 128) return set_error(MOEQ_ERR_UNSUPPORTED, "H must be a positive multiple of 128 (got %d)", H);
    if (I < 128 || I % 128) return set_error(MOEQ_ERR_UNSUPPORTED, "I must be a positive multiple of 128 (got %d)", I);
    return MOEQ_OK;
}

// Expert parallelism: the call holds experts [ep_base, ep_base + ep_local) of the E the routing
// picks from.
static int check_expert_range(int E, int ep_base, int ep_local)
{
    if (ep_local < 1 || ep_base < 0 || ep_base > E - ep_local)
        return set_error(MOEQ_ERR_INVALID_ARG,
                         "expert range [ep_base, ep_base + ep_local) = [%d, %d) must be non-empty and lie in [0, E = %d)",
                         ep_base, ep_base + ep_local, E);
    return MOEQ_OK;
}

#define MOEQ_REQUIRE(ptr)                                                                       \
    do {                                                                                        \
        if ((ptr) == nullptr) return set_error(MOEQ_ERR_INVALID_ARG, "%s must not be NULL", #ptr); \
    } while (0)

}  // namespace moeq

using namespace moeq;

extern "C" {

const char *moe_last_error(void) { return g_err; }

const char *moe_version(void) { return MOEQ_VERSION; }

int moe_route_topk(const float *logits, int T, int E, int k, int32_t *topk_ids, float *topk_w, void *stream)
{
    g_err[0] = 0;
    int rc = check_routing_shape(T, E, k);
    if (rc) return rc;
    if (T == 0) return MOEQ_OK;
    MOEQ_REQUIRE(logits);
    MOEQ_REQUIRE(topk_ids);
    MOEQ_REQUIRE(topk_w);
    launch_route_topk(logits, T, E, k, topk_ids, topk_w, (cudaStream_t)stream);
    return check_launch("moe_route_topk");
}

size_t moe_align_workspace_size(int T, int k, int E)
{
    if (T < 0 || k < 1 || E < 1 || E > kMaxExperts || (long)T * k > (1L << 24)) return 0;
    return align_scratch_bytes(T * k, E);
}

int moe_align(const int32_t *topk_ids, int T, int k, int E, int block_m, int32_t *sorted_ids, int32_t *expert_ids,
              int32_t *num_tokens_padded, void *ws, size_t ws_bytes, void *stream)
{
    g_err[0] = 0;
    if (T < 0 || k < 1) return set_error(MOEQ_ERR_INVALID_ARG, "need T >= 0 and k >= 1 (got T=%d, k=%d)", T, k);
    if (E < 1 || E > kMaxExperts) return set_error(MOEQ_ERR_UNSUPPORTED, "E must be in [1, %d] (got %d)", kMaxExperts, E);
    if (block_m < 1 || block_m > 256) return set_error(MOEQ_ERR_UNSUPPORTED, "block_m must be in [1, 256] (got %d)", block_m);
    if ((long)T * k > (1L << 24)) return set_error(MOEQ_ERR_UNSUPPORTED, "T*k must be <= 2^24");
    MOEQ_REQUIRE(sorted_ids);
    MOEQ_REQUIRE(expert_ids);
    MOEQ_REQUIRE(num_tokens_padded);
    if (T > 0) MOEQ_REQUIRE(topk_ids);
    const size_t need = align_scratch_bytes(T * k, E);
    if (need && ws && (reinterpret_cast<uintptr_t>(ws) & 255))
        return set_error(MOEQ_ERR_INVALID_ARG, "ws must be 256-byte aligned");
    int32_t *scratch = (need && ws && ws_bytes >= need) ? static_cast<int32_t *>(ws) : nullptr;
    launch_align(topk_ids, T * k, E, block_m, sorted_ids, expert_ids, num_tokens_padded, scratch,
                 (cudaStream_t)stream);
    return check_launch("moe_align");
}

int moe_fp8_act_quant(const uint16_t *x, int rows, int cols, uint8_t *q, float *s, void *stream)
{
    g_err[0] = 0;
    if (rows < 0) return set_error(MOEQ_ERR_INVALID_ARG, "rows must be >= 0 (got %d)", rows);
    if (cols < 128 || cols % 128) return set_error(MOEQ_ERR_UNSUPPORTED, "cols must be a positive multiple of 128 (got %d)", cols);
    if (rows == 0) return MOEQ_OK;
    MOEQ_REQUIRE(x);
    MOEQ_REQUIRE(q);
    MOEQ_REQUIRE(s);
    launch_fp8_act_quant(x, rows, cols, q, s, (cudaStream_t)stream);
    return check_launch("moe_fp8_act_quant");
}

size_t moe_w4a16_workspace_size(int T, int H, int I, int E, int k)
{
    if (check_layer_shape(T, H, I, E, k)) return 0;
    Carve c(nullptr);
    return w4a16_layout(c, T, H, I, E, k, nullptr, nullptr, nullptr);
}

size_t moe_w4a16_ep_workspace_size(int T, int H, int I, int E, int k, int ep_local)
{
    if (check_layer_shape(T, H, I, E, k) || check_expert_range(E, 0, ep_local)) return 0;
    Carve c(nullptr);
    return w4a16_layout(c, T, H, I, ep_local, k, nullptr, nullptr, nullptr, nullptr, nullptr, E);  // INT4: the largest
}

}  // extern "C"

namespace moeq {
// The 4-bit weight layer (fmt W4_INT4: codes - 8 times bf16 group scales; W4_FP4: E2M1 codes
// times the bf16 group factors 2^(s - 1) of moe_mxfp4_prepack_scales): one schedule, the format
// only changes the kernels' dequantization.
static int w4_layer_forward(int fmt, const char *name, const uint16_t *x, const float *logits, int T, int H, int I,
                            int E, int k, const int32_t *w13_q, const uint16_t *w13_s, const int32_t *w2_q,
                            const uint16_t *w2_s, uint16_t *out, int32_t *topk_ids_out, float *topk_w_out, void *ws,
                            size_t ws_bytes, void *stream, const float *g13 = nullptr, const float *g2 = nullptr,
                            int ep_base = 0, int ep_local = 0)
{
    host_time::Scope host_scope;
    g_err[0] = 0;
    int rc = check_layer_shape(T, H, I, E, k);
    if (rc) return rc;
    const bool ep = ep_local > 0 || ep_base != 0;  // expert parallelism: weights of ep_local experts
    if (ep && (rc = check_expert_range(E, ep_base, ep_local))) return rc;
    const int Ew = ep ? ep_local : E;  // experts whose weights this call holds
    if (T == 0) return MOEQ_OK;
    MOEQ_REQUIRE(x);
    MOEQ_REQUIRE(logits);
    MOEQ_REQUIRE(w13_q);
    MOEQ_REQUIRE(w13_s);
    MOEQ_REQUIRE(w2_q);
    MOEQ_REQUIRE(w2_s);
    MOEQ_REQUIRE(out);
    MOEQ_REQUIRE(ws);
    if (reinterpret_cast<uintptr_t>(ws) & 255) return set_error(MOEQ_ERR_INVALID_ARG, "ws must be 256-byte aligned");
    const size_t need = ep ? moe_w4a16_ep_workspace_size(T, H, I, E, k, ep_local) : moe_w4a16_workspace_size(T, H, I, E, k);
    if (ws_bytes < need) return set_error(MOEQ_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, need);

    cudaStream_t s = (cudaStream_t)stream;
    Carve c(ws);
    RouteBufs r;
    uint16_t *h, *xg, *h_small, *xh;
    uint16_t *ys;
    w4a16_layout(c, T, H, I, Ew, k, &r, &h, &ys, &xg, &h_small, E, fmt, &xh);
    // global picks to the caller's buffer (if any); under expert parallelism the alignment and the
    // combine take the local ids (-1 for experts held elsewhere) in the route scratch
    int32_t *ids = topk_ids_out ? topk_ids_out : (ep ? nullptr : r.ids);
    int32_t *lids = ep ? r.ids : nullptr;
    float *tw = topk_w_out ? topk_w_out : r.w;
    const int n = T * k;
    const bool tcp = w4_use_tc(T, k, E);

    {
        trace::Scope ts(trace::ROUTE, s);
        launch_route_topk(logits, T, E, k, ids, tw, s, lids, ep_base, ep_local, x, H, xh, fmt == W4_INT4);
    }
    {
        trace::Scope ts(trace::ALIGN, s);
        launch_align(ep ? lids : ids, n, Ew, r.block_m, r.sorted, r.eids, r.ntp, r.scratch, s);
    }

    if (tcp) {
        int *status = device_status_ptr();
        if (!status) return set_error(MOEQ_ERR_CUDA, "%s: no device status word", name);
        const int cap = r.max_blocks * r.block_m;
        {
            trace::Scope ts(trace::GATHER, s);
            launch_gather_bf16(x, H, k, r.sorted, r.ntp, n, cap, kW4SmallRows, xg, num_sms(), s, fmt == W4_INT4);
        }
        W4TcArgs t{};
        t.fmt = fmt;
        t.status = status;
        t.E = Ew;
        t.sorted_ids = r.sorted;
        t.expert_ids = r.eids;
        t.ntp = r.ntp;
        t.n_slots = n;
        t.topk_w = tw;
        t.M = cap;
        t.N = I;
        t.K = H;
        t.rows_per_expert = 2 * I;
        t.wq = w13_q;
        t.ws = w13_s;
        t.wglobal = g13;
        t.h_out = h;
        t.small_rows = kW4SmallRows;
        // the small blocks: register-fed kernel over the same 256-row alignment, h in slot order
        W4GroupedArgs g{};
        g.fmt = fmt;
        g.E = Ew;
        g.sorted_ids = r.sorted;
        g.expert_ids = r.eids;
        g.num_tokens_padded = r.ntp;
        g.n_slots = n;
        g.topk_w = tw;
        g.blk_stride = r.block_m;
        g.act = x;
        g.act_bf16 = 1;  // INT4: converted in registers (the few-row blocks only)
        g.act_row_div = k;
        g.wq = w13_q;
        g.ws = w13_s;
        g.wglobal = g13;
        g.K = H;
        g.n_out = I;
        g.n_rows = 2 * I;
        g.h_out = h_small;
        int rc;
        {
            trace::Scope ts(trace::GATE_UP, s);
            rc = launch_w4a16_tc(t, TC_GATEUP, xg, r.max_blocks, s);
        }
        {
            trace::Scope ts(trace::FEW_ROWS, s);
            launch_w4a16_grouped_mma(g, MODE_GATEUP, kW4SmallRows, r.max_blocks, s);
        }
        if (rc) return rc;
        t.N = H;
        t.K = I;
        t.rows_per_expert = H;
        t.wq = w2_q;
        t.ws = w2_s;
        t.wglobal = g2;
        t.ys = ys;
        g.act = h_small;
        g.act_bf16 = 0;
        g.act_row_div = 1;
        g.wq = w2_q;
        g.ws = w2_s;
        g.wglobal = g2;
        g.K = I;
        g.n_out = H;
        g.n_rows = H;
        g.y_out = ys;
        {
            trace::Scope ts(trace::DOWN, s);
            rc = launch_w4a16_tc(t, TC_DOWN, h, r.max_blocks, s);
        }
        {
            trace::Scope ts(trace::FEW_ROWS, s);
            launch_w4a16_grouped_mma(g, MODE_DOWN, kW4SmallRows, r.max_blocks, s);
        }
        if (rc) return rc;
    } else {
        W4GroupedArgs a{};
        a.fmt = fmt;
        a.E = Ew;
        a.sorted_ids = r.sorted;
        a.expert_ids = r.eids;
        a.num_tokens_padded = r.ntp;
        a.n_slots = n;
        a.topk_w = tw;
        // gate/up + SiLU*up on the routing kernel's copy of x (nibble-pair order; f16 for INT4)
        a.act = xh;
        a.act_row_div = k;
        a.wq = w13_q;
        a.ws = w13_s;
        a.wglobal = g13;
        a.K = H;
        a.n_out = I;
        a.n_rows = 2 * I;
        a.h_out = h;
        {
            trace::Scope ts(trace::GATE_UP, s);
            launch_w4a16_grouped_mma(a, MODE_GATEUP, r.block_m, r.max_blocks, s);
        }
        // down, routing weight applied per slot
        a.act = h;
        a.act_row_div = 1;
        a.after_gateup = 1;
        a.wq = w2_q;
        a.ws = w2_s;
        a.wglobal = g2;
        a.K = I;
        a.n_out = H;
        a.n_rows = H;
        a.y_out = ys;
        {
            trace::Scope ts(trace::DOWN, s);
            launch_w4a16_grouped_mma(a, MODE_DOWN, r.block_m, r.max_blocks, s);
        }
    }
    {
        trace::Scope ts(trace::COMBINE, s);
        launch_combine(ys, T, k, H, out, num_sms(), s, lids);
    }
    return check_launch(name);
}
}  // namespace moeq

extern "C" {

int moe_w4a16_forward(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                      const int32_t *w13_q, const uint16_t *w13_s, const int32_t *w2_q, const uint16_t *w2_s,
                      uint16_t *out, int32_t *topk_ids_out, float *topk_w_out, void *ws, size_t ws_bytes,
                      void *stream)
{
    return w4_layer_forward(W4_INT4, "moe_w4a16_forward", x, logits, T, H, I, E, k, w13_q, w13_s, w2_q, w2_s, out,
                            topk_ids_out, topk_w_out, ws, ws_bytes, stream);
}

size_t moe_mxfp4_workspace_size(int T, int H, int I, int E, int k) { return moe_w4a16_workspace_size(T, H, I, E, k); }

int moe_mxfp4_forward(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                      const int32_t *w13_q, const uint16_t *w13_f, const int32_t *w2_q, const uint16_t *w2_f,
                      uint16_t *out, int32_t *topk_ids_out, float *topk_w_out, void *ws, size_t ws_bytes,
                      void *stream)
{
    return w4_layer_forward(W4_FP4, "moe_mxfp4_forward", x, logits, T, H, I, E, k, w13_q, w13_f, w2_q, w2_f, out,
                            topk_ids_out, topk_w_out, ws, ws_bytes, stream);
}

size_t moe_nvfp4_workspace_size(int T, int H, int I, int E, int k) { return moe_w4a16_workspace_size(T, H, I, E, k); }

int moe_nvfp4_forward(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                      const int32_t *w13_q, const uint16_t *w13_f, const float *w13_g, const int32_t *w2_q,
                      const uint16_t *w2_f, const float *w2_g, uint16_t *out, int32_t *topk_ids_out, float *topk_w_out,
                      void *ws, size_t ws_bytes, void *stream)
{
    g_err[0] = 0;
    if (T > 0) {
        MOEQ_REQUIRE(w13_g);
        MOEQ_REQUIRE(w2_g);
    }
    return w4_layer_forward(W4_NV, "moe_nvfp4_forward", x, logits, T, H, I, E, k, w13_q, w13_f, w2_q, w2_f, out,
                            topk_ids_out, topk_w_out, ws, ws_bytes, stream, w13_g, w2_g);
}

int moe_w4a16_forward_ep(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k, int ep_base,
                         int ep_local, const int32_t *w13_q, const uint16_t *w13_s, const int32_t *w2_q,
                         const uint16_t *w2_s, uint16_t *out, int32_t *topk_ids_out, float *topk_w_out, void *ws,
                         size_t ws_bytes, void *stream)
{
    g_err[0] = 0;
    if (int rc = check_expert_range(E, ep_base, ep_local)) return rc;
    return w4_layer_forward(W4_INT4, "moe_w4a16_forward_ep", x, logits, T, H, I, E, k, w13_q, w13_s, w2_q, w2_s, out,
                            topk_ids_out, topk_w_out, ws, ws_bytes, stream, nullptr, nullptr, ep_base, ep_local);
}

int moe_mxfp4_forward_ep(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k, int ep_base,
                         int ep_local, const int32_t *w13_q, const uint16_t *w13_f, const int32_t *w2_q,
                         const uint16_t *w2_f, uint16_t *out, int32_t *topk_ids_out, float *topk_w_out, void *ws,
                         size_t ws_bytes, void *stream)
{
    g_err[0] = 0;
    if (int rc = check_expert_range(E, ep_base, ep_local)) return rc;
    return w4_layer_forward(W4_FP4, "moe_mxfp4_forward_ep", x, logits, T, H, I, E, k, w13_q, w13_f, w2_q, w2_f, out,
                            topk_ids_out, topk_w_out, ws, ws_bytes, stream, nullptr, nullptr, ep_base, ep_local);
}

int moe_nvfp4_forward_ep(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k, int ep_base,
                         int ep_local, const int32_t *w13_q, const uint16_t *w13_f, const float *w13_g,
                         const int32_t *w2_q, const uint16_t *w2_f, const float *w2_g, uint16_t *out,
                         int32_t *topk_ids_out, float *topk_w_out, void *ws, size_t ws_bytes, void *stream)
{
    g_err[0] = 0;
    if (int rc = check_expert_range(E, ep_base, ep_local)) return rc;
    if (T > 0) {
        MOEQ_REQUIRE(w13_g);
        MOEQ_REQUIRE(w2_g);
    }
    return w4_layer_forward(W4_NV, "moe_nvfp4_forward_ep", x, logits, T, H, I, E, k, w13_q, w13_f, w2_q, w2_f, out,
                            topk_ids_out, topk_w_out, ws, ws_bytes, stream, w13_g, w2_g, ep_base, ep_local);
}

int moe_nvfp4_prepack_scales(const uint8_t *e4m3, long long n, uint16_t *factors, void *stream)
{
    g_err[0] = 0;
    if (n < 0) return set_error(MOEQ_ERR_INVALID_ARG, "n must be >= 0 (got %lld)", n);
    if (n == 0) return MOEQ_OK;
    MOEQ_REQUIRE(e4m3);
    MOEQ_REQUIRE(factors);
    launch_nvfp4_scale_factors(e4m3, n, factors, num_sms(), (cudaStream_t)stream);
    return check_launch("moe_nvfp4_prepack_scales");
}

int moe_mxfp4_prepack_scales(const uint8_t *ue8m0, long long n, uint16_t *factors, void *stream)
{
    g_err[0] = 0;
    if (n < 0) return set_error(MOEQ_ERR_INVALID_ARG, "n must be >= 0 (got %lld)", n);
    if (n == 0) return MOEQ_OK;
    MOEQ_REQUIRE(ue8m0);
    MOEQ_REQUIRE(factors);
    launch_mxfp4_scale_factors(ue8m0, n, factors, num_sms(), (cudaStream_t)stream);
    return check_launch("moe_mxfp4_prepack_scales");
}

// ------------------------------------------------------------------------------------------
// Grouped W4A16 GEMM, contiguous and masked layouts (per-row expert map -> alignment with k = 1,
// then the down-mode kernels with unit weights write each real row of C).
// ------------------------------------------------------------------------------------------

static bool grouped_use_tc(int rows_hint) { return rows_hint >= 16; }  // same rule as the layer: rows per expert

static size_t grouped_layout(Carve &c, long M, int K, int G, int rows_hint, RouteBufs *rb, int32_t **ids,
                             uint16_t **xg)
{
    const bool tcp = grouped_use_tc(rows_hint);
    int32_t *idp = c.take<int32_t>((size_t)M);
    RouteBufs r = carve_route(c, M, 1, G, tcp ? 256 : pick_block_m((long)rows_hint * G, 1, G));
    uint16_t *xgp = tcp ? c.take<uint16_t>((size_t)r.max_blocks * r.block_m * K) : nullptr;
    if (rb) *rb = r;
    if (ids) *ids = idp;
    if (xg) *xg = xgp;
    return c.used;
}

static int check_grouped_shape(long M, int K, int N, int G)
{
    if (M < 0) return set_error(MOEQ_ERR_INVALID_ARG, "row count must be >= 0 (got %ld)", M);
    if (M > (1L << 24)) return set_error(MOEQ_ERR_UNSUPPORTED, "row count must be <= 2^24 (got %ld)", M);
    if (K < 128 || K % 128) return set_error(MOEQ_ERR_UNSUPPORTED, "K must be a positive multiple of 128 (got %d)", K);
    if (N < 128 || N % 128) return set_error(MOEQ_ERR_UNSUPPORTED, "N must be a positive multiple of 128 (got %d)", N);
    if (G < 1 || G > kMaxExperts) return set_error(MOEQ_ERR_UNSUPPORTED, "G must be in [1, %d] (got %d)", kMaxExperts, G);
    return MOEQ_OK;
}

size_t moe_w4a16_grouped_contiguous_workspace_size(int M, int K, int N, int G)
{
    if (check_grouped_shape(M, K, N, G)) return 0;
    Carve c(nullptr);
    return grouped_layout(c, M, K, G, M / G, nullptr, nullptr, nullptr);
}

size_t moe_w4a16_grouped_masked_workspace_size(int G, int max_m, int K, int N, int expected_m)
{
    if (max_m < 0 || check_grouped_shape((long)G * max_m, K, N, G)) return 0;
    Carve c(nullptr);
    return grouped_layout(c, (long)G * max_m, K, G, expected_m, nullptr, nullptr, nullptr);
}

static int grouped_forward(const char *name, const uint16_t *A, long M, int K, const int32_t *wq, const uint16_t *wsc,
                           int G, int N, const int32_t *m_indices, const int32_t *masked_m, int max_m, int rows_hint,
                           uint16_t *C, void *ws, size_t ws_bytes, void *stream)
{
    host_time::Scope host_scope;
    MOEQ_REQUIRE(A);
    MOEQ_REQUIRE(wq);
    MOEQ_REQUIRE(wsc);
    MOEQ_REQUIRE(C);
    MOEQ_REQUIRE(ws);
    if (!m_indices && !masked_m) return set_error(MOEQ_ERR_INVALID_ARG, "%s: no row-to-expert map", name);
    if (reinterpret_cast<uintptr_t>(ws) & 255) return set_error(MOEQ_ERR_INVALID_ARG, "ws must be 256-byte aligned");
    Carve need_c(nullptr);
    const size_t need = grouped_layout(need_c, M, K, G, rows_hint, nullptr, nullptr, nullptr);
    if (ws_bytes < need) return set_error(MOEQ_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, need);
    cudaStream_t s = (cudaStream_t)stream;
    Carve c(ws);
    RouteBufs r;
    int32_t *idp;
    uint16_t *xg;
    grouped_layout(c, M, K, G, rows_hint, &r, &idp, &xg);
    const int n = (int)M;
    const int32_t *ids = m_indices;
    {
        trace::Scope ts(trace::ALIGN, s);
        if (masked_m) {
            launch_masked_rows(masked_m, G, max_m, idp, num_sms(), s);
            ids = idp;
        }
        launch_align(ids, n, G, r.block_m, r.sorted, r.eids, r.ntp, r.scratch, s);
    }
    W4GroupedArgs g{};
    g.E = G;
    g.sorted_ids = r.sorted;
    g.expert_ids = r.eids;
    g.num_tokens_padded = r.ntp;
    g.n_slots = n;
    g.topk_w = nullptr;  // weight 1: plain grouped GEMM
    g.act = A;
    g.act_bf16 = 1;      // INT4 in f16: the bf16 rows are converted in registers
    g.act_row_div = 1;   // k = 1: the slot is the row
    g.wq = wq;
    g.ws = wsc;
    g.K = K;
    g.n_out = N;
    g.n_rows = N;
    g.y_out = C;
    trace::Scope ts(trace::DOWN, s);
    if (xg) {
        int *status = device_status_ptr();
        if (!status) return set_error(MOEQ_ERR_CUDA, "%s: no device status word", name);
        const int cap = r.max_blocks * r.block_m;
        launch_gather_bf16(A, K, 1, r.sorted, r.ntp, n, cap, kW4SmallRows, xg, num_sms(), s, true);
        W4TcArgs t{};
        t.status = status;
        t.E = G;
        t.sorted_ids = r.sorted;
        t.expert_ids = r.eids;
        t.ntp = r.ntp;
        t.n_slots = n;
        t.topk_w = nullptr;
        t.M = cap;
        t.N = N;
        t.K = K;
        t.rows_per_expert = N;
        t.wq = wq;
        t.ws = wsc;
        t.ys = C;
        t.small_rows = kW4SmallRows;
        const int rc = launch_w4a16_tc(t, TC_DOWN, xg, r.max_blocks, s);
        if (rc) return rc;
        g.blk_stride = r.block_m;
        launch_w4a16_grouped_mma(g, MODE_DOWN, kW4SmallRows, r.max_blocks, s);
    } else {
        launch_w4a16_grouped_mma(g, MODE_DOWN, r.block_m, r.max_blocks, s);
    }
    return check_launch(name);
}

int moe_w4a16_grouped_contiguous(const uint16_t *A, int M, int K, const int32_t *w_q, const uint16_t *w_s, int G, int N,
                                 const int32_t *m_indices, uint16_t *C, void *ws, size_t ws_bytes, void *stream)
{
    g_err[0] = 0;
    int rc = check_grouped_shape(M, K, N, G);
    if (rc) return rc;
    if (M == 0) return MOEQ_OK;
    MOEQ_REQUIRE(m_indices);
    return grouped_forward("moe_w4a16_grouped_contiguous", A, M, K, w_q, w_s, G, N, m_indices, nullptr, 0, M / G, C,
                           ws, ws_bytes, stream);
}

int moe_w4a16_grouped_masked(const uint16_t *A, int G, int max_m, int K, const int32_t *w_q, const uint16_t *w_s, int N,
                             const int32_t *masked_m, int expected_m, uint16_t *C, void *ws, size_t ws_bytes,
                             void *stream)
{
    g_err[0] = 0;
    if (max_m < 0) return set_error(MOEQ_ERR_INVALID_ARG, "max_m must be >= 0 (got %d)", max_m);
    if (expected_m < 0) return set_error(MOEQ_ERR_INVALID_ARG, "expected_m must be >= 0 (got %d)", expected_m);
    int rc = check_grouped_shape((long)G * max_m, K, N, G);
    if (rc) return rc;
    if (max_m == 0) return MOEQ_OK;
    MOEQ_REQUIRE(masked_m);
    return grouped_forward("moe_w4a16_grouped_masked", A, (long)G * max_m, K, w_q, w_s, G, N, nullptr, masked_m, max_m,
                           expected_m, C, ws, ws_bytes, stream);
}

size_t moe_w8a8_block_fp8_workspace_size(int T, int H, int I, int E, int k)
{
    if (check_layer_shape(T, H, I, E, k)) return 0;
    Carve c(nullptr);
    return fp8_layout(c, T, H, I, E, k, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
}

size_t moe_w8a8_block_fp8_ep_workspace_size(int T, int H, int I, int E, int k, int ep_local)
{
    if (check_layer_shape(T, H, I, E, k) || check_expert_range(E, 0, ep_local)) return 0;
    Carve c(nullptr);
    return fp8_layout(c, T, H, I, ep_local, k, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, E);
}

// The block-FP8 layer; ep_local > 0: expert parallelism over [ep_base, ep_base + ep_local).
static int fp8_layer_forward(const char *name, const uint16_t *x, const float *logits, int T, int H, int I, int E,
                             int k, const uint8_t *w13, const float *w13_s, const uint8_t *w2, const float *w2_s,
                             uint16_t *out, int32_t *topk_ids_out, float *topk_w_out, void *ws, size_t ws_bytes,
                             void *stream, int ep_base, int ep_local)
{
    host_time::Scope host_scope;
    g_err[0] = 0;
    int rc = check_layer_shape(T, H, I, E, k);
    if (rc) return rc;
    const bool ep = ep_local > 0 || ep_base != 0;
    if (ep && (rc = check_expert_range(E, ep_base, ep_local))) return rc;
    const int Ew = ep ? ep_local : E;  // experts whose weights this call holds
    if (T == 0) return MOEQ_OK;
    MOEQ_REQUIRE(x);
    MOEQ_REQUIRE(logits);
    MOEQ_REQUIRE(w13);
    MOEQ_REQUIRE(w13_s);
    MOEQ_REQUIRE(w2);
    MOEQ_REQUIRE(w2_s);
    MOEQ_REQUIRE(out);
    MOEQ_REQUIRE(ws);
    if (reinterpret_cast<uintptr_t>(ws) & 255) return set_error(MOEQ_ERR_INVALID_ARG, "ws must be 256-byte aligned");
    const size_t need = ep ? moe_w8a8_block_fp8_ep_workspace_size(T, H, I, E, k, ep_local)
                           : moe_w8a8_block_fp8_workspace_size(T, H, I, E, k);
    if (ws_bytes < need) return set_error(MOEQ_ERR_WORKSPACE, "workspace %zu bytes < required %zu", ws_bytes, need);

    cudaStream_t s = (cudaStream_t)stream;
    Carve c(ws);
    RouteBufs r;
    uint8_t *xq, *hq, *xg;
    float *xs, *hs, *xsg;
    uint16_t *ys;
    fp8_layout(c, T, H, I, Ew, k, &r, &xq, &xs, &hq, &hs, &ys, &xg, &xsg, E);
    int32_t *ids = topk_ids_out ? topk_ids_out : (ep ? nullptr : r.ids);
    int32_t *lids = ep ? r.ids : nullptr;
    float *tw = topk_w_out ? topk_w_out : r.w;
    const int n = T * k;
    const bool tcp = fp8_use_tc(T, k, E);

    {
        trace::Scope ts(trace::ROUTE, s);
        launch_route_topk(logits, T, E, k, ids, tw, s, lids, ep_base, ep_local);
    }
    {
        trace::Scope ts(trace::ALIGN, s);
        launch_align(ep ? lids : ids, n, Ew, r.block_m, r.sorted, r.eids, r.ntp, r.scratch, s);
    }
    {
        trace::Scope ts(trace::ACT_QUANT, s);
        launch_fp8_act_quant(x, T, H, xq, xs, s);
    }
    if (tcp) {
        trace::Scope ts(trace::GATHER, s);
        launch_gather_fp8_rows(xq, xs, H, k, r.sorted, r.ntp, n, r.max_blocks * 128, xg, xsg, num_sms(), s);
    }

    if (tcp) {
        int *status = device_status_ptr();
        if (!status) return set_error(MOEQ_ERR_CUDA, "%s: no device status word", name);
        const int cap = r.max_blocks * 128;
        Fp8TcArgs t{};
        t.status = status;
        t.E = Ew;
        t.sorted_ids = r.sorted;
        t.expert_ids = r.eids;
        t.ntp = r.ntp;
        t.n_slots = n;
        t.topk_w = tw;
        // gate/up + SiLU*up + E4M3 quantization of the intermediate (rows in aligned order)
        t.a_scale = xsg;
        t.b_scale = w13_s;
        t.M = cap;
        t.N = I;
        t.K = H;
        t.rows_per_expert = 2 * I;
        t.hq = hq;
        t.hs = hs;
        int rc;
        {
            trace::Scope ts(trace::GATE_UP, s);
            rc = launch_fp8_tc_grouped(t, TC_GATEUP, xg, w13, Ew, r.max_blocks, s);
        }
        if (rc) return rc;
        // down, routing weight applied, rows scattered back to their slots
        t.a_scale = hs;
        t.b_scale = w2_s;
        t.N = H;
        t.K = I;
        t.rows_per_expert = H;
        t.ys = ys;
        {
            trace::Scope ts(trace::DOWN, s);
            rc = launch_fp8_tc_grouped(t, TC_DOWN, hq, w2, Ew, r.max_blocks, s);
        }
        if (rc) return rc;
    } else {
        F8GroupedArgs a{};
        a.E = Ew;
        a.sorted_ids = r.sorted;
        a.expert_ids = r.eids;
        a.num_tokens_padded = r.ntp;
        a.n_slots = n;
        a.topk_w = tw;
        a.act = xq;
        a.act_s = xs;
        a.act_row_div = k;
        a.w = w13;
        a.w_s = w13_s;
        a.K = H;
        a.n_out = I;
        a.n_rows = 2 * I;
        a.hq_out = hq;
        a.hs_out = hs;
        {
            trace::Scope ts(trace::GATE_UP, s);
            launch_fp8_grouped_mma(a, MODE_GATEUP, r.block_m, r.max_blocks, s);
        }
        a.act = hq;
        a.act_s = hs;
        a.act_row_div = 1;
        a.w = w2;
        a.w_s = w2_s;
        a.K = I;
        a.n_out = H;
        a.n_rows = H;
        a.y_out = ys;
        {
            trace::Scope ts(trace::DOWN, s);
            launch_fp8_grouped_mma(a, MODE_DOWN, r.block_m, r.max_blocks, s);
        }
    }
    {
        trace::Scope ts(trace::COMBINE, s);
        launch_combine(ys, T, k, H, out, num_sms(), s, lids);
    }
    return check_launch(name);
}

int moe_w8a8_block_fp8_forward(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                               const uint8_t *w13, const float *w13_s, const uint8_t *w2, const float *w2_s,
                               uint16_t *out, int32_t *topk_ids_out, float *topk_w_out, void *ws, size_t ws_bytes,
                               void *stream)
{
    return fp8_layer_forward("moe_w8a8_block_fp8_forward", x, logits, T, H, I, E, k, w13, w13_s, w2, w2_s, out,
                             topk_ids_out, topk_w_out, ws, ws_bytes, stream, 0, 0);
}

int moe_w8a8_block_fp8_forward_ep(const uint16_t *x, const float *logits, int T, int H, int I, int E, int k,
                                  int ep_base, int ep_local, const uint8_t *w13, const float *w13_s, const uint8_t *w2,
                                  const float *w2_s, uint16_t *out, int32_t *topk_ids_out, float *topk_w_out, void *ws,
                                  size_t ws_bytes, void *stream)
{
    g_err[0] = 0;
    if (int rc = check_expert_range(E, ep_base, ep_local)) return rc;
    return fp8_layer_forward("moe_w8a8_block_fp8_forward_ep", x, logits, T, H, I, E, k, w13, w13_s, w2, w2_s, out,
                             topk_ids_out, topk_w_out, ws, ws_bytes, stream, ep_base, ep_local);
}

int w8a8_block_fp8_matmul(const uint8_t *A, const float *As, const uint8_t *B, const float *Bs, int M, int N, int K,
                          int block_n, int block_k, uint16_t *C, void *stream)
{
    host_time::Scope host_scope;
    g_err[0] = 0;
    if (block_n != 128 || block_k != 128)
        return set_error(MOEQ_ERR_UNSUPPORTED, "block_size must be [128, 128] (got [%d, %d])", block_n, block_k);
    if (M < 0 || N < 1 || K < 1) return set_error(MOEQ_ERR_INVALID_ARG, "bad sizes M=%d N=%d K=%d", M, N, K);
    if (K % 128) return set_error(MOEQ_ERR_UNSUPPORTED, "K must be a multiple of 128 (got %d)", K);
    if (N % 128) return set_error(MOEQ_ERR_UNSUPPORTED, "N must be a multiple of 128 (got %d)", N);
    if (M == 0) return MOEQ_OK;
    MOEQ_REQUIRE(A);
    MOEQ_REQUIRE(As);
    MOEQ_REQUIRE(B);
    MOEQ_REQUIRE(Bs);
    MOEQ_REQUIRE(C);
    if (reinterpret_cast<uintptr_t>(A) % 16 || reinterpret_cast<uintptr_t>(B) % 16 || reinterpret_cast<uintptr_t>(C) % 16)
        return set_error(MOEQ_ERR_UNSUPPORTED, "w8a8_block_fp8_matmul: A, B and C must be 16-byte aligned");
    // up to 32 rows: swap-AB tiles with K split over a cluster (HBM bound); more rows: 128-row
    // activation tiles
    Fp8TcArgs t{};
    t.a_scale = As;
    t.b_scale = Bs;
    t.C = C;
    t.M = M;
    t.N = N;
    t.K = K;
    t.status = device_status_ptr();
    if (!t.status) return set_error(MOEQ_ERR_CUDA, "w8a8_block_fp8_matmul: no device status word");
    trace::Scope ts(trace::DENSE, (cudaStream_t)stream);
    const int rc = M <= fp8_skinny_max_rows(false)
                       ? launch_fp8_tc_skinny(t, A, B, pick_skinny_split(M, N, K, false), false, (cudaStream_t)stream)
                       : launch_fp8_tc_gemm(t, A, B, (cudaStream_t)stream);
    if (rc) return rc;
    return check_launch("w8a8_block_fp8_matmul");
}

int w8a8_channel_fp8_matmul(const uint8_t *A, const float *As, const uint8_t *B, const float *Bs, int M, int N, int K,
                            uint16_t *C, void *stream)
{
    host_time::Scope host_scope;
    g_err[0] = 0;
    if (M < 0 || N < 1 || K < 1) return set_error(MOEQ_ERR_INVALID_ARG, "bad sizes M=%d N=%d K=%d", M, N, K);
    if (K % 128) return set_error(MOEQ_ERR_UNSUPPORTED, "K must be a multiple of 128 (got %d)", K);
    if (N % 128) return set_error(MOEQ_ERR_UNSUPPORTED, "N must be a multiple of 128 (got %d)", N);
    if (M == 0) return MOEQ_OK;
    MOEQ_REQUIRE(A);
    MOEQ_REQUIRE(As);
    MOEQ_REQUIRE(B);
    MOEQ_REQUIRE(Bs);
    MOEQ_REQUIRE(C);
    if (reinterpret_cast<uintptr_t>(A) % 16 || reinterpret_cast<uintptr_t>(B) % 16 || reinterpret_cast<uintptr_t>(C) % 16)
        return set_error(MOEQ_ERR_UNSUPPORTED, "w8a8_channel_fp8_matmul: A, B and C must be 16-byte aligned");
    // up to 64 rows: swap-AB tiles, K split over a cluster; more rows: 128-row activation tiles
    // (CTA pairs from 256 rows); both accumulate all of K in tensor memory and scale once
    Fp8TcArgs t{};
    t.a_scale = As;
    t.b_scale = Bs;
    t.C = C;
    t.M = M;
    t.N = N;
    t.K = K;
    t.status = device_status_ptr();
    if (!t.status) return set_error(MOEQ_ERR_CUDA, "w8a8_channel_fp8_matmul: no device status word");
    trace::Scope ts(trace::DENSE, (cudaStream_t)stream);
    const int rc = M <= fp8_skinny_max_rows(true)
                       ? launch_fp8_tc_skinny(t, A, B, pick_skinny_split(M, N, K, true), true, (cudaStream_t)stream)
                       : launch_fp8_tc_channel(t, A, B, (cudaStream_t)stream);
    if (rc) return rc;
    return check_launch("w8a8_channel_fp8_matmul");
}

int moe_trace_enable(int enable)
{
    g_err[0] = 0;
    std::lock_guard<std::mutex> g(trace::mu);
    trace::enabled = enable != 0;
    return MOEQ_OK;
}

int moe_trace_read(double *stage_ms, long long *stage_calls, int n_stages, int reset)
{
    g_err[0] = 0;
    std::lock_guard<std::mutex> g(trace::mu);
    for (const trace::Rec &r : trace::pending) {
        float ms = 0.f;
        cudaError_t e = cudaEventSynchronize(r.b);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
        if (e != cudaSuccess) {
            trace::pending.clear();
            return set_error(MOEQ_ERR_CUDA, "moe_trace_read: %s", cudaGetErrorString(e));
        }
        trace::sum_ms[r.stage] += ms;
        trace::calls[r.stage] += 1;
        trace::spare.push_back(r.a);
        trace::spare.push_back(r.b);
    }
    trace::pending.clear();
    for (int i = 0; i < n_stages && i < trace::NSTAGE; ++i) {
        if (stage_ms) stage_ms[i] = trace::sum_ms[i];
        if (stage_calls) stage_calls[i] = trace::calls[i];
    }
    if (reset)
        for (int i = 0; i < trace::NSTAGE; ++i) { trace::sum_ms[i] = 0.0; trace::calls[i] = 0; }
    return trace::NSTAGE;
}

int moe_host_stats(double *host_us, long long *calls, long long *tmap_encoded, long long *tmap_reused, int reset)
{
    g_err[0] = 0;
    long long hits = 0, misses = 0;
    tmap_memo_stats(&hits, &misses);
    const long long n = host_time::calls.load(std::memory_order_relaxed);
    if (host_us) *host_us = host_time::ns.load(std::memory_order_relaxed) * 1e-3;
    if (calls) *calls = n;
    if (tmap_encoded) *tmap_encoded = misses;
    if (tmap_reused) *tmap_reused = hits;
    if (reset) {
        host_time::ns.store(0, std::memory_order_relaxed);
        host_time::calls.store(0, std::memory_order_relaxed);
    }
    return MOEQ_OK;
}

int moe_selftest_bounded_wait(void *stream)
{
    g_err[0] = 0;
    const int rc = launch_selftest_bounded_wait((cudaStream_t)stream);
    if (rc) return rc;
    return check_launch("moe_selftest_bounded_wait");
}

int moe_device_status(int clear)
{
    g_err[0] = 0;
    int *p = device_status_ptr();
    if (!p) return set_error(MOEQ_ERR_CUDA, "moe_device_status: no device status word");
    int v = 0;
    cudaError_t e = cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return set_error(MOEQ_ERR_CUDA, "moe_device_status: %s", cudaGetErrorString(e));
    if (clear) {
        const int z = 0;
        e = cudaMemcpy(p, &z, sizeof z, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return set_error(MOEQ_ERR_CUDA, "moe_device_status: %s", cudaGetErrorString(e));
    }
    return v ? MOEQ_ERR_DEVICE_TIMEOUT : MOEQ_OK;
}

}  // extern "C"
