// moe_api.cu -- the extern "C" entry points of libmoe_b200.so: argument checks on the
// host, workspace layout, and the launch sequence of the layer.  See include/moe_api.h.
#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"

namespace moe {

std::atomic<unsigned long long> g_launches{0};
void count_launches(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

cudaError_t set_smem_limit(const void* fn, size_t bytes) {
    struct Entry {
        const void* fn;
        int dev;
        size_t bytes;
    };
    static std::mutex mu;
    static std::vector<Entry> set;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    Entry* e = nullptr;
    for (Entry& x : set)
        if (x.fn == fn && x.dev == dev) e = &x;
    if (e != nullptr && e->bytes >= bytes) return cudaSuccess;
    const cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(bytes));
    if (err != cudaSuccess) return err;
    if (e != nullptr) e->bytes = bytes;
    else set.push_back(Entry{fn, dev, bytes});
    return cudaSuccess;
}

constexpr unsigned long long kDefaultGridWaitNs = 2000000000ull;  // 2 s
std::atomic<unsigned long long> g_grid_wait_ns{kDefaultGridWaitNs};
unsigned long long grid_wait_budget_ns() { return g_grid_wait_ns.load(std::memory_order_relaxed); }

namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;

size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms_current() {
    static int cache[kMaxDevices] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// Workspace of the whole layer.  The status word is always at offset 0.
struct Layout {
    size_t status, counters, counts, tickets, perm_hist, logits, offsets, dense_offsets, topk_idx,
        topk_w, sgate, sorted_token, sorted_w, slot_to_row, x_sorted, h, h_s, out_acc, y_sorted,
        part, total;
    size_t zero_end;  // [0, zero_end) is cleared at the start of a layer call
};

// The routed gate_up may cut its tiles' K steps into up to kSplitMax slices when its tiles
// cannot fill the GPU (a few tokens, or a few experts), if the slices' fp32 partial sums
// (kSplitMax planes of [T*K, 2f]) take at most 64 MiB; one ticket per tile, bounded by the
// tiles of 16-row blocks: min(E, T*K) + T*K/16 + 1 row blocks of f/128 feature blocks.
constexpr int kSplitMax = 4;
bool gate_up_split_ok(long long T, long long K, long long f) {
    return 4ll * kSplitMax * T * K * 2 * f <= (64ll << 20);
}
long long gate_up_ticket_cap(long long T, long long E, long long K, long long f) {
    if (!gate_up_split_ok(T, K, f)) return 0;
    const long long rows = T * K;
    return (std::min(E, rows) + rows / 16 + 1) * (f / 128);
}

Layout layout(long long T, long long D, long long E, long long K, long long f, long long fs) {
    Layout L{};
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t r = o;
        o = align_up(o + bytes);
        return r;
    };
    L.status = take(kAlign);
    L.counters = take(sizeof(unsigned) * static_cast<size_t>((T + 7) / 8));
    L.counts = take(sizeof(int32_t) * E);
    L.tickets = take(sizeof(unsigned) * gate_up_ticket_cap(T, E, K, f));
    L.zero_end = o;
    // its offset depends on T, E, K and (through the split tickets) f; the single-step entry
    // points all lay the workspace out with f = 128, so they agree with each other
    L.perm_hist = take(sizeof(int32_t) * E * permute_chunks(T * K));
    // router logits: [T, E+1] (CUDA-core router) or partial-sum planes of [T, E]
    L.logits = take(sizeof(float) * T *
                    std::max<long long>(E + 1, router_uses_tensor_cores(static_cast<int>(T), static_cast<int>(E))
                                                   ? router_tc_max_planes(static_cast<int>(T)) * E
                                                   : 0));
    L.offsets = take(sizeof(int32_t) * (E + 1));
    L.dense_offsets = take(sizeof(int32_t) * 2);
    L.topk_idx = take(sizeof(int32_t) * T * K);
    L.topk_w = take(sizeof(float) * T * K);
    L.sgate = take(sizeof(float) * T);
    L.sorted_token = take(sizeof(int32_t) * T * K);
    L.sorted_w = take(sizeof(float) * T * K);
    L.slot_to_row = take(sizeof(int32_t) * T * K);
    L.x_sorted = take(2 * T * K * D);
    L.h = take(2 * T * K * f);
    L.h_s = take(2 * T * fs);
    L.out_acc = take(sizeof(float) * T * D);
    L.y_sorted = take(sizeof(float) * T * K * D);
    L.part = take(gate_up_split_ok(T, K, f) ? sizeof(float) * kSplitMax * T * K * 2 * f : 0);
    L.total = o;
    return L;
}

int check_shape(int T, int D, int E, int K, int f, int fs) {
    if (T < 0 || D <= 0 || E <= 0 || K <= 0 || f <= 0 || fs < 0) return MOE_ERR_ARG;
    if (E > 512 || K > 16 || K > E) return MOE_ERR_UNSUPPORTED;
    if (D % 128 || D > 8192 || f % 128 || f > 8192 || fs % 128 || fs > 8192)
        return MOE_ERR_UNSUPPORTED;
    if (static_cast<long long>(T) * K >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

template <class P>
P* at(void* ws, size_t off) {
    return reinterpret_cast<P*>(static_cast<uint8_t*>(ws) + off);
}

// Host checks of moe_layer_forward's parameters (out may be NULL when only planning).
int check_layer(const moe_layer_params* p, const moe_bf16* out) {
    if (!p) return MOE_ERR_ARG;
    const int T = p->T, E = p->E, K = p->K;
    int rc = check_shape(T, p->D, E, K, p->f, p->f_s);
    if (rc) return rc;
    const bool shared = p->f_s > 0;
    if (!p->w_router || !p->w_gate_up || !p->w_down) return MOE_ERR_ARG;
    if (shared && (!p->w_shared_gate || !p->w_shared_gate_up || !p->w_shared_down)) return MOE_ERR_ARG;
    if (!shared && (p->w_shared_gate || p->w_shared_gate_up || p->w_shared_down)) return MOE_ERR_ARG;
    if (p->score_mode != MOE_SCORE_SOFTMAX && p->score_mode != MOE_SCORE_SIGMOID) return MOE_ERR_ARG;
    if (!(p->capacity_factor >= 0.f) || !std::isfinite(p->capacity_factor) || p->min_capacity < 0)
        return MOE_ERR_ARG;
    if (!aligned16(p->x) || !aligned16(p->w_router) || !aligned16(p->w_gate_up) ||
        !aligned16(p->w_down) || !aligned16(out) || !aligned16(p->residual) ||
        (shared && (!aligned16(p->w_shared_gate) || !aligned16(p->w_shared_gate_up) ||
                    !aligned16(p->w_shared_down))))
        return MOE_ERR_ALIGN;
    return MOE_OK;
}

// Every launch of one layer call, and the choices that shape them.
struct LayerPlan {
    RouterLaunch r;
    PermuteLaunch pm;
    GroupedGemmLaunch up, dn, su, sd;
    CombineLaunch c;
    bool tc_router, det, shared_launches;
    bool rows_mode;  // down on CTA pairs writes weighted bf16 rows; the combine sums them
    bool combine;    // a combine launch ends the call
};

LayerPlan plan_layer(const moe_layer_params* p, moe_bf16* out, void* workspace, int sms) {
    const int T = p->T, D = p->D, E = p->E, K = p->K, f = p->f, fs = p->f_s;
    const Layout L = layout(T, D, E, K, f, fs);
    const bool shared = fs > 0;
    // expert capacity (assignments per expert), or -1: dropless
    const long long capacity = p->capacity_factor > 0.f
                                   ? moe_expert_capacity(T, K, E, p->capacity_factor, p->min_capacity)
                                   : -1;
    LayerPlan q{};
    q.det = (p->flags & MOE_FLAG_DETERMINISTIC) != 0;
    q.tc_router = router_uses_tensor_cores(T, E);
    int* status = at<int>(workspace, L.status);
    // the router counts into the workspace (cleared with the header); the permutation
    // copies the counts out when the caller asks for them
    int32_t* counts = at<int32_t>(workspace, L.counts);
    int32_t* idx = p->topk_idx_out ? p->topk_idx_out : at<int32_t>(workspace, L.topk_idx);
    float* tw = p->topk_w_out ? p->topk_w_out : at<float>(workspace, L.topk_w);
    float* sgate = at<float>(workspace, L.sgate);
    float* out_acc = at<float>(workspace, L.out_acc);
    const int rows = T * K;
    // When the down projection runs on CTA pairs (many rows per expert: the layer is
    // tensor-bound), its epilogue writes each row's weighted output as bf16 with plain
    // stores (into the expert-ordered x copy, free by then) and a fixed-order combine sums a
    // token's K rows: fp32 reductions of T*K*D values into a [T, D] accumulator larger than
    // L2 would keep the tensor pipe waiting.
    GroupedGemmLaunch probe{};
    probe.gate_up = false;
    probe.rows = rows; probe.E = E; probe.D = D; probe.f = f;
    q.rows_mode = !q.det && grouped_gemm_uses_pairs(probe, sms);
    q.combine = q.det || q.rows_mode;
    // the fp32 accumulator: every routed row's reductions, or only the shared expert's
    const bool use_acc = shared || (!q.det && !q.rows_mode);

    PermuteLaunch& pm = q.pm;
    pm.topk_idx = idx;
    pm.topk_w = tw;
    // tensor-core router (many tokens): no per-entry count atomics in the selection; the
    // permutation counts from its chunk histograms
    pm.counts = q.tc_router ? nullptr : counts;
    pm.counts_out = p->expert_counts_out;
    pm.T = T; pm.E = E; pm.K = K;
    pm.offsets = at<int32_t>(workspace, L.offsets);
    pm.sorted_token = at<int32_t>(workspace, L.sorted_token);
    pm.sorted_w = at<float>(workspace, L.sorted_w);
    pm.slot_to_row = at<int32_t>(workspace, L.slot_to_row);
    pm.dense_offsets = at<int32_t>(workspace, L.dense_offsets);
    pm.status = status;
    pm.hist = at<int32_t>(workspace, L.perm_hist);
    pm.capacity = capacity;

    RouterLaunch& r = q.r;
    r.x = reinterpret_cast<const bf16*>(p->x);
    r.w_router = reinterpret_cast<const bf16*>(p->w_router);
    r.logit_bias = p->logit_bias;
    r.w_shared_gate = shared ? reinterpret_cast<const bf16*>(p->w_shared_gate) : nullptr;
    r.T = T; r.D = D; r.E = E; r.K = K;
    r.logits = at<float>(workspace, L.logits);
    r.counters = at<unsigned>(workspace, L.counters);
    r.topk_idx = idx;
    r.topk_w = tw;
    r.counts = q.tc_router ? nullptr : counts;
    r.shared_gate = sgate;
    r.status = status;
    r.zero_acc = use_acc && !q.tc_router ? out_acc : nullptr;
    r.zero_cols = D;
    r.score_mode = p->score_mode;
    r.select_bias = p->select_bias;
    r.bf16_weights = (p->flags & MOE_FLAG_BF16_WEIGHTS) ? 1 : 0;

    GroupedGemmLaunch& up = q.up;
    up.gate_up = true;
    up.w = p->w_gate_up;
    up.act = p->x;
    up.gather_tok = pm.sorted_token;
    up.gather_buf = at<bf16>(workspace, L.x_sorted);
    up.offsets = pm.offsets;
    up.rows = rows; up.E = E; up.D = D; up.f = f;
    up.max_group_rows = capacity >= 0 && capacity < T ? static_cast<int>(capacity) : T;
    if (gate_up_split_ok(T, K, f)) {
        up.ksplit_max = kSplitMax;
        up.part = at<float>(workspace, L.part);
        up.tickets = at<unsigned>(workspace, L.tickets);
        up.ticket_cap = static_cast<int>(gate_up_ticket_cap(T, E, K, f));
    }
    up.h_out = at<bf16>(workspace, L.h);
    up.status = status;
    up.zero_acc = use_acc && q.tc_router ? out_acc : nullptr;
    up.zero_floats = static_cast<long long>(T) * D;
    q.shared_launches = shared;

    GroupedGemmLaunch& dn = q.dn;
    dn.gate_up = false;
    dn.w = p->w_down;
    dn.act = up.h_out;
    dn.offsets = pm.offsets;
    dn.sorted_token = pm.sorted_token;
    dn.sorted_w = q.det ? nullptr : pm.sorted_w;
    dn.rows = rows; dn.E = E; dn.D = D; dn.f = f;
    dn.max_group_rows = up.max_group_rows;
    dn.acc_out = q.det || q.rows_mode ? nullptr : out_acc;
    dn.y_out = q.det ? at<float>(workspace, L.y_sorted) : nullptr;
    dn.y16_out = q.rows_mode ? at<bf16>(workspace, L.x_sorted) : nullptr;
    dn.status = status;
    // K slices add into the accumulator in any order: not with the fixed-order combine
    dn.ksplit_max = q.det ? 1 : kSplitMax;
    // without the fixed-order combine, the last launch also writes the bf16 output after a
    // grid-wide step
    unsigned* done = at<unsigned>(workspace, L.status + 64);  // inside the cleared header
    const bf16* residual = reinterpret_cast<const bf16*>(p->residual);
    GroupedGemmLaunch& last = q.shared_launches ? q.sd : dn;
    if (!q.combine) {
        last.final_out = reinterpret_cast<bf16*>(out);
        last.final_rows = T;
        last.done = done;
        last.final_residual = residual;
        last.barrier_budget_ns = grid_wait_budget_ns();
    }
    if (q.shared_launches) {
        GroupedGemmLaunch& su = q.su;
        su.gate_up = true;
        su.w = p->w_shared_gate_up;
        su.act = p->x;
        su.offsets = pm.dense_offsets;
        su.rows = T; su.E = 1; su.D = D; su.f = fs;
        su.h_out = at<bf16>(workspace, L.h_s);
        su.status = status;
        GroupedGemmLaunch& sd = q.sd;
        sd.gate_up = false;
        sd.w = p->w_shared_down;
        sd.act = su.h_out;
        sd.offsets = pm.dense_offsets;
        sd.sorted_token = nullptr;
        sd.sorted_w = sgate;
        sd.rows = T; sd.E = 1; sd.D = D; sd.f = fs;
        sd.acc_out = out_acc;
        sd.status = status;
        sd.ksplit_max = q.det ? 1 : kSplitMax;
    }
    // fixed order: out_acc's shared part (if any) + the routed rows in slot order
    CombineLaunch& c = q.c;
    c.residual = residual;
    c.out_acc = use_acc ? out_acc : nullptr;
    c.y_sorted = q.det ? at<float>(workspace, L.y_sorted) : nullptr;
    c.y16_sorted = q.rows_mode ? at<bf16>(workspace, L.x_sorted) : nullptr;
    c.slot_to_row = pm.slot_to_row;
    c.topk_w = q.det ? tw : nullptr;
    c.T = T; c.D = D; c.K = K;
    c.out = reinterpret_cast<bf16*>(out);
    return q;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape";
        case MOE_ERR_ALIGN: return "pointer not 16-byte aligned";
        case MOE_ERR_CUDA: return "CUDA launch failed";
        case MOE_ERR_TIMEOUT: return "device wait timed out";
        case MOE_ERR_WORKSPACE: return "workspace missing or too small";
        case MOE_ERR_DEVICE: return "inconsistent routing table on the device";
        default: return "unknown status";
    }
}

int moe_version(void) { return 100; }

unsigned long long moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

unsigned long long moe_set_grid_wait_budget_ns(unsigned long long ns) {
    return g_grid_wait_ns.exchange(ns, std::memory_order_relaxed);
}

size_t moe_workspace_size(int T, int D, int E, int K, int f, int f_s) {
    if (check_shape(T, D, E, K, f, f_s) != MOE_OK) return 0;
    return layout(T, D, E, K, f, f_s).total;
}

int moe_route(const moe_bf16* x, const moe_bf16* w_router, const float* logit_bias,
              const moe_bf16* w_shared_gate, int T, int D, int E, int K, int32_t* topk_idx,
              float* topk_w, int32_t* expert_counts, float* shared_gate, void* workspace,
              size_t ws_bytes, void* stream) {
    return moe_route_ex(x, w_router, logit_bias, w_shared_gate, T, D, E, K, MOE_SCORE_SOFTMAX,
                        nullptr, 0u, topk_idx, topk_w, expert_counts, shared_gate, workspace,
                        ws_bytes, stream);
}

int moe_route_ex(const moe_bf16* x, const moe_bf16* w_router, const float* logit_bias,
                 const moe_bf16* w_shared_gate, int T, int D, int E, int K, int score_mode,
                 const float* select_bias, unsigned flags, int32_t* topk_idx, float* topk_w,
                 int32_t* expert_counts, float* shared_gate, void* workspace, size_t ws_bytes,
                 void* stream) {
    int rc = check_shape(T, D, E, K, 128, 0);
    if (rc) return rc;
    if (score_mode != MOE_SCORE_SOFTMAX && score_mode != MOE_SCORE_SIGMOID) return MOE_ERR_ARG;
    if (!w_router || !expert_counts) return MOE_ERR_ARG;
    if (T > 0 && (!x || !topk_idx || !topk_w || (w_shared_gate && !shared_gate))) return MOE_ERR_ARG;
    if (!aligned16(x) || !aligned16(w_router) || (w_shared_gate && !aligned16(w_shared_gate)))
        return MOE_ERR_ALIGN;
    const Layout L = layout(T, D, E, K, 128, 0);
    if (!workspace) return MOE_ERR_WORKSPACE;
    if (ws_bytes < L.offsets) return MOE_ERR_WORKSPACE;  // through the logits region
    cudaStream_t s = as_stream(stream);
    if (cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * E, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (T == 0) return MOE_OK;
    if (cudaMemsetAsync(workspace, 0, L.counts, s) != cudaSuccess) return MOE_ERR_CUDA;
    RouterLaunch a{};
    a.x = reinterpret_cast<const bf16*>(x);
    a.w_router = reinterpret_cast<const bf16*>(w_router);
    a.logit_bias = logit_bias;
    a.w_shared_gate = reinterpret_cast<const bf16*>(w_shared_gate);
    a.T = T; a.D = D; a.E = E; a.K = K;
    a.logits = at<float>(workspace, L.logits);
    a.counters = at<unsigned>(workspace, L.counters);
    a.topk_idx = topk_idx;
    a.topk_w = topk_w;
    a.counts = expert_counts;
    a.shared_gate = shared_gate;
    a.status = at<int>(workspace, L.status);
    a.score_mode = score_mode;
    a.select_bias = select_bias;
    a.bf16_weights = (flags & MOE_FLAG_BF16_WEIGHTS) ? 1 : 0;
    const int sms = num_sms_current();
    const cudaError_t err = router_uses_tensor_cores(T, E) ? launch_router_tc(a, sms, s)
                                                           : launch_router(a, sms, s);
    return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_permute(const int32_t* topk_idx, const float* topk_w, const int32_t* expert_counts, int T,
                int E, int K, int32_t* expert_offsets, int32_t* sorted_token, float* sorted_w,
                int32_t* slot_to_row, void* workspace, void* stream) {
    return moe_permute_ex(topk_idx, topk_w, expert_counts, T, E, K, -1, expert_offsets,
                          sorted_token, sorted_w, slot_to_row, workspace, stream);
}

long long moe_expert_capacity(int T, int K, int E, float capacity_factor, int min_capacity) {
    if (T < 0 || K <= 0 || E <= 0 || min_capacity < 0 || !(capacity_factor > 0.f) ||
        !std::isfinite(capacity_factor))
        return -1;
    const double c = std::ceil(static_cast<double>(capacity_factor) * static_cast<double>(T) *
                               static_cast<double>(K) / static_cast<double>(E));
    const long long cap = c > 9.0e18 ? static_cast<long long>(9.0e18) : static_cast<long long>(c);
    return cap < min_capacity ? min_capacity : cap;
}

int moe_permute_ex(const int32_t* topk_idx, const float* topk_w, const int32_t* expert_counts,
                   int T, int E, int K, long long capacity, int32_t* expert_offsets,
                   int32_t* sorted_token, float* sorted_w, int32_t* slot_to_row,
                   void* workspace, void* stream) {
    int rc = check_shape(T, 128, E, K, 128, 0);
    if (rc) return rc;
    if (!expert_counts || !expert_offsets) return MOE_ERR_ARG;
    if (T > 0 && (!topk_idx || !sorted_token || !slot_to_row || (topk_w && !sorted_w)))
        return MOE_ERR_ARG;
    PermuteLaunch a{};
    a.topk_idx = topk_idx;
    a.topk_w = topk_w;
    a.counts = expert_counts;
    a.T = T; a.E = E; a.K = K;
    a.offsets = expert_offsets;
    a.sorted_token = sorted_token;
    a.sorted_w = sorted_w;
    a.slot_to_row = slot_to_row;
    a.status = workspace ? at<int>(workspace, 0) : nullptr;
    a.hist = workspace ? at<int32_t>(workspace, layout(T, 128, E, K, 128, 0).perm_hist) : nullptr;
    a.capacity = capacity < 0 ? -1 : capacity;
    return launch_permute(a, as_stream(stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_grouped_swiglu(const moe_bf16* x, const int32_t* sorted_token,
                       const int32_t* expert_offsets, const float* sorted_w,
                       const moe_bf16* w_gate_up, const moe_bf16* w_down, int T, int rows, int D,
                       int E, int f, float* y_sorted, float* out_acc, void* workspace,
                       size_t ws_bytes, void* stream) {
    int rc = check_shape(T, D, E, 1, f, 0);
    if (rc) return rc;
    if (rows < 0 || (T == 0 && rows > 0)) return MOE_ERR_ARG;
    if (!sorted_token && rows > T) return MOE_ERR_ARG;
    if (!x || !expert_offsets || !w_gate_up || !w_down || (!y_sorted && !out_acc)) return MOE_ERR_ARG;
    if (!aligned16(x) || !aligned16(w_gate_up) || !aligned16(w_down) ||
        (y_sorted && !aligned16(y_sorted)))
        return MOE_ERR_ALIGN;
    if (!workspace) return MOE_ERR_WORKSPACE;
    const size_t h_off = kAlign;
    const size_t need = align_up(h_off + 2ull * rows * f);
    if (ws_bytes < need) return MOE_ERR_WORKSPACE;
    if (rows == 0) return MOE_OK;
    cudaStream_t s = as_stream(stream);
    const int sms = num_sms_current();
    int* status = at<int>(workspace, 0);
    GroupedGemmLaunch up{};
    up.gate_up = true;
    up.w = w_gate_up;
    up.act = x;
    up.gather_tok = sorted_token;
    up.offsets = expert_offsets;
    up.rows = rows; up.E = E; up.D = D; up.f = f;
    up.h_out = at<bf16>(workspace, h_off);
    up.status = status;
    if (launch_grouped_gemm(up, sms, s) != cudaSuccess) return MOE_ERR_CUDA;
    GroupedGemmLaunch dn{};
    dn.gate_up = false;
    dn.w = w_down;
    dn.act = at<bf16>(workspace, h_off);
    dn.offsets = expert_offsets;
    dn.sorted_token = sorted_token;
    dn.sorted_w = sorted_w;
    dn.rows = rows; dn.E = E; dn.D = D; dn.f = f;
    dn.acc_out = out_acc;
    dn.y_out = y_sorted;
    dn.status = status;
    return launch_grouped_gemm(dn, sms, s, true) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_combine(const float* out_acc, const float* y_sorted, const int32_t* slot_to_row,
                const float* topk_w, const moe_bf16* shared_out, const float* shared_gate, int T,
                int D, int K, moe_bf16* out, void* stream) {
    if (T < 0 || D <= 0 || D % 8 || K < 0) return MOE_ERR_ARG;
    if (!out || (y_sorted && (!slot_to_row || K <= 0)) || (shared_out && !shared_gate))
        return MOE_ERR_ARG;
    if (!aligned16(out) || (out_acc && !aligned16(out_acc)) || (y_sorted && !aligned16(y_sorted)) ||
        (shared_out && !aligned16(shared_out)))
        return MOE_ERR_ALIGN;
    CombineLaunch a{};
    a.out_acc = out_acc;
    a.y_sorted = y_sorted;
    a.slot_to_row = slot_to_row;
    a.topk_w = topk_w;
    a.shared_out = reinterpret_cast<const bf16*>(shared_out);
    a.shared_gate = shared_gate;
    a.T = T; a.D = D; a.K = K;
    a.out = reinterpret_cast<bf16*>(out);
    return launch_combine(a, num_sms_current(), as_stream(stream)) == cudaSuccess ? MOE_OK
                                                                                   : MOE_ERR_CUDA;
}

int moe_layer_forward(const moe_layer_params* p, moe_bf16* out, void* workspace, size_t ws_bytes,
                      void* stream) {
    int rc = check_layer(p, out);
    if (rc) return rc;
    if (p->T > 0 && (!p->x || !out)) return MOE_ERR_ARG;
    if (!workspace) return MOE_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return MOE_ERR_ALIGN;
    const Layout L = layout(p->T, p->D, p->E, p->K, p->f, p->f_s);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    if (p->T == 0) return MOE_OK;

    cudaStream_t s = as_stream(stream);
    const int sms = num_sms_current();
    LayerPlan q = plan_layer(p, out, workspace, sms);
    auto mark = [&](int i) {
        return p->step_events == nullptr || p->step_events[i] == nullptr ||
               cudaEventRecord(reinterpret_cast<cudaEvent_t>(p->step_events[i]), s) == cudaSuccess;
    };

    if (!mark(MOE_EV_START)) return MOE_ERR_CUDA;
    // the only clear: status word, router tickets, expert counts (a few KB); the fp32
    // accumulator is cleared by the CUDA-core router kernel, or (tensor-core router, many
    // tokens) by the gate_up kernel's epilogue warps while its first tiles accumulate
    if (cudaMemsetAsync(workspace, 0, L.zero_end, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (!mark(MOE_EV_ROUTER)) return MOE_ERR_CUDA;
    if ((q.tc_router ? launch_router_tc(q.r, sms, s) : launch_router(q.r, sms, s)) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (!mark(MOE_EV_PERMUTE)) return MOE_ERR_CUDA;
    if (launch_permute(q.pm, s, true) != cudaSuccess) return MOE_ERR_CUDA;
    if (!mark(MOE_EV_GATE_UP) || launch_grouped_gemm(q.up, sms, s, true) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (!mark(MOE_EV_DOWN) || launch_grouped_gemm(q.dn, sms, s, true) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (!mark(MOE_EV_SHARED)) return MOE_ERR_CUDA;
    if (q.shared_launches &&
        (launch_grouped_gemm(q.su, sms, s, true) != cudaSuccess ||
         launch_grouped_gemm(q.sd, sms, s, true) != cudaSuccess))
        return MOE_ERR_CUDA;
    if (!mark(MOE_EV_COMBINE)) return MOE_ERR_CUDA;
    if (q.combine && launch_combine(q.c, sms, s, true) != cudaSuccess) return MOE_ERR_CUDA;
    return mark(MOE_EV_END) ? MOE_OK : MOE_ERR_CUDA;
}

int moe_layer_plan(const moe_layer_params* p, unsigned* step_mask, int* launches) {
    int rc = check_layer(p, nullptr);
    if (rc) return rc;
    unsigned mask = 0;
    int n = 0;
    if (p->T > 0) {
        const int sms = num_sms_current();
        // nothing is dereferenced: the plan only needs the workspace's layout
        const LayerPlan q = plan_layer(p, nullptr, reinterpret_cast<void*>(kAlign), sms);
        const int nr = q.tc_router ? 2 : 1;
        const int np = permute_chunks(static_cast<long long>(p->T) * p->K) > 1 ? 2 : 1;
        const int nu = grouped_gemm_launches(q.up, sms), nd = grouped_gemm_launches(q.dn, sms);
        const int ns = q.shared_launches ? grouped_gemm_launches(q.su, sms) + grouped_gemm_launches(q.sd, sms) : 0;
        const int nc = q.combine ? 1 : 0;
        const int per[] = {nr, np, nu, nd, ns, nc};
        for (int i = 0; i < 6; ++i) {
            if (per[i]) mask |= 1u << (MOE_EV_ROUTER + i);
            n += per[i];
        }
    }
    if (step_mask) *step_mask = mask;
    if (launches) *launches = n;
    return MOE_OK;
}

int moe_ep_dispatch_rows(const moe_bf16* x, const int32_t* sorted_token, int rows, int D,
                         moe_bf16* x_sorted, void* stream) {
    if (rows < 0 || D <= 0 || D % 8) return MOE_ERR_ARG;
    if (rows > 0 && (!x || !sorted_token || !x_sorted)) return MOE_ERR_ARG;
    if (!aligned16(x) || !aligned16(x_sorted)) return MOE_ERR_ALIGN;
    return launch_gather_rows(reinterpret_cast<const bf16*>(x), sorted_token, rows, D,
                              reinterpret_cast<bf16*>(x_sorted), num_sms_current(),
                              as_stream(stream), false) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

int moe_ep_recv_layout(const int32_t* recv_counts, int G, int El, int n, int32_t* recv_offsets,
                       int32_t* recv_row, void* workspace, void* stream) {
    if (G <= 0 || El <= 0 || n < 0) return MOE_ERR_ARG;
    if (static_cast<long long>(G) * El > 512) return MOE_ERR_UNSUPPORTED;
    if (!recv_counts || !recv_offsets || (n > 0 && !recv_row)) return MOE_ERR_ARG;
    return launch_ep_recv_layout(recv_counts, G, El, n, recv_offsets, recv_row,
                                 workspace ? at<int>(workspace, 0) : nullptr,
                                 as_stream(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

int moe_ep_return_rows(const float* y, const int32_t* recv_row, int n, int D, float* y_ret,
                       void* stream) {
    if (n < 0 || D <= 0 || D % 4) return MOE_ERR_ARG;
    if (n > 0 && (!y || !recv_row || !y_ret)) return MOE_ERR_ARG;
    if (!aligned16(y) || !aligned16(y_ret)) return MOE_ERR_ALIGN;
    return launch_ep_return_rows(y, recv_row, n, D, y_ret, num_sms_current(),
                                 as_stream(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

int moe_read_device_status(void* workspace, void* stream) {
    if (!workspace) return MOE_ERR_WORKSPACE;
    cudaStream_t s = as_stream(stream);
    int h = 0;
    if (cudaMemcpyAsync(&h, workspace, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof(int), s) != cudaSuccess) return MOE_ERR_CUDA;
    return h;
}

}  // extern "C"
