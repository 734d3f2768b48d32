// route_noalloc.cu -- moe_route_noalloc: the router step with its scratch memory held in a
// fixed device array of this library, so the caller passes no workspace at all.
//
// The router needs scratch for the fp32 logits of every token ([T, E+1] floats, the last
// column is the shared-expert gate logit) and for one completion ticket per block of 8
// tokens.  moe_route takes that from the caller's workspace; this variant takes it from
// g_route_scratch below.  Nothing here allocates: the array exists in every device context
// that loads the library, for the life of the process.
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr size_t kScratchBytes = size_t(1) << 20;  // 1 MiB: logits, then tickets
constexpr size_t kScratchAlign = 256;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of g_route_scratch in the current device's context, looked up once per
// device (the host-side name of the array is only a stand-in, never a device address).
int scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr)
            return MOE_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

size_t round_up(size_t v) { return (v + kScratchAlign - 1) & ~(kScratchAlign - 1); }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" int moe_route_noalloc(const moe_bf16* x, const moe_bf16* w_router,
                                 const float* logit_bias, const moe_bf16* w_shared_gate, int T,
                                 int D, int E, int K, int32_t* topk_idx, float* topk_w,
                                 int32_t* expert_counts, float* shared_gate, void* stream) {
    if (T < 0 || D <= 0 || E <= 0 || K <= 0) return MOE_ERR_ARG;
    if (E > 512 || K > 16 || K > E || D % 128 || D > 8192) return MOE_ERR_UNSUPPORTED;
    if (!w_router || !expert_counts) return MOE_ERR_ARG;
    if (T > 0 && (!x || !topk_idx || !topk_w || (w_shared_gate && !shared_gate))) return MOE_ERR_ARG;
    auto misaligned = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
    if (misaligned(x) || misaligned(w_router) || (w_shared_gate && misaligned(w_shared_gate)))
        return MOE_ERR_ALIGN;
    const size_t logits_bytes = round_up(sizeof(float) * static_cast<size_t>(T) * (E + 1));
    const size_t ticket_bytes = sizeof(unsigned) * static_cast<size_t>((T + 7) / 8);
    if (logits_bytes + ticket_bytes > kScratchBytes) return MOE_ERR_UNSUPPORTED;

    void* scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != MOE_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * E, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (T == 0) return MOE_OK;
    unsigned* tickets = reinterpret_cast<unsigned*>(static_cast<unsigned char*>(scratch) + logits_bytes);
    // The tickets must start at zero; the logits are fully written before they are read.
    if (cudaMemsetAsync(tickets, 0, ticket_bytes, s) != cudaSuccess) return MOE_ERR_CUDA;

    RouterLaunch a{};
    a.x = reinterpret_cast<const bf16*>(x);
    a.w_router = reinterpret_cast<const bf16*>(w_router);
    a.logit_bias = logit_bias;
    a.w_shared_gate = reinterpret_cast<const bf16*>(w_shared_gate);
    a.T = T; a.D = D; a.E = E; a.K = K;
    a.logits = static_cast<float*>(scratch);
    a.counters = tickets;
    a.topk_idx = topk_idx;
    a.topk_w = topk_w;
    a.counts = expert_counts;
    a.shared_gate = shared_gate;
    a.status = nullptr;
    int sms = 0, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return MOE_ERR_CUDA;
    return launch_router(a, sms, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
