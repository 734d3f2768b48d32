// permute.cu -- group the (token, slot) pairs by expert and build the inverse map.
//
// "MoE" (llm.rainlin.net), section 3.2: each routed expert gathers the tokens routed to
// it (the expert loop's torch.where over the expert mask, then hidden_states[token_idx]).
// "1.6 混合专家（MoE）", section 2: tokens are first grouped by route, computed per
// expert, then merged back in their original order.
//
// The (token, slot) entries are cut into chunks of consecutive entries.  With one chunk a
// single CTA does everything; otherwise permute_hist_kernel counts each chunk's entries per
// expert and permute_scatter_kernel gives every entry its row:
//   row = offsets[e] + (entries of e in earlier chunks) + (entries of e earlier in this
//         chunk),
// offsets being the exclusive scan of the counts -- ascending (token, slot) order inside
// each group, i.e. a stable counting sort by expert.  With an expert capacity C
// ("1.6 混合专家（MoE）", section 三, expert capacity and token dropping) an entry whose
// place in its group is C or more is dropped (slot_to_row = -1) and the groups are the
// kept prefixes, min(count, C) rows each.
// The token rows themselves are never copied: the grouped GEMM gathers them from x.
#include <algorithm>

#include "common.cuh"
#include "permute_body.cuh"

namespace moe {
namespace {

constexpr int kPermThreads = 1024;
constexpr int kPermWarps = kPermThreads / 32;
constexpr int kSingleChunk = 4096;  // entries one CTA takes alone (decode sizes)
constexpr int kMaxChunks = 256;

// hist[c * E + e] = entries of chunk c routed to expert e
__global__ void __launch_bounds__(kPermThreads) permute_hist_kernel(PermuteLaunch a,
                                                                    int chunk_len) {
    extern __shared__ int cnt[];  // [E]
    const int tid = threadIdx.x, lane = tid & 31;
    const int E = a.E;
    grid_dep_wait();  // routing comes from the router
    grid_dep_launch();
    for (int e = tid; e < E; e += kPermThreads) cnt[e] = 0;
    __syncthreads();
    const ChunkRange r = chunk_range(blockIdx.x, chunk_len, a.T * a.K);
    for (int j0 = r.begin; j0 < r.end; j0 += kPermThreads) {
        const int j = j0 + tid;
        const int e = j < r.end ? __ldg(a.topk_idx + j) : -1;
        const bool ok = e >= 0 && e < E;
        const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1);
        if (ok && (peers & ((1u << lane) - 1u)) == 0) atomicAdd(&cnt[e], __popc(peers));
    }
    __syncthreads();
    for (int e = tid; e < E; e += kPermThreads)
        a.hist[static_cast<size_t>(blockIdx.x) * E + e] = cnt[e];
}

// Rows of chunk blockIdx.x (permute_scatter_chunk).
__global__ void __launch_bounds__(kPermThreads) permute_scatter_kernel(PermuteLaunch a,
                                                                       int chunk_len,
                                                                       int chunks) {
    extern __shared__ int sm[];
    grid_dep_wait();  // counts (router) and chunk histograms (previous kernel)
    grid_dep_launch();
    permute_scatter_chunk<kPermThreads>(a, chunk_len, chunks, blockIdx.x, sm);
}


// x_sorted[r] = x[sorted_token[r]]: the token rows in expert order, 16-byte vectors,
// grid-stride (for the CTA-pair GEMM, whose operand rows must be contiguous).
__global__ void __launch_bounds__(256) gather_rows_kernel(const bf16* x, const int32_t* tok,
                                                          int rows, int D, bf16* out) {
    grid_dep_wait();
    grid_dep_launch();
    const int vec = D / 8;
    const long long n = static_cast<long long>(rows) * vec;
    const uint4* src = reinterpret_cast<const uint4*>(x);
    uint4* dst = reinterpret_cast<uint4*>(out);
    for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n; i += 256ll * gridDim.x) {
        const int r = static_cast<int>(i / vec);
        const int c = static_cast<int>(i - static_cast<long long>(r) * vec);
        dst[i] = __ldg(src + static_cast<size_t>(__ldg(tok + r)) * vec + c);
    }
}

}  // namespace

int permute_chunks(long long entries) {
    if (entries <= kSingleChunk) return 1;
    const long long want = std::min<long long>(kMaxChunks, (entries + kPermThreads - 1) / kPermThreads);
    const long long len = (entries + want - 1) / want;
    return static_cast<int>((entries + len - 1) / len);
}

cudaError_t launch_permute(const PermuteLaunch& a, cudaStream_t s, bool pdl) {
    const long long entries = static_cast<long long>(a.T) * a.K;
    // without a histogram buffer one CTA walks every entry
    const int chunks = a.hist ? permute_chunks(entries) : 1;
    const int chunk_len = static_cast<int>(chunks > 1 ? (entries + chunks - 1) / chunks : entries);
    cudaError_t err;
    if (chunks > 1) {
        err = launch_kernel(permute_hist_kernel, dim3(chunks), dim3(kPermThreads),
                            sizeof(int) * static_cast<size_t>(a.E), s, pdl, a, chunk_len);
        count_launches(1);
        if (err != cudaSuccess) return err;
    }
    const size_t smem = sizeof(int) * (static_cast<size_t>(kPermWarps) * a.E + 3 * a.E + 1);
    err = set_smem_limit(reinterpret_cast<const void*>(permute_scatter_kernel), smem);
    if (err != cudaSuccess) return err;
    err = launch_kernel(permute_scatter_kernel, dim3(chunks), dim3(kPermThreads), smem, s,
                        pdl || chunks > 1, a, chunk_len, chunks);
    count_launches(1);
    return err;
}

cudaError_t launch_gather_rows(const bf16* x, const int32_t* tok, int rows, int D, bf16* out,
                               int num_sms, cudaStream_t s, bool pdl) {
    if (rows == 0) return cudaSuccess;
    const long long n = static_cast<long long>(rows) * (D / 8);
    const int blocks = static_cast<int>(std::min<long long>((n + 255) / 256, 8ll * num_sms));
    cudaError_t err = launch_kernel(gather_rows_kernel, dim3(blocks), dim3(256), 0, s, pdl, x, tok,
                                    rows, D, out);
    count_launches(1);
    return err;
}

}  // namespace moe
