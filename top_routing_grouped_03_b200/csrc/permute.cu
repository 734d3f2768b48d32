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

namespace moe {
namespace {

constexpr int kPermThreads = 1024;
constexpr int kPermWarps = kPermThreads / 32;
constexpr int kSingleChunk = 4096;  // entries one CTA takes alone (decode sizes)
constexpr int kMaxChunks = 256;

// [c*chunk_len, min(total, (c+1)*chunk_len)): the entries of chunk c
struct ChunkRange {
    int begin, end;
};
__device__ __forceinline__ ChunkRange chunk_range(int c, int chunk_len, int total) {
    const long long b = static_cast<long long>(c) * chunk_len;
    const long long e = b + chunk_len;
    return {static_cast<int>(b < total ? b : total), static_cast<int>(e < total ? e : total)};
}

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

// Rows of chunk blockIdx.x.  Inside a chunk, 1024 entries at a time: an entry's row is
// offsets[e] + base[e] (entries of e before this step) + (entries of e in earlier warps of
// this step) + (its rank among the lanes of its warp holding e, from __match_any_sync).
__global__ void __launch_bounds__(kPermThreads) permute_scatter_kernel(PermuteLaunch a,
                                                                       int chunk_len,
                                                                       int chunks) {
    extern __shared__ int sm[];
    int* warp_cnt = sm;                          // [kPermWarps][E]
    int* base = warp_cnt + kPermWarps * a.E;     // [E] entries of e placed before this step
    int* off = base + a.E;                       // [E + 1] first row of each (kept) group
    int* raw = off + a.E + 1;                    // [E] entries of each expert
    __shared__ int warp_sums[kPermWarps];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = a.E, total = a.T * a.K;
    const int c = blockIdx.x;
    const unsigned lt = (1u << lane) - 1u;

    grid_dep_wait();  // counts (router) and chunk histograms (previous kernel)
    grid_dep_launch();

    // counts: from the router, or counted here -- from every chunk's histogram, or (one
    // chunk) by a first pass over the entries
    int n = 0;
    if (a.counts) {
        n = tid < E ? a.counts[tid] : 0;
    } else {
        int* tot = warp_cnt;  // scratch until the walk below clears it
        for (int e = tid; e < E; e += kPermThreads) tot[e] = 0;
        __syncthreads();
        if (chunks > 1) {
            for (int i = tid; i < chunks * E; i += kPermThreads) {
                const int v = a.hist[i];
                if (v) atomicAdd(&tot[i % E], v);
            }
        } else {
            for (int j0 = 0; j0 < total; j0 += kPermThreads) {
                const int j = j0 + tid;
                const int e = j < total ? __ldg(a.topk_idx + j) : -1;
                const bool ok = e >= 0 && e < E;
                const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1);
                if (ok && (peers & lt) == 0) atomicAdd(&tot[e], __popc(peers));
            }
        }
        __syncthreads();
        n = tid < E ? tot[tid] : 0;
        if (c == 0 && a.counts_out && tid < E) a.counts_out[tid] = n;
        __syncthreads();
    }
    // rows each group keeps: all its entries, or the first `capacity` of them
    const int kept = (a.capacity >= 0 && n > a.capacity) ? static_cast<int>(a.capacity) : n;
    // offsets: exclusive scan of the kept counts (E <= 512 < kPermThreads)
    int incl = kept;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int sw = warp_sums[lane];
        int ws = sw;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, ws, o);
            if (lane >= o) ws += v;
        }
        warp_sums[lane] = ws - sw;  // exclusive prefix of the warps
    }
    __syncthreads();
    if (tid < E) {
        off[tid] = warp_sums[warp] + incl - kept;
        raw[tid] = n;
        base[tid] = 0;
        if (c == 0) a.offsets[tid] = off[tid];
        if (tid == E - 1) {
            off[E] = warp_sums[warp] + incl;  // rows kept in all (T*K without a capacity)
            if (c == 0) a.offsets[E] = off[E];
        }
    }
    if (tid == 0) {
        if (c == 0) {
            if (a.dense_offsets) {
                a.dense_offsets[0] = 0;
                a.dense_offsets[1] = a.T;
            }
        }
    }
    __syncthreads();
    // with a capacity, rows [kept total, T*K) belong to no group: token 0, weight 0
    if (c == 0 && a.capacity >= 0) {
        for (int row = off[E] + tid; row < total; row += kPermThreads) {
            a.sorted_token[row] = 0;
            if (a.topk_w) a.sorted_w[row] = 0.f;
        }
    }
    // entries of each expert in the chunks before this one
    for (int i = tid; i < c * E; i += kPermThreads) {
        const int v = a.hist[i];
        if (v) atomicAdd(&base[i % E], v);
    }
    const ChunkRange r = chunk_range(c, chunk_len, total);
    for (int j0 = r.begin; j0 < r.end; j0 += kPermThreads) {
        for (int i = tid; i < kPermWarps * E; i += kPermThreads) warp_cnt[i] = 0;
        __syncthreads();
        const int j = j0 + tid;
        const bool live = j < r.end;
        const int e = live ? __ldg(a.topk_idx + j) : -1;
        const bool ok = live && e >= 0 && e < E;
        const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1);
        const int rank = __popc(peers & lt);
        if (ok && rank == 0) warp_cnt[warp * E + e] = __popc(peers);
        if (live && !ok) set_status(a.status, MOE_ERR_DEVICE);
        __syncthreads();
        if (tid < E) {  // prefix over the warps of this step, per expert
            int run = base[tid];
            for (int w = 0; w < kPermWarps; ++w) {
                const int v = warp_cnt[w * E + tid];
                warp_cnt[w * E + tid] = run;
                run += v;
            }
            base[tid] = run;
        }
        __syncthreads();
        if (ok) {
            const int in_group = warp_cnt[warp * E + e] + rank;  // entries of e before it
            if (a.capacity >= 0 && in_group >= a.capacity) {
                a.slot_to_row[j] = -1;  // past the expert's capacity: dropped
            } else {
                const int row = off[e] + in_group;
                // counts that disagree with the entries can push a row out of its group,
                // or (when they do not sum to T*K) out of the arrays: flag it, write nothing
                if (row >= 0 && row < off[e + 1] && row < total) {
                    a.sorted_token[row] = j / a.K;
                    if (a.topk_w) a.sorted_w[row] = __ldg(a.topk_w + j);
                    a.slot_to_row[j] = row;
                } else {
                    set_status(a.status, MOE_ERR_DEVICE);
                }
            }
        }
        __syncthreads();
    }
    // the last chunk has seen every entry: each expert's entries must match its count
    if (c == chunks - 1 && tid < E && base[tid] != raw[tid]) set_status(a.status, MOE_ERR_DEVICE);
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
    err = cudaFuncSetAttribute(permute_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
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
