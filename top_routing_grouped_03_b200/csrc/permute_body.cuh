// permute_body.cuh -- the row placement of the permutation kernel (one chunk of entries
// per CTA), written for any CTA size NT >= E.
//
// "MoE" (llm.rainlin.net), section 3.2: each routed expert gathers the tokens routed to
// it; rows of a group are in ascending (token, slot) order, a stable counting sort by
// expert.  Within a chunk, NT entries at a time: an entry's row is offsets[e] + base[e]
// (entries of e before this step) + (entries of e in earlier warps of this step) + (its
// rank among the lanes of its warp holding e, from __match_any_sync).  With an expert
// capacity C ("1.6 混合专家（MoE）", section 三) an entry whose place in its group is C or
// more is dropped (slot_to_row = -1).
#pragma once

#include "common.cuh"

namespace moe {

// [c*chunk_len, min(total, (c+1)*chunk_len)): the entries of chunk c
struct ChunkRange {
    int begin, end;
};
__device__ __forceinline__ ChunkRange chunk_range(int c, int chunk_len, int total) {
    const long long b = static_cast<long long>(c) * chunk_len;
    const long long e = b + chunk_len;
    return {static_cast<int>(b < total ? b : total), static_cast<int>(e < total ? e : total)};
}

// Places the entries of chunk c.  Needs E <= NT and dynamic shared memory `sm` of
// (NT / 32 * E + 3 * E + 1) ints.  The routing (topk_idx, topk_w, counts) is read through
// L2 (ld.cg), so it may have been written earlier in the same kernel by other CTAs.
template <int NT>
__device__ __forceinline__ void permute_scatter_chunk(const PermuteLaunch& a, int chunk_len,
                                                      int chunks, int c, int* sm) {
    constexpr int kPermThreads = NT;
    constexpr int kPermWarps = NT / 32;
    static_assert(kPermWarps <= 32, "one warp scans the warp sums");
    int* warp_cnt = sm;                          // [kPermWarps][E]
    int* base = warp_cnt + kPermWarps * a.E;     // [E] entries of e placed before this step
    int* off = base + a.E;                       // [E + 1] first row of each (kept) group
    int* raw = off + a.E + 1;                    // [E] entries of each expert
    __shared__ int warp_sums[kPermWarps];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = a.E, total = a.T * a.K;
    const unsigned lt = (1u << lane) - 1u;

    // counts: from the router, or counted here -- from every chunk's histogram, or (one
    // chunk) by a first pass over the entries
    int n = 0;
    if (a.counts) {
        n = tid < E ? __ldcg(a.counts + tid) : 0;
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
                const int e = j < total ? __ldcg(a.topk_idx + j) : -1;
                const bool ok = e >= 0 && e < E;
                const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1);
                if (ok && (peers & lt) == 0) atomicAdd(&tot[e], __popc(peers));
            }
        }
        __syncthreads();
        n = tid < E ? tot[tid] : 0;
        __syncthreads();
    }
    if (c == 0 && a.counts_out && tid < E) a.counts_out[tid] = n;
    // rows each group keeps: all its entries, or the first `capacity` of them
    const int kept = (a.capacity >= 0 && n > a.capacity) ? static_cast<int>(a.capacity) : n;
    // offsets: exclusive scan of the kept counts (E <= NT: one expert per thread)
    int incl = kept;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int sw = lane < kPermWarps ? warp_sums[lane] : 0;
        int ws = sw;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, ws, o);
            if (lane >= o) ws += v;
        }
        if (lane < kPermWarps) warp_sums[lane] = ws - sw;  // exclusive prefix of the warps
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
        const int e = live ? __ldcg(a.topk_idx + j) : -1;
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
                    if (a.topk_w) a.sorted_w[row] = __ldcg(a.topk_w + j);
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

}  // namespace moe
