// permute.cu -- group the (token, slot) pairs by expert and build the inverse map.
//
// "MoE" (llm.rainlin.net), section 3.2: each routed expert gathers the tokens routed to
// it (the expert loop's torch.where over the expert mask, then hidden_states[token_idx]).
// "1.6 混合专家（MoE）", section 2: tokens are first grouped by route, computed per
// expert, then merged back in their original order.
//
// permute_kernel: one CTA per expert e.
//   offsets[e] = sum_{e' < e} counts[e']            (block reduction over <= 512 counts)
//   a block-wide ballot scan walks the T*K routing entries in order and writes the
//   entries equal to e to rows offsets[e] + rank  -> ascending token order (stable).
// permute_small_kernel: the same result from one CTA when T*K <= 4096 (decode sizes).
// The token rows themselves are never copied: the grouped GEMM gathers them from x.
#include <algorithm>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kPermThreads = 512;

__global__ void __launch_bounds__(kPermThreads) permute_kernel(PermuteLaunch a) {
    __shared__ int warp_tot[kPermThreads / 32];
    __shared__ int warp_pre[kPermThreads / 32];
    __shared__ int s_off;
    __shared__ int s_block_hits;
    const int e = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int total = a.T * a.K;

    grid_dep_wait();  // routing and counts come from the router
    grid_dep_launch();

    int v = 0;
    for (int i = tid; i < e; i += kPermThreads) v += a.counts[i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) warp_tot[warp] = v;
    __syncthreads();
    if (tid == 0) {
        int s = 0;
        for (int w = 0; w < kPermThreads / 32; ++w) s += warp_tot[w];
        s_off = s;
    }
    __syncthreads();
    const int off = s_off;
    const int n_e = a.counts[e];
    if (tid == 0) {
        a.offsets[e] = off;
        if (e == a.E - 1) {
            a.offsets[a.E] = off + n_e;
            if (off + n_e != total) set_status(a.status, MOE_ERR_DEVICE);
        }
        if (e == 0 && a.dense_offsets) {
            a.dense_offsets[0] = 0;
            a.dense_offsets[1] = a.T;
        }
    }
    if (n_e == 0) return;

    const unsigned lt_mask = (1u << lane) - 1u;
    int base = 0;
    for (int j0 = 0; j0 < total; j0 += kPermThreads) {
        const int j = j0 + tid;
        const bool hit = (j < total) && (__ldg(a.topk_idx + j) == e);
        const unsigned b = __ballot_sync(0xffffffffu, hit);
        if (lane == 0) warp_tot[warp] = __popc(b);
        __syncthreads();
        if (warp == 0) {
            const int c = (lane < kPermThreads / 32) ? warp_tot[lane] : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            if (lane < kPermThreads / 32) warp_pre[lane] = incl - c;
            if (lane == kPermThreads / 32 - 1) s_block_hits = incl;
        }
        __syncthreads();
        if (hit) {
            const int r = base + warp_pre[warp] + __popc(b & lt_mask);
            if (r < n_e) {
                const int row = off + r;
                a.sorted_token[row] = j / a.K;
                if (a.topk_w) a.sorted_w[row] = __ldg(a.topk_w + j);
                a.slot_to_row[j] = row;
            }
        }
        base += s_block_hits;
        __syncthreads();
    }
    if (tid == 0 && base != n_e) set_status(a.status, MOE_ERR_DEVICE);

}


// Small problems (T*K <= kSmallEntries): one CTA of 1024 threads does the whole
// permutation.  offsets = exclusive scan of the counts; then the entries are walked in
// chunks of 1024 in order, and an entry's row is offsets[e] + (entries of e in earlier
// chunks) + (entries of e in earlier warps of this chunk) + (its rank among the lanes of
// its warp holding e, from __match_any_sync) -- ascending token order, as the
// one-CTA-per-expert kernel gives.
constexpr int kSmallEntries = 4096;
constexpr int kSmallThreads = 1024;
constexpr int kSmallWarps = kSmallThreads / 32;

__global__ void __launch_bounds__(kSmallThreads) permute_small_kernel(PermuteLaunch a) {
    extern __shared__ int sm[];
    int* warp_cnt = sm;                          // [kSmallWarps][E]
    int* base = warp_cnt + kSmallWarps * a.E;    // [E] rows of e placed so far
    int* off = base + a.E;                       // [E + 1]
    __shared__ int warp_sums[kSmallWarps];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = a.E, total = a.T * a.K;

    grid_dep_wait();
    grid_dep_launch();

    // offsets: exclusive scan of counts (E <= 512 < kSmallThreads)
    const int c = tid < E ? a.counts[tid] : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int s = warp_sums[lane];
        int ws = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, ws, o);
            if (lane >= o) ws += v;
        }
        warp_sums[lane] = ws - s;  // exclusive prefix of the warps
    }
    __syncthreads();
    if (tid < E) {
        off[tid] = warp_sums[warp] + incl - c;
        base[tid] = 0;
        a.offsets[tid] = off[tid];
    }
    if (tid == 0) {
        off[E] = total;
        a.offsets[E] = total;
        if (a.dense_offsets) {
            a.dense_offsets[0] = 0;
            a.dense_offsets[1] = a.T;
        }
    }
    const unsigned lt = (1u << lane) - 1u;
    for (int j0 = 0; j0 < total; j0 += kSmallThreads) {
        for (int i = tid; i < kSmallWarps * E; i += kSmallThreads) warp_cnt[i] = 0;
        __syncthreads();
        const int j = j0 + tid;
        const bool live = j < total;
        const int e = live ? __ldg(a.topk_idx + j) : -1;
        const bool ok = live && e >= 0 && e < E;
        const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1);
        const int rank = __popc(peers & lt);
        if (ok && rank == 0) warp_cnt[warp * E + e] = __popc(peers);
        if (live && !ok) set_status(a.status, MOE_ERR_DEVICE);
        __syncthreads();
        if (tid < E) {  // prefix over the warps of this chunk, per expert
            int run = base[tid];
            for (int w = 0; w < kSmallWarps; ++w) {
                const int v = warp_cnt[w * E + tid];
                warp_cnt[w * E + tid] = run;
                run += v;
            }
            base[tid] = run;
        }
        __syncthreads();
        if (ok) {
            const int row = off[e] + warp_cnt[warp * E + e] + rank;
            if (row < off[e + 1]) {
                a.sorted_token[row] = j / a.K;
                if (a.topk_w) a.sorted_w[row] = __ldg(a.topk_w + j);
                a.slot_to_row[j] = row;
            } else {
                set_status(a.status, MOE_ERR_DEVICE);
            }
        }
        __syncthreads();
    }
    if (tid < E && base[tid] != off[tid + 1] - off[tid]) set_status(a.status, MOE_ERR_DEVICE);
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

cudaError_t launch_permute(const PermuteLaunch& a, cudaStream_t s, bool pdl) {
    cudaError_t err;
    if (static_cast<long long>(a.T) * a.K <= kSmallEntries) {
        const size_t smem = sizeof(int) * (static_cast<size_t>(kSmallWarps) * a.E + 2 * a.E + 1);
        err = cudaFuncSetAttribute(permute_small_kernel,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(smem));
        if (err != cudaSuccess) return err;
        err = launch_kernel(permute_small_kernel, dim3(1), dim3(kSmallThreads), smem, s, pdl, a);
    } else {
        err = launch_kernel(permute_kernel, dim3(a.E), dim3(kPermThreads), 0, s, pdl, a);
    }
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
