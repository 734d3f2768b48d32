// ep.cu -- the device-side layouts of expert parallelism.
//
// "1.6 混合专家（MoE）" (llm.satori-ai.cn), expert parallelism: the experts are spread over G
// devices; every device routes its own tokens, sends each token row to the devices that
// hold its experts (dispatch, an all-to-all), those run their experts on the rows they
// received, and the results travel back (combine, a second all-to-all) to be summed with
// the routing weights.  Rank r holds experts [r El, (r + 1) El), El = E / G.
//
// After the permutation of a rank's own tokens (moe_permute) the rows bound for rank d are
// already contiguous: [offsets[d El], offsets[(d + 1) El]) of the expert-sorted order, so
// the send side needs only the token rows gathered into that order (moe_ep_dispatch_rows).  The
// receive buffer holds, source by source, each source's rows for this rank's experts in
// expert order; ep_recv_layout_kernel turns the [G, El] table of received counts into the
// expert-major grouping the grouped GEMM takes (group offsets, and for every expert-major
// row the receive-buffer row it reads -- the GEMM gathers rows through that map, nothing is
// copied); ep_return_rows_kernel puts the per-row expert outputs back into receive-buffer
// order, which is the order the sources expect them back in.
#include <algorithm>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kLayoutThreads = 1024;

// One CTA.  recv_counts[s * El + e]: rows source s sent for local expert e.
//   src_start(s, e) = rows of sources before s + rows of s for experts before e
//   dst_start(e, s) = rows of experts before e (all sources) + rows of e from sources before s
// recv_offsets[e] = dst_start(e, 0); recv_offsets[El] = n; recv_row[dst_start(e, s) + i] =
// src_start(s, e) + i.  Counts that do not add up to n set MOE_ERR_DEVICE, leave every group
// empty and recv_row unwritten.
__global__ void __launch_bounds__(kLayoutThreads) ep_recv_layout_kernel(
    const int32_t* recv_counts, int G, int El, int n, int32_t* recv_offsets, int32_t* recv_row,
    int* status) {
    extern __shared__ int sm[];
    int* cnt = sm;                    // [G * El]
    int* src_start = cnt + G * El;    // [G * El]
    int* dst_start = src_start + G * El;  // [G * El]
    __shared__ int s_total;
    const int tid = threadIdx.x;
    const int GE = G * El;
    grid_dep_wait();
    for (int i = tid; i < GE; i += kLayoutThreads) cnt[i] = max(0, recv_counts[i]);
    __syncthreads();
    if (tid == 0) {
        // source-major running sum (receive-buffer order), then expert-major (group order)
        int run = 0;
        for (int i = 0; i < GE; ++i) {
            src_start[i] = run;
            run += cnt[i];
        }
        s_total = run;
        run = 0;
        for (int e = 0; e < El; ++e) {
            for (int s = 0; s < G; ++s) {
                dst_start[s * El + e] = run;
                run += cnt[s * El + e];
            }
        }
    }
    __syncthreads();
    // counts that do not add up to the rows received: report, and leave every group empty
    // (the grouped GEMM then reads nothing through recv_row)
    const bool consistent = s_total == n;
    if (tid == 0 && !consistent) set_status(status, MOE_ERR_DEVICE);
    for (int e = tid; e <= El; e += kLayoutThreads)
        recv_offsets[e] = !consistent ? 0 : (e < El ? dst_start[e] : n);
    // one warp per (source, expert) segment, lanes over its rows
    const int warp = tid >> 5, lane = tid & 31;
    for (int i = warp; i < GE && consistent; i += kLayoutThreads / 32) {
        const int c = cnt[i], src = src_start[i], dst = dst_start[i];
        for (int j = lane; j < c; j += 32) recv_row[dst + j] = src + j;
    }
}

// y_ret[recv_row[j]] = y[j] for every expert-major row j (fp32 rows of D, 16-byte vectors);
// a map entry outside [0, n) is skipped.
__global__ void __launch_bounds__(256) ep_return_rows_kernel(const float* y,
                                                             const int32_t* recv_row, int n,
                                                             int D, float* y_ret) {
    grid_dep_wait();
    grid_dep_launch();
    const int vec = D / 4;
    const long long total = static_cast<long long>(n) * vec;
    const float4* src = reinterpret_cast<const float4*>(y);
    float4* dst = reinterpret_cast<float4*>(y_ret);
    for (long long i = blockIdx.x * 256ll + threadIdx.x; i < total; i += 256ll * gridDim.x) {
        const int j = static_cast<int>(i / vec);
        const int c = static_cast<int>(i - static_cast<long long>(j) * vec);
        const int to = __ldg(recv_row + j);
        if (to >= 0 && to < n) dst[static_cast<size_t>(to) * vec + c] = __ldcs(src + i);
    }
}

}  // namespace

size_t ep_recv_layout_smem(int G, int El) { return sizeof(int) * 3ull * G * El; }

cudaError_t launch_ep_recv_layout(const int32_t* recv_counts, int G, int El, int n,
                                  int32_t* recv_offsets, int32_t* recv_row, int* status,
                                  cudaStream_t s) {
    const size_t smem = ep_recv_layout_smem(G, El);
    cudaError_t err = set_smem_limit(reinterpret_cast<const void*>(ep_recv_layout_kernel), smem);
    if (err != cudaSuccess) return err;
    err = launch_kernel(ep_recv_layout_kernel, dim3(1), dim3(kLayoutThreads), smem, s, false,
                        recv_counts, G, El, n, recv_offsets, recv_row, status);
    count_launches(1);
    return err;
}

cudaError_t launch_ep_return_rows(const float* y, const int32_t* recv_row, int n, int D,
                                  float* y_ret, int num_sms, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const long long total = static_cast<long long>(n) * (D / 4);
    const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, 8ll * num_sms));
    cudaError_t err = launch_kernel(ep_return_rows_kernel, dim3(blocks), dim3(256), 0, s, false,
                                    y, recv_row, n, D, y_ret);
    count_launches(1);
    return err;
}

}  // namespace moe
