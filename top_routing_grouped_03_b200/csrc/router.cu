// router.cu -- router logits, fp32 softmax/TopK/renormalisation and per-expert counts.
//
// "MoE" (llm.rainlin.net), section 2: r = x W_r^T, p = Softmax(r) in fp32,
// I = TopK(p, K), alpha = p_I / sum p_I; plus the shared-expert scalar gate
// sigma(w_s^T x) of section 4.
//
// One kernel.  CTA (tb, eb) computes the fp32 logits of 8 tokens against a slab of
// experts (the shared gate vector rides along as expert index E) and writes them to a
// workspace; in the layer call it also clears its tokens' rows of the fp32 accumulator.
// The CTA that finishes a token block last (atomic ticket, no waiting) then runs the
// selection for those 8 tokens, one warp per token, in registers:
//   * TopK on the logits: the softmax is strictly increasing, so the K largest
//     probabilities are the K largest logits; ties go to the lower expert index.
//   * alpha_k = exp(r_k - r_max) / sum_{j in I} exp(r_j - r_max): the full softmax
//     denominator cancels in the renormalisation, so only the K selected terms are
//     exponentiated.
//   * Variants ("1.6 混合专家（MoE）", sections 2-3): per-expert sigmoid affinities
//     s = sigma(r) normalised over the selected experts, and a bias added to the scores
//     for the selection only (the weights use the raw scores); optionally the weights are
//     rounded to bf16 as the reference's cast to the model dtype does.
//   * expert_counts[e] += 1 per selected expert (global atomics, for the permutation).
// For many tokens (T >= 256, E a multiple of 128) the logits instead come from the
// tcgen05 grouped GEMM as one dense [T, E] product, and router_select_kernel runs the
// same selection with one warp per token.
#include <algorithm>
#include <cfloat>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kTokensPerCta = 8;
constexpr int kRouterThreads = 256;
// E <= 512: at most 16 logits per lane in the selection (select_topk_warp)
constexpr int kExpertsPerWarp = 2;

// Brings the 128-byte line holding `p` into L2 (no register result, nothing waits on it).
__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// TopK of one token's logits by one warp, in registers, then the renormalised weights.
// lg: the token's E logits (bias already added when add_bias is NULL), or `planes` partial
// sums of them `plane_stride` floats apart, added in plane order.  Writes idx/w of the
// token and adds its K experts to the counts.
template <int NV>
__device__ __forceinline__ void select_topk_nv(const float* lg, int planes, size_t plane_stride,
                                               const float* add_bias, int E,
                                               int K, int token, int lane, int32_t* topk_idx,
                                               float* topk_w, int32_t* counts, int score_mode,
                                               const float* select_bias, int bf16_weights) {
    float v[NV];  // logits (+ the logit bias)
#pragma unroll
    for (int j = 0; j < NV; ++j) v[j] = 0.f;
    // plane by plane, each plane's NV loads in flight together; planes added in order
    for (int q = 0; q < planes; ++q) {
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const int e = j * 32 + lane;
            if (e < E) v[j] += __ldcg(lg + q * plane_stride + e);
        }
    }
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        const int e = j * 32 + lane;
        v[j] = (e < E) ? v[j] + (add_bias ? __ldg(add_bias + e) : 0.f) : -FLT_MAX;
    }
    // scores and selection keys.  Softmax without selection bias: the key is the logit
    // itself (softmax is increasing) and only the K selected terms are exponentiated.
    // Otherwise the scores are the full softmax or the sigmoids, keys = scores + bias.
    const bool on_logits = (score_mode == 0 && select_bias == nullptr);
    float sc[NV], key[NV];
    if (on_logits) {
#pragma unroll
        for (int j = 0; j < NV; ++j) { sc[j] = v[j]; key[j] = v[j]; }
    } else {
        if (score_mode == 0) {
            float m = -FLT_MAX;
#pragma unroll
            for (int j = 0; j < NV; ++j) m = fmaxf(m, v[j]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
            float z = 0.f;
#pragma unroll
            for (int j = 0; j < NV; ++j) {
                sc[j] = (j * 32 + lane < E) ? expf(v[j] - m) : 0.f;
                z += sc[j];
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
#pragma unroll
            for (int j = 0; j < NV; ++j) sc[j] /= z;
        } else {
#pragma unroll
            for (int j = 0; j < NV; ++j) sc[j] = 1.f / (1.f + expf(-v[j]));
        }
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const int e = j * 32 + lane;
            key[j] = (e < E) ? sc[j] + (select_bias ? __ldg(select_bias + e) : 0.f) : -FLT_MAX;
        }
    }
    float my_sc = 0.f;
    int my_i = 0;
    for (int k = 0; k < K; ++k) {
        float bv = -FLT_MAX;
        int bi = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const int e = j * 32 + lane;
            if (e < E && key[j] > bv) { bv = key[j]; bi = e; }  // strict: lowest e per lane
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        // the winner's score comes from its owner lane, which also retires it
        float wsc = 0.f;
#pragma unroll
        for (int j = 0; j < NV; ++j)
            if (j * 32 + lane == bi) { wsc = sc[j]; key[j] = -INFINITY; }
        wsc = __shfl_sync(0xffffffffu, wsc, bi & 31);
        if (lane == k) { my_sc = wsc; my_i = bi; }
    }
    // weights: the selected raw scores over their sum (for logits: exp(r - r_max) terms)
    float num;
    if (on_logits) {
        const float vmax = __shfl_sync(0xffffffffu, my_sc, 0);
        num = (lane < K) ? expf(my_sc - vmax) : 0.f;
    } else {
        num = (lane < K) ? my_sc : 0.f;
    }
    float sum = num;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < K) {
        float w = num / sum;
        if (bf16_weights) w = __bfloat162float(__float2bfloat16_rn(w));
        topk_idx[static_cast<size_t>(token) * K + lane] = my_i;
        topk_w[static_cast<size_t>(token) * K + lane] = w;
        if (counts) atomicAdd(&counts[my_i], 1);
    }
}

// NV = logits per lane = ceil(E / 32), so the selection loops run exactly as far as E needs.
__device__ __forceinline__ void select_topk_warp(const float* lg, int planes,
                                                 size_t plane_stride, const float* add_bias,
                                                 const RouterLaunch& a, int token, int lane) {
    const int nv = (a.E + 31) / 32;
#define MOE_SELECT(N)                                                                      \
    select_topk_nv<N>(lg, planes, plane_stride, add_bias, a.E, a.K, token, lane, a.topk_idx, \
                      a.topk_w, a.counts, a.score_mode, a.select_bias, a.bf16_weights)
    if (nv <= 1) MOE_SELECT(1);
    else if (nv <= 2) MOE_SELECT(2);
    else if (nv <= 4) MOE_SELECT(4);
    else if (nv <= 8) MOE_SELECT(8);
    else MOE_SELECT(16);
#undef MOE_SELECT
}

// dsplit: warps per expert pair, each over D / dsplit of the dot products (1, 2, 4 or 8)
__global__ void __launch_bounds__(kRouterThreads)
router_kernel(RouterLaunch a, int experts_per_cta, int dsplit) {
    extern __shared__ __align__(16) uint4 xs[];  // [8][D] bf16 tokens of this block
    __shared__ int s_last;
    // per-warp partial sums of a pass when the dot products are split over warps
    __shared__ float s_part[kRouterThreads / 32][kExpertsPerWarp][kTokensPerCta];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int D = a.D, E = a.E;
    const int t0 = blockIdx.x * kTokensPerCta;
    const int nt = min(kTokensPerCta, a.T - t0);
    const int rows_total = E + (a.w_shared_gate ? 1 : 0);

    grid_dep_wait();     // x and the zeroed tickets/counts come from earlier stream work
    grid_dep_launch();

    // ---- clear this token block's slice of the layer accumulator
    if (a.zero_acc) {
        const int n4 = nt * a.zero_cols / 4;
        const int per = (n4 + gridDim.y - 1) / gridDim.y;
        float4* dst = reinterpret_cast<float4*>(a.zero_acc + static_cast<size_t>(t0) * a.zero_cols);
        const int b = blockIdx.y * per, e = min(b + per, n4);
        for (int i = b + tid; i < e; i += kRouterThreads) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }

    const int e_begin = blockIdx.y * experts_per_cta;
    const int e_end = min(e_begin + experts_per_cta, rows_total);
    const int vec_per_row = D / 8;

    // ---- pull this CTA's weight rows towards L2 while the token rows are staged (they
    //      come from HBM on the first token block; 128-byte lines)
    {
        const int lines_per_row = D * 2 / 128;
        const int nlines = (e_end - e_begin) * lines_per_row;
        for (int i = tid; i < nlines; i += kRouterThreads) {
            const int e = e_begin + i / lines_per_row;
            const bf16* wrow = (e < E) ? a.w_router + static_cast<size_t>(e) * D : a.w_shared_gate;
            prefetch_l2(reinterpret_cast<const char*>(wrow) + (i % lines_per_row) * 128);
        }
    }

    // ---- stage the 8 token rows (zeros past T): kBatch loads in flight per thread
    {
        constexpr int kBatch = 8;
        const int nvec = kTokensPerCta * vec_per_row;
        const uint4* xsrc = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t0) * D);
        for (int i0 = tid; i0 < nvec; i0 += kBatch * kRouterThreads) {
            uint4 v[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int i = i0 + u * kRouterThreads;
                v[u] = (i < nvec && i / vec_per_row < nt) ? __ldg(xsrc + i) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int i = i0 + u * kRouterThreads;
                if (i < nvec) xs[i] = v[u];
            }
        }
    }
    __syncthreads();

    // ---- logits of this CTA's expert slab: each group of dsplit warps takes kExpertsPerWarp
    //      expert rows at a time (one unpack of x serves all of them), warp w of the group
    //      the w-th D / dsplit columns; each lane keeps kUnroll chunks of 16-byte weight loads
    //      per row in flight; the group's partial sums meet in shared memory
    constexpr int kUnroll = 4;
    const int groups = (kRouterThreads / 32) / dsplit;
    const int grp = warp / dsplit, part = warp % dsplit;
    const int c_lo = part * vec_per_row / dsplit, c_hi = (part + 1) * vec_per_row / dsplit;
    const int passes = (e_end - e_begin + groups * kExpertsPerWarp - 1) / (groups * kExpertsPerWarp);
    for (int pass = 0; pass < passes; ++pass) {
        const int e0 = e_begin + (pass * groups + grp) * kExpertsPerWarp;
        const uint4* wv[kExpertsPerWarp];
        bool has[kExpertsPerWarp];
#pragma unroll
        for (int u = 0; u < kExpertsPerWarp; ++u) {
            const int e = e0 + u;
            has[u] = e < e_end;
            const bf16* wrow = (e < E) ? a.w_router + static_cast<size_t>(e) * D : a.w_shared_gate;
            wv[u] = reinterpret_cast<const uint4*>(has[u] ? wrow : a.w_router);
        }
        float acc[kExpertsPerWarp][kTokensPerCta];
#pragma unroll
        for (int u = 0; u < kExpertsPerWarp; ++u)
#pragma unroll
            for (int t = 0; t < kTokensPerCta; ++t) acc[u][t] = 0.f;
        for (int c0 = c_lo + lane; c0 < c_hi; c0 += 32 * kUnroll) {
            uint4 w[kUnroll][kExpertsPerWarp];
#pragma unroll
            for (int v = 0; v < kUnroll; ++v)
#pragma unroll
                for (int u = 0; u < kExpertsPerWarp; ++u) {
                    const int c = c0 + 32 * v;
                    w[v][u] = (c < c_hi && has[u]) ? __ldg(wv[u] + c) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
            for (int v = 0; v < kUnroll; ++v) {
                const int c = c0 + 32 * v;
                if (c >= c_hi) break;
                float wf[kExpertsPerWarp][8];
#pragma unroll
                for (int u = 0; u < kExpertsPerWarp; ++u) {
                    wf[u][0] = bf16_lo(w[v][u].x); wf[u][1] = bf16_hi(w[v][u].x);
                    wf[u][2] = bf16_lo(w[v][u].y); wf[u][3] = bf16_hi(w[v][u].y);
                    wf[u][4] = bf16_lo(w[v][u].z); wf[u][5] = bf16_hi(w[v][u].z);
                    wf[u][6] = bf16_lo(w[v][u].w); wf[u][7] = bf16_hi(w[v][u].w);
                }
#pragma unroll
                for (int t = 0; t < kTokensPerCta; ++t) {
                    const uint4 xv = xs[t * vec_per_row + c];
                    const float x0 = bf16_lo(xv.x), x1 = bf16_hi(xv.x), x2 = bf16_lo(xv.y);
                    const float x3 = bf16_hi(xv.y), x4 = bf16_lo(xv.z), x5 = bf16_hi(xv.z);
                    const float x6 = bf16_lo(xv.w), x7 = bf16_hi(xv.w);
#pragma unroll
                    for (int u = 0; u < kExpertsPerWarp; ++u) {
                        float s2 = acc[u][t];
                        s2 = fmaf(wf[u][0], x0, s2);
                        s2 = fmaf(wf[u][1], x1, s2);
                        s2 = fmaf(wf[u][2], x2, s2);
                        s2 = fmaf(wf[u][3], x3, s2);
                        s2 = fmaf(wf[u][4], x4, s2);
                        s2 = fmaf(wf[u][5], x5, s2);
                        s2 = fmaf(wf[u][6], x6, s2);
                        s2 = fmaf(wf[u][7], x7, s2);
                        acc[u][t] = s2;
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kExpertsPerWarp; ++u)
#pragma unroll
            for (int t = 0; t < kTokensPerCta; ++t)
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
                    acc[u][t] += __shfl_xor_sync(0xffffffffu, acc[u][t], off);
        if (dsplit > 1) {
            if (lane == 0)
#pragma unroll
                for (int u = 0; u < kExpertsPerWarp; ++u)
#pragma unroll
                    for (int t = 0; t < kTokensPerCta; ++t) s_part[warp][u][t] = acc[u][t];
            __syncthreads();
            if (part == 0 && lane == 0)  // the group's parts in D order
                for (int q = 1; q < dsplit; ++q)
#pragma unroll
                    for (int u = 0; u < kExpertsPerWarp; ++u)
#pragma unroll
                        for (int t = 0; t < kTokensPerCta; ++t) acc[u][t] += s_part[warp + q][u][t];
            __syncthreads();
        }
        if (part == 0 && lane == 0) {
#pragma unroll
            for (int u = 0; u < kExpertsPerWarp; ++u) {
                const int e = e0 + u;
                if (!has[u]) continue;
                const float b = (e < E && a.logit_bias) ? a.logit_bias[e] : 0.f;
                for (int t = 0; t < nt; ++t)
                    a.logits[static_cast<size_t>(t0 + t) * (E + 1) + e] = acc[u][t] + b;
            }
        }
    }
    __threadfence();  // this thread's logits are visible device-wide before the ticket

    // ---- ticket: the last CTA of this token block does the selection
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned prev = atomicAdd(&a.counters[blockIdx.x], 1u);
        s_last = (prev == gridDim.y - 1) ? 1 : 0;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    for (int t = warp; t < nt; t += kRouterThreads / 32) {
        const int token = t0 + t;
        const float* lg = a.logits + static_cast<size_t>(token) * (E + 1);
        select_topk_warp(lg, 1, 0, nullptr, a, token, lane);
        if (a.w_shared_gate && lane == 0) {
            const float g = __ldcg(lg + E);
            a.shared_gate[token] = 1.f / (1.f + expf(-g));
        }
    }
}


// Selection after the tensor-core logits: one warp per token over the partial logit
// planes (no bias yet), the planes added in order and the bias on load; the shared gate's
// dot product w_s . x_t is done here by the same warp.  (The layer's accumulator is
// cleared by the gate_up kernel on this path.)
__global__ void __launch_bounds__(kRouterThreads, 4) router_select_kernel(RouterLaunch a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * (kRouterThreads / 32);
    const int nt = min(kRouterThreads / 32, a.T - t0);
    grid_dep_wait();  // logits come from the GEMM
    grid_dep_launch();
    if (warp >= nt) return;
    const int token = t0 + warp;
    select_topk_warp(a.logits + static_cast<size_t>(token) * a.E, a.logit_planes,
                     static_cast<size_t>(a.T) * a.E, a.logit_bias, a, token, lane);
    if (a.w_shared_gate) {
        const uint4* xv = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(token) * a.D);
        const uint4* wv = reinterpret_cast<const uint4*>(a.w_shared_gate);
        float acc = 0.f;
        // 8 chunks of x and w_s per lane in flight at a time (D = 4096 is 16 chunks a lane:
        // two round trips to memory instead of sixteen)
        constexpr int kBatch = 8;
        for (int c0 = lane; c0 < a.D / 8; c0 += 32 * kBatch) {
            uint4 x8[kBatch], w8[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int c = c0 + 32 * u;
                const bool in = c < a.D / 8;
                x8[u] = in ? __ldg(xv + c) : make_uint4(0, 0, 0, 0);
                w8[u] = in ? __ldg(wv + c) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                acc = fmaf(bf16_lo(x8[u].x), bf16_lo(w8[u].x), acc);
                acc = fmaf(bf16_hi(x8[u].x), bf16_hi(w8[u].x), acc);
                acc = fmaf(bf16_lo(x8[u].y), bf16_lo(w8[u].y), acc);
                acc = fmaf(bf16_hi(x8[u].y), bf16_hi(w8[u].y), acc);
                acc = fmaf(bf16_lo(x8[u].z), bf16_lo(w8[u].z), acc);
                acc = fmaf(bf16_hi(x8[u].z), bf16_hi(w8[u].z), acc);
                acc = fmaf(bf16_lo(x8[u].w), bf16_lo(w8[u].w), acc);
                acc = fmaf(bf16_hi(x8[u].w), bf16_hi(w8[u].w), acc);
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) a.shared_gate[token] = 1.f / (1.f + expf(-acc));
    }
}

}  // namespace

cudaError_t launch_router(const RouterLaunch& a, int num_sms, cudaStream_t s, bool pdl) {
    if (a.T == 0) return cudaSuccess;
    const int n_tb = ceil_div(a.T, kTokensPerCta);
    const int rows_total = a.E + (a.w_shared_gate ? 1 : 0);
    // Few token blocks: the dot products of an expert pair are split over dsplit warps (a
    // shorter chain per warp, at least 512 columns each) while one-pass CTAs would still
    // fill at most half the GPU
    int dsplit = 1;
    while (dsplit < 8 && a.D / (2 * dsplit) >= 512 &&
           2ll * n_tb * ceil_div(rows_total, (kRouterThreads / 32 / dsplit) * kExpertsPerWarp) <=
               num_sms)
        dsplit *= 2;
    const int rows_per_pass = (kRouterThreads / 32 / dsplit) * kExpertsPerWarp;
    // split the experts so that the grid covers about one wave of the GPU
    int n_eb = ceil_div(num_sms, n_tb);
    n_eb = max(1, min(n_eb, ceil_div(rows_total, rows_per_pass)));
    int per_cta = ceil_div(ceil_div(rows_total, n_eb), rows_per_pass) * rows_per_pass;
    n_eb = ceil_div(rows_total, per_cta);
    const size_t smem = static_cast<size_t>(kTokensPerCta) * a.D * sizeof(bf16);
    cudaError_t err = set_smem_limit(reinterpret_cast<const void*>(router_kernel), smem);
    if (err != cudaSuccess) return err;
    err = launch_kernel(router_kernel, dim3(n_tb, n_eb), dim3(kRouterThreads), smem, s, pdl, a,
                        per_cta, dsplit);
    count_launches(1);
    return err;
}


bool router_uses_tensor_cores(int T, int E) { return T >= 256 && E % 128 == 0; }


int router_tc_max_planes(int T) { return std::min(16, std::max(1, 512 / ceil_div(T, 128))); }

cudaError_t launch_router_tc(const RouterLaunch& a, int num_sms, cudaStream_t s, bool pdl) {
    if (a.T == 0) return cudaSuccess;
    // logits = x W_r^T: W_r's E rows on the MMA's M side, BN = 128 or 256 tokens on N, one
    // dense group.  Few tiles with a long reduction (D) would leave most SMs idle, so the D
    // steps are cut into S slices (partial planes).  (BN, S) minimises the bytes the busiest
    // CTA loads -- waves x (steps per slice x (128 + BN) rows of 128 B + a tile's fixed cost,
    // about 2048 such rows: pipeline fill, drain and epilogue) -- ties to fewer planes and the
    // narrower tile, with at least 4 steps per slice.  Wider token tiles re-read W_r less.
    constexpr long long kTileCost = 2048;
    const int nk = a.D / 64;
    int S = 1, BN = 128;
    long long best = -1;
    for (int bn = 128; bn <= 256; bn *= 2) {
        const int base = (a.E / 128) * ceil_div(a.T, bn);
        for (int c = 1; c <= router_tc_max_planes(a.T) && nk % c == 0 && nk / c >= 4; c *= 2) {
            const long long cost = static_cast<long long>(ceil_div(base * c, num_sms)) *
                                   (static_cast<long long>(nk / c) * (128 + bn) + kTileCost);
            if (best < 0 || cost < best) { best = cost; S = c; BN = bn; }
        }
    }
    GroupedGemmLaunch g{};
    g.gate_up = false;
    g.w = a.w_router;
    g.act = a.x;
    g.offsets = nullptr;
    g.rows = a.T;
    g.E = 1;
    g.D = a.E;  // output features
    g.f = a.D;  // reduction length
    g.y_out = a.logits;
    g.status = a.status;
    g.block_rows = BN;
    g.ksplit = S;
    cudaError_t err = launch_grouped_gemm(g, num_sms, s, pdl);
    if (err != cudaSuccess) return err;
    RouterLaunch sel = a;
    sel.logit_planes = S;
    err = launch_kernel(router_select_kernel, dim3(ceil_div(a.T, kRouterThreads / 32)),
                        dim3(kRouterThreads), 0, s, true, sel);
    count_launches(1);
    return err;
}

}  // namespace moe
