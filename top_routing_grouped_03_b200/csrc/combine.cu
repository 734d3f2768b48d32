// combine.cu -- back to token order.
//
// "MoE" (llm.rainlin.net), section 4: y_t = sum_{e in I_t} alpha_te E_e(x_t)
// + sigma(w_s^T x_t) E_s(x_t); section 3.2: the expert outputs are index-added back to
// their tokens.  One thread owns 8 consecutive features of one token (16-byte loads and
// stores) and sums, in this fixed order: the fp32 accumulator row (if any), the K routed
// rows in slot order (skipping pairs dropped by an expert capacity, slot_to_row = -1), the
// gated shared-expert row, then the decoder residual h (section 4: h_out = h + y); the
// result is rounded once to bf16 (round to nearest even).
#include <algorithm>

#include "common.cuh"

namespace moe {
namespace {

__device__ __forceinline__ void add8(float (&acc)[8], const uint4 v, float w) {
    acc[0] = fmaf(w, bf16_lo(v.x), acc[0]);
    acc[1] = fmaf(w, bf16_hi(v.x), acc[1]);
    acc[2] = fmaf(w, bf16_lo(v.y), acc[2]);
    acc[3] = fmaf(w, bf16_hi(v.y), acc[3]);
    acc[4] = fmaf(w, bf16_lo(v.z), acc[4]);
    acc[5] = fmaf(w, bf16_hi(v.z), acc[5]);
    acc[6] = fmaf(w, bf16_lo(v.w), acc[6]);
    acc[7] = fmaf(w, bf16_hi(v.w), acc[7]);
}

__global__ void __launch_bounds__(256) combine_kernel(CombineLaunch a) {
    grid_dep_wait();  // the rows to combine come from the grouped GEMM
    grid_dep_launch();
    const int vec = a.D / 8;
    const long long n = static_cast<long long>(a.T) * vec;
    for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n; i += 256ll * gridDim.x) {
        const int t = static_cast<int>(i / vec);
        const int c = static_cast<int>(i - static_cast<long long>(t) * vec);
        float acc[8];
        if (a.out_acc) {
            const float4* src = reinterpret_cast<const float4*>(a.out_acc) + 2 * i;
            const float4 lo = __ldcs(src), hi = __ldcs(src + 1);
            acc[0] = lo.x; acc[1] = lo.y; acc[2] = lo.z; acc[3] = lo.w;
            acc[4] = hi.x; acc[5] = hi.y; acc[6] = hi.z; acc[7] = hi.w;
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.f;
        }
        if (a.y_sorted) {
            const float4* ys = reinterpret_cast<const float4*>(a.y_sorted);
            for (int k = 0; k < a.K; ++k) {
                const int slot = t * a.K + k;
                const int row = __ldg(a.slot_to_row + slot);
                if (row < 0) continue;  // dropped past its expert's capacity
                const float w = a.topk_w ? __ldg(a.topk_w + slot) : 1.f;
                const size_t o = 2 * (static_cast<size_t>(row) * vec + c);
                const float4 lo = __ldg(ys + o), hi = __ldg(ys + o + 1);
                acc[0] = fmaf(w, lo.x, acc[0]);
                acc[1] = fmaf(w, lo.y, acc[1]);
                acc[2] = fmaf(w, lo.z, acc[2]);
                acc[3] = fmaf(w, lo.w, acc[3]);
                acc[4] = fmaf(w, hi.x, acc[4]);
                acc[5] = fmaf(w, hi.y, acc[5]);
                acc[6] = fmaf(w, hi.z, acc[6]);
                acc[7] = fmaf(w, hi.w, acc[7]);
            }
        }
        if (a.y16_sorted) {
            const uint4* ys = reinterpret_cast<const uint4*>(a.y16_sorted);
            for (int k = 0; k < a.K; ++k) {
                const int row = __ldg(a.slot_to_row + t * a.K + k);
                if (row < 0) continue;  // dropped past its expert's capacity
                add8(acc, __ldcs(ys + static_cast<size_t>(row) * vec + c), 1.f);
            }
        }
        if (a.shared_out) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(a.shared_out) + i);
            add8(acc, v, __ldg(a.shared_gate + t));
        }
        if (a.residual) add8(acc, __ldg(reinterpret_cast<const uint4*>(a.residual) + i), 1.f);
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        reinterpret_cast<uint4*>(a.out)[i] = o;
    }
}

}  // namespace

cudaError_t launch_combine(const CombineLaunch& a, int num_sms, cudaStream_t s, bool pdl) {
    if (a.T == 0) return cudaSuccess;
    const long long n = static_cast<long long>(a.T) * (a.D / 8);
    const int blocks = static_cast<int>(std::min<long long>((n + 255) / 256, 8ll * num_sms));
    cudaError_t err = launch_kernel(combine_kernel, dim3(blocks), dim3(256), 0, s, pdl, a);
    count_launches(1);
    return err;
}

}  // namespace moe
