// common.cuh -- types and small helpers shared by the kernels of libmoe_b200.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <utility>

#include "../../include/moe_api.h"

namespace moe {

using bf16 = __nv_bfloat16;

// Records the first device-side error in the status word (later errors are dropped).
__device__ __forceinline__ void set_status(int* status, int code) {
    if (status != nullptr) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float bf16_lo(uint32_t packed) {
    return __uint_as_float(packed << 16);
}

__device__ __forceinline__ float bf16_hi(uint32_t packed) {
    return __uint_as_float(packed & 0xFFFF0000u);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Programmatic dependent launch: a kernel launched with launch_kernel(..., pdl = true) may
// start while its predecessor on the stream is still running; it must call grid_dep_wait()
// before touching anything the predecessor writes (a no-op when launched without PDL).
// grid_dep_launch() lets the successor start as soon as every CTA of this grid issued it.
__device__ __forceinline__ void grid_dep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void grid_dep_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, bool pdl, Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Host-side count of kernel launches issued by the library (read by moe_launch_count).
void count_launches(unsigned n);

// Bound, in nanoseconds, of the layer's grid-wide wait (moe_set_grid_wait_budget_ns).
unsigned long long grid_wait_budget_ns();

// Lets kernel `fn` use `bytes` of dynamic shared memory on the current device: calls
// cudaFuncSetAttribute only when the limit this process last set there for fn is smaller
// (the attribute is per device and function; the layer would otherwise set it on every
// launch).
cudaError_t set_smem_limit(const void* fn, size_t bytes);

// ---------------------------------------------------------------- kernel launchers
// (defined in the .cu files, called by the C entry points in moe_api.cu)

struct PermuteLaunch {
    const int32_t* topk_idx;
    const float* topk_w;
    const int32_t* counts;   // [E] from the router, or NULL: counted here from topk_idx
    int32_t* counts_out;     // where the counts (given or derived) are copied, or NULL
    int T, E, K;
    int32_t* offsets;
    int32_t* sorted_token;
    float* sorted_w;
    int32_t* slot_to_row;
    int32_t* dense_offsets;  // optional [2] = {0, T} for a dense (shared) expert group
    int* status;
    int32_t* hist;           // [permute_chunks(T*K) * E] scratch, or NULL (one CTA)
    long long capacity;      // >= 0: each expert keeps its first `capacity` entries; < 0: all
};
// chunks the permutation cuts T*K entries into (1 at decode sizes, at most 256)
int permute_chunks(long long entries);
cudaError_t launch_permute(const PermuteLaunch& a, cudaStream_t s, bool pdl = false);

struct RouterLaunch {
    const bf16* x;
    const bf16* w_router;
    const float* logit_bias;
    const bf16* w_shared_gate;
    int T, D, E, K;
    float* logits;        // [T, E+1] workspace
    unsigned* counters;   // [ceil(T/8)] workspace, zeroed before the launch
    int32_t* topk_idx;
    float* topk_w;
    int32_t* counts;      // zeroed before the launch; NULL: not counted (the
                          // permutation derives them, tensor-core path)
    float* shared_gate;
    int* status;
    // optional: rows [T, zero_cols] of zero_acc are cleared by the CUDA-core router kernel
    // (the layer's fp32 accumulator); the tensor-core path leaves it to the gate_up kernel
    float* zero_acc;
    int zero_cols;
    int score_mode;           // 0: softmax over the experts; 1: per-expert sigmoid
    const float* select_bias; // [E] added to the scores for the selection only, or NULL
    int bf16_weights;         // round the renormalised weights to bf16
    int logit_planes;         // tensor-core path: partial-sum planes of [T, E] in logits
};
cudaError_t launch_router(const RouterLaunch& a, int num_sms, cudaStream_t s, bool pdl = false);

// Router for many tokens: the logits x W_r^T [T, E] (fp32) on the tensor cores through the
// grouped GEMM (one dense group, the reduction over D split into up to
// router_tc_max_planes(T) slices, each writing a partial [T, E] plane), then a selection
// kernel that adds the planes in slice order.  Needs E % 128 == 0 and a.logits with room
// for router_tc_max_planes(T) * T * E floats.
bool router_uses_tensor_cores(int T, int E);
int router_tc_max_planes(int T);
cudaError_t launch_router_tc(const RouterLaunch& a, int num_sms, cudaStream_t s, bool pdl = false);




struct GroupedGemmLaunch {
    bool gate_up;               // true: SiLU(gate)*up epilogue -> h; false: down epilogue
    const void* w;              // weights: gate_up [E, 2f, D] or down [E, D, f]
    const void* act;            // activations: x [T, D] (gathered via gather_tok) or h [rows, f]
    const int32_t* offsets;     // [E+1]; NULL: one dense group of `rows` rows (E must be 1)
    const int32_t* sorted_token;  // down only; NULL = identity
    const float* sorted_w;      // down only; NULL = 1
    int rows, E, D, f;
    bf16* h_out;                // gate_up: [rows, f]
    float* acc_out;             // down: [T, D] scatter-add target or NULL
    float* y_out;               // down: [rows, D] fp32 or NULL
    bf16* y16_out;              // down: [rows, D] bf16 (w * v per sorted row) or NULL
    int* status;
    // gate_up only: when gather_tok != NULL, act is the token matrix x [T, D] and row r of
    // the expert-ordered problem is x[gather_tok[r]] (gathered inside the kernel)
    const int32_t* gather_tok;
    int block_rows;   // weights on M: largest rows per tile (16..128); 0: from max_group_rows
    int max_group_rows;  // rows the largest group can have (T for routed experts); 0: rows
    int orientation;  // 0: auto; 1: weights on M; 2: tokens on M (one CTA); 3: CTA pairs
    // down with acc_out: when final_out and done are set, the kernel converts acc_out
    // [final_rows, D] to bf16 in final_out after all its CTAs finished (done = 0 at launch)
    bf16* final_out;
    int final_rows;
    unsigned* done;
    const bf16* final_residual;  // [final_rows, D] added in the conversion, or NULL
    unsigned long long barrier_budget_ns;  // bound of that grid-wide wait per CTA
    // gate_up with gather_tok: room for the rows in expert order [rows, D]; when given, the
    // CTA-pair kernel may be used (rows gathered by a copy kernel first)
    bf16* gather_buf;
    // down with y_out only (weights on M): split the reduction over f into ksplit equal
    // slices; slice s writes y_out + s * rows * D (0 or 1: no split)
    int ksplit;
    // gate_up: clear zero_acc[0, zero_floats) (a multiple of 4, 16-byte aligned) in the
    // kernel, before the down projection adds into it; NULL: nothing to clear
    float* zero_acc;
    long long zero_floats;
    // weights-on-M and one-CTA tokens-on-M kernels: let the kernel cut each tile's K steps
    // into up to ksplit_max slices (1 to 4) when the tiles cannot fill the grid.
    // gate_up needs `part` (ksplit_max planes of [rows, 2f] fp32) and `tickets` (ticket_cap
    // words, zero at launch, one per tile; more tiles than that: no split); down needs
    // acc_out without y_out / y16_out.  0 or 1: no split.
    int ksplit_max;
    float* part;
    unsigned* tickets;
    int ticket_cap;
};
// true when launch_grouped_gemm would run `a` on CTA pairs
bool grouped_gemm_uses_pairs(const GroupedGemmLaunch& a, int num_sms);
// kernels launch_grouped_gemm launches for `a` (0 when it has nothing to do)
int grouped_gemm_launches(const GroupedGemmLaunch& a, int num_sms);
cudaError_t launch_gather_rows(const bf16* x, const int32_t* tok, int rows, int D, bf16* out,
                               int num_sms, cudaStream_t s, bool pdl);
cudaError_t launch_grouped_gemm(const GroupedGemmLaunch& a, int num_sms, cudaStream_t s,
                                bool pdl = false);

// expert parallelism (ep.cu): receive-side grouping and the return of the expert rows
size_t ep_recv_layout_smem(int G, int El);
cudaError_t launch_ep_recv_layout(const int32_t* recv_counts, int G, int El, int n,
                                  int32_t* recv_offsets, int32_t* recv_row, int* status,
                                  cudaStream_t s);
cudaError_t launch_ep_return_rows(const float* y, const int32_t* recv_row, int n, int D,
                                  float* y_ret, int num_sms, cudaStream_t s);

struct CombineLaunch {
    const bf16* residual;  // [T, D] added before the bf16 rounding, or NULL
    const float* out_acc;
    const float* y_sorted;
    const bf16* y16_sorted;  // [T*K, D] bf16 rows already weighted (instead of y_sorted), or NULL
    const int32_t* slot_to_row;
    const float* topk_w;
    const bf16* shared_out;
    const float* shared_gate;
    int T, D, K;
    bf16* out;
};
cudaError_t launch_combine(const CombineLaunch& a, int num_sms, cudaStream_t s, bool pdl = false);

}  // namespace moe
