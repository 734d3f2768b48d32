// grouped_gemm.cu -- grouped SwiGLU expert GEMMs on tcgen05 tensor cores.
//
// "MoE" (llm.rainlin.net), section 3: E_e(x) = W_down (SiLU(W_gate x) (.) W_up x), the
// gate_up weight of an expert is one [2f, D] matrix (gate rows, then up rows); section
// 3.2: the routed output is scaled by the routing weight and index-added back to its
// token.  "MoE 到底省了什么" (clxhxhhr.top), section 3: with few rows per expert the
// layer is bound by reading the expert weights, with many rows it is bound by compute.
//
// Three persistent, warp-specialised kernels share one structure: warp 0 fills a ring of
// shared-memory stages (TMA, 128-byte swizzle, 64-deep K steps), warp 1 owns the tensor
// memory and one of its threads issues tcgen05.mma (bf16 in, fp32 accumulate), and the
// epilogue warps drain a double-buffered TMEM accumulator with tcgen05.ld while the next
// tile accumulates.  Epilogues: h = SiLU(g) * u -> bf16 for gate_up; w * v -> fp32
// reductions into the token's output row (and/or fp32 y_sorted) for down.  The work list
// (group, feature block, row block) is derived on the device from the group offsets, so no
// host synchronisation is needed, and every wait is bounded.
//   * grouped_gemm_kernel<BN, GATE_UP>, weights on M: 128 weight rows x BN token rows
//     (16..128), for groups of a handful of rows -- an expert with two rows still fills
//     the 128-lane tile.  gate_up keeps the gate block in accumulator columns [0, BN) and
//     the up block in [BN, 2BN) so one thread holds both halves of a feature.  Also the
//     router's logits GEMM (one dense group, the reduction split into partial planes).
//   * grouped_gemm_tm_kernel<GATE_UP>, tokens on M: 128 token rows x 256 weight rows (128
//     gate + 128 up features, or 256 output features), 8 epilogue warps; features lie
//     along the accumulator's columns, so h leaves as 16-byte stores and the down results
//     as 4-wide vector reductions.
//   * grouped_gemm_pair_kernel<GATE_UP>, CTA pairs: clusters of two with
//     tcgen05.mma.cta_group::2 over 256 token rows x 256 weight rows, each CTA loading its
//     own token rows and half of the weights (.cta_group::2 TMA, no multicast), commits
//     multicast to both CTAs' barriers; its token rows must be contiguous, so gate_up
//     reads an expert-ordered copy of x.
// The other two kernels gather gate_up's token rows themselves: the producer warp's lanes
// copy 16-byte chunks of x[token] with cp.async into the 128-byte swizzle the MMA
// descriptor expects, zero-filling rows past the group.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <unordered_map>

#include "common.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;          // weight rows per tile (MMA M)
constexpr int kBK = 64;           // K per stage: one 128-byte swizzle row of bf16
constexpr int kThreads = 192;     // 6 warps
constexpr int kEpiThreads = 128;  // warps 2..5
constexpr int kMaxGroups = 1024;

__host__ __device__ constexpr int pow2_at_least(int v) {
    int p = 32;
    while (p < v) p <<= 1;
    return p;
}

template <int BN, bool GATE_UP>
struct Cfg {
    static constexpr int kNumA = GATE_UP ? 2 : 1;
    static constexpr int kABytes = kBM * kBK * 2;
    static constexpr int kBBytes = BN * kBK * 2;
    static constexpr int kStageBytes = kNumA * kABytes + kBBytes;
    static constexpr int kStages0 = (200 * 1024) / kStageBytes;
    static constexpr int kStages = kStages0 > 8 ? 8 : kStages0;
    static constexpr int kAccCols = GATE_UP ? 2 * BN : BN;
    static constexpr int kTmemCols = pow2_at_least(2 * kAccCols);
    static_assert(kTmemCols <= 512, "accumulators exceed tensor memory");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M=128");
    static_assert(kStageBytes % 1024 == 0, "stage buffers must keep 1024-byte alignment");
};

struct Params {
    const int32_t* offsets;  // [G+1] row ranges; NULL: one group of rows_total rows
    int rows_total;
    const int32_t* sorted_token;
    const float* sorted_w;
    int G;             // groups
    int nf;            // feature blocks (of 128 weight rows) per group
    int nk;            // K steps of 64
    int w_group_rows;  // weight rows per group in the 2-D weight view (2f or D)
    int up_rows;       // gate_up: offset of the up rows inside a group (f)
    int out_cols;      // gate_up: f (h row length); down: D (output row length)
    bf16* h_out;
    float* acc_out;
    float* y_out;
    bf16* y16_out;     // down: w * v per sorted row as bf16 [rows, out_cols], or NULL
    int* status;
    const int32_t* gather_tok;  // gate_up: B rows are x[gather_tok[row]] (cp.async), or NULL
    const bf16* x;              // the token matrix the gather reads, [*, K] bf16
    bf16* final_out;            // down: when set, convert acc_out [final_rows, out_cols] to
    int final_rows;             //   bf16 here once every CTA of the grid has added its tiles
    unsigned* done;             //   (grid barrier counter, zero at launch)
    const bf16* final_residual; //   + this bf16 [final_rows, out_cols] when not NULL
    unsigned long long barrier_budget_ns;  // how long a CTA waits at that grid barrier
    // weights-on-M kernel, y_out only: the K steps are cut into ksplit equal slices, one
    // tile per slice, and slice s writes its partial sums to y_out + s * split_stride
    int ksplit;
    long long split_stride;
    // gate_up: the epilogue warps clear zero_acc[0, zero_n4) (float4s, the layer's fp32
    // accumulator) before their first tile -- they would otherwise wait for it idle
    float* zero_acc;
    long long zero_n4;
    // weights-on-M kernel with contiguous token rows: rows per activation TMA box (= BN)
    int act_box;
    // Split of each tile's K steps chosen on the device (weights-on-M kernel when ksplit is
    // 1, and the one-CTA tokens-on-M kernel): up to ksplit_max slices, picked from the tile
    // count so that the (tile, slice) units fill the grid's waves.  down: every slice adds
    // its partial products into acc_out.  gate_up: every slice writes its fp32 partial sums
    // to part, [slice][row][gate f | up f] with part_rows rows per slice; the slice that
    // completes a tile (tickets[tile], zero at launch, ticket_cap of them) adds them in
    // slice order and applies SwiGLU.
    int ksplit_max;
    float* part;
    int part_rows;
    unsigned* tickets;
    int ticket_cap;
};

// Epilogue threads of every CTA clear their grid-strided share of p.zero_acc.
__device__ __forceinline__ void clear_accumulator(const Params& p, int epi_tid, int epi_threads) {
    if (p.zero_acc == nullptr) return;
    float4* dst = reinterpret_cast<float4*>(p.zero_acc);
    const long long step = static_cast<long long>(gridDim.x) * epi_threads;
    for (long long i = static_cast<long long>(blockIdx.x) * epi_threads + epi_tid; i < p.zero_n4;
         i += step)
        __stcs(dst + i, make_float4(0.f, 0.f, 0.f, 0.f));
}

// tiles of a group of n rows cut into row blocks of `rows`
__device__ __forceinline__ int group_tiles(const Params& p, int n, int rows) {
    return ((n + rows - 1) / rows) * p.nf;
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// The layer's last down launch finishes the output: every thread fences its reductions,
// each CTA takes a ticket, all CTAs wait (bounded) until the whole grid has arrived --
// the grid is persistent with at most one CTA per SM, so all of it is resident -- and
// then convert a grid-stride share of the fp32 accumulator to bf16.
__device__ __noinline__ void finalize_output(const Params& p) {
    __shared__ int s_ok;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        atomicAdd(p.done, 1u);
        int ok = 1;
        const uint64_t t0 = global_timer_ns();
        while (ld_acquire_gpu(p.done) < gridDim.x) {
            // (a budget of 0 gives up at the first look that finds the grid incomplete)
            if (global_timer_ns() - t0 >= p.barrier_budget_ns) {
                set_status(p.status, MOE_ERR_TIMEOUT);
                ok = 0;
                break;
            }
            __nanosleep(64);
        }
        s_ok = ok;
    }
    __syncthreads();
    if (!s_ok) return;
    const long long n4 = static_cast<long long>(p.final_rows) * p.out_cols / 4;
    const float4* src = reinterpret_cast<const float4*>(p.acc_out);
    const uint2* res = reinterpret_cast<const uint2*>(p.final_residual);
    uint2* dst = reinterpret_cast<uint2*>(p.final_out);
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        float4 v = __ldcg(src + i);
        if (res) {
            const uint2 r = __ldg(res + i);
            v.x += bf16_lo(r.x); v.y += bf16_hi(r.x); v.z += bf16_lo(r.y); v.w += bf16_hi(r.y);
        }
        dst[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
    }
}

// Named barrier 1 of the four epilogue warps with an AND across their threads: all of
// them take the same branch afterwards, so a wait that gives up in one warp makes every
// epilogue warp unwind together.
template <int kThreadsInBar = kEpiThreads>
__device__ __forceinline__ bool epilogue_bar_and(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, 1, %2, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v)), "n"(kThreadsInBar)
        : "memory");
    return r != 0;
}

struct Tile {
    int g, i, row0, row_end;
};

__device__ __forceinline__ Tile decode_tile(int tile, const int* g_tile, const int* g_off, int G,
                                            int BN) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (g_tile[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    Tile t;
    t.g = lo;
    const int n = g_off[lo + 1] - g_off[lo];
    const int nb = (n + BN - 1) / BN;
    const int local = tile - g_tile[lo];
    t.i = local / nb;
    const int j = local - t.i * nb;
    t.row0 = g_off[lo] + j * BN;
    t.row_end = g_off[lo + 1];
    return t;
}

// The group table every role of a CTA walks: g_off = row offsets of the groups (from the
// device, or {0, rows_total} for one dense group); g_tile[g] = first tile of group g, where a
// group of n rows has ceil(n / rows_per_tile) * nf tiles; g_tile[G] = total.
__device__ __forceinline__ void build_tile_table(const Params& p, int rows_per_tile, int* g_off,
                                                 int* g_tile, int* total_slot, int warp,
                                                 int lane) {
    for (int i = threadIdx.x; i <= p.G; i += blockDim.x)
        g_off[i] = p.offsets ? p.offsets[i] : (i == 0 ? 0 : p.rows_total);
    __syncthreads();
    if (warp == 2) {
        // tile prefix over groups: lane l owns a contiguous run of groups
        const int per = (p.G + 31) / 32;
        const int gb = min(lane * per, p.G), ge = min(gb + per, p.G);
        int local = 0;
        for (int g = gb; g < ge; ++g) local += group_tiles(p, g_off[g + 1] - g_off[g], rows_per_tile);
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - local;
        for (int g = gb; g < ge; ++g) {
            g_tile[g] = run;
            run += group_tiles(p, g_off[g + 1] - g_off[g], rows_per_tile);
        }
        if (lane == 31) {
            g_tile[p.G] = incl;
            *total_slot = incl;
        }
    }
}

// Slices per tile (1 to 4, at most smax, each of at least kSplitMinSteps K steps; slice j
// of s takes steps [j nk / s, (j + 1) nk / s)) minimising the time of the (tile, slice)
// units over `ctas` CTAs: a unit costs its K steps (at most ceil(nk / s)) plus
// kSplitRampSteps for its pipeline ramp, epilogue and fix-up, and the units run in
// ceil(tiles s / ctas) waves.  Integer costs, so every thread gets the same answer; a tie
// keeps fewer slices.
constexpr int kSplitSlicesMax = 4;
constexpr int kSplitMinSteps = 4;
constexpr int kSplitRampSteps = 4;
__device__ __forceinline__ int slice_begin(int nk, int nsplit, int slice) {
    return slice * nk / nsplit;
}
__device__ __forceinline__ int choose_split(int tiles, int ctas, int nk, int smax) {
    int best = 1;
    if (tiles <= 0) return best;
    long long best_cost = static_cast<long long>((tiles + ctas - 1) / ctas) * (nk + kSplitRampSteps);
    for (int s = 2; s <= smax && s <= kSplitSlicesMax; ++s) {
        if (nk / s < kSplitMinSteps) break;
        const long long waves = (static_cast<long long>(tiles) * s + ctas - 1) / ctas;
        const long long cost = waves * ((nk + s - 1) / s + kSplitRampSteps);
        if (cost < best_cost) {
            best = s;
            best_cost = cost;
        }
    }
    return best;
}

// Work units of a launch: tiles [0, full) whole, then each remaining tile cut into s K
// slices, the slice varying fastest.  A host-fixed ksplit cuts every tile.  Otherwise,
// with fewer tiles than two waves of the grid, every tile is cut into the slices
// choose_split picks; with more, the tiles of the full waves stay whole and only the last,
// partial wave's tiles are cut, so that the tail of the launch is shared by more CTAs
// (measured: cutting every tile was faster below two waves, cutting the tail above).
struct Units {
    int full, s, total;
};
struct Unit {
    int tile, slice, nsl;
};
__device__ __forceinline__ Units plan_units(const Params& p, int tiles, bool gate_up) {
    if (p.ksplit > 1) return {0, p.ksplit, tiles * p.ksplit};
    Units w{tiles, 1, tiles};
    if (p.ksplit_max <= 1 || tiles == 0) return w;
    if (gate_up && (p.part == nullptr || p.tickets == nullptr || tiles > p.ticket_cap)) return w;
    const int ctas = gridDim.x;
    const int whole = tiles < 2 * ctas ? 0 : (tiles / ctas) * ctas;
    const int s = choose_split(tiles - whole, ctas, p.nk, p.ksplit_max);
    if (s > 1) w = {whole, s, whole + (tiles - whole) * s};
    return w;
}
__device__ __forceinline__ Unit unit_at(const Units& w, int u) {
    if (u < w.full) return {u, 0, 1};
    const int v = u - w.full;
    return {w.full + v / w.s, v % w.s, w.s};
}

// gate_up split: once every epilogue thread has written its partial sums of the tile, one
// ticket per slice (a release/acquire atomic by one thread, ordered with the other epilogue
// threads' stores and later loads by the barriers); true in every epilogue thread of the
// CTA that took the last one -- it then sees all slices' partial sums.
__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned* p, unsigned v) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
template <int kThreads>
__device__ __forceinline__ bool split_tile_done(const Params& p, int tile, int nsplit,
                                                int first_epi_tid) {
    epilogue_bar_and<kThreads>(true);
    bool last = true;
    if (threadIdx.x == first_epi_tid)
        last = atom_add_acq_rel_gpu(p.tickets + tile, 1u) == static_cast<unsigned>(nsplit - 1);
    return epilogue_bar_and<kThreads>(last);
}

// The one-CTA tokens-on-M kernel shares the fix-up among the tile's slices instead: each
// slice posts its ticket, waits (bounded) until all nsplit slices have posted -- the grid
// is persistent with at most one CTA per SM, so the tile's other slices are resident or
// will run once earlier work leaves the SMs, and a slice posts before it waits -- and then
// fixes up its own share of the tile's rows.  False on a wait that ran out of time.
template <int kThreads>
__device__ __forceinline__ bool split_tile_all_posted(const Params& p, int tile, int nsplit,
                                                      int first_epi_tid) {
    epilogue_bar_and<kThreads>(true);
    bool ok = true;
    if (threadIdx.x == first_epi_tid) {
        atom_add_acq_rel_gpu(p.tickets + tile, 1u);
        const uint64_t t0 = global_timer_ns();
        while (ld_acquire_gpu(p.tickets + tile) < static_cast<unsigned>(nsplit)) {
            if (global_timer_ns() - t0 > kWaitBudgetNs) {
                ok = false;
                break;
            }
        }
    }
    return epilogue_bar_and<kThreads>(ok);
}

// Per-lane plan for gathering ROWS token rows of x into a 128-byte-swizzled operand tile
// with cp.async: lane l owns 16-byte chunk c = l % 8 of tile rows l/8 + 4u; that chunk of
// tile row r lands at r*128 + ((c ^ (r % 8)) * 16).
template <int ROWS>
struct RowGather {
    static constexpr int kChunks = ROWS * 8 / 32;
    uint32_t src_off[kChunks];  // element offset of the chunk's row in x (< 2^31)
    uint32_t valid;

    __device__ __forceinline__ void plan(const int32_t* tok, int row0, int row_end, int row_len,
                                         int lane) {
        valid = 0;
#pragma unroll
        for (int u = 0; u < kChunks; ++u) {
            const int row = row0 + (lane >> 3) + 4 * u;
            const bool ok = row < row_end;
            const int t = ok ? __ldg(tok + row) : 0;
            src_off[u] = static_cast<uint32_t>(t) * row_len + (lane & 7) * 8;
            valid |= (ok ? 1u : 0u) << u;
        }
    }

    // copies columns [k0, k0 + 64) of the planned rows into the tile at smem_tile (rows
    // past the group are zero-filled)
    __device__ __forceinline__ void issue(uint32_t smem_tile, const bf16* x, int k0,
                                          int lane) const {
        const int c = lane & 7;
#pragma unroll
        for (int u = 0; u < kChunks; ++u) {
            // branch-free: rows past the group get a zero fill (no global read)
            const int r = (lane >> 3) + 4 * u;
            const bool live = (valid >> u) & 1u;
            cp_async_16(smem_tile + r * 128 + ((c ^ (r & 7)) << 4), x + src_off[u] + k0,
                        live ? 16u : 0u);
        }
    }
};

template <int BN, bool GATE_UP>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap map_w,
                    const __grid_constant__ CUtensorMap map_act, Params p) {
    using C = Cfg<BN, GATE_UP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
    uint64_t* empty = full + C::kStages;
    uint64_t* tfull = empty + C::kStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* total_slot = reinterpret_cast<int*>(tmem_slot + 2);
    int* g_off = reinterpret_cast<int*>(tmem_slot + 4);
    int* g_tile = g_off + (p.G + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // gate_up with gathered rows: the 32 producer lanes also arrive (after their cp.async)
    const bool gather = GATE_UP && p.gather_tok != nullptr;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], gather ? 1 + 32 : 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kEpiThreads);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_w);
        if (!gather) tma_prefetch_desc(&map_act);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    // everything above overlaps the previous kernel's tail; the offsets, the activations
    // and the accumulator are produced by earlier kernels of the stream
    grid_dep_wait();
    grid_dep_launch();
    build_tile_table(p, BN, g_off, g_tile, total_slot, warp, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // units: (group tile, K slice) with the slice varying fastest, so that CTAs working at
    // the same time read different K ranges of the weights
    const Units units = plan_units(p, *total_slot, GATE_UP);
    const int total = units.total;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        // Weights (operand A) always by TMA from lane 0.  Activation rows (operand B, the
        // tile's bn rows): 16-row TMA boxes when they are contiguous in expert order;
        // otherwise (gather) each lane copies 16-byte chunks of x[gather_tok[row]] with
        // cp.async into the swizzled tile (RowGather).
        if (gather || lane == 0) {
            const uint64_t pol_w = policy_evict_first();  // weights stream through once
            const uint64_t pol_a = policy_evict_last();   // activations are re-read
            const uint32_t a_bytes = C::kNumA * C::kABytes;
            int stage = 0;
            uint32_t phase = 0, filled = 0, fill_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const Unit un = unit_at(units, tile);
                const Tile t = decode_tile(un.tile, g_tile, g_off, p.G, BN);
                const int kb = slice_begin(p.nk, un.nsl, un.slice);
                const int ke = slice_begin(p.nk, un.nsl, un.slice + 1);
                const int wr0 = t.g * p.w_group_rows + t.i * kBM;
                RowGather<BN> rg;
                if (gather) rg.plan(p.gather_tok, t.row0, t.row_end, p.nk * kBK, lane);
                for (int kk = kb; kk < ke; ++kk) {
                    bool got = mbar_wait(&empty[stage], phase ^ 1u, kWaitBudgetNs, abort_flag);
                    if (gather) got = __all_sync(0xffffffffu, got);
                    if (!got) {
                        set_status(p.status, MOE_ERR_TIMEOUT);
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + stage * C::kStageBytes;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full[stage], gather ? a_bytes : C::kStageBytes);
                        tma_load_2d(st, &map_w, &full[stage], kk * kBK, wr0, pol_w);
                        if (GATE_UP)
                            tma_load_2d(st + C::kABytes, &map_w, &full[stage], kk * kBK,
                                        wr0 + p.up_rows, pol_w);
                        if (!gather)  // act_box rows per box: one box per stage
                            for (int b = 0; b < BN; b += p.act_box)
                                tma_load_2d(st + a_bytes + b * kBK * 2, &map_act, &full[stage],
                                            kk * kBK, t.row0 + b, pol_a);
                    }
                    if (gather) {
                        rg.issue(smem_u32(st + a_bytes), p.x, kk * kBK, lane);
                        cp_async_mbar_arrive_noinc(&full[stage]);
                    }
                    filled |= 1u << stage;
                    fill_phase = (fill_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
                }
            }
            if (gather) cp_async_wait_all();
            if (!ok && lane == 0) {  // let the copies already in flight land before exiting
                for (int s = 0; s < C::kStages; ++s)
                    if (filled & (1u << s))
                        mbar_wait(&full[s], (fill_phase >> s) & 1u, kDrainBudgetNs, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, abuf = 0, aphase = 0;
            bool ok = true, issued = false;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                if (!mbar_wait(&tempty[abuf], aphase ^ 1u, kWaitBudgetNs, abort_flag)) {
                    set_status(p.status, MOE_ERR_TIMEOUT);
                    *abort_flag = 1;
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d0 = tmem_base + abuf * C::kAccCols;
                constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN);
                const Unit un = unit_at(units, tile);
                const int nks = slice_begin(p.nk, un.nsl, un.slice + 1) -
                                slice_begin(p.nk, un.nsl, un.slice);
                for (int kk = 0; kk < nks; ++kk) {
                    if (!mbar_wait(&full[stage], phase, kWaitBudgetNs, abort_flag)) {
                        set_status(p.status, MOE_ERR_TIMEOUT);
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (gather) fence_proxy_async_smem();
                    const uint32_t a0 = smem_u32(smem + stage * C::kStageBytes);
                    const uint32_t a1 = a0 + C::kABytes;
                    const uint32_t b0 = a0 + C::kNumA * C::kABytes;
#pragma unroll
                    for (int s = 0; s < kBK / 16; ++s) {
                        const uint32_t acc = (kk | s) != 0 ? 1u : 0u;
                        const uint64_t bd = sdesc_k_sw128(b0 + s * 32);
                        umma_bf16(d0, sdesc_k_sw128(a0 + s * 32), bd, idesc, acc);
                        if (GATE_UP) umma_bf16(d0 + BN, sdesc_k_sw128(a1 + s * 32), bd, idesc, acc);
                    }
                    issued = true;
                    umma_commit(&empty[stage]);
                    if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit(&tfull[abuf]);
                abuf ^= 1u;
                if (abuf == 0) aphase ^= 1u;
            }
            if (!ok && issued) {  // the MMAs still read shared memory: wait for them
                umma_commit(drain);
                mbar_wait(drain, 0, kDrainBudgetNs, nullptr);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue
        const int q = warp & 3;  // tensor-memory lane quarter this warp may read
        const int feat_in_tile = q * 32 + lane;
        if (GATE_UP) clear_accumulator(p, threadIdx.x - 64, kEpiThreads);
        uint32_t abuf = 0, aphase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const Unit un = unit_at(units, tile);
            const Tile t = decode_tile(un.tile, g_tile, g_off, p.G, BN);
            float* y_slice = p.y_out ? p.y_out + un.slice * p.split_stride : nullptr;
            // gate_up cut into slices: this slice's partial sums, [row][gate f | up f]
            float* part = (GATE_UP && un.nsl > 1)
                              ? p.part + static_cast<size_t>(un.slice) * p.part_rows * 2 * p.out_cols
                              : nullptr;
            const int nsplit = un.nsl;
            const bool ready = mbar_wait(&tfull[abuf], aphase, kWaitBudgetNs, abort_flag);
            if (!epilogue_bar_and(ready)) {
                set_status(p.status, MOE_ERR_TIMEOUT);
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   abuf * C::kAccCols;
            const int feat = t.i * kBM + feat_in_tile;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 16) {
                uint32_t gv[16];
                uint32_t uv[16];
                tmem_ld16(tbase + c0, gv);
                if (GATE_UP) tmem_ld16(tbase + BN + c0, uv);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const int row = t.row0 + c0 + c;
                    if (row >= t.row_end) break;
                    const float g = __uint_as_float(gv[c]);
                    if (GATE_UP && part) {
                        float* pr = part + static_cast<size_t>(row) * 2 * p.out_cols;
                        __stcg(pr + feat, g);
                        __stcg(pr + p.out_cols + feat, __uint_as_float(uv[c]));
                    } else if (GATE_UP) {
                        const float u = __uint_as_float(uv[c]);
                        const float h = g / (1.f + __expf(-g)) * u;
                        p.h_out[static_cast<size_t>(row) * p.out_cols + feat] = __float2bfloat16_rn(h);
                    } else {
                        const float w = p.sorted_w ? __ldg(p.sorted_w + row) : 1.f;
                        const float v = w * g;
                        if (p.acc_out) {
                            const int tok = p.sorted_token ? __ldg(p.sorted_token + row) : row;
                            red_add_f32(p.acc_out + static_cast<size_t>(tok) * p.out_cols + feat, v);
                        }
                        if (y_slice) y_slice[static_cast<size_t>(row) * p.out_cols + feat] = v;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[abuf]);
            abuf ^= 1u;
            if (abuf == 0) aphase ^= 1u;
            // the slice that completes the tile: sum the slices' partial sums in slice
            // order, then SwiGLU into h
            if (GATE_UP && part && split_tile_done<kEpiThreads>(p, un.tile, nsplit, 64)) {
                // 4 rows' partial sums in flight at a time
                const int row_hi = min(t.row0 + BN, t.row_end);
#pragma unroll 1
                for (int r0 = t.row0; r0 < row_hi; r0 += 4) {
                    float gs[4][kSplitSlicesMax], us[4][kSplitSlicesMax];
#pragma unroll
                    for (int r = 0; r < 4; ++r)
#pragma unroll
                        for (int sl = 0; sl < kSplitSlicesMax; ++sl) {
                            gs[r][sl] = us[r][sl] = 0.f;
                            if (sl >= nsplit || r0 + r >= row_hi) continue;
                            const float* pr = p.part +
                                (static_cast<size_t>(sl) * p.part_rows + r0 + r) * 2 * p.out_cols;
                            gs[r][sl] = __ldcg(pr + feat);
                            us[r][sl] = __ldcg(pr + p.out_cols + feat);
                        }
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        if (r0 + r >= row_hi) break;
                        float g = 0.f, u = 0.f;
#pragma unroll
                        for (int sl = 0; sl < kSplitSlicesMax; ++sl) {
                            g += gs[r][sl];  // slices past nsplit hold 0
                            u += us[r][sl];
                        }
                        const float h = g / (1.f + __expf(-g)) * u;
                        p.h_out[static_cast<size_t>(r0 + r) * p.out_cols + feat] = __float2bfloat16_rn(h);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
    if (!GATE_UP && p.final_out != nullptr) finalize_output(p);
}

// ---------------------------------------------------------------- tokens-on-M variant
// For groups with more than a handful of rows: the MMA's M side holds 128 token rows and
// its N side 256 weight rows (gate_up: the gate and up rows of the same 128 features;
// down: 256 output features), one tcgen05.mma of 128 x 256 x 16 per 16 of K.  Each
// epilogue thread owns one row, so h is written with 16-byte stores and the down epilogue
// reduces 16-byte vectors (red.global.add.v4.f32) into the token's output row.  The
// CTA-pair kernel shares the tile shape.
constexpr int kTmRows = 128;  // token rows per tile (MMA M)
// weights on M while no group can exceed this many rows (a handful of tokens): measured
// faster than tokens on M there (one token: 47 vs 50 us for gate_up at the Zipf T=1 shape)
constexpr int kSwapMaxRows = 16;
constexpr int kTmN = 256;     // weight rows per tile (MMA N)
// 2 warps (producer, MMA) + 8 epilogue warps: two warps per tensor-memory lane quarter,
// each draining half of the accumulator's columns
constexpr int kTmThreads = 64 + 256;
constexpr int kTmEpiThreads = 256;


// Reductions into the fp32 accumulator keep its lines in L2 (evict-last) while the expert
// weights stream through (evict-first).
__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
    const uint64_t pol = policy_evict_last();
    asm volatile("red.global.add.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(addr),
                 "f"(a), "f"(b), "f"(c), "f"(d), "l"(pol)
                 : "memory");
}

// 16 SwiGLU values of one row (gate and up accumulators, fp32 bits) -> 16 bf16 in h.
__device__ __forceinline__ void swiglu_store16(const uint32_t* gv, const uint32_t* uv, bf16* dst) {
    uint32_t pk[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float g0 = __uint_as_float(gv[2 * j]);
        const float g1 = __uint_as_float(gv[2 * j + 1]);
        const float h0 = __fdividef(g0, 1.f + __expf(-g0)) * __uint_as_float(uv[2 * j]);
        const float h1 = __fdividef(g1, 1.f + __expf(-g1)) * __uint_as_float(uv[2 * j + 1]);
        pk[j] = pack_bf16x2(h0, h1);
    }
    uint4* d = reinterpret_cast<uint4*>(dst);
    d[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    d[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}

// The warp's 32 rows x 16 columns of w * v (v: fp32 bits, this lane's row) reduced into the
// token rows through shared memory: a thread holds one row, and a 4-wide reduction per
// thread and row would touch 32 rows' lines with 16 bytes each; transposed through
// `stage` (2 KB, 16-byte chunks XOR-swizzled so that both the row-wise writes and the
// transposed reads are free of bank conflicts) each reduction instruction covers 8 rows x
// 64 contiguous bytes: whole 32-byte sectors.
__device__ __forceinline__ void reduce16_transposed(const Params& p, const uint32_t* v, float w,
                                                    int tok, bool valid, int col, float* stage,
                                                    int lane) {
    const int rr0 = lane >> 2, kq = lane & 3;  // read side: row (of 8), chunk
#pragma unroll
    for (int k = 0; k < 4; ++k)
        *reinterpret_cast<float4*>(stage + lane * 16 + ((k ^ ((lane >> 1) & 3)) << 2)) =
            make_float4(w * __uint_as_float(v[4 * k]), w * __uint_as_float(v[4 * k + 1]),
                        w * __uint_as_float(v[4 * k + 2]), w * __uint_as_float(v[4 * k + 3]));
    __syncwarp();
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int rr = it * 8 + rr0;
        const float4 val =
            *reinterpret_cast<const float4*>(stage + rr * 16 + ((kq ^ ((rr >> 1) & 3)) << 2));
        const int tok_r = __shfl_sync(0xffffffffu, tok, rr);
        const bool valid_r = __shfl_sync(0xffffffffu, valid ? 1 : 0, rr) != 0;
        if (valid_r)
            red_add_v4(p.acc_out + static_cast<size_t>(tok_r) * p.out_cols + col + 4 * kq, val.x,
                       val.y, val.z, val.w);
    }
    __syncwarp();
}

// gate_up cut into K slices, slice `share` of nsplit once all slices have posted:
// h[row, feat0 + j] for its share of the (row, 8-feature chunk) items of the tile's rows
// [row0, row_end) and F features, from the slices' partial sums added in slice order.  The
// epilogue threads share the items, so that a share of a few rows costs one round trip to
// L2.
template <int kThreads>
__device__ __forceinline__ void split_fixup_tile(const Params& p, int row0, int row_end,
                                                 int feat0, int F, int nsplit, int share,
                                                 int epi_tid) {
    const int chunks = F / 8;
    const int items = (row_end - row0) * chunks;
    const int it_end = static_cast<int>(static_cast<long long>(items) * (share + 1) / nsplit);
#pragma unroll 1
    for (int it = static_cast<int>(static_cast<long long>(items) * share / nsplit) + epi_tid;
         it < it_end; it += kThreads) {
        const int row = row0 + it / chunks;
        const int f = feat0 + (it % chunks) * 8;
        float4 a[kSplitSlicesMax][2], b[kSplitSlicesMax][2];
#pragma unroll
        for (int sl = 0; sl < kSplitSlicesMax; ++sl) {
            if (sl >= nsplit) break;
            const float* pr =
                p.part + (static_cast<size_t>(sl) * p.part_rows + row) * 2 * p.out_cols + f;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                a[sl][j] = __ldcg(reinterpret_cast<const float4*>(pr) + j);
                b[sl][j] = __ldcg(reinterpret_cast<const float4*>(pr + p.out_cols) + j);
            }
        }
        float g[8], u[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) g[j] = u[j] = 0.f;
#pragma unroll
        for (int sl = 0; sl < kSplitSlicesMax; ++sl) {
            if (sl >= nsplit) break;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                g[4 * j] += a[sl][j].x; g[4 * j + 1] += a[sl][j].y;
                g[4 * j + 2] += a[sl][j].z; g[4 * j + 3] += a[sl][j].w;
                u[4 * j] += b[sl][j].x; u[4 * j + 1] += b[sl][j].y;
                u[4 * j + 2] += b[sl][j].z; u[4 * j + 3] += b[sl][j].w;
            }
        }
        uint32_t pk[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float h0 = __fdividef(g[2 * j], 1.f + __expf(-g[2 * j])) * u[2 * j];
            const float h1 = __fdividef(g[2 * j + 1], 1.f + __expf(-g[2 * j + 1])) * u[2 * j + 1];
            pk[j] = pack_bf16x2(h0, h1);
        }
        *reinterpret_cast<uint4*>(p.h_out + static_cast<size_t>(row) * p.out_cols + f) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
}

// Epilogue of one tokens-on-M tile (wn weight rows) for one epilogue warp: `half` selects
// the columns this warp drains (gate_up: features [wn/4 half, wn/4 (half + 1)) of the
// tile's wn/2; down: output columns [wn/2 half, wn/2 (half + 1)) of its wn).  The warp's
// 32 lanes are 32 rows.
// ROWS16: the kernel may write bf16 rows (p.y16_out; the CTA-pair kernel only).
template <bool GATE_UP, bool ROWS16 = false>
__device__ __forceinline__ void tm_epilogue(const Params& p, uint32_t tbase, int row, bool valid,
                                            int tile_i, int half, float* stage, int wn,
                                            float* part = nullptr) {
    const int lane = threadIdx.x & 31;
    if (GATE_UP && part) {
        // one K slice of the tile: fp32 partial sums of the gate and up features
        const int F = wn >> 1;
        const int hc = F >> 1;
        float* prow = part + static_cast<size_t>(row) * 2 * p.out_cols + tile_i * F + half * hc;
#pragma unroll 1
        for (int c0 = 0; c0 < hc; c0 += 32) {
            uint32_t gv[32], uv[32];
            tmem_ld32(tbase + half * hc + c0, gv);
            tmem_ld32(tbase + F + half * hc + c0, uv);
            tmem_ld_wait();
            if (valid) {
                float4* dg = reinterpret_cast<float4*>(prow + c0);
                float4* du = reinterpret_cast<float4*>(prow + p.out_cols + c0);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    __stcg(dg + j, make_float4(__uint_as_float(gv[4 * j]), __uint_as_float(gv[4 * j + 1]),
                                               __uint_as_float(gv[4 * j + 2]), __uint_as_float(gv[4 * j + 3])));
                    __stcg(du + j, make_float4(__uint_as_float(uv[4 * j]), __uint_as_float(uv[4 * j + 1]),
                                               __uint_as_float(uv[4 * j + 2]), __uint_as_float(uv[4 * j + 3])));
                }
            }
        }
    } else if (GATE_UP) {
        const int F = wn >> 1;        // features of the tile
        const int hc = F >> 1;        // features of this warp: 64, 32 or 16
        bf16* hrow = p.h_out + static_cast<size_t>(row) * p.out_cols + tile_i * F + half * hc;
        if (hc >= 32) {
#pragma unroll 1
            for (int c0 = 0; c0 < hc; c0 += 32) {
                uint32_t gv[32], uv[32];
                tmem_ld32(tbase + half * hc + c0, gv);
                tmem_ld32(tbase + F + half * hc + c0, uv);
                tmem_ld_wait();
                if (valid) {
                    swiglu_store16(gv, uv, hrow + c0);
                    swiglu_store16(gv + 16, uv + 16, hrow + c0 + 16);
                }
            }
        } else {
            uint32_t gv[16], uv[16];
            tmem_ld16(tbase + half * hc, gv);
            tmem_ld16(tbase + F + half * hc, uv);
            tmem_ld_wait();
            if (valid) swiglu_store16(gv, uv, hrow);
        }
    } else {
        const int hc = wn >> 1;  // output columns of this warp: 128, 64 or 32
        const float w = (valid && p.sorted_w) ? __ldg(p.sorted_w + row) : 1.f;
        const int tok = valid ? (p.sorted_token ? __ldg(p.sorted_token + row) : row) : 0;
        const int col0 = tile_i * wn + half * hc;
        const uint32_t tcol = tbase + half * hc;
        // a warp with a handful of rows (a few tokens per expert) reduces row by row: the
        // transpose would move 32 rows through shared memory for 2 or 3 of them
        const bool sparse = __popc(__ballot_sync(0xffffffffu, valid)) <= 4;
        if (p.acc_out && sparse) {
#pragma unroll 1
            for (int c0 = 0; c0 < hc; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tcol + c0, v);
                tmem_ld_wait();
                if (valid) {
                    float* dst = p.acc_out + static_cast<size_t>(tok) * p.out_cols + col0 + c0;
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        red_add_v4(dst + j, w * __uint_as_float(v[j]), w * __uint_as_float(v[j + 1]),
                                   w * __uint_as_float(v[j + 2]), w * __uint_as_float(v[j + 3]));
                }
            }
        } else if (p.acc_out) {
            // 16 columns at a time, the next 16 loaded from tensor memory while these are
            // reduced (tcgen05.wait::ld only after the shared-memory transpose)
            uint32_t va[16], vb[16];
            tmem_ld16(tcol, va);
            tmem_ld_wait_dep(va);
#pragma unroll 1
            for (int c0 = 0; c0 < hc; c0 += 32) {
                tmem_ld16(tcol + c0 + 16, vb);
                reduce16_transposed(p, va, w, tok, valid, col0 + c0, stage, lane);
                tmem_ld_wait_dep(vb);
                if (c0 + 32 < hc) tmem_ld16(tcol + c0 + 32, va);
                reduce16_transposed(p, vb, w, tok, valid, col0 + c0 + 16, stage, lane);
                tmem_ld_wait_dep(va);
            }
        }
#pragma unroll 1
        for (int c0 = 0; c0 < hc && ROWS16 && p.y16_out; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tcol + c0, v);
            tmem_ld_wait();
            if (valid) {
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    pk[j] = pack_bf16x2(w * __uint_as_float(v[2 * j]), w * __uint_as_float(v[2 * j + 1]));
                uint4* dst = reinterpret_cast<uint4*>(
                    p.y16_out + static_cast<size_t>(row) * p.out_cols + col0 + c0);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            }
        }
#pragma unroll 1
        for (int c0 = 0; c0 < hc && p.y_out; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tcol + c0, v);
            tmem_ld_wait();
            if (valid) {
                float4* dst = reinterpret_cast<float4*>(
                    p.y_out + static_cast<size_t>(row) * p.out_cols + col0 + c0);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    dst[j] = make_float4(w * __uint_as_float(v[4 * j]), w * __uint_as_float(v[4 * j + 1]),
                                         w * __uint_as_float(v[4 * j + 2]),
                                         w * __uint_as_float(v[4 * j + 3]));
            }
        }
    }
}

// down epilogue staging of the tokens-on-M kernels: 2 KB per epilogue warp, after the
// group table
constexpr int kStageFloatsPerWarp = 32 * 16;
constexpr size_t kEpiStageBytes = 16 + (kTmEpiThreads / 32) * kStageFloatsPerWarp * sizeof(float);
__device__ __forceinline__ float* epi_stage(int* table_end, int warp) {
    const uintptr_t a = (reinterpret_cast<uintptr_t>(table_end) + 15) & ~static_cast<uintptr_t>(15);
    return reinterpret_cast<float*>(a) + (warp - 2) * kStageFloatsPerWarp;
}

struct CfgTm {
    static constexpr int kABytes = kTmRows * kBK * 2;  // 16 KB of token rows
    static constexpr int kBBytes = kTmN * kBK * 2;     // 32 KB of weight rows
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = 4;
    static constexpr int kAccCols = kTmN;
    static constexpr int kTmemCols = 2 * kAccCols;
    static_assert(kTmemCols <= 512, "accumulators exceed tensor memory");
};

template <bool GATE_UP>
__global__ void __launch_bounds__(kTmThreads, 1)
grouped_gemm_tm_kernel(const __grid_constant__ CUtensorMap map_w,
                       const __grid_constant__ CUtensorMap map_act, Params p) {
    using C = CfgTm;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
    uint64_t* empty = full + C::kStages;
    uint64_t* tfull = empty + C::kStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* total_slot = reinterpret_cast<int*>(tmem_slot + 2);
    int* g_off = reinterpret_cast<int*>(tmem_slot + 4);
    int* g_tile = g_off + (p.G + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const bool gather = GATE_UP && p.gather_tok != nullptr;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], gather ? 1 + 32 : 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kTmEpiThreads);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_w);
        if (!gather) tma_prefetch_desc(&map_act);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    grid_dep_wait();
    grid_dep_launch();
    build_tile_table(p, kTmRows, g_off, g_tile, total_slot, warp, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // units: (tile, K slice), the slice varying fastest
    const Units units = plan_units(p, *total_slot, GATE_UP);
    const int total = units.total;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        // token rows (A): one TMA box of 128 rows when contiguous, else the lanes gather
        // them with cp.async; weight rows (B): two TMA boxes of 128 rows.
        if (gather || lane == 0) {
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_a = policy_evict_last();
            int stage = 0;
            uint32_t phase = 0, filled = 0, fill_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const Unit un = unit_at(units, tile);
                const Tile t = decode_tile(un.tile, g_tile, g_off, p.G, kTmRows);
                const int kb = slice_begin(p.nk, un.nsl, un.slice);
                const int ke = slice_begin(p.nk, un.nsl, un.slice + 1);
                // gate_up: gate rows g*2f + i*128 and up rows g*2f + f + i*128;
                // down: rows g*D + i*256 and the next 128
                const int wr0 = t.g * p.w_group_rows + t.i * (GATE_UP ? kBM : kTmN);
                const int wr1 = GATE_UP ? wr0 + p.up_rows : wr0 + kBM;
                RowGather<kTmRows> rg;
                if (gather) rg.plan(p.gather_tok, t.row0, t.row_end, p.nk * kBK, lane);
                for (int kk = kb; kk < ke; ++kk) {
                    bool got = mbar_wait(&empty[stage], phase ^ 1u, kWaitBudgetNs, abort_flag);
                    if (gather) got = __all_sync(0xffffffffu, got);
                    if (!got) {
                        set_status(p.status, MOE_ERR_TIMEOUT);
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + stage * C::kStageBytes;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full[stage], gather ? C::kBBytes : C::kStageBytes);
                        if (!gather)
                            tma_load_2d(st, &map_act, &full[stage], kk * kBK, t.row0, pol_a);
                        tma_load_2d(st + C::kABytes, &map_w, &full[stage], kk * kBK, wr0, pol_w);
                        tma_load_2d(st + C::kABytes + kBM * kBK * 2, &map_w, &full[stage],
                                    kk * kBK, wr1, pol_w);
                    }
                    if (gather) {
                        rg.issue(smem_u32(st), p.x, kk * kBK, lane);
                        cp_async_mbar_arrive_noinc(&full[stage]);
                    }
                    filled |= 1u << stage;
                    fill_phase = (fill_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
                }
            }
            if (gather) cp_async_wait_all();
            if (!ok && lane == 0) {
                for (int s = 0; s < C::kStages; ++s)
                    if (filled & (1u << s))
                        mbar_wait(&full[s], (fill_phase >> s) & 1u, kDrainBudgetNs, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kTmRows, kTmN);
            int stage = 0;
            uint32_t phase = 0, abuf = 0, aphase = 0;
            bool ok = true, issued = false;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                if (!mbar_wait(&tempty[abuf], aphase ^ 1u, kWaitBudgetNs, abort_flag)) {
                    set_status(p.status, MOE_ERR_TIMEOUT);
                    *abort_flag = 1;
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d0 = tmem_base + abuf * C::kAccCols;
                const Unit un = unit_at(units, tile);
                const int nks = slice_begin(p.nk, un.nsl, un.slice + 1) -
                                slice_begin(p.nk, un.nsl, un.slice);
                for (int kk = 0; kk < nks; ++kk) {
                    if (!mbar_wait(&full[stage], phase, kWaitBudgetNs, abort_flag)) {
                        set_status(p.status, MOE_ERR_TIMEOUT);
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (gather) fence_proxy_async_smem();
                    const uint32_t a0 = smem_u32(smem + stage * C::kStageBytes);
                    const uint32_t b0 = a0 + C::kABytes;
#pragma unroll
                    for (int s = 0; s < kBK / 16; ++s)
                        umma_bf16(d0, sdesc_k_sw128(a0 + s * 32), sdesc_k_sw128(b0 + s * 32), idesc,
                                  (kk | s) != 0 ? 1u : 0u);
                    issued = true;
                    umma_commit(&empty[stage]);
                    if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit(&tfull[abuf]);
                abuf ^= 1u;
                if (abuf == 0) aphase ^= 1u;
            }
            if (!ok && issued) {
                umma_commit(drain);
                mbar_wait(drain, 0, kDrainBudgetNs, nullptr);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue
        const int q = warp & 3;
        if (GATE_UP) clear_accumulator(p, threadIdx.x - 64, kTmEpiThreads);
        uint32_t abuf = 0, aphase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const Unit un = unit_at(units, tile);
            const Tile t = decode_tile(un.tile, g_tile, g_off, p.G, kTmRows);
            const bool ready = mbar_wait(&tfull[abuf], aphase, kWaitBudgetNs, abort_flag);
            if (!epilogue_bar_and<kTmEpiThreads>(ready)) {
                set_status(p.status, MOE_ERR_TIMEOUT);
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   abuf * C::kAccCols;
            const int row = t.row0 + q * 32 + lane;
            const bool valid = row < t.row_end;
            const int half = (warp - 2) >> 2;
            // gate_up cut into slices: this slice's partial sums, [row][gate f | up f]
            float* part = (GATE_UP && un.nsl > 1)
                              ? p.part + static_cast<size_t>(un.slice) * p.part_rows * 2 * p.out_cols
                              : nullptr;
            tm_epilogue<GATE_UP>(p, tbase, row, valid, t.i, half,
                                 GATE_UP ? nullptr : epi_stage(g_tile + p.G + 1, warp), kTmN, part);
            tc_fence_before();
            mbar_arrive(&tempty[abuf]);
            abuf ^= 1u;
            if (abuf == 0) aphase ^= 1u;
            // every slice of the tile, once all have posted, sums its share of the rows'
            // partial sums in slice order and applies SwiGLU
            if (GATE_UP && part) {
                if (split_tile_all_posted<kTmEpiThreads>(p, un.tile, un.nsl, 64))
                    split_fixup_tile<kTmEpiThreads>(p, t.row0, min(t.row0 + kTmRows, t.row_end),
                                                    t.i * (kTmN / 2), kTmN / 2, un.nsl, un.slice,
                                                    threadIdx.x - 64);
                else if (threadIdx.x == 64)
                    set_status(p.status, MOE_ERR_TIMEOUT);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
    if (!GATE_UP && p.final_out != nullptr) finalize_output(p);
}

// ---------------------------------------------------------------- CTA-pair variant
// For groups with many rows, two CTAs of a cluster share one tcgen05.mma of 256 x 256 x 16
// (cta_group::2): CTA r holds token rows [128 r, 128 r + 128) of a 256-row block (its half
// of A) and weight rows [128 r, 128 r + 128) of the 256-row block (its half of B) -- for
// gate_up the leader's half is the 128 gate rows and the peer's the 128 up rows of the same
// features -- and receives its 128 rows x 256 columns of D in its own tensor memory.  Each
// CTA loads 32 KB per K step instead of 48 KB, and 6 stages fit.  Both CTAs' TMA loads are
// counted on the leader's full barrier; the leader's single MMA thread commits to the
// empty and accumulator-full barriers of both CTAs; the peer's epilogue warps arrive on the
// leader's accumulator-empty barrier.  A's rows must be contiguous (x gathered into expert
// order beforehand for gate_up).
struct CfgPair {
    static constexpr int kABytes = kTmRows * kBK * 2;  // this CTA's 128 token rows: 16 KB
    static constexpr int kBBytes = kBM * kBK * 2;      // this CTA's 128 weight rows: 16 KB
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = 6;
    static constexpr int kAccCols = kTmN;
    static constexpr int kTmemCols = 2 * kAccCols;
    static constexpr int kPairRows = 2 * kTmRows;  // token rows per pair tile
};

template <bool GATE_UP>
__global__ void __launch_bounds__(kTmThreads, 1)
grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_w,
                         const __grid_constant__ CUtensorMap map_act, Params p) {
    using C = CfgPair;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
    uint64_t* empty = full + C::kStages;
    uint64_t* tfull = empty + C::kStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* total_slot = reinterpret_cast<int*>(tmem_slot + 2);
    int* g_off = reinterpret_cast<int*>(tmem_slot + 4);
    int* g_tile = g_off + (p.G + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: leader (issues the MMAs), 1: peer
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);   // leader: one expect-tx arrival; both CTAs' bytes
            mbar_init(&empty[s], 1);  // both: the leader's multicast commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);    // both: the leader's multicast commit
            mbar_init(&tempty[b], 16);  // leader: the 8 epilogue warps of each CTA
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&map_w);
        tma_prefetch_desc(&map_act);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, C::kTmemCols);
        tmem_relinquish_pair();
    }
    grid_dep_wait();
    grid_dep_launch();
    build_tile_table(p, C::kPairRows, g_off, g_tile, total_slot, warp, lane);
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers and tensor memory exist before any pair operation
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = *total_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer (both)
        if (lane == 0) {
            // a weight tile is read by every row block of its expert (consecutive tiles, run by
            // pairs at about the same time): kept in L2 like the token rows for the others
            const uint64_t pol_w = policy_evict_last();
            const uint64_t pol_a = policy_evict_last();
            int stage = 0;
            uint32_t phase = 0, filled = 0, fill_phase = 0;
            bool ok = true;
            for (int tile = pair; tile < total && ok; tile += npairs) {
                const Tile t = decode_tile(tile, g_tile, g_off, p.G, C::kPairRows);
                const int arow = t.row0 + static_cast<int>(rank) * kTmRows;
                // gate_up: leader = gate rows, peer = up rows of features i*128..+127;
                // down: rows i*256 + 128*rank
                const int wrow = GATE_UP ? t.g * p.w_group_rows + t.i * kBM + (rank ? p.up_rows : 0)
                                         : t.g * p.w_group_rows + t.i * kTmN + rank * kBM;
                for (int kk = 0; kk < p.nk; ++kk) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, kWaitBudgetNs, abort_flag)) {
                        set_status(p.status, MOE_ERR_TIMEOUT);
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + stage * C::kStageBytes;
                    const uint32_t leader_full = map_to_rank(smem_u32(&full[stage]), 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * C::kStageBytes);
                    tma_load_2d_pair(st, &map_act, leader_full, kk * kBK, arow, pol_a);
                    tma_load_2d_pair(st + C::kABytes, &map_w, leader_full, kk * kBK, wrow, pol_w);
                    filled |= 1u << stage;
                    fill_phase = (fill_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok && rank == 0) {
                for (int s = 0; s < C::kStages; ++s)
                    if (filled & (1u << s))
                        mbar_wait(&full[s], (fill_phase >> s) & 1u, kDrainBudgetNs, nullptr);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA (leader)
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(2 * kTmRows, kTmN);
            int stage = 0;
            uint32_t phase = 0, abuf = 0, aphase = 0;
            bool ok = true, issued = false;
            for (int tile = pair; tile < total && ok; tile += npairs) {
                if (!mbar_wait(&tempty[abuf], aphase ^ 1u, kWaitBudgetNs, abort_flag)) {
                    set_status(p.status, MOE_ERR_TIMEOUT);
                    *abort_flag = 1;
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d0 = tmem_base + abuf * C::kAccCols;
                for (int kk = 0; kk < p.nk; ++kk) {
                    if (!mbar_wait(&full[stage], phase, kWaitBudgetNs, abort_flag)) {
                        set_status(p.status, MOE_ERR_TIMEOUT);
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smem + stage * C::kStageBytes);
                    const uint32_t b0 = a0 + C::kABytes;
#pragma unroll
                    for (int s = 0; s < kBK / 16; ++s)
                        umma_bf16_pair(d0, sdesc_k_sw128(a0 + s * 32), sdesc_k_sw128(b0 + s * 32),
                                       idesc, (kk | s) != 0 ? 1u : 0u);
                    issued = true;
                    umma_commit_pair(&empty[stage]);
                    if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                umma_commit_pair(&tfull[abuf]);
                abuf ^= 1u;
                if (abuf == 0) aphase ^= 1u;
            }
            if (!ok && issued) {
                umma_commit_pair(drain);
                mbar_wait(drain, 0, kDrainBudgetNs, nullptr);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- epilogue (both)
        const int q = warp & 3;
        if (GATE_UP) clear_accumulator(p, threadIdx.x - 64, kTmEpiThreads);
        const uint32_t leader_tempty0 = map_to_rank(smem_u32(&tempty[0]), 0);
        uint32_t abuf = 0, aphase = 0;
        for (int tile = pair; tile < total; tile += npairs) {
            const Tile t = decode_tile(tile, g_tile, g_off, p.G, C::kPairRows);
            const bool ready = mbar_wait(&tfull[abuf], aphase, kWaitBudgetNs, abort_flag);
            if (!epilogue_bar_and<kTmEpiThreads>(ready)) {
                set_status(p.status, MOE_ERR_TIMEOUT);
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   abuf * C::kAccCols;
            const int row = t.row0 + static_cast<int>(rank) * kTmRows + q * 32 + lane;
            tm_epilogue<GATE_UP, true>(p, tbase, row, row < t.row_end, t.i, (warp - 2) >> 2,
                                       GATE_UP ? nullptr : epi_stage(g_tile + p.G + 1, warp),
                                       kTmN);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_tempty0 + abuf * 8);
            abuf ^= 1u;
            if (abuf == 0) aphase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the pair's MMAs and remote arrivals are over before tensor memory goes
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::kTmemCols);
    }
    if (!GATE_UP && p.final_out != nullptr) finalize_output(p);
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

cudaError_t get_encoder() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode ? cudaSuccess : cudaErrorNotSupported;
}

// 2-D bf16 view [rows, cols] (cols contiguous), box [box_rows, 64], 128-byte swizzle.
cudaError_t encode_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                       int box_rows) {
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// encode_map through a per-process cache keyed by (base, rows, cols, box): a descriptor
// depends on nothing else, and a layer call would otherwise encode 4 to 8 of them on the
// host.  The cache is bounded (cleared when full).
cudaError_t make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, int box_rows) {
    struct Key {
        const void* base;
        uint64_t rows, cols;
        int box;
        bool operator==(const Key& o) const {
            return base == o.base && rows == o.rows && cols == o.cols && box == o.box;
        }
    };
    struct Hash {
        size_t operator()(const Key& k) const {
            size_t h = std::hash<const void*>()(k.base);
            h = h * 1000003u ^ std::hash<uint64_t>()(k.rows);
            h = h * 1000003u ^ std::hash<uint64_t>()(k.cols);
            return h * 1000003u ^ static_cast<size_t>(k.box);
        }
    };
    static std::mutex mu;
    static std::unordered_map<Key, CUtensorMap, Hash> cache;
    const Key key{base, rows, cols, box_rows};
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find(key);
        if (it != cache.end()) {
            *m = it->second;
            return cudaSuccess;
        }
    }
    const cudaError_t err = encode_map(m, base, rows, cols, box_rows);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lock(mu);
    if (cache.size() >= 4096) cache.clear();
    cache.emplace(key, *m);
    return cudaSuccess;
}

template <int BN, bool GATE_UP>
cudaError_t launch_tpl(const CUtensorMap& mw, const CUtensorMap& ma, const Params& p, int grid,
                       cudaStream_t s, bool pdl) {
    using C = Cfg<BN, GATE_UP>;
    const size_t smem = 1024 + static_cast<size_t>(C::kStages) * C::kStageBytes +
                        (2 * C::kStages + 5) * 8 + 16 +
                        2 * (p.G + 1) * sizeof(int);
    auto kfn = grouped_gemm_kernel<BN, GATE_UP>;
    cudaError_t err = set_smem_limit(reinterpret_cast<const void*>(kfn), smem);
    if (err != cudaSuccess) return err;
    err = launch_kernel(kfn, dim3(grid), dim3(kThreads), smem, s, pdl, mw, ma, p);
    count_launches(1);
    return err;
}

template <bool GATE_UP>
cudaError_t launch_tm(const CUtensorMap& mw, const CUtensorMap& ma, const Params& p, int grid,
                      cudaStream_t s, bool pdl) {
    using C = CfgTm;
    const size_t smem = 1024 + static_cast<size_t>(C::kStages) * C::kStageBytes +
                        (2 * C::kStages + 5) * 8 + 16 + 2 * (p.G + 1) * sizeof(int) +
                        (GATE_UP ? 0 : kEpiStageBytes);
    auto kfn = grouped_gemm_tm_kernel<GATE_UP>;
    cudaError_t err = set_smem_limit(reinterpret_cast<const void*>(kfn), smem);
    if (err != cudaSuccess) return err;
    err = launch_kernel(kfn, dim3(grid), dim3(kTmThreads), smem, s, pdl, mw, ma, p);
    count_launches(1);
    return err;
}

template <bool GATE_UP>
cudaError_t launch_pair(const CUtensorMap& mw, const CUtensorMap& ma, const Params& p,
                        int npairs, cudaStream_t s, bool pdl) {
    using C = CfgPair;
    const size_t smem = 1024 + static_cast<size_t>(C::kStages) * C::kStageBytes +
                        (2 * C::kStages + 5) * 8 + 16 + 2 * (p.G + 1) * sizeof(int) +
                        (GATE_UP ? 0 : kEpiStageBytes);
    auto kfn = grouped_gemm_pair_kernel<GATE_UP>;
    cudaError_t err = set_smem_limit(reinterpret_cast<const void*>(kfn), smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * npairs);
    cfg.blockDim = dim3(kTmThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    err = cudaLaunchKernelEx(&cfg, kfn, mw, ma, p);
    count_launches(1);
    return err;
}

}  // namespace

int pick_block_rows(int rows, int groups) {
    const int avg = rows / (groups > 0 ? groups : 1);
    if (avg <= 16) return 16;
    if (avg <= 32) return 32;
    if (avg <= 64) return 64;
    return 128;
}

namespace {

enum class Kind { kSwap, kTm, kPair };

// One launch of one kernel kind over every group.  BN: largest rows per tile of the
// weights-on-M kernel.
cudaError_t launch_kind(const GroupedGemmLaunch& a, Kind kind, int BN, int num_sms,
                        cudaStream_t s, bool pdl) {
    const bool tm = kind != Kind::kSwap;
    const int K = a.gate_up ? a.D : a.f;
    const uint64_t w_group_rows = a.gate_up ? 2ull * a.f : static_cast<uint64_t>(a.D);
    CUtensorMap mw, ma;
    cudaError_t err;
    if ((err = make_map(&mw, a.w, w_group_rows * a.E, K, kBM)) != cudaSuccess) return err;  // 128-row boxes
    // the activation map is only read when the rows are contiguous (no gather); with a
    // gather it still has to be a valid descriptor, so it covers the first row of x
    const void* act = a.act;
    bool gather = a.gate_up && a.gather_tok != nullptr;
    if (kind == Kind::kPair && gather) {
        err = launch_gather_rows(reinterpret_cast<const bf16*>(a.act), a.gather_tok, a.rows, a.D,
                                 a.gather_buf, num_sms, s, pdl);
        if (err != cudaSuccess) return err;
        act = a.gather_buf;
        gather = false;
    }
    // activation boxes: 128 rows (tokens on M) or BN rows (weights on M: one box per stage)
    if ((err = make_map(&ma, act, gather ? 1 : a.rows, K, gather ? 1 : (tm ? kTmRows : BN))) !=
        cudaSuccess)
        return err;
    Params p{};
    p.offsets = a.offsets;
    p.rows_total = a.rows;
    p.sorted_token = a.sorted_token;
    p.sorted_w = a.sorted_w;
    p.G = a.E;
    p.nf = a.gate_up ? a.f / kBM : a.D / (tm ? kTmN : kBM);
    p.nk = K / kBK;
    p.w_group_rows = static_cast<int>(w_group_rows);
    p.up_rows = a.f;
    p.out_cols = a.gate_up ? a.f : a.D;
    p.h_out = a.h_out;
    p.acc_out = a.acc_out;
    p.y_out = a.y_out;
    p.y16_out = a.gate_up ? nullptr : a.y16_out;
    p.status = a.status;
    p.gather_tok = gather ? a.gather_tok : nullptr;
    p.x = reinterpret_cast<const bf16*>(act);
    p.final_out = (!a.gate_up && a.acc_out && a.done) ? a.final_out : nullptr;
    p.final_rows = a.final_rows;
    p.done = a.done;
    p.final_residual = a.final_residual;
    p.barrier_budget_ns = a.barrier_budget_ns;
    p.ksplit = kind == Kind::kSwap && a.ksplit > 1 ? a.ksplit : 1;
    p.zero_acc = a.gate_up ? a.zero_acc : nullptr;
    p.zero_n4 = a.zero_floats / 4;
    p.act_box = BN;
    p.split_stride = static_cast<long long>(a.rows) * p.out_cols;
    // K split chosen on the device: gate_up needs the partial-sum planes and tickets, down
    // adds its slices into the fp32 accumulator (not into per-row outputs)
    const bool auto_split =
        kind != Kind::kPair && p.ksplit == 1 && a.ksplit_max > 1 &&
        (a.gate_up ? (a.part != nullptr && a.tickets != nullptr && a.ticket_cap > 0)
                   : (a.acc_out != nullptr && a.y_out == nullptr && a.y16_out == nullptr));
    p.ksplit_max = auto_split ? std::min(a.ksplit_max, kSplitSlicesMax) : 1;
    p.part = a.part;
    p.part_rows = a.rows;
    p.tickets = a.tickets;
    p.ticket_cap = a.ticket_cap;
    // persistent grids: one CTA (or pair) per SM, fewer when the units cannot fill them
    const int rows_per_tile = kind == Kind::kPair ? CfgPair::kPairRows : (tm ? kTmRows : 16);
    const long long max_tiles = (static_cast<long long>(ceil_div(a.rows, rows_per_tile)) + p.G) *
                                p.nf * p.ksplit * p.ksplit_max;
    if (kind == Kind::kPair) {
        const int npairs = static_cast<int>(std::min<long long>(max_tiles, num_sms / 2));
        return a.gate_up ? launch_pair<true>(mw, ma, p, npairs, s, true)
                         : launch_pair<false>(mw, ma, p, npairs, s, true);
    }
    const int grid = static_cast<int>(max_tiles < num_sms ? max_tiles : num_sms);
    if (tm) return a.gate_up ? launch_tm<true>(mw, ma, p, grid, s, pdl)
                             : launch_tm<false>(mw, ma, p, grid, s, pdl);
    switch (BN) {
        case 16: return a.gate_up ? launch_tpl<16, true>(mw, ma, p, grid, s, pdl) : launch_tpl<16, false>(mw, ma, p, grid, s, pdl);
        case 32: return a.gate_up ? launch_tpl<32, true>(mw, ma, p, grid, s, pdl) : launch_tpl<32, false>(mw, ma, p, grid, s, pdl);
        case 64: return a.gate_up ? launch_tpl<64, true>(mw, ma, p, grid, s, pdl) : launch_tpl<64, false>(mw, ma, p, grid, s, pdl);
        case 128: return a.gate_up ? launch_tpl<128, true>(mw, ma, p, grid, s, pdl) : launch_tpl<128, false>(mw, ma, p, grid, s, pdl);
        // 256 token rows: down only (gate_up's two accumulators would not fit tensor memory)
        default: return a.gate_up ? cudaErrorInvalidValue : launch_tpl<256, false>(mw, ma, p, grid, s, pdl);
    }
}

}  // namespace

namespace {

// Kernel kind and weights-on-M tile height for a launch (see launch_grouped_gemm).
bool pick_kind(const GroupedGemmLaunch& a, int num_sms, Kind* kind, int* BN) {
    // tokens on M needs f (gate_up) or D (down) in 128- or 256-wide blocks
    const bool tm_ok = a.gate_up ? (a.f % 128 == 0) : (a.D % 256 == 0);
    const bool gathered = a.gate_up && a.gather_tok != nullptr;
    const bool pair_ok = tm_ok && (!gathered || a.gather_buf != nullptr) && num_sms >= 2;
    const int routed_rows = a.rows;
    // weights on M: tiles adapt per group up to BN, sized for groups up to 8x the average
    // (skewed routing) but never past the largest possible group
    const int max_rows = a.max_group_rows > 0 ? a.max_group_rows : routed_rows;
    const long long avg8 = 8ll * routed_rows / a.E;
    const int bn_rows = static_cast<int>(std::min<long long>(max_rows, std::max(avg8, 16ll)));
    *BN = a.block_rows ? a.block_rows : pick_block_rows(bn_rows, 1);
    if (*BN != 16 && *BN != 32 && *BN != 64 && *BN != 128 && !(*BN == 256 && !a.gate_up))
        return false;
    if (a.ksplit > 1 && (a.gate_up || !a.y_out || a.acc_out || a.final_out ||
                         (a.f / kBK) % a.ksplit != 0))
        return false;
    // Orientation.  Weights on M (token tiles of 16..128 rows) when asked for (the router's
    // split-reduction logits GEMM), or when the tokens-on-M tiles do not divide the shape.
    // Otherwise tokens on M: both orientations stream each weight tile once per row block
    // and are within a few percent of each other on 2-row groups, but tokens on M keeps
    // features along the accumulator's columns (16-byte stores and vector reductions in
    // the epilogue) and wins clearly once groups hold tens of rows; when a few experts (a
    // handful of tokens, or concentrated routing) give fewer tiles than the grid has CTAs,
    // both cut each tile's K steps on the device.  CTA pairs once the groups
    // average a full 256-row pair tile's half (their rows must be contiguous: x is
    // gathered first).
    if (a.orientation == 1 || a.block_rows || !tm_ok || a.ksplit > 1)
        *kind = Kind::kSwap;
    else if (a.orientation == 2)
        *kind = Kind::kTm;
    else if (a.orientation == 3 || routed_rows / a.E >= 128)
        *kind = pair_ok ? Kind::kPair : Kind::kTm;
    else
        *kind = max_rows <= kSwapMaxRows ? Kind::kSwap : Kind::kTm;
    return true;
}

}  // namespace

int grouped_gemm_launches(const GroupedGemmLaunch& a, int num_sms) {
    Kind kind;
    int BN;
    if (a.rows == 0 || a.E == 0 || !pick_kind(a, num_sms, &kind, &BN)) return 0;
    return (kind == Kind::kPair && a.gate_up && a.gather_tok != nullptr) ? 2 : 1;
}

bool grouped_gemm_uses_pairs(const GroupedGemmLaunch& a, int num_sms) {
    Kind kind;
    int BN;
    return pick_kind(a, num_sms, &kind, &BN) && kind == Kind::kPair;
}


cudaError_t launch_grouped_gemm(const GroupedGemmLaunch& a, int num_sms, cudaStream_t s,
                                bool pdl) {
    if (a.rows == 0 || a.E == 0) return cudaSuccess;
    if (a.E > kMaxGroups) return cudaErrorInvalidValue;
    cudaError_t err = get_encoder();
    if (err != cudaSuccess) return err;
    Kind kind;
    int BN;
    if (!pick_kind(a, num_sms, &kind, &BN)) return cudaErrorInvalidValue;
    return launch_kind(a, kind, BN, num_sms, s, pdl);
}

}  // namespace moe
