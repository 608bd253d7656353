// ep_group.cuh -- expert parallelism over G GPUs, one process each, on NVLink
// peer memory ("Low-Latency Mode API": every rank dispatches its tokens into
// the receive buffers of the ranks that own their experts and combines the
// experts' outputs back; "[Common][PyTorch] EP dispatch with unfused MXFP8
// quantization", Changes: symmetric-memory windows, and combine forward and
// backward as the reverse of the dispatch).
//
// Partitioning.  The R logical ranks of one configuration are split over the
// G GPUs in consecutive blocks of RG = R / G: GPU g holds the tokens of ranks
// g*RG .. (g+1)*RG - 1 (its N_loc = RG * T tokens, in the same order) and owns
// their experts g*EG .. (g+1)*EG - 1, EG = E / G.  Each GPU has one receive
// window of win_rows rows (and its scale region, source info, weights, expert
// outputs and gradient in the same row numbering).
//
// Virtual rows.  A row of GPU o's window is numbered o * win_rows + (row in
// the window), as if the G windows were one buffer.  With this numbering the
// single-GPU addressing is unchanged: the padded row of expert e, slot s,
// e * cap + s (cap = R * M), is the virtual row of its owner's window
// (win_rows = EG * cap), and in the packed layout expert_offset[e] holds
// owner * win_rows + (the expert's first row in its owner's window).  Kernels
// given a table of the G window bases split a virtual row into the owner and
// the row in its window.
//
// Slots.  The slot of an entry is its rank among all entries of its expert in
// (source rank, token, k) order, as on one GPU.  Each GPU first ranks its own
// entries (the single-GPU layout over its RG ranks); after every GPU's
// per-rank counts have been gathered, the entries of GPU g are shifted by the
// number of entries the ranks before g*RG send to the same expert.
#pragma once

#include <cstdint>

#include "ep_device.cuh"
#include "ep_mbar.cuh"

namespace ep {

constexpr int kGroupMaxGpus = 64;
// flag words of a GPU's window: [kind][source GPU]
enum { kFlagCounts = 0, kFlagDispatch = 1, kFlagExpertOut = 2, kFlagCombined = 3,
       kFlagBackward = 4, kGroupKinds = 5 };

// ---- the arithmetic of the partitioning, shared by the kernels and the host ----
struct GroupShape {
    int R, E, G, g, RG, EG;
    int64_t win_rows;
};

// entries the ranks before r0 send to expert e: sum_{r < r0} tpe[r][e]
__host__ __device__ inline int64_t group_prefix(const int32_t *tpe_all, int E, int r0, int e) {
    int64_t s = 0;
    for (int r = 0; r < r0; r++) s += tpe_all[(int64_t)r * E + e];
    return s;
}
__host__ __device__ inline int64_t group_total(const int32_t *tpe_all, int R, int E, int e) {
    return group_prefix(tpe_all, E, R, e);
}
// owner GPU of a virtual row, and the row in its window
__host__ __device__ inline int group_owner(int64_t vrow, int64_t win_rows) {
    return (int)(vrow / win_rows);
}

// Packed layout: virtual offsets of every expert from the per-expert totals.
// Experts of one owner follow one another in its window, each rounded up to
// `align` rows; expert_offset[E] = G * win_rows.  (The plain statement, run on
// the host; the plan kernel computes the same with a block-wide scan.)
__host__ __device__ inline void group_packed_offsets(const GroupShape &s, const int64_t *total,
                                                     int align, int64_t *expert_offset) {
    for (int o = 0; o < s.G; o++) {
        int64_t off = (int64_t)o * s.win_rows;
        for (int e = o * s.EG; e < (o + 1) * s.EG; e++) {
            expert_offset[e] = off;
            off += (total[e] + align - 1) / align * align;
        }
    }
    expert_offset[s.E] = (int64_t)s.G * s.win_rows;
}

struct GroupPlanArgs {
    GroupShape s;
    int packed, align;
    const uint64_t *my_flags;    // this GPU's flag words: the plan waits for every GPU's counts
    uint64_t epoch;
    uint32_t *status;
    int64_t n_loc, K;            // local entries: n_loc tokens x K
    const int32_t *tpe_all;      // [R][E] every rank's per-expert counts
    TopkIdx idx;                 // local topk_idx [n_loc][K]
    int32_t *slot;               // [n_loc][K]: local ranks in, global slots out
    int64_t *recv_count;         // [E]: entries of each expert over all GPUs
    int64_t *expert_offset;      // [E+1] virtual offsets (packed; may be null when padded)
    int64_t *stats;              // [E] += recv_count of the owned experts (nullable)
    int64_t *slot_base;          // [E] scratch: this GPU's shift per expert
};

constexpr int kPlanThreads = 1024;

// One block of kPlanThreads: a warp per expert sums the gathered counts (all
// ranks, and the ranks before this GPU's), then the packed offsets come from
// a block-wide inclusive scan of the rounded totals, restarted at each
// owner's first expert.
__device__ __forceinline__ void wait_flags(const uint64_t *my_flags, int kind, int G,
                                           uint64_t epoch, uint64_t limit_ns, uint32_t *status);

__global__ void __launch_bounds__(kPlanThreads) group_plan_kernel(GroupPlanArgs a) {
    pdl_enter();
    const GroupShape &s = a.s;
    // every GPU's counts have arrived in this GPU's counts window
    if (a.my_flags) wait_flags(a.my_flags, kFlagCounts, s.G, a.epoch, kWaitLimitNs, a.status);
    __syncthreads();
    __shared__ int64_t s_v[kPlanThreads];      // rounded totals, then their inclusive scan
    __shared__ int64_t s_wsum[kPlanThreads / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int r0 = s.g * s.RG;
    for (int e = warp; e < s.E; e += nw) {
        int64_t all = 0, before = 0;
        for (int r = lane; r < s.R; r += 32) {
            const int64_t c = a.tpe_all[(int64_t)r * s.E + e];
            all += c;
            if (r < r0) before += c;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            all += __shfl_xor_sync(kFull, all, o);
            before += __shfl_xor_sync(kFull, before, o);
        }
        if (lane == 0) {
            a.recv_count[e] = all;
            a.slot_base[e] = before;
            if (a.stats && e / s.EG == s.g) a.stats[e] += all;
            s_v[e] = (all + a.align - 1) / a.align * a.align;
        }
    }
    if (!a.packed) return;
    __syncthreads();
    // inclusive scan of s_v[0..E) (E <= kPlanThreads): warp scans, then the warp sums
    const int t = threadIdx.x;
    int64_t v = t < s.E ? s_v[t] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t u = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) s_wsum[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int64_t w = lane < nw ? s_wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t u = __shfl_up_sync(kFull, w, o);
            if (lane >= o) w += u;
        }
        if (lane < nw) s_wsum[lane] = w;
    }
    __syncthreads();
    if (warp > 0) v += s_wsum[warp - 1];
    const int64_t rounded = t < s.E ? s_v[t] : 0;
    __syncthreads();
    if (t < s.E) s_v[t] = v;  // inclusive scan
    __syncthreads();
    if (t < s.E) {
        const int o = t / s.EG, first = o * s.EG;
        const int64_t start = first > 0 ? s_v[first - 1] : 0;
        a.expert_offset[t] = (int64_t)o * s.win_rows + (v - rounded - start);
    }
    if (t == 0) a.expert_offset[s.E] = (int64_t)s.G * s.win_rows;
}

// every local entry's slot shifted by its expert's base (masked entries keep -1)
__global__ void group_shift_kernel(GroupPlanArgs a) {
    pdl_enter();
    const int64_t n = a.n_loc * a.K;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t sl = a.slot[i];
        const int64_t e = a.idx[i];
        if (sl >= 0 && e >= 0 && e < a.s.E) a.slot[i] = (int32_t)(sl + a.slot_base[e]);
    }
}

// ---- flags: release stores into the peers' windows, bounded acquiring waits ----
__device__ __forceinline__ void st_release_sys(uint64_t *p, uint64_t v) {
    asm volatile("st.release.sys.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint64_t ld_acquire_sys(const uint64_t *p) {
    uint64_t v;
    asm volatile("ld.acquire.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

// GPU g tells every GPU p that its step `epoch` of `kind` is done:
// flags[p][kind][g] = epoch.  Everything this GPU wrote before (in stream
// order) is visible to a GPU that has acquired the flag.
__device__ __forceinline__ void group_signal_all(uint64_t *const *flags, int kind, int g, int G,
                                                 uint64_t epoch) {
    __threadfence_system();
    for (int p = 0; p < G; p++) st_release_sys(flags[p] + (int64_t)kind * G + g, epoch);
}

__global__ void group_signal_kernel(uint64_t *const *flags, int kind, int g, int G,
                                    uint64_t epoch) {
    pdl_enter();
    if (threadIdx.x == 0) group_signal_all(flags, kind, g, G, epoch);
}

// Wait until every GPU has signalled `kind` for `epoch` (its flag word in
// this GPU's window at least epoch); threads p < G of the block each watch
// one GPU.  Gives up after `limit_ns`, sets kDevTimeout and returns: no
// kernel waits for ever.
__device__ __forceinline__ void wait_flags(const uint64_t *my_flags, int kind, int G,
                                           uint64_t epoch, uint64_t limit_ns, uint32_t *status) {
    for (int p = threadIdx.x; p < G; p += blockDim.x) {
        const uint64_t *f = my_flags + (int64_t)kind * G + p;
        const uint64_t t0 = gtimer();
#pragma unroll 1
        while (ld_acquire_sys(f) < epoch) {
            if (gtimer() - t0 > limit_ns) {
                atomicOr(status, kDevTimeout);
                break;
            }
            __nanosleep(256);
        }
    }
}

__global__ void group_wait_kernel(const uint64_t *my_flags, int kind, int G, uint64_t epoch,
                                  uint64_t limit_ns, uint32_t *status) {
    pdl_enter();
    wait_flags(my_flags, kind, G, epoch, limit_ns, status);
    __syncthreads();
}

// This GPU's per-rank counts (rows g*RG .. of the [R][E] table, already in
// its own counts window) copied into every other GPU's counts window, then
// the counts signal.  One block.
__global__ void group_push_counts_kernel(const int32_t *mine, int32_t *const *counts,
                                         int64_t offset, int64_t n, uint64_t *const *flags, int g,
                                         int G, uint64_t epoch) {
    pdl_enter();
    for (int p = 0; p < G; p++) {
        if (p == g) continue;
        int32_t *dst = counts[p] + offset;
        for (int64_t i = threadIdx.x; i < n; i += blockDim.x) dst[i] = mine[offset + i];
    }
    __threadfence_system();
    __syncthreads();
    if (threadIdx.x == 0) group_signal_all(flags, kFlagCounts, g, G, epoch);
}

// Kernels that write into peer windows end with this: every thread fences its
// own stores at system scope, the block's last thread counts the block, and
// the grid's last block signals every GPU (the counter is reset for the next
// step).  All threads of the grid must reach it.
__device__ __forceinline__ void group_grid_done(uint32_t *done, uint64_t *const *flags, int kind,
                                                int g, int G, uint64_t epoch) {
    __threadfence_system();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t prev = atomicAdd(done, 1u);
        if (prev == gridDim.x - 1) {
            *done = 0u;
            group_signal_all(flags, kind, g, G, epoch);
        }
    }
}

}  // namespace ep
