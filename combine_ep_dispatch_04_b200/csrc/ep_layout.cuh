// ep_layout.cuh -- routing layout and deterministic slot assignment.
//
// What it computes ("Low-Latency Mode API", low_latency_dispatch: topk_idx
// with -1 = no expert, recv_count per expert; the receive slots of an expert
// are ordered by (source rank, token), k breaking ties):
//   token_slot[n,k] = #{ valid entries (n',k') before (n,k) in (n, k) order
//                        with the same expert }.
//
// Design.  The N*K entries are cut into chunks of whole tokens of ONE source
// rank (chunk c = rank r, tokens [j*TC, j*TC+TC)).  Three launches, no
// inter-block waiting:
//   count  -- one block per chunk: per-expert and per-destination-rank
//             histograms in shared memory, is_token_in_rank rows, bad-index
//             flag.  Histograms go to the workspace transposed, [E][C].
//   scan   -- one block per expert: exclusive scan over chunks gives each
//             chunk's first slot; the total is recv_count, rank-segment
//             differences are tokens_per_expert.  One block per destination
//             rank sums tokens_per_rank.
//   assign -- one block per chunk: each warp owns a contiguous run of the
//             chunk's entries; warps count their run (match-any aggregated),
//             a per-expert scan over warps gives each warp its base, then each
//             warp walks its run again and ranks equal experts inside a step
//             with popc(match & lanemask_lt).  Block 0 also writes
//             expert_offset (packed layout).
// Every count is an integer sum, so the result never depends on timing.
#pragma once

#include "ep_device.cuh"

namespace ep {

struct LayoutArgs {
    int R, T, K, E, M, L;
    int TC, CR, C;  // tokens per chunk, chunks per rank, chunks
    int packed, align;
    int64_t cap;    // padded rows per expert (R*M)
    const int64_t *idx;
    int32_t *tpr, *tpe;
    uint8_t *itr;
    int32_t *slot;
    int64_t *recv_count, *eo, *stats;
    int32_t *ws_hist;  // [E][C]
    int32_t *ws_rk;    // [R][C]
    uint32_t *status;
};

constexpr int kLayoutThreads = 256;
constexpr int kMaxTopk = 16;

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kLayoutThreads) layout_count_kernel(LayoutArgs a) {
    extern __shared__ int sm[];
    int *hist = sm;         // [E]
    int *rk = sm + a.E;     // [R]
    for (int i = threadIdx.x; i < a.E + a.R; i += blockDim.x) sm[i] = 0;
    __syncthreads();

    const int c = blockIdx.x, r = c / a.CR, j = c % a.CR;
    const int t0 = j * a.TC, t1 = min(a.T, t0 + a.TC);
    bool bad = false;
    for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
        const int64_t n = (int64_t)r * a.T + t;
        int ev[kMaxTopk];
#pragma unroll
        for (int k = 0; k < kMaxTopk; k++) {
            ev[k] = -1;
            if (k < a.K) {
                int64_t e = a.idx[n * a.K + k];
                bad |= (e < -1 || e >= a.E);
                if (e >= 0 && e < a.E) {
                    ev[k] = (int)e;
                    atomicAdd(&hist[e], 1);
                }
            }
        }
        // destination ranks: count each rank once per token
#pragma unroll
        for (int k = 0; k < kMaxTopk; k++) {
            if (k < a.K && ev[k] >= 0) {
                const int d = ev[k] / a.L;
                bool first = true;
#pragma unroll
                for (int k2 = 0; k2 < kMaxTopk; k2++)
                    if (k2 < k && ev[k2] >= 0 && ev[k2] / a.L == d) first = false;
                if (first) atomicAdd(&rk[d], 1);
            }
        }
        if (a.itr) {
            uint8_t *row = a.itr + n * a.R;
            for (int d = 0; d < a.R; d++) row[d] = 0;
#pragma unroll
            for (int k = 0; k < kMaxTopk; k++)
                if (k < a.K && ev[k] >= 0) row[ev[k] / a.L] = 1;
        }
    }
    if (bad) atomicOr(a.status, kDevBadIndex);
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) a.ws_hist[(int64_t)e * a.C + c] = hist[e];
    for (int d = threadIdx.x; d < a.R; d += blockDim.x) a.ws_rk[(int64_t)d * a.C + c] = rk[d];
}

// Inclusive block scan of one int per thread (blockDim.x == kLayoutThreads).
__device__ __forceinline__ int block_inclusive_scan(int v, int *warp_sums, int &total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int u = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) warp_sums[w] = v;
    __syncthreads();
    if (w == 0) {
        int s = lane < kLayoutThreads / 32 ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int u = __shfl_up_sync(kFull, s, o);
            if (lane >= o) s += u;
        }
        if (lane < kLayoutThreads / 32) warp_sums[lane] = s;
    }
    __syncthreads();
    if (w > 0) v += warp_sums[w - 1];
    total = warp_sums[kLayoutThreads / 32 - 1];
    __syncthreads();
    return v;
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kLayoutThreads) layout_scan_kernel(LayoutArgs a) {
    __shared__ int warp_sums[kLayoutThreads / 32];
    const int b = blockIdx.x;
    if (b < a.E) {
        const int e = b;
        int32_t *h = a.ws_hist + (int64_t)e * a.C;
        int carry = 0;
        for (int base = 0; base < a.C; base += blockDim.x) {
            const int i = base + threadIdx.x;
            const int v = i < a.C ? h[i] : 0;
            int tot;
            const int incl = block_inclusive_scan(v, warp_sums, tot);
            if (i < a.C) h[i] = carry + incl - v;
            carry += tot;
        }
        if (threadIdx.x == 0) {
            a.recv_count[e] = carry;
            if (a.stats) a.stats[e] += carry;
        }
        __syncthreads();
        if (a.tpe) {
            for (int r = threadIdx.x; r < a.R; r += blockDim.x) {
                int v = 0;
                if (a.CR > 0) {
                    const int lo = h[r * a.CR];
                    const int hi = (r + 1 < a.R) ? h[(r + 1) * a.CR] : carry;
                    v = hi - lo;
                }
                a.tpe[(int64_t)r * a.E + e] = v;
            }
        }
    } else if (a.tpr) {
        const int d = b - a.E;
        for (int r = threadIdx.x; r < a.R; r += blockDim.x) {
            int s = 0;
            for (int j = 0; j < a.CR; j++) s += a.ws_rk[(int64_t)d * a.C + r * a.CR + j];
            a.tpr[(int64_t)r * a.R + d] = s;
        }
    }
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kLayoutThreads) layout_assign_kernel(LayoutArgs a) {
    extern __shared__ int sm[];  // off[W][E]
    __shared__ int warp_sums[kLayoutThreads / 32];
    constexpr int W = kLayoutThreads / 32;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int c = blockIdx.x;

    if (c < a.C) {
        int *off = sm + w * a.E;
        for (int e = lane; e < a.E; e += 32) off[e] = 0;
        __syncwarp();

        const int r = c / a.CR, j = c % a.CR;
        const int t0 = j * a.TC, t1 = min(a.T, t0 + a.TC);
        const int64_t f0 = ((int64_t)r * a.T + t0) * a.K;  // first entry of the chunk
        const int nent = (t1 - t0) * a.K;
        const int per = (nent + W - 1) / W;
        const int f_lo = min(nent, w * per), f_hi = min(nent, f_lo + per);

        // pass A: per-warp counts of its run
        for (int b0 = f_lo; b0 < f_hi; b0 += 32) {
            const int f = b0 + lane;
            int key = -1;
            if (f < f_hi) {
                const int64_t e = a.idx[f0 + f];
                if (e >= 0 && e < a.E) key = (int)e;
            }
            const uint32_t mask = __match_any_sync(kFull, key);
            if (key >= 0 && lane == __ffs(mask) - 1) off[key] += __popc(mask);
        }
        __syncthreads();
        // pass B: warp bases = chunk base + counts of the earlier warps
        for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
            int run = a.ws_hist[(int64_t)e * a.C + c];
#pragma unroll
            for (int w2 = 0; w2 < W; w2++) {
                const int cnt = sm[w2 * a.E + e];
                sm[w2 * a.E + e] = run;
                run += cnt;
            }
        }
        __syncthreads();
        // pass C: ranks inside each 32-entry step, in entry order
        bool over = false;
        for (int b0 = f_lo; b0 < f_hi; b0 += 32) {
            const int f = b0 + lane;
            int key = -1;
            if (f < f_hi) {
                const int64_t e = a.idx[f0 + f];
                if (e >= 0 && e < a.E) key = (int)e;
            }
            const uint32_t mask = __match_any_sync(kFull, key);
            int s = -1;
            if (key >= 0) s = off[key] + __popc(mask & lanemask_lt());
            __syncwarp();
            if (key >= 0 && lane == __ffs(mask) - 1) off[key] += __popc(mask);
            __syncwarp();
            if (f < f_hi) a.slot[f0 + f] = s;
            if (!a.packed && s >= 0 && s >= a.cap) over = true;
        }
        if (over) atomicOr(a.status, kDevCapacity);
    }

    // expert_offset: exclusive scan of recv_count rounded up to `align`
    if (c == 0 && a.eo) {
        __syncthreads();
        int64_t carry = 0;
        for (int base = 0; base < a.E; base += blockDim.x) {
            const int e = base + threadIdx.x;
            int64_t v = 0;
            if (e < a.E) v = (a.recv_count[e] + a.align - 1) / a.align * a.align;
            // rows per expert fit in int: recv_count <= N*K < 2^31
            int tot;
            const int incl = block_inclusive_scan((int)v, warp_sums, tot);
            if (e < a.E) a.eo[e] = carry + incl - v;
            carry += tot;
        }
        if (threadIdx.x == 0) a.eo[a.E] = carry;
    }
}


// ---------------------------------------------------------------------------
// One-block path for small routings (N*K up to a few tens of thousands of
// entries): the three phases above run inside a single block of
// kLayoutSingleThreads threads with __syncthreads between them, so the whole
// layout is one launch.  The entries are cut into one contiguous run per warp
// (the "chunk" is the whole problem and its base is 0); per-source-rank
// counts use warp-aggregated global atomics on outputs this block zeroes
// first.  Same result as the multi-block path, bit for bit.
constexpr int kLayoutSingleThreads = 1024;

__global__ void __launch_bounds__(kLayoutSingleThreads) layout_single_kernel(LayoutArgs a) {
    extern __shared__ int sm[];  // off[W][E]
    __shared__ int warp_sums[32];
    constexpr int W = kLayoutSingleThreads / 32;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t N = (int64_t)a.R * a.T;
    const int nent = (int)(N * a.K);

    for (int i = threadIdx.x; i < W * a.E; i += blockDim.x) sm[i] = 0;
    if (a.tpe) for (int i = threadIdx.x; i < a.R * a.E; i += blockDim.x) a.tpe[i] = 0;
    if (a.tpr) for (int i = threadIdx.x; i < a.R * a.R; i += blockDim.x) a.tpr[i] = 0;
    __syncthreads();

    // per token: is_token_in_rank row, distinct destination ranks, bad indices
    bool bad = false;
    for (int64_t n = threadIdx.x; n < N; n += blockDim.x) {
        const int r = (int)(n / a.T);
        int ev[kMaxTopk];
#pragma unroll
        for (int k = 0; k < kMaxTopk; k++) {
            ev[k] = -1;
            if (k < a.K) {
                const int64_t e = a.idx[n * a.K + k];
                bad |= (e < -1 || e >= a.E);
                if (e >= 0 && e < a.E) ev[k] = (int)e;
            }
        }
#pragma unroll
        for (int k = 0; k < kMaxTopk; k++) {
            if (k < a.K && ev[k] >= 0) {
                const int d = ev[k] / a.L;
                bool first = true;
#pragma unroll
                for (int k2 = 0; k2 < kMaxTopk; k2++)
                    if (k2 < k && ev[k2] >= 0 && ev[k2] / a.L == d) first = false;
                if (first && a.tpr) atomicAdd(&a.tpr[r * a.R + d], 1);
            }
        }
        if (a.itr) {
            uint8_t *row = a.itr + n * a.R;
            for (int d = 0; d < a.R; d++) row[d] = 0;
#pragma unroll
            for (int k = 0; k < kMaxTopk; k++)
                if (k < a.K && ev[k] >= 0) row[ev[k] / a.L] = 1;
        }
    }
    if (bad) atomicOr(a.status, kDevBadIndex);

    // pass A: per-warp counts of its run; per-(source rank, expert) counts
    int *off = sm + w * a.E;
    const int per = (nent + W - 1) / W;
    const int f_lo = min(nent, w * per), f_hi = min(nent, f_lo + per);
    for (int b0 = f_lo; b0 < f_hi; b0 += 32) {
        const int f = b0 + lane;
        int key = -1;
        if (f < f_hi) {
            const int64_t e = a.idx[f];
            if (e >= 0 && e < a.E) key = (int)e;
        }
        uint32_t mask = __match_any_sync(kFull, key);
        if (key >= 0 && lane == __ffs(mask) - 1) off[key] += __popc(mask);
        if (a.tpe) {
            const int rkey = key >= 0 ? (f / a.K / a.T) * a.E + key : -1;
            mask = __match_any_sync(kFull, rkey);
            if (rkey >= 0 && lane == __ffs(mask) - 1) atomicAdd(&a.tpe[rkey], __popc(mask));
        }
    }
    __syncthreads();
    // pass B: per expert, scan over warps; totals are recv_count
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int run = 0;
        for (int w2 = 0; w2 < W; w2++) {
            const int cnt = sm[w2 * a.E + e];
            sm[w2 * a.E + e] = run;
            run += cnt;
        }
        a.recv_count[e] = run;
        if (a.stats) a.stats[e] += run;
    }
    __syncthreads();
    // pass C: stable ranks
    bool over = false;
    for (int b0 = f_lo; b0 < f_hi; b0 += 32) {
        const int f = b0 + lane;
        int key = -1;
        if (f < f_hi) {
            const int64_t e = a.idx[f];
            if (e >= 0 && e < a.E) key = (int)e;
        }
        const uint32_t mask = __match_any_sync(kFull, key);
        int s = -1;
        if (key >= 0) s = off[key] + __popc(mask & lanemask_lt());
        __syncwarp();
        if (key >= 0 && lane == __ffs(mask) - 1) off[key] += __popc(mask);
        __syncwarp();
        if (f < f_hi) a.slot[f] = s;
        if (!a.packed && s >= 0 && s >= a.cap) over = true;
    }
    if (over) atomicOr(a.status, kDevCapacity);

    // expert_offset (recv_count was written by this block before the barrier)
    if (a.eo) {
        __syncthreads();
        int carry = 0;
        for (int base = 0; base < a.E; base += blockDim.x) {
            const int e = base + threadIdx.x;
            const int v = e < a.E ? (int)((a.recv_count[e] + a.align - 1) / a.align * a.align) : 0;
            int x = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(kFull, x, o);
                if (lane >= o) x += u;
            }
            if (lane == 31) warp_sums[w] = x;
            __syncthreads();
            if (w == 0) {
                int t = warp_sums[lane];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int u = __shfl_up_sync(kFull, t, o);
                    if (lane >= o) t += u;
                }
                warp_sums[lane] = t;
            }
            __syncthreads();
            const int incl = x + (w > 0 ? warp_sums[w - 1] : 0);
            if (e < a.E) a.eo[e] = carry + incl - v;
            carry += warp_sums[W - 1];
            __syncthreads();
        }
        if (threadIdx.x == 0) a.eo[a.E] = carry;
    }
}

}  // namespace ep
