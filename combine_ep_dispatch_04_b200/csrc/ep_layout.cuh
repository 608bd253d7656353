// ep_layout.cuh -- routing layout and deterministic slot assignment.
//
// What it computes ("Low-Latency Mode API", low_latency_dispatch: topk_idx
// with -1 = no expert, recv_count per expert; the receive slots of an expert
// are ordered by (source rank, token), k breaking ties):
//   token_slot[n,k] = #{ valid entries (n',k') before (n,k) in (n, k) order
//                        with the same expert }.
//
// Design.  Every block first stages the routing entries it owns into shared
// memory with one coalesced load (invalid and out-of-range values become -1
// there), so every later pass runs from shared memory.  Two paths:
//
//   one block (small routings, one launch): warps own chunks of whole tokens
//   of one source rank; per-chunk counts, a per-expert scan over chunks, then
//   a ranking pass in entry order (see layout_single_kernel).
//
//   three launches, no inter-block waiting (large routings): the N*K entries
//   are cut into chunks of whole tokens of ONE source rank.
//     count  -- one block per chunk: per-expert and per-destination-rank
//               histograms, is_token_in_rank rows, bad-index flag; histograms
//               go to the workspace transposed, [E][C].
//     scan   -- one block per expert: exclusive scan over chunks gives each
//               chunk's first slot; the total is recv_count and rank-segment
//               differences are tokens_per_expert.  One block per destination
//               rank sums tokens_per_rank.
//     assign -- one block per chunk: warps count their run of entries, a scan
//               over warps gives each warp its base, and each warp ranks its
//               run in entry order.  Block 0 also writes expert_offset.
//
// Ranking inside a 32-entry step uses warp_stable_rank (an order-free OR of
// lane bits into a per-warp word per expert), and every count is an integer
// sum of order-free atomics, so the result never depends on thread timing.
#pragma once

#include <cooperative_groups.h>

#include "ep_device.cuh"

namespace ep {

struct LayoutArgs {
    int R, T, K, E, M, L;
    int TC, CR, C;  // tokens per chunk, chunks per rank, chunks
    int packed, align;
    int64_t cap;    // padded rows per expert (R*M)
    TopkIdx idx;
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

// ---- shared helpers ------------------------------------------------------------

// keys[i] = expert of entry f0+i, or -1 when masked or out of range; returns
// true if a value outside [-1, E) was seen.  Coalesced loads, 8 in flight per
// thread.
__device__ __forceinline__ bool stage_keys(TopkIdx idx, int64_t f0, int nent, int E,
                                           int *keys) {
    constexpr int U = 8;
    bool bad = false;
    for (int base = threadIdx.x; base < nent; base += U * blockDim.x) {
        int64_t v[U];
#pragma unroll
        for (int u = 0; u < U; u++) {
            const int i = base + u * blockDim.x;
            v[u] = i < nent ? idx[f0 + i] : -1;
        }
#pragma unroll
        for (int u = 0; u < U; u++) {
            const int i = base + u * blockDim.x;
            if (i < nent) {
                bad |= (v[u] < -1 || v[u] >= E);
                keys[i] = (v[u] >= 0 && v[u] < E) ? (int)v[u] : -1;
            }
        }
    }
    return bad;
}

// One token's destination ranks: writes its is_token_in_rank row (if any)
// and adds 1 to rk[d] for each distinct destination rank d (if rk).
__device__ __forceinline__ void token_ranks(const int *keys, int K, int L, int R, uint8_t *row,
                                            int *rk) {
    if (R <= 64) {
        uint64_t mask = 0;
        for (int k = 0; k < K; k++)
            if (keys[k] >= 0) mask |= 1ull << (keys[k] / L);
        if (rk) {
            for (uint64_t m = mask; m; m &= m - 1) atomicAdd(&rk[__ffsll((long long)m) - 1], 1);
        }
        if (row) {
            if ((R & 3) == 0 && (reinterpret_cast<uintptr_t>(row) & 3) == 0) {
                for (int d = 0; d < R; d += 4) {
                    const uint32_t b = (uint32_t)(mask >> d);
                    reinterpret_cast<uint32_t *>(row)[d >> 2] =
                        (b & 1u) | ((b >> 1) & 1u) << 8 | ((b >> 2) & 1u) << 16 | ((b >> 3) & 1u) << 24;
                }
            } else {
                for (int d = 0; d < R; d++) row[d] = (uint8_t)((mask >> d) & 1u);
            }
        }
        return;
    }
    for (int k = 0; k < K; k++) {
        if (keys[k] < 0) continue;
        const int d = keys[k] / L;
        bool first = true;
        for (int k2 = 0; k2 < k; k2++)
            if (keys[k2] >= 0 && keys[k2] / L == d) first = false;
        if (first && rk) atomicAdd(&rk[d], 1);
    }
    if (row) {
        for (int d = 0; d < R; d++) row[d] = 0;
        for (int k = 0; k < K; k++)
            if (keys[k] >= 0) row[keys[k] / L] = 1;
    }
}

// Stable rank of each lane's key among the lanes of its warp holding the same
// key, without timing dependence: every lane ORs its bit into a per-warp word
// for its key (OR is order-free), then reads the word back.  Returns the
// number of lower lanes with the same key; *count gets the group size.  Key
// -1 means "no entry".  `msk` (one word per key, zero on entry) is zero again
// on return.
__device__ __forceinline__ int warp_stable_rank(int key, uint32_t *msk, int lane, int *count) {
    if (key >= 0) atomicOr(&msk[key], 1u << lane);
    __syncwarp();
    const uint32_t m = key >= 0 ? msk[key] : 0u;
    __syncwarp();
    const int rank = __popc(m & lanemask_lt());
    if (key >= 0 && rank == 0) msk[key] = 0u;
    __syncwarp();
    *count = __popc(m);
    return rank;
}

// Walks entries [f_lo, f_hi) of `keys` (one warp, 32 a step, in order) and
// writes slot[f0 + f] = off[key] + rank, advancing off.  Returns true when a
// padded-layout slot reached the capacity.
__device__ __forceinline__ bool rank_run(const int *keys, int f_lo, int f_hi, int *off,
                                         uint32_t *msk, int lane, int32_t *slot, int64_t f0,
                                         bool padded, int64_t cap) {
    bool over = false;
    for (int b0 = f_lo; b0 < f_hi; b0 += 32) {
        const int f = b0 + lane;
        const int key = f < f_hi ? keys[f] : -1;
        int cnt;
        const int rank = warp_stable_rank(key, msk, lane, &cnt);
        const int sl = key >= 0 ? off[key] + rank : -1;
        __syncwarp();
        if (key >= 0 && rank == 0) off[key] += cnt;
        __syncwarp();
        if (f < f_hi) slot[f0 + f] = sl;
        if (padded && sl >= cap) over = true;
    }
    return over;
}

// Inclusive scan of one int per thread over a block of W warps.
__device__ __forceinline__ int block_inclusive_scan(int v, int *warp_sums, int W, int &total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) warp_sums[w] = v;
    __syncthreads();
    if (w == 0) {
        int s = lane < W ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(kFull, s, o);
            if (lane >= o) s += u;
        }
        if (lane < W) warp_sums[lane] = s;
    }
    __syncthreads();
    if (w > 0) v += warp_sums[w - 1];
    total = warp_sums[W - 1];
    __syncthreads();
    return v;
}

// expert_offset[e] = exclusive scan of recv_count rounded up to align; the
// block's recv_count writes must be visible (a barrier before the call).
__device__ __forceinline__ void write_expert_offset(const LayoutArgs &a, int *warp_sums) {
    const int W = blockDim.x >> 5;
    int carry = 0;
    for (int base = 0; base < a.E; base += blockDim.x) {
        const int e = base + threadIdx.x;
        // rows per expert fit in int: the row capacity is validated below 2^31
        const int v = e < a.E ? (int)((a.recv_count[e] + a.align - 1) / a.align * a.align) : 0;
        int tot;
        const int incl = block_inclusive_scan(v, warp_sums, W, tot);
        if (e < a.E) a.eo[e] = carry + incl - v;
        carry += tot;
    }
    if (threadIdx.x == 0) a.eo[a.E] = carry;
}

// ---- multi-block path ------------------------------------------------------------

__global__ void __launch_bounds__(kLayoutThreads) layout_count_kernel(LayoutArgs a) {
    pdl_enter();
    extern __shared__ int sm[];
    const int c = blockIdx.x, r = c / a.CR, j = c % a.CR;
    const int t0 = j * a.TC, t1 = min(a.T, t0 + a.TC);
    const int nent = (t1 - t0) * a.K;
    int *keys = sm;                 // [TC*K]
    int *hist = sm + a.TC * a.K;    // [E]
    int *rk = hist + a.E;           // [R]
    for (int i = threadIdx.x; i < a.E + a.R; i += blockDim.x) hist[i] = 0;
    const bool bad = stage_keys(a.idx, ((int64_t)r * a.T + t0) * a.K, nent, a.E, keys);
    if (bad) atomicOr(a.status, kDevBadIndex);
    __syncthreads();

    for (int t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
        const int *tk = keys + (t - t0) * a.K;
        for (int k = 0; k < a.K; k++)
            if (tk[k] >= 0) atomicAdd(&hist[tk[k]], 1);
        token_ranks(tk, a.K, a.L, a.R, a.itr ? a.itr + ((int64_t)r * a.T + t) * a.R : nullptr, rk);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) a.ws_hist[(int64_t)e * a.C + c] = hist[e];
    for (int d = threadIdx.x; d < a.R; d += blockDim.x) a.ws_rk[(int64_t)d * a.C + c] = rk[d];
}

__global__ void __launch_bounds__(kLayoutThreads) layout_scan_kernel(LayoutArgs a) {
    pdl_enter();
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
            const int incl = block_inclusive_scan(v, warp_sums, kLayoutThreads / 32, tot);
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

__global__ void __launch_bounds__(kLayoutThreads) layout_assign_kernel(LayoutArgs a) {
    pdl_enter();
    extern __shared__ int sm[];
    __shared__ int warp_sums[kLayoutThreads / 32];
    constexpr int W = kLayoutThreads / 32;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int c = blockIdx.x;

    if (c < a.C) {
        const int r = c / a.CR, j = c % a.CR;
        const int t0 = j * a.TC, t1 = min(a.T, t0 + a.TC);
        const int64_t f0 = ((int64_t)r * a.T + t0) * a.K;  // first entry of the chunk
        const int nent = (t1 - t0) * a.K;
        int *keys = sm;                                              // [TC*K]
        int *off = sm + a.TC * a.K;                                  // [W][E]
        uint32_t *msk = reinterpret_cast<uint32_t *>(off + W * a.E); // [W][E]
        for (int i = threadIdx.x; i < 2 * W * a.E; i += blockDim.x) off[i] = 0;
        stage_keys(a.idx, f0, nent, a.E, keys);
        __syncthreads();

        const int per = (nent + W - 1) / W;
        const int f_lo = min(nent, w * per), f_hi = min(nent, f_lo + per);
        int *woff = off + w * a.E;
        // pass A: per-warp counts (order-free)
        for (int f = f_lo + lane; f < f_hi; f += 32)
            if (keys[f] >= 0) atomicAdd(&woff[keys[f]], 1);
        __syncthreads();
        // pass B: warp bases = chunk base + counts of the earlier warps
        for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
            int run = a.ws_hist[(int64_t)e * a.C + c];
#pragma unroll
            for (int w2 = 0; w2 < W; w2++) {
                const int cnt = off[w2 * a.E + e];
                off[w2 * a.E + e] = run;
                run += cnt;
            }
        }
        __syncthreads();
        // pass C: stable ranks in entry order
        if (rank_run(keys, f_lo, f_hi, woff, msk + w * a.E, lane, a.slot, f0, !a.packed, a.cap))
            atomicOr(a.status, kDevCapacity);
    }
    if (c == 0 && a.eo) {
        __syncthreads();
        write_expert_offset(a, warp_sums);
    }
}

// ---- one-block path ----------------------------------------------------------------
// The N tokens are cut into C chunks of whole tokens of one source rank
// (CR per rank); warp w owns chunks w, w+W, ...  Phase 1 (each warp, its
// chunks, a lane per token): per-chunk expert counts, is_token_in_rank rows,
// tokens_per_rank from ballots over the destination-rank masks.  Phase 2 (a
// thread per expert): exclusive scan over chunks gives every chunk's first
// slot and recv_count; tokens_per_expert[r][e] is the difference of the first
// slots of rank r+1 and rank r.  Phase 3 (each warp, its chunks in order):
// stable ranks, 32 entries a step.  The block is bound by instruction issue on
// its one SM, so the passes are written for few instructions: a shared table
// gives each expert's rank (no integer division), and zeroing uses 16-byte
// stores.  Same result as the multi-block path, bit for bit.
__global__ void __launch_bounds__(1024, 1) layout_single_kernel(LayoutArgs a) {
    pdl_enter();
    extern __shared__ __align__(16) int sm[];
    __shared__ int warp_sums[32];
    const int W = blockDim.x >> 5;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int E = a.E, R = a.R, K = a.K, T = a.T, C = a.C, CR = a.CR, TC = a.TC;
    const int64_t N = (int64_t)R * T;
    const int nent = (int)(N * K);
    // layout: [counters off: C*E][masks: W*E][rank_of: E][keys: N*K], each part
    // starting on a 16-byte boundary (the host sizes the block accordingly)
    const int off_n = (C * E + 3) & ~3, msk_n = (W * E + 3) & ~3, rk_n = (E + 3) & ~3;
    int *off = sm;
    uint32_t *msk = reinterpret_cast<uint32_t *>(sm + off_n);
    int *rank_of = sm + off_n + msk_n;
    int *keys = rank_of + rk_n;

    {
        int4 *z = reinterpret_cast<int4 *>(sm);
        const int n4 = (off_n + msk_n) >> 2;
        for (int i = threadIdx.x; i < n4; i += blockDim.x) z[i] = make_int4(0, 0, 0, 0);
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) rank_of[e] = e / a.L;
    if (a.tpr) for (int i = threadIdx.x; i < R * R; i += blockDim.x) a.tpr[i] = 0;
    if (stage_keys(a.idx, 0, nent, E, keys)) atomicOr(a.status, kDevBadIndex);
    __syncthreads();

    // phase 1
    for (int c = w; c < C; c += W) {
        const int r = c / CR, j = c - r * CR;
        const int t0 = j * TC, t1 = min(T, t0 + TC);
        int *coff = off + c * E;
        int rc0 = 0, rc1 = 0;  // this lane's share of tokens_per_rank[r][lane], [r][lane+32]
        for (int tb = t0; tb < t1; tb += 32) {
            const int t = tb + lane;
            uint64_t mask = 0;
            if (t < t1) {
                const int n = r * T + t;
                const int *tk = keys + n * K;
                for (int k = 0; k < K; k++) {
                    const int e = tk[k];
                    if (e >= 0) {
                        atomicAdd(&coff[e], 1);
                        mask |= 1ull << (rank_of[e] & 63);
                    }
                }
                if (R > 64) {
                    token_ranks(tk, K, a.L, R, a.itr ? a.itr + (int64_t)n * R : nullptr,
                                a.tpr ? a.tpr + (int64_t)r * R : nullptr);
                } else if (a.itr) {
                    uint8_t *row = a.itr + (int64_t)n * R;
                    if ((R & 3) == 0) {
                        for (int d = 0; d < R; d += 4) {
                            const uint32_t bits = (uint32_t)(mask >> d);
                            reinterpret_cast<uint32_t *>(row)[d >> 2] =
                                (bits & 1u) | ((bits >> 1) & 1u) << 8 | ((bits >> 2) & 1u) << 16 |
                                ((bits >> 3) & 1u) << 24;
                        }
                    } else {
                        for (int d = 0; d < R; d++) row[d] = (uint8_t)((mask >> d) & 1u);
                    }
                }
            }
            if (R <= 64) {
                for (int d = 0; d < R; d++) {
                    const int cnt = __popc(__ballot_sync(kFull, (mask >> d) & 1ull));
                    if (d == lane) rc0 += cnt;
                    if (d == lane + 32) rc1 += cnt;
                }
            }
        }
        if (R <= 64 && a.tpr) {
            if (lane < R && rc0) atomicAdd(&a.tpr[(int64_t)r * R + lane], rc0);
            if (lane + 32 < R && rc1) atomicAdd(&a.tpr[(int64_t)r * R + lane + 32], rc1);
        }
    }
    __syncthreads();

    // phase 2: per expert, exclusive scan over chunks
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        int c = 0;
        for (; c + 4 <= C; c += 4) {
            const int v0 = off[c * E + e], v1 = off[(c + 1) * E + e];
            const int v2 = off[(c + 2) * E + e], v3 = off[(c + 3) * E + e];
            off[c * E + e] = run;
            off[(c + 1) * E + e] = run + v0;
            off[(c + 2) * E + e] = run + v0 + v1;
            off[(c + 3) * E + e] = run + v0 + v1 + v2;
            run += v0 + v1 + v2 + v3;
        }
        for (; c < C; c++) {
            const int v = off[c * E + e];
            off[c * E + e] = run;
            run += v;
        }
        a.recv_count[e] = run;
        if (a.stats) a.stats[e] += run;
        if (a.tpe) {
            for (int r = 0; r < R; r++) {
                int v = 0;
                if (CR > 0) {  // no chunks when T == 0
                    const int lo = off[r * CR * E + e];
                    const int hi = r + 1 < R ? off[(r + 1) * CR * E + e] : run;
                    v = hi - lo;
                }
                a.tpe[(int64_t)r * E + e] = v;
            }
        }
    }
    __syncthreads();

    // phase 3: stable ranks, each warp over its chunks in order
    uint32_t *wmsk = msk + w * E;
    const uint32_t lt = lanemask_lt();
    bool over = false;
    for (int c = w; c < C; c += W) {
        const int r = c / CR, j = c - r * CR;
        const int t0 = j * TC, t1 = min(T, t0 + TC);
        const int f_lo = (r * T + t0) * K, f_hi = (r * T + t1) * K;
        int *coff = off + c * E;
        for (int b0 = f_lo; b0 < f_hi; b0 += 32) {
            const int f = b0 + lane;
            const int key = f < f_hi ? keys[f] : -1;
            if (key >= 0) atomicOr(&wmsk[key], 1u << lane);
            __syncwarp();
            uint32_t m = 0;
            int base = 0;
            if (key >= 0) {
                m = wmsk[key];
                base = coff[key];
            }
            __syncwarp();
            const int rank = __popc(m & lt);
            if (key >= 0 && rank == 0) {  // first holder: advance the base, clear the word
                coff[key] = base + __popc(m);
                wmsk[key] = 0u;
            }
            __syncwarp();
            const int sl = key >= 0 ? base + rank : -1;
            if (f < f_hi) a.slot[f] = sl;
            if (!a.packed && sl >= a.cap) over = true;
        }
    }
    if (over) atomicOr(a.status, kDevCapacity);
    if (a.eo) {
        __syncthreads();
        write_expert_offset(a, warp_sums);
    }
}

// ---- cluster path -------------------------------------------------------------------
// One thread-block cluster of Q blocks (Q <= 16, all co-scheduled, hardware
// cluster barriers) spreads the one-block design over Q SMs.  The N tokens
// are cut into C chunks of whole tokens of one source rank; block q owns the
// contiguous chunks [q*CPQ, (q+1)*CPQ) and warp w of a block owns its local
// chunks w, w+W, ...
//   0  every block stages its chunks' entries; block 0 zeroes the global
//      per-rank counters.                                       cluster barrier
//   1  per-chunk expert counts, is_token_in_rank rows, tokens_per_rank
//      (ballots, global atomics).
//   2a per expert: local exclusive scan over the block's chunks, the block
//      total tot[e], and each rank's share added to tokens_per_expert.
//                                                               cluster barrier
//   2b per expert: the block's base is the sum of tot[e] of the lower blocks,
//      read from their shared memory; block 0 sums all blocks for recv_count,
//      the stats and expert_offset.                              cluster barrier
//      (after it no block reads another block's shared memory)
//   3  stable ranks of each chunk, 32 entries a step.
// Counts are order-free integer sums, so the result is the one of the other
// paths, bit for bit.
struct ClusterPlan {
    int Q, TC, CR, C, CPQ;
};

__global__ void __launch_bounds__(512, 1) layout_cluster_kernel(LayoutArgs a, ClusterPlan cp) {
    pdl_enter();
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ __align__(16) int sm[];
    __shared__ int warp_sums[32];
    const int q = (int)cluster.block_rank();
    const int W = blockDim.x >> 5;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int E = a.E, R = a.R, K = a.K, T = a.T;
    const int TC = cp.TC, CR = cp.CR, C = cp.C, CPQ = cp.CPQ;
    const int c_lo = min(C, q * CPQ), c_hi = min(C, c_lo + CPQ), nloc = c_hi - c_lo;
    // entries of this block: chunks are contiguous in entry order
    auto chunk_first_entry = [&](int c) {
        const int r = c / CR, j = c - r * CR;
        return (r * T + min(T, j * TC)) * K;
    };
    const int f0 = nloc > 0 ? chunk_first_entry(c_lo) : 0;
    const int f1 = nloc > 0 ? (c_hi % CR == 0 ? (c_hi / CR) * T * K : chunk_first_entry(c_hi)) : 0;
    const int nent = f1 - f0;

    // shared memory: [off: CPQ*E][tot: E][msk: W*E][rank_of: E][keys: nent]
    const int off_n = (CPQ * E + 3) & ~3, e4 = (E + 3) & ~3, msk_n = (W * E + 3) & ~3;
    int *off = sm;
    int *tot = sm + off_n;
    uint32_t *msk = reinterpret_cast<uint32_t *>(sm + off_n + e4);
    int *rank_of = sm + off_n + e4 + msk_n;
    int *keys = rank_of + e4;

    {
        int4 *z = reinterpret_cast<int4 *>(sm);
        const int n4 = (off_n + e4 + msk_n) >> 2;
        for (int i = threadIdx.x; i < n4; i += blockDim.x) z[i] = make_int4(0, 0, 0, 0);
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) rank_of[e] = e / a.L;
    if (q == 0) {
        if (a.tpr) for (int i = threadIdx.x; i < R * R; i += blockDim.x) a.tpr[i] = 0;
        if (a.tpe) for (int i = threadIdx.x; i < R * E; i += blockDim.x) a.tpe[i] = 0;
    }
    if (stage_keys(a.idx, f0, nent, E, keys)) atomicOr(a.status, kDevBadIndex);
    cluster.sync();

    // phase 1
    for (int lc = w; lc < nloc; lc += W) {
        const int c = c_lo + lc;
        const int r = c / CR, j = c - r * CR;
        const int t0 = j * TC, t1 = min(T, t0 + TC);
        int *coff = off + lc * E;
        int rc0 = 0, rc1 = 0;
        for (int tb = t0; tb < t1; tb += 32) {
            const int t = tb + lane;
            uint64_t mask = 0;
            if (t < t1) {
                const int n = r * T + t;
                const int *tk = keys + (n * K - f0);
                for (int k = 0; k < K; k++) {
                    const int e = tk[k];
                    if (e >= 0) {
                        atomicAdd(&coff[e], 1);
                        mask |= 1ull << (rank_of[e] & 63);
                    }
                }
                if (R > 64) {
                    token_ranks(tk, K, a.L, R, a.itr ? a.itr + (int64_t)n * R : nullptr,
                                a.tpr ? a.tpr + (int64_t)r * R : nullptr);
                } else if (a.itr) {
                    uint8_t *row = a.itr + (int64_t)n * R;
                    if ((R & 3) == 0) {
                        for (int d = 0; d < R; d += 4) {
                            const uint32_t bits = (uint32_t)(mask >> d);
                            reinterpret_cast<uint32_t *>(row)[d >> 2] =
                                (bits & 1u) | ((bits >> 1) & 1u) << 8 | ((bits >> 2) & 1u) << 16 |
                                ((bits >> 3) & 1u) << 24;
                        }
                    } else {
                        for (int d = 0; d < R; d++) row[d] = (uint8_t)((mask >> d) & 1u);
                    }
                }
            }
            if (R <= 64) {
                for (int d = 0; d < R; d++) {
                    const int cnt = __popc(__ballot_sync(kFull, (mask >> d) & 1ull));
                    if (d == lane) rc0 += cnt;
                    if (d == lane + 32) rc1 += cnt;
                }
            }
        }
        if (R <= 64 && a.tpr) {
            if (lane < R && rc0) atomicAdd(&a.tpr[(int64_t)r * R + lane], rc0);
            if (lane + 32 < R && rc1) atomicAdd(&a.tpr[(int64_t)r * R + lane + 32], rc1);
        }
    }
    __syncthreads();

    // phase 2a: local scan over the block's chunks; per-rank shares of tpe
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0, rank_run = 0;
        int cur_r = nloc > 0 ? c_lo / CR : 0;
        for (int lc = 0; lc < nloc; lc++) {
            const int r = (c_lo + lc) / CR;
            if (r != cur_r) {
                if (a.tpe && rank_run) atomicAdd(&a.tpe[(int64_t)cur_r * E + e], rank_run);
                cur_r = r;
                rank_run = 0;
            }
            const int v = off[lc * E + e];
            off[lc * E + e] = run;
            run += v;
            rank_run += v;
        }
        if (a.tpe && rank_run) atomicAdd(&a.tpe[(int64_t)cur_r * E + e], rank_run);
        tot[e] = run;
    }
    cluster.sync();

    // phase 2b: bases from the lower blocks' totals (distributed shared memory);
    // the remote loads of all blocks are issued together, then summed
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int upto = q == 0 ? cp.Q : q;  // block 0 also sums every block
        int v[16];
#pragma unroll
        for (int q2 = 0; q2 < 16; q2++)
            v[q2] = q2 < upto ? cluster.map_shared_rank(tot, q2)[e] : 0;
        int base = 0, all = 0;
#pragma unroll
        for (int q2 = 0; q2 < 16; q2++) {
            base += q2 < q ? v[q2] : 0;
            all += v[q2];
        }
        for (int lc = 0; lc < nloc; lc++) off[lc * E + e] += base;
        if (q == 0) {
            a.recv_count[e] = all;
            if (a.stats) a.stats[e] += all;
        }
    }
    cluster.sync();  // no shared-memory reads across blocks after this point

    // phase 3: stable ranks, each warp over its local chunks in order
    uint32_t *wmsk = msk + w * E;
    const uint32_t lt = lanemask_lt();
    bool over = false;
    for (int lc = w; lc < nloc; lc += W) {
        const int c = c_lo + lc;
        const int r = c / CR, j = c - r * CR;
        const int t0 = j * TC, t1 = min(T, t0 + TC);
        const int g_lo = (r * T + t0) * K, g_hi = (r * T + t1) * K;  // global entry range
        int *coff = off + lc * E;
        for (int b0 = g_lo; b0 < g_hi; b0 += 32) {
            const int f = b0 + lane;
            const int key = f < g_hi ? keys[f - f0] : -1;
            if (key >= 0) atomicOr(&wmsk[key], 1u << lane);
            __syncwarp();
            uint32_t m = 0;
            int base = 0;
            if (key >= 0) {
                m = wmsk[key];
                base = coff[key];
            }
            __syncwarp();
            const int rank = __popc(m & lt);
            if (key >= 0 && rank == 0) {
                coff[key] = base + __popc(m);
                wmsk[key] = 0u;
            }
            __syncwarp();
            const int sl = key >= 0 ? base + rank : -1;
            if (f < g_hi) a.slot[f] = sl;
            if (!a.packed && sl >= a.cap) over = true;
        }
    }
    if (over) atomicOr(a.status, kDevCapacity);
    if (q == 0 && a.eo) {
        __syncthreads();
        write_expert_offset(a, warp_sums);
    }
}

}  // namespace ep
