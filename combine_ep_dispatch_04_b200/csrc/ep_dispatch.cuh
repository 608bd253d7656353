// ep_dispatch.cuh -- fused quantise + scatter (dispatch) and the reverse
// dispatch of the combine backward.
//
// Dispatch ("Low-Latency Mode API", low_latency_dispatch Return Values;
// "DeepEP FP8 Dispatch and Combine Operations", The Dispatch Stage;
// "EP dispatch with unfused MXFP8 quantization", Changes): every source token
// is read once, quantised once, and its row is stored to each of its <= K
// receive rows (data region) with its scales (scale region), src_info and the
// optional weight.
//
// Work split: a group of TPT threads owns one token (block_threads(TPT) / TPT
// tokens per block).  The row
// is cut into 16-element granules (32 bytes of bf16 input); thread lt of the
// group holds granules g = i*TPT + lt, i < GMAX, as two 16-byte loads.  A
// quantisation block of 128 elements is 8 consecutive threads and one of 32
// elements is 2, so block maxima are warp shuffles; the per-row int8 maximum
// crosses warps through shared memory.  Codes are computed once, then the
// group stores them to every destination row with 16-byte (8 for e2m1)
// coalesced stores: per warp instruction 512 (256) contiguous bytes.
#pragma once

#include "ep_device.cuh"
#include "ep_group.cuh"

namespace ep {

enum { Q_BF16 = 0, Q_E4M3_B128 = 1, Q_INT8 = 2, Q_MXFP8 = 3, Q_MXFP4 = 4 };

struct DispatchArgs {
    int64_t N;
    int T, K, E, M, H;
    int first_rank;          // logical rank of this GPU's first token (0 on one GPU)
    int packed;
    int64_t cap, rows;       // padded rows per expert, buffer row capacity
    int64_t D, S, scale_off; // row data bytes, row scale bytes, scale region offset
    float qmax;              // e4m3_b128 target max
    int sfmt;                // e4m3_b128 scales: 0 qmax/amax, 1 power of two, 2 e8m0 bytes
    int unweighted;          // combine backward only
    int early;               // load and quantise x before waiting for the previous grid
    const uint16_t *x;       // [N][H] bf16 (the gradient g for the backward)
    TopkIdx idx;
    const float *wts;
    const int32_t *slot;
    const int64_t *eo;
    uint8_t *out;            // recv_buf / grad_buf
    int32_t *src_info;
    float *recv_w;
    uint32_t *status;
    // expert parallelism over GPUs (ep_group.cuh); peer_out == nullptr on one GPU
    uint8_t *const *peer_out;  // [G] window bases (recv_buf / grad_buf of every GPU)
    int32_t *const *peer_src;  // [G] source-info windows (dispatch)
    float *const *peer_w;      // [G] weight windows (nullable)
    int64_t win_rows;          // rows of one window
    int experts_per_gpu;       // an expert's owner is e / experts_per_gpu
    uint32_t *done;            // this GPU's block counter for the end-of-grid signal
    uint64_t *const *flags;    // [G] flag words of every GPU
    int flag_kind, grp_g, grp_G;
    uint64_t epoch;
};

// Data and scale destinations of expert e's (virtual) row: in this GPU's
// buffer, or in the window of the GPU that owns e.  False (and the capacity
// bit) when the row lies past the end of the owner's window.
__device__ __forceinline__ bool row_dest(const DispatchArgs &a, int64_t e, int64_t row,
                                         uint8_t *&dst, uint8_t *&sdst, int32_t *&src,
                                         float *&rw, int64_t &lrow, uint32_t &flags) {
    uint8_t *base = a.out;
    src = a.src_info;
    rw = a.recv_w;
    lrow = row;
    if (a.peer_out) {
        const int o = (int)(e / a.experts_per_gpu);
        lrow = row - (int64_t)o * a.win_rows;
        if (lrow < 0 || lrow >= a.win_rows) {
            flags |= kDevCapacity;
            return false;
        }
        base = a.peer_out[o];
        src = a.peer_src ? a.peer_src[o] : nullptr;
        rw = a.peer_w ? a.peer_w[o] : nullptr;
    }
    dst = base + lrow * a.D;
    sdst = base + a.scale_off + lrow * a.S;
    return true;
}

// Row of entry (expert e, slot s) in the receive layout, or -1 (masked, or no row).
__device__ __forceinline__ int64_t row_of_entry(const DispatchArgs &a, int64_t e, int32_t s,
                                                uint32_t &flags) {
    if (e < -1 || e >= a.E) flags |= kDevBadIndex;
    if (e < 0 || e >= a.E) return -1;
    if (s < 0) return -1;
    int64_t row;
    if (!a.packed) {
        if (s >= a.cap) { flags |= kDevCapacity; return -1; }
        row = e * a.cap + s;
    } else {
        row = a.eo[e] + s;
        if (row >= a.eo[e + 1] || row >= a.rows) { flags |= kDevCapacity; return -1; }
    }
    return row;
}

template <int MODE>
struct GranOut;  // bytes a 16-element granule becomes
template <> struct GranOut<Q_BF16> { static constexpr int bytes = 32; };
template <> struct GranOut<Q_E4M3_B128> { static constexpr int bytes = 16; };
template <> struct GranOut<Q_INT8> { static constexpr int bytes = 16; };
template <> struct GranOut<Q_MXFP8> { static constexpr int bytes = 16; };
template <> struct GranOut<Q_MXFP4> { static constexpr int bytes = 8; };

// Largest magnitude of 16 bf16 values, NaNs left out, as a bf16 pair word
// (out of line: taken only for a granule with a NaN).
__device__ __noinline__ uint32_t nan_free_absmax16(const uint16_t *p) {
    uint32_t m = 0u;
    for (int q = 0; q < 8; q++) m = __vmaxu2(m, bf2_drop_nan(reinterpret_cast<const uint32_t *>(p)[q]));
    return m;
}

__device__ __forceinline__ uint32_t q_i8(float v, float s) {
    const float p = __fmul_rn(v, s);
    int q = p != p ? 0 : __float2int_rn(p);  // int8 has no NaN: a NaN product is 0
    q = q > 127 ? 127 : (q < -127 ? -127 : q);
    return (uint32_t)q & 0xFFu;
}

// With a.early (only set by ep_dispatch_with_layout, whose previous grid is
// the library's own layout kernel) the token is loaded and quantised before
// the wait for the previous grid: x is not produced by the layout, and the
// layout grid lets this grid launch only after its own wait for all earlier
// work returned.  The slots are read after the wait.
template <int MODE, int TPT, int GMAX>
__device__ __forceinline__ void dispatch_body(const DispatchArgs &a) {
    constexpr int TOKS = block_threads(TPT) / TPT;
    constexpr int WPG = TPT / 32;  // warps per token group
    constexpr int OB = GranOut<MODE>::bytes;
    __shared__ uint8_t *s_dst[TOKS][16];   // each entry's data row and scale row
    __shared__ uint8_t *s_sdst[TOKS][16];
    __shared__ float s_red[TOKS][WPG];

    const int grp = threadIdx.x / TPT, lt = threadIdx.x % TPT;
    const int64_t n = (int64_t)blockIdx.x * TOKS + grp;
    const bool active = n < a.N;
    const bool router = active && lt < a.K;  // thread lt reads entry (n, lt)
    const int ngran = a.H >> 4;

    // The entry's expert, slot and weight are loaded here and used after the
    // quantisation, so their latency overlaps the row loads.  topk_idx and the
    // weights are inputs; the slot comes from the layout and, in early mode,
    // is read only after the wait.
    int64_t r_e = -1;
    int32_t r_s = -1;
    float r_w = 0.0f;
    if (!a.early) pdl_enter();
    if (router) {
        r_e = a.idx[n * a.K + lt];
        if (a.recv_w || a.peer_w) r_w = a.wts[n * a.K + lt];
        if (!a.early) r_s = a.slot[n * a.K + lt];
    }

    // load the token's granules (two 16-byte loads each)
    uint32_t v[GMAX][8];
#pragma unroll
    for (int i = 0; i < GMAX; i++) {
        const int g = i * TPT + lt;
        if (active && g < ngran) {
            const uint16_t *p = a.x + n * a.H + (int64_t)g * 16;
            const uint4 u0 = ld_stream(p), u1 = ld_stream(p + 8);
            v[i][0] = u0.x; v[i][1] = u0.y; v[i][2] = u0.z; v[i][3] = u0.w;
            v[i][4] = u1.x; v[i][5] = u1.y; v[i][6] = u1.z; v[i][7] = u1.w;
        } else {
#pragma unroll
            for (int q = 0; q < 8; q++) v[i][q] = 0u;
        }
    }

    // per-granule block maxima (bf16 magnitudes, exact)
    float gmax[GMAX];
    uint32_t gm[GMAX];
    bool nan = false;
#pragma unroll
    for (int i = 0; i < GMAX; i++) {
        uint32_t m = 0u;
#pragma unroll
        for (int q = 0; q < 8; q++) m = bf2_absmax(m, v[i][q]);
        gm[i] = m;
        nan = nan || bf2_any_nan(m);
    }
    if (nan) {  // a NaN element (rare): the maxima again, NaN halves left out
#pragma unroll
        for (int i = 0; i < GMAX; i++) {
            const int g = i * TPT + lt;
            if (active && g < ngran) gm[i] = nan_free_absmax16(a.x + n * a.H + (int64_t)g * 16);
        }
    }
#pragma unroll
    for (int i = 0; i < GMAX; i++) gmax[i] = bf2_fold(gm[i]);

    // scales
    float rs = 1.0f, rsinv = 1.0f;  // int8: per row
    float bs[GMAX];                 // e4m3_b128: per 128-block multiplier; mx: 2^-X
    float bsinv[GMAX];              // e4m3_b128: stored scale_inv
    uint32_t bx[GMAX];              // mx: e8m0 byte
    if constexpr (MODE == Q_INT8) {
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < GMAX; i++) m = fmaxf(m, gmax[i]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
        if constexpr (WPG > 1) {
            if ((lt & 31) == 0) s_red[grp][lt >> 5] = m;
        }
        __syncthreads();
        if constexpr (WPG > 1) {
#pragma unroll
            for (int q = 0; q < WPG; q++) m = fmaxf(m, s_red[grp][q]);
        }
        if (m != 0.0f) {
            rs = fminf(__fdiv_rn(127.0f, m), FLT_MAX);
            rsinv = __fdiv_rn(m, 127.0f);
        }
    }
    if constexpr (MODE == Q_E4M3_B128) {
#pragma unroll
        for (int i = 0; i < GMAX; i++) {
            float m = gmax[i];
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 2));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 4));
            bs[i] = 1.0f;
            bsinv[i] = 1.0f;
            if (a.sfmt == 0) {
                if (m != 0.0f) {
                    bs[i] = fminf(__fdiv_rn(a.qmax, m), FLT_MAX);
                    bsinv[i] = __fdiv_rn(m, a.qmax);
                }
            } else {  // round_scale: the block's power of two by the MX rule
                const int X = a.qmax == 448.0f ? mx_exponent_fast<448>(m) : mx_exponent(m, a.qmax);
                bs[i] = exp2_neg(X);
                bsinv[i] = exp2_neg(-X);
                bx[i] = (uint32_t)(X + 127);
            }
        }
    }
    if constexpr (MODE == Q_MXFP8 || MODE == Q_MXFP4) {
#pragma unroll
        for (int i = 0; i < GMAX; i++) {
            float m = gmax[i];
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
            const int X = mx_exponent_fast<MODE == Q_MXFP8 ? 448 : 6>(m);
            bs[i] = exp2_neg(X);
            bx[i] = (uint32_t)(X + 127);
        }
    }

    // codes
    uint32_t c[GMAX][OB / 4];
#pragma unroll
    for (int i = 0; i < GMAX; i++) {
        if constexpr (MODE == Q_BF16) {
#pragma unroll
            for (int q = 0; q < 8; q++) c[i][q] = v[i][q];
        } else if constexpr (MODE == Q_INT8) {
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const uint32_t w0 = v[i][2 * q], w1 = v[i][2 * q + 1];
                c[i][q] = q_i8(bf_lo(w0), rs) | (q_i8(bf_hi(w0), rs) << 8) |
                          (q_i8(bf_lo(w1), rs) << 16) | (q_i8(bf_hi(w1), rs) << 24);
            }
        } else if constexpr (MODE == Q_E4M3_B128 || MODE == Q_MXFP8) {
            const float s = bs[i];
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const uint32_t w0 = v[i][2 * q], w1 = v[i][2 * q + 1];
                float p0 = bf_lo(w0), p1 = bf_hi(w0), p2 = bf_lo(w1), p3 = bf_hi(w1);
                mul2(p0, p1, s);
                mul2(p2, p3, s);
                c[i][q] = cvt_e4m3x2(p0, p1) | (cvt_e4m3x2(p2, p3) << 16);
            }
        } else {  // MXFP4: element 2i in the low nibble
            const float s = bs[i];
#pragma unroll
            for (int q = 0; q < 2; q++) {
                uint32_t word = 0u;
#pragma unroll
                for (int h = 0; h < 4; h++) {
                    const uint32_t wv = v[i][4 * q + h];
                    float p0 = bf_lo(wv), p1 = bf_hi(wv);
                    mul2(p0, p1, s);
                    word |= cvt_e2m1x2(p0, p1) << (8 * h);
                }
                c[i][q] = word;
            }
        }
    }

    if (a.early) {
        pdl_enter();
        if (router) r_s = a.slot[n * a.K + lt];
    }
    // destination rows of the token's entries
    if (router) {
        uint32_t flags = 0;
        const int64_t row = row_of_entry(a, r_e, r_s, flags);
        uint8_t *dst = nullptr, *sdst = nullptr;
        int32_t *src;
        float *rw;
        int64_t lrow;
        if (row >= 0 && row_dest(a, r_e, row, dst, sdst, src, rw, lrow, flags)) {
            // source rank and token; a GPU of a group holds ranks first_rank ..
            src[lrow] = (int32_t)((n / a.T + a.first_rank) * a.M + n % a.T);
            if (rw) rw[lrow] = r_w;
        }
        if (flags) atomicOr(a.status, flags);
        s_dst[grp][lt] = dst;
        s_sdst[grp][lt] = sdst;
    }
    __syncthreads();
    if (!active) return;
    // scatter to every destination row
    for (int k = 0; k < a.K; k++) {
        uint8_t *dst = s_dst[grp][k];
        if (!dst) continue;
        uint8_t *sdst = s_sdst[grp][k];
#pragma unroll
        for (int i = 0; i < GMAX; i++) {
            const int g = i * TPT + lt;
            if (g >= ngran) continue;
            uint8_t *p = dst + (int64_t)g * OB;
            if constexpr (OB == 32) {
                st_v4(p, make_uint4(c[i][0], c[i][1], c[i][2], c[i][3]));
                st_v4(p + 16, make_uint4(c[i][4], c[i][5], c[i][6], c[i][7]));
            } else if constexpr (OB == 16) {
                st_v4(p, make_uint4(c[i][0], c[i][1], c[i][2], c[i][3]));
            } else {
                st_v2(p, make_uint2(c[i][0], c[i][1]));
            }
            if constexpr (MODE == Q_E4M3_B128) {
                if ((g & 7) == 0) {
                    if (a.sfmt == 2) {  // e8m0 bytes, the row padded to whole int32 words with 0
                        sdst[g >> 3] = (uint8_t)bx[i];
                        if ((g >> 3) == (a.H >> 7) - 1)
                            for (int j = a.H >> 7; j < a.S; j++) sdst[j] = 0;
                    } else {
                        reinterpret_cast<float *>(sdst)[g >> 3] = bsinv[i];
                    }
                }
            }
            if constexpr (MODE == Q_MXFP8 || MODE == Q_MXFP4) {
                if ((g & 1) == 0) sdst[g >> 1] = (uint8_t)bx[i];
            }
        }
        if constexpr (MODE == Q_INT8) {
            if (lt == 0) *reinterpret_cast<float *>(sdst) = rsinv;
        }
    }
}

template <int MODE, int TPT, int GMAX>
__global__ void __launch_bounds__(block_threads(TPT)) dispatch_kernel(DispatchArgs a) {
    dispatch_body<MODE, TPT, GMAX>(a);
    // over GPUs: the grid's last block tells every GPU that the rows are there
    if (a.done) group_grid_done(a.done, a.flags, a.flag_kind, a.grp_g, a.grp_G, a.epoch);
}

// ---------------------------------------------------------------------------
// Combine backward ("EP dispatch with unfused MXFP8 quantization",
// Description): row(n,k) <- MXFP8(w[n,k] * g[n,:]).  The block maximum of
// |fl(w*g_h)| equals fl(|w| * max|g_h|) because rounding is monotone and sign
// symmetric, so it is taken once per token and scaled per entry.
template <int TPT, int GMAX, bool GROUP>
__device__ __forceinline__ void combine_bwd_body(const DispatchArgs &a) {
    pdl_enter();
    constexpr int TOKS = block_threads(TPT) / TPT;
    static_assert(TPT >= 32, "a warp belongs to one token");

    const int grp = threadIdx.x / TPT, lt = threadIdx.x % TPT;
    const int64_t n = (int64_t)blockIdx.x * TOKS + grp;
    const bool active = n < a.N;
    const int ngran = a.H >> 4;
    const int lane = lt & 31;

    // Every warp reads the token's entries itself (lane k holds entry k) and
    // hands them out by shuffles: no block barrier stands between a warp's
    // gradient loads and its stores.  The first warp reports the flags.
    // On one GPU the row index is handed out; over GPUs (peer_out) the two
    // destination pointers in the owner's window.
    int64_t my_row = -1;
    uint8_t *my_dst = nullptr, *my_sdst = nullptr;
    float my_w = 0.0f;
    if (active && lane < a.K) {
        uint32_t flags = 0;
        const int64_t e = a.idx[n * a.K + lane];
        const int32_t sl = (e >= 0 && e < a.E) ? a.slot[n * a.K + lane] : -1;
        my_row = row_of_entry(a, e, sl, flags);
        my_w = a.unweighted ? 1.0f : a.wts[n * a.K + lane];
        if (GROUP && my_row >= 0) {
            int32_t *src;
            float *rw;
            int64_t lrow;
            if (!row_dest(a, e, my_row, my_dst, my_sdst, src, rw, lrow, flags)) my_row = -1;
        }
        if (flags && lt < 32) atomicOr(a.status, flags);
    }

    // the token's gradient row, unpacked to fp32 once for all its entries
    float f[GMAX][16];
    float gmax[GMAX];
    uint32_t gm[GMAX];
#pragma unroll
    for (int i = 0; i < GMAX; i++) {
        const int g = i * TPT + lt;
        uint32_t v[8];
        if (active && g < ngran) {
            const uint16_t *p = a.x + n * a.H + (int64_t)g * 16;
            const uint4 u0 = ld_stream(p), u1 = ld_stream(p + 8);
            v[0] = u0.x; v[1] = u0.y; v[2] = u0.z; v[3] = u0.w;
            v[4] = u1.x; v[5] = u1.y; v[6] = u1.z; v[7] = u1.w;
        } else {
#pragma unroll
            for (int q = 0; q < 8; q++) v[q] = 0u;
        }
        uint32_t m = 0u;
#pragma unroll
        for (int q = 0; q < 8; q++) {
            m = bf2_absmax(m, v[q]);
            f[i][2 * q] = bf_lo(v[q]);
            f[i][2 * q + 1] = bf_hi(v[q]);
        }
        gm[i] = m;
    }
    // a NaN element (rare): the maxima again, NaN halves left out
    bool nan = false;
#pragma unroll
    for (int i = 0; i < GMAX; i++) nan = nan || bf2_any_nan(gm[i]);
    if (nan) {
#pragma unroll
        for (int i = 0; i < GMAX; i++) {
            const int g = i * TPT + lt;
            if (active && g < ngran) gm[i] = nan_free_absmax16(a.x + n * a.H + (int64_t)g * 16);
        }
    }
#pragma unroll
    for (int i = 0; i < GMAX; i++) {
        const float fm = bf2_fold(gm[i]);
        gmax[i] = fmaxf(fm, __shfl_xor_sync(kFull, fm, 1));
    }
    if (!active) return;  // a whole warp: tokens do not share warps

    const bool weighted = !a.unweighted;
    for (int k = 0; k < a.K; k++) {
        const int64_t row = __shfl_sync(kFull, my_row, k);
        const float w = __shfl_sync(kFull, my_w, k);
        if (row < 0) continue;
        uint8_t *dst, *sdst;
        if constexpr (GROUP) {
            dst = reinterpret_cast<uint8_t *>(
                __shfl_sync(kFull, reinterpret_cast<uintptr_t>(my_dst), k));
            sdst = reinterpret_cast<uint8_t *>(
                __shfl_sync(kFull, reinterpret_cast<uintptr_t>(my_sdst), k));
        } else {
            dst = a.out + row * (int64_t)a.H;
            sdst = a.out + a.scale_off + row * (int64_t)(a.H >> 5);
        }
        const float aw = fabsf(w);
#pragma unroll
        for (int i = 0; i < GMAX; i++) {
            const int g = i * TPT + lt;
            if (g >= ngran) continue;
            // NaN w (or inf w on a zero row) makes every product NaN: the
            // maximum of no element, X = 0 (mx_exponent's NaN case)
            const float amax = weighted ? __fmul_rn(aw, gmax[i]) : gmax[i];
            const int X = mx_exponent_fast<448>(amax);
            const float s = exp2_neg(X);
            uint32_t cw[4];
#pragma unroll
            for (int q = 0; q < 4; q++) {
                float p0 = f[i][4 * q], p1 = f[i][4 * q + 1], p2 = f[i][4 * q + 2], p3 = f[i][4 * q + 3];
                if (weighted) {  // fl(w * g), then fl(. * 2^-X): two multiplies, as defined
                    mul2(p0, p1, w);
                    mul2(p2, p3, w);
                }
                mul2(p0, p1, s);
                mul2(p2, p3, s);
                cw[q] = cvt_e4m3x2(p0, p1) | (cvt_e4m3x2(p2, p3) << 16);
            }
            st_v4(dst + (int64_t)g * 16, make_uint4(cw[0], cw[1], cw[2], cw[3]));
            if ((g & 1) == 0) sdst[g >> 1] = (uint8_t)(X + 127);
        }
    }
}

// GROUP: the rows go to the owners' windows over GPUs, and the grid ends with
// the signal (a separate instantiation: the one-GPU kernel carries neither)
template <int TPT, int GMAX, bool GROUP = false>
__global__ void __launch_bounds__(block_threads(TPT)) combine_bwd_kernel(DispatchArgs a) {
    combine_bwd_body<TPT, GMAX, GROUP>(a);
    if constexpr (GROUP) group_grid_done(a.done, a.flags, a.flag_kind, a.grp_g, a.grp_G, a.epoch);
}

}  // namespace ep
