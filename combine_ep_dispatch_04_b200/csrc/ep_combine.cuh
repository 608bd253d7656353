// ep_combine.cuh -- weighted top-k combine (bf16 or quantised expert outputs).
//
// "Low-Latency Mode API", low_latency_combine (Return Values: combined_x is
// the weighted sum across experts) and "DeepEP FP8 Dispatch and Combine
// Operations" (The FP8 Combine Operation: values are cast through fp32):
//   out[n,:] = bf16_rne( fma(w_{K-1}, y_{K-1}, ... fma(w_0, y_0, +0)) )
// over the valid entries in k order.
//
// Work split: a group of TPT = 128 threads owns one token; the row is cut
// into 8-element granules (16 bytes of bf16), thread lt holds granules
// g = i*TPT + lt.  For each granule the thread first issues the loads of all
// K expert rows (up to KB = 8 independent 16-byte loads in flight), then runs
// the fused multiply-adds in k order, so that memory latency is paid once per
// granule rather than once per expert.  Expert rows are read exactly once:
// loads are streaming (evict-first).
#pragma once

#include "ep_device.cuh"

namespace ep {

struct CombineArgs {
    int64_t N;
    int K, E, H;
    int packed;
    int64_t cap, rows;
    int64_t D, S, scale_off;  // quantised expert outputs: row bytes, scale bytes, scale region
    const uint16_t *y;        // bf16 rows, or the quantised buffer (data then scales)
    const int64_t *idx;
    const float *wts;
    const int32_t *slot;
    const int64_t *eo;
    uint16_t *out;
    uint32_t *status;
};

constexpr int kCombineThreads = 256;

enum { QIN_BF16 = 0, QIN_E4M3_B128 = 1, QIN_INT8 = 2, QIN_MXFP8 = 3, QIN_MXFP4 = 4 };

// Eight expert-output values of granule g of `row`, as fp32: bf16 widened, or
// quantised codes decoded and multiplied by their scale (one fp32 multiply --
// "DeepEP FP8 Dispatch and Combine Operations", The FP8 Combine Operation).
template <int QIN>
struct Granule {
    uint4 raw;   // bf16: 16 bytes; e4m3 / int8: 8 bytes in .x .y; e2m1: 4 bytes in .x
    float scale;
};

template <int QIN>
__device__ __forceinline__ Granule<QIN> load_granule(const CombineArgs &a, int64_t row, int g) {
    Granule<QIN> r;
    const uint8_t *base = reinterpret_cast<const uint8_t *>(a.y);
    if constexpr (QIN == QIN_BF16) {
        r.raw = ld_stream(a.y + row * a.H + (int64_t)g * 8);
        r.scale = 1.0f;
    } else {
        const uint8_t *sc = base + a.scale_off + row * a.S;
        if constexpr (QIN == QIN_MXFP4) {
            r.raw.x = __ldcs(reinterpret_cast<const unsigned int *>(base + row * a.D + (int64_t)g * 4));
            r.raw.y = r.raw.z = r.raw.w = 0u;
        } else {
            const uint2 d = __ldcs(reinterpret_cast<const uint2 *>(base + row * a.D + (int64_t)g * 8));
            r.raw = make_uint4(d.x, d.y, 0u, 0u);
        }
        if constexpr (QIN == QIN_INT8) r.scale = __ldg(reinterpret_cast<const float *>(sc));
        if constexpr (QIN == QIN_E4M3_B128)
            r.scale = __ldg(reinterpret_cast<const float *>(sc) + (g >> 4));
        if constexpr (QIN == QIN_MXFP8 || QIN == QIN_MXFP4)
            r.scale = exp2_neg(127 - (int)__ldg(sc + (g >> 2)));
    }
    return r;
}

template <int QIN>
__device__ __forceinline__ void decode_granule(const Granule<QIN> &r, float (&v)[8]) {
    if constexpr (QIN == QIN_BF16) {
        const uint32_t u[4] = {r.raw.x, r.raw.y, r.raw.z, r.raw.w};
#pragma unroll
        for (int q = 0; q < 4; q++) {
            v[2 * q] = bf_lo(u[q]);
            v[2 * q + 1] = bf_hi(u[q]);
        }
    } else if constexpr (QIN == QIN_INT8) {
        const uint32_t u[2] = {r.raw.x, r.raw.y};
#pragma unroll
        for (int q = 0; q < 8; q++)
            v[q] = __fmul_rn((float)(int8_t)((u[q >> 2] >> (8 * (q & 3))) & 0xFFu), r.scale);
    } else if constexpr (QIN == QIN_MXFP4) {
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const float2 f = e2m1x2_to_f32(r.raw.x >> (8 * q));
            v[2 * q] = __fmul_rn(f.x, r.scale);
            v[2 * q + 1] = __fmul_rn(f.y, r.scale);
        }
    } else {  // e4m3 codes
        const uint32_t u[2] = {r.raw.x, r.raw.y};
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const float2 f = e4m3x2_to_f32(u[q >> 1] >> (16 * (q & 1)));
            v[2 * q] = __fmul_rn(f.x, r.scale);
            v[2 * q + 1] = __fmul_rn(f.y, r.scale);
        }
    }
}

template <int TPT, int GMAX, int KB, int QIN>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(CombineArgs a) {
    pdl_enter();
    constexpr int TOKS = kCombineThreads / TPT;
    __shared__ int64_t s_row[TOKS][16];
    __shared__ float s_w[TOKS][16];

    const int grp = threadIdx.x / TPT, lt = threadIdx.x % TPT;
    const int64_t n = (int64_t)blockIdx.x * TOKS + grp;
    const bool active = n < a.N;

    if (active && lt < a.K) {
        uint32_t flags = 0;
        int64_t row = -1;
        const int64_t e = a.idx[n * a.K + lt];
        if (e < -1 || e >= a.E) flags |= kDevBadIndex;
        const int32_t s = (e >= 0 && e < a.E) ? a.slot[n * a.K + lt] : -1;
        if (s >= 0) {
            if (!a.packed) {
                if (s < a.cap) row = e * a.cap + s;
                else flags |= kDevCapacity;
            } else {
                const int64_t r = a.eo[e] + s;
                if (r < a.eo[e + 1] && r < a.rows) row = r;
                else flags |= kDevCapacity;
            }
        }
        if (flags) atomicOr(a.status, flags);
        s_row[grp][lt] = row;
        s_w[grp][lt] = a.wts[n * a.K + lt];
    }
    __syncthreads();
    if (!active) return;

    const int ngran = a.H >> 3;
#pragma unroll
    for (int i = 0; i < GMAX; i++) {
        const int g = i * TPT + lt;
        if (g >= ngran) break;
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; q++) acc[q] = 0.0f;
        for (int k0 = 0; k0 < a.K; k0 += KB) {
            if constexpr (QIN == QIN_BF16) {
                uint4 buf[KB];
#pragma unroll
                for (int kk = 0; kk < KB; kk++) {
                    const int k = k0 + kk;
                    const int64_t row = k < a.K ? s_row[grp][k] : -1;
                    buf[kk] = row >= 0 ? ld_stream(a.y + row * a.H + (int64_t)g * 8)
                                       : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int kk = 0; kk < KB; kk++) {
                    const int k = k0 + kk;
                    if (k >= a.K || s_row[grp][k] < 0) continue;
                    const float w = s_w[grp][k];
                    const uint32_t u[4] = {buf[kk].x, buf[kk].y, buf[kk].z, buf[kk].w};
#pragma unroll
                    for (int q = 0; q < 4; q++) {
                        acc[2 * q] = __fmaf_rn(w, bf_lo(u[q]), acc[2 * q]);
                        acc[2 * q + 1] = __fmaf_rn(w, bf_hi(u[q]), acc[2 * q + 1]);
                    }
                }
            } else {
                Granule<QIN> buf[KB];
#pragma unroll
                for (int kk = 0; kk < KB; kk++) {
                    const int k = k0 + kk;
                    const int64_t row = k < a.K ? s_row[grp][k] : -1;
                    if (row >= 0) buf[kk] = load_granule<QIN>(a, row, g);
                }
#pragma unroll
                for (int kk = 0; kk < KB; kk++) {
                    const int k = k0 + kk;
                    if (k >= a.K || s_row[grp][k] < 0) continue;
                    const float w = s_w[grp][k];
                    float v[8];
                    decode_granule<QIN>(buf[kk], v);
#pragma unroll
                    for (int q = 0; q < 8; q++) acc[q] = __fmaf_rn(w, v[q], acc[q]);
                }
            }
        }
        st_v4(a.out + n * a.H + (int64_t)g * 8,
              make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                         pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7])));
    }
}

}  // namespace ep
