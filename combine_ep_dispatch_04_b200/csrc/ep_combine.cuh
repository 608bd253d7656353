// ep_combine.cuh -- weighted top-k combine (bf16 or quantised expert outputs).
//
// "Low-Latency Mode API", low_latency_combine (Return Values: combined_x is
// the weighted sum across experts) and "DeepEP FP8 Dispatch and Combine
// Operations" (The FP8 Combine Operation: the sum is taken in fp32):
//   out[n,:] = bf16_rne( fma(w_{K-1}, y_{K-1}, ... fma(w_0, y_0, +0)) )
// over the valid entries in k order.
//
// Work split: a group of TPT threads owns one token (TPT is chosen per shape
// so that the grid fits in one wave where it can; a block holds
// block_threads(TPT) / TPT tokens); the row is cut into 8-element granules
// (16 bytes of bf16), thread lt holds granules g = i*TPT + lt.  For each granule the thread first issues the loads of all
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

enum { QIN_BF16 = 0, QIN_E4M3_B128 = 1, QIN_INT8 = 2, QIN_MXFP8 = 3, QIN_MXFP4 = 4 };

// Quantised expert outputs ("DeepEP FP8 Dispatch and Combine Operations",
// The FP8 Combine Operation): each code is decoded exactly (e4m3 / e2m1 via
// the hardware conversions to f16, int8 as an integer) and multiplied by its
// row / block scale as one fp32 multiply before the FMA.
template <int TPT, int GMAX, int KB, int QIN>
__global__ void __launch_bounds__(block_threads(TPT)) combine_kernel(CombineArgs a) {
    pdl_enter();
    constexpr int TOKS = block_threads(TPT) / TPT;
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
                // quantised rows: the codes of the granule (8 bytes, 4 for e2m1)
                // and their scale, loaded for all KB entries before any use
                const uint8_t *ybase = reinterpret_cast<const uint8_t *>(a.y);
                uint2 raw[KB];
                float sc[KB];
#pragma unroll
                for (int kk = 0; kk < KB; kk++) {
                    const int k = k0 + kk;
                    const int64_t row = k < a.K ? s_row[grp][k] : -1;
                    raw[kk] = make_uint2(0u, 0u);
                    sc[kk] = 0.0f;
                    if (row >= 0) {
                        const uint8_t *d = ybase + row * a.D;
                        const uint8_t *sp = ybase + a.scale_off + row * a.S;
                        if constexpr (QIN == QIN_MXFP4)
                            raw[kk].x = __ldcs(reinterpret_cast<const unsigned int *>(d + (int64_t)g * 4));
                        else
                            raw[kk] = __ldcs(reinterpret_cast<const uint2 *>(d + (int64_t)g * 8));
                        if constexpr (QIN == QIN_INT8) sc[kk] = __ldg(reinterpret_cast<const float *>(sp));
                        if constexpr (QIN == QIN_E4M3_B128)
                            sc[kk] = __ldg(reinterpret_cast<const float *>(sp) + (g >> 4));
                        if constexpr (QIN == QIN_MXFP8 || QIN == QIN_MXFP4)
                            sc[kk] = exp2_neg(127 - (int)__ldg(sp + (g >> 2)));
                    }
                }
#pragma unroll
                for (int kk = 0; kk < KB; kk++) {
                    const int k = k0 + kk;
                    if (k >= a.K || s_row[grp][k] < 0) continue;
                    const float w = s_w[grp][k];
                    float v[8];
                    if constexpr (QIN == QIN_INT8) {
#pragma unroll
                        for (int q = 0; q < 8; q++) {
                            const uint32_t word = q < 4 ? raw[kk].x : raw[kk].y;
                            v[q] = __fmul_rn((float)(int8_t)((word >> (8 * (q & 3))) & 0xFFu), sc[kk]);
                        }
                    } else if constexpr (QIN == QIN_MXFP4) {
#pragma unroll
                        for (int q = 0; q < 4; q++) {
                            const float2 f = e2m1x2_to_f32(raw[kk].x >> (8 * q));
                            v[2 * q] = __fmul_rn(f.x, sc[kk]);
                            v[2 * q + 1] = __fmul_rn(f.y, sc[kk]);
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; q++) {
                            const uint32_t word = q < 2 ? raw[kk].x : raw[kk].y;
                            const float2 f = e4m3x2_to_f32(word >> (16 * (q & 1)));
                            v[2 * q] = __fmul_rn(f.x, sc[kk]);
                            v[2 * q + 1] = __fmul_rn(f.y, sc[kk]);
                        }
                    }
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
