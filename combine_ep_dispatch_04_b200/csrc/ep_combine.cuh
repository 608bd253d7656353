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
// block_threads(TPT) / TPT tokens); the row is cut into granules of 16 bytes
// of expert output (8 bf16 elements; 16 e4m3 / int8 codes; 32 e2m1 codes),
// thread lt holds granules g = i*TPT + lt.  For each granule the thread first
// issues the loads of all K expert rows (up to KB = 8 independent 16-byte
// loads in flight), then runs the fused multiply-adds in k order, so that
// memory latency is paid once per granule rather than once per expert.
// Expert rows are read exactly once: loads are streaming (evict-first).
#pragma once

#include "ep_device.cuh"

namespace ep {

struct CombineArgs {
    int64_t N;
    int K, E, H;
    int packed;
    int64_t cap, rows;
    int64_t D, S, scale_off;  // quantised expert outputs: row bytes, scale bytes, scale region
    int sfmt;                 // e4m3_b128 scales: fp32 (0, 1) or e8m0 bytes (2)
    const uint16_t *y;        // bf16 rows, or the quantised buffer (data then scales)
    TopkIdx idx;
    const float *wts;
    const int32_t *slot;
    const int64_t *eo;
    uint16_t *out;
    uint32_t *status;
    // expert parallelism over GPUs (ep_group.cuh): y is read from the window of
    // the GPU that owns each virtual row; peer_y == nullptr on one GPU
    const uint8_t *const *peer_y;  // [G] expert-output windows
    int64_t win_rows;
    int experts_per_gpu;           // an expert's owner is e / experts_per_gpu
};

enum { QIN_BF16 = 0, QIN_E4M3_B128 = 1, QIN_INT8 = 2, QIN_MXFP8 = 3, QIN_MXFP4 = 4 };

// Elements of a granule: 16 bytes of bf16 expert output, or of codes.
__host__ __device__ constexpr int combine_granule(int qin) {
    return qin == QIN_BF16 ? 8 : (qin == QIN_MXFP4 ? 32 : 16);
}

// Quantised expert outputs ("DeepEP FP8 Dispatch and Combine Operations",
// The FP8 Combine Operation): every code is decoded exactly (e4m3 / e2m1 by
// the hardware conversions to f16 and then f32, which also turn the e4m3 NaN
// codes into NaN; int8 through the 2^23 constant of i8_exact) and multiplied
// by its row / block scale as one fp32 multiply, y = fl(decode(c) * s),
// before the FMA.
//
// Two elements at a time on the packed fp32 pipe (mul.rn.f32x2 / fma.rn.f32x2,
// sm_100): each lane is one IEEE multiply or fused multiply-add, rounded to
// nearest even, exactly the scalar __fmul_rn / __fmaf_rn.
// The weight and the scale are splat once per expert row ({w, w}, {s, s}) and
// the codes unpacked by vector moves (four e2m1 bytes, two e4m3 halves).
__device__ __forceinline__ uint64_t splat2(float v) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(v));
    return r;
}
// (a0, a1) <- fma(w, fl(x * s), a) lane by lane
__device__ __forceinline__ void dq2(float &a0, float &a1, uint64_t w2, uint64_t s2, float x0,
                                    float x1) {
    asm("{\n\t.reg .b64 a, x;\n\tmov.b64 a, {%0, %1};\n\tmov.b64 x, {%4, %5};\n\t"
        "mul.rn.f32x2 x, x, %3;\n\tfma.rn.f32x2 a, %2, x, a;\n\tmov.b64 {%0, %1}, a;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "l"(w2), "l"(s2), "f"(x0), "f"(x1));
}
// (a0, a1) <- fma(w, x, a) lane by lane
__device__ __forceinline__ void fma2(float &a0, float &a1, uint64_t w2, float x0, float x1) {
    asm("{\n\t.reg .b64 a, x;\n\tmov.b64 a, {%0, %1};\n\tmov.b64 x, {%3, %4};\n\t"
        "fma.rn.f32x2 a, %2, x, a;\n\tmov.b64 {%0, %1}, a;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "l"(w2), "f"(x0), "f"(x1));
}
// Codes widen exactly through f16 (every e4m3 and e2m1 value is an f16 value).
// The eight e2m1 codes of u (code j in nibble j) as four f16 pairs, h[b] from byte b.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t u, uint32_t (&h)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(u));
}
// The four e4m3 codes of u (code j in byte j) as two f16 pairs, h[b] from half b.
__device__ __forceinline__ void e4m3x4_to_f16x2(uint32_t u, uint32_t (&h)[2]) {
    asm("{\n\t.reg .b16 c0, c1;\n\tmov.b32 {c0, c1}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, c0;\n\tcvt.rn.f16x2.e4m3x2 %1, c1;\n\t}"
        : "=r"(h[0]), "=r"(h[1])
        : "r"(u));
}
__device__ __forceinline__ float2 f16x2_to_f32(uint32_t h) {
    return __half22float2(*reinterpret_cast<const __half2 *>(&h));
}

// acc <- fma(w, fl(decode(c) * s), acc) over the 16 bytes of codes in r.
template <int QIN>
__device__ __forceinline__ void dequant_fma(float (&acc)[combine_granule(QIN)], const uint4 &r,
                                            float s, float w) {
    const uint32_t u[4] = {r.x, r.y, r.z, r.w};
    const uint64_t w2 = splat2(w), s2 = splat2(s);
#pragma unroll
    for (int q = 0; q < 4; q++) {
        if constexpr (QIN == QIN_INT8) {
            const uint32_t wx = u[q] ^ 0x80808080u;
#pragma unroll
            for (int j = 0; j < 4; j += 2)
                dq2(acc[4 * q + j], acc[4 * q + j + 1], w2, s2, i8_exact(wx, j), i8_exact(wx, j + 1));
        } else if constexpr (QIN == QIN_MXFP4) {
            uint32_t h[4];
            e2m1x8_to_f16x2(u[q], h);
#pragma unroll
            for (int b = 0; b < 4; b++) {
                const float2 f = f16x2_to_f32(h[b]);
                dq2(acc[8 * q + 2 * b], acc[8 * q + 2 * b + 1], w2, s2, f.x, f.y);
            }
        } else {
            uint32_t h[2];
            e4m3x4_to_f16x2(u[q], h);
#pragma unroll
            for (int b = 0; b < 2; b++) {
                const float2 f = f16x2_to_f32(h[b]);
                dq2(acc[4 * q + 2 * b], acc[4 * q + 2 * b + 1], w2, s2, f.x, f.y);
            }
        }
    }
}

// Where s is a normal power of two 2^k (every MX scale; E4M3 per 128 with
// round_scale or UE8M0), y = decode(c) * s is exact (a code has at most four
// significant bits and k keeps it finite), and so is W = w * s when W is
// normal (or w is zero); then fma(W, decode(c), acc) equals the oracle's
// fma(w, y, acc), with one FFMA per element and no multiply.  Returns false,
// doing nothing, where that does not hold.
template <int QIN>
__device__ __forceinline__ bool pow2_fma(float (&acc)[combine_granule(QIN)], const uint4 &r,
                                         float s, float w) {
    constexpr int kMaxExp = QIN == QIN_MXFP4 ? 125 : 119;  // largest code * 2^k finite
    const uint32_t sb = __float_as_uint(s);
    const int ex = (int)(sb >> 23);  // a set sign bit makes ex > 255
    if ((sb & 0x007FFFFFu) != 0u || ex < 1 || ex - 127 > kMaxExp) return false;
    const float W = __fmul_rn(w, s);
    if (!((fabsf(W) >= FLT_MIN || w == 0.0f) && fabsf(W) <= FLT_MAX)) return false;
    const uint32_t u[4] = {r.x, r.y, r.z, r.w};
    const uint64_t W2 = splat2(W);
#pragma unroll
    for (int q = 0; q < 4; q++) {
        if constexpr (QIN == QIN_MXFP4) {
            uint32_t h[4];
            e2m1x8_to_f16x2(u[q], h);
#pragma unroll
            for (int b = 0; b < 4; b++) {
                const float2 f = f16x2_to_f32(h[b]);
                fma2(acc[8 * q + 2 * b], acc[8 * q + 2 * b + 1], W2, f.x, f.y);
            }
        } else {
            uint32_t h[2];
            e4m3x4_to_f16x2(u[q], h);
#pragma unroll
            for (int b = 0; b < 2; b++) {
                const float2 f = f16x2_to_f32(h[b]);
                fma2(acc[4 * q + 2 * b], acc[4 * q + 2 * b + 1], W2, f.x, f.y);
            }
        }
    }
    return true;
}

// Whether pow2_fma is worth trying: int8 scales are never used that way, and
// fp32 per-128 scales (amax / qmax, E4M3_B128 without round_scale) are almost
// never powers of two; pow2_fma's result equals dequant_fma's wherever it applies.
template <int QIN>
__device__ __forceinline__ bool use_pow2(int sfmt) {
    if constexpr (QIN == QIN_INT8 || QIN == QIN_BF16) return false;
    if constexpr (QIN == QIN_E4M3_B128) return sfmt != 0;
    return true;
}

template <int TPT, int GMAX, int KB, int QIN>
__global__ void __launch_bounds__(block_threads(TPT)) combine_kernel(CombineArgs a) {
    pdl_enter();
    constexpr int TOKS = block_threads(TPT) / TPT;
    constexpr int EPG = combine_granule(QIN);
    __shared__ int64_t s_row[TOKS][16];          // the row in its window (-1: none)
    __shared__ const uint8_t *s_ybase[TOKS][16];  // the window: y, or the owner GPU's
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
        const uint8_t *yb = reinterpret_cast<const uint8_t *>(a.y);
        if (a.peer_y && row >= 0) {  // virtual row -> the expert owner's window
            const int o = (int)(e / a.experts_per_gpu);
            row -= (int64_t)o * a.win_rows;
            yb = a.peer_y[o];
            if (row >= a.win_rows) {
                row = -1;
                flags |= kDevCapacity;
            }
        }
        if (flags) atomicOr(a.status, flags);
        s_row[grp][lt] = row;
        s_ybase[grp][lt] = yb;
        s_w[grp][lt] = a.wts[n * a.K + lt];
    }
    __syncthreads();
    if (!active) return;

    const int ngran = a.H / EPG;
#pragma unroll (QIN == QIN_BF16 ? GMAX : 1)
    for (int i = 0; i < GMAX; i++) {
        const int g = i * TPT + lt;
        if (g >= ngran) break;
        float acc[EPG];
#pragma unroll
        for (int q = 0; q < EPG; q++) acc[q] = 0.0f;
        for (int k0 = 0; k0 < a.K; k0 += KB) {
            if constexpr (QIN == QIN_BF16) {
                uint4 buf[KB];
#pragma unroll
                for (int kk = 0; kk < KB; kk++) {
                    const int k = k0 + kk;
                    const int64_t row = k < a.K ? s_row[grp][k] : -1;
                    buf[kk] = row >= 0 ? ld_stream(reinterpret_cast<const uint16_t *>(
                                                       s_ybase[grp][k]) +
                                                   row * a.H + (int64_t)g * 8)
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
                // quantised rows: 16 bytes of codes and their scale per entry,
                // loaded for all KB entries before any use
                uint4 raw[KB];
                float sc[KB];
#pragma unroll
                for (int kk = 0; kk < KB; kk++) {
                    const int k = k0 + kk;
                    const int64_t row = k < a.K ? s_row[grp][k] : -1;
                    raw[kk] = make_uint4(0u, 0u, 0u, 0u);
                    sc[kk] = 0.0f;
                    if (row >= 0) {
                        const uint8_t *ybase = s_ybase[grp][k];
                        const uint8_t *sp = ybase + a.scale_off + row * a.S;
                        raw[kk] = ld_stream(ybase + row * a.D + (int64_t)g * 16);
                        if constexpr (QIN == QIN_INT8) sc[kk] = __ldg(reinterpret_cast<const float *>(sp));
                        if constexpr (QIN == QIN_E4M3_B128)  // 128 elements a scale
                            sc[kk] = a.sfmt == 2 ? exp2_neg(127 - (int)__ldg(sp + (g >> 3)))
                                                 : __ldg(reinterpret_cast<const float *>(sp) + (g >> 3));
                        if constexpr (QIN == QIN_MXFP8)  // 32 elements a scale
                            sc[kk] = exp2_neg(127 - (int)__ldg(sp + (g >> 1)));
                        if constexpr (QIN == QIN_MXFP4)
                            sc[kk] = exp2_neg(127 - (int)__ldg(sp + g));
                    }
                }
#pragma unroll
                for (int kk = 0; kk < KB; kk++) {
                    const int k = k0 + kk;
                    if (k >= a.K || s_row[grp][k] < 0) continue;
                    if (use_pow2<QIN>(a.sfmt) && pow2_fma<QIN>(acc, raw[kk], sc[kk], s_w[grp][k]))
                        continue;
                    dequant_fma<QIN>(acc, raw[kk], sc[kk], s_w[grp][k]);
                }
            }
        }
        uint16_t *o = a.out + n * a.H + (int64_t)g * EPG;
#pragma unroll
        for (int q = 0; q < EPG; q += 8)
            st_v4(o + q, make_uint4(pack_bf16x2(acc[q], acc[q + 1]),
                                    pack_bf16x2(acc[q + 2], acc[q + 3]),
                                    pack_bf16x2(acc[q + 4], acc[q + 5]),
                                    pack_bf16x2(acc[q + 6], acc[q + 7])));
    }
}

// ---------------------------------------------------------------------------
// Combine of quantised expert outputs with the next granule's codes in flight
// while the current one is decoded.  Decoding costs several operations per
// element, so a thread that loaded, then decoded, would have no load in flight
// for much of its time: here each thread copies the codes of granule i+1 (16
// bytes per row) into its own slots of a two-stage shared-memory buffer
// (cp.async) before it decodes granule i.  The scales of the token's rows are
// copied once, with granule 0's codes.  Each thread reads only codes it copied
// itself, so its own cp.async.wait_group orders those copies before the reads;
// the scales, copied by all threads of the token, are read after a barrier.
// No spin wait is involved.  Power-of-two scales take pow2_fma (one FFMA per
// element), others dequant_fma.  Requires K <= 8 and scale rows of a multiple
// of 4 bytes (S % 4 == 0) and at most kPipeScaleBytes; the launcher takes
// combine_kernel otherwise.
constexpr int kPipeRows = 8;          // K bound of combine_q_kernel
constexpr int kPipeScaleBytes = 256;  // S bound (H <= 8192: 4*H/128 or H/32)

template <int QIN>
__device__ __forceinline__ float scale_at(const uint8_t *srow, int g, int sfmt) {
    if constexpr (QIN == QIN_INT8) return *reinterpret_cast<const float *>(srow);
    if constexpr (QIN == QIN_E4M3_B128) {
        if (sfmt != 2) return reinterpret_cast<const float *>(srow)[g >> 3];
        return exp2_neg(127 - (int)srow[g >> 3]);
    }
    if constexpr (QIN == QIN_MXFP8) return exp2_neg(127 - (int)srow[g >> 1]);
    return exp2_neg(127 - (int)srow[g]);  // MXFP4: one byte per granule of 32
}

template <int TPT, int GMAX, int QIN>
__global__ void __launch_bounds__(block_threads(TPT)) combine_q_kernel(CombineArgs a) {
    static_assert(QIN != QIN_BF16 && TPT <= 128, "quantised rows, blocks of 128 threads");
    pdl_enter();
    constexpr int NT = block_threads(TPT);
    constexpr int TOKS = NT / TPT;
    constexpr int EPG = combine_granule(QIN);
    constexpr int KB = kPipeRows;
    __shared__ int64_t s_row[TOKS][16];
    __shared__ float s_w[TOKS][16];
    __shared__ __align__(16) uint4 s_code[2][KB][NT];
    __shared__ __align__(16) uint8_t s_scl[TOKS][KB * kPipeScaleBytes];

    const int tid = threadIdx.x;
    const int grp = tid / TPT, lt = tid % TPT;
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

    const int ngran = a.H / EPG;
    const uint8_t *ybase = reinterpret_cast<const uint8_t *>(a.y);
    // the token's scale rows, whole, in 16- or 4-byte pieces
    if (active) {
        const uint8_t *sbase = ybase + a.scale_off;
        const int S = (int)a.S;
        if (S % 16 == 0) {
            const int per = S / 16;
            for (int w = lt; w < a.K * per; w += TPT) {
                const int kk = w / per, o = (w - kk * per) * 16;
                const int64_t row = s_row[grp][kk];
                if (row >= 0) cp_async16(&s_scl[grp][kk * S + o], sbase + row * a.S + o);
            }
        } else {
            const int per = S / 4;
            for (int w = lt; w < a.K * per; w += TPT) {
                const int kk = w / per, o = (w - kk * per) * 4;
                const int64_t row = s_row[grp][kk];
                if (row >= 0) cp_async4(&s_scl[grp][kk * S + o], sbase + row * a.S + o);
            }
        }
    }
    // copies of granule i's codes (if it exists) into stage i & 1, as one group
    auto issue = [&](int i) {
        const int g = i * TPT + lt;
        if (active && i < GMAX && g < ngran) {
#pragma unroll
            for (int kk = 0; kk < KB; kk++) {
                const int64_t row = kk < a.K ? s_row[grp][kk] : -1;
                if (row >= 0)
                    cp_async16(&s_code[i & 1][kk][tid], ybase + row * a.D + (int64_t)g * 16);
            }
        }
        cp_async_commit();
    };
    issue(0);
    cp_async_wait<0>();  // this thread's scale pieces and granule 0
    __syncthreads();     // every thread's scale pieces
    if (!active) return;

    // the token's weights and live rows, once (the unrolled entry loop below
    // keeps them in registers)
    float wk[KB];
    uint32_t live = 0;
#pragma unroll
    for (int kk = 0; kk < KB; kk++) {
        const bool ok = kk < a.K && s_row[grp][kk] >= 0;
        live |= ok ? (1u << kk) : 0u;
        wk[kk] = ok ? s_w[grp][kk] : 0.0f;
    }
    const bool try_pow2 = use_pow2<QIN>(a.sfmt);
#pragma unroll 1
    for (int i = 0; i < GMAX; i++) {
        const int g = i * TPT + lt;
        if (g >= ngran) break;
        issue(i + 1);
        cp_async_wait<1>();  // granule i's group has landed
        float acc[EPG];
#pragma unroll
        for (int q = 0; q < EPG; q++) acc[q] = 0.0f;
        // the entries' decode chains are independent: unrolled, they overlap
#pragma unroll
        for (int kk = 0; kk < KB; kk++) {
            if (!(live & (1u << kk))) continue;
            const uint4 r = s_code[i & 1][kk][tid];
            const float sc = scale_at<QIN>(&s_scl[grp][kk * (int)a.S], g, a.sfmt);
            if (try_pow2 && pow2_fma<QIN>(acc, r, sc, wk[kk])) continue;
            dequant_fma<QIN>(acc, r, sc, wk[kk]);
        }
        uint16_t *o = a.out + n * a.H + (int64_t)g * EPG;
#pragma unroll
        for (int q = 0; q < EPG; q += 8)
            st_v4(o + q, make_uint4(pack_bf16x2(acc[q], acc[q + 1]),
                                    pack_bf16x2(acc[q + 2], acc[q + 3]),
                                    pack_bf16x2(acc[q + 4], acc[q + 5]),
                                    pack_bf16x2(acc[q + 6], acc[q + 7])));
    }
    cp_async_wait<0>();  // nothing in flight when the thread exits
}

// ---------------------------------------------------------------------------
// Weight gradient of the combine: dw[n,k] = <g[n,:], y[row(n,k),:]>, the
// derivative of sum_k w_k y_k with respect to w_k.  Every bf16 x bf16
// product is exact in fp32 and enters an fp32 FMA chain per thread (its
// granules in order), then a shuffle / shared-memory tree over the token's
// threads; masked entries get 0.  Reads g once and each entry's expert row
// once (the bytes of a combine).
struct WgradArgs {
    int64_t N;
    int K, E, H;
    int packed;
    int64_t cap, rows;
    const uint16_t *g;  // [N][H] bf16
    const uint16_t *y;  // [rows][H] bf16
    TopkIdx idx;
    const int32_t *slot;
    const int64_t *eo;
    float *dw;          // [N][K]
    uint32_t *status;
};

template <int TPT, int GMAX>
__global__ void __launch_bounds__(block_threads(TPT)) combine_wgrad_kernel(WgradArgs a) {
    pdl_enter();
    constexpr int NT = block_threads(TPT);
    constexpr int TOKS = NT / TPT;
    constexpr int WPG = (TPT + 31) / 32;  // warps per token group
    constexpr int KB = 8;                 // row loads in flight per granule
    __shared__ int64_t s_row[TOKS][16];
    __shared__ float s_part[TOKS][WPG][16];

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
    }
    __syncthreads();

    float acc[16];
#pragma unroll
    for (int k = 0; k < 16; k++) acc[k] = 0.0f;
    const int ngran = a.H >> 3;
    if (active) {
#pragma unroll 1
        for (int i = 0; i < GMAX; i++) {
            const int g = i * TPT + lt;
            if (g >= ngran) break;
            const uint4 gv = ld_stream(a.g + n * a.H + (int64_t)g * 8);
            const uint32_t gu[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
            for (int k0 = 0; k0 < 16; k0 += KB) {
                if (k0 >= a.K) break;
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
                    const uint32_t u[4] = {buf[kk].x, buf[kk].y, buf[kk].z, buf[kk].w};
                    float t = acc[k0 + kk];
#pragma unroll
                    for (int q = 0; q < 4; q++) {
                        t = __fmaf_rn(bf_lo(gu[q]), bf_lo(u[q]), t);
                        t = __fmaf_rn(bf_hi(gu[q]), bf_hi(u[q]), t);
                    }
                    acc[k0 + kk] = t;
                }
            }
        }
    }
    // the token's threads: warp shuffles, then the warps' partial sums
#pragma unroll
    for (int k = 0; k < 16; k++) {
        float v = acc[k];
#pragma unroll
        for (int o = (TPT < 32 ? TPT : 32) / 2; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
        acc[k] = v;
    }
    if ((lt & 31) == 0) {
#pragma unroll
        for (int k = 0; k < 16; k++) s_part[grp][lt >> 5][k] = acc[k];
    }
    __syncthreads();
    if (active && lt < a.K) {
        float v = 0.0f;
#pragma unroll
        for (int wp = 0; wp < WPG; wp++) v += s_part[grp][wp][lt];
        a.dw[n * a.K + lt] = s_row[grp][lt] >= 0 ? v : 0.0f;
    }
}

}  // namespace ep
