/*
 * ep_oracle.c -- the oracle for MoE expert-parallel token dispatch and combine.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  This file is a plain, slow,
 * obviously-correct CPU statement of what the dispatch / combine path
 * computes.  Only the test suite, the package smoke check and the benchmark's
 * CPU-baseline leg may load it.  It shares no code, header, table or constant
 * generator with the CUDA library, and it never includes the library's
 * header.  Status-bit values are restated here from the meaning they carry.
 *
 * Sources (web pages, cited by title and section):
 *   [LL]   "Low-Latency Mode API" (DeepEP-Ascend, sgl-kernel-npu docs):
 *          low_latency_dispatch Parameters / Return Values / Constraints,
 *          low_latency_combine Parameters / Return Values.
 *   [FP8]  "DeepEP FP8 Dispatch and Combine Operations: Low-Precision
 *          All-to-All for MoE": The Dispatch Stage; The FP8 Combine
 *          Operation; Advanced Configuration Options; Summary.
 *   [TE]   "[Common][PyTorch] EP dispatch with unfused MXFP8 quantization"
 *          (TransformerEngine PR): Description; Changes.
 *   [A5]   "[feat] A5 deep fused moe supported" (sgl-kernel-npu PR): Testing;
 *          the operator's grouped matrix multiplications between dispatch
 *          and combine (the expert maps below, bf16 / MXFP8 / MXFP4).
 * The e4m3 / e2m1 / e8m0 encodings are written from the public OCP 8-bit
 * floating point and OCP Microscaling (MX) v1.0 format definitions.
 *
 * Arithmetic rules: every float operation here is a single IEEE-754 binary32
 * operation, round-to-nearest-even (the file is built with
 * -ffp-contract=off -fno-fast-math, so no multiply-add is fused unless
 * fmaf() is called by name); the dot products of the weight gradient and
 * the expert maps are summed in double (exact products) and rounded once.
 *
 * Parity: every function here is pinned by the CPU test suite against
 * brute force, closed forms, library routines or the pages' worked example.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- modes, layouts and status bits (restated from their meaning) ------- */
enum { ORC_BF16 = 0, ORC_E4M3_B128 = 1, ORC_INT8_TOKEN = 2, ORC_MXFP8 = 3, ORC_MXFP4 = 4,
       ORC_E4M3_B128_P2 = 5,     /* E4M3_B128 with round_scale: fp32 scales, powers of two */
       ORC_E4M3_B128_UE8M0 = 6 }; /* ... stored as e8m0 bytes, 4 to an int32 (use_ue8m0) */
enum { ORC_PADDED = 0, ORC_PACKED = 1 };
#define ORC_ST_BAD_INDEX 0x1u
#define ORC_ST_CAPACITY 0x2u

/* ---- scalar conversions ------------------------------------------------- */

static float bits_to_f32(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }

/* bf16 -> fp32 is exact: a bf16 is the top half of a binary32. */
float orc_bf16_to_f32(uint16_t h) { return bits_to_f32((uint32_t)h << 16); }

/* fp32 -> bf16, round to nearest, ties to even (NaN -> quiet NaN). */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t b = f32_to_bits(f);
    if (isnan(f)) return (uint16_t)((b >> 16) | 0x0040u);
    uint32_t lsb = (b >> 16) & 1u;
    return (uint16_t)((b + 0x7FFFu + lsb) >> 16);
}

/*
 * Generic round-to-nearest-even into a small float format with
 * `ebits` exponent bits, `mbits` mantissa bits, exponent bias `bias`,
 * and largest finite magnitude `maxval`; values beyond it saturate to it
 * ("satfinite").  Returns the unsigned code (exponent field << mbits |
 * mantissa).  Follows the OCP definitions: subnormals when the exponent
 * field is zero, value = m * 2^(1-bias-mbits); normals
 * value = (1 + m/2^mbits) * 2^(e-bias).
 */
static uint32_t small_float_code(float a /* >= 0, finite */, int mbits, int bias, float maxval,
                                 uint32_t maxcode)
{
    if (a >= maxval) return maxcode;
    int emin = 1 - bias; /* exponent of the smallest normal */
    if (a < ldexpf(1.0f, emin)) {
        /* subnormal range: count units of 2^(emin-mbits), RNE */
        float q = rintf(ldexpf(a, mbits - emin));
        return (uint32_t)q; /* q == 2^mbits lands exactly on the smallest normal code */
    }
    int e;
    float m = frexpf(a, &e); /* a = m * 2^e, m in [0.5, 1) */
    e -= 1;                  /* a = (2m) * 2^e, 2m in [1, 2) */
    float frac = ldexpf(2.0f * m - 1.0f, mbits); /* exact */
    float q = rintf(frac);                        /* RNE on the mantissa */
    if (q == ldexpf(1.0f, mbits)) { q = 0.0f; e += 1; }
    uint32_t code = ((uint32_t)(e + bias) << mbits) | (uint32_t)q;
    if (code > maxcode) code = maxcode; /* rounding carried past the largest finite */
    return code;
}

/* OCP FP8 E4M3 ("e4m3fn"): bias 7, 3 mantissa bits, max 448 (0x7E), NaN 0x7F,
 * no infinities.  Round to nearest even, saturate finite overflow. */
uint8_t orc_e4m3_encode(float x)
{
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    float a = fabsf(x);
    return (uint8_t)(sign | small_float_code(a, 3, 7, 448.0f, 0x7E));
}

/* OCP MX FP4 E2M1: bias 1, 1 mantissa bit, values {0,.5,1,1.5,2,3,4,6},
 * sign in bit 3.  Round to nearest even, saturate to 6 (infinities
 * included).  The format has no NaN and neither the OCP definition nor the
 * pages say which code a NaN input takes: it is unspecified, and this
 * encoder returns ORC_E2M1_NO_CODE (not a 4-bit code) so that a comparison
 * that forgets to leave such elements out fails. */
#define ORC_E2M1_NO_CODE 0xFFu
uint8_t orc_e2m1_encode(float x)
{
    if (isnan(x)) return ORC_E2M1_NO_CODE;
    uint8_t sign = signbit(x) ? 0x8 : 0x0;
    float a = fabsf(x);
    return (uint8_t)(sign | small_float_code(a, 1, 1, 6.0f, 0x7));
}

/* Decoders (used by the property tests to bound the quantisation error). */
float orc_e4m3_decode(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    float v = e ? ldexpf(1.0f + m / 8.0f, e - 7) : ldexpf((float)m, -9);
    return s ? -v : v;
}
float orc_e2m1_decode(uint8_t c)
{
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    float v = e ? ldexpf(1.0f + m / 2.0f, e - 1) : 0.5f * (float)m;
    return s ? -v : v;
}

/*
 * e8m0 exponent of an MX block: X = ceil(log2 v) for v > 0, where
 * v = amax / qmax.  [LL] use_ue8m0 / round_scale ask for power-of-two scales
 * without a rounding rule; the reading here rounds UP, so that every element of
 * the block fits: |x| * 2^-X <= qmax.  Written with frexp, which splits v into
 * m * 2^e exactly (m in [0.5, 1)); log2 v is an integer only when m == 0.5.
 * The exponent is clamped to the e8m0 range [-127, 127] (byte 255 = NaN is
 * never produced); an infinite quotient gives 127.  amax == 0 gives X = 0
 * (scale 1.0).
 */
int orc_mx_exponent(float amax, float qmax)
{
    if (amax == 0.0f) return 0;
    float v = amax / qmax; /* one IEEE division */
    if (v == 0.0f) return -127; /* underflowed: log2 v is below the e8m0 range */
    if (isinf(v)) return 127;   /* an infinite maximum: log2 v is above it */
    int e;
    float m = frexpf(v, &e);
    int X = (m == 0.5f) ? e - 1 : e;
    if (X < -127) X = -127;
    if (X > 127) X = 127;
    return X;
}

/* ---- per-row quantisation ([LL] use_fp8 / use_ue8m0 / use_mxfp4, [FP8]
 * The Dispatch Stage, [TE] Description) --------------------------------- */

/* bytes of one quantised row's data and scale parts */
long orc_row_data_bytes(int mode, int H)
{
    switch (mode) {
    case ORC_BF16: return 2L * H;
    case ORC_MXFP4: return H / 2;
    default: return H;
    }
}
long orc_row_scale_bytes(int mode, int H)
{
    switch (mode) {
    case ORC_BF16: return 0;
    case ORC_INT8_TOKEN: return 4;
    case ORC_E4M3_B128: return 4L * (H / 128);
    case ORC_E4M3_B128_P2: return 4L * (H / 128);
    case ORC_E4M3_B128_UE8M0: return 4L * ((H / 128 + 3) / 4); /* whole int32 words, pad bytes 0 */
    default: return H / 32; /* one e8m0 byte per 32 elements */
    }
}

/* Largest magnitude of a block; NaN elements are left out (the comparison
 * is false for them), as fmaxf does.  A NaN element still encodes as NaN. */
static float absmax(const float *x, int n)
{
    float a = 0.0f;
    for (int i = 0; i < n; i++) {
        float v = fabsf(x[i]);
        if (v > a) a = v;
    }
    return a;
}

/*
 * Quantise one fp32 row x[0..H) into `data` / `scale` bytes.
 *   BF16:       data = bf16 of each element (exact when x came from bf16).
 *   INT8_TOKEN: one scale per row ([LL] use_fp8: per-token dynamic
 *               quantisation, INT8 data, float32 scale).  s = 127/amax,
 *               q = clamp(rint(x*s), -127, 127), stored scale = amax/127.
 *   E4M3_B128:  per 128-element block ([FP8] The Dispatch Stage):
 *               s = qmax/amax_b, code = e4m3(x*s), stored scale_inv =
 *               amax_b/qmax (fp32).  qmax defaults to 448, the largest
 *               e4m3 value; 127 reproduces the page's printed constant.
 *   MXFP8:      e4m3 data, one e8m0 byte per 32 elements ([LL] use_ue8m0;
 *               [TE] Description): X = ceil(log2(amax/448)), code =
 *               e4m3(x * 2^-X), byte = X + 127.
 *   MXFP4:      as MXFP8 with e2m1 (max 6); two codes per byte, element 2i
 *               in the low nibble ([LL] use_mxfp4: data [rows, H/2]).
 *   E4M3_B128_P2: E4M3_B128 with round_scale ([LL] round_scale; [FP8]
 *               Advanced Configuration Options, Round-Scale Mode): the
 *               block's scale is the power of two of the MX rule, X =
 *               ceil(log2(amax_b/qmax)), code = e4m3(x * 2^-X), stored
 *               scale_inv = 2^X (fp32).
 *   E4M3_B128_UE8M0: the same codes, the scale stored as the e8m0 byte
 *               X + 127, one per block, four to an int32 ([FP8] Advanced
 *               Configuration Options, UE8M0 Support: 8-bit scales in a
 *               packed format); the row's unused pad bytes are 0.
 * amax == 0 uses the scale 1 (stored 1.0f or byte 127).  The int8/e4m3
 * scale s is limited to FLT_MAX so that a tiny amax cannot turn 0*s into NaN.
 */
void orc_quant_row_f32(int mode, int H, float e4m3_qmax, const float *x, uint8_t *data,
                       uint8_t *scale)
{
    if (mode == ORC_BF16) {
        for (int h = 0; h < H; h++) {
            uint16_t b = orc_f32_to_bf16(x[h]);
            memcpy(data + 2L * h, &b, 2);
        }
        return;
    }
    if (mode == ORC_INT8_TOKEN) {
        float amax = absmax(x, H);
        float s = 1.0f, sinv = 1.0f;
        if (amax != 0.0f) {
            s = 127.0f / amax;
            if (s > FLT_MAX) s = FLT_MAX;
            sinv = amax / 127.0f;
        }
        for (int h = 0; h < H; h++) {
            float q = rintf(x[h] * s);
            if (isnan(q)) q = 0.0f; /* int8 has no NaN: a NaN product (NaN x, or inf * 0) is 0 */
            if (q > 127.0f) q = 127.0f;
            if (q < -127.0f) q = -127.0f;
            data[h] = (uint8_t)(int8_t)q;
        }
        memcpy(scale, &sinv, 4);
        return;
    }
    if (mode == ORC_E4M3_B128) {
        float qmax = e4m3_qmax > 0.0f ? e4m3_qmax : 448.0f;
        for (int b = 0; b < H / 128; b++) {
            const float *xb = x + 128L * b;
            float amax = absmax(xb, 128);
            float s = 1.0f, sinv = 1.0f;
            if (amax != 0.0f) {
                s = qmax / amax;
                if (s > FLT_MAX) s = FLT_MAX;
                sinv = amax / qmax;
            }
            for (int i = 0; i < 128; i++) data[128L * b + i] = orc_e4m3_encode(xb[i] * s);
            memcpy(scale + 4L * b, &sinv, 4);
        }
        return;
    }
    if (mode == ORC_E4M3_B128_P2 || mode == ORC_E4M3_B128_UE8M0) {
        float qmax = e4m3_qmax > 0.0f ? e4m3_qmax : 448.0f;
        int nb = H / 128;
        if (mode == ORC_E4M3_B128_UE8M0)
            memset(scale, 0, (size_t)orc_row_scale_bytes(mode, H));
        for (int b = 0; b < nb; b++) {
            const float *xb = x + 128L * b;
            int X = orc_mx_exponent(absmax(xb, 128), qmax);
            float mult = ldexpf(1.0f, -X);
            for (int i = 0; i < 128; i++) data[128L * b + i] = orc_e4m3_encode(xb[i] * mult);
            if (mode == ORC_E4M3_B128_P2) {
                float sinv = ldexpf(1.0f, X);
                memcpy(scale + 4L * b, &sinv, 4);
            } else {
                scale[b] = (uint8_t)(X + 127);
            }
        }
        return;
    }
    /* MXFP8 / MXFP4 */
    float qmax = (mode == ORC_MXFP8) ? 448.0f : 6.0f;
    for (int b = 0; b < H / 32; b++) {
        const float *xb = x + 32L * b;
        int X = orc_mx_exponent(absmax(xb, 32), qmax);
        float mult = ldexpf(1.0f, -X); /* exact power of two (2^-127 is subnormal but exact) */
        scale[b] = (uint8_t)(X + 127);
        for (int i = 0; i < 32; i++) {
            float v = xb[i] * mult;
            if (mode == ORC_MXFP8) {
                data[32L * b + i] = orc_e4m3_encode(v);
            } else {
                uint8_t c = orc_e2m1_encode(v);
                if (c == ORC_E2M1_NO_CODE) c = 0; /* NaN element: unspecified nibble, 0 as a
                                                     placeholder that comparisons leave out */
                long byte = (32L * b + i) / 2;
                if (i % 2 == 0) data[byte] = c;                 /* low nibble */
                else data[byte] = (uint8_t)(data[byte] | (c << 4)); /* high nibble */
            }
        }
    }
}

/* Same, for a bf16 row (exact widening first). */
void orc_quant_row_bf16(int mode, int H, float e4m3_qmax, const uint16_t *x, uint8_t *data,
                        uint8_t *scale)
{
    float *xf = (float *)malloc(sizeof(float) * (size_t)H);
    for (int h = 0; h < H; h++) xf[h] = orc_bf16_to_f32(x[h]);
    orc_quant_row_f32(mode, H, e4m3_qmax, xf, data, scale);
    free(xf);
}

/* ---- routing layout and slots ------------------------------------------- */

/*
 * Routing layout ([LL] low_latency_dispatch: topk_idx with -1 = no expert,
 * recv_count per expert; [LL] low_latency_combine: x is
 * [num_local_experts, num_max_dispatch_tokens_per_rank * num_ranks, hidden]).
 *
 * R source ranks each hold T tokens (token n = r*T + t); E experts in
 * contiguous blocks of L = E/R per rank (expert e lives on rank e / L).
 * Entries are visited in (source rank, token, k) order and each valid entry
 * takes the next slot of its expert, so the slots inside an expert are
 * ordered by (source rank, token) with k breaking ties between duplicates.
 * Indices outside [-1, E) are counted as errors and treated as -1.
 *
 * Outputs: tokens_per_rank [R][R] (tokens of src r with >= 1 expert on dst
 * d), tokens_per_expert [R][E], is_token_in_rank [N][R] (0/1),
 * token_slot [N][K] (-1 for masked), recv_count [E].  For the packed
 * (grouped) layout, expert_offset [E+1] is the exclusive scan of
 * recv_count rounded up to `align` rows ([TE] Description: per-expert
 * grouped output; Changes: per-expert alignment).  In the padded layout a
 * slot >= cap = R*M has no row: it is flagged as a capacity overflow.
 * Returns the status bits.
 */
uint32_t orc_layout(int R, int T, int K, int E, int M, int layout, int align, const int64_t *idx,
                    int32_t *tokens_per_rank, int32_t *tokens_per_expert,
                    uint8_t *is_token_in_rank, int32_t *token_slot, int64_t *recv_count,
                    int64_t *expert_offset)
{
    uint32_t st = 0;
    long N = (long)R * T;
    int L = E / R;
    long cap = (long)R * M;
    memset(tokens_per_rank, 0, sizeof(int32_t) * (size_t)R * R);
    memset(tokens_per_expert, 0, sizeof(int32_t) * (size_t)R * E);
    memset(is_token_in_rank, 0, (size_t)N * R);
    memset(recv_count, 0, sizeof(int64_t) * (size_t)E);
    for (int r = 0; r < R; r++) {
        for (int t = 0; t < T; t++) {
            long n = (long)r * T + t;
            for (int k = 0; k < K; k++) {
                int64_t e = idx[n * K + k];
                if (e < -1 || e >= E) st |= ORC_ST_BAD_INDEX;
                if (e < 0 || e >= E) { token_slot[n * K + k] = -1; continue; }
                int64_t slot = recv_count[e]++;
                token_slot[n * K + k] = (int32_t)slot;
                if (layout == ORC_PADDED && slot >= cap) st |= ORC_ST_CAPACITY;
                tokens_per_expert[(long)r * E + e] += 1;
                is_token_in_rank[n * R + e / L] = 1;
            }
            for (int d = 0; d < R; d++) tokens_per_rank[r * R + d] += is_token_in_rank[n * R + d];
        }
    }
    if (expert_offset) {
        int64_t off = 0;
        for (int e = 0; e < E; e++) {
            expert_offset[e] = off;
            off += (recv_count[e] + align - 1) / align * align;
        }
        expert_offset[E] = off;
    }
    return st;
}

/* Row of (expert e, slot) in the receive buffer, or -1 when it has none. */
static long row_of(int layout, long cap, const int64_t *expert_offset, int64_t e, int32_t slot)
{
    if (slot < 0) return -1;
    if (layout == ORC_PADDED) return slot < cap ? e * cap + slot : -1;
    long row = expert_offset[e] + slot;
    return row < expert_offset[e + 1] ? row : -1;
}

/*
 * Dispatch ([LL] low_latency_dispatch Return Values; [TE] Changes: data and
 * block scales in one buffer, data region then scale region): each source
 * token is quantised once and its row is written to every valid expert slot.
 * Rows: padded row = e*cap + slot (= [rank][local expert][R*M] slots);
 * packed row = expert_offset[e] + slot.  src_info[row] = r*M + t.
 * recv_weights[row] = topk_weights of the entry when both are given.
 * Rows with no entry are left untouched.
 */
uint32_t orc_dispatch(int R, int T, int K, int E, int M, int H, int mode, float e4m3_qmax,
                      int layout, const uint16_t *x, const int64_t *idx, const float *topk_weights,
                      const int32_t *token_slot, const int64_t *expert_offset, uint8_t *recv_data,
                      uint8_t *recv_scale, int32_t *src_info, float *recv_weights)
{
    uint32_t st = 0;
    long cap = (long)R * M;
    long D = orc_row_data_bytes(mode, H), S = orc_row_scale_bytes(mode, H);
    uint8_t *qd = (uint8_t *)malloc((size_t)D);
    uint8_t *qs = (uint8_t *)malloc((size_t)(S > 0 ? S : 1));
    for (int r = 0; r < R; r++) {
        for (int t = 0; t < T; t++) {
            long n = (long)r * T + t;
            orc_quant_row_bf16(mode, H, e4m3_qmax, x + n * H, qd, qs);
            for (int k = 0; k < K; k++) {
                int64_t e = idx[n * K + k];
                int32_t slot = token_slot[n * K + k];
                if (e < 0 || e >= E || slot < 0) continue;
                long row = row_of(layout, cap, expert_offset, e, slot);
                if (row < 0) { st |= ORC_ST_CAPACITY; continue; }
                memcpy(recv_data + row * D, qd, (size_t)D);
                if (S) memcpy(recv_scale + row * S, qs, (size_t)S);
                src_info[row] = r * M + t;
                if (recv_weights && topk_weights) recv_weights[row] = topk_weights[n * K + k];
            }
        }
    }
    free(qd);
    free(qs);
    return st;
}

/*
 * Weighted top-k combine of one token ([LL] low_latency_combine: combined_x
 * is the weighted sum across experts; [FP8] The FP8 Combine Operation: the
 * sum is taken in fp32).  acc starts at +0 and, for k = 0..K-1 in order, each valid
 * entry adds w_k * y_k with one fused multiply-add; the sum is rounded to
 * bf16 (RNE).  Masked entries add nothing; weights are used as given.
 */
void orc_combine_row(int H, int K, const uint16_t *const *yrows, const float *w,
                     const uint8_t *valid, uint16_t *out)
{
    for (int h = 0; h < H; h++) {
        float acc = 0.0f;
        for (int k = 0; k < K; k++) {
            if (!valid[k]) continue;
            acc = fmaf(w[k], orc_bf16_to_f32(yrows[k][h]), acc);
        }
        out[h] = orc_f32_to_bf16(acc);
    }
}

uint32_t orc_combine(int R, int T, int K, int E, int M, int H, int layout, const uint16_t *y,
                     const int64_t *idx, const float *topk_weights, const int32_t *token_slot,
                     const int64_t *expert_offset, uint16_t *out)
{
    uint32_t st = 0;
    long N = (long)R * T, cap = (long)R * M;
    const uint16_t **rows = (const uint16_t **)malloc(sizeof(void *) * (size_t)K);
    uint8_t *valid = (uint8_t *)malloc((size_t)K);
    for (long n = 0; n < N; n++) {
        for (int k = 0; k < K; k++) {
            int64_t e = idx[n * K + k];
            int32_t slot = token_slot[n * K + k];
            long row = (e >= 0 && e < E) ? row_of(layout, cap, expert_offset, e, slot) : -1;
            if (e >= 0 && e < E && slot >= 0 && row < 0) st |= ORC_ST_CAPACITY;
            valid[k] = row >= 0;
            rows[k] = row >= 0 ? y + row * H : NULL;
        }
        orc_combine_row(H, K, rows, topk_weights + n * K, valid, out + n * H);
    }
    free(rows);
    free(valid);
    return st;
}

/*
 * Combine backward ([TE] Description: the result-grad is scattered back to
 * the expert positions through the reverse dispatch and quantised to
 * MXFP8).  For entry (n, k) the expert-output grad is w_k * g_n (each
 * product one fp32 multiply); `unweighted` gives the plain re-dispatch of
 * g_n.  The row is MXFP8-quantised and written at the forward's slot.
 */
/* One entry of the combine backward: MXFP8(w * g) (or MXFP8(g) unweighted). */
void orc_bwd_row(int H, float w, int unweighted, const uint16_t *g, uint8_t *data, uint8_t *scale)
{
    float *p = (float *)malloc(sizeof(float) * (size_t)H);
    for (int h = 0; h < H; h++) {
        float gv = orc_bf16_to_f32(g[h]);
        p[h] = unweighted ? gv : w * gv;
    }
    orc_quant_row_f32(ORC_MXFP8, H, 0.0f, p, data, scale);
    free(p);
}

/* Combine of N tokens whose K expert rows are already gathered:
 * yrows [N][K][H], w [N][K], valid [N][K] -> out [N][H]. */
void orc_combine_gathered(long N, int K, int H, const uint16_t *yrows, const float *w,
                          const uint8_t *valid, uint16_t *out)
{
    const uint16_t **rows = (const uint16_t **)malloc(sizeof(void *) * (size_t)K);
    for (long n = 0; n < N; n++) {
        for (int k = 0; k < K; k++) rows[k] = yrows + (n * K + k) * (long)H;
        orc_combine_row(H, K, rows, w + n * K, valid + n * K, out + n * H);
    }
    free(rows);
}

uint32_t orc_combine_bwd(int R, int T, int K, int E, int M, int H, int layout, int unweighted,
                         const uint16_t *g, const int64_t *idx, const float *topk_weights,
                         const int32_t *token_slot, const int64_t *expert_offset,
                         uint8_t *grad_data, uint8_t *grad_scale)
{
    uint32_t st = 0;
    long N = (long)R * T, cap = (long)R * M;
    long D = orc_row_data_bytes(ORC_MXFP8, H), S = orc_row_scale_bytes(ORC_MXFP8, H);
    for (long n = 0; n < N; n++) {
        for (int k = 0; k < K; k++) {
            int64_t e = idx[n * K + k];
            int32_t slot = token_slot[n * K + k];
            if (e < 0 || e >= E || slot < 0) continue;
            long row = row_of(layout, cap, expert_offset, e, slot);
            if (row < 0) { st |= ORC_ST_CAPACITY; continue; }
            float w = unweighted ? 1.0f : topk_weights[n * K + k];
            orc_bwd_row(H, w, unweighted, g + n * H, grad_data + row * D, grad_scale + row * S);
        }
    }
    return st;
}

/*
 * Gradient of the combine with respect to the top-k weights (the reading of
 * the "grad w.r.t. topk_weights" extension of the combine backward: the
 * combine is out[n] = sum_k w[n,k] * y_k, so d out / d w[n,k] = y_k and the
 * weight gradient is the dot product of the output gradient g[n,:] with the
 * entry's expert row).  Every product of two bf16 values is exact in double
 * and the sum is taken in double in h order, rounded to fp32 once.  Masked
 * entries get 0.
 */
uint32_t orc_combine_wgrad(int R, int T, int K, int E, int M, int H, int layout,
                           const uint16_t *g, const uint16_t *y, const int64_t *idx,
                           const int32_t *token_slot, const int64_t *expert_offset, float *dw)
{
    uint32_t st = 0;
    long N = (long)R * T, cap = (long)R * M;
    for (long n = 0; n < N; n++) {
        for (int k = 0; k < K; k++) {
            dw[n * K + k] = 0.0f;
            int64_t e = idx[n * K + k];
            if (e < -1 || e >= E) st |= ORC_ST_BAD_INDEX;
            int32_t slot = token_slot[n * K + k];
            if (e < 0 || e >= E || slot < 0) continue;
            long row = row_of(layout, cap, expert_offset, e, slot);
            if (row < 0) { st |= ORC_ST_CAPACITY; continue; }
            double acc = 0.0;
            for (int h = 0; h < H; h++)
                acc += (double)orc_bf16_to_f32(g[n * H + h]) * (double)orc_bf16_to_f32(y[row * H + h]);
            dw[n * K + k] = (float)acc;
        }
    }
    return st;
}

/* The same for tokens whose K expert rows are gathered: g [N][H], yrows
 * [N][K][H], valid [N][K] -> dw [N][K]; also sum_h |g*y| per entry (the
 * scale of the rounding error of any fp32 summation order) in absdot. */
void orc_combine_wgrad_gathered(long N, int K, int H, const uint16_t *g, const uint16_t *yrows,
                                const uint8_t *valid, float *dw, double *absdot)
{
    for (long n = 0; n < N; n++) {
        for (int k = 0; k < K; k++) {
            double acc = 0.0, mag = 0.0;
            if (valid[n * K + k]) {
                const uint16_t *y = yrows + (n * K + k) * (long)H;
                for (int h = 0; h < H; h++) {
                    double p = (double)orc_bf16_to_f32(g[n * H + h]) * (double)orc_bf16_to_f32(y[h]);
                    acc += p;
                    mag += fabs(p);
                }
            }
            dw[n * K + k] = (float)acc;
            absdot[n * K + k] = mag;
        }
    }
}

/*
 * The experts between dispatch and combine (each expert a single linear
 * map, standing in for the grouped matrix multiplications that the deep-fused
 * MoE operator of "[feat] A5 deep fused moe supported" runs between its
 * dispatch and combine): for every expert e and each of its rows r (rows
 * expert_offset[e] .. + count[e] of the packed receive layout),
 *   y[r, j] = bf16_rne( sum_h x[r, h] * w[e, j, h] ),  j < Nout,
 * the products exact in double, summed in double in h order, rounded to
 * fp32 and then to bf16.  Rows past count[e] are left untouched.
 */
void orc_expert_gemm(int E, int H, int Nout, const int64_t *expert_offset, const int64_t *count,
                     const uint16_t *x, const uint16_t *w, uint16_t *y)
{
    for (int e = 0; e < E; e++) {
        for (int64_t i = 0; i < count[e]; i++) {
            int64_t r = expert_offset[e] + i;
            for (int j = 0; j < Nout; j++) {
                const uint16_t *wr = w + ((int64_t)e * Nout + j) * H;
                double acc = 0.0;
                for (int h = 0; h < H; h++)
                    acc += (double)orc_bf16_to_f32(x[r * H + h]) * (double)orc_bf16_to_f32(wr[h]);
                y[r * Nout + j] = orc_f32_to_bf16((float)acc);
            }
        }
    }
}

/*
 * The same linear maps on MXFP8 operands ("[feat] A5 deep fused moe
 * supported": the deep-fused operator's grouped matrix multiplications take
 * e4m3 codes with one e8m0 scale per 32 elements, as its MX dispatch emits).
 * Element h of row r is decode_e4m3(xc[r, h]) * 2^(xs[r, h/32] - 127); weight
 * element (j, h) of expert e is decode_e4m3(wc[e, j, h]) * 2^(ws[e, j, h/32] - 127);
 *   y[r, j] = bf16_rne( sum_h x[r, h] * w[e, j, h] )
 * with every product exact in double (3-bit mantissas, power-of-two scales),
 * summed in double in h order, rounded to fp32 and then to bf16.  A NaN code
 * or scale byte 255 (NaN in the MX format) gives NaN.  Rows past count[e] are
 * left untouched.
 */
static double orc_e8m0_value(uint8_t b)
{
    return b == 255 ? NAN : ldexp(1.0, (int)b - 127);
}
void orc_expert_gemm_mx(int E, int H, int Nout, const int64_t *expert_offset, const int64_t *count,
                        const uint8_t *xc, const uint8_t *xs, const uint8_t *wc,
                        const uint8_t *ws, uint16_t *y)
{
    const int S = H / 32;
    for (int e = 0; e < E; e++) {
        for (int64_t i = 0; i < count[e]; i++) {
            int64_t r = expert_offset[e] + i;
            for (int j = 0; j < Nout; j++) {
                const int64_t wrow = (int64_t)e * Nout + j;
                double acc = 0.0;
                for (int h = 0; h < H; h++) {
                    double xv = (double)orc_e4m3_decode(xc[r * H + h]) * orc_e8m0_value(xs[r * S + h / 32]);
                    double wv = (double)orc_e4m3_decode(wc[wrow * H + h]) * orc_e8m0_value(ws[wrow * S + h / 32]);
                    acc += xv * wv;
                }
                y[r * Nout + j] = orc_f32_to_bf16((float)acc);
            }
        }
    }
}

/*
 * The same linear maps on MXFP4 operands (the deep-fused operator's MX
 * formats include e2m1 with an e8m0 scale per 32 elements, as its MX
 * dispatch emits): codes are packed two to a byte, element h in the low
 * nibble of byte h/2 when h is even and in the high nibble when h is odd.
 * Element h of row r is decode_e2m1(code) * 2^(xs[r, h/32] - 127), likewise
 * for the weights; y[r, j] = bf16_rne( sum_h x[r, h] * w[e, j, h] ), the
 * products exact in double, summed in h order, rounded to fp32 then bf16.
 * A scale byte 255 gives NaN.  Rows past count[e] are left untouched.
 */
static double orc_e2m1_at(const uint8_t *row, int h)
{
    uint8_t b = row[h / 2];
    return (double)orc_e2m1_decode((uint8_t)(h % 2 == 0 ? (b & 0xF) : (b >> 4)));
}
void orc_expert_gemm_mxfp4(int E, int H, int Nout, const int64_t *expert_offset,
                           const int64_t *count, const uint8_t *xc, const uint8_t *xs,
                           const uint8_t *wc, const uint8_t *ws, uint16_t *y)
{
    const int S = H / 32, D = H / 2;
    for (int e = 0; e < E; e++) {
        for (int64_t i = 0; i < count[e]; i++) {
            int64_t r = expert_offset[e] + i;
            for (int j = 0; j < Nout; j++) {
                const int64_t wrow = (int64_t)e * Nout + j;
                double acc = 0.0;
                for (int h = 0; h < H; h++) {
                    double xv = orc_e2m1_at(xc + r * D, h) * orc_e8m0_value(xs[r * S + h / 32]);
                    double wv = orc_e2m1_at(wc + wrow * D, h) * orc_e8m0_value(ws[wrow * S + h / 32]);
                    acc += xv * wv;
                }
                y[r * Nout + j] = orc_f32_to_bf16((float)acc);
            }
        }
    }
}

/*
 * The experts' gated two-layer MLP on MXFP8 operands ("[feat] A5 deep fused
 * moe supported": Testing, the per-stage table -- Dispatch, GMM1, SwiGLU,
 * Requant, GMM2, Combine; Benchmarking and Profiling -- hidden 7168,
 * moe-intermediate-size 3072, FP8 quantisation; its review notes that the
 * GMM1 operands are e4m3 codes with one e8m0 scale per 32 elements).
 * I is the intermediate size.  For each expert e and each of its rows r
 * (expert_offset[e] .. + count[e]):
 *   GMM1     h[j] = fl32( sum_k x[r,k] * W1[e][j,k] ),   j < 2I
 *            (exact products, summed in double in k order, one rounding)
 *   SwiGLU   z[j] = fl32( silu(h[j]) * h[I + j] ),        j < I
 *            silu(a) = a / (1 + exp(-a)), evaluated in double from the fp32
 *            h; the first I outputs of GMM1 are the gate, the last I the up
 *            projection
 *   Requant  the row z[0..I) quantised to MXFP8 exactly as the MX dispatch
 *            quantises a token (orc_quant_row_f32, one e8m0 scale per 32)
 *   GMM2     y[r, j] = bf16( fl32( sum_i zq[i] * W2[e][j,i] ) ),  j < H
 *            (the MXFP8 maps above with the intermediate size as depth)
 * W1 codes [E][2I][H] with e8m0 scales [E][2I][H/32]; W2 codes [E][H][I]
 * with scales [E][H][I/32].  Outputs per row: h_out (fp32 [rows][2I],
 * nullable), z_out (fp32 [rows][I], nullable), zc / zs (the requantised
 * codes [rows][I] and scales [rows][I/32]) and y (bf16 [rows][H]); rows past
 * count[e] are left untouched.
 */
void orc_expert_ffn_mx(int E, int H, int I, const int64_t *expert_offset, const int64_t *count,
                       const uint8_t *xc, const uint8_t *xs, const uint8_t *w1c,
                       const uint8_t *w1s, const uint8_t *w2c, const uint8_t *w2s, float *h_out,
                       float *z_out, uint8_t *zc, uint8_t *zs, uint16_t *y)
{
    const int SH = H / 32, SI = I / 32, N1 = 2 * I;
    float *h = (float *)malloc(sizeof(float) * (size_t)N1);
    float *z = (float *)malloc(sizeof(float) * (size_t)I);
    for (int e = 0; e < E; e++) {
        for (int64_t i = 0; i < count[e]; i++) {
            const int64_t r = expert_offset[e] + i;
            for (int j = 0; j < N1; j++) { /* GMM1 */
                const int64_t wrow = (int64_t)e * N1 + j;
                double acc = 0.0;
                for (int k = 0; k < H; k++) {
                    double xv = (double)orc_e4m3_decode(xc[r * H + k]) * orc_e8m0_value(xs[r * SH + k / 32]);
                    double wv = (double)orc_e4m3_decode(w1c[wrow * H + k]) * orc_e8m0_value(w1s[wrow * SH + k / 32]);
                    acc += xv * wv;
                }
                h[j] = (float)acc;
            }
            for (int j = 0; j < I; j++) { /* SwiGLU */
                const double g = (double)h[j], u = (double)h[I + j];
                z[j] = (float)(g / (1.0 + exp(-g)) * u);
            }
            orc_quant_row_f32(ORC_MXFP8, I, 0.0f, z, zc + r * I, zs + r * SI); /* Requant */
            for (int j = 0; j < H; j++) { /* GMM2 */
                const int64_t wrow = (int64_t)e * H + j;
                double acc = 0.0;
                for (int k = 0; k < I; k++) {
                    double zv = (double)orc_e4m3_decode(zc[r * I + k]) * orc_e8m0_value(zs[r * SI + k / 32]);
                    double wv = (double)orc_e4m3_decode(w2c[wrow * I + k]) * orc_e8m0_value(w2s[wrow * SI + k / 32]);
                    acc += zv * wv;
                }
                y[r * H + j] = orc_f32_to_bf16((float)acc);
            }
            if (h_out) memcpy(h_out + r * N1, h, sizeof(float) * (size_t)N1);
            if (z_out) memcpy(z_out + r * I, z, sizeof(float) * (size_t)I);
        }
    }
    free(h);
    free(z);
}

/*
 * Dequantisation of one row stored in a quantised format ([FP8] The FP8
 * Combine Operation: the received codes times the stored inverse scale, in
 * fp32).  Each element is decode(code) * scale_inv as
 * one fp32 multiply: int8 codes and e4m3 / e2m1 values times the row's or
 * block's fp32 scale_inv, MX codes times 2^(byte-127).  BF16 rows widen
 * exactly.
 */
void orc_dequant_row(int mode, int H, const uint8_t *data, const uint8_t *scale, float *out)
{
    for (int h = 0; h < H; h++) {
        float v, s;
        switch (mode) {
        case ORC_BF16: {
            uint16_t b;
            memcpy(&b, data + 2L * h, 2);
            out[h] = orc_bf16_to_f32(b);
            continue;
        }
        case ORC_INT8_TOKEN:
            v = (float)(int8_t)data[h];
            memcpy(&s, scale, 4);
            break;
        case ORC_E4M3_B128:
        case ORC_E4M3_B128_P2:
            v = orc_e4m3_decode(data[h]);
            memcpy(&s, scale + 4L * (h / 128), 4);
            break;
        case ORC_E4M3_B128_UE8M0:
            v = orc_e4m3_decode(data[h]);
            s = ldexpf(1.0f, (int)scale[h / 128] - 127);
            break;
        case ORC_MXFP8:
            v = orc_e4m3_decode(data[h]);
            s = ldexpf(1.0f, (int)scale[h / 32] - 127);
            break;
        default: /* MXFP4: element 2i in the low nibble */
            v = orc_e2m1_decode((uint8_t)((h % 2 == 0) ? (data[h / 2] & 0xF) : (data[h / 2] >> 4)));
            s = ldexpf(1.0f, (int)scale[h / 32] - 127);
            break;
        }
        out[h] = v * s;
    }
}

/*
 * Weighted top-k combine of quantised expert outputs: as orc_combine_row, with
 * each expert row dequantised first (rows: data [K][D], scales [K][S]).
 */
void orc_combine_row_q(int mode, int H, int K, const uint8_t *data, const uint8_t *scale,
                       const float *w, const uint8_t *valid, uint16_t *out)
{
    long D = orc_row_data_bytes(mode, H), S = orc_row_scale_bytes(mode, H);
    float *y = (float *)malloc(sizeof(float) * (size_t)H * (size_t)K);
    for (int k = 0; k < K; k++)
        if (valid[k]) orc_dequant_row(mode, H, data + k * D, scale + k * S, y + (long)k * H);
    for (int h = 0; h < H; h++) {
        float acc = 0.0f;
        for (int k = 0; k < K; k++)
            if (valid[k]) acc = fmaf(w[k], y[(long)k * H + h], acc);
        out[h] = orc_f32_to_bf16(acc);
    }
    free(y);
}

/* Tokens whose K quantised rows are gathered: data [N][K][D], scale [N][K][S]. */
void orc_combine_gathered_q(int mode, long N, int K, int H, const uint8_t *data,
                            const uint8_t *scale, const float *w, const uint8_t *valid,
                            uint16_t *out)
{
    long D = orc_row_data_bytes(mode, H), S = orc_row_scale_bytes(mode, H);
    for (long n = 0; n < N; n++)
        orc_combine_row_q(mode, H, K, data + n * K * D, scale + n * K * S, w + n * K,
                          valid + n * K, out + n * H);
}

/* ---- array helpers for the tests (loops over the scalar functions) ------ */
void orc_e4m3_encode_array(const float *x, uint8_t *out, long n)
{
    for (long i = 0; i < n; i++) out[i] = orc_e4m3_encode(x[i]);
}
void orc_e2m1_encode_array(const float *x, uint8_t *out, long n)
{
    for (long i = 0; i < n; i++) out[i] = orc_e2m1_encode(x[i]);
}
/* Encode the fp32 values with bit patterns start .. start+n-1 (a sweep of
 * the whole binary32 space in chunks); NaN patterns give the e4m3 NaN code,
 * and ORC_E2M1_NO_CODE for e2m1 (unspecified there). */
void orc_e4m3_encode_bits(uint32_t start, uint8_t *out, long n)
{
    for (long i = 0; i < n; i++) out[i] = orc_e4m3_encode(bits_to_f32(start + (uint32_t)i));
}
void orc_e2m1_encode_bits(uint32_t start, uint8_t *out, long n)
{
    for (long i = 0; i < n; i++) {
        float f = bits_to_f32(start + (uint32_t)i);
        out[i] = orc_e2m1_encode(f);
    }
}
/* e8m0 byte (X + 127) of a block whose maximum is |value of bit pattern
 * start+i|; 0xFF marks non-finite patterns (not an amax). */
void orc_mx_exponent_bits(uint32_t start, float qmax, uint8_t *out, long n)
{
    for (long i = 0; i < n; i++) {
        float a = fabsf(bits_to_f32(start + (uint32_t)i));
        out[i] = isfinite(a) ? (uint8_t)(orc_mx_exponent(a, qmax) + 127) : 0xFF;
    }
}
void orc_mx_exponent_array(const float *amax, float qmax, int32_t *out, long n)
{
    for (long i = 0; i < n; i++) out[i] = orc_mx_exponent(amax[i], qmax);
}
void orc_f32_to_bf16_array(const float *x, uint16_t *out, long n)
{
    for (long i = 0; i < n; i++) out[i] = orc_f32_to_bf16(x[i]);
}
