/*
 * ep.h -- C ABI of libep: MoE expert-parallel token dispatch and combine on
 * one NVIDIA B200 (sm_100a).
 *
 * On one GPU the R "ranks" of expert parallelism are logical partitions of
 * buffers that all sit in this GPU's memory: no inter-GPU traffic exists.
 * The ep_group_* calls (near the end) split the same ranks over several GPUs.
 * Token n = r*T + t is token t of source rank r.  Expert e (of E) lives on
 * rank e / L, L = E / R, as local expert e % L.
 *
 * Page citations (title, section):
 *   [LL]  "Low-Latency Mode API" (DeepEP-Ascend docs): low_latency_dispatch
 *         and low_latency_combine -- Parameters, Return Values, Constraints.
 *   [FP8] "DeepEP FP8 Dispatch and Combine Operations: Low-Precision
 *         All-to-All for MoE": The Dispatch Stage, The FP8 Combine Operation.
 *   [TE]  "[Common][PyTorch] EP dispatch with unfused MXFP8 quantization"
 *         (TransformerEngine PR): Description, Changes.
 *   [IDX] "DeepEP topk_idx_t Custom Dtype Requirements": Tensor Requirements
 *         and Constraints, Runtime Validation.
 *   [A5]  "[feat] A5 deep fused moe supported" (sgl-kernel-npu PR): review
 *         comments on tiling validation.
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers unless stated; every buffer is allocated
 *     and owned by the caller.  The library allocates no device memory and
 *     keeps no per-call state.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and is asynchronous; outputs are valid in stream order.
 *   - Host-side checks run before any launch and before any division by a
 *     caller value ([A5] review: validate before dividing); a failed check
 *     returns an error and launches nothing.  Vector buffers (x, y, out,
 *     recv_buf, grad_buf) must be 16-byte aligned (EP_ERR_MISALIGNED).
 *   - Every buffer whose size follows from the receive layout (workspace,
 *     recv_buf, src_info, recv_weights, grad_buf, the expert outputs y) comes
 *     with the number of bytes the caller allocated for it (a `*_bytes`
 *     argument after the pointer).  A count below what the configuration
 *     needs (ep_buffer_sizes) gives EP_ERR_BUFFER_TOO_SMALL before any launch
 *     ([IDX] Runtime Validation: sizes are checked before GPU work).  Arrays
 *     sized by the configuration alone (x, out, topk_idx, token_slot, ...:
 *     [N][H], [N][K], [E] ...) carry no count.
 *   - Conditions found on the device (an expert index outside [-1, E), a
 *     slot beyond the receive capacity) never trap: the offending entry is
 *     skipped and a bit is OR-ed into *dev_status (a caller-owned uint32_t in
 *     device memory, zero before first use).  ep_get_status reads it.
 *   - Combine and combine-backward must be given the configuration and the
 *     layout outputs (token_slot, expert_offset) of the dispatch whose rows
 *     they read ([LL] low_latency_combine: indices must match dispatch; the
 *     handle is passed unchanged).
 */
#ifndef EP_H
#define EP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *ep_stream_t; /* identical to cudaStream_t */

typedef enum {
    EP_OK = 0,
    EP_ERR_INVALID_ARG = 1,   /* a size, enum or pointer argument is out of range */
    EP_ERR_UNSUPPORTED = 2,   /* valid request outside what this build implements */
    EP_ERR_MISALIGNED = 3,    /* a vector buffer is not 16-byte aligned */
    EP_ERR_CUDA = 4,          /* a CUDA runtime call failed (launch, copy, sync) */
    EP_ERR_DEVICE_STATUS = 5, /* ep_get_status found device-side error bits */
    EP_ERR_TIMEOUT = 6,       /* ep_get_status: a bounded wait gave up (EP_DEV_TIMEOUT) */
    EP_ERR_BUFFER_TOO_SMALL = 7 /* a *_bytes argument is below what the configuration needs */
} ep_status_t;

/* Quantisation of dispatched rows.  Values 2..4 equal the DeepEP-Ascend
 * quant_mode numbers ([LL] use_fp8 / use_ue8m0 / use_mxfp4). */
typedef enum {
    EP_Q_BF16 = 0,       /* plain bf16 rows ([LL] use_fp8=False) */
    EP_Q_E4M3_B128 = 1,  /* e4m3 + one fp32 scale_inv per 128 elements ([FP8] Dispatch Stage) */
    EP_Q_INT8_TOKEN = 2, /* int8 + one fp32 scale per row ([LL] use_fp8, quant_mode 2) */
    EP_Q_MXFP8 = 3,      /* e4m3 + one e8m0 byte per 32 elements ([LL] use_ue8m0; [TE]) */
    EP_Q_MXFP4 = 4       /* e2m1 x2 per byte + one e8m0 byte per 32 ([LL] use_mxfp4);
                          * e2m1 has no NaN: the nibble a NaN element takes is unspecified
                          * (the block's scale and its other elements are not affected) */
} ep_quant_t;

/* Receive-buffer layouts. */
typedef enum {
    EP_LAYOUT_PADDED = 0, /* [R][L][R*M] rows: per rank [L, R*M, H] ([LL] combine x) */
    EP_LAYOUT_PACKED = 1  /* rows of expert e at expert_offset[e] .. ([TE] grouped tensor) */
} ep_layout_t;

/* Bits of *dev_status. */
#define EP_DEV_BAD_INDEX 0x1u         /* topk_idx value < -1 or >= E (entry skipped) */
#define EP_DEV_CAPACITY_OVERFLOW 0x2u /* slot >= R*M in the padded layout (row skipped) */
#define EP_DEV_TIMEOUT 0x4u           /* a bounded wait (tensor-core kernels, ep_group_wait) gave up */

/* ep_config_t.flags */
#define EP_F_BWD_UNWEIGHTED 0x1u    /* combine-backward re-dispatches g without w */
#define EP_F_COMBINE_QUANTIZED 0x2u /* ep_combine's y is in cfg->quant's format (recv_buf layout) */
#define EP_F_IDX_I32 0x4u           /* topk_idx is int32 [N][K] instead of int64 ([IDX]) */
#define EP_F_ROUND_SCALE 0x8u       /* E4M3_B128: power-of-two scales ([LL] round_scale) */
#define EP_F_UE8M0 0x10u            /* E4M3_B128: the power-of-two scales as e8m0 bytes */
#define EP_F_LAYOUT_SINGLE_CTA 0x100u /* force the one-block layout path */
#define EP_F_LAYOUT_MULTI_CTA 0x200u  /* force the multi-block layout path */
#define EP_F_LAYOUT_CLUSTER 0x400u    /* force the thread-block-cluster layout path */
#define EP_F_GEMM_CTA_PAIRS 0x800u    /* ep_expert_gemm: two-CTA MMAs on CTA pairs */

/*
 * Flags on the formats:
 *   EP_F_IDX_I32      every topk_idx argument is int32 [N][K] ([IDX]: the
 *                     index type may be built with 32 or 64 bits); values
 *                     have the same meaning.
 *   EP_F_ROUND_SCALE  E4M3_B128 ([LL] round_scale; [FP8] Advanced Configuration
 *                     Options, Round-Scale Mode): each 128-block's scale is the
 *                     smallest power of two 2^X with amax/qmax <= 2^X (amax 0:
 *                     X = 0; X clamped to [-127, 127]), codes = e4m3(x * 2^-X),
 *                     stored scale_inv = 2^X (fp32).  The pages ask for
 *                     power-of-two scales without fixing the rounding; rounding
 *                     up keeps every element within qmax.  Allowed and without
 *                     effect for MXFP8 / MXFP4 (their scales are powers of two);
 *                     invalid for BF16 and INT8_TOKEN.
 *   EP_F_UE8M0        E4M3_B128 only, implies EP_F_ROUND_SCALE ([FP8] Advanced
 *                     Configuration Options, UE8M0 Support: 8-bit scales in a
 *                     packed format): the scale of block j is the e8m0 byte
 *                     X + 127 at byte j of the row's scales, four to an int32;
 *                     S = 4 * ceil(H/128 / 4) bytes, pad bytes written as 0.
 */
typedef struct {
    int32_t num_ranks;           /* R > 0 */
    int32_t num_tokens;          /* T tokens per rank, 0 <= T <= M */
    int32_t max_tokens_per_rank; /* M > 0 ([LL] num_max_dispatch_tokens_per_rank) */
    int32_t num_topk;            /* K in [1, 16] ([LL] Constraints) */
    int32_t num_experts;         /* E in [1, 1024], E % R == 0 */
    int32_t hidden;              /* H in [32, 8192], H % 32 == 0; % 128 for E4M3_B128 */
    int32_t quant;               /* ep_quant_t */
    int32_t layout;              /* ep_layout_t */
    int32_t expert_align;        /* packed layout: rows per expert rounded up to this (>= 1) */
    float e4m3_qmax;             /* E4M3_B128 target max, (0, 448]; 0 selects 448 */
    uint32_t flags;              /* EP_F_* */
} ep_config_t;

/* Byte sizes of the caller-owned buffers for one configuration.  "rows" is
 * the row capacity of every receive-layout buffer: E*R*M (padded) or
 * R*T*K + E*(expert_align-1) (packed, enough for every entry). */
typedef struct {
    int64_t rows;
    int64_t data_row_bytes;     /* D: 2H bf16, H int8/e4m3, H/2 e2m1 */
    int64_t scale_row_bytes;    /* S: 0 bf16, 4 int8, 4*H/128 e4m3_b128 (UE8M0: above), H/32 mx */
    int64_t recv_scale_offset;  /* recv_buf: data region [rows][D] then, here, scales [rows][S] */
    int64_t recv_bytes;
    int64_t src_info_bytes;     /* int32 [rows] */
    int64_t recv_weights_bytes; /* float [rows] */
    int64_t expert_out_bytes;   /* y for ep_combine: bf16 [rows][H] */
    int64_t grad_scale_offset;  /* grad_buf: e4m3 [rows][H] then e8m0 [rows][H/32] here */
    int64_t grad_bytes;
    int64_t workspace_bytes;    /* scratch for ep_dispatch_layout */
    int64_t token_slot_bytes;   /* int32 [N][K] */
    int64_t is_token_in_rank_bytes; /* uint8 [N][R] */
} ep_sizes_t;

/* Buffer sizes for `cfg` (validates it).  Host only; no device work. */
ep_status_t ep_buffer_sizes(const ep_config_t *cfg, ep_sizes_t *out);

/*
 * Routing layout and slot assignment ([LL] low_latency_dispatch: topk_idx
 * [num_tokens, num_topk] int64, -1 = no expert; recv_count [num_local_experts]
 * int64; cumulative_local_expert_recv_stats).
 *   topk_idx            int64 [N][K], N = R*T (int32 with EP_F_IDX_I32)
 *   tokens_per_rank     int32 [R][R]: tokens of src r with >= 1 expert on rank d (nullable)
 *   tokens_per_expert   int32 [R][E]: entries of src r routed to e (nullable)
 *   is_token_in_rank    uint8 [N][R]: 1 if token n has an expert on rank d (nullable)
 *   token_slot          int32 [N][K]: rank of entry (n,k) among its expert's entries
 *                       ordered by (source rank, token, k); -1 when masked
 *   recv_count          int64 [E]
 *   expert_offset       int64 [E+1]: exclusive scan of recv_count rounded up to
 *                       expert_align (required for PACKED, nullable for PADDED)
 *   cumulative_recv_stats int64 [E]: += recv_count (nullable; [LL] load-balance stats)
 *   workspace           scratch (contents undefined after) of workspace_bytes
 *                       >= ep_sizes_t.workspace_bytes
 * Deterministic: the result never depends on thread timing.
 */
ep_status_t ep_dispatch_layout(const ep_config_t *cfg, const void *topk_idx,
                               int32_t *tokens_per_rank, int32_t *tokens_per_expert,
                               uint8_t *is_token_in_rank, int32_t *token_slot,
                               int64_t *recv_count, int64_t *expert_offset,
                               int64_t *cumulative_recv_stats, void *workspace,
                               size_t workspace_bytes, uint32_t *dev_status, ep_stream_t stream);

/*
 * Quantise each token once and scatter it to its experts' receive rows
 * ([LL] low_latency_dispatch Return Values; [FP8] The Dispatch Stage; [TE]
 * Changes: data region then scale region in one caller buffer).
 *   x              bf16 [N][H]
 *   topk_idx       int64 [N][K] (int32 with EP_F_IDX_I32); token_slot /
 *                  expert_offset from ep_dispatch_layout
 *   topk_weights   float [N][K] (nullable; needed for recv_weights)
 *   recv_buf       recv_bytes >= ep_sizes_t.recv_bytes: row (e, slot) holds the
 *                  token's quantised row; padded row = e*R*M + slot, packed row =
 *                  expert_offset[e] + slot.  Rows without an entry are not written.
 *   src_info       int32 [rows], src_info_bytes >= 4*rows: r*M + t of the
 *                  row's source token
 *   recv_weights   float [rows] (nullable; recv_weights_bytes >= 4*rows, ignored
 *                  when NULL): the entry's top-k weight
 */
ep_status_t ep_dispatch(const ep_config_t *cfg, const uint16_t *x, const void *topk_idx,
                        const float *topk_weights, const int32_t *token_slot,
                        const int64_t *expert_offset, void *recv_buf, size_t recv_bytes,
                        int32_t *src_info, size_t src_info_bytes, float *recv_weights,
                        size_t recv_weights_bytes, uint32_t *dev_status, ep_stream_t stream);

/*
 * ep_dispatch_layout followed by ep_dispatch in one call, with the same
 * arguments and results as the two calls ([LL] low_latency_dispatch returns
 * the received tokens and recv_count from one call).  Because the call
 * launches the layout itself, the dispatch kernel may start while the layout
 * runs: it loads and quantises its tokens first and waits for the layout only
 * before reading token_slot / expert_offset.
 */
ep_status_t ep_dispatch_with_layout(const ep_config_t *cfg, const uint16_t *x,
                                    const void *topk_idx, const float *topk_weights,
                                    int32_t *tokens_per_rank, int32_t *tokens_per_expert,
                                    uint8_t *is_token_in_rank, int32_t *token_slot,
                                    int64_t *recv_count, int64_t *expert_offset,
                                    int64_t *cumulative_recv_stats, void *workspace,
                                    size_t workspace_bytes, void *recv_buf, size_t recv_bytes,
                                    int32_t *src_info, size_t src_info_bytes, float *recv_weights,
                                    size_t recv_weights_bytes, uint32_t *dev_status,
                                    ep_stream_t stream);

/*
 * Weighted top-k combine ([LL] low_latency_combine: combined_x [T, H] bf16 is
 * the weighted sum across experts; `out` written in place):
 *   out[n,:] = bf16_rne( sum over valid k = 0..K-1, in order, of
 *                        w[n,k] * y[row(n,k), :] )
 * accumulated in fp32 with one fused multiply-add per term.  Masked entries
 * add nothing; a token with no valid entry gets +0.  Weights are used as given.
 *   y      bf16 [rows][H] expert outputs in the receive layout (y_bytes >=
 *          ep_sizes_t.expert_out_bytes); with EP_F_COMBINE_QUANTIZED (and
 *          cfg->quant != EP_Q_BF16) y is instead a buffer of y_bytes >=
 *          ep_sizes_t.recv_bytes in cfg->quant's format (data region
 *          then scale region, as ep_dispatch writes it) and each expert value
 *          is decode(code) * scale as one fp32 multiply before the FMA ([FP8]
 *          The FP8 Combine Operation: codes times the stored inverse scale,
 *          in fp32).  An e8m0 scale byte of 255 (NaN) is not a valid input.
 *   out    bf16 [N][H]
 */
ep_status_t ep_combine(const ep_config_t *cfg, const uint16_t *y, size_t y_bytes,
                       const void *topk_idx, const float *topk_weights, const int32_t *token_slot,
                       const int64_t *expert_offset, uint16_t *out, uint32_t *dev_status,
                       ep_stream_t stream);

/*
 * Combine backward ([TE] Description: the result gradient goes back to the
 * expert positions through the reverse dispatch, quantised to MXFP8): for
 * each valid entry, row(n,k) of grad_buf receives MXFP8(w[n,k] * g[n,:])
 * (MXFP8(g[n,:]) with EP_F_BWD_UNWEIGHTED).  cfg->quant is ignored: the
 * gradient is always MXFP8.
 *   g          bf16 [N][H]
 *   grad_buf   grad_bytes >= ep_sizes_t.grad_bytes: e4m3 [rows][H] then e8m0
 *              [rows][H/32]
 */
ep_status_t ep_combine_backward(const ep_config_t *cfg, const uint16_t *g,
                                const void *topk_idx, const float *topk_weights,
                                const int32_t *token_slot, const int64_t *expert_offset,
                                void *grad_buf, size_t grad_bytes, uint32_t *dev_status,
                                ep_stream_t stream);

/*
 * Gradient of the combine with respect to the top-k weights (the combine is
 * out[n] = sum_k w[n,k] * y[row(n,k)], so d out / d w[n,k] is the entry's
 * expert row; no page defines this call: it completes the combine backward
 * of [TE] Description, whose other half is ep_combine_backward):
 *   topk_weights_grad[n,k] = sum_h g[n,h] * y[row(n,k),h]
 * for each valid entry, 0 for masked ones.  Each bf16 x bf16 product is exact
 * in fp32; the sum is taken in fp32 (an FMA chain per thread over its part of
 * the row, then a tree over the token's threads), so its rounding depends on
 * the order: within 128 * 2^-24 * sum_h |g[n,h] * y[row,h]| of the exact sum.
 *   g                  bf16 [N][H]: gradient of the combined output
 *   y                  bf16 [rows][H]: the expert outputs ep_combine read
 *                      (y_bytes >= ep_sizes_t.expert_out_bytes)
 *   topk_weights_grad  float [N][K]
 * EP_F_COMBINE_QUANTIZED is not supported here (EP_ERR_UNSUPPORTED).
 */
ep_status_t ep_combine_backward_weights(const ep_config_t *cfg, const uint16_t *g,
                                        const uint16_t *y, size_t y_bytes, const void *topk_idx,
                                        const int32_t *token_slot, const int64_t *expert_offset,
                                        float *topk_weights_grad, uint32_t *dev_status,
                                        ep_stream_t stream);

/*
 * The experts between dispatch and combine, each one linear map ("[feat] A5
 * deep fused moe supported": grouped matrix multiplications of the experts run
 * between the operator's dispatch and combine).  For each expert e and each of
 * its received rows r (expert_offset[e] .. + recv_count[e] of the packed
 * receive layout):
 *   y[r, :] = bf16_rne( x[r, :] . W[e]^T )
 * with fp32 accumulation on the tensor cores (tcgen05: 128 x 256 tiles on
 * single CTAs; with EP_F_GEMM_CTA_PAIRS in cfg->flags, where pairs of SMs can
 * be scheduled, 256 x 256 tiles on CTA pairs with the two-CTA MMA);
 * padding rows of y (past recv_count[e]) are not written.  The summation
 * order of the fp32 accumulation is the hardware's: every product is exact
 * and H/16 partial sums are chained through one fp32 accumulator, so results
 * are within (H/16 + 16) * 2^-23 * sum_h |x*w| + 1 bf16 ulp of the exact sum.
 *   cfg          quant EP_Q_BF16 and layout EP_LAYOUT_PACKED (the dispatch that
 *                wrote recv_buf), H % 64 == 0; otherwise EP_ERR_UNSUPPORTED
 *   recv_buf     the dispatch's receive buffer: bf16 [rows][H] (recv_bytes >=
 *                rows * 2H)
 *   expert_offset, recv_count   from ep_dispatch_layout
 *   weights      bf16 [E][n_out][H] (row j of W[e] is output column j)
 *   n_out        output columns, a multiple of 256
 *   y            bf16 [rows][n_out] (y_bytes >= rows * n_out * 2; n_out = H
 *                gives ep_combine's input)
 * A wait inside the kernel that exceeds 2 s sets EP_DEV_TIMEOUT and the
 * kernel returns; it never traps.
 */
ep_status_t ep_expert_gemm(const ep_config_t *cfg, const void *recv_buf, size_t recv_bytes,
                           const int64_t *expert_offset, const int64_t *recv_count,
                           const uint16_t *weights, int32_t n_out, uint16_t *y, size_t y_bytes,
                           uint32_t *dev_status, ep_stream_t stream);

/*
 * The same linear maps on MX operands ("[feat] A5 deep fused moe supported":
 * the deep-fused operator's grouped matrix multiplications take the codes and
 * e8m0 block scales its MX dispatch emits): MXFP8 (e4m3 codes) or MXFP4 (e2m1
 * codes two a byte, element h in the low nibble of byte h/2 when h is even).
 * Element h of received row r is code value * 2^(scale[r][h/32] - 127), and
 * likewise for the weights; for each expert e and each of its received rows r
 *   y[r, j] = bf16_rne( sum_h x[r, h] * W[e][j, h] )
 * on the block-scaled tensor-core MMA (tcgen05 kind::mxf8f6f4 or kind::mxf4,
 * fp32 accumulation); padding rows of y are not written.  Every product is
 * exact and H/32 block sums are chained through one fp32 accumulator: results
 * are within (H/32 + 32) * 2^-23 * sum_h |x*w| + 1 bf16 ulp of the exact sum.
 * NaN codes, and scale bytes of 255 (NaN in the MX format), give unspecified
 * values in the rows or columns they touch.
 *   cfg          quant EP_Q_MXFP8 (H % 128 == 0) or EP_Q_MXFP4 (H % 256 == 0) and
 *                layout EP_LAYOUT_PACKED (the dispatch that wrote recv_buf);
 *                otherwise EP_ERR_UNSUPPORTED
 *   recv_buf     the dispatch's receive buffer (recv_bytes >= ep_sizes_t.recv_bytes):
 *                codes [rows][D] (D = H, or H/2 for MXFP4), then at
 *                ep_sizes_t.recv_scale_offset e8m0 [rows][H/32]
 *   expert_offset, recv_count   from ep_dispatch_layout
 *   w_codes      [E][n_out][D] in cfg's code format (row j of W[e] is output
 *                column j)
 *   w_scales     e8m0 [E][n_out][H/32]
 *   n_out        output columns, a multiple of 224, 256 or 128 (tiles of 224
 *                columns where they divide n_out, else 256, else 128; MXFP8
 *                with at least 256 entries an expert on average takes 256)
 *   y            bf16 [rows][n_out] (y_bytes >= rows * n_out * 2; n_out = H
 *                gives ep_combine's input)
 * recv_buf, w_codes, w_scales and y 16-byte aligned (EP_ERR_MISALIGNED).
 * A wait inside the kernel that exceeds 2 s sets EP_DEV_TIMEOUT and the
 * kernel returns; it never traps.
 */
ep_status_t ep_expert_gemm_mx(const ep_config_t *cfg, const void *recv_buf, size_t recv_bytes,
                              const int64_t *expert_offset, const int64_t *recv_count,
                              const uint8_t *w_codes, const uint8_t *w_scales, int32_t n_out,
                              uint16_t *y, size_t y_bytes, uint32_t *dev_status,
                              ep_stream_t stream);

/*
 * The experts' gated two-layer MLP on MXFP8 operands ("[feat] A5 deep fused
 * moe supported": the operator's stages GMM1, SwiGLU, Requant and GMM2
 * between its dispatch and combine, with moe-intermediate-size I; its review:
 * GMM1 takes e4m3 codes with one e8m0 scale per 32 elements).  For each
 * expert e and each of its received rows r (packed layout):
 *   GMM1     h = x[r] . W1[e]^T                       (2I outputs, fp32)
 *   SwiGLU   z[j] = silu(h[j]) * h[I + j], j < I        silu(a) = a / (1 + e^-a)
 *   Requant  z to MXFP8 per 32 with the MX dispatch's rule (written to z_buf)
 *   GMM2     y[r] = bf16( zq . W2[e]^T )               (H outputs)
 * The first I rows of W1[e] are the gate projection, the last I the up
 * projection.  SwiGLU and the requant run in GMM1's epilogue on the fp32
 * accumulator (tcgen05 block-scaled MMA); GMM2 is ep_expert_gemm_mx's kernel
 * with depth I.  Accuracy: GMM1's sums are chained as in ep_expert_gemm_mx
 * ((H/32 + 32) * 2^-23 * sum |x*w| of the exact sum, before the fp32
 * rounding), silu uses the library expf (a few fp32 ulps), so an element of z
 * may round to a neighbouring e4m3 code (and a block to the neighbouring
 * scale) where the exact value lies that close to a rounding boundary.
 *   cfg          quant EP_Q_MXFP8, layout EP_LAYOUT_PACKED, H % 128 == 0 and a
 *                multiple of 224, 256 or 128 (GMM2's column tiles);
 *                otherwise EP_ERR_UNSUPPORTED / EP_ERR_INVALID_ARG
 *   recv_buf     the dispatch's receive buffer (recv_bytes >= ep_sizes_t.recv_bytes)
 *   expert_offset, recv_count   from ep_dispatch_layout
 *   w1_codes     e4m3 [E][2I][H], w1_scales e8m0 [E][2I][H/32]
 *   w2_codes     e4m3 [E][H][I],  w2_scales e8m0 [E][H][I/32]
 *   inter        I, a multiple of 128, at most 8192
 *   z_buf        z_bytes >= ep_ffn_buffer_bytes(): the requantised z, e4m3
 *                [rows][I] then, at z_scale_offset, e8m0 [rows][I/32]
 *                (rows past recv_count not written)
 *   y            bf16 [rows][H] (y_bytes >= ep_sizes_t.expert_out_bytes): the
 *                input of ep_combine
 * All weight and buffer pointers 16-byte aligned (EP_ERR_MISALIGNED).  A wait
 * inside the kernels that exceeds 2 s sets EP_DEV_TIMEOUT; they never trap.
 */
ep_status_t ep_ffn_buffer_bytes(const ep_config_t *cfg, int32_t inter, int64_t *z_bytes,
                                int64_t *z_scale_offset);
ep_status_t ep_expert_ffn_mx(const ep_config_t *cfg, const void *recv_buf, size_t recv_bytes,
                             const int64_t *expert_offset, const int64_t *recv_count,
                             const uint8_t *w1_codes, const uint8_t *w1_scales,
                             const uint8_t *w2_codes, const uint8_t *w2_scales, int32_t inter,
                             void *z_buf, size_t z_bytes, uint16_t *y, size_t y_bytes,
                             uint32_t *dev_status, ep_stream_t stream);

/*
 * The page's whole forward path in one call ("[feat] A5 deep fused moe
 * supported": Dispatch, GMM1, SwiGLU, Requant, GMM2, Combine in one
 * operator): ep_dispatch_with_layout (MXFP8), ep_expert_ffn_mx, then
 * ep_combine of its bf16 outputs, launched back to back on `stream` with
 * programmatic dependent launch.  Every argument is checked before the first
 * launch; the result equals the calls made one by one.  Arguments as those
 * calls; cfg as ep_expert_ffn_mx (EP_F_COMBINE_QUANTIZED unsupported).
 */
ep_status_t ep_moe_forward_ffn(const ep_config_t *cfg, const uint16_t *x, const void *topk_idx,
                               const float *topk_weights, const uint8_t *w1_codes,
                               const uint8_t *w1_scales, const uint8_t *w2_codes,
                               const uint8_t *w2_scales, int32_t inter, int32_t *token_slot,
                               int64_t *recv_count, int64_t *expert_offset, void *workspace,
                               size_t workspace_bytes, void *recv_buf, size_t recv_bytes,
                               int32_t *src_info, size_t src_info_bytes, void *z_buf,
                               size_t z_bytes, uint16_t *y, size_t y_bytes, uint16_t *out,
                               uint32_t *dev_status, ep_stream_t stream);

/*
 * One call for the whole forward path with the experts between dispatch and
 * combine ("[feat] A5 deep fused moe supported": one operator runs the
 * dispatch, the experts' grouped matrix multiplications and the combine):
 * ep_dispatch_with_layout, then the experts' maps (ep_expert_gemm for
 * cfg->quant EP_Q_BF16, ep_expert_gemm_mx for EP_Q_MXFP8 / EP_Q_MXFP4) with
 * n_out = H, then ep_combine of their bf16 outputs.  The launches follow one
 * another on `stream` with programmatic dependent launch: each kernel's
 * set-up overlaps the previous kernel's tail.  Every argument is checked
 * before the first launch; the result equals the four calls made one by one.
 *   cfg          layout EP_LAYOUT_PACKED; quant EP_Q_BF16 (H % 256 == 0),
 *                EP_Q_MXFP8 (H % 128 == 0) or EP_Q_MXFP4 (H % 256 == 0);
 *                EP_F_COMBINE_QUANTIZED is not supported (EP_ERR_UNSUPPORTED)
 *   x, topk_idx, topk_weights    as ep_dispatch / ep_combine
 *   w_codes      bf16 [E][H][H] (w_scales NULL) or the MX codes [E][H][D]
 *   w_scales     e8m0 [E][H][H/32] for the MX formats
 *   token_slot, recv_count, expert_offset, workspace(_bytes)   as ep_dispatch_layout
 *   recv_buf(_bytes), src_info(_bytes)                          as ep_dispatch
 *   y            bf16 [rows][H]: the experts' outputs (scratch owned by the
 *                caller; y_bytes >= ep_sizes_t.expert_out_bytes)
 *   out          bf16 [N][H]
 * A wait inside the GEMM kernel that exceeds 2 s sets EP_DEV_TIMEOUT.
 */
ep_status_t ep_moe_forward(const ep_config_t *cfg, const uint16_t *x, const void *topk_idx,
                           const float *topk_weights, const void *w_codes,
                           const uint8_t *w_scales, int32_t *token_slot, int64_t *recv_count,
                           int64_t *expert_offset, void *workspace, size_t workspace_bytes,
                           void *recv_buf, size_t recv_bytes, int32_t *src_info,
                           size_t src_info_bytes, uint16_t *y, size_t y_bytes, uint16_t *out,
                           uint32_t *dev_status, ep_stream_t stream);

/*
 * Diagnostic of the bounded waits in the tensor-core kernels (ep_expert_gemm,
 * ep_expert_gemm_mx, ep_moe_forward): one block waits, with the helper those
 * kernels use, on a shared-memory barrier that nothing completes.  After 2 s
 * the wait gives up, EP_DEV_TIMEOUT is set in *dev_status and the kernel
 * returns; the context stays usable.  Takes about 2 s of one SM.
 *   dev_status   device uint32, read and cleared by ep_get_status
 */
ep_status_t ep_wait_probe(uint32_t *dev_status, ep_stream_t stream);

/*
 * Allocation-free variant of ep_dispatch_layout.  The pages have no
 * counterpart to this call; it exists for callers that cannot allocate
 * device memory when they route tokens -- for example a serving loop whose
 * device memory is reserved in full up front, or a plugin running inside a
 * host framework that owns every device allocation -- and so cannot provide
 * the `workspace` buffer.  Arguments and results are those of
 * ep_dispatch_layout without `workspace`; the multi-block layout kernels run
 * with their scratch in a static device array of EP_STATIC_SCRATCH_BYTES
 * inside this library (every GPU that loads the library holds it until the
 * process exits).  The caller still owns and passes all inputs and outputs.
 *   - A configuration whose ep_sizes_t.workspace_bytes exceeds
 *     EP_STATIC_SCRATCH_BYTES is rejected with EP_ERR_UNSUPPORTED before any
 *     launch.
 *   - The first call on a device looks up the array's device address with
 *     that device current (the device of `stream` must be the current
 *     device); make that first call before any stream capture.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind.  Each launch writes every scratch word it reads, so nothing has
 *     to start at zero; but calls that overlap on the GPU (different streams,
 *     or several host threads) race on the array: serialise them.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *     The array itself comes into being when CUDA loads this library's
 *     device code on a device, which under CUDA's default lazy loading is
 *     the first call into the library there.  A caller that reserves the
 *     whole device up front should make one call into the library per device
 *     first (for example this call on a tiny configuration), so that the
 *     array already exists when memory runs out.
 */
#define EP_STATIC_SCRATCH_BYTES (1u << 20)
ep_status_t ep_dispatch_layout_static(const ep_config_t *cfg, const void *topk_idx,
                                      int32_t *tokens_per_rank, int32_t *tokens_per_expert,
                                      uint8_t *is_token_in_rank, int32_t *token_slot,
                                      int64_t *recv_count, int64_t *expert_offset,
                                      int64_t *cumulative_recv_stats, uint32_t *dev_status,
                                      ep_stream_t stream);

/*
 * ---- Expert parallelism over G GPUs (one process per GPU, NVLink peer memory)
 * ("Low-Latency Mode API": each rank dispatches its tokens into the receive
 * buffers of the ranks that own their experts and combines the experts'
 * outputs back; "[Common][PyTorch] EP dispatch with unfused MXFP8
 * quantization", Changes: symmetric-memory windows, combine forward and
 * backward as the reverse of the dispatch.)
 *
 * Partitioning.  `cfg` describes the whole job (R ranks of T tokens, E
 * experts).  GPU g of G (R % G == 0) holds the tokens of ranks g*RG ..
 * (g+1)*RG - 1, RG = R/G (its N_loc = RG*T tokens: x, topk_idx, topk_weights,
 * token_slot and out are [N_loc] arrays), and owns experts g*EG .. (g+1)*EG - 1,
 * EG = E/G.  Every GPU has one window per buffer kind, all of ep_group_sizes()'s
 * `rows` rows in the single-GPU row format: receive window (data then scales),
 * source info, optional weights, expert outputs y, gradient window.  Rows are
 * numbered virtually: row r of GPU o's window is o*rows + r; expert_offset and
 * the padded addressing e*R*M + slot are virtual rows.  Slots are global
 * (ranked over all GPUs' entries of the expert in (source rank, token, k)
 * order), so every GPU's window holds what one GPU's buffer would hold for
 * those experts, row for row.
 *
 * One step, every GPU (epoch = 1, 2, ... one more each step; flags are never
 * reset), all of it in this library's kernels over peer memory:
 *   ep_group_layout      local ranks of this GPU's entries and its per-rank
 *                        counts, stored into every GPU's counts window
 *                        (signal COUNTS)
 *   ep_group_plan        waits for every GPU's counts, then global slots,
 *                        totals and virtual packed offsets
 *   ep_group_dispatch    quantise and store rows into the owners' windows;
 *                        the grid's last block signals every GPU (DISPATCH)
 *   ep_group_wait(DISPATCH)              every GPU's rows have arrived
 *   (the experts of this GPU write y in its window)
 *   ep_group_signal / wait(EXPERT_OUT)   every GPU's expert outputs are there
 *   ep_group_combine     read the tokens' rows from the owners' y windows
 *   ep_group_signal / wait(COMBINED)     windows may be reused next step
 * and for the backward: ep_group_combine_backward (stores into the owners'
 * gradient windows, signals BACKWARD), ep_group_wait(BACKWARD).
 * Waits are bounded: one that gives up sets EP_DEV_TIMEOUT, and ep_get_status
 * then returns EP_ERR_TIMEOUT; kernels never trap.  Windows of other GPUs
 * are mapped with ep_ipc_export / ep_ipc_import.  No transfer uses TMA
 * multicast; stores and loads to peers are plain 16-byte accesses.
 */
#define EP_GROUP_KIND_COUNTS 0
#define EP_GROUP_KIND_DISPATCH 1
#define EP_GROUP_KIND_EXPERT_OUT 2
#define EP_GROUP_KIND_COMBINED 3
#define EP_GROUP_KIND_BACKWARD 4
#define EP_GROUP_KINDS 5

typedef struct {
    int32_t world;       /* G, 1 .. 64, R % G == 0 */
    int32_t rank;        /* this GPU, 0 .. G-1 */
    uint64_t epoch;      /* step number, >= 1, the same on every GPU */
    int64_t window_rows; /* packed layout: rows of every window; 0 = room for every entry
                          * of the job (R*T*K + EG*(expert_align-1)).  Rows past a window
                          * are skipped with EP_DEV_CAPACITY_OVERFLOW.  Padded: 0 (the
                          * window is EG*R*M rows). */
} ep_group_t;

/* Every GPU's windows as this process sees them: device arrays of G device
 * pointers (entry g: GPU g's window, mapped into this process), written once
 * at set-up.  Window layouts as ep_group_sizes(). */
typedef struct {
    void *const *recv;            /* receive windows (data, then scales at recv_scale_offset) */
    int32_t *const *src_info;     /* int32 [rows]: global r*M + t of each row's token */
    float *const *recv_weights;   /* float [rows] or NULL (array pointer NULL: not written) */
    const void *const *y;         /* bf16 [rows][H] expert outputs */
    void *const *grad;            /* gradient windows (MXFP8, as ep_combine_backward) or NULL */
    int32_t *const *counts;       /* int32 [R][E] counts tables of every GPU */
    uint64_t *const *flags;       /* uint64 [EP_GROUP_KINDS][G] flag words of every GPU */
    int32_t *my_counts;           /* this GPU's counts table (its entry of `counts`) */
    uint64_t *my_flags;           /* this GPU's flag words (zero before the first step) */
    uint32_t *done;               /* uint32 [EP_GROUP_KINDS] block counters, zero before first use */
} ep_peers_t;

/* Sizes for GPU grp->rank: `rows` and every *_bytes of one window, the
 * workspace of ep_group_layout, token_slot_bytes of N_loc*K (no
 * is_token_in_rank over GPUs). */
ep_status_t ep_group_sizes(const ep_config_t *cfg, const ep_group_t *grp, ep_sizes_t *out);
/* This GPU's entries ranked within their experts (the single-GPU layout over
 * its RG ranks: token_slot int32 [N_loc][K] receives local ranks, which
 * ep_group_plan makes global) and its per-rank counts: rows g*RG .. of the
 * [R][E] counts table (tokens_per_expert of ep_dispatch_layout), written in
 * its own counts window and stored into every other GPU's, then the COUNTS
 * signal. */
ep_status_t ep_group_layout(const ep_config_t *cfg, const ep_group_t *grp,
                            const ep_peers_t *peers, const void *topk_idx, int32_t *token_slot,
                            void *workspace, size_t workspace_bytes, uint32_t *dev_status,
                            ep_stream_t stream);
/* Waits (bounded) for every GPU's COUNTS, then from the [R][E] table:
 * token_slot += the entries the ranks before this GPU's send to the same
 * expert; recv_count int64 [E] = entries of each expert over all GPUs;
 * expert_offset int64 [E+1] = virtual packed offsets (each owner's experts in
 * order, rounded up to expert_align; [E] = G*rows; required when packed);
 * cumulative_recv_stats [E] += recv_count of this GPU's experts (nullable).
 * workspace: 8*E bytes of scratch.  E <= 1024. */
ep_status_t ep_group_plan(const ep_config_t *cfg, const ep_group_t *grp,
                          const ep_peers_t *peers, const void *topk_idx, int32_t *token_slot,
                          int64_t *recv_count, int64_t *expert_offset,
                          int64_t *cumulative_recv_stats, void *workspace, size_t workspace_bytes,
                          uint32_t *dev_status, ep_stream_t stream);
/* The same plan on the host (host pointers, no device work): slot_base [E]
 * (the shift of this GPU's slots), recv_count [E], expert_offset [E+1]. */
ep_status_t ep_group_plan_host(const ep_config_t *cfg, const ep_group_t *grp,
                               const int32_t *tokens_per_expert_all, int64_t *slot_base,
                               int64_t *recv_count, int64_t *expert_offset);
/* ep_dispatch of this GPU's tokens into the owners' windows (peers->recv,
 * src_info, recv_weights), then the EP_GROUP_KIND_DISPATCH signal. */
ep_status_t ep_group_dispatch(const ep_config_t *cfg, const ep_group_t *grp,
                              const ep_peers_t *peers, const uint16_t *x, const void *topk_idx,
                              const float *topk_weights, const int32_t *token_slot,
                              const int64_t *expert_offset, uint32_t *dev_status,
                              ep_stream_t stream);
/* ep_combine of this GPU's tokens, reading each entry's bf16 row from its
 * owner's y window (EP_F_COMBINE_QUANTIZED unsupported). */
ep_status_t ep_group_combine(const ep_config_t *cfg, const ep_group_t *grp,
                             const ep_peers_t *peers, const void *topk_idx,
                             const float *topk_weights, const int32_t *token_slot,
                             const int64_t *expert_offset, uint16_t *out, uint32_t *dev_status,
                             ep_stream_t stream);
/* ep_combine_backward of this GPU's tokens into the owners' gradient
 * windows, then the EP_GROUP_KIND_BACKWARD signal. */
ep_status_t ep_group_combine_backward(const ep_config_t *cfg, const ep_group_t *grp,
                                      const ep_peers_t *peers, const uint16_t *g,
                                      const void *topk_idx, const float *topk_weights,
                                      const int32_t *token_slot, const int64_t *expert_offset,
                                      uint32_t *dev_status, ep_stream_t stream);
/* Tell every GPU that this GPU's work of `kind` for grp->epoch is done (its
 * earlier writes in stream order are visible to a GPU that sees the flag). */
ep_status_t ep_group_signal(const ep_group_t *grp, const ep_peers_t *peers, int32_t kind,
                            ep_stream_t stream);
/* Wait (on the device, in stream order) until every GPU has signalled `kind`
 * for grp->epoch; gives up after timeout_ns (0: 2 s; at most 10 s), sets
 * EP_DEV_TIMEOUT in *dev_status and returns. */
ep_status_t ep_group_wait(const ep_group_t *grp, const ep_peers_t *peers, int32_t kind,
                          uint64_t timeout_ns, uint32_t *dev_status, ep_stream_t stream);
/* CUDA IPC of windows: export gives the 64-byte handle of the allocation that
 * holds ptr and ptr's offset in it; import (in another process) maps it and
 * returns the same address's mapping; close unmaps (pass the mapping's base,
 * i.e. the imported pointer minus its offset). */
ep_status_t ep_ipc_export(const void *ptr, uint8_t *handle, uint64_t *offset);
ep_status_t ep_ipc_import(const uint8_t *handle, uint64_t offset, void **ptr);
ep_status_t ep_ipc_close(void *base);

/* Synchronise `stream`, read *dev_status into *host_flags (host pointer) and
 * clear it.  Returns EP_ERR_TIMEOUT when EP_DEV_TIMEOUT was set,
 * else EP_ERR_DEVICE_STATUS when any bit was set. */
ep_status_t ep_get_status(uint32_t *dev_status, uint32_t *host_flags, ep_stream_t stream);

/* Static description of a status code. */
const char *ep_status_string(ep_status_t status);

/* ---- diagnostics ---------------------------------------------------------
 * ep_copy: a plain 16-byte-vector device copy, the same-run HBM bandwidth
 * reference for the kernels above (bytes % 16 == 0, both pointers aligned).
 * ep_cvt_sweep: out[i] = the kernels' conversion of the binary32 value with
 * bit pattern start+i (format 0: e4m3 satfinite byte; 1: e2m1 satfinite code
 * in the low nibble; 2 and 3: the e8m0 byte X+127 of an MX block whose
 * maximum is |value|, for qmax 448 and 6), for checking the hardware
 * conversions and the exponent arithmetic against their definitions.
 * ep_kernel_launches: kernels launched by this library in this process. */
ep_status_t ep_copy(void *dst, const void *src, size_t bytes, ep_stream_t stream);
ep_status_t ep_cvt_sweep(int32_t format, uint32_t start, int64_t n, uint8_t *out,
                         ep_stream_t stream);
uint64_t ep_kernel_launches(void);

#ifdef __cplusplus
}
#endif
#endif /* EP_H */
