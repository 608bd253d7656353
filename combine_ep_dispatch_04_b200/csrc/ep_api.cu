// ep_api.cu -- the C ABI of libep (declared in include/ep.h): argument
// validation, buffer sizing and kernel selection.  Every hot step runs in the
// kernels of ep_layout.cuh, ep_dispatch.cuh and ep_combine.cuh.
#include <atomic>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>

#include "ep.h"
#include "ep_combine.cuh"
#include "ep_device.cuh"
#include "ep_dispatch.cuh"
#include "ep_gemm.cuh"
#include "ep_group.cuh"
#include "ep_layout.cuh"

namespace {

std::atomic<uint64_t> g_launches{0};

constexpr int kMaxExperts = 1024;
constexpr int kMaxHidden = 8192;
constexpr int64_t kIntLimit = (int64_t(1) << 31) - 1;
// Layout paths by routing size: one block up to kSingleMaxEntries entries, one
// thread-block cluster up to kClusterMaxEntries, three multi-block launches
// beyond.
constexpr int64_t kSingleMaxEntries = 2048;
constexpr int64_t kClusterMaxEntries = 131072;
constexpr size_t kDefaultSmem = 48 * 1024;
constexpr size_t kMaxSmem = 200 * 1024;
constexpr size_t kMaxSmemOptin = 227 * 1024;  // the GEMMs' rings

cudaStream_t cs(ep_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

// Launch with programmatic stream serialisation (see pdl_enter in
// ep_device.cuh): the kernel may begin while the previous grid on the stream
// drains, and waits for it before touching memory.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                   Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// A caller buffer of `have` bytes where `want` are needed ([IDX] Runtime
// Validation: sizes are checked before any GPU work).
ep_status_t need(size_t have, int64_t want) {
    return (int64_t)have >= want ? EP_OK : EP_ERR_BUFFER_TOO_SMALL;
}

ep_status_t launched() {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError() == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

// Derived quantities of a validated configuration.
struct Plan {
    int R, T, M, K, E, H, L;
    int64_t N, cap, rows, D, S, scale_off, recv_bytes, grad_scale_off, grad_bytes;
    int TC, CR, C;
    int64_t ws_bytes;
};

int64_t data_row_bytes(int quant, int H) {
    return quant == EP_Q_BF16 ? 2LL * H : (quant == EP_Q_MXFP4 ? H / 2 : H);
}
int64_t scale_row_bytes(int quant, int H, uint32_t flags) {
    switch (quant) {
    case EP_Q_BF16: return 0;
    case EP_Q_INT8_TOKEN: return 4;
    case EP_Q_E4M3_B128:  // fp32 per 128, or e8m0 bytes in whole int32 words
        return (flags & EP_F_UE8M0) ? 4LL * ((H / 128 + 3) / 4) : 4LL * (H / 128);
    default: return H / 32;
    }
}

// E4M3_B128 scale format: 0 = qmax/amax in fp32, 1 = power of two in fp32,
// 2 = e8m0 bytes.
int e4m3_scale_format(const ep_config_t *cfg) {
    if (cfg->quant != EP_Q_E4M3_B128) return 0;
    if (cfg->flags & EP_F_UE8M0) return 2;
    return (cfg->flags & EP_F_ROUND_SCALE) ? 1 : 0;
}

ep::TopkIdx topk_idx_view(const ep_config_t *cfg, const void *topk_idx) {
    return ep::TopkIdx{topk_idx, (cfg->flags & EP_F_IDX_I32) ? 1 : 0};
}

// Every check happens before any arithmetic that uses the values.
ep_status_t make_plan(const ep_config_t *c, Plan &p) {
    if (!c) return EP_ERR_INVALID_ARG;
    if (c->num_ranks <= 0 || c->max_tokens_per_rank <= 0 || c->num_tokens < 0 ||
        c->num_tokens > c->max_tokens_per_rank)
        return EP_ERR_INVALID_ARG;
    if (c->num_topk < 1 || c->num_topk > ep::kMaxTopk) return EP_ERR_INVALID_ARG;
    if (c->num_experts < 1 || c->num_experts > kMaxExperts) return EP_ERR_INVALID_ARG;
    if (c->num_experts % c->num_ranks != 0) return EP_ERR_INVALID_ARG;
    if (c->hidden < 32 || c->hidden > kMaxHidden || c->hidden % 32 != 0) return EP_ERR_INVALID_ARG;
    if (c->quant < EP_Q_BF16 || c->quant > EP_Q_MXFP4) return EP_ERR_INVALID_ARG;
    if (c->quant == EP_Q_E4M3_B128 && c->hidden % 128 != 0) return EP_ERR_INVALID_ARG;
    if (c->layout != EP_LAYOUT_PADDED && c->layout != EP_LAYOUT_PACKED) return EP_ERR_INVALID_ARG;
    if (c->expert_align < 1) return EP_ERR_INVALID_ARG;
    if (!(c->e4m3_qmax >= 0.0f && c->e4m3_qmax <= 448.0f)) return EP_ERR_INVALID_ARG;  // NaN fails
    const uint32_t paths = EP_F_LAYOUT_SINGLE_CTA | EP_F_LAYOUT_MULTI_CTA | EP_F_LAYOUT_CLUSTER;
    const uint32_t known = EP_F_BWD_UNWEIGHTED | EP_F_COMBINE_QUANTIZED | EP_F_IDX_I32 |
                           EP_F_ROUND_SCALE | EP_F_UE8M0 | EP_F_GEMM_CTA_PAIRS | paths;
    if (c->flags & ~known) return EP_ERR_INVALID_ARG;
    // power-of-two scales exist for the e4m3 / e2m1 formats only (MX scales
    // already are); e8m0 storage of the per-128 scales only for E4M3_B128
    if ((c->flags & EP_F_ROUND_SCALE) && (c->quant == EP_Q_BF16 || c->quant == EP_Q_INT8_TOKEN))
        return EP_ERR_INVALID_ARG;
    if ((c->flags & EP_F_UE8M0) && c->quant != EP_Q_E4M3_B128) return EP_ERR_INVALID_ARG;
    const uint32_t forced = c->flags & paths;
    if (forced & (forced - 1)) return EP_ERR_INVALID_ARG;  // at most one path flag

    p.R = c->num_ranks;
    p.T = c->num_tokens;
    p.M = c->max_tokens_per_rank;
    p.K = c->num_topk;
    p.E = c->num_experts;
    p.H = c->hidden;
    p.L = p.E / p.R;
    p.N = (int64_t)p.R * p.T;
    if (p.N * p.K > kIntLimit) return EP_ERR_INVALID_ARG;
    p.cap = (int64_t)p.R * p.M;
    if (c->layout == EP_LAYOUT_PADDED) {
        if (p.cap > kIntLimit) return EP_ERR_INVALID_ARG;  // slots are int32
        p.rows = (int64_t)p.E * p.cap;
    } else {
        if ((int64_t)c->expert_align > kIntLimit / p.E) return EP_ERR_INVALID_ARG;
        p.rows = p.N * p.K + (int64_t)p.E * (c->expert_align - 1);
        if (p.rows > kIntLimit) return EP_ERR_INVALID_ARG;  // expert_offset scan is int32 per tile
    }
    p.D = data_row_bytes(c->quant, p.H);
    p.S = scale_row_bytes(c->quant, p.H, c->flags);
    p.scale_off = round_up(p.rows * p.D, 256);
    p.recv_bytes = p.scale_off + p.rows * p.S;
    p.grad_scale_off = round_up(p.rows * p.H, 256);
    p.grad_bytes = p.grad_scale_off + p.rows * (p.H / 32);
    // layout chunks: whole tokens of one source rank, about 2048 entries each
    p.TC = (2048 + p.K - 1) / p.K;
    if (p.TC > p.T) p.TC = p.T > 0 ? p.T : 1;
    p.CR = (p.T + p.TC - 1) / p.TC;
    p.C = p.R * p.CR;
    p.ws_bytes = round_up((int64_t)(p.E + p.R) * p.C * 4, 256);
    if (p.ws_bytes == 0) p.ws_bytes = 256;
    return EP_OK;
}


struct ClusterChoice;
ep_status_t check_layout_args(const ep_config_t *, const Plan &, const void *, const int32_t *,
                              const int64_t *, const int64_t *, const void *, size_t,
                              const uint32_t *);
ep::LayoutArgs layout_args(const ep_config_t *, const Plan &, const void *, int32_t *, int32_t *,
                           uint8_t *, int32_t *, int64_t *, int64_t *, int64_t *, void *,
                           uint32_t *);
ep_status_t run_layout(const ep_config_t *, const Plan &, const ep::LayoutArgs &, cudaStream_t);

// ---- layout launch helpers -------------------------------------------------------
// The one-block layout cuts the N tokens into chunks of whole tokens of one
// source rank, about one chunk per warp (ceil(W/R) per rank).  Its shared
// memory holds the per-chunk counters (C*E ints), one mask word per warp and
// expert (W*E), the expert-to-rank table (E) and the staged keys (N*K), each
// part rounded up to a multiple of 4 ints.
struct SinglePlan {
    int warps, TC, CR, C;
    size_t smem;
    bool ok;
};

SinglePlan single_chunks(const Plan &p, int W) {
    SinglePlan sp{};
    sp.warps = W;
    sp.CR = (W + p.R - 1) / p.R;
    if (sp.CR > p.T) sp.CR = p.T > 0 ? p.T : 1;
    sp.TC = p.T > 0 ? (p.T + sp.CR - 1) / sp.CR : 1;
    sp.CR = p.T > 0 ? (p.T + sp.TC - 1) / sp.TC : 0;
    sp.C = p.R * sp.CR;
    auto r4 = [](int64_t v) { return (v + 3) & ~int64_t(3); };
    const int64_t ints = r4((int64_t)sp.C * p.E) + r4((int64_t)W * p.E) + r4(p.E) + r4(p.N * p.K);
    sp.smem = (size_t)ints * sizeof(int);
    sp.ok = sp.smem <= kMaxSmem;
    return sp;
}

SinglePlan plan_single(const Plan &p) {
    for (int W : {32, 16, 8, 4}) {
        const SinglePlan sp = single_chunks(p, W);
        if (sp.ok) return sp;
    }
    SinglePlan none{};
    return none;
}

// Kernels that may ask for more than the default 48 KB of shared memory get
// the larger limit once per device (the attribute is per function and device).
constexpr int kMaxDevices = 64;
std::atomic<uint32_t> g_smem_done[kMaxDevices];

template <typename Kernel>
bool allow_smem(Kernel k, int which, size_t bytes) {
    if (bytes <= kDefaultSmem) return true;
    if (bytes > kMaxSmemOptin) return false;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
    if (g_smem_done[dev].load() & (1u << which)) return true;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)std::max(bytes, kMaxSmem)) != cudaSuccess)
        return false;
    g_smem_done[dev].fetch_or(1u << which);
    return true;
}

ep_status_t launch_layout_single(ep::LayoutArgs a, const SinglePlan &sp, cudaStream_t s) {
    if (!sp.ok) return EP_ERR_UNSUPPORTED;
    a.TC = sp.TC;
    a.CR = sp.CR;
    a.C = sp.C;
    if (!allow_smem(ep::layout_single_kernel, 0, sp.smem)) return EP_ERR_CUDA;
    launch(ep::layout_single_kernel, 1, sp.warps * 32, sp.smem, s, a);
    return launched();
}

// One cluster of Q blocks of 512 threads: chunks of whole tokens of one
// source rank, about one per warp of the cluster, contiguous per block.
// Shared memory per block: [off: CPQ*E][tot: E][msk: W*E][rank_of: E][keys],
// each part rounded up to a multiple of 4 ints.
constexpr int kClusterThreads = 512;

struct ClusterChoice {
    bool ok;
    ep::ClusterPlan cp;
    size_t smem;
};

// Largest cluster size that can be resident (16 needs the non-portable
// attribute), checked once per device.
int cluster_size_limit() {
    static std::mutex mu;
    static int limit[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 8;
    std::lock_guard<std::mutex> lock(mu);
    if (limit[dev]) return limit[dev];
    int q = 8;
    if (cudaFuncSetAttribute(ep::layout_cluster_kernel,
                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
        cudaFuncSetAttribute(ep::layout_cluster_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxSmem) ==
            cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(16);
        cfg.blockDim = dim3(kClusterThreads);
        cfg.dynamicSmemBytes = kMaxSmem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 16;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, ep::layout_cluster_kernel, &cfg) == cudaSuccess &&
            n >= 1)
            q = 16;
    }
    cudaGetLastError();  // a refused query leaves no sticky error
    limit[dev] = q;
    return q;
}

ClusterChoice plan_cluster(const Plan &p) {
    const int W = kClusterThreads / 32;
    auto r4 = [](int64_t v) { return (v + 3) & ~int64_t(3); };
    for (int Q = cluster_size_limit(); Q >= 2; Q /= 2) {
        ep::ClusterPlan cp{};
        cp.Q = Q;
        int cr = (Q * W + p.R - 1) / p.R;
        if (cr > p.T) cr = p.T > 0 ? p.T : 1;
        cp.TC = p.T > 0 ? (p.T + cr - 1) / cr : 1;
        cp.CR = p.T > 0 ? (p.T + cp.TC - 1) / cp.TC : 0;
        cp.C = p.R * cp.CR;
        cp.CPQ = (cp.C + Q - 1) / Q;
        const int64_t ints = r4((int64_t)cp.CPQ * p.E) + r4(p.E) + r4((int64_t)W * p.E) + r4(p.E) +
                             r4((int64_t)cp.CPQ * cp.TC * p.K);
        const size_t smem = (size_t)ints * sizeof(int);
        if (smem <= kMaxSmem) return {true, cp, smem};
    }
    ClusterChoice none{};
    return none;
}

ep_status_t launch_layout_cluster(const ep::LayoutArgs &a, const ClusterChoice &cc,
                                  cudaStream_t s) {
    if (!cc.ok) return EP_ERR_UNSUPPORTED;
    if (cc.cp.Q > 8 &&
        cudaFuncSetAttribute(ep::layout_cluster_kernel,
                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
        return EP_ERR_CUDA;
    if (!allow_smem(ep::layout_cluster_kernel, 4, cc.smem)) return EP_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cc.cp.Q);
    cfg.blockDim = dim3(kClusterThreads);
    cfg.dynamicSmemBytes = cc.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cc.cp.Q;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaLaunchKernelEx(&cfg, ep::layout_cluster_kernel, a, cc.cp);
    return launched();
}

ep_status_t launch_layout_multi(const ep::LayoutArgs &a, const Plan &p, cudaStream_t s) {
    ep_status_t st;
    if (p.C > 0) {
        const size_t smem = (size_t)(p.TC * p.K + p.E + p.R) * sizeof(int);
        if (!allow_smem(ep::layout_count_kernel, 2, smem)) return EP_ERR_CUDA;
        launch(ep::layout_count_kernel, p.C, ep::kLayoutThreads, smem, s, a);
        if ((st = launched()) != EP_OK) return st;
    }
    launch(ep::layout_scan_kernel, p.E + p.R, ep::kLayoutThreads, 0, s, a);
    if ((st = launched()) != EP_OK) return st;
    const size_t smem = (size_t)(p.TC * p.K + 2 * (ep::kLayoutThreads / 32) * p.E) * sizeof(int);
    if (!allow_smem(ep::layout_assign_kernel, 3, smem)) return EP_ERR_CUDA;
    launch(ep::layout_assign_kernel, p.C > 0 ? p.C : 1, ep::kLayoutThreads, smem, s, a);
    return launched();
}

}  // namespace

extern "C" {

const char *ep_status_string(ep_status_t s) {
    switch (s) {
    case EP_OK: return "ok";
    case EP_ERR_INVALID_ARG: return "invalid argument";
    case EP_ERR_UNSUPPORTED: return "unsupported";
    case EP_ERR_MISALIGNED: return "buffer not 16-byte aligned";
    case EP_ERR_CUDA: return "CUDA runtime error";
    case EP_ERR_DEVICE_STATUS: return "device reported bad indices or capacity overflow";
    case EP_ERR_TIMEOUT: return "timed out";
    case EP_ERR_BUFFER_TOO_SMALL: return "a caller buffer is smaller than the configuration needs";
    }
    return "unknown status";
}

uint64_t ep_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

ep_status_t ep_buffer_sizes(const ep_config_t *cfg, ep_sizes_t *out) {
    Plan p;
    ep_status_t st = make_plan(cfg, p);
    if (st != EP_OK) return st;
    if (!out) return EP_ERR_INVALID_ARG;
    std::memset(out, 0, sizeof(*out));
    out->rows = p.rows;
    out->data_row_bytes = p.D;
    out->scale_row_bytes = p.S;
    out->recv_scale_offset = p.scale_off;
    out->recv_bytes = p.recv_bytes;
    out->src_info_bytes = p.rows * 4;
    out->recv_weights_bytes = p.rows * 4;
    out->expert_out_bytes = p.rows * p.H * 2;
    out->grad_scale_offset = p.grad_scale_off;
    out->grad_bytes = p.grad_bytes;
    out->workspace_bytes = p.ws_bytes;
    out->token_slot_bytes = p.N * p.K * 4;
    out->is_token_in_rank_bytes = p.N * p.R;
    return EP_OK;
}

ep_status_t ep_dispatch_layout(const ep_config_t *cfg, const void *topk_idx,
                               int32_t *tokens_per_rank, int32_t *tokens_per_expert,
                               uint8_t *is_token_in_rank, int32_t *token_slot,
                               int64_t *recv_count, int64_t *expert_offset,
                               int64_t *cumulative_recv_stats, void *workspace,
                               size_t workspace_bytes, uint32_t *dev_status, ep_stream_t stream) {
    Plan p;
    ep_status_t st = make_plan(cfg, p);
    if (st != EP_OK) return st;
    if ((st = check_layout_args(cfg, p, topk_idx, token_slot, recv_count, expert_offset, workspace,
                                workspace_bytes, dev_status)) != EP_OK)
        return st;
    const ep::LayoutArgs a =
        layout_args(cfg, p, topk_idx, tokens_per_rank, tokens_per_expert, is_token_in_rank,
                    token_slot, recv_count, expert_offset, cumulative_recv_stats, workspace, dev_status);
    return run_layout(cfg, p, a, cs(stream));
}

}  // extern "C"

namespace {

// Threads per token (TPT) and granules per thread (G).  When the grid can
// fit in one wave of resident blocks, take the largest TPT that does (few
// tokens -- decode -- then spread each row over up to 8 warps, and no second,
// partial wave doubles the tail); otherwise (many waves) the smallest TPT
// with G <= max_g.  TPT never exceeds the granule count by more than a warp.
struct Split {
    int tpt, gmax;
};

int pow2_at_least(int g) { return g <= 1 ? 1 : (g <= 2 ? 2 : (g <= 4 ? 4 : 8)); }

// Resident blocks per SM of a kernel, queried once per function and device.
int blocks_per_sm(const void *fn, int threads) {
    static std::mutex mu;
    static std::map<std::pair<const void *, int>, int> cache;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find({fn, dev});
    if (it != cache.end()) return it->second;
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, threads, 0) != cudaSuccess || nb < 1)
        nb = 1;
    cache[{fn, dev}] = nb;
    return nb;
}

int sm_count();

// `kernel_of(tpt, gmax)` returns the kernel instance (nullptr if none).
template <typename KernelOf>
Split split_rows(int64_t N, int ngran, int max_g, KernelOf kernel_of) {
    const int64_t sms = sm_count();
    for (int tpt = 256; tpt >= 32; tpt >>= 1) {
        if (tpt > 32 && tpt / 2 >= ngran) continue;  // more than a warp of idle threads
        const int g = (ngran + tpt - 1) / tpt;
        if (g > max_g) break;
        const int gmax = pow2_at_least(g);
        const void *fn = kernel_of(tpt, gmax);
        if (!fn) continue;
        const int threads = ep::block_threads(tpt);
        const int64_t ctas = (N + threads / tpt - 1) / (threads / tpt);
        if (ctas <= sms * blocks_per_sm(fn, threads)) return {tpt, gmax};
    }
    int tpt = 32;
    while (tpt < 256 && (ngran + tpt - 1) / tpt > max_g) tpt *= 2;
    return {tpt, pow2_at_least((ngran + tpt - 1) / tpt)};
}

unsigned grid_for(int64_t N, int tpt) {
    const int toks = ep::block_threads(tpt) / tpt;
    return (unsigned)((N + toks - 1) / toks);
}

// Instantiated (TPT, GMAX) pairs: every split_rows result for H <= 8192 with
// 16-element granules (dispatch, backward: at most 512) and 8-element
// granules (combine: at most 1024).
#define EP_SPLITS(X) X(32, 1) X(32, 2) X(32, 4) X(32, 8) X(64, 1) X(64, 2) X(64, 4) X(64, 8) \
    X(128, 1) X(128, 2) X(128, 4) X(128, 8) X(256, 1) X(256, 2) X(256, 4)

template <int MODE>
ep_status_t launch_dispatch(const ep::DispatchArgs &a, cudaStream_t s) {
    auto kernel_of = [](int t, int g) -> const void * {
#define EP_FN(T_, G_) if (t == T_ && g == G_) return (const void *)ep::dispatch_kernel<MODE, T_, G_>;
        EP_SPLITS(EP_FN)
#undef EP_FN
        return nullptr;
    };
    const Split sp = split_rows(a.N, a.H / 16, 8, kernel_of);
    const unsigned grid = grid_for(a.N, sp.tpt);
#define EP_CASE(T_, G_)                                                                     \
    if (sp.tpt == T_ && sp.gmax == G_) {                                                    \
        launch(ep::dispatch_kernel<MODE, T_, G_>, grid, ep::block_threads(T_), 0, s, a);     \
        return launched();                                                                  \
    }
    EP_SPLITS(EP_CASE)
#undef EP_CASE
    return EP_ERR_UNSUPPORTED;
}

// The backward quantises every entry separately (K scaled copies of the
// row), so its per-thread state grows with G: keep G <= 2 (about 60
// registers) for occupancy.
template <bool GROUP>
ep_status_t launch_combine_bwd_as(const ep::DispatchArgs &a, cudaStream_t s) {
    auto kernel_of = [](int t, int g) -> const void * {
#define EP_FN(T_, G_) \
    if (t == T_ && g == G_) return (const void *)ep::combine_bwd_kernel<T_, G_, GROUP>;
        EP_SPLITS(EP_FN)
#undef EP_FN
        return nullptr;
    };
    const Split sp = split_rows(a.N, a.H / 16, 2, kernel_of);
    const unsigned grid = grid_for(a.N, sp.tpt);
#define EP_CASE(T_, G_)                                                                        \
    if (sp.tpt == T_ && sp.gmax == G_) {                                                       \
        launch(ep::combine_bwd_kernel<T_, G_, GROUP>, grid, ep::block_threads(T_), 0, s, a);    \
        return launched();                                                                     \
    }
    EP_SPLITS(EP_CASE)
#undef EP_CASE
    return EP_ERR_UNSUPPORTED;
}

ep_status_t launch_combine_bwd(const ep::DispatchArgs &a, cudaStream_t s) {
    return a.peer_out ? launch_combine_bwd_as<true>(a, s) : launch_combine_bwd_as<false>(a, s);
}

ep::DispatchArgs dispatch_args(const ep_config_t *cfg, const Plan &p) {
    ep::DispatchArgs a;
    std::memset(&a, 0, sizeof(a));
    a.N = p.N; a.T = p.T; a.K = p.K; a.E = p.E; a.M = p.M; a.H = p.H;
    a.packed = cfg->layout == EP_LAYOUT_PACKED;
    a.cap = p.cap;
    a.rows = p.rows;
    a.qmax = cfg->e4m3_qmax > 0.0f ? cfg->e4m3_qmax : 448.0f;
    a.sfmt = e4m3_scale_format(cfg);
    return a;
}


// ---- argument checks and launch bodies shared by the entry points ----------------
ep_status_t check_layout_args(const ep_config_t *cfg, const Plan &p, const void *topk_idx,
                              const int32_t *token_slot, const int64_t *recv_count,
                              const int64_t *expert_offset, const void *workspace,
                              size_t workspace_bytes, const uint32_t *dev_status) {
    if (!recv_count || !workspace || !dev_status) return EP_ERR_INVALID_ARG;
    if (p.N > 0 && (!topk_idx || !token_slot)) return EP_ERR_INVALID_ARG;
    if (cfg->layout == EP_LAYOUT_PACKED && !expert_offset) return EP_ERR_INVALID_ARG;
    return need(workspace_bytes, p.ws_bytes);
}

ep::LayoutArgs layout_args(const ep_config_t *cfg, const Plan &p, const void *topk_idx,
                           int32_t *tokens_per_rank, int32_t *tokens_per_expert,
                           uint8_t *is_token_in_rank, int32_t *token_slot, int64_t *recv_count,
                           int64_t *expert_offset, int64_t *cumulative_recv_stats,
                           void *workspace, uint32_t *dev_status) {
    ep::LayoutArgs a;
    a.R = p.R; a.T = p.T; a.K = p.K; a.E = p.E; a.M = p.M; a.L = p.L;
    a.TC = p.TC; a.CR = p.CR; a.C = p.C;
    a.packed = cfg->layout == EP_LAYOUT_PACKED;
    a.align = cfg->expert_align;
    a.cap = p.cap;
    a.idx = topk_idx_view(cfg, topk_idx);
    a.tpr = tokens_per_rank;
    a.tpe = tokens_per_expert;
    a.itr = is_token_in_rank;
    a.slot = token_slot;
    a.recv_count = recv_count;
    a.eo = expert_offset;
    a.stats = cumulative_recv_stats;
    a.ws_hist = static_cast<int32_t *>(workspace);
    a.ws_rk = a.ws_hist ? a.ws_hist + (int64_t)p.E * p.C : nullptr;
    a.status = dev_status;
    return a;
}

// Layout path by routing size (or the path a flag forces).
ep_status_t run_layout(const ep_config_t *cfg, const Plan &p, const ep::LayoutArgs &a,
                       cudaStream_t s) {
    if (cfg->flags & EP_F_LAYOUT_SINGLE_CTA) return launch_layout_single(a, plan_single(p), s);
    if (cfg->flags & EP_F_LAYOUT_MULTI_CTA) return launch_layout_multi(a, p, s);
    if (cfg->flags & EP_F_LAYOUT_CLUSTER) return launch_layout_cluster(a, plan_cluster(p), s);
    const int64_t entries = p.N * p.K;
    if (entries <= kSingleMaxEntries) {
        const SinglePlan sp = plan_single(p);
        if (sp.ok) return launch_layout_single(a, sp, s);
    }
    if (entries <= kClusterMaxEntries) {
        const ClusterChoice cc = plan_cluster(p);
        if (cc.ok) return launch_layout_cluster(a, cc, s);
    }
    return launch_layout_multi(a, p, s);
}

ep_status_t check_dispatch_args(const ep_config_t *cfg, const Plan &p, const uint16_t *x,
                                const void *topk_idx, const float *topk_weights,
                                const int32_t *token_slot, const int64_t *expert_offset,
                                const void *recv_buf, size_t recv_bytes, const int32_t *src_info,
                                size_t src_info_bytes, const float *recv_weights,
                                size_t recv_weights_bytes) {
    if (!x || !topk_idx || !token_slot || !recv_buf || !src_info) return EP_ERR_INVALID_ARG;
    if (cfg->layout == EP_LAYOUT_PACKED && !expert_offset) return EP_ERR_INVALID_ARG;
    if (recv_weights && !topk_weights) return EP_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(recv_buf)) return EP_ERR_MISALIGNED;
    ep_status_t st;
    if ((st = need(recv_bytes, p.recv_bytes)) != EP_OK) return st;
    if ((st = need(src_info_bytes, p.rows * 4)) != EP_OK) return st;
    if (recv_weights && (st = need(recv_weights_bytes, p.rows * 4)) != EP_OK) return st;
    return EP_OK;
}

ep::DispatchArgs full_dispatch_args(const ep_config_t *cfg, const Plan &p, const uint16_t *x,
                                    const void *topk_idx, const float *topk_weights,
                                    const int32_t *token_slot, const int64_t *expert_offset,
                                    void *recv_buf, int32_t *src_info, float *recv_weights,
                                    uint32_t *dev_status) {
    ep::DispatchArgs a = dispatch_args(cfg, p);
    a.D = p.D; a.S = p.S; a.scale_off = p.scale_off;
    a.x = x; a.idx = topk_idx_view(cfg, topk_idx);
    a.wts = topk_weights; a.slot = token_slot; a.eo = expert_offset;
    a.out = static_cast<uint8_t *>(recv_buf);
    a.src_info = src_info;
    a.recv_w = recv_weights;
    a.status = dev_status;
    return a;
}

// Quantised expert outputs with K <= 8 and 4-byte aligned scale rows: the
// kernel that keeps the next granule's copies in flight (blocks of 128).
template <int QIN>
ep_status_t launch_combine_pipelined(const ep::CombineArgs &a, cudaStream_t s) {
    auto kernel_of = [](int t, int g) -> const void * {
#define EP_FN(T_, G_)                                                                      \
    if (T_ <= 128 && t == T_ && g == G_) return (const void *)ep::combine_q_kernel<(T_ <= 128 ? T_ : 128), G_, QIN>;
        EP_SPLITS(EP_FN)
#undef EP_FN
        return nullptr;
    };
    const Split sp = split_rows(a.N, a.H / ep::combine_granule(QIN), 8, kernel_of);
    const unsigned grid = grid_for(a.N, sp.tpt);
#define EP_CASE(T_, G_)                                                                     \
    if (T_ <= 128 && sp.tpt == T_ && sp.gmax == G_) {                                       \
        launch(ep::combine_q_kernel<(T_ <= 128 ? T_ : 128), G_, QIN>, grid, ep::block_threads(T_), 0, s, a); \
        return launched();                                                                  \
    }
    EP_SPLITS(EP_CASE)
#undef EP_CASE
    return EP_ERR_UNSUPPORTED;
}

// Granules of 16 bytes of expert output (combine_granule elements).
template <int QIN>
ep_status_t launch_combine(const ep::CombineArgs &a, cudaStream_t s) {
    if constexpr (QIN != ep::QIN_BF16) {
        // The pipelined kernel's shared-memory stages cap it near 900 threads an
        // SM; below about a million granules (decode-sized batches) the
        // register kernel's higher occupancy wins.  (Rows in other GPUs'
        // windows are read by the register kernel.)
        if (!a.peer_y && a.K <= ep::kPipeRows && a.S % 4 == 0 && a.S <= ep::kPipeScaleBytes &&
            a.N * (int64_t)(a.H / ep::combine_granule(QIN)) > ((int64_t)1 << 20))
            return launch_combine_pipelined<QIN>(a, s);
    }
    auto kernel_of = [](int t, int g) -> const void * {
#define EP_FN(T_, G_) if (t == T_ && g == G_) return (const void *)ep::combine_kernel<T_, G_, 8, QIN>;
        EP_SPLITS(EP_FN)
#undef EP_FN
        return nullptr;
    };
    const Split sp = split_rows(a.N, a.H / ep::combine_granule(QIN), 8, kernel_of);
    const unsigned grid = grid_for(a.N, sp.tpt);
#define EP_CASE(T_, G_)                                                                     \
    if (sp.tpt == T_ && sp.gmax == G_) {                                                    \
        launch(ep::combine_kernel<T_, G_, 8, QIN>, grid, ep::block_threads(T_), 0, s, a);     \
        return launched();                                                                  \
    }
    EP_SPLITS(EP_CASE)
#undef EP_CASE
    return EP_ERR_UNSUPPORTED;
}

ep_status_t run_dispatch(const ep_config_t *cfg, const ep::DispatchArgs &a, cudaStream_t s) {
    switch (cfg->quant) {
    case EP_Q_BF16: return launch_dispatch<ep::Q_BF16>(a, s);
    case EP_Q_E4M3_B128: return launch_dispatch<ep::Q_E4M3_B128>(a, s);
    case EP_Q_INT8_TOKEN: return launch_dispatch<ep::Q_INT8>(a, s);
    case EP_Q_MXFP8: return launch_dispatch<ep::Q_MXFP8>(a, s);
    default: return launch_dispatch<ep::Q_MXFP4>(a, s);
    }
}

}  // namespace

extern "C" {

ep_status_t ep_dispatch(const ep_config_t *cfg, const uint16_t *x, const void *topk_idx,
                        const float *topk_weights, const int32_t *token_slot,
                        const int64_t *expert_offset, void *recv_buf, size_t recv_bytes,
                        int32_t *src_info, size_t src_info_bytes, float *recv_weights,
                        size_t recv_weights_bytes, uint32_t *dev_status, ep_stream_t stream) {
    Plan p;
    ep_status_t st = make_plan(cfg, p);
    if (st != EP_OK) return st;
    if (!dev_status) return EP_ERR_INVALID_ARG;
    if (p.N == 0) return EP_OK;
    if ((st = check_dispatch_args(cfg, p, x, topk_idx, topk_weights, token_slot, expert_offset,
                                  recv_buf, recv_bytes, src_info, src_info_bytes, recv_weights,
                                  recv_weights_bytes)) != EP_OK)
        return st;
    ep::DispatchArgs a = full_dispatch_args(cfg, p, x, topk_idx, topk_weights, token_slot,
                                            expert_offset, recv_buf, src_info, recv_weights,
                                            dev_status);
    return run_dispatch(cfg, a, cs(stream));
}

ep_status_t ep_dispatch_with_layout(const ep_config_t *cfg, const uint16_t *x,
                                    const void *topk_idx, const float *topk_weights,
                                    int32_t *tokens_per_rank, int32_t *tokens_per_expert,
                                    uint8_t *is_token_in_rank, int32_t *token_slot,
                                    int64_t *recv_count, int64_t *expert_offset,
                                    int64_t *cumulative_recv_stats, void *workspace,
                                    size_t workspace_bytes, void *recv_buf, size_t recv_bytes,
                                    int32_t *src_info, size_t src_info_bytes, float *recv_weights,
                                    size_t recv_weights_bytes, uint32_t *dev_status,
                                    ep_stream_t stream) {
    Plan p;
    ep_status_t st = make_plan(cfg, p);
    if (st != EP_OK) return st;
    if ((st = check_layout_args(cfg, p, topk_idx, token_slot, recv_count, expert_offset, workspace,
                                workspace_bytes, dev_status)) != EP_OK)
        return st;
    if (p.N > 0 &&
        (st = check_dispatch_args(cfg, p, x, topk_idx, topk_weights, token_slot, expert_offset,
                                  recv_buf, recv_bytes, src_info, src_info_bytes, recv_weights,
                                  recv_weights_bytes)) != EP_OK)
        return st;
    cudaStream_t s = cs(stream);
    const ep::LayoutArgs la =
        layout_args(cfg, p, topk_idx, tokens_per_rank, tokens_per_expert, is_token_in_rank,
                    token_slot, recv_count, expert_offset, cumulative_recv_stats, workspace, dev_status);
    if ((st = run_layout(cfg, p, la, s)) != EP_OK) return st;
    if (p.N == 0) return EP_OK;
    ep::DispatchArgs a = full_dispatch_args(cfg, p, x, topk_idx, topk_weights, token_slot,
                                            expert_offset, recv_buf, src_info, recv_weights,
                                            dev_status);
    a.early = 1;  // the previous grid is the layout launched just above
    return run_dispatch(cfg, a, s);
}

ep_status_t ep_combine(const ep_config_t *cfg, const uint16_t *y, size_t y_bytes,
                       const void *topk_idx, const float *topk_weights, const int32_t *token_slot,
                       const int64_t *expert_offset, uint16_t *out, uint32_t *dev_status,
                       ep_stream_t stream) {
    Plan p;
    ep_status_t st = make_plan(cfg, p);
    if (st != EP_OK) return st;
    if (!dev_status) return EP_ERR_INVALID_ARG;
    if (p.N == 0) return EP_OK;
    if (!y || !topk_idx || !topk_weights || !token_slot || !out) return EP_ERR_INVALID_ARG;
    if (cfg->layout == EP_LAYOUT_PACKED && !expert_offset) return EP_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(out)) return EP_ERR_MISALIGNED;

    const int qin = (cfg->flags & EP_F_COMBINE_QUANTIZED) ? cfg->quant : EP_Q_BF16;
    if ((st = need(y_bytes, qin == EP_Q_BF16 ? p.rows * p.H * 2 : p.recv_bytes)) != EP_OK)
        return st;
    ep::CombineArgs a;
    std::memset(&a, 0, sizeof(a));
    a.N = p.N; a.K = p.K; a.E = p.E; a.H = p.H;
    a.packed = cfg->layout == EP_LAYOUT_PACKED;
    a.cap = p.cap; a.rows = p.rows;
    a.D = p.D; a.S = p.S; a.scale_off = p.scale_off;
    a.sfmt = e4m3_scale_format(cfg);
    a.y = y; a.idx = topk_idx_view(cfg, topk_idx);
    a.wts = topk_weights; a.slot = token_slot; a.eo = expert_offset;
    a.out = out; a.status = dev_status;
    cudaStream_t s = cs(stream);
    switch (qin) {
    case EP_Q_BF16: return launch_combine<ep::QIN_BF16>(a, s);
    case EP_Q_E4M3_B128: return launch_combine<ep::QIN_E4M3_B128>(a, s);
    case EP_Q_INT8_TOKEN: return launch_combine<ep::QIN_INT8>(a, s);
    case EP_Q_MXFP8: return launch_combine<ep::QIN_MXFP8>(a, s);
    default: return launch_combine<ep::QIN_MXFP4>(a, s);
    }
}

ep_status_t ep_combine_backward(const ep_config_t *cfg, const uint16_t *g,
                                const void *topk_idx, const float *topk_weights,
                                const int32_t *token_slot, const int64_t *expert_offset,
                                void *grad_buf, size_t grad_bytes, uint32_t *dev_status,
                                ep_stream_t stream) {
    Plan p;
    ep_status_t st = make_plan(cfg, p);
    if (st != EP_OK) return st;
    if (!dev_status) return EP_ERR_INVALID_ARG;
    if (p.N == 0) return EP_OK;
    const bool unweighted = (cfg->flags & EP_F_BWD_UNWEIGHTED) != 0;
    if (!g || !topk_idx || !token_slot || !grad_buf) return EP_ERR_INVALID_ARG;
    if (!unweighted && !topk_weights) return EP_ERR_INVALID_ARG;
    if (cfg->layout == EP_LAYOUT_PACKED && !expert_offset) return EP_ERR_INVALID_ARG;
    if (!aligned16(g) || !aligned16(grad_buf)) return EP_ERR_MISALIGNED;
    if ((st = need(grad_bytes, p.grad_bytes)) != EP_OK) return st;

    ep::DispatchArgs a = dispatch_args(cfg, p);
    a.D = p.H; a.S = p.H / 32; a.scale_off = p.grad_scale_off;
    a.unweighted = unweighted;
    a.x = g; a.idx = topk_idx_view(cfg, topk_idx);
    a.wts = topk_weights; a.slot = token_slot; a.eo = expert_offset;
    a.out = static_cast<uint8_t *>(grad_buf);
    a.status = dev_status;
    return launch_combine_bwd(a, cs(stream));
}

ep_status_t ep_combine_backward_weights(const ep_config_t *cfg, const uint16_t *g,
                                        const uint16_t *y, size_t y_bytes, const void *topk_idx,
                                        const int32_t *token_slot, const int64_t *expert_offset,
                                        float *topk_weights_grad, uint32_t *dev_status,
                                        ep_stream_t stream) {
    Plan p;
    ep_status_t st = make_plan(cfg, p);
    if (st != EP_OK) return st;
    if (!dev_status) return EP_ERR_INVALID_ARG;
    if (cfg->flags & EP_F_COMBINE_QUANTIZED) return EP_ERR_UNSUPPORTED;  // bf16 y only
    if (p.N == 0) return EP_OK;
    if (!g || !y || !topk_idx || !token_slot || !topk_weights_grad) return EP_ERR_INVALID_ARG;
    if (cfg->layout == EP_LAYOUT_PACKED && !expert_offset) return EP_ERR_INVALID_ARG;
    if (!aligned16(g) || !aligned16(y)) return EP_ERR_MISALIGNED;
    if ((st = need(y_bytes, p.rows * p.H * 2)) != EP_OK) return st;

    ep::WgradArgs a;
    a.N = p.N; a.K = p.K; a.E = p.E; a.H = p.H;
    a.packed = cfg->layout == EP_LAYOUT_PACKED;
    a.cap = p.cap; a.rows = p.rows;
    a.g = g; a.y = y; a.idx = topk_idx_view(cfg, topk_idx);
    a.slot = token_slot; a.eo = expert_offset;
    a.dw = topk_weights_grad; a.status = dev_status;
    auto kernel_of = [](int t, int gm) -> const void * {
#define EP_FN(T_, G_) if (t == T_ && gm == G_) return (const void *)ep::combine_wgrad_kernel<T_, G_>;
        EP_SPLITS(EP_FN)
#undef EP_FN
        return nullptr;
    };
    const Split sp = split_rows(a.N, a.H / 8, 8, kernel_of);
    const unsigned grid = grid_for(a.N, sp.tpt);
    cudaStream_t s = cs(stream);
#define EP_CASE(T_, G_)                                                                     \
    if (sp.tpt == T_ && sp.gmax == G_) {                                                    \
        launch(ep::combine_wgrad_kernel<T_, G_>, grid, ep::block_threads(T_), 0, s, a);     \
        return launched();                                                                  \
    }
    EP_SPLITS(EP_CASE)
#undef EP_CASE
    return EP_ERR_UNSUPPORTED;
}

// ---- the experts between dispatch and combine -----------------------------------
namespace {
using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                 const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                 const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link to
// the driver library)
EncodeTiled encode_tiled() {
    static EncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    });
    return fn;
}

// bf16 matrix [outer][inner] (rows of `inner` elements), tiles of 64 x
// box_rows, 128-byte swizzle (the layout the kernel's matrix descriptors describe)
bool bf16_tile_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer,
                   uint32_t box_rows) {
    const EncodeTiled enc = encode_tiled();
    if (!enc) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner * 2};
    const cuuint32_t box[2] = {(cuuint32_t)ep::kGemmBK, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// u8 matrix [outer][inner], tiles of 128 x box_rows, 128-byte swizzle
bool u8_tile_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer,
                 uint32_t box_rows) {
    const EncodeTiled enc = encode_tiled();
    if (!enc) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner};
    const cuuint32_t box[2] = {(cuuint32_t)ep::kMxBK, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// An MX operand of the maps: codes [rows][K bytes or K/2] and the e8m0 scales
// [rows][K/32] of the same rows.
struct MxOperand {
    const void *codes;
    const uint8_t *scales;
    int K;  // elements of a row
};

// one launch of the MX kernel (e4m3 or packed e2m1 codes) with tiles of BM
// rows and BN columns; GLU: the first layer of the gated MLP (n_out = 2I
// outputs of which the epilogue writes z = silu(gate) * up requantised to
// zc / zs, BN/2 of each half per tile)
extern "C++" template <int BN, bool FP4, bool GLU = false, int BM = ep::kGemmBM>
ep_status_t launch_gemm_mx(const Plan &p, const MxOperand &x, const int64_t *expert_offset,
                           const int64_t *recv_count, const uint8_t *w_codes,
                           const uint8_t *w_scales, int n_out, uint16_t *y, uint8_t *zc,
                           uint8_t *zs, uint32_t *dev_status, cudaStream_t s, int slot) {
    const uint64_t D = FP4 ? (uint64_t)x.K / 2 : (uint64_t)x.K;  // code bytes of a row
    constexpr int TN = GLU ? BN / 2 : BN;
    CUtensorMap ma, mb;
    if (!u8_tile_map(&ma, x.codes, D, (uint64_t)p.rows, ep::kGemmBM) ||
        !u8_tile_map(&mb, w_codes, D, (uint64_t)p.E * n_out, TN))
        return EP_ERR_CUDA;
    ep::MxArgs a;
    std::memset(&a, 0, sizeof(a));
    a.E = p.E; a.K = x.K; a.N = n_out; a.rows = p.rows;
    a.I = GLU ? n_out / 2 : 0;
    a.ntn = GLU ? a.I / TN : n_out / BN;
    a.eo = expert_offset; a.cnt = recv_count;
    a.xs = x.scales;
    a.ws = w_scales; a.y = y; a.zc = zc; a.zs = zs; a.status = dev_status;
    const size_t smem = ep::MxCfg<BN, FP4, BM>::smem();
    if (!allow_smem(ep::expert_gemm_mx_kernel<BN, FP4, GLU, BM>, slot, smem)) return EP_ERR_CUDA;
    launch(ep::expert_gemm_mx_kernel<BN, FP4, GLU, BM>, (unsigned)sm_count(), ep::kMxThreads, smem,
           s, ma, mb, a);
    return launched();
}

// Pairs of CTAs the two-CTA GEMM can hold resident at once (0: none, then
// the one-CTA kernel runs), asked of the occupancy calculator once per device.
int gemm_pairs() {
    static std::atomic<int> pairs[kMaxDevices];
    static std::atomic<bool> asked[kMaxDevices];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    if (asked[dev].load()) return pairs[dev].load();
    int n = 0;
    const size_t smem = ep::gemm2_smem_bytes();
    if (allow_smem(ep::expert_gemm2_kernel, 12, smem)) {
        cudaLaunchConfig_t lc = {};
        lc.gridDim = dim3(2 * (unsigned)(sm_count() / 2));
        lc.blockDim = dim3(ep::kGemmThreads);
        lc.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        lc.attrs = attr;
        lc.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, ep::expert_gemm2_kernel, &lc) != cudaSuccess) n = 0;
    }
    cudaGetLastError();  // a refused query leaves no sticky error
    n = std::max(0, std::min(n, sm_count() / 2));
    pairs[dev].store(n);
    asked[dev].store(true);
    return n;
}

// N tile of the MX kernels (0: none divides n_out).  Two accumulators of 224
// columns let a tile's epilogue overlap the next tile's MMAs, which matters
// where the weights stream past few rows (decode-sized experts); MXFP8 with
// at least 256 rows an expert on average takes one accumulator of 256
// columns, the most FLOPs per byte of A (measured faster there, not for
// MXFP4).  Otherwise 256, then 128, where 224 does not divide n_out.
// Average rows an expert from which 256-row tiles pay (measured on one B200:
// MXFP4 gains from 256 rows, MXFP8 from about twice that).
constexpr int64_t mx_tall_rows(bool fp4) { return fp4 ? 256 : 448; }

int mx_tile_n(int n_out, bool fp4 = false, int64_t rows_per_expert = 0) {
    if (rows_per_expert >= mx_tall_rows(fp4) && n_out % 224 == 0) return 224;
    if (!fp4 && rows_per_expert >= 256 && n_out % 256 == 0) return 256;
    for (int bn : {224, 256, 128})
        if (n_out % bn == 0) return bn;
    return 0;
}
// Row tiles of 256 (two M = 128 MMAs sharing each B tile: a third fewer
// operand bytes per FLOP than 128 x 224; a tile whose upper half holds no row
// runs as a 128-row tile) where the experts hold at least mx_tall_rows rows
// on average.  With 224 columns a half, the two halves fill 448 TMEM columns:
// one accumulator, so the epilogue does not overlap the next tile's MMAs.
int mx_tile_m(int bn, bool fp4, int64_t rows_per_expert) {
    return (bn == 224 && rows_per_expert >= mx_tall_rows(fp4)) ? 256 : ep::kGemmBM;
}

// The experts' maps: argument checks (EP_OK: a launch may follow, or there is
// nothing to do when p.N == 0), then the launches.  `w_scales` null selects
// the bf16 maps, else the MX ones (cfg->quant MXFP8 / MXFP4).
ep_status_t check_gemm_args(const ep_config_t *cfg, const Plan &p, bool mx, int n_out,
                            const void *recv_buf, size_t recv_bytes,
                            const int64_t *expert_offset, const int64_t *recv_count,
                            const void *w_codes, const void *w_scales, const void *y,
                            size_t y_bytes, const uint32_t *dev_status) {
    const bool fp4 = cfg->quant == EP_Q_MXFP4;
    if (cfg->layout != EP_LAYOUT_PACKED) return EP_ERR_UNSUPPORTED;
    if (mx) {
        if (cfg->quant != EP_Q_MXFP8 && !fp4) return EP_ERR_UNSUPPORTED;
        if (p.H % (fp4 ? 2 * ep::kMxBK : ep::kMxBK) != 0) return EP_ERR_UNSUPPORTED;
        if (n_out <= 0 || mx_tile_n(n_out) == 0) return EP_ERR_INVALID_ARG;
    } else {
        if (cfg->quant != EP_Q_BF16) return EP_ERR_UNSUPPORTED;
        if (p.H % ep::kGemmBK != 0) return EP_ERR_UNSUPPORTED;
        if (n_out < ep::kGemmBN || n_out % ep::kGemmBN != 0) return EP_ERR_INVALID_ARG;
    }
    if ((int64_t)n_out * p.E > kIntLimit || p.E > ep::kGemmMaxExperts) return EP_ERR_INVALID_ARG;
    if (!dev_status) return EP_ERR_INVALID_ARG;
    if (p.N == 0) return EP_OK;  // nothing to multiply (empty buffers may be null)
    if (!recv_buf || !expert_offset || !recv_count || !w_codes || !y || (mx && !w_scales))
        return EP_ERR_INVALID_ARG;
    if (!aligned16(recv_buf) || !aligned16(w_codes) || !aligned16(y) ||
        (mx && !aligned16(w_scales)))
        return EP_ERR_MISALIGNED;
    // the bf16 maps read the data region only; the MX maps also the scales after it
    ep_status_t st = need(recv_bytes, mx ? p.recv_bytes : p.rows * p.D);
    if (st != EP_OK) return st;
    return need(y_bytes, p.rows * (int64_t)n_out * 2);
}

ep_status_t run_gemm_bf16(const ep_config_t *cfg, const Plan &p, const void *recv_buf,
                          const int64_t *expert_offset, const int64_t *recv_count,
                          const uint16_t *weights, int n_out, uint16_t *y, uint32_t *dev_status,
                          cudaStream_t s) {
    ep::GemmArgs a;
    a.E = p.E; a.H = p.H; a.N = n_out; a.ntn = n_out / ep::kGemmBN;
    a.eo = expert_offset; a.cnt = recv_count; a.y = y; a.status = dev_status;
    const int pairs = (cfg->flags & EP_F_GEMM_CTA_PAIRS) ? gemm_pairs() : 0;
    if (pairs > 0) {
        CUtensorMap ma, mb;  // each CTA's halves: 128-row boxes
        if (!bf16_tile_map(&ma, recv_buf, (uint64_t)p.H, (uint64_t)p.rows, 128) ||
            !bf16_tile_map(&mb, weights, (uint64_t)p.H, (uint64_t)p.E * n_out, 128))
            return EP_ERR_CUDA;
        const size_t smem2 = ep::gemm2_smem_bytes();
        if (!allow_smem(ep::expert_gemm2_kernel, 12, smem2)) return EP_ERR_CUDA;
        cudaLaunchConfig_t lc = {};
        lc.gridDim = dim3(2 * pairs);
        lc.blockDim = dim3(ep::kGemmThreads);
        lc.dynamicSmemBytes = smem2;
        lc.stream = s;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        lc.attrs = attr;
        lc.numAttrs = 2;
        cudaLaunchKernelEx(&lc, ep::expert_gemm2_kernel, ma, mb, a);
        return launched();
    }
    CUtensorMap ma, mb;
    if (!bf16_tile_map(&ma, recv_buf, (uint64_t)p.H, (uint64_t)p.rows, ep::kGemmBM) ||
        !bf16_tile_map(&mb, weights, (uint64_t)p.H, (uint64_t)p.E * n_out, ep::kGemmBN))
        return EP_ERR_CUDA;
    const size_t smem = ep::gemm_smem_bytes();
    if (!allow_smem(ep::expert_gemm_kernel, 5, smem)) return EP_ERR_CUDA;
    launch(ep::expert_gemm_kernel, (unsigned)sm_count(), ep::kGemmThreads, smem, s, ma, mb, a);
    return launched();
}

ep_status_t run_gemm_mx(const ep_config_t *cfg, const Plan &p, const void *recv_buf,
                        const int64_t *expert_offset, const int64_t *recv_count,
                        const uint8_t *w_codes, const uint8_t *w_scales, int n_out, uint16_t *y,
                        uint32_t *dev_status, cudaStream_t s, const MxOperand *x_in = nullptr) {
    const bool fp4 = cfg->quant == EP_Q_MXFP4;
    const int bn = mx_tile_n(n_out, fp4, p.N * p.K / p.E);
    const int bm = mx_tile_m(bn, fp4, p.N * p.K / p.E);
    const MxOperand x = x_in ? *x_in
                             : MxOperand{recv_buf,
                                         static_cast<const uint8_t *>(recv_buf) + p.scale_off,
                                         p.H};
#define EP_MX(BN_, FP4_, SLOT_, ...)                                                         \
    return launch_gemm_mx<BN_, FP4_, false, ##__VA_ARGS__>(p, x, expert_offset, recv_count, w_codes, \
                                                       w_scales, n_out, y, nullptr, nullptr,      \
                                                       dev_status, s, SLOT_)
    if (bm == 256) {
        if (fp4) EP_MX(224, true, 15, 256);
        EP_MX(224, false, 16, 256);
    }
    if (fp4) {
        if (bn == 224) EP_MX(224, true, 9);
        if (bn == 256) EP_MX(256, true, 10);
        EP_MX(128, true, 11);
    }
    if (bn == 224) EP_MX(224, false, 6);
    if (bn == 256) EP_MX(256, false, 7);
    EP_MX(128, false, 8);
#undef EP_MX
}
}  // namespace

ep_status_t ep_expert_gemm(const ep_config_t *cfg, const void *recv_buf, size_t recv_bytes,
                           const int64_t *expert_offset, const int64_t *recv_count,
                           const uint16_t *weights, int32_t n_out, uint16_t *y, size_t y_bytes,
                           uint32_t *dev_status, ep_stream_t stream) {
    Plan p;
    ep_status_t st = make_plan(cfg, p);
    if (st != EP_OK) return st;
    if ((st = check_gemm_args(cfg, p, false, n_out, recv_buf, recv_bytes, expert_offset,
                              recv_count, weights, nullptr, y, y_bytes, dev_status)) != EP_OK ||
        p.N == 0)
        return st;
    return run_gemm_bf16(cfg, p, recv_buf, expert_offset, recv_count, weights, n_out, y,
                         dev_status, cs(stream));
}

ep_status_t ep_expert_gemm_mx(const ep_config_t *cfg, const void *recv_buf, size_t recv_bytes,
                              const int64_t *expert_offset, const int64_t *recv_count,
                              const uint8_t *w_codes, const uint8_t *w_scales, int32_t n_out,
                              uint16_t *y, size_t y_bytes, uint32_t *dev_status,
                              ep_stream_t stream) {
    Plan p;
    ep_status_t st = make_plan(cfg, p);
    if (st != EP_OK) return st;
    if ((st = check_gemm_args(cfg, p, true, n_out, recv_buf, recv_bytes, expert_offset,
                              recv_count, w_codes, w_scales, y, y_bytes, dev_status)) != EP_OK ||
        p.N == 0)
        return st;
    return run_gemm_mx(cfg, p, recv_buf, expert_offset, recv_count, w_codes, w_scales, n_out, y,
                       dev_status, cs(stream));
}

// ---- the experts' gated MLP ----------------------------------------------------
namespace {
// z buffer of the gated MLP: e4m3 codes [rows][I], then at a 256-byte aligned
// offset the e8m0 scales [rows][I/32]
int64_t ffn_z_scale_offset(const Plan &p, int I) { return round_up(p.rows * I, 256); }
int64_t ffn_z_bytes(const Plan &p, int I) { return ffn_z_scale_offset(p, I) + p.rows * (I / 32); }

ep_status_t check_ffn_args(const ep_config_t *cfg, const Plan &p, int I, const void *recv_buf,
                           size_t recv_bytes, const int64_t *expert_offset,
                           const int64_t *recv_count, const uint8_t *w1c, const uint8_t *w1s,
                           const uint8_t *w2c, const uint8_t *w2s, const void *z_buf,
                           size_t z_bytes, const void *y, size_t y_bytes,
                           const uint32_t *dev_status) {
    if (cfg->quant != EP_Q_MXFP8 || cfg->layout != EP_LAYOUT_PACKED) return EP_ERR_UNSUPPORTED;
    if (p.H % ep::kMxBK != 0) return EP_ERR_UNSUPPORTED;
    if (I <= 0 || I % ep::kMxBK != 0 || I > kMaxHidden) return EP_ERR_INVALID_ARG;
    if (mx_tile_n(p.H) == 0) return EP_ERR_INVALID_ARG;
    if ((int64_t)2 * I * p.E > kIntLimit || (int64_t)p.H * p.E > kIntLimit ||
        p.E > ep::kGemmMaxExperts)
        return EP_ERR_INVALID_ARG;
    if (!dev_status) return EP_ERR_INVALID_ARG;
    if (p.N == 0) return EP_OK;
    if (!recv_buf || !expert_offset || !recv_count || !w1c || !w1s || !w2c || !w2s || !z_buf ||
        !y)
        return EP_ERR_INVALID_ARG;
    if (!aligned16(recv_buf) || !aligned16(w1c) || !aligned16(w1s) || !aligned16(w2c) ||
        !aligned16(w2s) || !aligned16(z_buf) || !aligned16(y))
        return EP_ERR_MISALIGNED;
    ep_status_t st;
    if ((st = need(recv_bytes, p.recv_bytes)) != EP_OK) return st;
    if ((st = need(z_bytes, ffn_z_bytes(p, I))) != EP_OK) return st;
    return need(y_bytes, p.rows * p.H * 2);
}

// GMM1 with SwiGLU and the requant in its epilogue (tiles of 128 gate + 128 up
// columns where the experts average 256 rows or more, else 64 + 64 with two
// accumulators so that a tile's epilogue overlaps the next tile's MMAs), then
// GMM2 on the requantised z.
ep_status_t run_ffn(const Plan &p, int I, const void *recv_buf, const int64_t *expert_offset,
                    const int64_t *recv_count, const uint8_t *w1c, const uint8_t *w1s,
                    const uint8_t *w2c, const uint8_t *w2s, void *z_buf, uint16_t *y,
                    uint32_t *dev_status, cudaStream_t s) {
    uint8_t *zc = static_cast<uint8_t *>(z_buf);
    uint8_t *zs = zc + ffn_z_scale_offset(p, I);
    const MxOperand x{recv_buf, static_cast<const uint8_t *>(recv_buf) + p.scale_off, p.H};
    // GMM1 tiles: 256 columns (128 gate + 128 up, one accumulator) for experts of
    // 256 rows and more; else 192 (96 + 96) where I allows, which keeps two
    // accumulators (the SwiGLU epilogue overlaps the next tile's MMAs) with a
    // quarter fewer operand bytes per FLOP than 128-column tiles
    const bool wide = p.N * p.K / p.E >= 256 && I % 128 == 0;
    ep_status_t st;
    if (wide)
        st = launch_gemm_mx<256, false, true>(p, x, expert_offset, recv_count, w1c, w1s, 2 * I,
                                              nullptr, zc, zs, dev_status, s, 13);
    else if (I % 96 == 0)
        st = launch_gemm_mx<192, false, true>(p, x, expert_offset, recv_count, w1c, w1s, 2 * I,
                                              nullptr, zc, zs, dev_status, s, 17);
    else
        st = launch_gemm_mx<128, false, true>(p, x, expert_offset, recv_count, w1c, w1s, 2 * I,
                                              nullptr, zc, zs, dev_status, s, 14);
    if (st != EP_OK) return st;
    const MxOperand z{zc, zs, I};
    ep_config_t c2 = {};
    c2.quant = EP_Q_MXFP8;
    return run_gemm_mx(&c2, p, nullptr, expert_offset, recv_count, w2c, w2s, p.H, y, dev_status,
                       s, &z);
}
}  // namespace

ep_status_t ep_ffn_buffer_bytes(const ep_config_t *cfg, int32_t inter, int64_t *z_bytes,
                                int64_t *z_scale_offset) {
    Plan p;
    ep_status_t st = make_plan(cfg, p);
    if (st != EP_OK) return st;
    if (inter <= 0 || inter % ep::kMxBK != 0 || inter > kMaxHidden || !z_bytes)
        return EP_ERR_INVALID_ARG;
    *z_bytes = ffn_z_bytes(p, inter);
    if (z_scale_offset) *z_scale_offset = ffn_z_scale_offset(p, inter);
    return EP_OK;
}

ep_status_t ep_expert_ffn_mx(const ep_config_t *cfg, const void *recv_buf, size_t recv_bytes,
                             const int64_t *expert_offset, const int64_t *recv_count,
                             const uint8_t *w1_codes, const uint8_t *w1_scales,
                             const uint8_t *w2_codes, const uint8_t *w2_scales, int32_t inter,
                             void *z_buf, size_t z_bytes, uint16_t *y, size_t y_bytes,
                             uint32_t *dev_status, ep_stream_t stream) {
    Plan p;
    ep_status_t st = make_plan(cfg, p);
    if (st != EP_OK) return st;
    if ((st = check_ffn_args(cfg, p, inter, recv_buf, recv_bytes, expert_offset, recv_count,
                             w1_codes, w1_scales, w2_codes, w2_scales, z_buf, z_bytes, y, y_bytes,
                             dev_status)) != EP_OK ||
        p.N == 0)
        return st;
    return run_ffn(p, inter, recv_buf, expert_offset, recv_count, w1_codes, w1_scales, w2_codes,
                   w2_scales, z_buf, y, dev_status, cs(stream));
}

ep_status_t ep_moe_forward_ffn(const ep_config_t *cfg, const uint16_t *x, const void *topk_idx,
                               const float *topk_weights, const uint8_t *w1_codes,
                               const uint8_t *w1_scales, const uint8_t *w2_codes,
                               const uint8_t *w2_scales, int32_t inter, int32_t *token_slot,
                               int64_t *recv_count, int64_t *expert_offset, void *workspace,
                               size_t workspace_bytes, void *recv_buf, size_t recv_bytes,
                               int32_t *src_info, size_t src_info_bytes, void *z_buf,
                               size_t z_bytes, uint16_t *y, size_t y_bytes, uint16_t *out,
                               uint32_t *dev_status, ep_stream_t stream) {
    Plan p;
    ep_status_t st = make_plan(cfg, p);
    if (st != EP_OK) return st;
    if (cfg->flags & EP_F_COMBINE_QUANTIZED) return EP_ERR_UNSUPPORTED;  // y is bf16 here
    // every argument is checked before the first launch
    if ((st = check_layout_args(cfg, p, topk_idx, token_slot, recv_count, expert_offset, workspace,
                                workspace_bytes, dev_status)) != EP_OK)
        return st;
    if ((st = check_ffn_args(cfg, p, inter, recv_buf, recv_bytes, expert_offset, recv_count,
                             w1_codes, w1_scales, w2_codes, w2_scales, z_buf, z_bytes, y, y_bytes,
                             dev_status)) != EP_OK)
        return st;
    if (p.N > 0) {
        if ((st = check_dispatch_args(cfg, p, x, topk_idx, topk_weights, token_slot,
                                      expert_offset, recv_buf, recv_bytes, src_info,
                                      src_info_bytes, nullptr, 0)) != EP_OK)
            return st;
        if (!topk_weights || !out) return EP_ERR_INVALID_ARG;
        if (!aligned16(out)) return EP_ERR_MISALIGNED;
    }
    if ((st = ep_dispatch_with_layout(cfg, x, topk_idx, topk_weights, nullptr, nullptr, nullptr,
                                      token_slot, recv_count, expert_offset, nullptr, workspace,
                                      workspace_bytes, recv_buf, recv_bytes, src_info,
                                      src_info_bytes, nullptr, 0, dev_status, stream)) != EP_OK ||
        p.N == 0)
        return st;
    if ((st = run_ffn(p, inter, recv_buf, expert_offset, recv_count, w1_codes, w1_scales,
                      w2_codes, w2_scales, z_buf, y, dev_status, cs(stream))) != EP_OK)
        return st;
    return ep_combine(cfg, y, y_bytes, topk_idx, topk_weights, token_slot, expert_offset, out,
                      dev_status, stream);
}

ep_status_t ep_moe_forward(const ep_config_t *cfg, const uint16_t *x, const void *topk_idx,
                           const float *topk_weights, const void *w_codes,
                           const uint8_t *w_scales, int32_t *token_slot, int64_t *recv_count,
                           int64_t *expert_offset, void *workspace, size_t workspace_bytes,
                           void *recv_buf, size_t recv_bytes, int32_t *src_info,
                           size_t src_info_bytes, uint16_t *y, size_t y_bytes, uint16_t *out,
                           uint32_t *dev_status, ep_stream_t stream) {
    Plan p;
    ep_status_t st = make_plan(cfg, p);
    if (st != EP_OK) return st;
    if (cfg->flags & EP_F_COMBINE_QUANTIZED) return EP_ERR_UNSUPPORTED;  // y is bf16 here
    const bool mx = cfg->quant != EP_Q_BF16;
    // every argument is checked before the first launch
    if ((st = check_layout_args(cfg, p, topk_idx, token_slot, recv_count, expert_offset, workspace,
                                workspace_bytes, dev_status)) != EP_OK)
        return st;
    if ((st = check_gemm_args(cfg, p, mx, p.H, recv_buf, recv_bytes, expert_offset, recv_count,
                              w_codes, w_scales, y, y_bytes, dev_status)) != EP_OK)
        return st;
    if (p.N > 0) {
        if ((st = check_dispatch_args(cfg, p, x, topk_idx, topk_weights, token_slot,
                                      expert_offset, recv_buf, recv_bytes, src_info,
                                      src_info_bytes, nullptr, 0)) != EP_OK)
            return st;
        if (!topk_weights || !out) return EP_ERR_INVALID_ARG;
        if (!aligned16(out)) return EP_ERR_MISALIGNED;
    }
    if ((st = ep_dispatch_with_layout(cfg, x, topk_idx, topk_weights, nullptr, nullptr, nullptr,
                                      token_slot, recv_count, expert_offset, nullptr, workspace,
                                      workspace_bytes, recv_buf, recv_bytes, src_info,
                                      src_info_bytes, nullptr, 0, dev_status, stream)) != EP_OK ||
        p.N == 0)
        return st;
    const cudaStream_t s = cs(stream);
    st = mx ? run_gemm_mx(cfg, p, recv_buf, expert_offset, recv_count,
                          static_cast<const uint8_t *>(w_codes), w_scales, p.H, y, dev_status, s)
            : run_gemm_bf16(cfg, p, recv_buf, expert_offset, recv_count,
                            static_cast<const uint16_t *>(w_codes), p.H, y, dev_status, s);
    if (st != EP_OK) return st;
    return ep_combine(cfg, y, y_bytes, topk_idx, topk_weights, token_slot, expert_offset, out,
                      dev_status, stream);
}

// ---- expert parallelism over GPUs (ep_group.cuh) ---------------------------------
}  // extern "C"
namespace {

// The group's shape from the global configuration: GPU g holds ranks
// g*RG .. (g+1)*RG - 1 and owns experts g*EG .. (g+1)*EG - 1.  A window holds
// every row its experts can receive: EG * R * M (padded) or all N * K entries
// plus the alignment of its experts (packed).
ep_status_t make_group(const ep_config_t *cfg, const ep_group_t *grp, Plan &p,
                       ep::GroupShape &s) {
    ep_status_t st = make_plan(cfg, p);
    if (st != EP_OK) return st;
    if (!grp || grp->world < 1 || grp->world > ep::kGroupMaxGpus || grp->rank < 0 ||
        grp->rank >= grp->world || p.R % grp->world != 0)
        return EP_ERR_INVALID_ARG;
    if (cfg->flags & (EP_F_LAYOUT_SINGLE_CTA | EP_F_LAYOUT_MULTI_CTA | EP_F_LAYOUT_CLUSTER))
        return EP_ERR_INVALID_ARG;
    s.R = p.R; s.E = p.E; s.G = grp->world; s.g = grp->rank;
    s.RG = p.R / s.G; s.EG = p.E / s.G;
    if (cfg->layout == EP_LAYOUT_PACKED) {  // every entry, unless the caller sizes it
        const int64_t all = p.N * p.K + (int64_t)s.EG * (cfg->expert_align - 1);
        if (grp->window_rows < 0) return EP_ERR_INVALID_ARG;
        s.win_rows = grp->window_rows > 0 ? std::min(grp->window_rows, all) : all;
    } else {  // the padded addressing fixes it
        s.win_rows = (int64_t)s.EG * p.cap;
        if (grp->window_rows != 0 && grp->window_rows != s.win_rows) return EP_ERR_INVALID_ARG;
    }
    if ((int64_t)s.G * s.win_rows > kIntLimit) return EP_ERR_INVALID_ARG;  // int32 slots
    return EP_OK;
}

// the configuration of this GPU's own tokens: RG ranks, packed (no capacity:
// the local ranks of the entries are all the layout is run for)
ep_config_t local_config(const ep_config_t *cfg, const ep::GroupShape &s) {
    ep_config_t c = *cfg;
    c.num_ranks = s.RG;
    c.layout = EP_LAYOUT_PACKED;
    c.expert_align = 1;
    return c;
}

int64_t group_ws_bytes(const ep_config_t *cfg, const ep::GroupShape &s) {
    const ep_config_t lc = local_config(cfg, s);
    Plan lp;
    if (make_plan(&lc, lp) != EP_OK) return -1;
    // + the local layout's expert_offset and recv_count (scratch)
    return lp.ws_bytes + round_up((int64_t)(2 * s.E + 1) * 8, 256);
}

bool peers_ok(const ep_peers_t *pe) { return pe && pe->flags && pe->my_flags && pe->done; }

bool group_ok(const ep_group_t *grp) {
    return grp && grp->world >= 1 && grp->world <= ep::kGroupMaxGpus && grp->rank >= 0 &&
           grp->rank < grp->world && grp->epoch > 0;
}

}  // namespace
extern "C" {

ep_status_t ep_group_sizes(const ep_config_t *cfg, const ep_group_t *grp, ep_sizes_t *out) {
    Plan p;
    ep::GroupShape s;
    ep_status_t st = make_group(cfg, grp, p, s);
    if (st != EP_OK) return st;
    if (!out) return EP_ERR_INVALID_ARG;
    const int64_t rows = s.win_rows;
    std::memset(out, 0, sizeof(*out));
    out->rows = rows;
    out->data_row_bytes = p.D;
    out->scale_row_bytes = p.S;
    out->recv_scale_offset = round_up(rows * p.D, 256);
    out->recv_bytes = out->recv_scale_offset + rows * p.S;
    out->src_info_bytes = rows * 4;
    out->recv_weights_bytes = rows * 4;
    out->expert_out_bytes = rows * p.H * 2;
    out->grad_scale_offset = round_up(rows * p.H, 256);
    out->grad_bytes = out->grad_scale_offset + rows * (p.H / 32);
    out->workspace_bytes = group_ws_bytes(cfg, s);
    out->token_slot_bytes = (int64_t)s.RG * p.T * p.K * 4;
    out->is_token_in_rank_bytes = 0;  // not produced over GPUs
    return EP_OK;
}

ep_status_t ep_group_layout(const ep_config_t *cfg, const ep_group_t *grp,
                            const ep_peers_t *peers, const void *topk_idx, int32_t *token_slot,
                            void *workspace, size_t workspace_bytes, uint32_t *dev_status,
                            ep_stream_t stream) {
    Plan p;
    ep::GroupShape s;
    ep_status_t st = make_group(cfg, grp, p, s);
    if (st != EP_OK) return st;
    if (!group_ok(grp) || !peers_ok(peers) || !peers->counts || !peers->my_counts || !workspace ||
        !dev_status)
        return EP_ERR_INVALID_ARG;
    // this GPU's rows of the [R][E] counts table, in its own counts window
    int32_t *tokens_per_expert = peers->my_counts + (int64_t)s.g * s.RG * s.E;
    if ((st = need(workspace_bytes, group_ws_bytes(cfg, s))) != EP_OK) return st;
    const ep_config_t lc = local_config(cfg, s);
    Plan lp;
    if ((st = make_plan(&lc, lp)) != EP_OK) return st;
    if (lp.N > 0 && (!topk_idx || !token_slot)) return EP_ERR_INVALID_ARG;
    // local ranks, per-rank counts and (scratch) local counts and offsets
    int64_t *eo_loc = reinterpret_cast<int64_t *>(static_cast<uint8_t *>(workspace) + lp.ws_bytes);
    int64_t *cnt_loc = eo_loc + (s.E + 1);
    ep::LayoutArgs a = layout_args(&lc, lp, topk_idx, nullptr, tokens_per_expert, nullptr,
                                   token_slot, cnt_loc, eo_loc, nullptr, workspace, dev_status);
    cudaStream_t cstr = cs(stream);
    if ((st = run_layout(&lc, lp, a, cstr)) != EP_OK) return st;
    // the counts to every GPU, then the counts signal
    launch(ep::group_push_counts_kernel, 1, 256, 0, cstr, (const int32_t *)peers->my_counts,
           peers->counts, (int64_t)s.g * s.RG * s.E, (int64_t)s.RG * s.E, peers->flags, s.g, s.G,
           grp->epoch);
    return launched();
}

ep_status_t ep_group_plan_host(const ep_config_t *cfg, const ep_group_t *grp,
                               const int32_t *tokens_per_expert_all, int64_t *slot_base,
                               int64_t *recv_count, int64_t *expert_offset) {
    Plan p;
    ep::GroupShape s;
    ep_status_t st = make_group(cfg, grp, p, s);
    if (st != EP_OK) return st;
    if (!tokens_per_expert_all || !slot_base || !recv_count) return EP_ERR_INVALID_ARG;
    if (cfg->layout == EP_LAYOUT_PACKED && !expert_offset) return EP_ERR_INVALID_ARG;
    for (int e = 0; e < s.E; e++) {
        slot_base[e] = ep::group_prefix(tokens_per_expert_all, s.E, s.g * s.RG, e);
        recv_count[e] = ep::group_total(tokens_per_expert_all, s.R, s.E, e);
    }
    if (cfg->layout == EP_LAYOUT_PACKED)
        ep::group_packed_offsets(s, recv_count, cfg->expert_align, expert_offset);
    return EP_OK;
}

ep_status_t ep_group_plan(const ep_config_t *cfg, const ep_group_t *grp,
                          const ep_peers_t *peers, const void *topk_idx, int32_t *token_slot,
                          int64_t *recv_count, int64_t *expert_offset,
                          int64_t *cumulative_recv_stats, void *workspace, size_t workspace_bytes,
                          uint32_t *dev_status, ep_stream_t stream) {
    Plan p;
    ep::GroupShape s;
    ep_status_t st = make_group(cfg, grp, p, s);
    if (st != EP_OK) return st;
    if (!group_ok(grp) || !peers_ok(peers) || !peers->my_counts || !recv_count || !workspace ||
        !dev_status)
        return EP_ERR_INVALID_ARG;
    const int32_t *tokens_per_expert_all = peers->my_counts;
    if (cfg->layout == EP_LAYOUT_PACKED && !expert_offset) return EP_ERR_INVALID_ARG;
    if (s.E > ep::kPlanThreads) return EP_ERR_UNSUPPORTED;
    if ((st = need(workspace_bytes, (int64_t)s.E * 8)) != EP_OK) return st;
    const int64_t n_loc = (int64_t)s.RG * p.T;
    if (n_loc > 0 && (!topk_idx || !token_slot)) return EP_ERR_INVALID_ARG;
    ep::GroupPlanArgs a;
    std::memset(&a, 0, sizeof(a));
    a.s = s;
    a.packed = cfg->layout == EP_LAYOUT_PACKED;
    a.align = cfg->expert_align;
    a.my_flags = peers->my_flags;
    a.epoch = grp->epoch;
    a.status = dev_status;
    a.n_loc = n_loc;
    a.K = p.K;
    a.tpe_all = tokens_per_expert_all;
    a.idx = topk_idx_view(cfg, topk_idx);
    a.slot = token_slot;
    a.recv_count = recv_count;
    a.expert_offset = expert_offset;
    a.stats = cumulative_recv_stats;
    a.slot_base = static_cast<int64_t *>(workspace);
    cudaStream_t cstr = cs(stream);
    launch(ep::group_plan_kernel, 1, ep::kPlanThreads, 0, cstr, a);
    if ((st = launched()) != EP_OK || n_loc == 0) return st;
    const int64_t entries = n_loc * p.K;
    const unsigned grid = (unsigned)std::min<int64_t>((entries + 255) / 256, 4 * sm_count());
    launch(ep::group_shift_kernel, grid, 256, 0, cstr, a);
    return launched();
}

ep_status_t ep_group_dispatch(const ep_config_t *cfg, const ep_group_t *grp,
                              const ep_peers_t *peers, const uint16_t *x, const void *topk_idx,
                              const float *topk_weights, const int32_t *token_slot,
                              const int64_t *expert_offset, uint32_t *dev_status,
                              ep_stream_t stream) {
    Plan p;
    ep::GroupShape s;
    ep_status_t st = make_group(cfg, grp, p, s);
    if (st != EP_OK) return st;
    if (!group_ok(grp) || !dev_status || !peers_ok(peers) || !peers->recv || !peers->src_info)
        return EP_ERR_INVALID_ARG;
    if (cfg->layout == EP_LAYOUT_PACKED && !expert_offset) return EP_ERR_INVALID_ARG;
    if (peers->recv_weights && !topk_weights) return EP_ERR_INVALID_ARG;
    const int64_t n_loc = (int64_t)s.RG * p.T;
    cudaStream_t cstr = cs(stream);
    if (n_loc == 0) {  // nothing to send: the others still learn that this GPU is done
        launch(ep::group_signal_kernel, 1, 32, 0, cstr, peers->flags, (int)ep::kFlagDispatch, s.g,
               s.G, grp->epoch);
        return launched();
    }
    if (!x || !topk_idx || !token_slot) return EP_ERR_INVALID_ARG;
    if (!aligned16(x)) return EP_ERR_MISALIGNED;
    ep::DispatchArgs a = dispatch_args(cfg, p);
    a.N = n_loc;
    a.first_rank = s.g * s.RG;
    a.rows = (int64_t)s.G * s.win_rows;  // virtual rows
    a.D = p.D; a.S = p.S; a.scale_off = round_up(s.win_rows * p.D, 256);
    a.x = x; a.idx = topk_idx_view(cfg, topk_idx);
    a.wts = topk_weights; a.slot = token_slot; a.eo = expert_offset;
    a.status = dev_status;
    a.peer_out = reinterpret_cast<uint8_t *const *>(peers->recv);
    a.peer_src = peers->src_info;
    a.peer_w = peers->recv_weights;
    a.win_rows = s.win_rows;
    a.experts_per_gpu = s.EG;
    a.done = peers->done + ep::kFlagDispatch;
    a.flags = peers->flags;
    a.flag_kind = ep::kFlagDispatch;
    a.grp_g = s.g; a.grp_G = s.G;
    a.epoch = grp->epoch;
    return run_dispatch(cfg, a, cstr);
}

ep_status_t ep_group_combine(const ep_config_t *cfg, const ep_group_t *grp,
                             const ep_peers_t *peers, const void *topk_idx,
                             const float *topk_weights, const int32_t *token_slot,
                             const int64_t *expert_offset, uint16_t *out, uint32_t *dev_status,
                             ep_stream_t stream) {
    Plan p;
    ep::GroupShape s;
    ep_status_t st = make_group(cfg, grp, p, s);
    if (st != EP_OK) return st;
    if (!group_ok(grp) || !dev_status || !peers || !peers->y) return EP_ERR_INVALID_ARG;
    if (cfg->flags & EP_F_COMBINE_QUANTIZED) return EP_ERR_UNSUPPORTED;
    const int64_t n_loc = (int64_t)s.RG * p.T;
    if (n_loc == 0) return EP_OK;
    if (!topk_idx || !topk_weights || !token_slot || !out) return EP_ERR_INVALID_ARG;
    if (cfg->layout == EP_LAYOUT_PACKED && !expert_offset) return EP_ERR_INVALID_ARG;
    if (!aligned16(out)) return EP_ERR_MISALIGNED;
    ep::CombineArgs a;
    std::memset(&a, 0, sizeof(a));
    a.N = n_loc; a.K = p.K; a.E = p.E; a.H = p.H;
    a.packed = cfg->layout == EP_LAYOUT_PACKED;
    a.cap = p.cap; a.rows = (int64_t)s.G * s.win_rows;
    a.idx = topk_idx_view(cfg, topk_idx);
    a.wts = topk_weights; a.slot = token_slot; a.eo = expert_offset;
    a.out = out; a.status = dev_status;
    a.peer_y = reinterpret_cast<const uint8_t *const *>(peers->y);
    a.win_rows = s.win_rows;
    a.experts_per_gpu = s.EG;
    return launch_combine<ep::QIN_BF16>(a, cs(stream));
}

ep_status_t ep_group_combine_backward(const ep_config_t *cfg, const ep_group_t *grp,
                                      const ep_peers_t *peers, const uint16_t *g,
                                      const void *topk_idx, const float *topk_weights,
                                      const int32_t *token_slot, const int64_t *expert_offset,
                                      uint32_t *dev_status, ep_stream_t stream) {
    Plan p;
    ep::GroupShape s;
    ep_status_t st = make_group(cfg, grp, p, s);
    if (st != EP_OK) return st;
    if (!group_ok(grp) || !dev_status || !peers_ok(peers) || !peers->grad)
        return EP_ERR_INVALID_ARG;
    const bool unweighted = (cfg->flags & EP_F_BWD_UNWEIGHTED) != 0;
    const int64_t n_loc = (int64_t)s.RG * p.T;
    cudaStream_t cstr = cs(stream);
    if (n_loc == 0) {
        launch(ep::group_signal_kernel, 1, 32, 0, cstr, peers->flags, (int)ep::kFlagBackward, s.g,
               s.G, grp->epoch);
        return launched();
    }
    if (!g || !topk_idx || !token_slot || (!unweighted && !topk_weights)) return EP_ERR_INVALID_ARG;
    if (cfg->layout == EP_LAYOUT_PACKED && !expert_offset) return EP_ERR_INVALID_ARG;
    if (!aligned16(g)) return EP_ERR_MISALIGNED;
    ep::DispatchArgs a = dispatch_args(cfg, p);
    a.N = n_loc;
    a.rows = (int64_t)s.G * s.win_rows;
    a.D = p.H; a.S = p.H / 32; a.scale_off = round_up(s.win_rows * p.H, 256);
    a.unweighted = unweighted;
    a.x = g; a.idx = topk_idx_view(cfg, topk_idx);
    a.wts = topk_weights; a.slot = token_slot; a.eo = expert_offset;
    a.status = dev_status;
    a.peer_out = reinterpret_cast<uint8_t *const *>(peers->grad);
    a.win_rows = s.win_rows;
    a.experts_per_gpu = s.EG;
    a.done = peers->done + ep::kFlagBackward;
    a.flags = peers->flags;
    a.flag_kind = ep::kFlagBackward;
    a.grp_g = s.g; a.grp_G = s.G;
    a.epoch = grp->epoch;
    return launch_combine_bwd(a, cstr);
}

ep_status_t ep_group_signal(const ep_group_t *grp, const ep_peers_t *peers, int32_t kind,
                            ep_stream_t stream) {
    if (!group_ok(grp) || !peers || !peers->flags) return EP_ERR_INVALID_ARG;
    if (kind < 0 || kind >= ep::kGroupKinds) return EP_ERR_INVALID_ARG;
    launch(ep::group_signal_kernel, 1, 32, 0, cs(stream), peers->flags, (int)kind, grp->rank,
           grp->world, grp->epoch);
    return launched();
}

ep_status_t ep_group_wait(const ep_group_t *grp, const ep_peers_t *peers, int32_t kind,
                          uint64_t timeout_ns, uint32_t *dev_status, ep_stream_t stream) {
    if (!group_ok(grp) || !peers || !peers->my_flags || !dev_status) return EP_ERR_INVALID_ARG;
    if (kind < 0 || kind >= ep::kGroupKinds) return EP_ERR_INVALID_ARG;
    const uint64_t limit = timeout_ns ? std::min<uint64_t>(timeout_ns, ep::kWaitLimitNs * 5)
                                      : ep::kWaitLimitNs;
    launch(ep::group_wait_kernel, 1, 64, 0, cs(stream), (const uint64_t *)peers->my_flags,
           (int)kind, (int)grp->world, grp->epoch, limit, dev_status);
    return launched();
}

// CUDA IPC of a window: the handle of the allocation that holds `ptr` and the
// offset of ptr inside it, and the mapping of a peer's window from them.
ep_status_t ep_ipc_export(const void *ptr, uint8_t *handle, uint64_t *offset) {
    if (!ptr || !handle || !offset) return EP_ERR_INVALID_ARG;
    using GetRange = CUresult (*)(CUdeviceptr *, size_t *, CUdeviceptr);
    static GetRange get_range = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_range = reinterpret_cast<GetRange>(f);
    });
    if (!get_range) return EP_ERR_CUDA;
    CUdeviceptr base = 0;
    size_t size = 0;
    if (get_range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS)
        return EP_ERR_CUDA;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base)) != cudaSuccess) return EP_ERR_CUDA;
    std::memcpy(handle, &h, sizeof(h));
    *offset = (uint64_t)(reinterpret_cast<uintptr_t>(ptr) - (uintptr_t)base);
    return EP_OK;
}

ep_status_t ep_ipc_import(const uint8_t *handle, uint64_t offset, void **ptr) {
    if (!handle || !ptr) return EP_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof(h));
    void *base = nullptr;
    if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess)
        return EP_ERR_CUDA;
    *ptr = static_cast<uint8_t *>(base) + offset;
    return EP_OK;
}

ep_status_t ep_ipc_close(void *base) {
    if (!base) return EP_ERR_INVALID_ARG;
    return cudaIpcCloseMemHandle(base) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

ep_status_t ep_get_status(uint32_t *dev_status, uint32_t *host_flags, ep_stream_t stream) {
    if (!dev_status || !host_flags) return EP_ERR_INVALID_ARG;
    cudaStream_t s = cs(stream);
    uint32_t h = 0;
    if (cudaMemcpyAsync(&h, dev_status, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return EP_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return EP_ERR_CUDA;
    if (cudaMemsetAsync(dev_status, 0, sizeof(uint32_t), s) != cudaSuccess) return EP_ERR_CUDA;
    *host_flags = h;
    if (h & EP_DEV_TIMEOUT) return EP_ERR_TIMEOUT;
    return h ? EP_ERR_DEVICE_STATUS : EP_OK;
}

}  // extern "C"

// ---- diagnostics -------------------------------------------------------------
namespace ep {

__global__ void __launch_bounds__(512) copy_kernel(uint4 *__restrict__ dst,
                                                   const uint4 *__restrict__ src, int64_t n) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (; i + 3 * stride < n; i += 4 * stride) {
        const uint4 a = ld_stream(src + i), b = ld_stream(src + i + stride);
        const uint4 c = ld_stream(src + i + 2 * stride), d = ld_stream(src + i + 3 * stride);
        dst[i] = a; dst[i + stride] = b; dst[i + 2 * stride] = c; dst[i + 3 * stride] = d;
    }
    for (; i < n; i += stride) dst[i] = ld_stream(src + i);
}

__global__ void cvt_sweep_kernel(int format, uint32_t start, int64_t n, uint8_t *out) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const float v = __uint_as_float(start + (uint32_t)i);
        const float av = __uint_as_float((start + (uint32_t)i) & 0x7FFFFFFFu);
        uint8_t r;
        switch (format) {
        case 0: r = (uint8_t)(cvt_e4m3x2(v, 0.0f) & 0xFFu); break;
        case 1: r = (uint8_t)(cvt_e2m1x2(v, 0.0f) & 0xFu); break;
        case 2: r = (uint8_t)(mx_exponent_fast<448>(av) + 127); break;
        default: r = (uint8_t)(mx_exponent_fast<6>(av) + 127); break;
        }
        out[i] = r;
    }
}

}  // namespace ep

namespace {
int sm_count() {  // declared above
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}
}  // namespace

extern "C" ep_status_t ep_copy(void *dst, const void *src, size_t bytes, ep_stream_t stream) {
    if (!dst || !src || bytes % 16 != 0) return EP_ERR_INVALID_ARG;
    if (!aligned16(dst) || !aligned16(src)) return EP_ERR_MISALIGNED;
    if (bytes == 0) return EP_OK;
    const int64_t n = (int64_t)(bytes / 16);
    int64_t blocks = (n + 511) / 512;
    const int64_t cap = (int64_t)sm_count() * 4;
    if (blocks > cap) blocks = cap;
    ep::copy_kernel<<<(unsigned)blocks, 512, 0, cs(stream)>>>(
        static_cast<uint4 *>(dst), static_cast<const uint4 *>(src), n);
    return launched();
}

extern "C" ep_status_t ep_cvt_sweep(int32_t format, uint32_t start, int64_t n, uint8_t *out,
                                    ep_stream_t stream) {
    if (format < 0 || format > 3 || n < 0 || !out) return EP_ERR_INVALID_ARG;
    if (n > (int64_t(1) << 32) - (int64_t)start) return EP_ERR_INVALID_ARG;
    if (n == 0) return EP_OK;
    int64_t blocks = (n + 255) / 256;
    const int64_t cap = (int64_t)sm_count() * 16;
    if (blocks > cap) blocks = cap;
    ep::cvt_sweep_kernel<<<(unsigned)blocks, 256, 0, cs(stream)>>>(format, start, n, out);
    return launched();
}

// ---- allocation-free layout ------------------------------------------------------
// The multi-block layout path with its scratch in a static device array, for
// callers that cannot allocate device memory (see ep_dispatch_layout_static in
// ep.h).  The array's device address is looked up once per device, with that
// device current, and cached.
namespace {

__device__ __align__(256) unsigned char g_static_scratch[EP_STATIC_SCRATCH_BYTES];

std::mutex g_static_mu;
void *g_static_ptr[kMaxDevices] = {};

ep_status_t static_scratch(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return EP_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return EP_ERR_CUDA;
        g_static_ptr[dev] = p;
    }
    *out = g_static_ptr[dev];
    return EP_OK;
}

}  // namespace

extern "C" ep_status_t ep_dispatch_layout_static(
    const ep_config_t *cfg, const void *topk_idx, int32_t *tokens_per_rank,
    int32_t *tokens_per_expert, uint8_t *is_token_in_rank, int32_t *token_slot,
    int64_t *recv_count, int64_t *expert_offset, int64_t *cumulative_recv_stats,
    uint32_t *dev_status, ep_stream_t stream) {
    Plan p;
    ep_status_t st = make_plan(cfg, p);
    if (st != EP_OK) return st;
    if (!recv_count || !dev_status) return EP_ERR_INVALID_ARG;
    if (p.N > 0 && (!topk_idx || !token_slot)) return EP_ERR_INVALID_ARG;
    if (cfg->layout == EP_LAYOUT_PACKED && !expert_offset) return EP_ERR_INVALID_ARG;
    if (p.ws_bytes > (int64_t)EP_STATIC_SCRATCH_BYTES) return EP_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if ((st = static_scratch(&scratch)) != EP_OK) return st;

    ep::LayoutArgs a;
    a.R = p.R; a.T = p.T; a.K = p.K; a.E = p.E; a.M = p.M; a.L = p.L;
    a.TC = p.TC; a.CR = p.CR; a.C = p.C;
    a.packed = cfg->layout == EP_LAYOUT_PACKED;
    a.align = cfg->expert_align;
    a.cap = p.cap;
    a.idx = topk_idx_view(cfg, topk_idx);
    a.tpr = tokens_per_rank;
    a.tpe = tokens_per_expert;
    a.itr = is_token_in_rank;
    a.slot = token_slot;
    a.recv_count = recv_count;
    a.eo = expert_offset;
    a.stats = cumulative_recv_stats;
    a.ws_hist = static_cast<int32_t *>(scratch);
    a.ws_rk = a.ws_hist + (int64_t)p.E * p.C;
    a.status = dev_status;

    return launch_layout_multi(a, p, cs(stream));
}
