"""Thin Python binding of libep (include/ep.h): argument checks and marshalling.

Every step of the path runs in libep's CUDA kernels; this module only turns
torch tensors into device pointers and the caller's stream into a
cudaStream_t.  Tensor checks follow "DeepEP topk_idx_t Custom Dtype
Requirements" (Tensor Requirements and Constraints: exact dtype, 2-D,
contiguous, matching top-k, checked before any GPU work) and "EP dispatch
with unfused MXFP8 quantization" (Changes: a pre-quantised input is
rejected -- x must be bfloat16).  If libep.so is missing the import fails:
there is no fallback path.
"""
import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libep.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"libep.so not built at {LIB_PATH}: run combine_ep_dispatch_04_b200/build.py")
lib = C.CDLL(LIB_PATH)

QUANT = {"bf16": 0, "e4m3_b128": 1, "int8_token": 2, "mxfp8": 3, "mxfp4": 4}
LAYOUT = {"padded": 0, "packed": 1}
DEV_BAD_INDEX = 0x1
DEV_CAPACITY_OVERFLOW = 0x2
DEV_TIMEOUT = 0x4
F_BWD_UNWEIGHTED = 0x1
F_COMBINE_QUANTIZED = 0x2
F_IDX_I32 = 0x4
F_ROUND_SCALE = 0x8
F_UE8M0 = 0x10
F_LAYOUT_SINGLE_CTA = 0x100
F_LAYOUT_MULTI_CTA = 0x200
F_LAYOUT_CLUSTER = 0x400
F_GEMM_CTA_PAIRS = 0x800

STATIC_SCRATCH_BYTES = 1 << 20  # EP_STATIC_SCRATCH_BYTES of include/ep.h

STATUS = {0: "EP_OK", 1: "EP_ERR_INVALID_ARG", 2: "EP_ERR_UNSUPPORTED", 3: "EP_ERR_MISALIGNED",
          4: "EP_ERR_CUDA", 5: "EP_ERR_DEVICE_STATUS", 6: "EP_ERR_TIMEOUT",
          7: "EP_ERR_BUFFER_TOO_SMALL"}
ERR_BUFFER_TOO_SMALL = 7


class EpError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = lib.ep_status_string(status).decode()
        super().__init__(f"{where}: {STATUS.get(status, status)} ({msg})")


class EpConfig(C.Structure):
    _fields_ = [("num_ranks", C.c_int32), ("num_tokens", C.c_int32),
                ("max_tokens_per_rank", C.c_int32), ("num_topk", C.c_int32),
                ("num_experts", C.c_int32), ("hidden", C.c_int32), ("quant", C.c_int32),
                ("layout", C.c_int32), ("expert_align", C.c_int32), ("e4m3_qmax", C.c_float),
                ("flags", C.c_uint32)]


class EpSizes(C.Structure):
    _fields_ = [(n, C.c_int64) for n in (
        "rows", "data_row_bytes", "scale_row_bytes", "recv_scale_offset", "recv_bytes",
        "src_info_bytes", "recv_weights_bytes", "expert_out_bytes", "grad_scale_offset",
        "grad_bytes", "workspace_bytes", "token_slot_bytes", "is_token_in_rank_bytes")]


class EpGroupT(C.Structure):
    _fields_ = [("world", C.c_int32), ("rank", C.c_int32), ("epoch", C.c_uint64),
                ("window_rows", C.c_int64)]


class EpPeers(C.Structure):
    """ep_peers_t: device arrays of G window pointers and this GPU's flags."""
    _fields_ = [("recv", C.c_void_p), ("src_info", C.c_void_p), ("recv_weights", C.c_void_p),
                ("y", C.c_void_p), ("grad", C.c_void_p), ("counts", C.c_void_p),
                ("flags", C.c_void_p), ("my_counts", C.c_void_p), ("my_flags", C.c_void_p),
                ("done", C.c_void_p)]


GROUP_KIND_COUNTS, GROUP_KIND_DISPATCH, GROUP_KIND_EXPERT_OUT, GROUP_KIND_COMBINED, \
    GROUP_KIND_BACKWARD = 0, 1, 2, 3, 4
GROUP_KINDS = 5

_P = C.c_void_p
_Z = C.c_size_t
_CFG = C.POINTER(EpConfig)
lib.ep_status_string.restype = C.c_char_p
lib.ep_status_string.argtypes = [C.c_int]
lib.ep_buffer_sizes.restype = C.c_int
lib.ep_buffer_sizes.argtypes = [_CFG, C.POINTER(EpSizes)]
lib.ep_dispatch_layout.restype = C.c_int
lib.ep_dispatch_layout.argtypes = [_CFG] + [_P] * 9 + [_Z, _P, _P]
lib.ep_dispatch_layout_static.restype = C.c_int
lib.ep_dispatch_layout_static.argtypes = [_CFG] + [_P] * 10
lib.ep_dispatch_with_layout.restype = C.c_int
lib.ep_dispatch_with_layout.argtypes = [_CFG] + [_P] * 11 + [_Z, _P, _Z, _P, _Z, _P, _Z, _P, _P]
lib.ep_dispatch.restype = C.c_int
lib.ep_dispatch.argtypes = [_CFG] + [_P] * 6 + [_Z, _P, _Z, _P, _Z, _P, _P]
lib.ep_combine.restype = C.c_int
lib.ep_combine.argtypes = [_CFG, _P, _Z] + [_P] * 7
lib.ep_combine_backward.restype = C.c_int
lib.ep_combine_backward.argtypes = [_CFG] + [_P] * 6 + [_Z, _P, _P]
lib.ep_expert_gemm.restype = C.c_int
lib.ep_expert_gemm.argtypes = [_CFG, _P, _Z, _P, _P, _P, C.c_int32, _P, _Z, _P, _P]
lib.ep_wait_probe.restype = C.c_int
lib.ep_wait_probe.argtypes = [_P, _P]
lib.ep_moe_forward.restype = C.c_int
lib.ep_moe_forward.argtypes = [_CFG] + [_P] * 9 + [_Z, _P, _Z, _P, _Z, _P, _Z, _P, _P, _P]
lib.ep_expert_gemm_mx.restype = C.c_int
lib.ep_expert_gemm_mx.argtypes = [_CFG, _P, _Z, _P, _P, _P, _P, C.c_int32, _P, _Z, _P, _P]
lib.ep_ffn_buffer_bytes.restype = C.c_int
lib.ep_ffn_buffer_bytes.argtypes = [_CFG, C.c_int32, C.POINTER(C.c_int64), C.POINTER(C.c_int64)]
lib.ep_expert_ffn_mx.restype = C.c_int
lib.ep_expert_ffn_mx.argtypes = [_CFG, _P, _Z, _P, _P, _P, _P, _P, _P, C.c_int32, _P, _Z, _P, _Z,
                                 _P, _P]
lib.ep_moe_forward_ffn.restype = C.c_int
lib.ep_moe_forward_ffn.argtypes = [_CFG] + [_P] * 7 + [C.c_int32] + [_P] * 4 + \
    [_Z, _P, _Z, _P, _Z, _P, _Z, _P, _Z, _P, _P, _P]
lib.ep_combine_backward_weights.restype = C.c_int
lib.ep_combine_backward_weights.argtypes = [_CFG, _P, _P, _Z] + [_P] * 6
_G = C.POINTER(EpGroupT)
_PE = C.POINTER(EpPeers)
lib.ep_group_sizes.restype = C.c_int
lib.ep_group_sizes.argtypes = [_CFG, _G, C.POINTER(EpSizes)]
lib.ep_group_layout.restype = C.c_int
lib.ep_group_layout.argtypes = [_CFG, _G, _PE, _P, _P, _P, _Z, _P, _P]
lib.ep_group_plan.restype = C.c_int
lib.ep_group_plan.argtypes = [_CFG, _G, _PE, _P, _P, _P, _P, _P, _P, _Z, _P, _P]
lib.ep_group_plan_host.restype = C.c_int
lib.ep_group_plan_host.argtypes = [_CFG, _G, _P, _P, _P, _P]
lib.ep_group_dispatch.restype = C.c_int
lib.ep_group_dispatch.argtypes = [_CFG, _G, _PE, _P, _P, _P, _P, _P, _P, _P]
lib.ep_group_combine.restype = C.c_int
lib.ep_group_combine.argtypes = [_CFG, _G, _PE, _P, _P, _P, _P, _P, _P, _P]
lib.ep_group_combine_backward.restype = C.c_int
lib.ep_group_combine_backward.argtypes = [_CFG, _G, _PE, _P, _P, _P, _P, _P, _P, _P]
lib.ep_group_signal.restype = C.c_int
lib.ep_group_signal.argtypes = [_G, _PE, C.c_int32, _P]
lib.ep_group_wait.restype = C.c_int
lib.ep_group_wait.argtypes = [_G, _PE, C.c_int32, C.c_uint64, _P, _P]
lib.ep_ipc_export.restype = C.c_int
lib.ep_ipc_export.argtypes = [_P, _P, C.POINTER(C.c_uint64)]
lib.ep_ipc_import.restype = C.c_int
lib.ep_ipc_import.argtypes = [_P, C.c_uint64, C.POINTER(C.c_void_p)]
lib.ep_ipc_close.restype = C.c_int
lib.ep_ipc_close.argtypes = [_P]
lib.ep_get_status.restype = C.c_int
lib.ep_get_status.argtypes = [_P, C.POINTER(C.c_uint32), _P]
lib.ep_copy.restype = C.c_int
lib.ep_copy.argtypes = [_P, _P, C.c_size_t, _P]
lib.ep_cvt_sweep.restype = C.c_int
lib.ep_cvt_sweep.argtypes = [C.c_int32, C.c_uint32, C.c_int64, _P, _P]
lib.ep_kernel_launches.restype = C.c_uint64
lib.ep_kernel_launches.argtypes = []


def make_config(R, T, M, K, E, H, quant="bf16", layout="padded", expert_align=1, e4m3_qmax=0.0,
                flags=0):
    q = QUANT[quant] if isinstance(quant, str) else int(quant)
    lay = LAYOUT[layout] if isinstance(layout, str) else int(layout)
    return EpConfig(R, T, M, K, E, H, q, lay, expert_align, float(e4m3_qmax), flags)


def _check(st, where):
    if st != 0:
        raise EpError(st, where)


class Bound:
    """One entry-point call with its arguments checked and marshalled once.
    Calling it replays the C call with the same pointers and stream (for loops
    that run the same step many times, e.g. a timing loop)."""

    def __init__(self, fn, cfg, args, where):
        self._fn, self._cfg, self._args, self._where = fn, cfg, tuple(args), where
        self._ref = C.byref(cfg)

    def __call__(self):
        st = self._fn(self._ref, *self._args)
        if st != 0:
            raise EpError(st, self._where)


def _call(fn, cfg, args, where, bind):
    if bind:
        return Bound(fn, cfg, args, where)
    _check(fn(C.byref(cfg), *args), where)
    return None


def ep_buffer_sizes(cfg):
    s = EpSizes()
    _check(lib.ep_buffer_sizes(C.byref(cfg), C.byref(s)), "ep_buffer_sizes")
    return {n: getattr(s, n) for n, _ in EpSizes._fields_}


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _dev(t, name, dtype, shape=None, optional=False):
    """Device pointer of a contiguous CUDA tensor of the given dtype (and shape)."""
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return C.c_void_p(t.data_ptr())


def _buf(t, name, optional=False):
    """(device pointer, byte count) of a contiguous CUDA buffer; libep checks the
    count against what the configuration needs (EP_ERR_BUFFER_TOO_SMALL)."""
    if t is None and optional:
        return [None, C.c_size_t(0)]
    if t is None or not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    return [C.c_void_p(t.data_ptr()), C.c_size_t(t.numel() * t.element_size())]


def _nk(cfg):
    return cfg.num_ranks * cfg.num_tokens, cfg.num_topk


def idx_dtype(cfg):
    """dtype of topk_idx for this configuration: int64, or int32 with F_IDX_I32."""
    return torch.int32 if cfg.flags & F_IDX_I32 else torch.int64


def ep_dispatch_layout(cfg, topk_idx, token_slot, recv_count, workspace, dev_status,
                       tokens_per_rank=None, tokens_per_expert=None, is_token_in_rank=None,
                       expert_offset=None, cumulative_recv_stats=None, stream=None, bind=False):
    N, K = _nk(cfg)
    R, E = cfg.num_ranks, cfg.num_experts
    args = [
        _dev(topk_idx, "topk_idx", idx_dtype(cfg), (N, K)),
        _dev(tokens_per_rank, "tokens_per_rank", torch.int32, (R, R), optional=True),
        _dev(tokens_per_expert, "tokens_per_expert", torch.int32, (R, E), optional=True),
        _dev(is_token_in_rank, "is_token_in_rank", torch.uint8, (N, R), optional=True),
        _dev(token_slot, "token_slot", torch.int32, (N, K)),
        _dev(recv_count, "recv_count", torch.int64, (E,)),
        _dev(expert_offset, "expert_offset", torch.int64, (E + 1,),
             optional=cfg.layout == LAYOUT["padded"]),
        _dev(cumulative_recv_stats, "cumulative_recv_stats", torch.int64, (E,), optional=True),
        *_buf(workspace, "workspace"),
        _dev(dev_status, "dev_status", torch.int32, (1,)),
        _stream(stream),
    ]
    return _call(lib.ep_dispatch_layout, cfg, args, "ep_dispatch_layout", bind)


def ep_dispatch_layout_static(cfg, topk_idx, token_slot, recv_count, dev_status,
                              tokens_per_rank=None, tokens_per_expert=None, is_token_in_rank=None,
                              expert_offset=None, cumulative_recv_stats=None, stream=None,
                              bind=False):
    """ep_dispatch_layout without a workspace: for callers that cannot allocate
    device memory.  Its scratch is a static array inside libep.so, shared by
    every call on the device (serialise calls; see include/ep.h)."""
    N, K = _nk(cfg)
    R, E = cfg.num_ranks, cfg.num_experts
    args = [
        _dev(topk_idx, "topk_idx", idx_dtype(cfg), (N, K)),
        _dev(tokens_per_rank, "tokens_per_rank", torch.int32, (R, R), optional=True),
        _dev(tokens_per_expert, "tokens_per_expert", torch.int32, (R, E), optional=True),
        _dev(is_token_in_rank, "is_token_in_rank", torch.uint8, (N, R), optional=True),
        _dev(token_slot, "token_slot", torch.int32, (N, K)),
        _dev(recv_count, "recv_count", torch.int64, (E,)),
        _dev(expert_offset, "expert_offset", torch.int64, (E + 1,),
             optional=cfg.layout == LAYOUT["padded"]),
        _dev(cumulative_recv_stats, "cumulative_recv_stats", torch.int64, (E,), optional=True),
        _dev(dev_status, "dev_status", torch.int32, (1,)),
        _stream(stream),
    ]
    return _call(lib.ep_dispatch_layout_static, cfg, args, "ep_dispatch_layout_static", bind)


def ep_dispatch(cfg, x, topk_idx, token_slot, recv_buf, src_info, dev_status, topk_weights=None,
                expert_offset=None, recv_weights=None, stream=None, bind=False):
    N, K = _nk(cfg)
    args = [
        _dev(x, "x", torch.bfloat16, (N, cfg.hidden)),
        _dev(topk_idx, "topk_idx", idx_dtype(cfg), (N, K)),
        _dev(topk_weights, "topk_weights", torch.float32, (N, K), optional=True),
        _dev(token_slot, "token_slot", torch.int32, (N, K)),
        _dev(expert_offset, "expert_offset", torch.int64, (cfg.num_experts + 1,),
             optional=cfg.layout == LAYOUT["padded"]),
        *_buf(recv_buf, "recv_buf"),
        *_buf(src_info, "src_info"),
        *_buf(recv_weights, "recv_weights", optional=True),
        _dev(dev_status, "dev_status", torch.int32, (1,)),
        _stream(stream),
    ]
    return _call(lib.ep_dispatch, cfg, args, "ep_dispatch", bind)


def ep_dispatch_with_layout(cfg, x, topk_idx, token_slot, recv_count, workspace, recv_buf,
                            src_info, dev_status, topk_weights=None, tokens_per_rank=None,
                            tokens_per_expert=None, is_token_in_rank=None, expert_offset=None,
                            cumulative_recv_stats=None, recv_weights=None, stream=None,
                            bind=False):
    """ep_dispatch_layout + ep_dispatch in one call (the dispatch kernel
    overlaps the layout; see include/ep.h)."""
    N, K = _nk(cfg)
    R, E = cfg.num_ranks, cfg.num_experts
    args = [
        _dev(x, "x", torch.bfloat16, (N, cfg.hidden)),
        _dev(topk_idx, "topk_idx", idx_dtype(cfg), (N, K)),
        _dev(topk_weights, "topk_weights", torch.float32, (N, K), optional=True),
        _dev(tokens_per_rank, "tokens_per_rank", torch.int32, (R, R), optional=True),
        _dev(tokens_per_expert, "tokens_per_expert", torch.int32, (R, E), optional=True),
        _dev(is_token_in_rank, "is_token_in_rank", torch.uint8, (N, R), optional=True),
        _dev(token_slot, "token_slot", torch.int32, (N, K)),
        _dev(recv_count, "recv_count", torch.int64, (E,)),
        _dev(expert_offset, "expert_offset", torch.int64, (E + 1,),
             optional=cfg.layout == LAYOUT["padded"]),
        _dev(cumulative_recv_stats, "cumulative_recv_stats", torch.int64, (E,), optional=True),
        *_buf(workspace, "workspace"),
        *_buf(recv_buf, "recv_buf"),
        *_buf(src_info, "src_info"),
        *_buf(recv_weights, "recv_weights", optional=True),
        _dev(dev_status, "dev_status", torch.int32, (1,)),
        _stream(stream),
    ]
    return _call(lib.ep_dispatch_with_layout, cfg, args, "ep_dispatch_with_layout", bind)


def ep_combine(cfg, y, topk_idx, topk_weights, token_slot, out, dev_status, expert_offset=None,
               stream=None, bind=False):
    N, K = _nk(cfg)
    quantized = bool(cfg.flags & F_COMBINE_QUANTIZED) and cfg.quant != QUANT["bf16"]
    if y is None or (not quantized and y.dtype != torch.bfloat16):
        raise TypeError("y (expert outputs) must be bfloat16 unless F_COMBINE_QUANTIZED")
    args = [
        *_buf(y, "y"),
        _dev(topk_idx, "topk_idx", idx_dtype(cfg), (N, K)),
        _dev(topk_weights, "topk_weights", torch.float32, (N, K)),
        _dev(token_slot, "token_slot", torch.int32, (N, K)),
        _dev(expert_offset, "expert_offset", torch.int64, (cfg.num_experts + 1,),
             optional=cfg.layout == LAYOUT["padded"]),
        _dev(out, "out", torch.bfloat16, (N, cfg.hidden)),
        _dev(dev_status, "dev_status", torch.int32, (1,)),
        _stream(stream),
    ]
    return _call(lib.ep_combine, cfg, args, "ep_combine", bind)


def ep_combine_backward(cfg, g, topk_idx, topk_weights, token_slot, grad_buf, dev_status,
                        expert_offset=None, stream=None, bind=False):
    N, K = _nk(cfg)
    args = [
        _dev(g, "g", torch.bfloat16, (N, cfg.hidden)),
        _dev(topk_idx, "topk_idx", idx_dtype(cfg), (N, K)),
        _dev(topk_weights, "topk_weights", torch.float32, (N, K),
             optional=bool(cfg.flags & F_BWD_UNWEIGHTED)),
        _dev(token_slot, "token_slot", torch.int32, (N, K)),
        _dev(expert_offset, "expert_offset", torch.int64, (cfg.num_experts + 1,),
             optional=cfg.layout == LAYOUT["padded"]),
        *_buf(grad_buf, "grad_buf"),
        _dev(dev_status, "dev_status", torch.int32, (1,)),
        _stream(stream),
    ]
    return _call(lib.ep_combine_backward, cfg, args, "ep_combine_backward", bind)


def ep_expert_gemm(cfg, recv_buf, expert_offset, recv_count, weights, y, dev_status, stream=None,
                   bind=False):
    """y[r] = bf16(x[r] . W[e]^T) for the rows of every expert (packed bf16 receive layout);
    weights bf16 [E, n_out, H], y bf16 [rows, n_out]."""
    sz = ep_buffer_sizes(cfg)
    E, H = cfg.num_experts, cfg.hidden
    if weights is None or weights.dim() != 3:
        raise ValueError("weights must be a [E, n_out, H] tensor")
    n_out = int(weights.shape[1])
    args = [
        *_buf(recv_buf, "recv_buf"),
        _dev(expert_offset, "expert_offset", torch.int64, (E + 1,)),
        _dev(recv_count, "recv_count", torch.int64, (E,)),
        _dev(weights, "weights", torch.bfloat16, (E, n_out, H)),
        C.c_int32(n_out),
        _dev(y, "y", torch.bfloat16, (sz["rows"], n_out)), C.c_size_t(sz["rows"] * n_out * 2),
        _dev(dev_status, "dev_status", torch.int32, (1,)),
        _stream(stream),
    ]
    return _call(lib.ep_expert_gemm, cfg, args, "ep_expert_gemm", bind)


def ep_expert_gemm_mx(cfg, recv_buf, expert_offset, recv_count, w_codes, w_scales, y, dev_status,
                      stream=None, bind=False):
    """The same maps on MX operands (packed MXFP8 or MXFP4 receive layout): w_codes
    [E, n_out, D] as uint8 (D = H for e4m3, H/2 for packed e2m1), w_scales e8m0
    [E, n_out, H/32] as uint8, y bf16 [rows, n_out]."""
    sz = ep_buffer_sizes(cfg)
    E, H = cfg.num_experts, cfg.hidden
    D = sz["data_row_bytes"]
    if w_codes is None or w_codes.dim() != 3:
        raise ValueError("w_codes must be a [E, n_out, D] tensor")
    n_out = int(w_codes.shape[1])
    args = [
        *_buf(recv_buf, "recv_buf"),
        _dev(expert_offset, "expert_offset", torch.int64, (E + 1,)),
        _dev(recv_count, "recv_count", torch.int64, (E,)),
        _dev(w_codes, "w_codes", torch.uint8, (E, n_out, D)),
        _dev(w_scales, "w_scales", torch.uint8, (E, n_out, H // 32)),
        C.c_int32(n_out),
        _dev(y, "y", torch.bfloat16, (sz["rows"], n_out)), C.c_size_t(sz["rows"] * n_out * 2),
        _dev(dev_status, "dev_status", torch.int32, (1,)),
        _stream(stream),
    ]
    return _call(lib.ep_expert_gemm_mx, cfg, args, "ep_expert_gemm_mx", bind)


def ep_ffn_buffer_bytes(cfg, inter):
    """(z_bytes, z_scale_offset) of the gated MLP's intermediate buffer."""
    zb, zo = C.c_int64(0), C.c_int64(0)
    _check(lib.ep_ffn_buffer_bytes(C.byref(cfg), int(inter), C.byref(zb), C.byref(zo)),
           "ep_ffn_buffer_bytes")
    return zb.value, zo.value


def _ffn_weights(cfg, w1_codes, w1_scales, w2_codes, w2_scales):
    E, H = cfg.num_experts, cfg.hidden
    if w1_codes is None or w1_codes.dim() != 3 or w1_codes.shape[1] % 2:
        raise ValueError("w1_codes must be a [E, 2I, H] tensor")
    inter = int(w1_codes.shape[1]) // 2
    return inter, [
        _dev(w1_codes, "w1_codes", torch.uint8, (E, 2 * inter, H)),
        _dev(w1_scales, "w1_scales", torch.uint8, (E, 2 * inter, H // 32)),
        _dev(w2_codes, "w2_codes", torch.uint8, (E, H, inter)),
        _dev(w2_scales, "w2_scales", torch.uint8, (E, H, inter // 32)),
        C.c_int32(inter),
    ]


def ep_expert_ffn_mx(cfg, recv_buf, expert_offset, recv_count, w1_codes, w1_scales, w2_codes,
                     w2_scales, z_buf, y, dev_status, stream=None, bind=False):
    """The experts' gated MLP on the packed MXFP8 receive rows: GMM1 (w1 [E, 2I, H],
    gate rows first) with SwiGLU and the MXFP8 requant of z in its epilogue (z_buf:
    codes [rows, I] then scales, ep_ffn_buffer_bytes), then GMM2 (w2 [E, H, I]) into
    y bf16 [rows, H]."""
    sz = ep_buffer_sizes(cfg)
    E, H = cfg.num_experts, cfg.hidden
    _, wargs = _ffn_weights(cfg, w1_codes, w1_scales, w2_codes, w2_scales)
    args = [
        *_buf(recv_buf, "recv_buf"),
        _dev(expert_offset, "expert_offset", torch.int64, (E + 1,)),
        _dev(recv_count, "recv_count", torch.int64, (E,)),
        *wargs,
        *_buf(z_buf, "z_buf"),
        _dev(y, "y", torch.bfloat16, (sz["rows"], H)), C.c_size_t(sz["rows"] * H * 2),
        _dev(dev_status, "dev_status", torch.int32, (1,)),
        _stream(stream),
    ]
    return _call(lib.ep_expert_ffn_mx, cfg, args, "ep_expert_ffn_mx", bind)


def ep_moe_forward_ffn(cfg, x, topk_idx, topk_weights, w1_codes, w1_scales, w2_codes, w2_scales,
                       token_slot, recv_count, expert_offset, workspace, recv_buf, src_info,
                       z_buf, y, out, dev_status, stream=None, bind=False):
    """Layout + MXFP8 dispatch -> the experts' gated MLP (ep_expert_ffn_mx) ->
    combine in one call; out bf16 [N, H]."""
    N, K = _nk(cfg)
    sz = ep_buffer_sizes(cfg)
    E, H = cfg.num_experts, cfg.hidden
    _, wargs = _ffn_weights(cfg, w1_codes, w1_scales, w2_codes, w2_scales)
    args = [
        _dev(x, "x", torch.bfloat16, (N, H)),
        _dev(topk_idx, "topk_idx", idx_dtype(cfg), (N, K)),
        _dev(topk_weights, "topk_weights", torch.float32, (N, K)),
        *wargs,
        _dev(token_slot, "token_slot", torch.int32, (N, K)),
        _dev(recv_count, "recv_count", torch.int64, (E,)),
        _dev(expert_offset, "expert_offset", torch.int64, (E + 1,)),
        *_buf(workspace, "workspace"),
        *_buf(recv_buf, "recv_buf"),
        *_buf(src_info, "src_info"),
        *_buf(z_buf, "z_buf"),
        _dev(y, "y", torch.bfloat16, (sz["rows"], H)), C.c_size_t(sz["rows"] * H * 2),
        _dev(out, "out", torch.bfloat16, (N, H)),
        _dev(dev_status, "dev_status", torch.int32, (1,)),
        _stream(stream),
    ]
    return _call(lib.ep_moe_forward_ffn, cfg, args, "ep_moe_forward_ffn", bind)


def ep_wait_probe(dev_status, stream=None):
    """One block waits on a barrier nothing completes: after 2 s the wait gives
    up and sets DEV_TIMEOUT in dev_status (read it with ep_get_status)."""
    st = lib.ep_wait_probe(_dev(dev_status, "dev_status", torch.int32, (1,)), _stream(stream))
    if st != 0:
        raise EpError(st, "ep_wait_probe")


def ep_moe_forward(cfg, x, topk_idx, topk_weights, w_codes, w_scales, token_slot, recv_count,
                   expert_offset, workspace, recv_buf, src_info, y, out, dev_status, stream=None,
                   bind=False):
    """Layout + dispatch -> the experts' maps (n_out = H) -> combine in one call:
    w_codes bf16 [E, H, H] with w_scales None, or MX codes uint8 [E, H, D] with
    e8m0 w_scales uint8 [E, H, H/32]; y bf16 [rows, H] scratch; out bf16 [N, H]."""
    N, K = _nk(cfg)
    sz = ep_buffer_sizes(cfg)
    E, H = cfg.num_experts, cfg.hidden
    if cfg.quant == QUANT["bf16"]:
        if w_scales is not None:
            raise ValueError("bf16 weights take no scales")
        wc = _dev(w_codes, "w_codes", torch.bfloat16, (E, H, H))
        ws = None
    else:
        wc = _dev(w_codes, "w_codes", torch.uint8, (E, H, sz["data_row_bytes"]))
        ws = _dev(w_scales, "w_scales", torch.uint8, (E, H, H // 32))
    args = [
        _dev(x, "x", torch.bfloat16, (N, H)),
        _dev(topk_idx, "topk_idx", idx_dtype(cfg), (N, K)),
        _dev(topk_weights, "topk_weights", torch.float32, (N, K)),
        wc, ws,
        _dev(token_slot, "token_slot", torch.int32, (N, K)),
        _dev(recv_count, "recv_count", torch.int64, (E,)),
        _dev(expert_offset, "expert_offset", torch.int64, (E + 1,)),
        *_buf(workspace, "workspace"),
        *_buf(recv_buf, "recv_buf"),
        *_buf(src_info, "src_info"),
        _dev(y, "y", torch.bfloat16, (sz["rows"], H)), C.c_size_t(sz["rows"] * H * 2),
        _dev(out, "out", torch.bfloat16, (N, H)),
        _dev(dev_status, "dev_status", torch.int32, (1,)),
        _stream(stream),
    ]
    return _call(lib.ep_moe_forward, cfg, args, "ep_moe_forward", bind)


def ep_combine_backward_weights(cfg, g, y, topk_idx, token_slot, topk_weights_grad, dev_status,
                                expert_offset=None, stream=None, bind=False):
    """topk_weights_grad[n, k] = <g[n, :], y[row(n, k), :]> (0 for masked entries)."""
    N, K = _nk(cfg)
    sz = ep_buffer_sizes(cfg)
    args = [
        _dev(g, "g", torch.bfloat16, (N, cfg.hidden)),
        _dev(y, "y", torch.bfloat16, (sz["rows"], cfg.hidden)),
        C.c_size_t(sz["rows"] * cfg.hidden * 2),
        _dev(topk_idx, "topk_idx", idx_dtype(cfg), (N, K)),
        _dev(token_slot, "token_slot", torch.int32, (N, K)),
        _dev(expert_offset, "expert_offset", torch.int64, (cfg.num_experts + 1,),
             optional=cfg.layout == LAYOUT["padded"]),
        _dev(topk_weights_grad, "topk_weights_grad", torch.float32, (N, K)),
        _dev(dev_status, "dev_status", torch.int32, (1,)),
        _stream(stream),
    ]
    return _call(lib.ep_combine_backward_weights, cfg, args, "ep_combine_backward_weights", bind)


def ep_get_status(dev_status, stream=None):
    """Synchronise, read and clear the device status word; returns its bits."""
    flags = C.c_uint32(0)
    st = lib.ep_get_status(_dev(dev_status, "dev_status", torch.int32, (1,)), C.byref(flags),
                           _stream(stream))
    if st not in (0, 5, 6):
        raise EpError(st, "ep_get_status")
    return flags.value


# ---- expert parallelism over GPUs (include/ep.h, ep_group_*) ----------------------
def make_group(world, rank, epoch=1, window_rows=0):
    return EpGroupT(world, rank, epoch, window_rows)


def ep_group_sizes(cfg, grp):
    s = EpSizes()
    _check(lib.ep_group_sizes(C.byref(cfg), C.byref(grp), C.byref(s)), "ep_group_sizes")
    return {n: getattr(s, n) for n, _ in EpSizes._fields_}


def _gnk(cfg, grp):
    return (cfg.num_ranks // grp.world) * cfg.num_tokens, cfg.num_topk


def ep_group_layout(cfg, grp, peers, topk_idx, token_slot, workspace, dev_status, stream=None,
                    bind=False):
    """Local ranks of this GPU's entries; its per-rank counts to every GPU's
    counts window (then the COUNTS signal)."""
    n, K = _gnk(cfg, grp)
    args = [C.byref(peers),
            _dev(topk_idx, "topk_idx", idx_dtype(cfg), (n, K)),
            _dev(token_slot, "token_slot", torch.int32, (n, K)),
            *_buf(workspace, "workspace"),
            _dev(dev_status, "dev_status", torch.int32, (1,)), _stream(stream)]
    return _gcall(lib.ep_group_layout, cfg, grp, args, "ep_group_layout", bind)


def ep_group_plan(cfg, grp, peers, topk_idx, token_slot, recv_count, expert_offset, slot_scratch,
                  dev_status, cumulative_recv_stats=None, stream=None, bind=False):
    """After every GPU's counts: global slots, totals and virtual packed offsets."""
    n, K = _gnk(cfg, grp)
    E = cfg.num_experts
    args = [C.byref(peers),
            _dev(topk_idx, "topk_idx", idx_dtype(cfg), (n, K)),
            _dev(token_slot, "token_slot", torch.int32, (n, K)),
            _dev(recv_count, "recv_count", torch.int64, (E,)),
            _dev(expert_offset, "expert_offset", torch.int64, (E + 1,),
                 optional=cfg.layout == LAYOUT["padded"]),
            _dev(cumulative_recv_stats, "cumulative_recv_stats", torch.int64, (E,), optional=True),
            *_buf(slot_scratch, "slot_scratch"),
            _dev(dev_status, "dev_status", torch.int32, (1,)), _stream(stream)]
    return _gcall(lib.ep_group_plan, cfg, grp, args, "ep_group_plan", bind)


def ep_group_plan_host(cfg, grp, tokens_per_expert_all):
    """The plan on the host (numpy): (slot_base [E], recv_count [E], expert_offset [E+1])."""
    import numpy as np
    E = cfg.num_experts
    tpe = np.ascontiguousarray(tokens_per_expert_all, np.int32)
    assert tpe.shape == (cfg.num_ranks, E)
    base, cnt = np.zeros(E, np.int64), np.zeros(E, np.int64)
    eo = np.zeros(E + 1, np.int64)
    p = lambda a: a.ctypes.data_as(C.c_void_p)  # noqa: E731
    _check(lib.ep_group_plan_host(C.byref(cfg), C.byref(grp), p(tpe), p(base), p(cnt), p(eo)),
           "ep_group_plan_host")
    return base, cnt, eo


def ep_group_dispatch(cfg, grp, peers, x, topk_idx, token_slot, dev_status, topk_weights=None,
                      expert_offset=None, stream=None, bind=False):
    n, K = _gnk(cfg, grp)
    args = [C.byref(peers),
            _dev(x, "x", torch.bfloat16, (n, cfg.hidden)),
            _dev(topk_idx, "topk_idx", idx_dtype(cfg), (n, K)),
            _dev(topk_weights, "topk_weights", torch.float32, (n, K), optional=True),
            _dev(token_slot, "token_slot", torch.int32, (n, K)),
            _dev(expert_offset, "expert_offset", torch.int64, (cfg.num_experts + 1,),
                 optional=cfg.layout == LAYOUT["padded"]),
            _dev(dev_status, "dev_status", torch.int32, (1,)), _stream(stream)]
    return _gcall(lib.ep_group_dispatch, cfg, grp, args, "ep_group_dispatch", bind)


def ep_group_combine(cfg, grp, peers, topk_idx, topk_weights, token_slot, out, dev_status,
                     expert_offset=None, stream=None, bind=False):
    n, K = _gnk(cfg, grp)
    args = [C.byref(peers),
            _dev(topk_idx, "topk_idx", idx_dtype(cfg), (n, K)),
            _dev(topk_weights, "topk_weights", torch.float32, (n, K)),
            _dev(token_slot, "token_slot", torch.int32, (n, K)),
            _dev(expert_offset, "expert_offset", torch.int64, (cfg.num_experts + 1,),
                 optional=cfg.layout == LAYOUT["padded"]),
            _dev(out, "out", torch.bfloat16, (n, cfg.hidden)),
            _dev(dev_status, "dev_status", torch.int32, (1,)), _stream(stream)]
    return _gcall(lib.ep_group_combine, cfg, grp, args, "ep_group_combine", bind)


def ep_group_combine_backward(cfg, grp, peers, g, topk_idx, topk_weights, token_slot, dev_status,
                              expert_offset=None, stream=None, bind=False):
    n, K = _gnk(cfg, grp)
    args = [C.byref(peers),
            _dev(g, "g", torch.bfloat16, (n, cfg.hidden)),
            _dev(topk_idx, "topk_idx", idx_dtype(cfg), (n, K)),
            _dev(topk_weights, "topk_weights", torch.float32, (n, K),
                 optional=bool(cfg.flags & F_BWD_UNWEIGHTED)),
            _dev(token_slot, "token_slot", torch.int32, (n, K)),
            _dev(expert_offset, "expert_offset", torch.int64, (cfg.num_experts + 1,),
                 optional=cfg.layout == LAYOUT["padded"]),
            _dev(dev_status, "dev_status", torch.int32, (1,)), _stream(stream)]
    return _gcall(lib.ep_group_combine_backward, cfg, grp, args, "ep_group_combine_backward",
                  bind)


def ep_group_signal(grp, peers, kind, stream=None, bind=False):
    args = [C.byref(peers), C.c_int32(int(kind)), _stream(stream)]
    if bind:
        return _Plain(lib.ep_group_signal, [C.byref(grp)] + args, "ep_group_signal")
    _check(lib.ep_group_signal(C.byref(grp), *args), "ep_group_signal")


def ep_group_wait(grp, peers, kind, dev_status, timeout_ns=0, stream=None, bind=False):
    args = [C.byref(peers), C.c_int32(int(kind)), C.c_uint64(int(timeout_ns)),
            _dev(dev_status, "dev_status", torch.int32, (1,)), _stream(stream)]
    if bind:
        return _Plain(lib.ep_group_wait, [C.byref(grp)] + args, "ep_group_wait")
    _check(lib.ep_group_wait(C.byref(grp), *args), "ep_group_wait")


class _Plain:
    """A bound call without a configuration argument."""

    def __init__(self, fn, args, where):
        self._fn, self._args, self._where = fn, tuple(args), where

    def __call__(self):
        st = self._fn(*self._args)
        if st != 0:
            raise EpError(st, self._where)


class _GBound(Bound):
    def __init__(self, fn, cfg, grp, args, where):
        super().__init__(fn, cfg, args, where)
        self._grp = C.byref(grp)

    def __call__(self):
        st = self._fn(self._ref, self._grp, *self._args)
        if st != 0:
            raise EpError(st, self._where)


def _gcall(fn, cfg, grp, args, where, bind):
    if bind:
        return _GBound(fn, cfg, grp, args, where)
    _check(fn(C.byref(cfg), C.byref(grp), *args), where)
    return None


def ep_ipc_export(t):
    """(64-byte handle, offset) of a CUDA tensor's memory, for another process."""
    h = (C.c_uint8 * 64)()
    off = C.c_uint64(0)
    _check(lib.ep_ipc_export(C.c_void_p(t.data_ptr()), h, C.byref(off)), "ep_ipc_export")
    return bytes(h), off.value


def ep_ipc_import(handle, offset):
    """Device address of another process's exported memory, mapped here."""
    h = (C.c_uint8 * 64).from_buffer_copy(handle)
    p = C.c_void_p(0)
    _check(lib.ep_ipc_import(h, int(offset), C.byref(p)), "ep_ipc_import")
    return p.value


def ep_ipc_close(base):
    _check(lib.ep_ipc_close(C.c_void_p(base)), "ep_ipc_close")


def ep_copy(dst, src, stream=None):
    n = src.numel() * src.element_size()
    (pd, nd), (ps, _) = _buf(dst, "dst"), _buf(src, "src")
    if nd.value < n:
        raise ValueError(f"dst holds {nd.value} bytes, needs {n}")
    _check(lib.ep_copy(pd, ps, n, _stream(stream)), "ep_copy")


def ep_cvt_sweep(fmt, start, out, stream=None):
    _check(lib.ep_cvt_sweep(fmt, start, out.numel(), _dev(out, "out", torch.uint8), _stream(stream)),
           "ep_cvt_sweep")


def ep_kernel_launches():
    return int(lib.ep_kernel_launches())


class Buffers:
    """Caller-owned device buffers for one configuration (plain torch allocations)."""

    def __init__(self, cfg, device="cuda", recv_weights=False, expert_out=True, grad=False):
        sz = ep_buffer_sizes(cfg)
        self.sizes = sz
        N, K = _nk(cfg)
        R, E, H = cfg.num_ranks, cfg.num_experts, cfg.hidden
        u8 = dict(dtype=torch.uint8, device=device)
        self.tokens_per_rank = torch.empty((R, R), dtype=torch.int32, device=device)
        self.tokens_per_expert = torch.empty((R, E), dtype=torch.int32, device=device)
        self.is_token_in_rank = torch.empty((N, R), **u8)
        self.token_slot = torch.empty((N, K), dtype=torch.int32, device=device)
        self.recv_count = torch.empty(E, dtype=torch.int64, device=device)
        self.expert_offset = torch.empty(E + 1, dtype=torch.int64, device=device) \
            if cfg.layout == LAYOUT["packed"] else None
        self.workspace = torch.empty(sz["workspace_bytes"], **u8)
        self.recv_buf = torch.empty(sz["recv_bytes"], **u8)
        self.src_info = torch.empty(sz["rows"], dtype=torch.int32, device=device)
        self.recv_weights = torch.empty(sz["rows"], dtype=torch.float32, device=device) \
            if recv_weights else None
        self.y = torch.empty((sz["rows"], H), dtype=torch.bfloat16, device=device) \
            if expert_out else None
        self.out = torch.empty((N, H), dtype=torch.bfloat16, device=device)
        self.grad_buf = torch.empty(sz["grad_bytes"], **u8) if grad else None
        self.dev_status = torch.zeros(1, dtype=torch.int32, device=device)

    def recv_data(self):
        """View of the data region: [rows, D] bytes."""
        s = self.sizes
        return self.recv_buf[: s["rows"] * s["data_row_bytes"]].view(s["rows"], s["data_row_bytes"])

    def recv_scale(self):
        s = self.sizes
        a = s["recv_scale_offset"]
        return self.recv_buf[a: a + s["rows"] * s["scale_row_bytes"]].view(s["rows"], s["scale_row_bytes"])

    def grad_data(self, H):
        s = self.sizes
        return self.grad_buf[: s["rows"] * H].view(s["rows"], H)

    def grad_scale(self, H):
        s = self.sizes
        a = s["grad_scale_offset"]
        return self.grad_buf[a: a + s["rows"] * (H // 32)].view(s["rows"], H // 32)
