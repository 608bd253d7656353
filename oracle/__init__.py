"""The oracle: a plain, slow CPU statement of MoE dispatch / combine.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  The product path
(``combine_ep_dispatch_04_b200``) never imports it, and it never imports the
product.  The arithmetic lives in ``ep_oracle.c``; this module only builds and
loads it and marshals numpy arrays.

Modes and layouts use the names of the product's enums, mapped here by value:
bf16=0, e4m3_b128=1, int8_token=2, mxfp8=3, mxfp4=4; padded=0, packed=1.  Two
more modes are e4m3_b128 with the scale options: e4m3_b128_p2 (round_scale:
power-of-two fp32 scales) and e4m3_b128_ue8m0 (the same as e8m0 bytes).
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

MODES = {"bf16": 0, "e4m3_b128": 1, "int8_token": 2, "mxfp8": 3, "mxfp4": 4,
         "e4m3_b128_p2": 5, "e4m3_b128_ue8m0": 6}
LAYOUTS = {"padded": 0, "packed": 1}
ST_BAD_INDEX = 0x1
ST_CAPACITY = 0x2

# EP_ORACLE_LIB names another build of ep_oracle.c (the mutation tests load
# copies with planted mistakes through it); normally the library is built here.
_lib = C.CDLL(os.environ.get("EP_ORACLE_LIB") or _build.build())

_p = C.c_void_p
_i = C.c_int
_f = C.c_float
_l = C.c_long

_lib.orc_bf16_to_f32.restype = C.c_float
_lib.orc_bf16_to_f32.argtypes = [C.c_uint16]
_lib.orc_f32_to_bf16.restype = C.c_uint16
_lib.orc_f32_to_bf16.argtypes = [C.c_float]
_lib.orc_e4m3_encode.restype = C.c_uint8
_lib.orc_e4m3_encode.argtypes = [C.c_float]
_lib.orc_e2m1_encode.restype = C.c_uint8
_lib.orc_e2m1_encode.argtypes = [C.c_float]
_lib.orc_e4m3_decode.restype = C.c_float
_lib.orc_e4m3_decode.argtypes = [C.c_uint8]
_lib.orc_e2m1_decode.restype = C.c_float
_lib.orc_e2m1_decode.argtypes = [C.c_uint8]
_lib.orc_mx_exponent.restype = C.c_int
_lib.orc_mx_exponent.argtypes = [C.c_float, C.c_float]
_lib.orc_row_data_bytes.restype = C.c_long
_lib.orc_row_data_bytes.argtypes = [_i, _i]
_lib.orc_row_scale_bytes.restype = C.c_long
_lib.orc_row_scale_bytes.argtypes = [_i, _i]
_lib.orc_quant_row_f32.restype = None
_lib.orc_quant_row_f32.argtypes = [_i, _i, _f, _p, _p, _p]
_lib.orc_quant_row_bf16.restype = None
_lib.orc_quant_row_bf16.argtypes = [_i, _i, _f, _p, _p, _p]
_lib.orc_layout.restype = C.c_uint32
_lib.orc_layout.argtypes = [_i, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p]
_lib.orc_dispatch.restype = C.c_uint32
_lib.orc_dispatch.argtypes = [_i, _i, _i, _i, _i, _i, _i, _f, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p]
_lib.orc_combine_row.restype = None
_lib.orc_combine_row.argtypes = [_i, _i, _p, _p, _p, _p]
_lib.orc_combine.restype = C.c_uint32
_lib.orc_combine.argtypes = [_i, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p]
_lib.orc_combine_bwd.restype = C.c_uint32
_lib.orc_combine_bwd.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p]
_lib.orc_combine_wgrad.restype = C.c_uint32
_lib.orc_combine_wgrad.argtypes = [_i, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p]
_lib.orc_combine_wgrad_gathered.restype = None
_lib.orc_combine_wgrad_gathered.argtypes = [_l, _i, _i, _p, _p, _p, _p, _p]
_lib.orc_expert_gemm.restype = None
_lib.orc_expert_gemm.argtypes = [_i, _i, _i, _p, _p, _p, _p, _p]
_lib.orc_expert_gemm_mx.restype = None
_lib.orc_expert_gemm_mx.argtypes = [_i, _i, _i, _p, _p, _p, _p, _p, _p, _p]
_lib.orc_expert_gemm_mxfp4.restype = None
_lib.orc_expert_gemm_mxfp4.argtypes = [_i, _i, _i, _p, _p, _p, _p, _p, _p, _p]
_lib.orc_bwd_row.restype = None
_lib.orc_expert_ffn_mx.restype = None
_lib.orc_expert_ffn_mx.argtypes = [_i, _i, _i] + [_p] * 13
_lib.orc_bwd_row.argtypes = [_i, _f, _i, _p, _p, _p]
_lib.orc_combine_gathered.restype = None
_lib.orc_combine_gathered.argtypes = [_l, _i, _i, _p, _p, _p, _p]
_lib.orc_dequant_row.restype = None
_lib.orc_dequant_row.argtypes = [_i, _i, _p, _p, _p]
_lib.orc_combine_gathered_q.restype = None
_lib.orc_combine_gathered_q.argtypes = [_i, _l, _i, _i, _p, _p, _p, _p, _p]
for _n in ("orc_e4m3_encode_array", "orc_e2m1_encode_array"):
    getattr(_lib, _n).restype = None
    getattr(_lib, _n).argtypes = [_p, _p, _l]
for _n in ("orc_e4m3_encode_bits", "orc_e2m1_encode_bits"):
    getattr(_lib, _n).restype = None
    getattr(_lib, _n).argtypes = [C.c_uint32, _p, _l]
_lib.orc_mx_exponent_bits.restype = None
_lib.orc_mx_exponent_bits.argtypes = [C.c_uint32, _f, _p, _l]
_lib.orc_mx_exponent_array.restype = None
_lib.orc_mx_exponent_array.argtypes = [_p, _f, _p, _l]
_lib.orc_f32_to_bf16_array.restype = None
_lib.orc_f32_to_bf16_array.argtypes = [_p, _p, _l]


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _mode(m):
    return MODES[m] if isinstance(m, str) else int(m)


def _layout(l):
    return LAYOUTS[l] if isinstance(l, str) else int(l)


# ---- scalar formats -------------------------------------------------------

def e4m3_encode(x):
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    _lib.orc_e4m3_encode_array(_ptr(x), _ptr(out), x.size)
    return out


def e2m1_encode(x):
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    _lib.orc_e2m1_encode_array(_ptr(x), _ptr(out), x.size)
    return out


def e4m3_encode_bits(start, n):
    """Codes of the binary32 values whose bit patterns are start .. start+n-1."""
    out = np.empty(n, np.uint8)
    _lib.orc_e4m3_encode_bits(start, _ptr(out), n)
    return out


def e2m1_encode_bits(start, n):
    out = np.empty(n, np.uint8)
    _lib.orc_e2m1_encode_bits(start, _ptr(out), n)
    return out


def mx_exponent_bits(start, n, qmax):
    """e8m0 bytes of blocks whose maxima are |bit patterns start .. start+n-1| (0xFF: not finite)."""
    out = np.empty(n, np.uint8)
    _lib.orc_mx_exponent_bits(start, float(qmax), _ptr(out), n)
    return out


def e4m3_decode(c):
    return np.array([_lib.orc_e4m3_decode(int(v)) for v in np.ravel(c)], np.float32).reshape(np.shape(c))


def e2m1_decode(c):
    return np.array([_lib.orc_e2m1_decode(int(v)) for v in np.ravel(c)], np.float32).reshape(np.shape(c))


def mx_exponent(amax, qmax):
    a = _c(amax, np.float32)
    out = np.empty(a.shape, np.int32)
    _lib.orc_mx_exponent_array(_ptr(a), float(qmax), _ptr(out), a.size)
    return out


def f32_to_bf16(x):
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    _lib.orc_f32_to_bf16_array(_ptr(x), _ptr(out), x.size)
    return out


def bf16_to_f32(b):
    return (_c(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---- rows -----------------------------------------------------------------

def row_bytes(mode, H):
    """(data bytes, scale bytes) of one quantised row."""
    m = _mode(mode)
    return int(_lib.orc_row_data_bytes(m, H)), int(_lib.orc_row_scale_bytes(m, H))


def quant_row(mode, x, e4m3_qmax=0.0):
    """Quantise one row: bf16 bits (uint16) or fp32 values.  Returns (data, scale) bytes."""
    m = _mode(mode)
    H = int(np.size(x))
    D, S = row_bytes(m, H)
    data = np.zeros(D, np.uint8)
    scale = np.zeros(max(S, 1), np.uint8)
    if np.asarray(x).dtype == np.uint16:
        xb = _c(x, np.uint16)
        _lib.orc_quant_row_bf16(m, H, float(e4m3_qmax), _ptr(xb), _ptr(data), _ptr(scale))
    else:
        xf = _c(x, np.float32)
        _lib.orc_quant_row_f32(m, H, float(e4m3_qmax), _ptr(xf), _ptr(data), _ptr(scale))
    return data, scale[:S]


def rows_max(R, T, K, E, M, layout, align=1):
    """Rows a receive buffer must hold (padded: E*R*M; packed: every entry valid)."""
    if _layout(layout) == 0:
        return E * R * M
    return R * T * K + E * (align - 1)


def row_index(layout, R, M, e, slot, expert_offset=None):
    """Row of (expert e, slot) in the receive layout (no validity check)."""
    if _layout(layout) == 0:
        return np.asarray(e, np.int64) * (R * M) + np.asarray(slot, np.int64)
    return np.asarray(expert_offset, np.int64)[np.asarray(e, np.int64)] + np.asarray(slot, np.int64)


# ---- the path -------------------------------------------------------------

def layout(R, T, K, E, M, topk_idx, layout="padded", align=1):
    idx = _c(topk_idx, np.int64).reshape(R * T, K)
    N = R * T
    out = dict(
        tokens_per_rank=np.zeros((R, R), np.int32),
        tokens_per_expert=np.zeros((R, E), np.int32),
        is_token_in_rank=np.zeros((N, R), np.uint8),
        token_slot=np.zeros((N, K), np.int32),
        recv_count=np.zeros(E, np.int64),
        expert_offset=np.zeros(E + 1, np.int64) if _layout(layout) == 1 else None,
    )
    st = _lib.orc_layout(R, T, K, E, M, _layout(layout), align, _ptr(idx),
                         _ptr(out["tokens_per_rank"]), _ptr(out["tokens_per_expert"]),
                         _ptr(out["is_token_in_rank"]), _ptr(out["token_slot"]),
                         _ptr(out["recv_count"]), _ptr(out["expert_offset"]))
    out["status"] = int(st)
    return out


def dispatch_buffers(R, T, K, E, M, H, mode, layout="padded", align=1, weights=False, fill=True):
    """Output arrays for dispatch().  With fill, rows keep 0xAB bytes / -7 / nan
    until written, so tests can see which rows were written; without, the
    arrays are left uninitialised (only written rows are touched)."""
    rows = rows_max(R, T, K, E, M, layout, align)
    D, S = row_bytes(_mode(mode), H)
    mk = (lambda shape, dt, v: np.full(shape, v, dt)) if fill else \
        (lambda shape, dt, v: np.empty(shape, dt))
    return dict(recv_data=mk((rows, D), np.uint8, 0xAB),
                recv_scale=mk((rows, max(S, 1)), np.uint8, 0xAB),
                src_info=mk(rows, np.int32, -7),
                recv_weights=mk(rows, np.float32, np.nan) if weights else None)


def dispatch(R, T, K, E, M, H, mode, x, topk_idx, token_slot, expert_offset=None,
             topk_weights=None, layout="padded", align=1, e4m3_qmax=0.0, out=None):
    """Returns dict(recv_data [rows, D] u8, recv_scale [rows, S] u8, src_info, recv_weights, status).

    `out` may hold arrays from dispatch_buffers(); otherwise they are made here."""
    m = _mode(mode)
    D, S = row_bytes(m, H)
    x = _c(x, np.uint16).reshape(R * T, H)
    idx = _c(topk_idx, np.int64)
    slot = _c(token_slot, np.int32)
    eo = None if expert_offset is None else _c(expert_offset, np.int64)
    w = None if topk_weights is None else _c(topk_weights, np.float32)
    if out is None:
        out = dispatch_buffers(R, T, K, E, M, H, m, layout, align, weights=w is not None)
    out = dict(out)
    if eo is not None and layout in ("packed", 1):  # the rows the offsets address must exist
        assert int(eo[-1]) <= out["recv_data"].shape[0], "expert_offset beyond the buffers' rows"
    st = _lib.orc_dispatch(R, T, K, E, M, H, m, float(e4m3_qmax), _layout(layout), _ptr(x),
                           _ptr(idx), _ptr(w), _ptr(slot), _ptr(eo), _ptr(out["recv_data"]),
                           _ptr(out["recv_scale"]), _ptr(out["src_info"]), _ptr(out["recv_weights"]))
    out["recv_scale"] = out["recv_scale"][:, :S]
    out["status"] = int(st)
    return out


def combine(R, T, K, E, M, H, y, topk_idx, topk_weights, token_slot, expert_offset=None,
            layout="padded", out=None):
    """y: expert outputs, bf16 bits [rows, H] in the receive layout.  Returns (out [N, H] u16, status)."""
    y = _c(y, np.uint16)
    idx = _c(topk_idx, np.int64)
    w = _c(topk_weights, np.float32)
    slot = _c(token_slot, np.int32)
    eo = None if expert_offset is None else _c(expert_offset, np.int64)
    if out is None:
        out = np.zeros((R * T, H), np.uint16)
    st = _lib.orc_combine(R, T, K, E, M, H, _layout(layout), _ptr(y), _ptr(idx), _ptr(w),
                          _ptr(slot), _ptr(eo), _ptr(out))
    return out, int(st)


def combine_row(yrows, w, valid):
    """One token: yrows [K, H] bf16 bits, w [K] f32, valid [K] bool -> [H] bf16 bits."""
    yrows = _c(yrows, np.uint16)
    K, H = yrows.shape
    ptrs = (C.c_void_p * K)(*[yrows.ctypes.data + k * H * 2 for k in range(K)])
    w = _c(w, np.float32)
    v = _c(valid, np.uint8)
    out = np.zeros(H, np.uint16)
    _lib.orc_combine_row(H, K, C.cast(ptrs, C.c_void_p), _ptr(w), _ptr(v), _ptr(out))
    return out


def combine_bwd(R, T, K, E, M, H, g, topk_idx, topk_weights, token_slot, expert_offset=None,
                layout="padded", align=1, unweighted=False):
    """Returns dict(grad_data [rows, H] u8, grad_scale [rows, H/32] u8, status)."""
    rows = rows_max(R, T, K, E, M, layout, align)
    g = _c(g, np.uint16).reshape(R * T, H)
    idx = _c(topk_idx, np.int64)
    w = _c(topk_weights, np.float32)
    slot = _c(token_slot, np.int32)
    eo = None if expert_offset is None else _c(expert_offset, np.int64)
    gd = np.full((rows, H), 0xAB, np.uint8)
    gs = np.full((rows, H // 32), 0xAB, np.uint8)
    st = _lib.orc_combine_bwd(R, T, K, E, M, H, _layout(layout), int(bool(unweighted)), _ptr(g),
                              _ptr(idx), _ptr(w), _ptr(slot), _ptr(eo), _ptr(gd), _ptr(gs))
    return dict(grad_data=gd, grad_scale=gs, status=int(st))


def combine_wgrad(R, T, K, E, M, H, g, y, topk_idx, token_slot, expert_offset=None,
                  layout="padded"):
    """Weight gradient dw [N, K] f32 (dot products of g [N, H] with the entries'
    expert rows y [rows, H], bf16 bits), and the status bits."""
    g = _c(g, np.uint16).reshape(R * T, H)
    y = _c(y, np.uint16)
    idx = _c(topk_idx, np.int64)
    slot = _c(token_slot, np.int32)
    eo = None if expert_offset is None else _c(expert_offset, np.int64)
    dw = np.zeros((R * T, K), np.float32)
    st = _lib.orc_combine_wgrad(R, T, K, E, M, H, _layout(layout), _ptr(g), _ptr(y), _ptr(idx),
                                _ptr(slot), _ptr(eo), _ptr(dw))
    return dw, int(st)


def combine_wgrad_gathered(g, yrows, valid):
    """g [N, H], yrows [N, K, H] bf16 bits, valid [N, K] -> (dw [N, K] f32,
    sum_h |g * y| [N, K] f64)."""
    yrows = _c(yrows, np.uint16)
    N, K, H = yrows.shape
    g = _c(g, np.uint16).reshape(N, H)
    v = _c(valid, np.uint8)
    dw = np.zeros((N, K), np.float32)
    mag = np.zeros((N, K), np.float64)
    _lib.orc_combine_wgrad_gathered(N, K, H, _ptr(g), _ptr(yrows), _ptr(v), _ptr(dw), _ptr(mag))
    return dw, mag


def expert_gemm(x, w, expert_offset, count, n_out, y=None):
    """Per-expert linear maps on packed rows: x [rows, H] bf16 bits, w [E, n_out, H]
    bf16 bits; rows expert_offset[e] .. + count[e] -> y [rows, n_out] bf16 bits
    (other rows of y untouched)."""
    x = _c(x, np.uint16)
    rows, H = x.shape
    w = _c(w, np.uint16)
    E = w.shape[0]
    eo = _c(expert_offset, np.int64)
    cnt = _c(count, np.int64)
    if y is None:
        y = np.zeros((rows, n_out), np.uint16)
    _lib.orc_expert_gemm(E, H, n_out, _ptr(eo), _ptr(cnt), _ptr(x), _ptr(w), _ptr(y))
    return y


def expert_gemm_mx(xc, xs, wc, ws, expert_offset, count, n_out, y=None):
    """Per-expert linear maps on MXFP8 operands: xc [rows, H] e4m3 codes,
    xs [rows, H/32] e8m0 bytes, wc [E, n_out, H] e4m3 codes, ws [E, n_out, H/32]
    e8m0 bytes; rows expert_offset[e] .. + count[e] -> y [rows, n_out] bf16 bits
    (other rows of y untouched)."""
    xc = _c(xc, np.uint8)
    rows, H = xc.shape
    xs = _c(xs, np.uint8)
    wc = _c(wc, np.uint8)
    ws = _c(ws, np.uint8)
    E = wc.shape[0]
    assert xs.shape == (rows, H // 32) and wc.shape == (E, n_out, H) and ws.shape == (E, n_out, H // 32)
    eo = _c(expert_offset, np.int64)
    cnt = _c(count, np.int64)
    if y is None:
        y = np.zeros((rows, n_out), np.uint16)
    _lib.orc_expert_gemm_mx(E, H, n_out, _ptr(eo), _ptr(cnt), _ptr(xc), _ptr(xs), _ptr(wc),
                            _ptr(ws), _ptr(y))
    return y


def expert_ffn_mx(xc, xs, w1c, w1s, w2c, w2s, expert_offset, count):
    """The experts' gated MLP on MXFP8 operands: GMM1 (h = x . W1^T, fp32),
    SwiGLU (z = silu(gate) * up, gate = h[:, :I], up = h[:, I:]), MXFP8 requant
    of z, GMM2 (y = zq . W2^T, bf16).  xc [rows, H] e4m3 codes, xs [rows, H/32];
    w1c [E, 2I, H], w1s [E, 2I, H/32]; w2c [E, H, I], w2s [E, H, I/32].
    Returns dict(h [rows, 2I] f32, z [rows, I] f32, zc [rows, I] u8,
    zs [rows, I/32] u8, y [rows, H] bf16 bits); rows outside every expert stay 0."""
    xc, xs = _c(xc, np.uint8), _c(xs, np.uint8)
    w1c, w1s, w2c, w2s = (_c(a, np.uint8) for a in (w1c, w1s, w2c, w2s))
    rows, H = xc.shape
    E, N1 = w1c.shape[0], w1c.shape[1]
    I = N1 // 2
    assert xs.shape == (rows, H // 32) and w1c.shape == (E, N1, H) and w1s.shape == (E, N1, H // 32)
    assert w2c.shape == (E, H, I) and w2s.shape == (E, H, I // 32) and I % 32 == 0
    eo, cnt = _c(expert_offset, np.int64), _c(count, np.int64)
    out = dict(h=np.zeros((rows, N1), np.float32), z=np.zeros((rows, I), np.float32),
               zc=np.zeros((rows, I), np.uint8), zs=np.zeros((rows, I // 32), np.uint8),
               y=np.zeros((rows, H), np.uint16))
    _lib.orc_expert_ffn_mx(E, H, I, _ptr(eo), _ptr(cnt), _ptr(xc), _ptr(xs), _ptr(w1c), _ptr(w1s),
                           _ptr(w2c), _ptr(w2s), _ptr(out["h"]), _ptr(out["z"]), _ptr(out["zc"]),
                           _ptr(out["zs"]), _ptr(out["y"]))
    return out


def expert_gemm_mxfp4(xc, xs, wc, ws, expert_offset, count, n_out, y=None):
    """Per-expert linear maps on MXFP4 operands: xc [rows, H/2] packed e2m1 codes
    (even element in the low nibble), xs [rows, H/32] e8m0 bytes, wc [E, n_out, H/2],
    ws [E, n_out, H/32]; rows expert_offset[e] .. + count[e] -> y [rows, n_out] bf16
    bits (other rows of y untouched)."""
    xc = _c(xc, np.uint8)
    rows, D = xc.shape
    H = 2 * D
    xs = _c(xs, np.uint8)
    wc = _c(wc, np.uint8)
    ws = _c(ws, np.uint8)
    E = wc.shape[0]
    assert xs.shape == (rows, H // 32) and wc.shape == (E, n_out, D) and ws.shape == (E, n_out, H // 32)
    eo = _c(expert_offset, np.int64)
    cnt = _c(count, np.int64)
    if y is None:
        y = np.zeros((rows, n_out), np.uint16)
    _lib.orc_expert_gemm_mxfp4(E, H, n_out, _ptr(eo), _ptr(cnt), _ptr(xc), _ptr(xs), _ptr(wc),
                               _ptr(ws), _ptr(y))
    return y


def combine_gathered(yrows, w, valid):
    """Tokens whose K expert rows are gathered: yrows [N, K, H] bf16 bits,
    w [N, K] f32, valid [N, K] -> out [N, H] bf16 bits."""
    yrows = _c(yrows, np.uint16)
    N, K, H = yrows.shape
    w = _c(w, np.float32)
    v = _c(valid, np.uint8)
    out = np.zeros((N, H), np.uint16)
    _lib.orc_combine_gathered(N, K, H, _ptr(yrows), _ptr(w), _ptr(v), _ptr(out))
    return out


def bwd_row(g_row, w, unweighted=False):
    """One entry of the combine backward: (e4m3 data [H], e8m0 scales [H/32])."""
    g_row = _c(g_row, np.uint16)
    H = g_row.size
    d = np.zeros(H, np.uint8)
    s = np.zeros(H // 32, np.uint8)
    _lib.orc_bwd_row(H, float(w), int(bool(unweighted)), _ptr(g_row), _ptr(d), _ptr(s))
    return d, s


def dequant_row(mode, data, scale, H):
    """fp32 values of one quantised row (data bytes, scale bytes)."""
    d = _c(data, np.uint8)
    sc = _c(scale, np.uint8) if np.size(scale) else np.zeros(1, np.uint8)
    out = np.zeros(H, np.float32)
    _lib.orc_dequant_row(_mode(mode), H, _ptr(d), _ptr(sc), _ptr(out))
    return out


def combine_gathered_q(mode, data, scale, w, valid, H):
    """Tokens whose K rows are quantised: data [N, K, D] u8, scale [N, K, S] u8,
    w [N, K] f32, valid [N, K] -> out [N, H] bf16 bits."""
    m = _mode(mode)
    d = _c(data, np.uint8)
    N, K = d.shape[0], d.shape[1]
    D, S = row_bytes(m, H)
    sc = _c(scale, np.uint8) if S else np.zeros((N, K, 1), np.uint8)
    w = _c(w, np.float32)
    v = _c(valid, np.uint8)
    out = np.zeros((N, H), np.uint16)
    _lib.orc_combine_gathered_q(m, N, K, H, _ptr(d), _ptr(sc), _ptr(w), _ptr(v), _ptr(out))
    return out
