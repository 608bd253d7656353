"""The C ABI without a GPU: libep.so loads, exports every function that
include/ep.h declares, sizes buffers, and rejects invalid arguments on the
host before any launch (no CUDA call is reached on these paths)."""
import ctypes as C
import os
import re

import pytest

import combine_ep_dispatch_04_b200 as ep
from combine_ep_dispatch_04_b200.ep import lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(ep_[a-z0-9_]+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported():
    names = _declared_functions()
    assert {"ep_dispatch_layout", "ep_dispatch", "ep_combine", "ep_combine_backward",
            "ep_buffer_sizes", "ep_get_status"} <= names
    for n in sorted(names):
        assert hasattr(lib, n), n


def _cfg(**kw):
    base = dict(R=8, T=128, M=128, K=8, E=256, H=7168, quant="e4m3_b128")
    base.update(kw)
    return ep.make_config(base["R"], base["T"], base["M"], base["K"], base["E"], base["H"],
                          base["quant"], base.get("layout", "padded"), base.get("expert_align", 1),
                          base.get("e4m3_qmax", 0.0), base.get("flags", 0))


def test_sizes_padded_decode_shape():
    s = ep.ep_buffer_sizes(_cfg())
    assert s["rows"] == 256 * 8 * 128
    assert s["data_row_bytes"] == 7168 and s["scale_row_bytes"] == 4 * 56
    assert s["recv_scale_offset"] % 256 == 0
    assert s["recv_bytes"] == s["recv_scale_offset"] + s["rows"] * 224
    assert s["expert_out_bytes"] == s["rows"] * 7168 * 2
    assert s["grad_bytes"] == s["grad_scale_offset"] + s["rows"] * 7168 // 32


@pytest.mark.parametrize("quant,D,S", [("bf16", 2048, 0), ("int8_token", 1024, 4),
                                        ("e4m3_b128", 1024, 32), ("mxfp8", 1024, 32),
                                        ("mxfp4", 512, 32)])
def test_sizes_packed_every_mode(quant, D, S):
    s = ep.ep_buffer_sizes(_cfg(R=4, T=10, M=16, K=3, E=8, H=1024, quant=quant, layout="packed",
                                expert_align=4))
    assert s["rows"] == 4 * 10 * 3 + 8 * 3
    assert (s["data_row_bytes"], s["scale_row_bytes"]) == (D, S)


@pytest.mark.parametrize("bad", [
    dict(R=0), dict(M=0), dict(T=-1), dict(T=129), dict(K=0), dict(K=17), dict(E=0),
    dict(E=1025 * 8), dict(E=255), dict(H=0), dict(H=48), dict(H=8224), dict(H=7168 + 32),
    dict(quant=7), dict(layout=2), dict(expert_align=0), dict(e4m3_qmax=449.0),
    dict(e4m3_qmax=float("nan")), dict(e4m3_qmax=-1.0), dict(flags=0x8000),
    dict(flags=ep.F_LAYOUT_MULTI_CTA | ep.F_LAYOUT_SINGLE_CTA),
    dict(flags=ep.F_LAYOUT_CLUSTER | ep.F_LAYOUT_SINGLE_CTA),
    dict(flags=ep.F_LAYOUT_CLUSTER | ep.F_LAYOUT_MULTI_CTA),
    dict(quant="e4m3_b128", H=96),
    dict(quant="bf16", flags=ep.F_ROUND_SCALE), dict(quant="int8_token", flags=ep.F_ROUND_SCALE),
    dict(quant="mxfp8", flags=ep.F_UE8M0), dict(quant="int8_token", flags=ep.F_UE8M0),
    dict(quant="bf16", flags=ep.F_UE8M0 | ep.F_ROUND_SCALE),
])
def test_invalid_configs_rejected(bad):
    with pytest.raises(ep.EpError) as ei:
        ep.ep_buffer_sizes(_cfg(**bad))
    assert ei.value.status == 1


@pytest.mark.parametrize("H,flags,S", [
    (7168, 0, 224), (7168, ep.F_ROUND_SCALE, 224), (7168, ep.F_UE8M0, 56),
    (7168, ep.F_UE8M0 | ep.F_ROUND_SCALE, 56), (384, ep.F_UE8M0, 4), (640, ep.F_UE8M0, 8),
])
def test_sizes_e4m3_scale_options(H, flags, S):
    s = ep.ep_buffer_sizes(_cfg(H=H, flags=flags))
    assert s["scale_row_bytes"] == S and s["data_row_bytes"] == H
    assert s["recv_bytes"] == s["recv_scale_offset"] + s["rows"] * S


@pytest.mark.parametrize("quant", ["mxfp8", "mxfp4"])
def test_round_scale_accepted_for_mx(quant):
    a = ep.ep_buffer_sizes(_cfg(H=1024, quant=quant))
    b = ep.ep_buffer_sizes(_cfg(H=1024, quant=quant, flags=ep.F_ROUND_SCALE))
    assert a == b


def test_index_dtype_follows_the_flag():
    import torch
    assert ep.idx_dtype(_cfg()) == torch.int64
    assert ep.idx_dtype(_cfg(flags=ep.F_IDX_I32)) == torch.int32


def test_entry_points_reject_before_any_launch():
    """Null buffers, a null config and a bad config are refused on the host:
    these calls reach no CUDA API (there is no device here)."""
    cfg = _cfg()
    null = C.c_void_p(0)
    z = C.c_size_t(0)
    n0 = ep.ep_kernel_launches()
    assert lib.ep_dispatch_layout(None, *([null] * 9), z, null, null) == 1
    assert lib.ep_dispatch_layout(C.byref(cfg), *([null] * 9), z, null, null) == 1
    assert lib.ep_dispatch(C.byref(cfg), *([null] * 6), z, null, z, null, z, null, null) == 1
    assert lib.ep_combine(C.byref(cfg), null, z, *([null] * 7)) == 1
    assert lib.ep_combine_backward(C.byref(cfg), *([null] * 6), z, null, null) == 1
    assert lib.ep_combine_backward_weights(C.byref(cfg), null, null, z, *([null] * 6)) == 1
    qcfg = _cfg(quant="mxfp8", flags=ep.F_COMBINE_QUANTIZED)
    fake = C.c_void_p(0x1000)
    assert lib.ep_combine_backward_weights(C.byref(qcfg), fake, fake, z, *([fake] * 5), null) == 2
    assert lib.ep_get_status(null, None, null) == 1
    bad = _cfg(E=255)
    big = C.c_size_t(1 << 40)
    assert lib.ep_dispatch(C.byref(bad), *([fake] * 6), big, fake, big, fake, big, fake,
                           null) == 1
    # misaligned vector buffers
    odd = C.c_void_p(0x1008)
    assert lib.ep_dispatch(C.byref(cfg), odd, *([fake] * 5), big, fake, big, fake, big, fake,
                           null) == 3
    assert lib.ep_copy(fake, fake, 24, null) == 1
    assert lib.ep_copy(odd, fake, 32, null) == 3
    assert lib.ep_cvt_sweep(4, 0, 16, fake, null) == 1
    assert lib.ep_cvt_sweep(0, 0xFFFFFFF0, 17, fake, null) == 1
    assert ep.ep_kernel_launches() == n0


# ---------------------------------------------------------------------------
# buffer sizes stated by a C caller: one byte short -> EP_ERR_BUFFER_TOO_SMALL
# before any launch ("DeepEP topk_idx_t Custom Dtype Requirements", Runtime
# Validation: checks come before GPU work)
# ---------------------------------------------------------------------------
_F = C.c_void_p(0x10000)   # a non-null, 16-byte aligned pointer that is never dereferenced
_N = C.c_void_p(0)


def _short_calls():
    """(name, which buffer, call(sizes) -> status) for every sized buffer of every
    entry point; `sizes` maps buffer -> byte count."""
    pad = _cfg(R=4, T=16, M=16, K=4, E=16, H=1024, quant="mxfp8")
    pk = _cfg(R=4, T=16, M=16, K=4, E=16, H=1024, quant="mxfp8", layout="packed")
    pkq = _cfg(R=4, T=16, M=16, K=4, E=16, H=1024, quant="mxfp8", layout="packed",
               flags=ep.F_COMBINE_QUANTIZED)
    bfp = _cfg(R=4, T=16, M=16, K=4, E=16, H=1024, quant="bf16", layout="packed")
    Z = C.c_size_t
    out = []

    def add(name, cfg, need, fn):
        out.append((name, cfg, need, fn))
    for cfg in (pad, pk):
        s = ep.ep_buffer_sizes(cfg)
        add("ep_dispatch_layout", cfg, {"workspace": s["workspace_bytes"]},
            lambda c, z: lib.ep_dispatch_layout(C.byref(c), _F, _F, _F, _F, _F, _F, _F, _N, _F,
                                                Z(z["workspace"]), _F, _N))
        need = {"recv_buf": s["recv_bytes"], "src_info": s["src_info_bytes"],
                "recv_weights": s["recv_weights_bytes"]}
        add("ep_dispatch", cfg, need,
            lambda c, z: lib.ep_dispatch(C.byref(c), _F, _F, _F, _F, _F, _F, Z(z["recv_buf"]), _F,
                                         Z(z["src_info"]), _F, Z(z["recv_weights"]), _F, _N))
        add("ep_dispatch_with_layout", cfg, dict(need, workspace=s["workspace_bytes"]),
            lambda c, z: lib.ep_dispatch_with_layout(
                C.byref(c), _F, _F, _F, _F, _F, _F, _F, _F, _F, _N, _F, Z(z["workspace"]), _F,
                Z(z["recv_buf"]), _F, Z(z["src_info"]), _F, Z(z["recv_weights"]), _F, _N))
        add("ep_combine", cfg, {"y": s["expert_out_bytes"]},
            lambda c, z: lib.ep_combine(C.byref(c), _F, Z(z["y"]), _F, _F, _F, _F, _F, _F, _N))
        add("ep_combine_backward", cfg, {"grad_buf": s["grad_bytes"]},
            lambda c, z: lib.ep_combine_backward(C.byref(c), _F, _F, _F, _F, _F, _F,
                                                 Z(z["grad_buf"]), _F, _N))
        add("ep_combine_backward_weights", cfg, {"y": s["expert_out_bytes"]},
            lambda c, z: lib.ep_combine_backward_weights(C.byref(c), _F, _F, Z(z["y"]), _F, _F,
                                                         _F, _F, _F, _N))
    s = ep.ep_buffer_sizes(pkq)
    add("ep_combine (quantised y)", pkq, {"y": s["recv_bytes"]},
        lambda c, z: lib.ep_combine(C.byref(c), _F, Z(z["y"]), _F, _F, _F, _F, _F, _F, _N))
    s = ep.ep_buffer_sizes(bfp)
    rows = s["rows"]
    add("ep_expert_gemm", bfp, {"recv_buf": rows * 2048, "y": rows * 512 * 2},
        lambda c, z: lib.ep_expert_gemm(C.byref(c), _F, Z(z["recv_buf"]), _F, _F, _F, 512, _F,
                                        Z(z["y"]), _F, _N))
    add("ep_moe_forward", bfp, {"workspace": s["workspace_bytes"], "recv_buf": s["recv_bytes"],
                                "src_info": s["src_info_bytes"], "y": s["expert_out_bytes"]},
        lambda c, z: lib.ep_moe_forward(C.byref(c), _F, _F, _F, _F, _N, _F, _F, _F, _F,
                                        Z(z["workspace"]), _F, Z(z["recv_buf"]), _F,
                                        Z(z["src_info"]), _F, Z(z["y"]), _F, _F, _N))
    s = ep.ep_buffer_sizes(pk)
    zb, _ = ep.ep_ffn_buffer_bytes(pk, 256)
    add("ep_expert_ffn_mx", pk, {"recv_buf": s["recv_bytes"], "z_buf": zb,
                                 "y": s["expert_out_bytes"]},
        lambda c, z: lib.ep_expert_ffn_mx(C.byref(c), _F, Z(z["recv_buf"]), _F, _F, _F, _F, _F, _F,
                                          256, _F, Z(z["z_buf"]), _F, Z(z["y"]), _F, _N))
    add("ep_moe_forward_ffn", pk, {"workspace": s["workspace_bytes"], "recv_buf": s["recv_bytes"],
                                   "src_info": s["src_info_bytes"], "z_buf": zb,
                                   "y": s["expert_out_bytes"]},
        lambda c, z: lib.ep_moe_forward_ffn(C.byref(c), _F, _F, _F, _F, _F, _F, _F, 256, _F, _F, _F,
                                            _F, Z(z["workspace"]), _F, Z(z["recv_buf"]), _F,
                                            Z(z["src_info"]), _F, Z(z["z_buf"]), _F, Z(z["y"]), _F,
                                            _F, _N))
    rows = s["rows"]
    add("ep_expert_gemm_mx", pk, {"recv_buf": s["recv_bytes"], "y": rows * 224 * 2},
        lambda c, z: lib.ep_expert_gemm_mx(C.byref(c), _F, Z(z["recv_buf"]), _F, _F, _F, _F, 224,
                                           _F, Z(z["y"]), _F, _N))
    return out


_CASES = [(name, cfg, need, fn, buf) for name, cfg, need, fn in _short_calls() for buf in need]


@pytest.mark.parametrize("case", _CASES,
                         ids=[f"{c[0]}-{'padded' if c[1].layout == 0 else 'packed'}-{c[4]}"
                              for c in _CASES])
def test_one_byte_short_buffer_is_refused_before_any_launch(case):
    name, cfg, need, fn, buf = case
    sizes = dict(need)
    sizes[buf] = need[buf] - 1
    n0 = ep.ep_kernel_launches()
    assert fn(cfg, sizes) == ep.ERR_BUFFER_TOO_SMALL, (name, buf)
    assert ep.ep_kernel_launches() == n0


def test_status_strings():
    for s in range(8):
        assert lib.ep_status_string(s)
    assert b"unknown" in lib.ep_status_string(99)


def test_gemm_pair_flag_is_known():
    """EP_F_GEMM_CTA_PAIRS is a valid flag of any configuration (no launch)."""
    cfg = ep.make_config(2, 16, 16, 2, 4, 256, "bf16", "packed", 1, 0.0, ep.F_GEMM_CTA_PAIRS)
    assert ep.ep_buffer_sizes(cfg)["rows"] > 0
