"""Parity of the CUDA path with the oracle, through the C ABI, on cuda:0.

Bit-exact: layout outputs, slots, counts, src_info, recv weights, quantised
codes and scales, combine-backward rows and the device status word.  Combine:
within 1 bf16 ulp of the oracle (both accumulate in fp32 with one FMA per
entry in k order, so the results are expected to be identical).

Sizes: every named workload at full size where the oracle finishes in
seconds (tiny, decode, skewed, large), reduced-T variants with a ragged tail
for the others, and the full prefill workload checked on sampled tokens.
"""
import numpy as np
import pytest
import torch

import combine_ep_dispatch_04_b200 as ep
import oracle
import synth
from harness import Guards, Run, bf16_dev, to_np_u16, ulp_distance

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mode", ["bf16", "int8_token"])
@pytest.mark.parametrize("layout", ["padded", "packed"])
def test_tiny_workload(mode, layout):
    w = synth.workload("tiny")
    r = Run(w, mode, layout=layout, stats=True)
    r.check_layout()
    assert r.check_dispatch() == (r.idx >= 0).sum()
    r.check_combine()


@pytest.mark.parametrize("qmax", [0.0, 127.0])
def test_decode_workload_full_size(qmax):
    w = synth.workload("decode")
    r = Run(w, "e4m3_b128", qmax=qmax)
    r.check_layout()
    assert r.check_dispatch() == w["N"] * w["K"]
    r.check_combine()


def test_skewed_workload_full_size():
    w = synth.workload("skewed")
    r = Run(w, "int8_token")
    r.check_layout()
    r.check_dispatch()
    r.check_combine()


@pytest.mark.parametrize("align", [1, 16])
@pytest.mark.parametrize("unweighted", [False, True])
def test_prefill_workload_ragged(align, unweighted):
    w = synth.workload("prefill", T=97)  # 3104 tokens: many layout chunks, ragged tail
    r = Run(w, "mxfp8", layout="packed", align=align, backward=True, bwd_unweighted=unweighted)
    r.check_layout()
    r.check_dispatch()
    r.check_combine()
    r.check_backward()


def test_large_workload_full_size():
    w = synth.workload("large")
    r = Run(w, "mxfp4", layout="packed")
    r.check_layout()
    r.check_dispatch()
    sample = np.random.default_rng(5).choice(w["N"], 2048, replace=False)
    r.check_combine(tokens=np.sort(sample))
    # the benchmark's quantised combine (pipelined kernel) of the dispatched MXFP4 rows
    from harness import combine_dispatched_check
    combine_dispatched_check(r, np.sort(sample[:600]))


def test_prefill_workload_full_size_sampled():
    """The full prefill workload (131072 tokens, ~1M entries) in the launch
    configuration the benchmark uses; outputs checked on sampled tokens and the
    layout checked in full."""
    w = synth.workload("prefill")
    r = Run(w, "mxfp8", layout="packed", backward=True)
    r.check_layout()
    rng = np.random.default_rng(11)
    sample = np.sort(np.concatenate([rng.choice(w["N"], 1500, replace=False),
                                     [0, w["N"] - 1]]))
    r.check_dispatch(tokens=sample)
    r.check_combine(tokens=sample)
    r.check_backward(tokens=sample[:300])
    # the benchmark's quantised combine (pipelined kernel) of the dispatched MXFP8 rows
    from harness import combine_dispatched_check
    combine_dispatched_check(r, sample[::3])


# ---------------------------------------------------------------------------
# both layout paths agree with the oracle (and so with each other)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name,override", [
    ("decode", {}), ("skewed", dict(T=100)), ("large", dict(T=40)), ("tiny", {}),
    ("prefill", dict(T=33, E=1024)), ("skewed", dict(R=3, E=6, K=4, T=1000, M=1000)),
])
@pytest.mark.parametrize("path", [ep.F_LAYOUT_SINGLE_CTA, ep.F_LAYOUT_MULTI_CTA,
                                  ep.F_LAYOUT_CLUSTER])
def test_layout_paths(name, override, path):
    w = synth.workload(name, **override)
    r = Run(w, "bf16", layout="packed", align=4, flags=path)
    r.check_layout()


# ---------------------------------------------------------------------------
# edge cases
# ---------------------------------------------------------------------------
def _edge(R=2, T=8, M=8, K=3, E=8, H=256, x="normal"):
    w = synth.workload("tiny", R=R, T=T, M=M, K=K, E=E, H=H)
    w["x"] = x
    return w


@pytest.mark.parametrize("mode", ["bf16", "int8_token", "e4m3_b128", "mxfp8", "mxfp4"])
@pytest.mark.parametrize("layout", ["padded", "packed"])
def test_every_mode_small_ragged(mode, layout):
    w = _edge(R=3, T=13, M=16, K=4, E=12, H=640)
    r = Run(w, mode, layout=layout, backward=True)
    r.check_layout()
    r.check_dispatch()
    r.check_combine()
    r.check_backward()


@pytest.mark.parametrize("path", [ep.F_LAYOUT_SINGLE_CTA, ep.F_LAYOUT_MULTI_CTA,
                                  ep.F_LAYOUT_CLUSTER])
def test_zero_tokens(path):
    w = _edge(T=0)
    r = Run(w, "mxfp8", layout="packed", flags=path)
    r.check_layout()
    assert r.b.recv_count.sum().item() == 0
    assert r.b.expert_offset.cpu().numpy().tolist() == [0] * (w["E"] + 1)


def test_all_entries_masked():
    w = _edge()
    idx = np.full((w["N"], w["K"]), -1, np.int64)
    r = Run(w, "int8_token", idx=idx)
    r.check_layout()
    r.check_dispatch()
    assert not r.b.out.view(torch.int16).any().item()  # +0 everywhere


@pytest.mark.parametrize("mode", ["bf16", "mxfp4"])
def test_k1_r1_and_one_expert_per_rank(mode):
    for (R, E, K) in [(1, 4, 1), (4, 4, 2), (1, 1, 1)]:
        w = _edge(R=R, E=E, K=K, T=7, M=9, H=128)
        r = Run(w, mode)
        r.check_layout()
        r.check_dispatch()
        r.check_combine()


@pytest.mark.parametrize("mode,H", [("bf16", 32), ("int8_token", 32), ("mxfp8", 32),
                                    ("mxfp4", 32), ("e4m3_b128", 128), ("mxfp8", 8192),
                                    ("int8_token", 8192)])
def test_min_and_max_hidden(mode, H):
    w = _edge(H=H, T=5, M=5)
    r = Run(w, mode, layout="packed", backward=True)
    r.check_layout()
    r.check_dispatch()
    r.check_combine()
    r.check_backward()


def test_duplicates_overflow_padded_capacity():
    # every entry of every token on expert 0: 2*6*3 entries > cap = 2*6
    w = _edge(R=2, T=6, M=6, K=3, E=4)
    idx = np.zeros((w["N"], w["K"]), np.int64)
    r = Run(w, "bf16", idx=idx)
    assert r.status & ep.DEV_CAPACITY_OVERFLOW
    r.check_layout()
    r.check_dispatch()
    r.check_combine()  # entries beyond the capacity contribute nothing


def test_duplicates_fit_packed():
    w = _edge(R=2, T=6, M=6, K=3, E=4)
    idx = np.zeros((w["N"], w["K"]), np.int64)
    idx[::2, 1] = 3
    r = Run(w, "mxfp8", layout="packed", idx=idx, backward=True)
    assert r.status == 0
    r.check_layout()
    r.check_dispatch()
    r.check_combine()
    r.check_backward()


def test_full_capacity_expert():
    # T == M and every token of every rank picks expert 0 once: slot R*M-1 is used
    w = _edge(R=4, T=8, M=8, K=2, E=8)
    idx = np.stack([np.zeros(w["N"], np.int64), np.arange(w["N"]) % 7 + 1], axis=1)
    r = Run(w, "int8_token", idx=idx)
    assert r.status == 0
    assert r.b.recv_count[0].item() == w["R"] * w["M"]
    r.check_layout()
    r.check_dispatch()
    r.check_combine()


def test_bad_indices_flagged_and_skipped():
    w = _edge()
    idx, wts = synth.make_routing(w)
    idx[1, 0] = w["E"]
    idx[3, 2] = -5
    idx[4, 1] = 1 << 40
    r = Run(w, "e4m3_b128", idx=idx, wts=wts)
    assert r.status & ep.DEV_BAD_INDEX
    r.check_layout()
    r.check_dispatch()
    r.check_combine()
    assert ep.ep_get_status(r.b.dev_status) == 0  # read-and-clear


def test_zero_and_signed_zero_rows():
    w = _edge(H=256)
    x = synth.make_x(w)
    x[0] = 0
    x[1] = 0x8000  # -0.0 everywhere
    x[2, :128] = 0  # one zero 128-block, one normal block
    x[3, 32:64] = 0x8000
    for mode in ["int8_token", "e4m3_b128", "mxfp8", "mxfp4", "bf16"]:
        r = Run(w, mode, layout="packed", x=x)
        r.check_dispatch()


def test_tiny_magnitudes_and_outliers():
    w = _edge(H=512)
    x = synth.make_x(w)
    f = oracle.bf16_to_f32(x).copy()
    f[0] *= np.float32(2.0 ** -120)    # subnormal block maxima after the scale division
    f[1] *= np.float32(2.0 ** -126)
    f[2] *= np.float32(2.0 ** 100)
    f[3, ::7] *= 50
    x = synth.to_bf16_bits(f)
    for mode in ["int8_token", "e4m3_b128", "mxfp8", "mxfp4"]:
        r = Run(w, mode, layout="packed", x=x, backward=True)
        r.check_dispatch()
        r.check_backward()


def test_recv_weights_optional_and_deterministic():
    w = synth.workload("skewed", T=64)
    a = Run(w, "int8_token", with_weights=False)
    b = Run(w, "int8_token", with_weights=False)
    for name in ("token_slot", "recv_count", "recv_buf", "src_info", "out"):
        assert torch.equal(getattr(a.b, name), getattr(b.b, name)), name


def test_stats_accumulate():
    w = synth.workload("decode", T=16)
    r = Run(w, "bf16", stats=True)
    cnt = r.b.recv_count.clone()
    ep.ep_dispatch_layout(r.cfg, r.idx_d, r.b.token_slot, r.b.recv_count, r.b.workspace,
                          r.b.dev_status, cumulative_recv_stats=r.stats_d)
    torch.cuda.synchronize()
    assert torch.equal(r.stats_d, 2 * cnt)


def test_python_checks_reject_prequantised_input():
    w = _edge()
    cfg = ep.make_config(w["R"], w["T"], w["M"], w["K"], w["E"], w["H"], "mxfp8")
    b = ep.Buffers(cfg)
    x8 = torch.zeros((w["N"], w["H"]), dtype=torch.float8_e4m3fn, device="cuda")
    idx = torch.zeros((w["N"], w["K"]), dtype=torch.int64, device="cuda")
    with pytest.raises(TypeError):
        ep.ep_dispatch(cfg, x8, idx, b.token_slot, b.recv_buf, b.src_info, b.dev_status)
    with pytest.raises(TypeError):
        ep.ep_dispatch_layout(cfg, idx.int(), b.token_slot, b.recv_count, b.workspace,
                              b.dev_status)
    with pytest.raises(ValueError):
        ep.ep_dispatch_layout(cfg, idx.t().contiguous().t(), b.token_slot, b.recv_count,
                              b.workspace, b.dev_status)


@pytest.mark.parametrize("path", [ep.F_LAYOUT_SINGLE_CTA, ep.F_LAYOUT_MULTI_CTA,
                                  ep.F_LAYOUT_CLUSTER])
def test_layout_paths_bad_indices_and_duplicates(path):
    w = _edge(R=4, T=37, M=40, K=5, E=8)
    idx, wts = synth.make_routing(w)
    idx[::3, 1] = idx[::3, 0]          # duplicates
    idx[5, 2] = w["E"] + 3             # out of range
    idx[7, 0] = -9
    r = Run(w, "mxfp8", layout="packed", align=3, idx=idx, wts=wts, flags=path, stats=True)
    assert r.status & ep.DEV_BAD_INDEX
    r.check_layout()
    r.check_dispatch()


@pytest.mark.parametrize("mode", ["bf16", "int8_token", "e4m3_b128", "mxfp8", "mxfp4"])
@pytest.mark.parametrize("name,override,path", [
    ("decode", {}, 0), ("tiny", {}, 0), ("skewed", dict(T=64), ep.F_LAYOUT_MULTI_CTA),
    ("large", dict(T=40), ep.F_LAYOUT_SINGLE_CTA), ("prefill", dict(T=50), 0),
])
def test_dispatch_with_layout_equals_separate_calls(mode, name, override, path):
    """The one-call dispatch (whose kernel overlaps the layout) gives the bytes
    of ep_dispatch_layout + ep_dispatch, and so the oracle's."""
    w = synth.workload(name, **override)
    r = Run(w, mode, layout=w["layout"], flags=path, stats=True)
    r.check_layout()
    _check_one_call(r, w)


def _check_one_call(r, w, cfg=None):
    """ep_dispatch_with_layout on r's inputs (r.cfg unless cfg is given) against
    r's separate calls, every output byte for byte, the device status and a
    cumulative_recv_stats accumulated twice."""
    cfg = cfg or r.cfg
    b = ep.Buffers(cfg, recv_weights=True, expert_out=False)
    b.recv_buf.fill_(0xAB)
    b.src_info.fill_(-7)
    b.recv_weights.fill_(float("nan"))
    b.is_token_in_rank.fill_(7)
    b.tokens_per_rank.fill_(-3)
    b.tokens_per_expert.fill_(-3)
    stats = torch.full((w["E"],), 5, dtype=torch.int64, device="cuda")
    for _ in range(2):
        b.token_slot.fill_(-5)
        b.recv_count.fill_(-5)
        ep.ep_dispatch_with_layout(cfg, r.x_d, r.idx_d, b.token_slot, b.recv_count, b.workspace,
                                   b.recv_buf, b.src_info, b.dev_status, topk_weights=r.wts_d,
                                   tokens_per_rank=b.tokens_per_rank,
                                   tokens_per_expert=b.tokens_per_expert,
                                   is_token_in_rank=b.is_token_in_rank,
                                   expert_offset=b.expert_offset, cumulative_recv_stats=stats,
                                   recv_weights=b.recv_weights)
        assert ep.ep_get_status(b.dev_status) == r.status
    for name_ in ("token_slot", "recv_count", "tokens_per_rank", "tokens_per_expert",
                  "is_token_in_rank", "recv_buf", "src_info"):
        assert torch.equal(getattr(b, name_), getattr(r.b, name_)), name_
    assert torch.equal(b.recv_weights.nan_to_num(-1), r.b.recv_weights.nan_to_num(-1))
    if b.expert_offset is not None:
        assert torch.equal(b.expert_offset, r.b.expert_offset)
    if r.stats_d is not None:
        assert torch.equal(stats, 5 + 2 * r.stats_d)


@pytest.mark.parametrize("mode", ["bf16", "int8_token", "e4m3_b128", "mxfp8", "mxfp4"])
@pytest.mark.parametrize("case", ["dup_bad_masked", "capacity", "idx_i32", "k1_r1", "wide_e"])
def test_dispatch_with_layout_edges(mode, case):
    """The one-call layout + dispatch on edge routings, against the separate
    calls through a forced layout kernel and the oracle: duplicates within a
    token, out-of-range and negative indices, masked entries; slots past the
    capacity; int32 topk_idx; K = 1 on one rank; E = 1024 on 2 ranks."""
    flags, path = 0, ep.F_LAYOUT_SINGLE_CTA
    if case == "dup_bad_masked":
        w = _edge(R=4, T=37, M=40, K=5, E=8, H=2048)
        idx, wts = synth.make_routing(w)
        idx[::3, 1] = idx[::3, 0]
        idx[5, 2] = w["E"] + 3
        idx[7, 0] = -9
        idx[11, :] = -1
    elif case == "capacity":
        w = _edge(R=2, T=64, M=64, K=4, E=4, H=2048)
        idx = np.zeros((128, 4), np.int64)
        idx[:, 1:] = np.random.default_rng(2).integers(0, 4, (128, 3))
        wts = np.ones_like(idx, dtype=np.float32)
    elif case == "idx_i32":
        w = _edge(R=8, T=64, M=64, K=8, E=64, H=4096)
        idx, wts = synth.make_routing(w)
        flags = ep.F_IDX_I32
    elif case == "k1_r1":
        w = _edge(R=1, T=200, M=200, K=1, E=4, H=2048)
        idx, wts = synth.make_routing(w)
    else:
        w = _edge(R=2, T=100, M=100, K=8, E=1024, H=2048)
        idx, wts = synth.make_routing(w)
    r = Run(w, mode, layout="padded", idx=idx, wts=wts, flags=flags | path, stats=True)
    r.check_layout()
    r.check_dispatch()
    if case == "dup_bad_masked":
        assert r.status & ep.DEV_BAD_INDEX
    if case == "capacity":
        assert r.status & ep.DEV_CAPACITY_OVERFLOW
    cfg = ep.make_config(w["R"], w["T"], w["M"], w["K"], w["E"], w["H"], mode, "padded",
                         flags=flags)
    _check_one_call(r, w, cfg)


@pytest.mark.parametrize("mode", ["int8_token", "e4m3_b128", "mxfp8", "mxfp4"])
@pytest.mark.parametrize("name,override", [("decode", {}), ("tiny", {}), ("large", dict(T=40)),
                                           ("skewed", dict(T=64))])
def test_combine_of_quantized_expert_outputs(mode, name, override):
    w = synth.workload(name, **override)
    if mode == "e4m3_b128" and w["H"] % 128:
        pytest.skip("H % 128")
    from harness import combine_quantized_check
    r = Run(w, mode, layout=w["layout"])
    combine_quantized_check(r, seed=31 * len(mode) + len(name))


@pytest.mark.parametrize("special_weights", [False, True])
@pytest.mark.parametrize("mode", ["int8_token", "e4m3_b128", "mxfp8", "mxfp4"])
def test_combine_of_quantized_pipelined_kernel(mode, special_weights):
    """More than 2^20 granules a launch: the pipelined kernel (codes copied a
    granule ahead into shared memory, scale rows staged once) rather than the
    register kernel the smaller cases take.  Sampled tokens; random and special
    rows; ordinary and special weights."""
    from harness import combine_quantized_check, special_quantized_rows
    T = 80 if mode == "mxfp4" else 40
    w = synth.workload("large", T=T)
    gran = 32 if mode == "mxfp4" else 16
    assert w["R"] * T * (w["H"] // gran) > (1 << 20)
    idx, wts = synth.make_routing(w)
    if special_weights:
        pick = np.float32([0.0, -0.0, 1e-45, 1e-39, 1e-30, 0.5, -2.0, 3e38, np.inf, -np.inf,
                           np.nan, 7.0, 0.125])
        wts = pick[np.random.default_rng(13).integers(0, len(pick), wts.shape)]
    r = Run(w, mode, layout="packed", idx=idx, wts=wts)
    sample = np.sort(np.random.default_rng(3).choice(w["R"] * T, 400, replace=False))
    combine_quantized_check(r, tokens=sample, seed=41 + len(mode))
    combine_quantized_check(r, tokens=sample, seed=43 + len(mode), rows_fn=special_quantized_rows)


@pytest.mark.parametrize("mode", ["int8_token", "e4m3_b128", "mxfp8", "mxfp4"])
def test_combine_of_quantized_special_values(mode):
    """NaN codes, zero / subnormal / huge / infinite / NaN / negative scales,
    and every e8m0 byte: the decoder's exact fast path and its fallback."""
    from harness import combine_quantized_check, special_quantized_rows
    w = synth.workload("decode", T=24)
    r = Run(w, mode, layout="packed")
    combine_quantized_check(r, seed=7 + len(mode), rows_fn=special_quantized_rows)


# ---------------------------------------------------------------------------
# int32 topk_idx, and the E4M3-per-128 scale options (round_scale, UE8M0)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("mode", ["bf16", "e4m3_b128", "mxfp4"])
@pytest.mark.parametrize("path", [ep.F_LAYOUT_SINGLE_CTA, ep.F_LAYOUT_MULTI_CTA,
                                  ep.F_LAYOUT_CLUSTER])
def test_int32_topk_idx(mode, path):
    w = _edge(R=4, T=37, M=40, K=5, E=8, H=384)
    idx, wts = synth.make_routing(w)
    idx[::3, 1] = idx[::3, 0]          # duplicates
    idx[5, 2] = w["E"] + 3             # out of range
    idx[7, 0] = -9
    idx[9, 1] = -(1 << 31)
    r = Run(w, mode, layout="packed", align=2, idx=idx, wts=wts, flags=path | ep.F_IDX_I32,
            backward=True, stats=True)
    assert r.idx_d.dtype == torch.int32
    assert r.status & ep.DEV_BAD_INDEX
    r.check_layout()
    r.check_dispatch()
    r.check_combine()
    r.check_backward()


def test_int32_topk_idx_decode_and_one_call_dispatch():
    w = synth.workload("decode")
    r = Run(w, "e4m3_b128", flags=ep.F_IDX_I32)
    r.check_layout()
    r.check_dispatch(check_unwritten=False)
    r.check_combine()
    b = ep.Buffers(r.cfg)
    ep.ep_dispatch_with_layout(r.cfg, r.x_d, r.idx_d, b.token_slot, b.recv_count, b.workspace,
                               b.recv_buf, b.src_info, b.dev_status)
    assert torch.equal(b.token_slot, r.b.token_slot)
    ns, ks, rows = r.entries()
    rows_d = torch.from_numpy(rows).cuda()
    assert torch.equal(b.recv_data().index_select(0, rows_d), r.b.recv_data().index_select(0, rows_d))
    assert torch.equal(b.recv_scale().index_select(0, rows_d), r.b.recv_scale().index_select(0, rows_d))


def test_int64_index_rejected_when_int32_expected():
    w = _edge()
    cfg = ep.make_config(w["R"], w["T"], w["M"], w["K"], w["E"], w["H"], "bf16",
                         flags=ep.F_IDX_I32)
    b = ep.Buffers(cfg)
    idx64 = torch.zeros((w["N"], w["K"]), dtype=torch.int64, device="cuda")
    with pytest.raises(TypeError):
        ep.ep_dispatch_layout(cfg, idx64, b.token_slot, b.recv_count, b.workspace, b.dev_status)


@pytest.mark.parametrize("flags", [ep.F_ROUND_SCALE, ep.F_UE8M0, ep.F_ROUND_SCALE | ep.F_UE8M0])
@pytest.mark.parametrize("qmax", [0.0, 240.0])
@pytest.mark.parametrize("H", [384, 7168])
def test_e4m3_round_scale_and_ue8m0(flags, qmax, H):
    w = _edge(R=3, T=13, M=16, K=4, E=12, H=H)
    r = Run(w, "e4m3_b128", layout="packed", qmax=qmax, flags=flags)
    assert r.sizes["scale_row_bytes"] == (4 * ((H // 128 + 3) // 4) if flags & ep.F_UE8M0
                                          else 4 * (H // 128))
    r.check_layout()
    r.check_dispatch()
    r.check_combine()


def test_e4m3_round_scale_extreme_magnitudes():
    w = _edge(H=512)
    x = synth.make_x(w)
    f = oracle.bf16_to_f32(x).copy()
    f[0] *= np.float32(2.0 ** -120)
    f[1] *= np.float32(2.0 ** -126)
    f[2] *= np.float32(2.0 ** 100)
    f[3, ::7] *= 50
    x = synth.to_bf16_bits(f)
    x[4] = 0
    x[5, :128] = 0x8000
    for flags in (ep.F_ROUND_SCALE, ep.F_UE8M0):
        for qmax in (0.0, 3.5):
            r = Run(w, "e4m3_b128", layout="packed", x=x, qmax=qmax, flags=flags)
            r.check_dispatch()


def test_e4m3_ue8m0_decode_workload():
    r = Run(synth.workload("decode"), "e4m3_b128", flags=ep.F_UE8M0)
    r.check_dispatch(check_unwritten=False)


@pytest.mark.parametrize("mode", ["mxfp8", "mxfp4"])
def test_round_scale_changes_nothing_for_mx(mode):
    w = _edge(R=3, T=13, M=16, K=4, E=12, H=640)
    a = Run(w, mode, layout="packed")
    b = Run(w, mode, layout="packed", flags=ep.F_ROUND_SCALE)
    assert torch.equal(a.b.recv_buf, b.b.recv_buf)


@pytest.mark.parametrize("flags", [ep.F_ROUND_SCALE, ep.F_UE8M0])
def test_combine_of_quantized_round_scale_rows(flags):
    from harness import combine_quantized_check, special_quantized_rows
    r = Run(synth.workload("decode", T=24), "e4m3_b128", layout="packed", flags=flags)
    combine_quantized_check(r, seed=3 + flags)
    combine_quantized_check(r, seed=5 + flags, rows_fn=special_quantized_rows)


@pytest.mark.parametrize("mode,flags", [("mxfp8", 0), ("mxfp4", 0), ("e4m3_b128", ep.F_UE8M0),
                                        ("e4m3_b128", ep.F_ROUND_SCALE), ("e4m3_b128", 0),
                                        ("int8_token", 0)])
def test_combine_of_quantized_special_weights(mode, flags):
    """Weights that are zero, negative zero, subnormal, huge, infinite or NaN,
    against scales of every kind: the weight-folded path must hand every case
    it cannot do exactly to the scale multiply."""
    from harness import combine_quantized_check, special_quantized_rows
    w = synth.workload("decode", T=24)
    idx, wts = synth.make_routing(w)
    pick = np.float32([0.0, -0.0, 1e-45, 1e-39, 1e-30, 0.5, -2.0, 3e38, np.inf, -np.inf, np.nan,
                       7.0, 0.125])
    wts = pick[np.random.default_rng(9).integers(0, len(pick), wts.shape)]
    r = Run(w, mode, layout="packed", idx=idx, wts=wts, flags=flags)
    combine_quantized_check(r, seed=11, rows_fn=special_quantized_rows)
    combine_quantized_check(r, seed=12)


# ---------------------------------------------------------------------------
# non-finite inputs and weights
# ---------------------------------------------------------------------------
def _nonfinite_x(w, with_nan=True):
    x = synth.make_x(w)
    f = oracle.bf16_to_f32(x).copy()
    f[0, 5] = np.inf                      # an infinite block maximum
    f[1, 130] = -np.inf
    f[2, ::97] = np.inf
    if with_nan:
        f[3, 17] = np.nan                 # NaN elements: left out of the block maximum
        f[4, ::13] = np.nan
        f[5, :128] = np.nan               # a block of NaNs only
    return synth.to_bf16_bits(f)


@pytest.mark.parametrize("mode,flags", [("bf16", 0), ("int8_token", 0), ("e4m3_b128", 0),
                                        ("e4m3_b128", ep.F_UE8M0), ("mxfp8", 0), ("mxfp4", 0)])
def test_nonfinite_inputs(mode, flags):
    w = _edge(R=2, T=8, M=8, K=3, E=8, H=512)
    x = _nonfinite_x(w)
    r = Run(w, mode, layout="packed", x=x, flags=flags, backward=True)
    r.check_dispatch()
    r.check_backward()


def test_backward_special_weights():
    """Weights that are zero, signed zero, subnormal, huge (products overflow),
    infinite or NaN, on gradients with large and non-finite values: the folded
    scale multiply must leave every such case to the two-multiply path."""
    w = _edge(R=2, T=16, M=16, K=4, E=8, H=512)
    idx, wts = synth.make_routing(w)
    pick = np.float32([0.0, -0.0, 1e-45, 1e-39, 3e38, -2.0, np.inf, -np.inf, np.nan, 0.25,
                       1.0, 7.5])
    wts = pick[np.random.default_rng(5).integers(0, len(pick), wts.shape)]
    r = Run(w, "mxfp8", layout="packed", idx=idx, wts=wts, backward=True,
            x=_nonfinite_x(w, with_nan=False))
    g = oracle.bf16_to_f32(r.g).copy()
    g[0] *= np.float32(2.0 ** 100)
    g[1, 3] = np.inf
    g[2, 9] = np.nan
    g[3] = 0.0
    r.g = synth.to_bf16_bits(g)
    r.g_d = bf16_dev(r.g)
    ep.ep_combine_backward(r.cfg, r.g_d, r.idx_d, r.wts_d, r.b.token_slot, r.b.grad_buf,
                           r.b.dev_status, expert_offset=r.b.expert_offset)
    r.check_backward()


# ---------------------------------------------------------------------------
# weight gradient of the combine
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name,override,layout", [
    ("decode", {}, "padded"), ("tiny", {}, "padded"), ("skewed", dict(T=64), "padded"),
    ("prefill", dict(T=40), "packed"), ("large", dict(T=24), "packed")])
def test_weights_grad(name, override, layout):
    w = synth.workload(name, **override)
    r = Run(w, "bf16", layout=layout)
    r.check_weights_grad()


def test_weights_grad_ragged_masked_bad_and_int32():
    w = _edge(R=3, T=13, M=16, K=5, E=12, H=608)
    idx, wts = synth.make_routing(w)
    idx[2, :] = -1
    idx[4, 1] = w["E"] + 1
    r = Run(w, "bf16", layout="packed", align=3, idx=idx, wts=wts, flags=ep.F_IDX_I32)
    assert r.status & ep.DEV_BAD_INDEX
    r.check_weights_grad()


def test_weights_grad_rejects_quantized_outputs():
    w = _edge()
    cfg = ep.make_config(w["R"], w["T"], w["M"], w["K"], w["E"], w["H"], "mxfp8",
                         flags=ep.F_COMBINE_QUANTIZED)
    b = ep.Buffers(cfg)
    g = torch.zeros((w["N"], w["H"]), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((w["N"], w["K"]), dtype=torch.int64, device="cuda")
    dw = torch.zeros((w["N"], w["K"]), dtype=torch.float32, device="cuda")
    with pytest.raises(ep.EpError) as ei:
        ep.ep_combine_backward_weights(cfg, g, b.y, idx, b.token_slot, dw, b.dev_status)
    assert ei.value.status == 2


def test_variable_tokens_per_rank_by_masking():
    """Ranks with different token counts T_r <= M ("Low-Latency Mode API",
    low_latency_combine: num_combined_tokens is the rank's dispatched token
    count): the ranks share T = max T_r and the missing tokens' topk_idx rows
    are -1.  They then take no slot, count nowhere, and combine to +0."""
    w = _edge(R=3, T=13, M=16, K=4, E=12, H=256)
    t_r = [13, 5, 0]
    idx, wts = synth.make_routing(w)
    for r, tr in enumerate(t_r):
        idx[r * w["T"] + tr:(r + 1) * w["T"]] = -1
    r = Run(w, "e4m3_b128", layout="packed", idx=idx, wts=wts, backward=True)
    r.check_layout()
    r.check_dispatch()
    r.check_combine()
    r.check_backward()
    out = r.b.out.view(torch.int16).cpu().numpy()
    for rr, tr in enumerate(t_r):
        assert np.all(out[rr * w["T"] + tr:(rr + 1) * w["T"]] == 0)
    tpr = r.b.tokens_per_rank.cpu().numpy()
    assert tpr[1].max() <= t_r[1] and tpr[2].sum() == 0
    assert r.b.recv_count.sum().item() == int((idx >= 0).sum())


# ---------------------------------------------------------------------------
# K = 16 (the largest top-k) and the quantised combine's fallback kernel
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("mode", ["bf16", "int8_token", "e4m3_b128", "mxfp8", "mxfp4"])
def test_k16_every_mode(mode):
    w = _edge(R=4, T=21, M=24, K=16, E=32, H=640)
    r = Run(w, mode, layout="packed", align=2, backward=True)
    r.check_layout()
    r.check_dispatch()
    r.check_combine()
    r.check_backward()
    if mode == "bf16":
        r.check_weights_grad()


@pytest.mark.parametrize("mode,flags", [("int8_token", 0), ("e4m3_b128", 0),
                                        ("e4m3_b128", ep.F_UE8M0), ("mxfp8", 0), ("mxfp4", 0)])
def test_quantized_combine_k_above_eight(mode, flags):
    """K > 8 takes the one-stage kernel (the pipelined one holds 8 rows)."""
    from harness import combine_quantized_check, special_quantized_rows
    w = _edge(R=4, T=21, M=24, K=12, E=32, H=640)
    r = Run(w, mode, layout="packed", flags=flags)
    combine_quantized_check(r, seed=21)
    combine_quantized_check(r, seed=22, rows_fn=special_quantized_rows)


@pytest.mark.parametrize("mode", ["mxfp8", "mxfp4"])
def test_quantized_combine_unaligned_scale_rows(mode):
    """H = 96 gives 3-byte MX scale rows: the one-stage kernel."""
    from harness import combine_quantized_check
    w = _edge(R=2, T=9, M=12, K=4, E=8, H=96 if mode == "mxfp8" else 224)
    r = Run(w, mode, layout="packed")
    assert r.sizes["scale_row_bytes"] % 4 != 0
    combine_quantized_check(r, seed=23)


# ---------------------------------------------------------------------------
# the experts between dispatch and combine: grouped tcgen05 GEMM
# ---------------------------------------------------------------------------
def _seeded_weights(E, n_out, H, scale, seed):
    """Synthetic expert weights, N(0, scale^2) in bf16, from a seeded generator."""
    gen = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn(E, n_out, H, device="cuda", dtype=torch.bfloat16, generator=gen).mul_(scale)


def _seeded_mx_weights(E, n_out, H, seed, lo=118, hi=134, fp4=False):
    """Synthetic MX weights from a seeded generator: e4m3 codes uniform over the
    bit patterns (the two NaN codes replaced by zero) or packed e2m1 bytes
    uniform over all 256 (fp4: [E, n_out, H/2]), e8m0 scales uniform in [lo, hi)."""
    gen = torch.Generator(device="cuda").manual_seed(seed)
    c = torch.randint(0, 256, (E, n_out, H // 2 if fp4 else H), device="cuda", dtype=torch.int16,
                      generator=gen).to(torch.uint8)
    if not fp4:
        c[(c & 0x7F) == 0x7F] = 0
    sc = torch.randint(lo, hi, (E, n_out, H // 32), device="cuda", dtype=torch.int16,
                       generator=gen).to(torch.uint8)
    return c, sc


def _e4m3_table():
    return oracle.e4m3_decode(np.arange(256, dtype=np.uint8)).astype(np.float64)


def _e2m1_values(c):
    """Values of packed e2m1 bytes (even element in the low nibble)."""
    t = oracle.e2m1_decode(np.arange(16, dtype=np.uint8)).astype(np.float64)
    v = np.empty(c.shape[:-1] + (2 * c.shape[-1],), np.float64)
    v[..., 0::2] = t[c & 0xF]
    v[..., 1::2] = t[c >> 4]
    return v


def _check_expert_gemm(r, y, n_out, W=None, wc=None, ws=None, sample_rows=None):
    """y from the GPU against the oracle's maps of the oracle's own receive rows
    (its layout and its quantisation of the seeded x), on every valid row or a
    sample; rows outside every expert untouched (0x7777).

    Bound, from the arithmetic: every product is exact in fp32 and the kernel
    chains H/16 (bf16: 16 products per tensor-core step) or H/32 (MXFP8: one
    32-element scale block per step) partial sums through one fp32
    accumulator, the sum inside a step taking at most 16 or 32 additions more;
    with at most one fp32 ulp lost per addition (truncation allowed)
    |acc - exact| <= chain * 2^-23 * sum_h |x*w|, and the final bf16 rounding
    adds at most one bf16 ulp.  Besides the bound, at least 90% of the outputs
    equal the oracle's correctly rounded ones."""
    r.check_layout()
    o = r.lay
    E, H = r.w["E"], r.w["H"]
    mx = wc is not None
    fp4 = r.mode == "mxfp4"
    eo, cnt = o["expert_offset"], o["recv_count"]
    rows = r.sizes["rows"]
    got = y.view(torch.int16).cpu().numpy().view(np.uint16)
    valid = np.zeros(rows, bool)
    for e in range(E):
        valid[eo[e]:eo[e] + cnt[e]] = True
    assert np.all(got[~valid] == 0x7777)
    ns, _, rr = r.entries()
    tok_of_row = np.full(rows, -1, np.int64)
    tok_of_row[rr] = ns
    expert_of = np.repeat(np.arange(E), np.diff(eo[:E + 1]))
    pick = np.nonzero(valid)[0]
    if sample_rows is not None and len(pick) > sample_rows:
        pick = np.sort(np.random.default_rng(0).choice(pick, sample_rows, replace=False))
    lut = _e4m3_table()

    def f(u):
        return (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)

    def mxv(c, sc):
        v = _e2m1_values(c) if fp4 else lut[c]
        return v * np.ldexp(1.0, np.repeat(sc.astype(np.int64) - 127, 32, axis=-1))
    same = 0
    for e in np.unique(expert_of[pick]):
        rs = pick[expert_of[pick] == e]
        q = [oracle.quant_row(r.omode, r.x[n], e4m3_qmax=r.qmax) for n in tok_of_row[rs]]
        one, cnt1 = np.zeros(1, np.int64), np.array([len(rs)], np.int64)
        if mx:
            xc, xs = np.stack([d for d, _ in q]), np.stack([sc for _, sc in q])
            wce, wse = wc[e].cpu().numpy(), ws[e].cpu().numpy()
            gemm = oracle.expert_gemm_mxfp4 if fp4 else oracle.expert_gemm_mx
            want = gemm(xc, xs, wce[None], wse[None], one, cnt1, n_out)
            xv, wv = mxv(xc, xs), mxv(wce, wse)
            chain = H // 32 + 32
        else:
            xb = np.stack([d.view(np.uint16) for d, _ in q])
            We = W[e].view(torch.int16).cpu().numpy().view(np.uint16)
            want = oracle.expert_gemm(xb, We[None], one, cnt1, n_out)
            xv, wv = f(xb), f(We)
            chain = H // 16 + 16
        mag = np.abs(xv).astype(np.float32) @ np.abs(wv).astype(np.float32).T
        del wv
        wf, gf = f(want), f(got[rs])
        ulp = np.ldexp(1.0, np.floor(np.log2(np.maximum(np.abs(wf), 2.0 ** -126))).astype(np.int64) - 7)
        tol = ulp + mag.astype(np.float64) * (chain * 2.0 ** -23) * (1 + 2.0 ** -10)
        assert np.all(np.abs(gf - wf) <= tol), int(e)
        same += int((got[rs] == want).sum())
    frac = same / (len(pick) * n_out)
    assert frac >= 0.9, frac
    return frac


def _sentinel_y(r, n_out):
    y = r.guards.alloc((r.sizes["rows"], n_out), torch.bfloat16, "y (expert outputs)")
    y.view(torch.int16).fill_(0x7777)
    return y


@pytest.mark.parametrize("pairs", [False, True])   # single CTAs / CTA pairs (two-CTA MMA)
@pytest.mark.parametrize("n_out", [256, 768, 1280])
def test_expert_gemm_small(n_out, pairs):
    w = synth.workload("tiny", R=4, T=40, M=48, K=4, E=8, H=640)
    idx, wts = synth.make_routing(w)
    idx[idx == 3] = 5                      # expert 3 receives nothing
    r = Run(w, "bf16", layout="packed", align=8, idx=idx, wts=wts,
            flags=ep.F_GEMM_CTA_PAIRS if pairs else 0)
    W = _seeded_weights(w["E"], n_out, w["H"], 0.05, seed=n_out)
    y = _sentinel_y(r, n_out)
    ep.ep_expert_gemm(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, W, y, r.b.dev_status)
    assert ep.ep_get_status(r.b.dev_status) == 0
    assert r.lay["recv_count"][3] == 0
    _check_expert_gemm(r, y, n_out, W=W)


@pytest.mark.parametrize("pairs", [False, True])
def test_expert_gemm_many_row_tiles(pairs):
    """Experts of several hundred rows: several row tiles, partial last tiles."""
    w = synth.workload("tiny", R=2, T=512, M=512, K=4, E=8, H=512)
    r = Run(w, "bf16", layout="packed", flags=ep.F_GEMM_CTA_PAIRS if pairs else 0)
    W = _seeded_weights(w["E"], 512, w["H"], 0.05, seed=21)
    y = _sentinel_y(r, 512)
    ep.ep_expert_gemm(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, W, y, r.b.dev_status)
    assert ep.ep_get_status(r.b.dev_status) == 0
    assert r.lay["recv_count"].max() > 256
    _check_expert_gemm(r, y, 512, W=W, sample_rows=200)


def test_expert_gemm_decode_shape_sampled():
    w = synth.workload("decode", layout="packed")
    r = Run(w, "bf16", layout="packed")
    W = _seeded_weights(w["E"], w["H"], w["H"], 0.02, seed=7)
    y = _sentinel_y(r, w["H"])
    ep.ep_expert_gemm(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, W, y, r.b.dev_status)
    assert ep.ep_get_status(r.b.dev_status) == 0
    _check_expert_gemm(r, y, w["H"], W=W, sample_rows=12)


@pytest.mark.parametrize("n_out", [448, 256, 384])   # N tiles of 224, 256 and 128 columns
def test_expert_gemm_mx_small(n_out):
    w = synth.workload("tiny", R=4, T=40, M=48, K=4, E=8, H=640)
    idx, wts = synth.make_routing(w)
    idx[idx == 3] = 5                      # expert 3 receives nothing
    r = Run(w, "mxfp8", layout="packed", align=8, idx=idx, wts=wts)
    wc, ws = _seeded_mx_weights(w["E"], n_out, w["H"], seed=n_out)
    y = _sentinel_y(r, n_out)
    ep.ep_expert_gemm_mx(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, wc, ws, y,
                         r.b.dev_status)
    assert ep.ep_get_status(r.b.dev_status) == 0
    _check_expert_gemm(r, y, n_out, wc=wc, ws=ws)


def test_expert_gemm_mx_decode_shape_sampled():
    w = synth.workload("decode", layout="packed")
    r = Run(w, "mxfp8", layout="packed")
    wc, ws = _seeded_mx_weights(w["E"], w["H"], w["H"], seed=9)
    y = _sentinel_y(r, w["H"])
    ep.ep_expert_gemm_mx(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, wc, ws, y,
                         r.b.dev_status)
    assert ep.ep_get_status(r.b.dev_status) == 0
    _check_expert_gemm(r, y, w["H"], wc=wc, ws=ws, sample_rows=12)


@pytest.mark.parametrize("n_out", [448, 256, 384])   # N tiles of 224, 256 and 128 columns
def test_expert_gemm_mxfp4_small(n_out):
    w = synth.workload("tiny", R=4, T=40, M=48, K=4, E=8, H=768)
    idx, wts = synth.make_routing(w)
    idx[idx == 3] = 5                      # expert 3 receives nothing
    r = Run(w, "mxfp4", layout="packed", align=8, idx=idx, wts=wts)
    wc, ws = _seeded_mx_weights(w["E"], n_out, w["H"], seed=n_out + 1, fp4=True)
    y = _sentinel_y(r, n_out)
    ep.ep_expert_gemm_mx(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, wc, ws, y,
                         r.b.dev_status)
    assert ep.ep_get_status(r.b.dev_status) == 0
    _check_expert_gemm(r, y, n_out, wc=wc, ws=ws)


def test_expert_gemm_mxfp4_large_shape_sampled():
    w = synth.workload("large")
    r = Run(w, "mxfp4", layout="packed")
    wc, ws = _seeded_mx_weights(w["E"], w["H"], w["H"], seed=10, fp4=True)
    y = _sentinel_y(r, w["H"])
    ep.ep_expert_gemm_mx(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, wc, ws, y,
                         r.b.dev_status)
    assert ep.ep_get_status(r.b.dev_status) == 0
    _check_expert_gemm(r, y, w["H"], wc=wc, ws=ws, sample_rows=12)


@pytest.mark.parametrize("mode,H", [("mxfp8", 1024), ("mxfp8", 640), ("mxfp4", 1024),
                                    ("mxfp4", 768)])
def test_expert_gemm_mx_tall_tiles(mode, H):
    """About 490 rows an expert on average and N tiles of 224: 256-row tiles,
    two M = 128 MMAs sharing each B tile (MXFP8 and MXFP4).  Expert sizes put
    tile ends on and around the 128-row half (129: one row in the upper half;
    556, 555: a last tile whose upper half holds nothing; 384, 640: exactly a
    half tile more), an empty expert, and H with and without whole groups of
    scale loads."""
    counts = np.array([1200, 556, 129, 0, 384, 640, 555, 440])
    w = synth.workload("tiny", R=2, T=int(counts.sum()) // 2, M=int(counts.sum()) // 2, K=1,
                       E=8, H=H)
    idx = np.repeat(np.arange(8), counts)[np.random.default_rng(5).permutation(counts.sum())]
    idx = idx.reshape(-1, 1).astype(np.int64)
    wts = np.ones_like(idx, dtype=np.float32)
    r = Run(w, mode, layout="packed", idx=idx, wts=wts)
    assert np.array_equal(r.lay["recv_count"], counts)
    wc, ws = _seeded_mx_weights(w["E"], 448, H, seed=H + len(mode), fp4=mode == "mxfp4")
    y = _sentinel_y(r, 448)
    ep.ep_expert_gemm_mx(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, wc, ws, y,
                         r.b.dev_status)
    assert ep.ep_get_status(r.b.dev_status) == 0
    _check_expert_gemm(r, y, 448, wc=wc, ws=ws, sample_rows=400)


def test_expert_gemm_empty_batch_launches_nothing():
    w = synth.workload("tiny", R=2, T=0, M=16, K=2, E=4, H=256)
    for mode in ("bf16", "mxfp8"):
        r = Run(w, mode, layout="packed")
        y = _sentinel_y(r, 256)
        n0 = ep.ep_kernel_launches()
        if mode == "bf16":
            W = _seeded_weights(w["E"], 256, w["H"], 0.05, seed=1)
            ep.ep_expert_gemm(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, W, y,
                              r.b.dev_status)
        else:
            wc, ws = _seeded_mx_weights(w["E"], 256, w["H"], seed=1)
            ep.ep_expert_gemm_mx(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, wc, ws,
                                 y, r.b.dev_status)
        assert ep.ep_kernel_launches() == n0
        assert torch.all(y.view(torch.int16) == 0x7777)


@pytest.mark.parametrize("mode", ["bf16", "mxfp8", "mxfp4"])
def test_expert_gemm_one_expert_takes_every_token(mode):
    """Every token to expert 2: one expert with many row tiles (a partial last
    one), every other expert empty."""
    w = synth.workload("tiny", R=2, T=300, M=300, K=1, E=8, H=512)
    idx = np.full((w["R"] * w["T"], 1), 2, np.int64)
    wts = np.ones((w["R"] * w["T"], 1), np.float32)
    r = Run(w, mode, layout="packed", idx=idx, wts=wts)
    y = _sentinel_y(r, 256)
    if mode == "bf16":
        W = _seeded_weights(w["E"], 256, w["H"], 0.05, seed=3)
        ep.ep_expert_gemm(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, W, y,
                          r.b.dev_status)
        kw = dict(W=W)
    else:
        wc, ws = _seeded_mx_weights(w["E"], 256, w["H"], seed=3, fp4=mode == "mxfp4")
        ep.ep_expert_gemm_mx(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, wc, ws, y,
                             r.b.dev_status)
        kw = dict(wc=wc, ws=ws)
    assert ep.ep_get_status(r.b.dev_status) == 0
    assert r.lay["recv_count"][2] == 600
    _check_expert_gemm(r, y, 256, sample_rows=160, **kw)


def test_expert_gemm_most_experts():
    """E = 1024 (the limit): the per-expert tile prefix over 32 experts a lane."""
    w = synth.workload("tiny", R=4, T=64, M=64, K=4, E=1024, H=256)
    r = Run(w, "bf16", layout="packed")
    W = _seeded_weights(w["E"], 256, w["H"], 0.05, seed=4)
    y = _sentinel_y(r, 256)
    ep.ep_expert_gemm(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, W, y, r.b.dev_status)
    assert ep.ep_get_status(r.b.dev_status) == 0
    _check_expert_gemm(r, y, 256, W=W, sample_rows=200)


def test_expert_gemm_mx_rejects_other_formats():
    w = synth.workload("tiny", R=2, T=16, M=16, K=2, E=4, H=256)
    r = Run(w, "bf16", layout="packed")
    # codes shaped as the binding expects for this format, so that the library rejects it
    wc = torch.zeros((w["E"], 256, 2 * w["H"]), dtype=torch.uint8, device="cuda")
    _, ws = _seeded_mx_weights(w["E"], 256, w["H"], seed=1)
    y = _sentinel_y(r, 256)
    with pytest.raises(ep.EpError):
        ep.ep_expert_gemm_mx(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, wc, ws, y,
                             r.b.dev_status)
    wc2, ws2 = _seeded_mx_weights(w["E"], 96, w["H"], seed=1)    # no N tile divides 96
    r2 = Run(w, "mxfp8", layout="packed")
    with pytest.raises(ep.EpError):
        ep.ep_expert_gemm_mx(r2.cfg, r2.b.recv_buf, r2.b.expert_offset, r2.b.recv_count, wc2, ws2,
                             _sentinel_y(r2, 96), r2.b.dev_status)
    assert torch.all(y.view(torch.int16) == 0x7777)


def _bf16_ulp(bits):
    v = np.abs((bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    return np.ldexp(1.0, np.floor(np.log2(np.maximum(v, 2.0 ** -126))).astype(np.int64) - 7)


def _chain_check(got, want, yw, mag, chain, idx, wts, rows_of):
    """The GPU's chain against the oracle's, element by element, within a bound
    derived from the arithmetic: each expert output the GPU combines may differ
    from the oracle's by its own allowance (one bf16 ulp plus
    chain * 2^-23 * sum_h |x*w|, the GEMM bound), which the combine scales by
    |w_k|; the combine's own rounding adds up to two bf16 ulps of the result
    (its fp32 sum of perturbed terms, then bf16)."""
    N, K = idx.shape
    bound = 2.0 * _bf16_ulp(want)
    for n in range(N):
        for k in range(K):
            row = rows_of.get((n, k))
            if row is None:
                continue
            allow = _bf16_ulp(yw[row]) + mag[row] * (chain * 2.0 ** -23)
            bound[n] += abs(float(wts[n, k])) * allow
    gf = (got.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    wf = (want.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.all(np.abs(gf - wf) <= bound)


def _pipeline_check(r, maps_fn, n_out, chain):
    """The GPU's combine of its expert outputs against the oracle's combine of
    the oracle's expert outputs (oracle layout and quantisation of the seeded x),
    within _chain_check's bound.  maps_fn(e, rows) -> (bf16 outputs, sum_h |x*w|)."""
    w = r.w
    o = r.lay
    E, H = w["E"], w["H"]
    eo, cnt = o["expert_offset"], o["recv_count"]
    rows = r.sizes["rows"]
    ns, ks, rr = r.entries()
    tok = {int(a): int(b) for a, b in zip(rr, ns)}
    yw = np.zeros((rows, n_out), np.uint16)
    mag = np.zeros((rows, n_out), np.float64)
    for e in range(E):
        rs = np.sort(rr[(rr >= eo[e]) & (rr < eo[e] + cnt[e])])
        if len(rs) == 0:
            continue
        q = [oracle.quant_row(r.omode, r.x[tok[int(x)]], e4m3_qmax=r.qmax) for x in rs]
        yw[rs], mag[rs] = maps_fn(e, q)
    want, st = oracle.combine(w["R"], w["T"], w["K"], E, w["M"], H, yw, r.idx, r.wts,
                              o["token_slot"], o["expert_offset"], layout="packed")
    assert st == 0
    _chain_check(to_np_u16(r.b.out), want, yw, mag, chain, r.idx, r.wts,
                 {(int(n), int(k)): int(x) for n, k, x in zip(ns, ks, rr)})


def test_dispatch_experts_combine_pipeline():
    """dispatch -> the experts' linear maps -> combine on the GPU, against the
    oracle's chain (one bf16 ulp for the experts' rounding, one for the
    combine's)."""
    w = synth.workload("tiny", R=2, T=32, M=32, K=4, E=8, H=256)
    r = Run(w, "bf16", layout="packed")
    n_out = w["H"]
    W = _seeded_weights(w["E"], n_out, w["H"], 0.06, seed=11)
    ep.ep_expert_gemm(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, W, r.b.y,
                      r.b.dev_status)
    ep.ep_combine(r.cfg, r.b.y, r.idx_d, r.wts_d, r.b.token_slot, r.b.out, r.b.dev_status,
                  expert_offset=r.b.expert_offset)
    assert ep.ep_get_status(r.b.dev_status) == 0
    Wh = W.view(torch.int16).cpu().numpy().view(np.uint16)

    def maps(e, q):
        xb = np.stack([d.view(np.uint16) for d, _ in q])
        y = oracle.expert_gemm(xb, Wh[e][None], np.zeros(1, np.int64),
                               np.array([len(q)], np.int64), n_out)
        f = lambda u: (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        return y, np.abs(f(xb)) @ np.abs(f(Wh[e])).T
    _pipeline_check(r, maps, n_out, w["H"] // 16 + 16)


def test_dispatch_mxfp4_experts_combine_pipeline():
    """MXFP4 dispatch -> the experts' block-scaled maps -> combine on the GPU,
    against the oracle's chain."""
    w = synth.workload("tiny", R=2, T=32, M=32, K=4, E=8, H=512)
    r = Run(w, "mxfp4", layout="packed")
    n_out = w["H"]
    wc, ws = _seeded_mx_weights(w["E"], n_out, w["H"], seed=13, lo=112, hi=124, fp4=True)
    ep.ep_expert_gemm_mx(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, wc, ws, r.b.y,
                         r.b.dev_status)
    ep.ep_combine(r.cfg, r.b.y, r.idx_d, r.wts_d, r.b.token_slot, r.b.out, r.b.dev_status,
                  expert_offset=r.b.expert_offset)
    assert ep.ep_get_status(r.b.dev_status) == 0
    wch, wsh = wc.cpu().numpy(), ws.cpu().numpy()

    def maps(e, q):
        xc, xs = np.stack([d for d, _ in q]), np.stack([sc for _, sc in q])
        y = oracle.expert_gemm_mxfp4(xc, xs, wch[e][None], wsh[e][None], np.zeros(1, np.int64),
                                     np.array([len(q)], np.int64), n_out)
        sv = lambda c, sc: _e2m1_values(c) * np.ldexp(1.0, np.repeat(sc.astype(np.int64) - 127, 32, axis=-1))
        return y, np.abs(sv(xc, xs)) @ np.abs(sv(wch[e], wsh[e])).T
    _pipeline_check(r, maps, n_out, w["H"] // 32 + 32)


def test_dispatch_mx_experts_combine_pipeline():
    """MXFP8 dispatch -> the experts' block-scaled maps -> combine on the GPU,
    against the oracle's chain."""
    w = synth.workload("tiny", R=2, T=32, M=32, K=4, E=8, H=256)
    r = Run(w, "mxfp8", layout="packed")
    n_out = w["H"]
    wc, ws = _seeded_mx_weights(w["E"], n_out, w["H"], seed=12, lo=112, hi=124)
    ep.ep_expert_gemm_mx(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, wc, ws, r.b.y,
                         r.b.dev_status)
    ep.ep_combine(r.cfg, r.b.y, r.idx_d, r.wts_d, r.b.token_slot, r.b.out, r.b.dev_status,
                  expert_offset=r.b.expert_offset)
    assert ep.ep_get_status(r.b.dev_status) == 0
    wch, wsh = wc.cpu().numpy(), ws.cpu().numpy()

    def maps(e, q):
        xc, xs = np.stack([d for d, _ in q]), np.stack([sc for _, sc in q])
        y = oracle.expert_gemm_mx(xc, xs, wch[e][None], wsh[e][None], np.zeros(1, np.int64),
                                  np.array([len(q)], np.int64), n_out)
        lut = _e4m3_table()
        sv = lambda c, sc: lut[c] * np.ldexp(1.0, np.repeat(sc.astype(np.int64) - 127, 32, axis=-1))
        return y, np.abs(sv(xc, xs)) @ np.abs(sv(wch[e], wsh[e])).T
    _pipeline_check(r, maps, n_out, w["H"] // 32 + 32)


# ---------------------------------------------------------------------------
# the whole forward path in one call
# ---------------------------------------------------------------------------
def _moe_case(mode, seed):
    w = synth.workload("tiny", R=2, T=48, M=48, K=4, E=8, H=512)
    idx, wts = synth.make_routing(w)
    x = synth.make_x(w)
    cfg = ep.make_config(w["R"], w["T"], w["M"], w["K"], w["E"], w["H"], mode, "packed")
    if mode == "bf16":
        wc, ws = _seeded_weights(w["E"], w["H"], w["H"], 0.05, seed), None
    else:
        wc, ws = _seeded_mx_weights(w["E"], w["H"], w["H"], seed, lo=112, hi=124,
                                    fp4=mode == "mxfp4")
    return w, cfg, bf16_dev(x), torch.from_numpy(idx).cuda(), torch.from_numpy(wts).cuda(), wc, ws, idx, wts, x


@pytest.mark.parametrize("mode", ["bf16", "mxfp8", "mxfp4"])
def test_moe_forward_equals_the_calls_one_by_one(mode):
    w, cfg, x_d, idx_d, wts_d, wc, ws, idx, wts, x = _moe_case(mode, 31)
    H = w["H"]
    outs = []
    for one_call in (True, False):
        guards = Guards()
        b = guards.wrap(ep.Buffers(cfg))
        b.recv_buf.fill_(0xAB)
        y = guards.alloc((b.sizes["rows"], H), torch.bfloat16, "y")
        out = guards.alloc((w["N"], H), torch.bfloat16, "out")
        out.fill_(7.0)
        if one_call:
            n0 = ep.ep_kernel_launches()
            ep.ep_moe_forward(cfg, x_d, idx_d, wts_d, wc, ws, b.token_slot, b.recv_count,
                              b.expert_offset, b.workspace, b.recv_buf, b.src_info, y, out,
                              b.dev_status)
            assert ep.ep_kernel_launches() - n0 == 4   # layout, dispatch, experts, combine
        else:
            ep.ep_dispatch_layout(cfg, idx_d, b.token_slot, b.recv_count, b.workspace,
                                  b.dev_status, expert_offset=b.expert_offset)
            ep.ep_dispatch(cfg, x_d, idx_d, b.token_slot, b.recv_buf, b.src_info, b.dev_status,
                           expert_offset=b.expert_offset)
            if mode == "bf16":
                ep.ep_expert_gemm(cfg, b.recv_buf, b.expert_offset, b.recv_count, wc, y,
                                  b.dev_status)
            else:
                ep.ep_expert_gemm_mx(cfg, b.recv_buf, b.expert_offset, b.recv_count, wc, ws, y,
                                     b.dev_status)
            ep.ep_combine(cfg, y, idx_d, wts_d, b.token_slot, b.out, b.dev_status,
                          expert_offset=b.expert_offset)
            out = b.out
        assert ep.ep_get_status(b.dev_status) == 0
        guards.check()
        outs.append(to_np_u16(out))
    assert np.array_equal(outs[0], outs[1])


def test_moe_forward_against_the_oracle_chain():
    """bf16: the one call against the oracle's layout, dispatch, maps and combine."""
    w, cfg, x_d, idx_d, wts_d, W, _, idx, wts, x = _moe_case("bf16", 32)
    H, E = w["H"], w["E"]
    b = ep.Buffers(cfg)
    y = torch.empty((b.sizes["rows"], H), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((w["N"], H), dtype=torch.bfloat16, device="cuda")
    ep.ep_moe_forward(cfg, x_d, idx_d, wts_d, W, None, b.token_slot, b.recv_count, b.expert_offset,
                      b.workspace, b.recv_buf, b.src_info, y, out, b.dev_status)
    assert ep.ep_get_status(b.dev_status) == 0
    lay = oracle.layout(w["R"], w["T"], w["K"], E, w["M"], idx, layout="packed")
    eo, cnt = lay["expert_offset"], lay["recv_count"]
    rows = b.sizes["rows"]
    xr = np.zeros((rows, H), np.uint16)
    for n in range(w["N"]):
        for k in range(w["K"]):
            e = idx[n, k]
            if 0 <= e < E:
                xr[eo[e] + lay["token_slot"][n, k]] = x[n]       # bf16 dispatch is a scatter
    Wh = W.view(torch.int16).cpu().numpy().view(np.uint16)
    yw = oracle.expert_gemm(xr, Wh, eo[:E], cnt, H)
    want, st = oracle.combine(w["R"], w["T"], w["K"], E, w["M"], H, yw, idx, wts,
                              lay["token_slot"], eo, layout="packed")
    assert st == 0
    f = lambda u: (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    mag = np.zeros((rows, H))
    rows_of = {}
    for e in range(E):
        rs = np.arange(eo[e], eo[e] + cnt[e])
        if len(rs):
            mag[rs] = np.abs(f(xr[rs])) @ np.abs(f(Wh[e])).T
    for n in range(w["N"]):
        for k in range(w["K"]):
            if 0 <= idx[n, k] < E:
                rows_of[(n, k)] = int(eo[idx[n, k]] + lay["token_slot"][n, k])
    _chain_check(to_np_u16(out), want, yw, mag, H // 16 + 16, idx, wts, rows_of)


def test_moe_forward_checks_before_launching():
    w, cfg, x_d, idx_d, wts_d, wc, ws, *_ = _moe_case("bf16", 33)
    b = ep.Buffers(cfg)
    y = torch.empty((b.sizes["rows"], w["H"]), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((w["N"], w["H"]), dtype=torch.bfloat16, device="cuda")
    bad = ep.make_config(w["R"], w["T"], w["M"], w["K"], w["E"], w["H"], "bf16", "packed",
                         flags=ep.F_COMBINE_QUANTIZED)
    n0 = ep.ep_kernel_launches()
    with pytest.raises(ep.EpError):
        ep.ep_moe_forward(bad, x_d, idx_d, wts_d, wc, None, b.token_slot, b.recv_count,
                          b.expert_offset, b.workspace, b.recv_buf, b.src_info, y, out, b.dev_status)
    assert ep.ep_kernel_launches() == n0


# ---------------------------------------------------------------------------
# the bounded waits of the tensor-core kernels
# ---------------------------------------------------------------------------
def test_bounded_wait_gives_up_reports_and_leaves_the_context_usable():
    """A wait on a barrier that nothing completes (the GEMMs' own wait helper)
    gives up after about 2 s and sets DEV_TIMEOUT; the kernel returns and the
    next calls run normally."""
    import time
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.monotonic()
    ep.ep_wait_probe(st)
    flags = ep.ep_get_status(st)
    dt = time.monotonic() - t0
    assert flags == ep.DEV_TIMEOUT
    assert 1.5 < dt < 60, dt
    assert ep.ep_get_status(st) == 0                   # read and cleared
    r = Run(synth.workload("tiny"), "bf16")             # the context is still usable
    r.check_layout()
    r.check_dispatch()
    r.check_combine()
