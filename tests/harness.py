"""Shared helpers for the GPU parity tests: run the path on cuda:0 through the
C ABI, and compare it with the oracle on the same seeded inputs.

The oracle never sees a value produced on the device: its inputs are the host
arrays the seeded recipes build, and expert outputs are rebuilt on the host
from the same pool windows the device gathered."""
import numpy as np
import torch

import combine_ep_dispatch_04_b200 as ep
import oracle
import synth


def bf16_dev(a_u16):
    return torch.from_numpy(np.ascontiguousarray(a_u16).view(np.int16)).cuda().view(torch.bfloat16)


def to_np_u16(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


GUARD_BYTES = 4096
GUARD_FILL = 0x5C
BUFFER_FIELDS = ("tokens_per_rank", "tokens_per_expert", "is_token_in_rank", "token_slot",
                 "recv_count", "expert_offset", "workspace", "recv_buf", "src_info",
                 "recv_weights", "y", "out", "grad_buf", "dev_status")


class Guards:
    """Guard bands around the device buffers a test hands to the library (the
    stand-in for a memory checker): each buffer is carved out of a larger
    allocation with GUARD_BYTES of a fill pattern on both sides (plus the
    rounding up to 16 bytes after it); check() asserts that no kernel wrote
    into a band.  The byte count each buffer reports is its own, so the
    library's size checks see the exact size."""

    def __init__(self):
        self.items = []

    def alloc(self, shape, dtype, name):
        nbytes = int(np.prod(shape, dtype=np.int64)) * torch.empty((), dtype=dtype).element_size()
        span = (nbytes + 15) // 16 * 16
        base = torch.full((2 * GUARD_BYTES + span,), GUARD_FILL, dtype=torch.uint8,
                          device="cuda")
        self.items.append((name, base, nbytes))
        return base[GUARD_BYTES:GUARD_BYTES + nbytes].view(dtype).view(shape)

    def like(self, t, name):
        g = self.alloc(tuple(t.shape), t.dtype, name)
        g.copy_(t)
        return g

    def wrap(self, buffers):
        """Replace every buffer of an ep.Buffers with a guarded copy."""
        for f in BUFFER_FIELDS:
            t = getattr(buffers, f, None)
            if isinstance(t, torch.Tensor):
                setattr(buffers, f, self.like(t, f))
        torch.cuda.empty_cache()
        return buffers

    def check(self):
        torch.cuda.synchronize()
        for name, base, nbytes in self.items:
            lo = base[:GUARD_BYTES]
            hi = base[GUARD_BYTES + nbytes:]
            assert bool((lo == GUARD_FILL).all()), f"write below {name}"
            assert bool((hi == GUARD_FILL).all()), f"write past the end of {name}"


def oracle_mode(mode, flags):
    """The oracle's name for a quantisation mode with its scale flags."""
    if mode == "e4m3_b128" and flags & ep.F_UE8M0:
        return "e4m3_b128_ue8m0"
    if mode == "e4m3_b128" and flags & ep.F_ROUND_SCALE:
        return "e4m3_b128_p2"
    return mode


class Run:
    """One pass of layout -> dispatch -> combine (-> combine backward) on the GPU."""

    def __init__(self, w, mode, layout="padded", align=1, qmax=0.0, flags=0, idx=None, wts=None,
                 x=None, with_weights=True, backward=False, bwd_unweighted=False, stats=False,
                 replica=0, fill=0xAB):
        self.w, self.mode, self.layout, self.align, self.qmax = w, mode, layout, align, qmax
        R, T, M, K, E, H = w["R"], w["T"], w["M"], w["K"], w["E"], w["H"]
        if idx is None or wts is None:
            i2, w2 = synth.make_routing(w, replica)
            idx = i2 if idx is None else idx
            wts = w2 if wts is None else wts
        self.idx = np.ascontiguousarray(idx, np.int64)
        if flags & ep.F_IDX_I32:  # the values the device sees
            self.idx = self.idx.astype(np.int32).astype(np.int64)
        self.wts = np.ascontiguousarray(wts, np.float32)
        self.x = synth.make_x(w, replica) if x is None else np.ascontiguousarray(x, np.uint16)
        self.cfg = ep.make_config(R, T, M, K, E, H, mode, layout, align, qmax,
                                  flags | (ep.F_BWD_UNWEIGHTED if bwd_unweighted else 0))
        self.bwd_unweighted = bwd_unweighted
        self.omode = oracle_mode(mode, flags)
        self.guards = Guards()
        b = self.guards.wrap(ep.Buffers(self.cfg, recv_weights=with_weights, grad=backward))
        self.b = b
        b.recv_buf.fill_(fill)
        if b.recv_weights is not None:
            b.recv_weights.fill_(float("nan"))
        b.src_info.fill_(-7)
        self.sizes = b.sizes
        N = R * T
        self.idx_d = torch.from_numpy(self.idx).cuda().to(ep.idx_dtype(self.cfg))
        self.wts_d = torch.from_numpy(self.wts).cuda()
        self.x_d = bf16_dev(self.x)
        self.stats_d = torch.zeros(E, dtype=torch.int64, device="cuda") if stats else None
        ep.ep_dispatch_layout(self.cfg, self.idx_d, b.token_slot, b.recv_count, b.workspace,
                              b.dev_status, b.tokens_per_rank, b.tokens_per_expert,
                              b.is_token_in_rank, b.expert_offset, self.stats_d)
        ep.ep_dispatch(self.cfg, self.x_d, self.idx_d, b.token_slot, b.recv_buf, b.src_info,
                       b.dev_status, topk_weights=self.wts_d if with_weights else None,
                       expert_offset=b.expert_offset, recv_weights=b.recv_weights)
        # expert outputs: pool windows for every buffer row
        rows = self.sizes["rows"]
        self.y_pool, self.y_off = synth.y_source(w, rows, replica)
        pool_d = torch.from_numpy(self.y_pool.view(np.int16)).cuda()
        off_d = torch.from_numpy(self.y_off).cuda()
        torch.index_select(pool_d.as_strided((synth.POOL, H), (1, 1)), 0, off_d,
                           out=b.y.view(torch.int16))
        del pool_d, off_d
        b.out.fill_(1.0)
        ep.ep_combine(self.cfg, b.y, self.idx_d, self.wts_d, b.token_slot, b.out, b.dev_status,
                      expert_offset=b.expert_offset)
        self.g = None
        if backward:
            gp, go = synth.g_source(w, replica)
            self.g = synth.windows(gp, go, H)
            self.g_d = bf16_dev(self.g)
            b.grad_buf.fill_(fill)
            ep.ep_combine_backward(self.cfg, self.g_d, self.idx_d, self.wts_d, b.token_slot,
                                   b.grad_buf, b.dev_status, expert_offset=b.expert_offset)
        self.status = ep.ep_get_status(b.dev_status)
        self.lay = oracle.layout(R, T, K, E, M, self.idx, layout=layout, align=align)

    # ---- comparisons ----------------------------------------------------------
    def check_layout(self):
        self.guards.check()
        b, o = self.b, self.lay
        assert np.array_equal(b.token_slot.cpu().numpy(), o["token_slot"])
        assert np.array_equal(b.recv_count.cpu().numpy(), o["recv_count"])
        assert np.array_equal(b.tokens_per_expert.cpu().numpy(), o["tokens_per_expert"])
        assert np.array_equal(b.tokens_per_rank.cpu().numpy(), o["tokens_per_rank"])
        assert np.array_equal(b.is_token_in_rank.cpu().numpy(), o["is_token_in_rank"])
        if self.layout == "packed":
            assert np.array_equal(b.expert_offset.cpu().numpy(), o["expert_offset"])
        assert self.status == o["status"], (self.status, o["status"])
        if self.stats_d is not None:
            assert np.array_equal(self.stats_d.cpu().numpy(), o["recv_count"])

    def entries(self, tokens=None):
        """(n, k, row) of every valid entry of the given tokens, from the oracle layout."""
        w, o = self.w, self.lay
        idx = self.idx
        n_all = np.arange(idx.shape[0]) if tokens is None else np.asarray(tokens)
        ns, ks = np.nonzero((idx[n_all] >= 0) & (idx[n_all] < w["E"]))
        ns = n_all[ns]
        slots = o["token_slot"][ns, ks]
        rows = oracle.row_index(self.layout, w["R"], w["M"], idx[ns, ks], slots, o["expert_offset"])
        if self.layout == "padded":
            ok = slots < w["R"] * w["M"]
            ns, ks, rows = ns[ok], ks[ok], rows[ok]
        return ns, ks, rows

    def check_dispatch(self, tokens=None, check_unwritten=True):
        self.guards.check()
        w, b = self.w, self.b
        ns, ks, rows = self.entries(tokens)
        rows_d = torch.from_numpy(rows).cuda()
        data = b.recv_data().index_select(0, rows_d).cpu().numpy()
        S = self.sizes["scale_row_bytes"]
        scale = b.recv_scale().index_select(0, rows_d).cpu().numpy() if S else None
        src = b.src_info.index_select(0, rows_d).cpu().numpy()
        expect_cache = {}
        for i, (n, k, row) in enumerate(zip(ns, ks, rows)):
            if n not in expect_cache:
                d, s = oracle.quant_row(self.omode, self.x[n], e4m3_qmax=self.qmax)
                if self.mode == "mxfp4":  # a NaN element's nibble is unspecified
                    keep = mxfp4_defined_nibbles(self.x[n])
                    d = d & keep
                else:
                    keep = None
                expect_cache[n] = (d, s, keep)
            d, s, keep = expect_cache[n]
            got_d = data[i] if keep is None else data[i] & keep
            assert np.array_equal(got_d, d), f"data row {row} (token {n}, k {k})"
            if S:
                assert np.array_equal(scale[i], s), f"scale row {row} (token {n}, k {k})"
            assert src[i] == (n // w["T"]) * w["M"] + n % w["T"]
        if b.recv_weights is not None:
            rw = b.recv_weights.index_select(0, rows_d).cpu().numpy()
            assert np.array_equal(rw, self.wts[ns, ks])
        if check_unwritten and tokens is None:
            written = (b.recv_data() != 0xAB).any(dim=1).cpu().numpy()
            want = np.zeros(self.sizes["rows"], bool)
            want[rows] = True
            assert np.array_equal(written, want)
        return len(rows)

    def y_rows_host(self, rows):
        return synth.windows(self.y_pool, self.y_off[np.asarray(rows, np.int64)], self.w["H"])

    def check_combine(self, tokens=None, max_ulp=1):
        self.guards.check()
        w, b = self.w, self.b
        K, H = w["K"], w["H"]
        tokens = np.arange(self.idx.shape[0]) if tokens is None else np.asarray(tokens)
        got = to_np_u16(b.out.index_select(0, torch.from_numpy(tokens).cuda()))
        worst = 0
        for a in range(0, len(tokens), 512):
            tk = tokens[a:a + 512]
            yr = np.zeros((len(tk), K, H), np.uint16)
            valid = np.zeros((len(tk), K), np.uint8)
            ns, ks, rows = self.entries(tk)
            pos = {n: i for i, n in enumerate(tk)}
            if len(rows):
                ys = self.y_rows_host(rows)
                for j, (n, k) in enumerate(zip(ns, ks)):
                    yr[pos[n], k] = ys[j]
                    valid[pos[n], k] = 1
            want = oracle.combine_gathered(yr, self.wts[tk], valid)
            d = ulp_distance(got[a:a + 512], want)
            worst = max(worst, int(d.max()) if d.size else 0)
        assert worst <= max_ulp, worst
        return worst

    def check_weights_grad(self, tokens=None, g=None):
        """Weight gradient on the GPU against the oracle: within 128 * 2^-24 *
        sum_h |g*y| of the exact dot product (any fp32 summation order of at
        most ~80 additions per term stays inside it), masked entries 0."""
        w, b = self.w, self.b
        K, H = w["K"], w["H"]
        if g is None:
            gp, go = synth.g_source(w)
            g = synth.windows(gp, go, H)
        g_d = bf16_dev(g)
        dw = self.guards.alloc((w["N"], K), torch.float32, "topk_weights_grad")
        dw.fill_(float("nan"))
        ep.ep_combine_backward_weights(self.cfg, g_d, b.y, self.idx_d, b.token_slot, dw,
                                       b.dev_status, expert_offset=b.expert_offset)
        assert ep.ep_get_status(b.dev_status) == self.status
        self.guards.check()
        tokens = np.arange(w["N"]) if tokens is None else np.asarray(tokens)
        got = dw.cpu().numpy()[tokens]
        worst = 0.0
        for a in range(0, len(tokens), 256):
            tk = tokens[a:a + 256]
            yr = np.zeros((len(tk), K, H), np.uint16)
            valid = np.zeros((len(tk), K), np.uint8)
            ns, ks, rows = self.entries(tk)
            pos = {n: i for i, n in enumerate(tk)}
            if len(rows):
                ys = self.y_rows_host(rows)
                for j, (n, k) in enumerate(zip(ns, ks)):
                    yr[pos[n], k] = ys[j]
                    valid[pos[n], k] = 1
            want, mag = oracle.combine_wgrad_gathered(g[tk], yr, valid)
            err = np.abs(got[a:a + 256].astype(np.float64) - want.astype(np.float64))
            bound = 128 * 2.0 ** -24 * mag + np.abs(want.astype(np.float64)) * 2.0 ** -24
            assert np.all(err <= bound), float((err - bound).max())
            assert np.all(got[a:a + 256][valid == 0] == 0.0)
            worst = max(worst, float((err / np.maximum(mag, 1e-300)).max()) if err.size else 0.0)
        return worst

    def check_backward(self, tokens=None):
        self.guards.check()
        w, b = self.w, self.b
        H = w["H"]
        ns, ks, rows = self.entries(tokens)
        rows_d = torch.from_numpy(rows).cuda()
        gd = b.grad_data(H).index_select(0, rows_d).cpu().numpy()
        gs = b.grad_scale(H).index_select(0, rows_d).cpu().numpy()
        for i, (n, k) in enumerate(zip(ns, ks)):
            d, s = oracle.bwd_row(self.g[n], self.wts[n, k], self.bwd_unweighted)
            assert np.array_equal(gd[i], d), f"grad row {rows[i]} (token {n}, k {k})"
            assert np.array_equal(gs[i], s), f"grad scale row {rows[i]}"
        return len(rows)


def mxfp4_defined_nibbles(x_row_u16):
    """Byte mask over a packed MXFP4 row: 0xF for each nibble whose element is
    not NaN, 0 for a NaN element (e2m1 has no NaN; its code is unspecified)."""
    nan = ((x_row_u16 & 0x7F80) == 0x7F80) & ((x_row_u16 & 0x007F) != 0)
    m = np.where(nan, 0, 0xF).astype(np.uint8)
    return (m[0::2] | (m[1::2] << 4)).astype(np.uint8)


def ulp_distance(a, b):
    """Distance in bf16 ulps between arrays of bf16 bit patterns."""
    def key(u):
        u = u.astype(np.int64)
        return np.where(u & 0x8000, -(u & 0x7FFF), u)
    return np.abs(key(a) - key(b))


def quantized_rows(mode, H, nrows, seed):
    """Random expert outputs stored in a quantised format: (data [n, D], scale [n, S])
    bytes.  Every code value occurs; NaN codes and NaN scales do not."""
    r = np.random.default_rng(seed)
    D, S = oracle.row_bytes(mode, H)
    data = r.integers(0, 256, (nrows, D), dtype=np.uint8)
    if mode.startswith("e4m3") or mode == "mxfp8":
        data[(data & 0x7F) == 0x7F] ^= 0x01          # 0x7F / 0xFF are NaN in e4m3
    if mode == "int8_token":
        scale = (r.random((nrows, 1)) * 0.05 + 1e-3).astype(np.float32).view(np.uint8)
    elif mode == "e4m3_b128":
        scale = (r.random((nrows, S // 4)) * 0.02 + 1e-4).astype(np.float32).view(np.uint8)
    elif mode == "e4m3_b128_p2":
        scale = np.ldexp(1.0, r.integers(-20, 5, (nrows, S // 4))).astype(np.float32).view(np.uint8)
    else:
        scale = r.integers(112, 140, (nrows, S), dtype=np.uint8)
    return data, scale.reshape(nrows, S)


def special_quantized_rows(mode, H, nrows, seed):
    """Quantised rows with the values a decoder can get wrong: every code
    (NaN codes included), and scales that are zero, subnormal, huge, infinite,
    NaN or negative (fp32 scales), or every e8m0 byte from 0 to 255."""
    r = np.random.default_rng(seed)
    D, S = oracle.row_bytes(mode, H)
    data = r.integers(0, 256, (nrows, D), dtype=np.uint8)
    if mode in ("int8_token", "e4m3_b128", "e4m3_b128_p2"):
        pick = np.array([0.0, 1e-45, 1e-40, 3e-39, 1e-3, 0.5, 1.0, 200.0, 255.9, 256.0, 1e30,
                         3e38, np.inf, np.nan, -0.75, -np.inf], np.float32)
        scale = pick[r.integers(0, len(pick), (nrows, S // 4))].view(np.uint8)
    else:
        scale = r.integers(0, 256, (nrows, S), dtype=np.uint8)
        scale[:, 0] = np.arange(nrows) % 256
    return data, scale.reshape(nrows, S)


def _quantized_combine_matches(run, out, tokens, ns, ks, data, scale):
    """The GPU combine `out` of quantised rows (data / scale of entry i = (ns[i],
    ks[i])) against the oracle on `tokens`: within 1 bf16 ulp, NaN exactly where
    the oracle gives NaN.  Returns the largest distance."""
    K, H = run.w["K"], run.w["H"]
    D, S = data.shape[1], scale.shape[1]
    where = {(int(n), int(k)): i for i, (n, k) in enumerate(zip(ns, ks))}
    qd = np.zeros((len(tokens), K, D), np.uint8)
    qs = np.zeros((len(tokens), K, S), np.uint8)
    valid = np.zeros((len(tokens), K), np.uint8)
    for j, n in enumerate(tokens):
        for k in range(K):
            i = where.get((int(n), k))
            if i is not None:
                qd[j, k], qs[j, k], valid[j, k] = data[i], scale[i], 1
    want = oracle.combine_gathered_q(run.omode, qd, qs, run.wts[tokens], valid, H)
    got = to_np_u16(out)[tokens]
    nan_g = (got & 0x7FFF) > 0x7F80
    nan_w = (want & 0x7FFF) > 0x7F80
    assert np.array_equal(nan_g, nan_w), int((nan_g != nan_w).sum())
    d = np.where(nan_w, 0, ulp_distance(got, want))
    assert d.max() <= 1, int(d.max())
    return int(d.max())


def combine_dispatched_check(run, tokens):
    """The combine of the dispatched rows themselves read as quantised expert
    outputs (the benchmark's quantised-combine launch), on the given tokens:
    within 1 bf16 ulp of the oracle, NaN exactly where the oracle gives NaN."""
    w, b = run.w, run.b
    K, H = w["K"], w["H"]
    cfg = ep.make_config(w["R"], w["T"], w["M"], K, w["E"], H, run.mode, run.layout, run.align,
                         run.qmax, run.cfg.flags | ep.F_COMBINE_QUANTIZED)
    out = run.guards.alloc((w["N"], H), torch.bfloat16, "out (combine of dispatched rows)")
    out.fill_(1.0)
    ep.ep_combine(cfg, b.recv_buf, run.idx_d, run.wts_d, b.token_slot, out, b.dev_status,
                  expert_offset=b.expert_offset)
    assert ep.ep_get_status(b.dev_status) == run.status
    run.guards.check()
    tokens = np.asarray(tokens)
    ns, ks, rows = run.entries(tokens)
    sz = run.sizes
    D, S = sz["data_row_bytes"], sz["scale_row_bytes"]
    rows_d = torch.from_numpy(np.ascontiguousarray(rows, np.int64)).cuda()
    data = b.recv_buf[: sz["rows"] * D].view(sz["rows"], D).index_select(0, rows_d).cpu().numpy()
    a = sz["recv_scale_offset"]
    scale = b.recv_buf[a: a + sz["rows"] * S].view(sz["rows"], S).index_select(0, rows_d) \
        .cpu().numpy() if S else np.zeros((len(rows), 0), np.uint8)
    return _quantized_combine_matches(run, out, tokens, ns, ks, data, scale)


def combine_quantized_check(run, tokens=None, seed=0, rows_fn=None):
    """Combine of quantised expert outputs on the GPU against the oracle:
    within 1 bf16 ulp, and NaN exactly where the oracle gives NaN."""
    w, b = run.w, run.b
    K, H = w["K"], w["H"]
    mode = run.omode
    cfg = ep.make_config(w["R"], w["T"], w["M"], K, w["E"], H, run.mode, run.layout, run.align,
                         run.qmax, run.cfg.flags | ep.F_COMBINE_QUANTIZED)
    ns, ks, rows = run.entries(None)
    data, scale = (rows_fn or quantized_rows)(mode, H, len(rows), seed)
    sz = run.sizes
    yq = torch.zeros(sz["recv_bytes"], dtype=torch.uint8, device="cuda")
    D, S = sz["data_row_bytes"], sz["scale_row_bytes"]
    rows_d = torch.from_numpy(rows).cuda()
    yq[: sz["rows"] * D].view(sz["rows"], D).index_copy_(0, rows_d, torch.from_numpy(data).cuda())
    if S:
        a = sz["recv_scale_offset"]
        yq[a: a + sz["rows"] * S].view(sz["rows"], S).index_copy_(0, rows_d, torch.from_numpy(scale).cuda())
    out = run.guards.alloc((w["N"], H), torch.bfloat16, "out (quantised combine)")
    out.fill_(1.0)
    ep.ep_combine(cfg, yq, run.idx_d, run.wts_d,
                  b.token_slot, out, b.dev_status, expert_offset=b.expert_offset)
    assert ep.ep_get_status(b.dev_status) == run.status
    run.guards.check()
    tokens = np.arange(w["N"]) if tokens is None else np.asarray(tokens)
    return _quantized_combine_matches(run, out, tokens, ns, ks, data, scale)
