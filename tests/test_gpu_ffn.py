"""The experts' gated MLP on the GPU ("[feat] A5 deep fused moe supported":
GMM1, SwiGLU, Requant, GMM2 between the dispatch and the combine) against the
oracle, through the C ABI.

The GPU's GMM1 sums in the tensor cores' order and its SwiGLU uses the fp32
expf, so its z differs from the oracle's (exact sums rounded once, silu in
double) by a bounded amount, derived here from the oracle's own values:
  h:  (H/32 + 32) * 2^-23 * sum_k |x*w1| (the chained block sums) + 1 fp32 ulp
  z:  silu' <= 1.1, so |dz| <= 1.1 (|u| + du) dg + (|silu(g)| + 1.1 dg) du
      + 8 fp32 ulps of z (the kernel's own expf, division and products)
Every requantised code must then be the MXFP8 rounding of some value inside
z's window: its block's scale between the scales of the window's smallest and
largest block maxima, and its value between the e4m3 roundings of the
window's ends at that scale.  At least 99% of the codes and scales equal the
oracle's.  The bf16 outputs y are bounded by the second GEMM's chain plus, per
element of z, the window and one e4m3 step at the largest admissible scale,
weighted by |w2|.  The oracle's inputs are its own layout and quantisation of
the seeded x; nothing it sees comes from the device."""
import numpy as np
import pytest
import torch

import combine_ep_dispatch_04_b200 as ep
import oracle
import synth
from harness import Guards, Run, bf16_dev, to_np_u16

pytestmark = pytest.mark.gpu


def _mx_weights(E, n, k, lo, hi, seed):
    gen = torch.Generator(device="cuda").manual_seed(seed)
    c = torch.randint(0, 256, (E, n, k), device="cuda", dtype=torch.int16,
                      generator=gen).to(torch.uint8)
    c[(c & 0x7F) == 0x7F] = 0                      # no NaN codes
    s = torch.randint(lo, hi, (E, n, k // 32), device="cuda", dtype=torch.int16,
                      generator=gen).to(torch.uint8)
    return c, s


def _lut():
    return oracle.e4m3_decode(np.arange(256, dtype=np.uint8)).astype(np.float64)


def _mxv(c, s):
    """Values of MXFP8 codes c with e8m0 scales s (exact in float32 for the
    scales used here: e4m3 values times powers of two in range)."""
    lut = _lut().astype(np.float32)
    return lut[c] * np.ldexp(np.float32(1.0), np.repeat(s.astype(np.int32) - 127, 32, axis=-1))


def _ulp32(v):
    return np.spacing(np.abs(v).astype(np.float32)).astype(np.float64)


def _e4m3_step(a):
    """e4m3 spacing at magnitude a (a in units of the block scale)."""
    return np.ldexp(1.0, np.floor(np.log2(np.maximum(a, 2.0 ** -6))).astype(np.int64) - 3)


class Ffn:
    """One dispatch (GPU, checked bit-exact against the oracle) followed by the
    experts' gated MLP on the GPU, and the oracle's chain on its own rows."""

    def __init__(self, w, I, seed=1, w1_scales=(115, 119), w2_scales=(112, 116), sample=None,
                 idx=None, wts=None, weights=None, experts=None):
        self.w, self.I = w, I
        self.r = r = Run(w, "mxfp8", layout="packed", idx=idx, wts=wts)
        r.check_layout()
        r.check_dispatch(check_unwritten=False)
        E, H = w["E"], w["H"]
        if weights is None:
            weights = _mx_weights(E, 2 * I, H, *w1_scales, seed) + \
                _mx_weights(E, H, I, *w2_scales, seed + 1)
        self.w1c, self.w1s, self.w2c, self.w2s = weights
        zb, zoff = ep.ep_ffn_buffer_bytes(r.cfg, I)
        rows = r.sizes["rows"]
        self.z_buf = r.guards.alloc((zb,), torch.uint8, "z_buf")
        self.z_buf.fill_(0xCD)
        self.zoff = zoff
        self.y = r.guards.alloc((rows, H), torch.bfloat16, "y")
        self.y.view(torch.int16).fill_(0x7777)
        ep.ep_expert_ffn_mx(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, self.w1c,
                            self.w1s, self.w2c, self.w2s, self.z_buf, self.y, r.b.dev_status)
        assert ep.ep_get_status(r.b.dev_status) == 0
        r.guards.check()
        # the oracle on its own quantisation of the seeded x, row by row
        o = r.lay
        eo, cnt = o["expert_offset"], o["recv_count"]
        valid = np.zeros(rows, bool)
        for e in range(E):
            valid[eo[e]:eo[e] + cnt[e]] = True
        self.valid = valid
        ns, _, rr = r.entries()
        tok_of_row = np.full(rows, -1, np.int64)
        tok_of_row[rr] = ns
        expert_of = np.repeat(np.arange(E), np.diff(eo[:E + 1]))
        pick = np.nonzero(valid)[0]
        if experts is not None:  # sample from a few experts: the oracle dequantises each once
            chosen = np.random.default_rng(seed).choice(np.unique(expert_of[pick]), experts,
                                                        replace=False)
            pick = pick[np.isin(expert_of[pick], chosen)]
        if sample is not None and len(pick) > sample:
            pick = np.sort(np.random.default_rng(seed).choice(pick, sample, replace=False))
        self.pick = pick
        w1c, w1s = self.w1c.cpu().numpy(), self.w1s.cpu().numpy()
        w2c, w2s = self.w2c.cpu().numpy(), self.w2s.cpu().numpy()
        self.o = {k: [] for k in ("h", "z", "zc", "zs", "y", "xv", "e")}
        for e in np.unique(expert_of[pick]):
            rs = pick[expert_of[pick] == e]
            q = [oracle.quant_row("mxfp8", r.x[n]) for n in tok_of_row[rs]]
            xc, xs = np.stack([d for d, _ in q]), np.stack([s_ for _, s_ in q])
            oo = oracle.expert_ffn_mx(xc, xs, w1c[e][None], w1s[e][None], w2c[e][None],
                                      w2s[e][None], np.zeros(1, np.int64),
                                      np.array([len(rs)], np.int64))
            for k in ("h", "z", "zc", "zs", "y"):
                self.o[k].append(oo[k])
            self.o["xv"].append(_mxv(xc, xs))
            self.o["e"].append(np.full(len(rs), e))
        self.order = np.concatenate([pick[expert_of[pick] == e] for e in np.unique(expert_of[pick])])
        for k in self.o:
            self.o[k] = np.concatenate(self.o[k])
        self.wh = (w1c, w1s, w2c, w2s)

    def _per_expert(self, which, fn):
        """fn(|W| of expert e as float32, sampled rows of e) for each expert in the
        sample, one expert's weights in memory at a time; rows stacked in order."""
        w1c, w1s, w2c, w2s = self.wh
        out = []
        for e in np.unique(self.o["e"]):
            sel = np.nonzero(self.o["e"] == e)[0]
            c, sc = (w1c[e], w1s[e]) if which == 1 else (w2c[e], w2s[e])
            W = np.abs(_mxv(c, sc)).astype(np.float32)
            out.append((sel, fn(W, sel)))
            del W
        res = np.empty((len(self.o["e"]),) + out[0][1].shape[1:])
        for sel, v in out:
            res[sel] = v
        return res

    def gpu_z(self):
        rows, I = self.r.sizes["rows"], self.I
        zb = self.z_buf.cpu().numpy()
        zc = zb[:rows * I].reshape(rows, I)
        zs = zb[self.zoff:self.zoff + rows * (I // 32)].reshape(rows, I // 32)
        return zc, zs

    def check_z(self):
        """Every code and scale admissible, >= 99% equal; untouched rows stay 0xCD.
        Returns (z window, largest admissible scale exponent) per sampled row."""
        I, H = self.I, self.w["H"]
        zc_all, zs_all = self.gpu_z()
        assert np.all(zc_all[~self.valid] == 0xCD) and np.all(zs_all[~self.valid] == 0xCD)
        zc, zs = zc_all[self.order], zs_all[self.order]
        h, z = self.o["h"].astype(np.float64), self.o["z"].astype(np.float64)
        chain = H // 32 + 32
        xa = np.abs(self.o["xv"]).astype(np.float32)  # float32 sums: the 1 + 2^-10 margin covers them
        mag = self._per_expert(1, lambda W, sel: (xa[sel] @ W.T).astype(np.float64))
        dh = chain * 2.0 ** -23 * mag * (1 + 2.0 ** -10) + _ulp32(h)
        g, u, dg, du = h[:, :I], h[:, I:], dh[:, :I], dh[:, I:]
        silu = g / (1.0 + np.exp(-g))
        dz = 1.1 * (np.abs(u) + du) * dg + (np.abs(silu) + 1.1 * dg) * du + 8 * _ulp32(z)
        lut = _lut()
        Xg = zs.astype(np.int64) - 127
        Xhi = np.empty_like(Xg)
        for b in range(I // 32):
            sl = slice(32 * b, 32 * b + 32)
            lo_max = np.maximum(np.abs(z[:, sl]) - dz[:, sl], 0).max(axis=1).astype(np.float32)
            hi_max = (np.abs(z[:, sl]) + dz[:, sl]).max(axis=1).astype(np.float32)
            x_lo = oracle.mx_exponent(lo_max, 448.0)
            x_hi = oracle.mx_exponent(np.minimum(hi_max, np.float32(3e38)), 448.0)
            assert np.all((Xg[:, b] >= x_lo) & (Xg[:, b] <= x_hi)), b
            Xhi[:, b] = x_hi
            sc = np.ldexp(1.0, -Xg[:, b])[:, None]
            lo_c = oracle.e4m3_encode(((z[:, sl] - dz[:, sl]) * sc).astype(np.float32))
            hi_c = oracle.e4m3_encode(((z[:, sl] + dz[:, sl]) * sc).astype(np.float32))
            v = lut[zc[:, sl]]
            assert np.all((v >= lut[lo_c]) & (v <= lut[hi_c])), b
        same_c = float((zc == self.o["zc"]).mean())
        same_s = float((zs == self.o["zs"]).mean())
        assert same_c >= 0.99 and same_s >= 0.99, (same_c, same_s)
        return dz, Xhi

    def y_allowance(self, dz, Xhi):
        """Per sampled row and output: how far the GPU's y may be from the oracle's."""
        I, H = self.I, self.w["H"]
        q = _mxv(self.o["zc"], self.o["zs"])
        step = _e4m3_step((np.abs(self.o["z"]) + dz) * np.ldexp(1.0, -np.repeat(Xhi, 32, axis=1))) * \
            np.ldexp(1.0, np.repeat(Xhi, 32, axis=1))
        dq = (dz + step).astype(np.float32)
        qa = (np.abs(q) + dq).astype(np.float32)
        chain = (I // 32 + 32) * 2.0 ** -23
        allow = self._per_expert(2, lambda W, sel: (dq[sel] @ W.T).astype(np.float64) * 1.001 +
                                 chain * (qa[sel] @ W.T).astype(np.float64) * 1.001)
        return allow + 2.0 * _bf16_ulp(self.o["y"])

    def check_y(self, dz, Xhi):
        got = to_np_u16(self.y)
        assert np.all(got[~self.valid] == 0x7777)
        g, o = _f(got[self.order]), _f(self.o["y"])
        allow = self.y_allowance(dz, Xhi)
        assert np.all(np.abs(g - o) <= allow), float((np.abs(g - o) - allow).max())
        return float((got[self.order] == self.o["y"]).mean())


def _f(u16):
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _bf16_ulp(bits):
    v = np.abs(_f(bits))
    return np.ldexp(1.0, np.floor(np.log2(np.maximum(v, 2.0 ** -126))).astype(np.int64) - 7)


@pytest.mark.parametrize("I", [128, 256, 384])
def test_ffn_small_ragged(I):
    """Several column tiles of GMM1 (64 gate + 64 up columns each), ragged experts
    (one past a 128-row tile, one empty), against the oracle."""
    w = synth.workload("tiny", R=2, T=96, M=96, K=4, E=8, H=512)
    idx, wts = synth.make_routing(w)
    idx[idx == 5] = 2                      # expert 5 receives nothing, expert 2 over 128 rows
    f = Ffn(w, I, idx=idx, wts=wts)
    dz, xhi = f.check_z()
    frac = f.check_y(dz, xhi)
    assert frac >= 0.5, frac


def test_ffn_wide_tiles():
    """At least 256 entries an expert on average: GMM1 takes 128 gate + 128 up
    columns per tile (one accumulator)."""
    w = synth.workload("tiny", R=4, T=256, M=256, K=4, E=4, H=256)
    f = Ffn(w, 256, w1_scales=(117, 121), sample=400)
    dz, xhi = f.check_z()
    f.check_y(dz, xhi)


def test_ffn_page_shape_sampled():
    """The benchmark case of the deep fused MoE page on one GPU: 8 ranks x 128
    tokens, hidden 7168, intermediate 3072, top-6 of 48 experts (6 a rank),
    MXFP8; 24 rows of three experts against the oracle."""
    w = synth.workload("a5", T=128)
    f = Ffn(w, 3072, w1_scales=(112, 116), w2_scales=(110, 114), sample=24, experts=3)
    dz, xhi = f.check_z()
    f.check_y(dz, xhi)


def test_ffn_rejects_other_formats_and_short_buffers():
    w = synth.workload("tiny", R=2, T=16, M=16, K=2, E=4, H=256)
    r = Run(w, "bf16", layout="packed")
    w1c, w1s = _mx_weights(4, 256, 256, 115, 119, 3)
    w2c, w2s = _mx_weights(4, 256, 128, 115, 119, 4)
    y = torch.empty((r.sizes["rows"], 256), dtype=torch.bfloat16, device="cuda")
    z = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    r2 = Run(w, "mxfp8", layout="packed")
    n0 = ep.ep_kernel_launches()
    with pytest.raises(ep.EpError) as ei:
        ep.ep_expert_ffn_mx(r.cfg, r.b.recv_buf, r.b.expert_offset, r.b.recv_count, w1c, w1s,
                            w2c, w2s, z, y, r.b.dev_status)
    assert ei.value.status == 2                       # bf16 rows: unsupported
    zb, _ = ep.ep_ffn_buffer_bytes(r2.cfg, 128)
    with pytest.raises(ep.EpError) as ei:
        ep.ep_expert_ffn_mx(r2.cfg, r2.b.recv_buf, r2.b.expert_offset, r2.b.recv_count, w1c,
                            w1s, w2c, w2s, z[:zb - 1], y, r2.b.dev_status)
    assert ei.value.status == ep.ERR_BUFFER_TOO_SMALL
    assert ep.ep_kernel_launches() == n0


def test_moe_forward_ffn_equals_the_calls_one_by_one_and_the_oracle_chain():
    """Layout + dispatch, the gated MLP and the combine in one call: bit for
    bit the calls made one by one, and within the chain's bound of the
    oracle's chain (each expert output within its allowance, scaled by |w_k|,
    plus two bf16 ulps of the combined value)."""
    w = synth.workload("tiny", R=2, T=48, M=48, K=4, E=8, H=512)
    I = 256
    idx, wts = synth.make_routing(w)
    x = synth.make_x(w)
    cfg = ep.make_config(w["R"], w["T"], w["M"], w["K"], w["E"], w["H"], "mxfp8", "packed")
    w1c, w1s = _mx_weights(w["E"], 2 * I, w["H"], 115, 119, 21)
    w2c, w2s = _mx_weights(w["E"], w["H"], I, 112, 116, 22)
    x_d, idx_d, wts_d = bf16_dev(x), torch.from_numpy(idx).cuda(), torch.from_numpy(wts).cuda()
    zb, _ = ep.ep_ffn_buffer_bytes(cfg, I)
    outs = []
    for one_call in (True, False):
        guards = Guards()
        b = guards.wrap(ep.Buffers(cfg))
        z = guards.alloc((zb,), torch.uint8, "z_buf")
        y = guards.alloc((b.sizes["rows"], w["H"]), torch.bfloat16, "y")
        out = guards.alloc((w["N"], w["H"]), torch.bfloat16, "out")
        if one_call:
            n0 = ep.ep_kernel_launches()
            ep.ep_moe_forward_ffn(cfg, x_d, idx_d, wts_d, w1c, w1s, w2c, w2s, b.token_slot,
                                  b.recv_count, b.expert_offset, b.workspace, b.recv_buf,
                                  b.src_info, z, y, out, b.dev_status)
            assert ep.ep_kernel_launches() - n0 == 5   # layout, dispatch, GMM1, GMM2, combine
        else:
            ep.ep_dispatch_layout(cfg, idx_d, b.token_slot, b.recv_count, b.workspace,
                                  b.dev_status, expert_offset=b.expert_offset)
            ep.ep_dispatch(cfg, x_d, idx_d, b.token_slot, b.recv_buf, b.src_info, b.dev_status,
                           expert_offset=b.expert_offset)
            ep.ep_expert_ffn_mx(cfg, b.recv_buf, b.expert_offset, b.recv_count, w1c, w1s, w2c,
                                w2s, z, y, b.dev_status)
            ep.ep_combine(cfg, y, idx_d, wts_d, b.token_slot, out, b.dev_status,
                          expert_offset=b.expert_offset)
        assert ep.ep_get_status(b.dev_status) == 0
        guards.check()
        outs.append(to_np_u16(out))
    assert np.array_equal(outs[0], outs[1])
    # the oracle's chain: its layout, quantisation, gated MLP and combine
    f = Ffn(w, I, idx=idx, wts=wts, weights=(w1c, w1s, w2c, w2s))
    o = f.r.lay
    rows = f.r.sizes["rows"]
    yo = np.zeros((rows, w["H"]), np.uint16)
    yo[f.order] = f.o["y"]
    want, st = oracle.combine(w["R"], w["T"], w["K"], w["E"], w["M"], w["H"], yo, idx, wts,
                              o["token_slot"], o["expert_offset"], layout="packed")
    assert st == 0
    dz, xhi = f.check_z()
    allow_rows = np.zeros((rows, w["H"]))
    allow_rows[f.order] = f.y_allowance(dz, xhi)
    bound = 2.0 * _bf16_ulp(want)
    ns, ks, rr = f.r.entries()
    for n, k, row in zip(ns, ks, rr):
        bound[n] += abs(float(wts[n, k])) * allow_rows[row]
    got = outs[0]
    err = np.abs(_f(got) - _f(want))
    assert np.all(err <= bound), float((err - bound).max())
