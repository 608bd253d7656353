"""Seeded synthetic inputs for MoE dispatch / combine.

Shared by the tests, the smoke check and the benchmark.  This module holds
input recipes only -- token activations, routing, weights, expert outputs
and gradients -- and none of the dispatch / combine arithmetic.  Every draw
comes from numpy's Philox4x32-10 counter-based generator (Salmon et al.,
"Parallel random numbers: as easy as 1, 2, 3", SC'11), keyed by
(workload id, tensor tag, replica), so that any tensor can be rebuilt on any
host from its key alone.

Matrices (x, expert outputs y, gradients g) are rows cut from a seeded pool:
row i is ``pool[off_i : off_i + H]`` with ``off_i`` uniform in [0, 2^24).
Each element is an independent draw of the stated distribution; rows are
windows of one long iid sequence, which lets a device rebuild a 15 GB
expert-output buffer from a 32 MB pool while a host rebuilds only the rows it
samples.

Workloads (the five named MoE dispatch / combine shapes, and the deep fused MoE
page's benchmark case):
  tiny     R=1  T=128  H=1024 K=2 E=8   M=128  N(0,1) x, uniform top-2, 5% -1
  decode   R=8  T=128  H=7168 K=8 E=256 M=128  N(0,1) x, uniform top-8
  skewed   R=16 T=512  H=4096 K=6 E=64  M=512  N(0,1) x with 1% channels x50,
                                              Zipf(1.2) expert popularity
  prefill  R=32 T=4096 H=7168 K=8 E=256 M=4096 N(0,1) x, uniform, 2% -1
  large    R=64 T=256  H=7168 K=8 E=256 M=256  0.5*Student-t(3) x, Zipf(0.8)
  a5       R=8  T=128  H=7168 K=6 E=48  M=128  N(0,1) x, uniform top-6; the experts'
                                              gated MLP has intermediate size 3072
Routing draws K distinct experts per token without replacement with
probabilities p_e (uniform, or p_e ~ 1/rank(e)^s with a seeded rank
permutation) by the Gumbel-top-K construction; the order of the K picks is the
order of the sequential draw.  Each entry is then replaced by -1 with
probability mask_p.  Weights are the softmax over K of N(0,1) draws, taken
before masking and never renormalised.
"""
import copy

import numpy as np

POOL = 1 << 24

WORKLOADS = {
    "tiny": dict(wid=1, R=1, T=128, H=1024, K=2, E=8, M=128, routing="uniform", zipf_s=0.0,
                 mask_p=0.05, x="normal", modes=("bf16", "int8_token"), layout="padded"),
    "decode": dict(wid=2, R=8, T=128, H=7168, K=8, E=256, M=128, routing="uniform", zipf_s=0.0,
                   mask_p=0.0, x="normal", modes=("e4m3_b128",), layout="padded"),
    "skewed": dict(wid=3, R=16, T=512, H=4096, K=6, E=64, M=512, routing="zipf", zipf_s=1.2,
                   mask_p=0.0, x="outlier", modes=("int8_token",), layout="padded"),
    "prefill": dict(wid=4, R=32, T=4096, H=7168, K=8, E=256, M=4096, routing="uniform",
                    zipf_s=0.0, mask_p=0.02, x="normal", modes=("mxfp8",), layout="packed",
                    backward=True),
    "large": dict(wid=5, R=64, T=256, H=7168, K=8, E=256, M=256, routing="zipf", zipf_s=0.8,
                  mask_p=0.0, x="student_t", modes=("mxfp4",), layout="packed"),
    # the deep fused MoE page's benchmark case on one GPU: EP 8 (logical ranks),
    # 128 tokens a rank, hidden 7168, top-6 of 48 experts (6 a rank), uniform
    # routing, FP8 (MXFP8), moe-intermediate-size 3072
    "a5": dict(wid=6, R=8, T=128, H=7168, K=6, E=48, M=128, routing="uniform", zipf_s=0.0,
               mask_p=0.0, x="normal", modes=("mxfp8",), layout="packed", inter=3072),
}

# tensor tags inside one workload's key space
_T_XPOOL, _T_XOFF, _T_ROUTE, _T_MASK, _T_W, _T_YPOOL, _T_YOFF, _T_GPOOL, _T_GOFF, _T_OUTLIER, \
    _T_ZIPF = range(1, 12)


def workload(name, **override):
    """A copy of a named workload, optionally with fields replaced (e.g. a
    reduced T for a test that the oracle finishes in seconds)."""
    w = copy.deepcopy(WORKLOADS[name])
    w.update(override)
    w["name"] = name
    w["N"] = w["R"] * w["T"]
    return w


def rng(wid, tag, replica=0):
    key = np.array([(int(wid) << 32) | int(tag), int(replica)], dtype=np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def to_bf16_bits(f32):
    """float32 -> bf16 bit patterns, round to nearest even (input recipe only)."""
    b = np.ascontiguousarray(f32, np.float32).view(np.uint32)
    return ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


# ---- pools and windows ------------------------------------------------------

def _pool_f32(kind, wid, tag, H, replica):
    g = rng(wid, tag, replica)
    n = POOL + H
    if kind in ("normal", "outlier"):
        return g.standard_normal(n, dtype=np.float32)
    if kind == "student_t":
        return (0.5 * g.standard_t(3, size=n)).astype(np.float32)
    raise ValueError(kind)


def windows(pool, offsets, H):
    """Rows pool[off : off + H] for each offset (host gather, one slice copy per row)."""
    offsets = np.asarray(offsets, np.int64).reshape(-1)
    out = np.empty((offsets.size, H), pool.dtype)
    for i, o in enumerate(offsets.tolist()):
        out[i] = pool[o:o + H]
    return out


def windows_torch(pool_dev, offsets_dev, H):
    """The same rows gathered on a device from a device copy of the pool."""
    view = pool_dev.as_strided((POOL, H), (1, 1))
    return view.index_select(0, offsets_dev)


def offsets(wid, tag, rows, replica=0):
    return rng(wid, tag, replica).integers(0, POOL, size=rows, dtype=np.int64)


def outlier_channels(w, replica=0):
    """1% of the channels (41 of 4096), the same for every token."""
    n = max(1, int(round(0.01 * w["H"])))
    return np.sort(rng(w["wid"], _T_OUTLIER, replica).permutation(w["H"])[:n])


def x_source(w, replica=0):
    """(pool of bf16 bits, row offsets) for the activations x; None for the
    outlier recipe, whose rows are built on the host by make_x."""
    if w["x"] == "outlier":
        return None
    pool = to_bf16_bits(_pool_f32(w["x"], w["wid"], _T_XPOOL, w["H"], replica))
    return pool, offsets(w["wid"], _T_XOFF, w["N"], replica)


def make_x(w, replica=0, rows=None):
    """x as bf16 bits [N, H] (or only the listed rows)."""
    H = w["H"]
    if w["x"] == "outlier":
        pool = _pool_f32("normal", w["wid"], _T_XPOOL, H, replica)
        off = offsets(w["wid"], _T_XOFF, w["N"], replica)
        if rows is not None:
            off = off[np.asarray(rows)]
        z = windows(pool, off, H)
        factor = np.ones(H, np.float32)
        factor[outlier_channels(w, replica)] = np.float32(50.0)
        return to_bf16_bits(z * factor)
    pool, off = x_source(w, replica)
    if rows is not None:
        off = off[np.asarray(rows)]
    return windows(pool, off, H)


def y_source(w, rows, replica=0):
    """Expert outputs: (pool of N(0,1) bf16 bits, offsets for `rows` buffer rows)."""
    pool = to_bf16_bits(_pool_f32("normal", w["wid"], _T_YPOOL, w["H"], replica))
    return pool, offsets(w["wid"], _T_YOFF, rows, replica)


def g_source(w, replica=0):
    """Result gradient g [N, H] for the combine backward: N(0,1) bf16 rows."""
    pool = to_bf16_bits(_pool_f32("normal", w["wid"], _T_GPOOL, w["H"], replica))
    return pool, offsets(w["wid"], _T_GOFF, w["N"], replica)


# ---- routing ------------------------------------------------------------------

def make_routing(w, replica=0):
    """(topk_idx int64 [N, K], topk_weights float32 [N, K])."""
    N, K, E = w["N"], w["K"], w["E"]
    g = rng(w["wid"], _T_ROUTE, replica)
    logp = np.zeros(E)
    if w["routing"] == "zipf":
        rank = rng(w["wid"], _T_ZIPF, replica).permutation(E) + 1
        logp = -w["zipf_s"] * np.log(rank.astype(np.float64))
    idx = np.empty((N, K), np.int64)
    chunk = 1 << 14
    for a in range(0, N, chunk):
        b = min(N, a + chunk)
        u = g.random((b - a, E))
        keys = logp[None, :] - np.log(-np.log(u))      # Gumbel-perturbed log-probabilities
        top = np.argpartition(-keys, K - 1, axis=1)[:, :K]
        order = np.argsort(-np.take_along_axis(keys, top, axis=1), axis=1, kind="stable")
        idx[a:b] = np.take_along_axis(top, order, axis=1)
    if w["mask_p"] > 0:
        drop = rng(w["wid"], _T_MASK, replica).random((N, K)) < w["mask_p"]
        idx[drop] = -1
    z = rng(w["wid"], _T_W, replica).standard_normal((N, K))
    z = np.exp(z - z.max(axis=1, keepdims=True))
    wts = (z / z.sum(axis=1, keepdims=True)).astype(np.float32)
    return idx, wts
