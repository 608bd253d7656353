"""Expert parallelism over several GPUs, on one GPU: the G GPUs' windows are
emulated by G sets of buffers in this GPU's memory (no GPU waits on another:
every member's calls are issued one after another in stream order, and every
flag a wait looks at has been set by work issued before it).  The group's
kernels -- counts pushed to every window, the plan, the dispatch into the
owners' windows, the combine from them, the backward into them -- must give,
row for row and bit for bit, what the single-GPU path gives (itself checked
against the oracle by the harness).  Also: the plan kernel against the host
plan, waits that give up (EP_ERR_TIMEOUT) and leave the context usable, and
the CUDA IPC mapping between two processes (one reads the other's memory; no
kernel waits)."""
import ctypes as C
import os
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import combine_ep_dispatch_04_b200 as ep
import synth
from combine_ep_dispatch_04_b200.ep import lib
from combine_ep_dispatch_04_b200.group import EmulatedGroup
from harness import Run, to_np_u16

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class Members:
    """Per emulated GPU: its slice of the inputs and its own layout buffers."""

    def __init__(self, r, G, window_rows=0):
        self.r, self.G = r, G
        w, cfg = r.w, r.cfg
        self.cfg = cfg
        self.eg = EmulatedGroup(cfg, G, "cuda", grad=r.g is not None, weights=False,
                                window_rows=window_rows)
        R, T, K, E = w["R"], w["T"], w["K"], w["E"]
        self.RG, self.EG, self.T = R // G, E // G, T
        self.grps = [ep.make_group(G, g, 1, window_rows) for g in range(G)]
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        n = self.RG * T
        sl = [slice(g * n, (g + 1) * n) for g in range(G)]
        self.idx = [r.idx_d[s] for s in sl]
        self.x = [r.x_d[s] for s in sl]
        self.wts = [r.wts_d[s] for s in sl]
        self.g_in = [r.g_d[s] for s in sl] if r.g is not None else None
        self.slot = [torch.full((n, K), -9, dtype=torch.int32, device="cuda") for _ in range(G)]
        self.cnt = [torch.empty(E, dtype=torch.int64, device="cuda") for _ in range(G)]
        self.eo = [torch.empty(E + 1, dtype=torch.int64, device="cuda") for _ in range(G)]
        ws = self.eg.wins[0].sizes["workspace_bytes"]
        self.ws = [torch.empty(ws, dtype=torch.uint8, device="cuda") for _ in range(G)]
        self.scratch = [torch.empty(E, dtype=torch.int64, device="cuda") for _ in range(G)]
        self.sizes = self.eg.wins[0].sizes
        self.packed = cfg.layout == ep.LAYOUT["packed"]

    def eo_arg(self, g):
        return self.eo[g] if self.packed else None

    def dispatch(self, members=None):
        G, c, pe = self.G, self.cfg, self.eg.peers
        gs = range(G) if members is None else members
        for g in gs:
            ep.ep_group_layout(c, self.grps[g], pe[g], self.idx[g], self.slot[g], self.ws[g],
                               self.status)
        for g in gs:
            ep.ep_group_plan(c, self.grps[g], pe[g], self.idx[g], self.slot[g], self.cnt[g],
                             self.eo_arg(g), self.scratch[g], self.status)
        for g in gs:
            ep.ep_group_dispatch(c, self.grps[g], pe[g], self.x[g], self.idx[g], self.slot[g],
                                 self.status, expert_offset=self.eo_arg(g))
        for g in gs:
            ep.ep_group_wait(self.grps[g], pe[g], ep.GROUP_KIND_DISPATCH, self.status)

    def row_maps(self):
        """(owner, window row, single-GPU row) of every received row."""
        r, G, EG = self.r, self.G, self.EG
        lay = r.lay
        cap = r.w["R"] * r.w["M"]
        rows = self.sizes["rows"]
        eo_v = self.eo[0].cpu().numpy() if self.packed else None
        own, wrow, srow = [], [], []
        for e in range(r.w["E"]):
            o = e // EG
            for s in range(int(lay["recv_count"][e])):
                own.append(o)
                if self.packed:
                    wrow.append(int(eo_v[e]) - o * rows + s)
                    srow.append(int(lay["expert_offset"][e]) + s)
                else:
                    wrow.append((e - o * EG) * cap + s)
                    srow.append(e * cap + s)
        return np.array(own), np.array(wrow), np.array(srow)


def _window_rows(buf, rows, D, S, scale_off):
    data = buf[: rows * D].view(rows, D)
    scale = buf[scale_off: scale_off + rows * S].view(rows, S) if S else None
    return data, scale


CASES = [("mxfp8", "packed", 1, 2), ("mxfp8", "packed", 4, 4), ("e4m3_b128", "padded", 1, 2),
         ("bf16", "padded", 1, 4), ("int8_token", "packed", 1, 1), ("mxfp4", "packed", 2, 2)]


@pytest.mark.parametrize("mode,layout,align,G", CASES)
def test_group_equals_the_single_gpu_path(mode, layout, align, G):
    w = synth.workload("tiny", R=4, T=24, M=24, K=4, E=16, H=512)
    idx, wts = synth.make_routing(w)
    idx[5, 2] = -1
    r = Run(w, mode, layout=layout, align=align, idx=idx, wts=wts, backward=True)
    r.check_layout()
    r.check_dispatch(check_unwritten=False)
    r.check_combine()
    m = Members(r, G)
    m.dispatch()
    assert ep.ep_get_status(m.status) == 0
    # global slots and totals: the single-GPU layout's
    single_slot = r.b.token_slot.cpu().numpy()
    n = m.RG * m.T
    for g in range(G):
        assert np.array_equal(m.slot[g].cpu().numpy(), single_slot[g * n:(g + 1) * n])
        assert np.array_equal(m.cnt[g].cpu().numpy(), r.lay["recv_count"])
    # the plan kernel's offsets equal the host plan's
    tpe = r.b.tokens_per_expert.cpu().numpy()
    for g in range(G):
        _, total, eo_h = ep.ep_group_plan_host(m.cfg, m.grps[g], tpe)
        assert np.array_equal(total, r.lay["recv_count"])
        if m.packed:
            assert np.array_equal(m.eo[g].cpu().numpy(), eo_h)
    # every window row equals the single-GPU row of the same expert and slot
    sz = m.sizes
    own, wrow, srow = m.row_maps()
    D, S = sz["data_row_bytes"], sz["scale_row_bytes"]
    sd, ss = r.b.recv_data().cpu().numpy(), (r.b.recv_scale().cpu().numpy() if S else None)
    si = r.b.src_info.cpu().numpy()
    for o in range(G):
        win = m.eg.wins[o]
        data, scale = _window_rows(win.recv, sz["rows"], D, S, sz["recv_scale_offset"])
        sel = own == o
        assert np.array_equal(data.cpu().numpy()[wrow[sel]], sd[srow[sel]]), o
        if S:
            assert np.array_equal(scale.cpu().numpy()[wrow[sel]], ss[srow[sel]]), o
        assert np.array_equal(win.src_info.cpu().numpy()[wrow[sel]], si[srow[sel]]), o
    # expert outputs: each owner's y rows are the single-GPU y rows of its experts
    for o in range(G):
        sel = own == o
        m.eg.wins[o].y[torch.from_numpy(wrow[sel]).cuda()] = \
            r.b.y[torch.from_numpy(srow[sel]).cuda()]
    for g in range(G):
        ep.ep_group_signal(m.grps[g], m.eg.peers[g], ep.GROUP_KIND_EXPERT_OUT)
    outs = []
    for g in range(G):
        ep.ep_group_wait(m.grps[g], m.eg.peers[g], ep.GROUP_KIND_EXPERT_OUT, m.status)
        out = torch.full((n, w["H"]), 3.0, dtype=torch.bfloat16, device="cuda")
        ep.ep_group_combine(m.cfg, m.grps[g], m.eg.peers[g], m.idx[g], m.wts[g], m.slot[g], out,
                            m.status, expert_offset=m.eo_arg(g))
        outs.append(out)
    for g in range(G):
        ep.ep_group_signal(m.grps[g], m.eg.peers[g], ep.GROUP_KIND_COMBINED)
    for g in range(G):
        ep.ep_group_wait(m.grps[g], m.eg.peers[g], ep.GROUP_KIND_COMBINED, m.status)
    assert ep.ep_get_status(m.status) == 0
    assert np.array_equal(to_np_u16(torch.cat(outs)), to_np_u16(r.b.out))
    # backward into the owners' gradient windows
    for g in range(G):
        ep.ep_group_combine_backward(m.cfg, m.grps[g], m.eg.peers[g], m.g_in[g], m.idx[g],
                                     m.wts[g], m.slot[g], m.status, expert_offset=m.eo_arg(g))
    for g in range(G):
        ep.ep_group_wait(m.grps[g], m.eg.peers[g], ep.GROUP_KIND_BACKWARD, m.status)
    assert ep.ep_get_status(m.status) == 0
    H = w["H"]
    gd, gs = r.b.grad_data(H).cpu().numpy(), r.b.grad_scale(H).cpu().numpy()
    for o in range(G):
        win = m.eg.wins[o]
        data, scale = _window_rows(win.grad, sz["rows"], H, H // 32, sz["grad_scale_offset"])
        sel = own == o
        assert np.array_equal(data.cpu().numpy()[wrow[sel]], gd[srow[sel]]), o
        assert np.array_equal(scale.cpu().numpy()[wrow[sel]], gs[srow[sel]]), o


def test_group_two_steps_reuse_the_windows():
    """Epoch 2 on the same windows and flags, with a new routing: again the
    single-GPU rows."""
    w = synth.workload("tiny", R=4, T=16, M=16, K=3, E=8, H=256)
    idx1, wts1 = synth.make_routing(w, replica=1)
    r1 = Run(w, "mxfp8", layout="packed", idx=idx1, wts=wts1)
    m = Members(r1, 2)
    m.dispatch()
    for g in range(2):
        ep.ep_group_signal(m.grps[g], m.eg.peers[g], ep.GROUP_KIND_EXPERT_OUT)
        ep.ep_group_signal(m.grps[g], m.eg.peers[g], ep.GROUP_KIND_COMBINED)
    idx2, wts2 = synth.make_routing(w, replica=2)
    r2 = Run(w, "mxfp8", layout="packed", idx=idx2, wts=wts2)
    n = m.RG * m.T
    for g in range(2):
        m.grps[g].epoch = 2
        m.idx[g] = r2.idx_d[g * n:(g + 1) * n]
        m.x[g] = r2.x_d[g * n:(g + 1) * n]
    m.r = r2
    m.dispatch()
    assert ep.ep_get_status(m.status) == 0
    own, wrow, srow = m.row_maps()
    sz = m.sizes
    sd = r2.b.recv_data().cpu().numpy()
    for o in range(2):
        data, _ = _window_rows(m.eg.wins[o].recv, sz["rows"], sz["data_row_bytes"],
                               sz["scale_row_bytes"], sz["recv_scale_offset"])
        sel = own == o
        assert np.array_equal(data.cpu().numpy()[wrow[sel]], sd[srow[sel]])


def test_rows_past_a_window_are_skipped_and_flagged():
    """Windows smaller than their owners' rows: the rows that fit are the
    single-GPU rows, the others are skipped and the capacity bit is set."""
    w = synth.workload("tiny", R=4, T=24, M=24, K=4, E=8, H=256)
    r = Run(w, "mxfp8", layout="packed")
    need = int(r.lay["recv_count"][:4].sum())
    small = need // 2
    m = Members(r, 2, window_rows=small)
    m.dispatch()
    assert ep.ep_get_status(m.status) & ep.DEV_CAPACITY_OVERFLOW
    own, wrow, srow = m.row_maps()
    sz = m.sizes
    assert sz["rows"] == small
    sd = r.b.recv_data().cpu().numpy()
    for o in range(2):
        data, _ = _window_rows(m.eg.wins[o].recv, sz["rows"], sz["data_row_bytes"],
                               sz["scale_row_bytes"], sz["recv_scale_offset"])
        sel = (own == o) & (wrow < small)
        assert np.array_equal(data.cpu().numpy()[wrow[sel]], sd[srow[sel]]), o


def test_plan_kernel_equals_the_host_plan_on_many_shapes():
    """The plan kernel (one block: warp sums and a block-wide scan) against the
    host plan (the plain loops), for every member of several group sizes, on
    counts of real routings; the counts table is written into the window
    directly (no other member takes part: its COUNTS flags are set by hand)."""
    rng = np.random.default_rng(5)
    for (R, E, G, align) in [(8, 64, 4, 1), (16, 256, 8, 4), (4, 1024, 2, 3), (32, 256, 1, 1)]:
        T, K = 8, 4
        cfg = ep.make_config(R, T, T, K, E, 256, "mxfp8", "packed", align)
        eg = EmulatedGroup(cfg, G, "cuda")
        idx = rng.integers(-1, E, (R * T, K))
        tpe = np.stack([np.bincount(idx[r * T:(r + 1) * T][idx[r * T:(r + 1) * T] >= 0],
                                    minlength=E) for r in range(R)]).astype(np.int32)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        for g in range(G):
            win = eg.wins[g]
            win.counts.copy_(torch.from_numpy(tpe))
            win.flags[ep.GROUP_KIND_COUNTS].fill_(1)
            grp = ep.make_group(G, g, 1)
            n = (R // G) * T
            idx_g = torch.from_numpy(idx[g * n:(g + 1) * n].copy()).cuda()
            slot = torch.zeros((n, K), dtype=torch.int32, device="cuda")
            cnt = torch.empty(E, dtype=torch.int64, device="cuda")
            eo = torch.empty(E + 1, dtype=torch.int64, device="cuda")
            scratch = torch.empty(E, dtype=torch.int64, device="cuda")
            ep.ep_group_plan(cfg, grp, eg.peers[g], idx_g, slot, cnt, eo, scratch, status)
            base, total, eo_h = ep.ep_group_plan_host(cfg, grp, tpe)
            assert ep.ep_get_status(status) == 0
            assert np.array_equal(cnt.cpu().numpy(), total)
            assert np.array_equal(eo.cpu().numpy(), eo_h)
            valid = idx[g * n:(g + 1) * n] >= 0
            want = np.where(valid, base[np.maximum(idx[g * n:(g + 1) * n], 0)], 0)
            assert np.array_equal(slot.cpu().numpy(), want)


def test_a_member_that_withholds_its_counts_times_out():
    """Of two emulated GPUs only the first lays out its tokens and sends its
    counts: its plan waits for the second's counts, gives up after the bound,
    and ep_get_status reports EP_ERR_TIMEOUT (the DEV_TIMEOUT bit); the
    context stays usable.  A wait for a signal nobody sends gives up the same
    way after its own short limit."""
    w = synth.workload("tiny", R=2, T=16, M=16, K=2, E=4, H=256)
    r = Run(w, "mxfp8", layout="packed")
    m = Members(r, 2)
    c, pe = m.cfg, m.eg.peers
    ep.ep_group_layout(c, m.grps[0], pe[0], m.idx[0], m.slot[0], m.ws[0], m.status)
    ep.ep_group_plan(c, m.grps[0], pe[0], m.idx[0], m.slot[0], m.cnt[0], m.eo[0], m.scratch[0],
                     m.status)
    flags = ep.ep_get_status(m.status)
    assert flags & ep.DEV_TIMEOUT
    assert lib.ep_get_status(C.c_void_p(m.status.data_ptr()), C.byref(C.c_uint32(0)),
                                C.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    ep.ep_group_wait(m.grps[0], pe[0], ep.GROUP_KIND_EXPERT_OUT, m.status, timeout_ns=50_000_000)
    st = C.c_uint32(0)
    assert lib.ep_get_status(C.c_void_p(m.status.data_ptr()), C.byref(st),
                                C.c_void_p(torch.cuda.current_stream().cuda_stream)) == 6
    assert st.value & ep.DEV_TIMEOUT
    r2 = Run(w, "mxfp8", layout="packed")   # the context is still usable
    r2.check_layout()
    r2.check_dispatch()


def _ipc_owner(q_out, q_in):
    sys.path.insert(0, ROOT)
    import combine_ep_dispatch_04_b200 as ep_
    t = torch.arange(1 << 20, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    q_out.put(ep_.ep_ipc_export(t[4096:]))
    assert q_in.get(timeout=120) == "done"      # keep the memory alive until read


def _ipc_reader(q_in, q_out, res):
    sys.path.insert(0, ROOT)
    import combine_ep_dispatch_04_b200 as ep_
    h, off = q_in.get(timeout=120)
    addr = ep_.ep_ipc_import(h, off)
    dst = torch.zeros((1 << 20) - 4096, dtype=torch.int32, device="cuda")
    st = ep_.ep.lib.ep_copy(C.c_void_p(dst.data_ptr()), C.c_void_p(addr), dst.numel() * 4,
                         C.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    ok = st == 0 and bool(torch.equal(dst.cpu(), torch.arange(4096, 1 << 20, dtype=torch.int32)))
    ep_.ep_ipc_close(addr - off)
    q_out.put("done")
    res.put(ok)


def test_ipc_export_and_import_between_two_processes():
    """One process exports a buffer (an offset into its allocation); another maps
    it and copies it out with the library's copy kernel: the same bytes."""
    ctx = mp.get_context("spawn")
    q1, q2, res = ctx.Queue(), ctx.Queue(), ctx.Queue()
    a = ctx.Process(target=_ipc_owner, args=(q1, q2))
    b = ctx.Process(target=_ipc_reader, args=(q1, q2, res))
    a.start()
    b.start()
    ok = res.get(timeout=180)
    a.join(timeout=60)
    b.join(timeout=60)
    assert ok and a.exitcode == 0 and b.exitcode == 0
