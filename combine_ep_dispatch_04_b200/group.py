"""Expert parallelism over several GPUs, one process each ("Low-Latency Mode
API": each rank dispatches its tokens into the receive buffers of the ranks
that own their experts and combines the experts' outputs back; "[Common]
[PyTorch] EP dispatch with unfused MXFP8 quantization", Changes: symmetric
windows, combine forward and backward as the reverse of the dispatch).

Every step of the data path runs in libep's kernels over peer memory
(include/ep.h, ep_group_*): the counts exchange, the slot plan, the dispatch
into the owners' windows, the combine from them, and the bounded waits
between.  This module holds the plumbing around them: the caller-owned
windows of one GPU (torch allocations), the tables of every GPU's window
addresses, the one-time exchange of CUDA IPC handles over torch.distributed,
and the order of the calls in one step.

Windows of GPU g (rows = ep_group_sizes()["rows"], the single-GPU row format):
  recv      receive window: codes [rows][D], then scales [rows][S]
  src_info  int32 [rows]
  y         bf16 [rows][H]: the expert outputs the owners' experts write
  grad      MXFP8 gradient window (optional)
  counts    int32 [R][E]: every rank's per-expert counts
  flags     uint64 [kinds][G]; done uint32 [kinds]
"""
import datetime

import torch

from . import ep

KINDS = ep.GROUP_KINDS


class Windows:
    """The windows of one GPU of the group, allocated by the caller (torch)."""

    def __init__(self, cfg, grp, device, grad=False, weights=False):
        self.sizes = sz = ep.ep_group_sizes(cfg, grp)
        u8 = dict(dtype=torch.uint8, device=device)
        rows, H = sz["rows"], cfg.hidden
        self.recv = torch.empty(sz["recv_bytes"], **u8)
        self.src_info = torch.empty(rows, dtype=torch.int32, device=device)
        self.recv_weights = torch.empty(rows, dtype=torch.float32, device=device) \
            if weights else None
        self.y = torch.empty((rows, H), dtype=torch.bfloat16, device=device)
        self.grad = torch.empty(sz["grad_bytes"], **u8) if grad else None
        self.counts = torch.zeros((cfg.num_ranks, cfg.num_experts), dtype=torch.int32,
                                  device=device)
        self.flags = torch.zeros((KINDS, grp.world), dtype=torch.int64, device=device)
        self.done = torch.zeros(KINDS, dtype=torch.int32, device=device)

    FIELDS = ("recv", "src_info", "recv_weights", "y", "grad", "counts", "flags")

    def pointers(self):
        return {f: (getattr(self, f).data_ptr() if getattr(self, f) is not None else 0)
                for f in self.FIELDS}


def peer_struct(tables, mine, device):
    """An EpPeers from per-field lists of G device addresses (`tables`) and this
    GPU's own Windows.  The address arrays live in device memory (returned
    with the struct, which keeps them alive)."""
    keep = {}
    st = ep.EpPeers()
    for f in Windows.FIELDS:
        addrs = tables[f]
        if all(a == 0 for a in addrs):
            setattr(st, f, None)
            continue
        t = torch.tensor(addrs, dtype=torch.int64, device=device)
        keep[f] = t
        setattr(st, f, t.data_ptr())
    st.my_counts = mine.counts.data_ptr()
    st.my_flags = mine.flags.data_ptr()
    st.done = mine.done.data_ptr()
    return st, keep


class EmulatedGroup:
    """G GPUs' windows on one device: every 'GPU' is the same process, so its
    peers' windows are plain local buffers.  For tests of the partitioning on
    one GPU: each member's calls run one after another in stream order, so no
    kernel waits on work that has not been issued before it."""

    def __init__(self, cfg, world, device, grad=False, weights=False, window_rows=0):
        self.cfg, self.world = cfg, world
        self.wins = [Windows(cfg, ep.make_group(world, g, 1, window_rows), device, grad, weights)
                     for g in range(world)]
        ptrs = [w.pointers() for w in self.wins]
        tables = {f: [p[f] for p in ptrs] for f in Windows.FIELDS}
        self.peers, self._keep = [], []
        for g in range(world):
            st, keep = peer_struct(tables, self.wins[g], device)
            self.peers.append(st)
            self._keep.append(keep)


def _world(pg):
    """(size, rank) of the process group; one GPU alone without one."""
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return 1, 0
    return dist.get_world_size(pg), dist.get_rank(pg)


def _exchange(obj, pg, what):
    """all_gather_object over the process group; a peer that does not take part
    before the group's timeout turns into EP_ERR_TIMEOUT."""
    import torch.distributed as dist
    if _world(pg)[0] == 1:
        return [obj]
    out = [None] * dist.get_world_size(pg)
    try:
        dist.all_gather_object(out, obj, group=pg)
    except RuntimeError as ex:  # gloo / NCCL raise on a timed-out collective
        raise ep.EpError(6, f"{what}: a peer did not take part ({str(ex).splitlines()[0][:120]})")
    return out


class EpGroup:
    """This process's member of a G-GPU group (G = the process group's size):
    its windows, the other GPUs' windows mapped through CUDA IPC, and one
    step of the path as the sequence of libep calls on `stream`."""

    def __init__(self, cfg, pg=None, device=None, grad=False, weights=False, stream=None,
                 timeout_ns=0, window_rows=0):
        self.cfg = cfg
        G, g = _world(pg)
        self.world, self.rank = G, g
        self.grp = ep.make_group(G, g, 1, window_rows)
        self.device = device or torch.device("cuda", torch.cuda.current_device())
        self.stream = stream or torch.cuda.current_stream(self.device)
        self.timeout_ns = timeout_ns
        self.win = Windows(cfg, self.grp, self.device, grad, weights)
        mine = {}
        for f, p in self.win.pointers().items():
            mine[f] = ep.ep_ipc_export(getattr(self.win, f)) if p else None
        torch.cuda.synchronize(self.device)
        allh = _exchange(mine, pg, "window handles")
        self._mapped = []
        bases = {}  # one mapping per peer allocation (windows may share one)
        tables = {f: [0] * G for f in Windows.FIELDS}
        for p in range(G):
            for f in Windows.FIELDS:
                if p == g:
                    tables[f][p] = self.win.pointers()[f]
                elif allh[p][f] is not None:
                    h, off = allh[p][f]
                    if (p, h) not in bases:
                        bases[(p, h)] = ep.ep_ipc_import(h, 0)
                        self._mapped.append(bases[(p, h)])
                    tables[f][p] = bases[(p, h)] + off
        self.peers, self._keep = peer_struct(tables, self.win, self.device)
        n_loc = (cfg.num_ranks // G) * cfg.num_tokens
        K, E = cfg.num_topk, cfg.num_experts
        dev = self.device
        self.token_slot = torch.empty((n_loc, K), dtype=torch.int32, device=dev)
        self.recv_count = torch.empty(E, dtype=torch.int64, device=dev)
        self.expert_offset = torch.empty(E + 1, dtype=torch.int64, device=dev) \
            if cfg.layout == ep.LAYOUT["packed"] else None
        self.workspace = torch.empty(self.win.sizes["workspace_bytes"], dtype=torch.uint8,
                                     device=dev)
        self.slot_scratch = torch.empty(E, dtype=torch.int64, device=dev)
        self.dev_status = torch.zeros(1, dtype=torch.int32, device=dev)
        _exchange(True, pg, "set-up")  # every peer has mapped every window

    def close(self):
        torch.cuda.synchronize(self.device)
        for base in self._mapped:
            ep.ep_ipc_close(base)
        self._mapped = []

    # ---- one step ----------------------------------------------------------------
    def dispatch(self, x, topk_idx, topk_weights=None):
        """Layout, counts to every GPU, plan, rows to the owners' windows, and
        the wait for every GPU's rows.  The experts then read this GPU's recv
        window (its expert_offset rows) and write its y window."""
        c, g, s, pe = self.cfg, self.grp, self.stream, self.peers
        ep.ep_group_layout(c, g, pe, topk_idx, self.token_slot, self.workspace, self.dev_status,
                           stream=s)
        ep.ep_group_plan(c, g, pe, topk_idx, self.token_slot, self.recv_count, self.expert_offset,
                         self.slot_scratch, self.dev_status, stream=s)
        ep.ep_group_dispatch(c, g, pe, x, topk_idx, self.token_slot, self.dev_status,
                             topk_weights=topk_weights, expert_offset=self.expert_offset,
                             stream=s)
        ep.ep_group_wait(g, pe, ep.GROUP_KIND_DISPATCH, self.dev_status, self.timeout_ns, stream=s)

    def combine(self, topk_idx, topk_weights, out):
        """After this GPU's experts have written its y window: the signal and the
        wait for every GPU's outputs, the combine from the owners' windows, and
        the end-of-step barrier (the windows may be reused)."""
        c, g, s, pe = self.cfg, self.grp, self.stream, self.peers
        ep.ep_group_signal(g, pe, ep.GROUP_KIND_EXPERT_OUT, stream=s)
        ep.ep_group_wait(g, pe, ep.GROUP_KIND_EXPERT_OUT, self.dev_status, self.timeout_ns,
                         stream=s)
        ep.ep_group_combine(c, g, pe, topk_idx, topk_weights, self.token_slot, out,
                            self.dev_status, expert_offset=self.expert_offset, stream=s)
        ep.ep_group_signal(g, pe, ep.GROUP_KIND_COMBINED, stream=s)
        ep.ep_group_wait(g, pe, ep.GROUP_KIND_COMBINED, self.dev_status, self.timeout_ns,
                         stream=s)
        self.grp.epoch += 1

    def status(self):
        """Device status bits since the last call (EP_ERR_TIMEOUT shows as DEV_TIMEOUT)."""
        return ep.ep_get_status(self.dev_status, self.stream)


def init_timeout(seconds):
    return datetime.timedelta(seconds=seconds)


__all__ = ["Windows", "EmulatedGroup", "EpGroup", "peer_struct", "init_timeout"]
