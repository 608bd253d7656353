"""Expert parallelism over several GPUs, the host side, on the CPU: two gloo
ranks split one R-rank problem (each holds R/2 ranks' tokens and owns E/2
experts), rank their own entries (the oracle's layout of their tokens),
exchange their per-rank counts over gloo, take libep's plan of the group
(ep_group_plan_host: the same arithmetic the plan kernel runs) and send each
entry's quantised row to the window of the rank that owns its expert.  Each
rank's window must equal, row for row, what the single-process oracle puts in
the rows of those experts; the global slots must equal the single-process
ones.  Also: the group's set-up gives EP_ERR_TIMEOUT when a peer never takes
part."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = [("bf16", "padded", 1), ("mxfp8", "packed", 1), ("mxfp8", "packed", 4),
         ("int8_token", "padded", 1), ("e4m3_b128", "packed", 2)]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _shape(mode):
    import synth
    H = 256 if mode == "e4m3_b128" else 64
    return synth.workload("tiny", R=4, T=7, M=8, K=3, E=8, H=H)


def _rank_main(rank, world, port, mode, layout, align, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import combine_ep_dispatch_04_b200 as ep
    import oracle
    import synth

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    w = _shape(mode)
    R, T, M, K, E, H = w["R"], w["T"], w["M"], w["K"], w["E"], w["H"]
    idx, _ = synth.make_routing(w)
    idx[3, 1] = -1
    x = synth.make_x(w)
    cfg = ep.make_config(R, T, M, K, E, H, mode, layout, align)
    grp = ep.make_group(world, rank)
    RG, EG = R // world, E // world
    mine = slice(rank * RG * T, (rank + 1) * RG * T)
    # this rank's entries ranked within their experts, and its per-rank counts
    loc = oracle.layout(RG, T, K, E, M, idx[mine], layout="packed")
    counts = torch.from_numpy(loc["tokens_per_expert"].astype(np.int32))
    gathered = [torch.empty_like(counts) for _ in range(world)]
    dist.all_gather(gathered, counts)
    tpe_all = torch.cat(gathered).numpy()
    base, total, eo_v = ep.ep_group_plan_host(cfg, grp, tpe_all)
    win = ep.ep_group_sizes(cfg, grp)
    rows, cap = win["rows"], R * M
    # global slots and the owner's window row of every entry
    gslot = np.where(loc["token_slot"] >= 0,
                     loc["token_slot"] + base[np.maximum(idx[mine], 0)], -1)
    msgs = []
    for n in range(RG * T):
        xr = oracle.quant_row(mode, x[mine][n])
        for k in range(K):
            e = int(idx[mine][n, k])
            if e < 0:
                continue
            s = int(gslot[n, k])
            vrow = e * cap + s if layout == "padded" else int(eo_v[e]) + s
            owner, wrow = divmod(vrow, rows)
            r_glob, t = (rank * RG * T + n) // T, (rank * RG * T + n) % T
            msgs.append((owner, wrow, xr[0].tobytes(), xr[1].tobytes(), r_glob * M + t))
    everyone = [None] * world
    dist.all_gather_object(everyone, msgs)
    got = {}
    for m in everyone:
        for owner, wrow, d, sc, src in m:
            if owner == rank:
                assert wrow not in got
                got[wrow] = (d, sc, src)
    q.put((rank, got, gslot, total, eo_v, rows))
    dist.destroy_process_group()


@pytest.mark.parametrize("mode,layout,align", CASES)
def test_two_ranks_reassemble_the_single_gpu_dispatch(mode, layout, align):
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, mode, layout, align, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in procs:
        r = q.get(timeout=300)
        res[r[0]] = r[1:]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = _shape(mode)
    R, T, M, K, E, H = w["R"], w["T"], w["M"], w["K"], w["E"], w["H"]
    idx, _ = synth.make_routing(w)
    idx[3, 1] = -1
    x = synth.make_x(w)
    lay = oracle.layout(R, T, K, E, M, idx, layout=layout, align=align)
    ref = oracle.dispatch(R, T, K, E, M, H, mode, x, idx, lay["token_slot"], lay["expert_offset"],
                          layout=layout, align=align)
    EG, RG, cap = E // world, R // world, R * M
    for g in range(world):
        got, gslot, total, eo_v, rows = res[g]
        # global slots, totals
        assert np.array_equal(gslot, lay["token_slot"][g * RG * T:(g + 1) * RG * T])
        assert np.array_equal(total, lay["recv_count"])
        # every row of this rank's experts, as the single process holds it
        want_rows = 0
        for e in range(g * EG, (g + 1) * EG):
            for s in range(int(lay["recv_count"][e])):
                single = e * cap + s if layout == "padded" else int(lay["expert_offset"][e]) + s
                wrow = (e - g * EG) * cap + s if layout == "padded" else int(eo_v[e]) - g * rows + s
                d, sc, src = got[wrow]
                assert d == ref["recv_data"][single].tobytes(), (g, e, s)
                assert sc == ref["recv_scale"][single].tobytes(), (g, e, s)
                assert src == ref["src_info"][single], (g, e, s)
                want_rows += 1
        assert len(got) == want_rows
        if layout == "packed":   # each owner's experts start at its window, aligned
            assert eo_v[g * EG] == g * rows
            assert all(eo_v[e] % align == 0 for e in range(g * EG, (g + 1) * EG))


def test_plan_host_against_its_definition():
    """ep_group_plan_host on random counts: shifts are the counts of the ranks
    before this GPU's, totals the column sums, offsets the owner-relative
    running sums of the rounded totals (written out here with numpy)."""
    sys.path.insert(0, ROOT)
    import combine_ep_dispatch_04_b200 as ep
    r = np.random.default_rng(3)
    for (R, E, G, align, layout) in [(4, 8, 2, 1, "packed"), (8, 16, 4, 3, "packed"),
                                     (4, 8, 1, 1, "padded"), (6, 12, 3, 8, "packed")]:
        T, K = 4, 2
        cfg = ep.make_config(R, T, 8, K, E, 64, "bf16", layout, align)
        idx = r.integers(-1, E, (R, T * K))          # any routing, duplicates and -1 included
        tpe = np.stack([np.bincount(row[row >= 0], minlength=E) for row in idx]).astype(np.int32)
        for g in range(G):
            grp = ep.make_group(G, g)
            base, total, eo = ep.ep_group_plan_host(cfg, grp, tpe)
            rows = ep.ep_group_sizes(cfg, grp)["rows"]
            assert np.array_equal(total, tpe.sum(axis=0))
            assert np.array_equal(base, tpe[: g * (R // G)].sum(axis=0))
            if layout == "packed":
                EG = E // G
                rnd = (total + align - 1) // align * align
                for o in range(G):
                    seg = rnd[o * EG:(o + 1) * EG]
                    want = o * rows + np.concatenate([[0], np.cumsum(seg)[:-1]])
                    assert np.array_equal(eo[o * EG:(o + 1) * EG], want)
                    assert seg.sum() <= rows          # every owner's rows fit its window
                assert eo[E] == G * rows


def _withholding_rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import time

    import torch.distributed as dist

    import combine_ep_dispatch_04_b200 as ep
    from combine_ep_dispatch_04_b200 import group as grp_mod

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=3))
    if rank == 1:          # never takes part in the exchange; leaves after the others gave up
        time.sleep(8)
        q.put((rank, None))
        return
    try:
        grp_mod._exchange({"counts": [1, 2, 3]}, None, "counts")
        q.put((rank, "no error"))
    except ep.EpError as ex:
        q.put((rank, ex.status))


def test_a_peer_that_withholds_its_part_gives_a_timeout():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_withholding_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert res[0] == 6          # EP_ERR_TIMEOUT
