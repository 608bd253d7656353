#!/usr/bin/env python
"""Benchmark of MoE expert-parallel dispatch + combine on B200.

One step = the whole hot path over one batch: routing layout, quantise +
scatter (dispatch), weighted combine (and combine-backward for the prefill
workload).  Default workload (the headline): prefill, the largest of the five
named workloads that fits one GPU (R=32 logical ranks x T=4096 tokens,
H=7168, top-8 of 256 experts, MXFP8 dispatch into the packed receive layout,
weighted combine and the MXFP8 combine-backward), on one GPU.  After the
headline, every other named workload (tiny in both of its modes, decode,
skewed, large) is run through the same per-kernel protocol and reported in
the line's "workloads" object, with the combine of quantised expert outputs
of every quantised mode.

Timing: CUDA events on the stream the kernels run on.  The timed region
brackets each step with one event pair (the reported value); a second pass
times every kernel alone, between its own event pair, after its own L2 flush,
for the per-kernel durations behind the roofline figures (a kernel that
follows the dispatch in the same step would otherwise also pay the write-back
of the dispatch's dirty L2 lines, which the step-level value already counts).
A third pass, for workloads that move under 1 GiB a step, launches each
kernel 4 times back to back on 4 distinct copies of its buffers between one
pair of events: the per-launch time with the launch overhead amortised as in
the step (an isolated launch carries ~6 us of launch and drain that the
dependent launches of a step overlap); the roofline reports it, with the
isolated figure beside it.
Between steps, outside the step's events, L2 is flushed by writing one
512 MiB buffer and then reading another: the read evicts the write's dirty
lines, so every step starts from a cold L2 holding only clean lines (a
write-only flush would leave ~126 MB of dirty lines whose write-back the next
step's kernels would pay for).
The K timed steps are bracketed by a barrier and a synchronize on both sides;
the reported time is the max over ranks.  With --gpus N > 1 (torchrun), each
rank runs an independent replica of the workload (different seed): the path
has no exchange step on one GPU, so no collective is added ("weak" scaling).

  python bench.py [--steps K] [--warmup W] [--workload prefill] [--impl reference]
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "dispatch+combine tokens/s and achieved HBM GB/s (% of B200 peak), 1 GPU"
FALLBACK_HBM_GBS = 6650.0
WORKLOAD_MODE = {"tiny": "int8_token", "decode": "e4m3_b128", "skewed": "int8_token",
                 "prefill": "mxfp8", "large": "mxfp4", "a5": "mxfp8"}
KERNEL_SOURCES = ["combine_ep_dispatch_04_b200/csrc/" + f for f in
                  ("ep_api.cu", "ep_device.cuh", "ep_layout.cuh", "ep_dispatch.cuh", "ep_combine.cuh",
                   "ep_group.cuh")]


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=300)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--workload", default="prefill", choices=sorted(synth.WORKLOADS))
    p.add_argument("--tokens-per-rank", type=int, default=None,
                   help="override T (profiling a reduced case; the reported workload says so)")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--flush-mib", type=int, default=512)
    p.add_argument("--cpu-seconds", type=float, default=10.0)
    p.add_argument("--quantized-combine", action="store_true",
                   help="combine reads expert outputs stored in the dispatch format")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--only", choices=["ffn"], default=None,
                   help="run one leg alone and print its object (profiler captures)")
    p.add_argument("--ep-group", action="store_true",
                   help="run the expert-parallel group path also on one GPU (a group of one)")
    p.add_argument("--replicas", action="store_true",
                   help="with --gpus N > 1: N independent single-GPU replicas instead of one "
                        "expert-parallel job over the N GPUs")
    p.add_argument("--no-workloads", action="store_true",
                   help="skip the per-kernel pass over the other named workloads")
    p.add_argument("--gemm-workload", default="decode", choices=sorted(synth.WORKLOADS),
                   help="the workload whose routing the GEMM legs use")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--weights-grad", action="store_true",
                   help="also time the combine's weight gradient (outside the step)")
    p.add_argument("--gemm", action="store_true",
                   help="time the experts' grouped GEMMs (bf16, MXFP8, MXFP4; packed, N = H) and "
                        "the one-call forward path outside the step, also when N > 1 (one GPU: "
                        "the default)")
    p.add_argument("--no-gemm", action="store_true",
                   help="skip the experts' GEMM legs on one GPU")
    p.add_argument("--gemm-experts", type=int, default=0,
                   help="with --gemm: route the tokens onto this many experts (expert id "
                        "modulo E) for the GEMM legs only, a small case for profilers")
    p.add_argument("--no-steady", action="store_true",
                   help="skip the steady-state pass and its buffer copies (profiling runs)")
    p.add_argument("--no-copy", action="store_true",
                   help="skip the same-run copy-bandwidth measurement (profiling runs)")
    return p.parse_args()


# ---------------------------------------------------------------------------
# algorithmic bytes (what the method must move; unwritten capacity not counted)
# ---------------------------------------------------------------------------
def algorithmic_bytes(w, mode, idx, quantized_combine=False, weights_grad=False):
    """Bytes per launch of each kernel, from the per-token counts."""
    import oracle

    N, K, H, R = w["N"], w["K"], w["H"], w["R"]
    D, S = oracle.row_bytes(mode, H)
    v = int(((idx >= 0) & (idx < w["E"])).sum())
    y_row = (D + S) if quantized_combine else 2 * H
    out = {
        "layout": N * (8 * K + 4 * K + R),
        "dispatch": N * (2 * H + 8 * K + 4 * K) + v * (D + S + 4),
        "combine": v * y_row + N * (8 * K + 4 * K + 4 * K + 2 * H),
    }
    if mode != "bf16":  # the combine of expert outputs stored in the dispatch format
        out["combine_q"] = v * (D + S) + N * (8 * K + 4 * K + 4 * K + 2 * H)
    if w.get("backward"):
        out["combine_bwd"] = N * (2 * H + 4 * K + 4 * K + 8 * K) + v * (H + H // 32)
    if weights_grad:  # g, idx, slots, dw; one expert row per valid entry
        out["combine_bwd_w"] = N * (2 * H + 8 * K + 4 * K + 4 * K) + v * 2 * H
    return out, v


def source_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except (OSError, ValueError):
        return None


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dispatch_combine_traffic.json")


def ncu_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    e = t.get(workload, {}).get(kernel)
    if not e or e.get("source_hash") != source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ---------------------------------------------------------------------------
REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index):
        self.samples, self.reasons, self.ok = [], 0, False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            h = None
            uuid = getattr(props, "uuid", None)
            if uuid is not None:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(uuid))
                except Exception:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv, self.h = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as exc:  # no NVML: report what is known
            self.err = str(exc)

    def _run(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(0.005)

    def sample(self):
        try:
            mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
            r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            self.samples.append(mhz)
            self.reasons |= int(r)
        except Exception:
            pass

    def __enter__(self):
        if self.ok:
            self.sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()
            self.sample()

    def report(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for b, n in REASONS.items() if self.reasons & b and b != 0x1]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas; no data-path collective)
# ---------------------------------------------------------------------------
def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value, world):
    """Max of a float over ranks (the timed duration)."""
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_done(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# the oracle as the CPU baseline / reference arm
# ---------------------------------------------------------------------------
SAMPLE_TOKENS = 1024  # tokens of one oracle step (a bounded sample of the workload)


def sample_tokens_per_rank(w):
    """Tokens per source rank in the oracle's sample: about SAMPLE_TOKENS in all."""
    return max(1, min(w["T"], SAMPLE_TOKENS // w["R"]))


class OracleStep:
    """The oracle (plain single-threaded C) running one step of the workload --
    layout, dispatch and combine -- on a bounded sample: the first `sub_t`
    tokens of every source rank (same ranks, experts, capacity and hidden
    size).  Inputs and output arrays are built before timing; only rows that
    hold entries are ever touched."""

    def __init__(self, w, mode, sub_t, replica=0):
        import oracle
        self.o, self.mode = oracle, mode
        R, T, M, K, E, H = w["R"], w["T"], w["M"], w["K"], w["E"], w["H"]
        sub_t = max(1, min(sub_t, T))
        take = (np.arange(R)[:, None] * T + np.arange(sub_t)[None, :]).reshape(-1)
        idx, wts = synth.make_routing(w, replica)
        self.w = synth.workload(w["name"], T=sub_t)
        self.idx, self.wts = idx[take], wts[take]
        self.x = synth.make_x(w, replica, rows=take)
        self.n = take.size
        lay = oracle.layout(R, sub_t, K, E, M, self.idx, layout=w["layout"])
        rows = oracle.rows_max(R, sub_t, K, E, M, w["layout"])
        self.bufs = oracle.dispatch_buffers(R, sub_t, K, E, M, H, mode, w["layout"], fill=False)
        self.y = np.zeros((rows, H), np.uint16)   # pages of rows never read stay unmapped
        pool, off = synth.y_source(w, rows, replica)
        used = (self.idx >= 0) & (self.idx < E)
        r_used = oracle.row_index(w["layout"], R, M, self.idx[used], lay["token_slot"][used],
                                  lay["expert_offset"])
        for r in np.asarray(r_used).tolist():
            self.y[r] = pool[off[r]: off[r] + H]
        self.out = np.empty((self.n, H), np.uint16)
        self.sample = (f"first {sub_t} of {T} tokens of each of the {R} ranks "
                       f"({self.n} tokens): layout, dispatch and combine per step")

    def step(self):
        o, w = self.o, self.w
        R, T, M, K, E, H = w["R"], w["T"], w["M"], w["K"], w["E"], w["H"]
        lay = o.layout(R, T, K, E, M, self.idx, layout=w["layout"])
        o.dispatch(R, T, K, E, M, H, self.mode, self.x, self.idx, lay["token_slot"],
                   lay["expert_offset"], layout=w["layout"], out=self.bufs)
        o.combine(R, T, K, E, M, H, self.y, self.idx, self.wts, lay["token_slot"],
                  lay["expert_offset"], layout=w["layout"], out=self.out)
        return self.n


def cpu_baseline(w, mode, seconds, replica=0):
    st = OracleStep(w, mode, sample_tokens_per_rank(w), replica=replica)
    st.step()
    t0 = time.perf_counter()
    done, reps = 0, 0
    while True:
        done += st.step()
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return {"value": done / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{st.sample}; {reps} steps in {el:.1f} s, single thread"}


def _oracle_worker(job, barrier, results):
    """One independent oracle instance (a spawned process): the seeded inputs
    of its sample rebuilt here and one warm-up step, then, after every instance
    has reached the barrier, steps for `seconds`."""
    wname, t_override, mode, replica, sub_t, seconds = job
    w = synth.workload(wname) if t_override is None else synth.workload(wname, T=t_override)
    st = OracleStep(w, mode, sub_t, replica=replica)
    st.step()
    barrier.wait(timeout=600)
    t0 = time.perf_counter()
    done = 0
    while True:
        done += st.step()
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    results.put((done, el))


def cpu_baseline_all_cores(wname, t_override, mode, seconds, replica=0):
    """The oracle on the host's cores (up to 32): as many independent instances as
    cores (spawned processes, each on the same bounded sample), released
    together by a barrier and timed over the same interval; tokens/s summed."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    cores = min(os.cpu_count() or 1, 32)  # each instance is a process with its own imports
    w = synth.workload(wname) if t_override is None else synth.workload(wname, T=t_override)
    sub_t = sample_tokens_per_rank(w)
    barrier, results = ctx.Barrier(cores), ctx.Queue()
    job = (wname, t_override, mode, replica, sub_t, seconds)
    procs = [ctx.Process(target=_oracle_worker, args=(job, barrier, results)) for _ in range(cores)]
    for pr in procs:
        pr.start()
    res = [results.get(timeout=900) for _ in procs]
    for pr in procs:
        pr.join(timeout=60)
    total = sum(d for d, _ in res)
    el = max(e for _, e in res)
    return {"value": total / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{cores} independent instances, each the first {sub_t} of {w['T']} tokens "
                      f"of each of the {w['R']} ranks, started together; {seconds:.0f} s, summed"}


# ---------------------------------------------------------------------------
# one workload on the device: inputs, buffers and the bound C-ABI calls
# ---------------------------------------------------------------------------
class WorkloadRun:
    """Device inputs, caller-owned buffers and bound C-ABI calls of one
    workload.  Kernels (each a bound call, timed separately):
      layout, dispatch, combine     the step (layout + dispatch run as the
                                    one-call dispatch inside a step)
      combine_bwd                   the step, for workloads with a backward
      combine_q                     the combine of expert outputs stored in
                                    the dispatch's quantised format (outside
                                    the step), quantised modes only
      combine_bwd_w                 the weight gradient (outside the step,
                                    with --weights-grad)"""

    def __init__(self, ep, wname, args, dev, stream, replica, mode=None, t_override=None,
                 with_q=True, quantized_step=False, weights_grad=False):
        w = synth.workload(wname) if t_override is None else synth.workload(wname, T=t_override)
        self.ep, self.w, self.dev, self.stream = ep, w, dev, stream
        self.mode = mode or WORKLOAD_MODE[wname]
        R, T, M, K, E, H = w["R"], w["T"], w["M"], w["K"], w["E"], w["H"]
        self.idx, self.wts = synth.make_routing(w, replica)
        self.x = synth.make_x(w, replica)
        self.cfg = cfg = ep.make_config(R, T, M, K, E, H, self.mode, w["layout"])
        self.b = b = ep.Buffers(cfg, device=dev, grad=bool(w.get("backward")))
        self.idx_d = torch.from_numpy(self.idx).to(dev)
        self.wts_d = torch.from_numpy(self.wts).to(dev)
        self.x_d = torch.from_numpy(self.x.view(np.int16)).to(dev).view(torch.bfloat16)
        ypool, yoff = synth.y_source(w, b.sizes["rows"], replica)
        pool_d = torch.from_numpy(ypool.view(np.int16)).to(dev)
        torch.index_select(pool_d.as_strided((synth.POOL, H), (1, 1)), 0,
                           torch.from_numpy(yoff).to(dev), out=b.y.view(torch.int16))
        del pool_d
        quantized = self.mode != "bf16"
        self.qcfg = ep.make_config(R, T, M, K, E, H, self.mode, w["layout"],
                                   flags=ep.F_COMBINE_QUANTIZED) if quantized else None
        self.y_q = None
        if quantized and (with_q or quantized_step):
            # expert outputs in the dispatch format: the dispatched rows of one
            # pass, copied to their own buffer (cold after every L2 flush)
            ep.ep_dispatch_with_layout(cfg, self.x_d, self.idx_d, b.token_slot, b.recv_count,
                                       b.workspace, b.recv_buf, b.src_info, b.dev_status,
                                       expert_offset=b.expert_offset, stream=stream)
            self.y_q = b.recv_buf.clone()
        self.g_d = None
        if w.get("backward"):
            gp, go = synth.g_source(w, replica)
            self.g_d = torch.from_numpy(synth.windows(gp, go, H).view(np.int16)).to(dev) \
                .view(torch.bfloat16)
        self.gw_d = self.dw_d = None
        if weights_grad:
            gp, go = synth.g_source(w, replica)
            self.gw_d = torch.from_numpy(synth.windows(gp, go, H).view(np.int16)).to(dev) \
                .view(torch.bfloat16)
            self.dw_d = torch.empty((w["N"], K), dtype=torch.float32, device=dev)
        eo = b.expert_offset
        self.step_ccfg, self.step_y = (self.qcfg, self.y_q) if quantized_step and quantized \
            else (cfg, b.y)
        self.kernels = ["layout", "dispatch", "combine"]
        if self.g_d is not None:
            self.kernels.append("combine_bwd")
        if quantized and with_q:
            self.kernels.append("combine_q")
        if weights_grad:
            self.kernels.append("combine_bwd_w")
        self.calls = {k: self.bound(k, 0) for k in self.kernels}
        self.step_calls = [
            ep.ep_dispatch_with_layout(cfg, self.x_d, self.idx_d, b.token_slot, b.recv_count,
                                       b.workspace, b.recv_buf, b.src_info, b.dev_status,
                                       expert_offset=eo, stream=stream, bind=True),
            ep.ep_combine(self.step_ccfg, self.step_y, self.idx_d, self.wts_d, b.token_slot,
                          b.out, b.dev_status, expert_offset=eo, stream=stream, bind=True),
        ]
        if self.g_d is not None:
            self.step_calls.append(self.calls["combine_bwd"])
        self.keep = []

    def name(self):
        w = self.w
        return (f"{w['name']}: R={w['R']} T={w['T']} H={w['H']} K={w['K']} E={w['E']} "
                f"M={w['M']} {self.mode} {w['layout']}")

    def bound(self, k, copy):
        """The bound call of kernel k; copy > 0 gives it its own copies of the
        data-path buffers it reads and writes (for back-to-back launches whose
        data is all cold)."""
        ep, b, eo, s = self.ep, self.b, self.b.expert_offset, self.stream
        cfg = self.cfg

        def fresh(t, clone):
            if not copy:
                return t
            u = t.clone() if clone else torch.empty_like(t)
            self.keep.append(u)
            return u
        if k == "layout":
            return ep.ep_dispatch_layout(cfg, self.idx_d, b.token_slot, b.recv_count, b.workspace,
                                         b.dev_status, expert_offset=eo, stream=s, bind=True)
        if k == "dispatch":
            return ep.ep_dispatch(cfg, fresh(self.x_d, True), self.idx_d, b.token_slot,
                                  fresh(b.recv_buf, False), fresh(b.src_info, False), b.dev_status,
                                  expert_offset=eo, stream=s, bind=True)
        if k == "combine":
            return ep.ep_combine(cfg, fresh(b.y, True), self.idx_d, self.wts_d, b.token_slot,
                                 fresh(b.out, False), b.dev_status, expert_offset=eo, stream=s,
                                 bind=True)
        if k == "combine_q":
            return ep.ep_combine(self.qcfg, fresh(self.y_q, True), self.idx_d, self.wts_d,
                                 b.token_slot, fresh(b.out, False), b.dev_status,
                                 expert_offset=eo, stream=s, bind=True)
        if k == "combine_bwd":
            return ep.ep_combine_backward(cfg, fresh(self.g_d, True), self.idx_d, self.wts_d,
                                          b.token_slot, fresh(b.grad_buf, False), b.dev_status,
                                          expert_offset=eo, stream=s, bind=True)
        if k == "combine_bwd_w":
            return ep.ep_combine_backward_weights(cfg, fresh(self.gw_d, True), fresh(b.y, True),
                                                  self.idx_d, b.token_slot, fresh(self.dw_d, False),
                                                  b.dev_status, expert_offset=eo, stream=s,
                                                  bind=True)
        raise KeyError(k)

    def step(self):
        for c in self.step_calls:
            c()

    def release(self):
        self.keep.clear()
        self.calls.clear()
        self.step_calls = []
        for a in ("b", "x_d", "idx_d", "wts_d", "y_q", "g_d", "gw_d", "dw_d"):
            setattr(self, a, None)
        torch.cuda.empty_cache()


def run_group_bench(ep, args, wname, world, rank, local, dev):
    """One expert-parallel job over the N GPUs (weak scaling): every GPU holds
    the named workload's R ranks of T tokens (the job has R * N ranks and the
    workload's E experts, E / N on each GPU), its tokens drawn with its own
    replica of the routing and activations.  A step is the library's group
    path: layout with the counts exchange, plan, dispatch into the owners'
    windows over NVLink, (the expert outputs stand in the windows), combine
    from the owners' windows, and the combine-backward for the prefill
    workload; every transfer and wait is in the library's kernels.  Timed with
    CUDA events on the stream, L2 flushed before each step, max over ranks."""
    import torch.distributed as dist

    from combine_ep_dispatch_04_b200.group import EpGroup
    w1 = synth.workload(wname) if args.tokens_per_rank is None else \
        synth.workload(wname, T=args.tokens_per_rank)
    mode = WORKLOAD_MODE[wname]
    R1, T, M, K, E, H = w1["R"], w1["T"], w1["M"], w1["K"], w1["E"], w1["H"]
    R = R1 * world
    if E % R:
        raise SystemExit(f"{wname}: {E} experts cannot be split over {R} ranks")
    cfg = ep.make_config(R, T, M, K, E, H, mode, w1["layout"])
    n_loc = R1 * T
    stream = torch.cuda.current_stream(dev)
    idx, wts = synth.make_routing(w1, rank)
    x = synth.make_x(w1, rank)
    idx_d, wts_d = torch.from_numpy(idx).to(dev), torch.from_numpy(wts).to(dev)
    x_d = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    backward = bool(w1.get("backward"))
    g_d = None
    if backward:
        gp, go = synth.g_source(w1, rank)
        g_d = torch.from_numpy(synth.windows(gp, go, H).view(np.int16)).to(dev).view(torch.bfloat16)
    # packed windows for the expected load (each owner receives about n_loc * K
    # rows under uniform routing) with room to spare; padded: fixed by R * M
    slack = 2.0 if w1["routing"] == "zipf" else 1.5
    win = int(slack * n_loc * K) + (E // world) * 8 if w1["layout"] == "packed" else 0
    eg = EpGroup(cfg, device=dev, grad=backward, stream=stream, timeout_ns=5_000_000_000,
                 window_rows=win)
    ypool, yoff = synth.y_source(w1, eg.win.sizes["rows"], rank)
    pool_d = torch.from_numpy(ypool.view(np.int16)).to(dev)
    torch.index_select(pool_d.as_strided((synth.POOL, H), (1, 1)), 0,
                       torch.from_numpy(yoff).to(dev), out=eg.win.y.view(torch.int16))
    del pool_d
    out = torch.empty((n_loc, H), dtype=torch.bfloat16, device=dev)
    flush_w = torch.empty(args.flush_mib << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(args.flush_mib << 20, dtype=torch.uint8, device=dev)

    def step():
        eg.dispatch(x_d, idx_d, wts_d)
        eg.combine(idx_d, wts_d, out)
        if backward:
            ep.ep_group_combine_backward(cfg, eg.grp, eg.peers, g_d, idx_d, wts_d, eg.token_slot,
                                         eg.dev_status, expert_offset=eg.expert_offset,
                                         stream=stream)
            ep.ep_group_wait(eg.grp, eg.peers, ep.GROUP_KIND_BACKWARD, eg.dev_status,
                             eg.timeout_ns, stream=stream)

    for _ in range(max(args.warmup, 3)):
        flush_w.fill_(1)
        flush_r.max()
        step()
    torch.cuda.synchronize(dev)
    if eg.status() != 0:
        raise SystemExit("device status reported errors during warm-up (timeout or capacity)")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize(dev)
    launches0 = ep.ep_kernel_launches()
    with clocks:
        for s_ in range(args.steps):
            flush_w.fill_(s_ & 0xFF)
            flush_r.max()
            evs[s_][0].record(stream)
            step()
            evs[s_][1].record(stream)
        torch.cuda.synchronize(dev)
    launches = ep.ep_kernel_launches() - launches0
    barrier(world)
    total_ms = max_over_ranks(sum(a.elapsed_time(c) for a, c in evs), world)
    bad = max_over_ranks(float(eg.status() != 0), world)
    eg.close()
    ms = total_ms / args.steps
    if rank == 0:
        out_line = {
            "metric": METRIC, "value": round(world * n_loc * args.steps / (total_ms / 1e3), 1),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"{wname}: {R1} ranks x T={T} a GPU ({R} ranks), H={H} K={K} "
                                   f"E={E} M={M} {mode} {w1['layout']}",
                       "tokens_per_step": world * n_loc,
                       "parallelism": f"ep{world}: expert parallel over NVLink peer memory",
                       "window_rows": eg.win.sizes["rows"],
                       "l2": "flushed before each step outside the events"},
            "clocks": clocks.report(), "gpu_launches": launches,
            "device_status_clean": bad == 0.0,
        }
        print(json.dumps(out_line), flush=True)
    dist_done(world)


def run_ffn_leg(ep, flush, stream, dev, args, replica):
    """The deep fused MoE page's benchmark case on one GPU ("[feat] A5 deep fused
    moe supported", Benchmarking: EP 8, hidden 7168, moe-intermediate-size 3072,
    top-6, 6 experts a rank, FP8, uniform routing; 128 tokens a rank): the
    experts' gated MLP alone (ep_expert_ffn_mx: GMM1 with SwiGLU and the
    requant in its epilogue, GMM2) and the whole forward path in one call
    (ep_moe_forward_ffn: layout + MXFP8 dispatch, the MLP, combine), each timed
    alone between events after an L2 flush.  Seeded random MXFP8 weights.
    FLOPs = 2 * entries * (H * 2I + I * H); the bytes that must move at least
    once are the codes and scales of every used expert's weights, the received
    rows, z (written and read) and y; the tensor peak is the measured bf16 peak
    times the nominal fp8 / bf16 ratio 2."""
    w = synth.workload("a5")
    R, T, M, K, E, H, I = w["R"], w["T"], w["M"], w["K"], w["E"], w["H"], w["inter"]
    idx, wts = synth.make_routing(w, replica)
    x = synth.make_x(w, replica)
    cfg = ep.make_config(R, T, M, K, E, H, "mxfp8", "packed")
    b = ep.Buffers(cfg, device=dev)
    x_d = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    idx_d, wts_d = torch.from_numpy(idx).to(dev), torch.from_numpy(wts).to(dev)
    gen = torch.Generator(device=dev).manual_seed(77)

    def mxw(n, k, lo, hi):
        c = torch.randint(0, 256, (E, n, k), device=dev, dtype=torch.int16,
                          generator=gen).to(torch.uint8)
        c[(c & 0x7F) == 0x7F] = 0
        sc = torch.randint(lo, hi, (E, n, k // 32), device=dev, dtype=torch.int16,
                           generator=gen).to(torch.uint8)
        return c, sc
    w1c, w1s = mxw(2 * I, H, 112, 116)
    w2c, w2s = mxw(H, I, 110, 114)
    zb, _ = ep.ep_ffn_buffer_bytes(cfg, I)
    z = torch.empty(zb, dtype=torch.uint8, device=dev)
    ep.ep_dispatch_with_layout(cfg, x_d, idx_d, b.token_slot, b.recv_count, b.workspace,
                               b.recv_buf, b.src_info, b.dev_status,
                               expert_offset=b.expert_offset, stream=stream)
    mlp = ep.ep_expert_ffn_mx(cfg, b.recv_buf, b.expert_offset, b.recv_count, w1c, w1s, w2c, w2s,
                              z, b.y, b.dev_status, stream=stream, bind=True)
    fwd = ep.ep_moe_forward_ffn(cfg, x_d, idx_d, wts_d, w1c, w1s, w2c, w2s, b.token_slot,
                                b.recv_count, b.expert_offset, b.workspace, b.recv_buf,
                                b.src_info, z, b.y, b.out, b.dev_status, stream=stream,
                                bind=True)

    def timed(call):
        for _ in range(3):
            flush(1)
            call()
        torch.cuda.synchronize(dev)
        if ep.ep_get_status(b.dev_status) != 0:
            raise RuntimeError("device status reported errors")
        reps = max(3, min(args.steps, 20))
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        for s_ in range(reps):
            flush(s_ & 0xFF)
            evs[s_][0].record(stream)
            call()
            evs[s_][1].record(stream)
        torch.cuda.synchronize(dev)
        return statistics.mean(a.elapsed_time(c) for a, c in evs)
    ms_mlp = timed(mlp)
    ms_fwd = timed(fwd)
    v = int(b.recv_count.sum().item())
    used = int((b.recv_count > 0).sum().item())
    flops = 2.0 * v * (H * 2 * I + I * H)
    wbytes = used * (2 * I * H + H * I) * (1 + 1 / 32)
    nbytes = wbytes + v * (H + H / 32) + 2 * v * (I + I / 32) + 2.0 * v * H
    peaks = measured_peaks() or {}
    peak = (peaks.get("bf16_tflops") or 1590.0) * 2.0
    hbm = peaks.get("hbm_gbs") or FALLBACK_HBM_GBS
    t_tensor, t_hbm = flops / (peak * 1e12), nbytes / (hbm * 1e9)
    del w1c, w1s, w2c, w2s, z, b
    torch.cuda.empty_cache()
    return {"workload": f"a5: R={R} T={T} H={H} K={K} E={E} M={M} mxfp8 packed, intermediate {I}",
            "mlp_ms": round(ms_mlp, 4), "forward_ms": round(ms_fwd, 4),
            "tokens_per_s": round(R * T / (ms_fwd * 1e-3), 1),
            "flops": flops, "bytes": nbytes, "tflops": round(flops / (ms_mlp * 1e-3) / 1e12, 1),
            "gbs": round(nbytes / (ms_mlp * 1e-3) / 1e9, 1),
            "bound": "tensor" if t_tensor >= t_hbm else "hbm", "peak_tflops": peak,
            "peak_gbs": hbm, "peak_source": ("measured bf16 x 2 (nominal fp8 / bf16)"
                                              if peaks.get("bf16_tflops") else "fallback bf16 x 2"),
            "frac": round(max(t_tensor, t_hbm) / (ms_mlp * 1e-3), 4),
            "launches": {"mlp": 2, "forward": 5},
            "what": "mlp: GMM1 + SwiGLU + requant, GMM2; forward: layout + dispatch, mlp, combine"}


STEADY_SETS = 4
STEADY_MAX_BYTES = 1 << 30


def isolated_launches(run, steps, flush):
    """Each kernel alone between its own pair of events, after its own L2 flush,
    `steps` times: {kernel: [ms]}."""
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in run.kernels] for _ in range(steps)]
    torch.cuda.synchronize(run.dev)
    for s in range(steps):
        for i, k in enumerate(run.kernels):
            flush(s & 0xFF)
            evs[s][i][0].record(run.stream)
            run.calls[k]()
            evs[s][i][1].record(run.stream)
    torch.cuda.synchronize(run.dev)
    return {k: [e[i][0].elapsed_time(e[i][1]) for e in evs] for i, k in enumerate(run.kernels)}


def steady_launches(run, steps, flush, step_bytes, skip=False):
    """Per-launch durations with the launch overhead amortised as in the step:
    each kernel is launched STEADY_SETS times back to back, on as many
    distinct copies of the buffers it reads and writes (each launch's data is
    cold: the group starts after an L2 flush and no two launches share a
    buffer of the data path), between one pair of events; the dependent
    launches overlap the tail of the previous grid, as the kernels of a step
    do.  Workloads that move more than STEADY_MAX_BYTES a step are not timed
    this way: there the launch overhead is already a negligible part of an
    isolated launch.  Returns ({kernel: [ms per launch]}, sets)."""
    if step_bytes > STEADY_MAX_BYTES or skip:
        return {}, 1
    sets = STEADY_SETS
    per_set = {k: [run.calls[k]] + [run.bound(k, j) for j in range(1, sets)] for k in run.kernels}
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in run.kernels] for _ in range(steps)]
    for s in range(steps):
        for i, k in enumerate(run.kernels):
            flush(s & 0xFF)
            evs[s][i][0].record(run.stream)
            for c in per_set[k]:
                c()
            evs[s][i][1].record(run.stream)
    torch.cuda.synchronize(run.dev)
    out = {k: [e[i][0].elapsed_time(e[i][1]) / sets for e in evs]
           for i, k in enumerate(run.kernels)}
    del per_set
    run.keep.clear()
    torch.cuda.empty_cache()
    return out, sets


def kernel_stats(run, per_kernel, steady, sets, alg, peak, peak_src):
    ks = {}
    for k in run.kernels:
        mean_ms = statistics.mean(per_kernel[k])
        gbs = alg[k] / (mean_ms * 1e-3) / 1e9
        ks[k] = {"us_mean": round(mean_ms * 1e3, 2),
                 "us_p10": round(float(np.percentile(per_kernel[k], 10)) * 1e3, 2),
                 "us_p90": round(float(np.percentile(per_kernel[k], 90)) * 1e3, 2),
                 "alg_bytes": alg[k], "gbs": round(gbs, 1),
                 "frac_of_" + peak_src: round(gbs / peak, 4)}
        if sets > 1:
            st_ms = statistics.mean(steady[k])
            ks[k].update({"us_steady": round(st_ms * 1e3, 2),
                          "gbs_steady": round(alg[k] / (st_ms * 1e-3) / 1e9, 1),
                          "frac_steady_of_" + peak_src:
                              round(alg[k] / (st_ms * 1e-3) / 1e9 / peak, 4)})
    return ks


def step_bytes_of(alg):
    """Algorithmic bytes of one step: the kernels of the step only."""
    return sum(v for k, v in alg.items() if k not in ("combine_bwd_w", "combine_q"))


def hbm_peak():
    peaks = measured_peaks()
    if peaks and peaks.get("hbm_gbs"):
        return peaks["hbm_gbs"], "measured"
    return FALLBACK_HBM_GBS, "fallback"


def timed_steps(run, steps, flush):
    """`steps` steps, one event pair each, L2 flushed before each outside the
    events: [ms per step]."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for s in range(steps):
        flush(s & 0xFF)
        evs[s][0].record(run.stream)
        run.step()
        evs[s][1].record(run.stream)
    torch.cuda.synchronize(run.dev)
    return [a.elapsed_time(c) for a, c in evs]


def other_workload(ep, wname, mode, args, dev, stream, flush, local):
    """One of the other named workloads at full size: warm-up, the step timed
    `steps` times, then the per-kernel passes; its own clock record."""
    run = WorkloadRun(ep, wname, args, dev, stream, replica=0, mode=mode)
    try:
        for _ in range(max(args.warmup, 3)):
            flush(1)
            run.step()
            for k in run.kernels:
                run.calls[k]()
        torch.cuda.synchronize(dev)
        if ep.ep_get_status(run.b.dev_status) != 0:
            raise RuntimeError("device status reported errors")
        alg, v = algorithmic_bytes(run.w, run.mode, run.idx)
        peak, peak_src = hbm_peak()
        clocks = ClockSampler(local)
        with clocks:
            step_ms = timed_steps(run, args.steps, flush)
            iso = isolated_launches(run, args.steps, flush)
            steady, sets = steady_launches(run, args.steps, flush, step_bytes_of(alg),
                                           skip=args.no_steady)
        ms = statistics.mean(step_ms)
        return {"workload": run.name(), "tokens_per_step": run.w["N"], "valid_entries": v,
                "step_us": round(ms * 1e3, 2),
                "tokens_per_s": round(run.w["N"] / (ms * 1e-3), 1),
                "step_frac_of_" + peak_src: round(step_bytes_of(alg) / (ms * 1e-3) / 1e9 / peak, 4),
                "kernels": kernel_stats(run, iso, steady, sets, alg, peak, peak_src),
                "clocks": clocks.report()}
    finally:
        run.release()


OTHER_WORKLOADS = [("tiny", "int8_token"), ("tiny", "bf16"), ("decode", None), ("skewed", None),
                   ("large", None), ("prefill", None)]


# ---------------------------------------------------------------------------
def main():
    args = parse()
    world, rank, local = dist_init()
    wname = args.workload
    w = synth.workload(wname) if args.tokens_per_rank is None else \
        synth.workload(wname, T=args.tokens_per_rank)
    mode = WORKLOAD_MODE[wname]
    replica = rank

    if args.impl == "reference":
        run_reference(args, w, mode, world, rank)
        return

    import combine_ep_dispatch_04_b200 as ep

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.only == "ffn":
        stream = torch.cuda.current_stream(dev)
        flush_w = torch.empty(args.flush_mib << 20, dtype=torch.uint8, device=dev)
        flush_r = torch.ones(args.flush_mib << 20, dtype=torch.uint8, device=dev)

        def flush_only(v):
            flush_w.fill_(v)
            flush_r.max()
        leg = run_ffn_leg(ep, flush_only, stream, dev, args, replica)
        if rank == 0:
            print(json.dumps({"expert_ffn": leg}), flush=True)
        dist_done(world)
        return
    if (world > 1 and not args.replicas) or args.ep_group:
        run_group_bench(ep, args, wname, world, rank, local, dev)
        return
    if args.weights_grad and args.quantized_combine:
        raise SystemExit("--weights-grad reads bf16 expert outputs: not with --quantized-combine")
    stream = torch.cuda.current_stream(dev)
    flush_w = torch.empty(args.flush_mib << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(args.flush_mib << 20, dtype=torch.uint8, device=dev)

    def flush(v):
        flush_w.fill_(v)
        flush_r.max()

    run = WorkloadRun(ep, wname, args, dev, stream, replica, t_override=args.tokens_per_rank,
                      quantized_step=args.quantized_combine, weights_grad=args.weights_grad)
    N = run.w["N"]
    for _ in range(max(args.warmup, 3)):
        flush(1)
        run.step()
    torch.cuda.synchronize(dev)
    if ep.ep_get_status(run.b.dev_status) != 0:
        raise SystemExit("device status reported errors during warm-up")

    # timed region: K steps, one event pair per step (events between the
    # kernels would add their own ~2 us each to the step)
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize(dev)
    launches0 = ep.ep_kernel_launches()
    with clocks:
        step_ms = timed_steps(run, args.steps, flush)
    launches = ep.ep_kernel_launches() - launches0
    barrier(world)
    total_ms = max_over_ranks(sum(step_ms), world)
    ms_per_step = total_ms / args.steps
    value = world * N * args.steps / (total_ms / 1e3)

    graph = graph_steps(ep, args, run, flush, world)

    # per-kernel durations (for the roofline): each kernel after its own flush
    # and between its own pair of events, then back to back where the step is small
    per_kernel = isolated_launches(run, args.steps, flush)
    alg, v = algorithmic_bytes(run.w, run.mode, run.idx, quantized_combine=args.quantized_combine,
                               weights_grad=args.weights_grad)
    step_bytes = step_bytes_of(alg)
    steady, sets = steady_launches(run, args.steps, flush, step_bytes, skip=args.no_steady)
    peak, peak_src = hbm_peak()
    kstats = kernel_stats(run, per_kernel, steady, sets, alg, peak, peak_src)
    step_kernels = [k for k in run.kernels if k not in ("combine_bwd_w", "combine_q")]
    dom = max(step_kernels, key=lambda k: alg[k])
    iso_achieved = alg[dom] / (statistics.mean(per_kernel[dom]) * 1e-3) / 1e9
    if sets > 1:
        achieved = alg[dom] / (statistics.mean(steady[dom]) * 1e-3) / 1e9
        duration = (f"per launch: {sets} launches back to back on {sets} distinct copies of the "
                    f"kernel's inputs and outputs between one pair of events, L2 flushed before "
                    f"each group")
    else:
        achieved = iso_achieved
        duration = "per launch: each launch alone between its own events, after an L2 flush"

    e2e = None if args.no_e2e else run_e2e(ep, run, flush, args, world, step_bytes)
    workload_name = run.name() + (", combine of quantised expert outputs"
                                  if args.quantized_combine else "")
    run.release()
    del run

    # same-run copy bandwidth (reference for the fractions above)
    copy_gbs = None
    try:
        if args.no_copy:
            raise RuntimeError("skipped")
        src = torch.empty(2 << 30, dtype=torch.uint8, device=dev)
        dst = torch.empty_like(src)
        for _ in range(3):
            ep.ep_copy(dst, src, stream=stream)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        best = None
        for _ in range(10):
            e0.record(stream)
            ep.ep_copy(dst, src, stream=stream)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            t = e0.elapsed_time(e1)
            best = t if best is None or t < best else best
        copy_gbs = round(2 * src.numel() / (best * 1e-3) / 1e9, 1)
        del src, dst
        torch.cuda.empty_cache()
    except Exception:
        pass

    # every other named workload through the same per-kernel protocol (one GPU)
    workloads = None
    if world == 1 and not args.no_workloads and args.tokens_per_rank is None:
        workloads = {}
        for wn, md in OTHER_WORKLOADS:
            key = wn if md is None or md == WORKLOAD_MODE[wn] else f"{wn}_{md}"
            if wn == wname and (md is None or md == mode):
                workloads[key] = {"see": "headline (kernels, roofline)"}
                continue
            try:
                workloads[key] = other_workload(ep, wn, md, args, dev, stream, flush, local)
            except Exception as ex:  # noqa: BLE001 -- reported in the line
                workloads[key] = {"error": f"{type(ex).__name__}: {ex}"[:300]}
                torch.cuda.empty_cache()

    # the experts between dispatch and combine, outside the step: by default on
    # one GPU, on the routing of --gemm-workload; a leg that fails reports its
    # error instead of ending the bench
    gemm_on = args.gemm or (world == 1 and not args.no_gemm)
    gemm = gemm_mx = gemm_mx4 = None
    if gemm_on:
        gw = synth.workload(args.gemm_workload)
        gidx, gwts = synth.make_routing(gw, replica)
        gx = synth.make_x(gw, replica)
        gidx_d = torch.from_numpy(gidx).to(dev)
        gwts_d = torch.from_numpy(gwts).to(dev)
        gx_d = torch.from_numpy(gx.view(np.int16)).to(dev).view(torch.bfloat16)

        def leg(fn, *a):
            try:
                return fn(*a)
            except Exception as ex:  # noqa: BLE001 -- reported in the line
                torch.cuda.empty_cache()
                return {"error": f"{type(ex).__name__}: {ex}"[:300]}
        gemm = leg(run_gemm, ep, gw, gx_d, gidx_d, gwts_d, flush, stream, dev, args)
        gemm_mx = leg(run_gemm_mx, ep, gw, gx_d, gidx_d, gwts_d, flush, stream, dev, args)
        gemm_mx4 = (leg(run_gemm_mx, ep, gw, gx_d, gidx_d, gwts_d, flush, stream, dev, args,
                        "mxfp4") if gw["H"] % 256 == 0 else None)
        del gx_d, gidx_d, gwts_d
        torch.cuda.empty_cache()
    ffn = None
    if gemm_on:
        try:
            ffn = run_ffn_leg(ep, flush, stream, dev, args, replica)
        except Exception as ex:  # noqa: BLE001 -- reported in the line
            torch.cuda.empty_cache()
            ffn = {"error": f"{type(ex).__name__}: {ex}"[:300]}

    out = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {
            "workload": workload_name,
            "tokens_per_step": N, "valid_entries": v,
            "l2": f"flushed between steps outside the step events ({args.flush_mib} MiB write, "
                  f"then {args.flush_mib} MiB read); per-kernel timings: each kernel after its "
                  f"own flush",
            "parallelism": "replicas" if world > 1 else "single",
        },
        "hbm_gbs": round(step_bytes / (ms_per_step * 1e-3) / 1e9, 1),
        "hbm_frac_of_" + peak_src: round(step_bytes / (ms_per_step * 1e-3) / 1e9 / peak, 4),
        "clocks": clocks.report(),
        "gpu_launches": launches,
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1),
                     "peak": peak, "peak_source": peak_src, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": ncu_traffic(dom, wname), "duration": duration,
                     "isolated_launch": {"achieved": round(iso_achieved, 1),
                                         "frac": round(iso_achieved / peak, 4)}},
        "kernels": kstats,
        "workloads": workloads,
        "graph": graph,
        "expert_gemm": gemm,
        "expert_gemm_mx": gemm_mx,
        "expert_gemm_mxfp4": gemm_mx4,
        "expert_ffn": ffn,
        "copy_gbs_same_run": copy_gbs,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, mode, args.cpu_seconds, replica)
        try:
            out["cpu_baseline_all_cores"] = cpu_baseline_all_cores(
                wname, args.tokens_per_rank, mode, args.cpu_seconds, replica)
        except Exception as e:  # a host without process support: report, do not fail
            out["cpu_baseline_all_cores"] = {"unavailable": f"{type(e).__name__}: {e}"[:160]}
    if rank == 0:
        print(json.dumps(out), flush=True)
    dist_done(world)


def graph_steps(ep, args, run, flush, world):
    """The timed step captured once in a CUDA graph and replayed, with the same
    flush and event protocol: the step without the host's per-launch work (the
    device-side gaps between the kernels remain).  Every rank takes the same
    collective steps: the capture's outcome is agreed on first (a failure on
    any rank reports it on all and times nothing)."""
    dev, stream, b = run.dev, run.stream, run.b
    graph, why = None, None
    try:
        gs = torch.cuda.Stream(dev)
        gcalls = [
            ep.ep_dispatch_with_layout(run.cfg, run.x_d, run.idx_d, b.token_slot, b.recv_count,
                                       b.workspace, b.recv_buf, b.src_info, b.dev_status,
                                       expert_offset=b.expert_offset, stream=gs, bind=True),
            ep.ep_combine(run.step_ccfg, run.step_y, run.idx_d, run.wts_d, b.token_slot, b.out,
                          b.dev_status, expert_offset=b.expert_offset, stream=gs, bind=True),
        ]
        if run.g_d is not None:
            gcalls.append(ep.ep_combine_backward(run.cfg, run.g_d, run.idx_d, run.wts_d,
                                                 b.token_slot, b.grad_buf, b.dev_status,
                                                 expert_offset=b.expert_offset, stream=gs,
                                                 bind=True))
        gs.wait_stream(stream)
        for c in gcalls:  # warm, outside capture
            c()
        stream.wait_stream(gs)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=gs):
            for c in gcalls:
                c()
        torch.cuda.synchronize(dev)
    except Exception as e:  # report, do not fail the bench
        graph, why = None, f"{type(e).__name__}: {str(e).splitlines()[0][:120]}" if str(e) else \
            type(e).__name__
    if max_over_ranks(0.0 if graph is not None else 1.0, world) > 0.0:
        return {"unavailable": why or "capture failed on another rank"}
    for _ in range(3):
        flush(1)
        graph.replay()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    for s in range(args.steps):
        flush(s & 0xFF)
        evs[s][0].record(stream)
        graph.replay()
        evs[s][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    total = max_over_ranks(sum(a.elapsed_time(c) for a, c in evs), world)
    del graph
    N = run.w["N"]
    return {"ms_per_step": round(total / args.steps, 5),
            "value": round(world * N * args.steps / (total / 1e3), 1), "unit": "tokens/s"}


def gemm_routing(E, idx_d, args):
    """The GEMM legs' experts: the workload's, or --gemm-experts of them (expert
    id modulo E; a token may then reach one expert twice, which the packed
    layout receives as two rows)."""
    if not args.gemm_experts or args.gemm_experts == E:
        return E, idx_d
    E2 = args.gemm_experts
    return E2, torch.where(idx_d >= 0, torch.remainder(idx_d, E2), idx_d)


def time_moe_forward(ep, cfg, b, x_d, idx_d, wts_d, wc, ws, y, flush, stream, dev, args):
    """The whole forward path in one call (ep_moe_forward: layout + dispatch ->
    the experts' maps -> combine) with the GEMM leg's weights, timed alone
    between events after an L2 flush; tokens/s = N / time."""
    N, H = cfg.num_ranks * cfg.num_tokens, cfg.hidden
    out = torch.empty((N, H), dtype=torch.bfloat16, device=dev)
    call = ep.ep_moe_forward(cfg, x_d, idx_d, wts_d, wc, ws, b.token_slot, b.recv_count,
                             b.expert_offset, b.workspace, b.recv_buf, b.src_info, y, out,
                             b.dev_status, stream=stream, bind=True)
    for _ in range(3):
        flush(1)
        call()
    torch.cuda.synchronize(dev)
    if ep.ep_get_status(b.dev_status) != 0:
        raise RuntimeError("ep_moe_forward reported a device error")
    reps = max(3, min(args.steps, 20))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for s in range(reps):
        flush(s & 0xFF)
        evs[s][0].record(stream)
        call()
        evs[s][1].record(stream)
    torch.cuda.synchronize(dev)
    ms = statistics.mean(a.elapsed_time(c) for a, c in evs)
    del out
    return {"ms": round(ms, 4), "tokens_per_s": round(N / (ms * 1e-3), 1),
            "launches": 4, "what": "layout + dispatch, the experts' maps (n_out = H), combine"}


def run_gemm(ep, w, x_d, idx_d, wts_d, flush, stream, dev, args):
    """The experts between dispatch and combine (ep_expert_gemm): the workload's
    tokens dispatched as bf16 into the packed layout, one seeded random linear
    map of H x H per expert, timed alone between events after an L2 flush.
    FLOPs = 2 * (valid entries) * H * H."""
    R, T, M, K, E, H = w["R"], w["T"], w["M"], w["K"], w["E"], w["H"]
    E, idx_d = gemm_routing(E, idx_d, args)
    cfg = ep.make_config(R, T, M, K, E, H, "bf16", "packed")
    b = ep.Buffers(cfg, device=dev, expert_out=False)
    ep.ep_dispatch_with_layout(cfg, x_d, idx_d, b.token_slot, b.recv_count, b.workspace,
                               b.recv_buf, b.src_info, b.dev_status,
                               expert_offset=b.expert_offset, stream=stream)
    gen = torch.Generator(device=dev).manual_seed(1234)
    W = torch.randn(E, H, H, device=dev, dtype=torch.bfloat16, generator=gen).mul_(0.02)
    y = torch.empty((b.sizes["rows"], H), dtype=torch.bfloat16, device=dev)
    call = ep.ep_expert_gemm(cfg, b.recv_buf, b.expert_offset, b.recv_count, W, y, b.dev_status,
                             stream=stream, bind=True)
    for _ in range(3):
        flush(1)
        call()
    torch.cuda.synchronize(dev)
    if ep.ep_get_status(b.dev_status) != 0:
        raise RuntimeError("ep_expert_gemm reported a device error")
    v = int(b.recv_count.sum().item())
    reps = max(3, min(args.steps, 20))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for s in range(reps):
        flush(s & 0xFF)
        evs[s][0].record(stream)
        call()
        evs[s][1].record(stream)
    torch.cuda.synchronize(dev)
    ms = statistics.mean(a.elapsed_time(c) for a, c in evs)
    flops = 2.0 * v * H * H
    # bytes that must move at least once: the weights of every expert that
    # received a row, the received rows, the outputs
    used = int((b.recv_count > 0).sum().item())
    nbytes = 2.0 * used * H * H + 2.0 * 2 * v * H
    peaks = measured_peaks() or {}
    peak = peaks.get("bf16_tflops") or 1590.0
    hbm = peaks.get("hbm_gbs") or 6650.0
    tf = flops / (ms * 1e-3) / 1e12
    t_tensor, t_hbm = flops / (peak * 1e12), nbytes / (hbm * 1e9)
    moe = time_moe_forward(ep, cfg, b, x_d, idx_d, wts_d, W, None, y, flush, stream, dev, args)
    del W, y, b
    torch.cuda.empty_cache()
    return {"ms": round(ms, 4), "flops": flops, "bytes": nbytes, "tflops": round(tf, 1),
            "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
            "bound": "tensor" if t_tensor >= t_hbm else "hbm",
            "peak_tflops": peak, "peak_gbs": hbm,
            "peak_source": "measured" if peaks.get("bf16_tflops") else "fallback",
            "frac": round(max(t_tensor, t_hbm) / (ms * 1e-3), 4),
            "shape": f"{E} experts, {v} rows, {H} x {H} bf16 each", "moe_forward": moe}


def run_gemm_mx(ep, w, x_d, idx_d, wts_d, flush, stream, dev, args, fmt="mxfp8"):
    """The experts' maps on MX operands (ep_expert_gemm_mx): the workload's
    tokens dispatched as MXFP8 or MXFP4 into the packed layout, seeded random
    weights of H x H per expert in the same format (e4m3 codes uniform over
    the finite bit patterns, or packed e2m1 bytes uniform over all 256; e8m0
    scales in [118, 134)), timed alone between events after an L2 flush.
    FLOPs = 2 * (valid entries) * H * H; the tensor peak is the measured bf16
    peak times the nominal ratio (fp8 4.5 / 2.25, fp4 9 / 2.25)."""
    R, T, M, K, E, H = w["R"], w["T"], w["M"], w["K"], w["E"], w["H"]
    E, idx_d = gemm_routing(E, idx_d, args)
    fp4 = fmt == "mxfp4"
    cfg = ep.make_config(R, T, M, K, E, H, fmt, "packed")
    b = ep.Buffers(cfg, device=dev, expert_out=False)
    ep.ep_dispatch_with_layout(cfg, x_d, idx_d, b.token_slot, b.recv_count, b.workspace,
                               b.recv_buf, b.src_info, b.dev_status,
                               expert_offset=b.expert_offset, stream=stream)
    gen = torch.Generator(device=dev).manual_seed(4321)
    D = H // 2 if fp4 else H
    wc = torch.randint(0, 256, (E, H, D), device=dev, dtype=torch.int16, generator=gen).to(torch.uint8)
    if not fp4:
        wc[(wc & 0x7F) == 0x7F] = 0
    ws = torch.randint(118, 134, (E, H, H // 32), device=dev, dtype=torch.int16,
                       generator=gen).to(torch.uint8)
    y = torch.empty((b.sizes["rows"], H), dtype=torch.bfloat16, device=dev)
    call = ep.ep_expert_gemm_mx(cfg, b.recv_buf, b.expert_offset, b.recv_count, wc, ws, y,
                                b.dev_status, stream=stream, bind=True)
    for _ in range(3):
        flush(1)
        call()
    torch.cuda.synchronize(dev)
    if ep.ep_get_status(b.dev_status) != 0:
        raise RuntimeError(f"ep_expert_gemm_mx ({fmt}) reported a device error")
    v = int(b.recv_count.sum().item())
    reps = max(3, min(args.steps, 20))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for s in range(reps):
        flush(s & 0xFF)
        evs[s][0].record(stream)
        call()
        evs[s][1].record(stream)
    torch.cuda.synchronize(dev)
    ms = statistics.mean(a.elapsed_time(c) for a, c in evs)
    flops = 2.0 * v * H * H
    used = int((b.recv_count > 0).sum().item())
    row = D + H / 32                      # codes and scales of one row
    nbytes = used * H * row + v * row + 2.0 * v * H
    peaks = measured_peaks() or {}
    ratio = 4.0 if fp4 else 2.0
    peak = (peaks.get("bf16_tflops") or 1590.0) * ratio
    hbm = peaks.get("hbm_gbs") or 6650.0
    tf = flops / (ms * 1e-3) / 1e12
    t_tensor, t_hbm = flops / (peak * 1e12), nbytes / (hbm * 1e9)
    moe = time_moe_forward(ep, cfg, b, x_d, idx_d, wts_d, wc, ws, y, flush, stream, dev, args)
    del wc, ws, y, b
    torch.cuda.empty_cache()
    return {"ms": round(ms, 4), "flops": flops, "bytes": nbytes, "tflops": round(tf, 1),
            "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
            "bound": "tensor" if t_tensor >= t_hbm else "hbm",
            "peak_tflops": peak, "peak_gbs": hbm,
            "peak_source": (f"measured bf16 x {ratio:g} (nominal {'fp4' if fp4 else 'fp8'} / bf16)"
                            if peaks.get("bf16_tflops") else f"fallback bf16 x {ratio:g}"),
            "frac": round(max(t_tensor, t_hbm) / (ms * 1e-3), 4),
            "shape": f"{E} experts, {v} rows, {H} x {H} {fmt.upper()} each", "moe_forward": moe}


L2_BYTES = 126 << 20


def run_e2e(ep, run, flush, args, world, step_bytes):
    """The same step through the public API with host buffers: every step
    copies its inputs in from pinned host memory and its combined output and
    counts back, inside the timed region.  Steps are pipelined as a serving
    loop would run them: two complete buffer sets, the copy-in of step i+1 and
    the copy-out of step i-1 overlapping the kernels of step i (three streams,
    events guarding each buffer's reuse).  Expert outputs (and the gradient)
    stay on the device: in a MoE layer the experts produce them there.  Two
    alternating sets move more than three L2s of data per pair of steps, so
    no step finds its data in L2; smaller workloads flush L2 before each
    step's kernels instead."""
    w, b, cfg, ccfg, g_d = run.w, run.b, run.cfg, run.step_ccfg, run.g_d
    dev, stream = run.dev, run.stream
    N, H = w["N"], w["H"]
    x_h = torch.from_numpy(run.x.view(np.int16)).view(torch.bfloat16).pin_memory()
    idx_h = torch.from_numpy(run.idx).to(ep.idx_dtype(cfg)).pin_memory()
    wts_h = torch.from_numpy(run.wts).pin_memory()
    h2d = x_h.numel() * 2 + idx_h.numel() * idx_h.element_size() + wts_h.numel() * 4
    d2h = N * H * 2 + w["E"] * 8
    flush_each = 2 * step_bytes < 3 * L2_BYTES

    sets = []
    for j in range(2):
        bj = b if j == 0 else ep.Buffers(cfg, device=dev, expert_out=False,
                                          grad=g_d is not None)
        yj = run.step_y if j == 0 else run.step_y.clone()
        st = {"b": bj, "y": yj,
              "x": torch.empty((N, H), dtype=torch.bfloat16, device=dev),
              "idx": torch.empty_like(idx_h, device=dev),
              "wts": torch.empty_like(wts_h, device=dev),
              "out_h": torch.empty((N, H), dtype=torch.bfloat16).pin_memory(),
              "cnt_h": torch.empty(w["E"], dtype=torch.int64).pin_memory(),
              "in_done": torch.cuda.Event(), "comp_done": torch.cuda.Event(),
              "out_done": torch.cuda.Event()}
        calls = [
            ep.ep_dispatch_with_layout(cfg, st["x"], st["idx"], bj.token_slot, bj.recv_count,
                                       bj.workspace, bj.recv_buf, bj.src_info, bj.dev_status,
                                       expert_offset=bj.expert_offset, stream=stream, bind=True),
            ep.ep_combine(ccfg, yj, st["idx"], st["wts"], bj.token_slot, bj.out, bj.dev_status,
                          expert_offset=bj.expert_offset, stream=stream, bind=True),
        ]
        if g_d is not None:
            calls.append(ep.ep_combine_backward(cfg, g_d, st["idx"], st["wts"], bj.token_slot,
                                                bj.grad_buf, bj.dev_status,
                                                expert_offset=bj.expert_offset, stream=stream,
                                                bind=True))
        st["calls"] = calls
        sets.append(st)
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)

    def one(i):
        st = sets[i % 2]
        s_in.wait_event(st["comp_done"])       # step i-2's kernels are done with this set
        with torch.cuda.stream(s_in):
            st["x"].copy_(x_h, non_blocking=True)
            st["idx"].copy_(idx_h, non_blocking=True)
            st["wts"].copy_(wts_h, non_blocking=True)
            st["in_done"].record(s_in)
        stream.wait_event(st["in_done"])
        stream.wait_event(st["out_done"])      # step i-2's output has left this set
        if flush_each:
            flush(i & 0xFF)
        for c in st["calls"]:
            c()
        st["comp_done"].record(stream)
        s_out.wait_event(st["comp_done"])
        with torch.cuda.stream(s_out):
            st["out_h"].copy_(st["b"].out, non_blocking=True)
            st["cnt_h"].copy_(st["b"].recv_count, non_blocking=True)
            st["out_done"].record(s_out)

    for i in range(4):
        one(i)
    torch.cuda.synchronize(dev)
    steps = max(10, min(args.steps, 100))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for i in range(steps):
        one(i)
    stream.wait_stream(s_out)
    stream.wait_stream(s_in)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    total_ms = max_over_ranks(e0.elapsed_time(e1), world)
    del sets
    torch.cuda.empty_cache()
    return {"value": round(world * N * steps / (total_ms / 1e3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "pipelined": "2 buffer sets; copy-in, kernels and copy-out of consecutive steps "
                         "overlap on three streams",
            "l2": "flushed before each step's kernels" if flush_each else
                  "not flushed: two alternating buffer sets move over 3x L2 per pair of steps"}


def run_reference(args, w, mode, world, rank):
    """The reference arm: the oracle on the host cores, rank 0 only, each step
    a bounded sample of the workload (about SAMPLE_TOKENS tokens)."""
    if rank != 0:
        dist_done(world)
        return
    st = OracleStep(w, mode, sample_tokens_per_rank(w))
    for _ in range(args.warmup):
        st.step()
    t0 = time.perf_counter()
    done = 0
    for _ in range(args.steps):
        done += st.step()
    el = time.perf_counter() - t0
    value = done / el
    R, T, M, K, E, H = w["R"], w["T"], w["M"], w["K"], w["E"], w["H"]
    out = {
        "impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"{w['name']}: R={R} T={T} H={H} K={K} E={E} M={M} {mode} "
                               f"{w['layout']}", "tokens_per_step": st.n},
        "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "cores": 1,
                         "kind": "oracle", "sample": st.sample},
        "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)
    dist_done(world)


if __name__ == "__main__":
    main()
