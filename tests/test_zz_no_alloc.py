"""The allocation-free layout entry point, ep_dispatch_layout_static.

Some callers cannot allocate device memory at the moment they route tokens:
a serving loop that reserved all of its device memory up front, or a plugin
inside a host framework that owns every device allocation (and cudaMalloc
would also stall the whole device).  Such callers cannot hand the layout a
workspace, so this entry point keeps its scratch in a static array inside
libep.so instead.  The test calls it through the C ABI twice in a row, on two
different routings so that the second call starts from the first call's
leftover scratch, and checks every output against the regular
ep_dispatch_layout (integer outputs: bit-exact).  It runs the same alone in
a fresh process or after the rest of the suite.  The static array comes into
being when CUDA loads the library's device code on the device (lazily, at
the first call into the library there); a caller that reserves the whole
device up front makes one such call first, which is what the first case
here is in a fresh process.
"""
import numpy as np
import pytest
import torch

import combine_ep_dispatch_04_b200 as ep
import synth

pytestmark = pytest.mark.gpu

OUTPUTS = ("token_slot", "recv_count", "tokens_per_rank", "tokens_per_expert",
           "is_token_in_rank", "expert_offset")


def _outputs(cfg, idx_d, static):
    b = ep.Buffers(cfg, expert_out=False)
    for name in OUTPUTS:
        t = getattr(b, name)
        if t is not None:
            t.fill_(-3)
    stats = torch.zeros(cfg.num_experts, dtype=torch.int64, device="cuda")
    if static:
        ep.ep_dispatch_layout_static(cfg, idx_d, b.token_slot, b.recv_count, b.dev_status,
                                     b.tokens_per_rank, b.tokens_per_expert, b.is_token_in_rank,
                                     b.expert_offset, stats)
    else:
        ep.ep_dispatch_layout(cfg, idx_d, b.token_slot, b.recv_count, b.workspace, b.dev_status,
                              b.tokens_per_rank, b.tokens_per_expert, b.is_token_in_rank,
                              b.expert_offset, stats)
    flags = ep.ep_get_status(b.dev_status)
    out = {n: getattr(b, n).cpu().numpy() for n in OUTPUTS if getattr(b, n) is not None}
    out["stats"] = stats.cpu().numpy()
    out["flags"] = flags
    return out


def _case(name, **override):
    w = synth.workload(name, **override)
    idx, _ = synth.make_routing(w)
    cfg = ep.make_config(w["R"], w["T"], w["M"], w["K"], w["E"], w["H"], "mxfp8", "packed", 8)
    return cfg, torch.from_numpy(idx).cuda()


def test_static_scratch_layout_matches_workspace_layout_twice():
    # first call: a routing with many chunks; second call: a different one that
    # reuses (and must overwrite) the scratch the first call left behind
    cases = [_case("prefill", T=512), _case("large", T=100)]
    for cfg, idx_d in cases:
        assert ep.ep_buffer_sizes(cfg)["workspace_bytes"] <= ep.STATIC_SCRATCH_BYTES
        got = _outputs(cfg, idx_d, static=True)
        want = _outputs(cfg, idx_d, static=False)
        for k in want:
            assert np.array_equal(got[k], want[k]), k


def test_static_scratch_rejects_oversized_requests():
    # E = 1024 experts over 131072 tokens needs more scratch than the static array holds
    cfg = ep.make_config(32, 4096, 4096, 8, 1024, 7168, "mxfp8", "packed")
    assert ep.ep_buffer_sizes(cfg)["workspace_bytes"] > ep.STATIC_SCRATCH_BYTES
    b_slot = torch.empty((32 * 4096, 8), dtype=torch.int32, device="cuda")
    cnt = torch.empty(1024, dtype=torch.int64, device="cuda")
    eo = torch.empty(1025, dtype=torch.int64, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx = torch.zeros((32 * 4096, 8), dtype=torch.int64, device="cuda")
    n0 = ep.ep_kernel_launches()
    with pytest.raises(ep.EpError) as ei:
        ep.ep_dispatch_layout_static(cfg, idx, b_slot, cnt, st, expert_offset=eo)
    assert ei.value.status == 2  # EP_ERR_UNSUPPORTED, before any launch
    assert ep.ep_kernel_launches() == n0
