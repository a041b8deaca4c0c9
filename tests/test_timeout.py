"""The error path of the bounded device-side waits, driven by the library's test hook
(hs2_debug_stall_waits): a wait that nothing will satisfy runs out after a short limit,
the kernel records HS2_ERR_DEVICE_TIMEOUT, finishes without leaving a copy or an MMA in
flight, and the context stays usable (a normal call on a re-zeroed workspace matches the
oracle).  No GPU is faulted or hung: every wait is bounded and the hook only shortens
the limit of a wait that would otherwise never end."""
import pytest
import torch

import oracle  # noqa: F401  (the parity helpers below use it)
from long_context_token_b200 import hs2, workloads
from test_parity import compare, run_gpu

pytestmark = [pytest.mark.gpu, pytest.mark.filterwarnings("ignore::RuntimeWarning")]

HS2_ERR_DEVICE_TIMEOUT = 5


@pytest.mark.parametrize("mode", [1, 2], ids=["mbarrier-wait", "row-barrier"])
def test_wait_runs_out_reports_timeout_and_context_stays_usable(mode):
    inp = workloads.make_inputs(2, 5000, n_q=1, h_q=16, kv="bf16", n_sparse=1, seed=161,
                                lens=[5000, 3333])
    dev = torch.device("cuda:0")
    cache = hs2.Cache(inp.k.to(dev), inp.v.to(dev), inp.lens.to(dev))
    assert hs2.select_fused(cache, 1, 16)  # one launch: stream, merge and selection
    ws = hs2.alloc_workspace(cache, 1, 16)
    L = hs2.lib()
    L.hs2_debug_stall_waits(mode)
    try:
        hs2.full_attn_select(inp.q.to(dev), cache, inp.window, inp.k_sel, inp.sm_scale, ws)
        torch.cuda.synchronize()
    finally:
        L.hs2_debug_stall_waits(0)
    assert hs2.check_device_status(ws) == HS2_ERR_DEVICE_TIMEOUT
    assert hs2.check_device_status(ws) == 0  # the check cleared it
    # The context is intact: the same sizes on a fresh workspace match the oracle.
    runs, status = run_gpu(inp)
    assert status == 0
    compare(inp, runs[0])


def test_status_check_returns_lowest_code_and_clears_all():
    dev = torch.device("cuda:0")
    k = torch.zeros(1, 512, 128, dtype=torch.bfloat16, device=dev)
    cache = hs2.Cache(k, k.clone(), torch.full((1,), 512, dtype=torch.int32, device=dev))
    ws = hs2.alloc_workspace(cache, 1, 16)
    # Two kinds of error recorded (bits 7 and 6: bad length, index out of range).
    ws[:4].view(torch.int32)[0] = (1 << 7) | (1 << 6)
    assert hs2.check_device_status(ws) == 6
    assert hs2.check_device_status(ws) == 0
