"""Stage markers (wildcat_set_stage_events): a forward records the caller's
events after its select and after its weights on its own stream; the output
is the same as without markers, and the three stage times add up to the
whole call."""
import pytest
import torch

import nystr_coreset_approximate_b200 as wc
import workloads
from tests import gpu_common as gc

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nbins", [1, 4])
def test_stage_events_split_a_forward(nbins):
    w = gc.case("stage_ev", "iid", 4, 4096, 512, 64, 64, "bf16")
    dev, _ = workloads.make(w)
    d = gc.cuda_inputs(dev)
    plan = (wc.ForwardPlan(w.BH, w.m, w.n, w.d, w.r, w.dtype) if nbins == 1
            else wc.BinnedForwardPlan(w.BH, w.m, w.n, w.d, w.r, nbins, w.dtype))
    O_ref = plan.run(d["Q"], d["K"], d["V"], w.beta, w.pivot_seed)[0].clone()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for e in ev:
        e.record()
    torch.cuda.synchronize()
    wc.set_stage_events(ev[1], ev[2])
    try:
        ev[0].record()
        O = plan.run(d["Q"], d["K"], d["V"], w.beta, w.pivot_seed)[0]
        ev[3].record()
    finally:
        wc.set_stage_events(None, None)
    torch.cuda.synchronize()
    assert torch.equal(O, O_ref)
    t = [ev[k].elapsed_time(ev[k + 1]) for k in range(3)]
    assert all(x > 0 for x in t)
    assert abs(sum(t) - ev[0].elapsed_time(ev[3])) < 5e-3
    assert wc.device_status() == 0


def test_stage_events_need_a_recorded_handle():
    with pytest.raises(ValueError):
        wc.set_stage_events(torch.cuda.Event(enable_timing=True), None)
