"""Failure detection without a GPU fault: a pipeline wait that nothing will
ever satisfy gives up after its time limit, the timeout reaches the host
through the workspace status word, and the context stays usable for the
next layer call."""
import pytest
import torch

from mixture_experts_layer_49_b200 import native as nat
from mixture_experts_layer_49_b200 import synthetic as syn

from helpers import make_case

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(cuda_device):
    wl = syn.Workload("after_timeout", T=300, d_model=128, E=8, d_ff=128, top_k=2)
    cfg = nat.config_from_workload(wl)
    ws = nat.alloc_workspace(cfg, cuda_device)
    nat.moe_check_wait_timeout(ws, 20_000_000)              # 20 ms
    assert nat.moe_get_device_status(ws) == nat.MOE_ERR_TIMEOUT
    assert nat.moe_get_device_status(ws) == nat.MOE_OK       # reading clears it
    inp, _ = make_case(wl, cuda_device, seed=3)
    out = nat.Outputs(cfg, cuda_device)
    nat.forward(cfg, inp, out, ws)
    torch.cuda.synchronize(cuda_device)
    assert nat.moe_get_device_status(ws) == nat.MOE_OK
    assert torch.isfinite(out.y.float()).all()
