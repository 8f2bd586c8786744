"""Bounded waits: a kernel whose barrier never completes gives up after its
limit, reports LORA_ERR_TIMEOUT through the status word, and leaves the
context usable.  The wait runs out on purpose; nothing faults or hangs."""
import pytest
import torch

import workloads as WL
from gpu_helpers import run_fwd

pytestmark = pytest.mark.gpu


def test_wait_gives_up_and_reports_timeout(gpu):
    code = gpu.lora_selftest_wait_timeout(20_000_000)   # 20 ms
    assert gpu.STATUS[code] == "LORA_ERR_TIMEOUT"
    assert gpu.lora_get_device_status() == 0            # the flag was cleared
    sh = WL.LayerShape(128, 256, 256, 16, 32.0)
    t = WL.make_layer_inputs(sh, seed=0)
    Y = run_fwd(gpu, t["X"], t["W"], t["A"], t["B"], sh.alpha)
    assert torch.isfinite(Y.float()).all()


def test_unsupported_arguments_raise_before_launch(gpu):
    X = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    A = torch.zeros((12, 64), dtype=torch.bfloat16, device="cuda")   # r = 12: not a multiple of 8
    B = torch.zeros((64, 12), dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gpu.LoraError) as e:
        gpu.lora_fwd(X, W, A, B, Y, 24.0)
    assert e.value.code == gpu.STATUS_CODE["LORA_ERR_RANK"]
