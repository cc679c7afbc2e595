"""Runs only in the checked build (MOE_LIB_VARIANT=checks; see
test_gpu_checks.py): an expert-offsets table that is not non-decreasing --
every value still inside the slot range, so even a kernel without the check
stays in bounds -- is reported as MOE_ERR_DEVICE_CHECK by the grouped GEMMs'
offsets check."""
import os

import pytest
import torch

from routed_expert_layer_route_b200 import moe, synth

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(os.environ.get("MOE_LIB_VARIANT") != "checks",
                                 reason="checked build only (MOE_LIB_VARIANT=checks)")]
DEV = torch.device("cuda:0")


def test_checked_build_is_loaded():
    assert moe.LIB_PATH.endswith("libmoe_checks.so")
    moe.lib()


def test_checked_build_reports_decreasing_offsets():
    T, d, E, I, k1 = 8, 256, 8, 128, 2
    L = synth.make_layer(T, d, E, I, seed=1, device=DEV)
    n = T * k1
    off = torch.tensor([0, 4, 2, 6, 8, 10, 12, 14, n], dtype=torch.int32, device=DEV)
    ss = torch.arange(n, dtype=torch.int32, device=DEV)
    out = torch.zeros(n, d, dtype=torch.float32, device=DEV)
    ws = moe.workspace(T, d, E, I, k1, device=DEV)
    moe.moe_expert_ffn(L.x, off, ss, L.w_gate, L.w_up, L.w_down, k1, out, ws,
                       flags=moe.MOE_PATH_GROUPED)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == moe.MOE_ERR_DEVICE_CHECK
    # the workspace serves a consistent call afterwards
    moe.moe_workspace_init(ws)
    off_ok = torch.tensor([0, 2, 4, 6, 8, 10, 12, 14, n], dtype=torch.int32, device=DEV)
    moe.moe_expert_ffn(L.x, off_ok, ss, L.w_gate, L.w_up, L.w_down, k1, out, ws,
                       flags=moe.MOE_PATH_GROUPED)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == 0
