"""The bounded device waits give up instead of hanging: with the wait limit
shortened to 1 ms, a kernel that waits on something nothing ever completes (a
header flag, an mbarrier phase, the one-token layer's router exchange for a
tag no CTA publishes) returns, the workspace's status word reads
MOE_ERR_TIMEOUT, and after moe_workspace_init the same workspace serves a
normal layer call with status OK and oracle-matching output.  No fault, trap
or hang is involved: each wait is the library's own, bounded by the limit."""
import pytest
import torch

from routed_expert_layer_route_b200 import moe, synth

from parity import check_layer_full

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture
def short_waits():
    moe.moe_test_set_wait_limit_ns(1_000_000)
    try:
        yield
    finally:
        moe.moe_test_set_wait_limit_ns(2_000_000_000)


@pytest.mark.parametrize("which", [0, 1, 2], ids=["flag", "mbarrier", "router-exchange"])
def test_wait_that_never_completes_times_out(short_waits, which):
    ws = moe.workspace(1, 256, 16, 64, 2, device=DEV)
    moe.moe_test_wait_never_set(ws, which)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == moe.MOE_ERR_TIMEOUT
    # the context and the workspace are usable again after re-initialisation
    moe.moe_workspace_init(ws)
    L = synth.make_layer(1, 256, 16, 64, seed=which, device=DEV)
    wdc = moe.moe_pack_w_down(L.w_down)
    check_layer_full(L, 2, 4, flags=moe.MOE_WDOWN_CHANNEL_MAJOR, w_down=wdc)
    moe.moe_layer(L.x, L.w_router, L.bias, L.w_gate, L.w_up, wdc, 2, 4,
                  torch.empty(1, 256, device=DEV), ws, flags=moe.MOE_WDOWN_CHANNEL_MAJOR)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(ws) == 0
