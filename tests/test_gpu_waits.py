"""The kernels' bounded waits, made to run out on the GPU without a fault.

moe_selftest_wait_timeout has one warp wait, with the wait routine the FFN
kernels use, on a shared-memory barrier that nothing arrives at.  The wait
gives up after its budget, records MOE_DEV_TIMEOUT_FULL in the workspace's
status word and the kernel returns; the host reads the code through
moe_workspace_status, and the context keeps working (a layer call after it
matches the oracle).
"""
import numpy as np
import pytest
import torch

import synthetic as S
from helpers import dev_x
from test_gpu_parity import _check_layer, _layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda(moe):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_bounded_wait_runs_out_and_is_reported(moe):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert moe.workspace_status(ws) == (0, moe.DEV_OK)
    moe.selftest_wait_timeout(ws, 2_000_000)          # about a millisecond of SM clock
    st, code = moe.workspace_status(ws, clear=False)
    assert code == moe.DEV_TIMEOUT_FULL
    assert st == 6                                     # MOE_ERR_TIMEOUT
    # still set until cleared, then clear
    assert moe.workspace_status(ws, clear=True)[1] == moe.DEV_TIMEOUT_FULL
    assert moe.workspace_status(ws) == (0, moe.DEV_OK)
    # the first recorded code stays: a second timeout does not overwrite it
    moe.selftest_wait_timeout(ws, 1_000_000)
    moe.selftest_wait_timeout(ws, 1_000_000)
    assert moe.workspace_status(ws)[1] == moe.DEV_TIMEOUT_FULL


def test_context_is_usable_after_a_timeout(moe):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    moe.selftest_wait_timeout(ws, 2_000_000)
    assert moe.workspace_status(ws)[1] == moe.DEV_TIMEOUT_FULL
    cfg = S.LayerConfig("after", T=4, D=512, E=8, k=2, F=256, qtype="q4_0", x_dtype="bf16",
                        y_dtype="f32", router_std=0.05, seed=91)
    L = S.make_layer(cfg)
    lay = _layer(moe, L)
    y = lay.forward(dev_x(L))
    torch.cuda.synchronize()
    _check_layer(moe, L, y, lay.ids, 4)
    assert moe.workspace_status(lay.ws) == (0, moe.DEV_OK)
