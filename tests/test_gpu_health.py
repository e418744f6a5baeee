"""The failure path of the bounded device waits, exercised without faulting the GPU.

Every kernel of the library bounds its waits; one that runs out records
MOE_ERR_DEVICE_TIMEOUT in the workspace's status word and returns.  moe_wait_selftest
runs such a wait on a barrier that nothing completes (a flag nobody sets), with a short
bound; the test checks that the timeout is reported, that the report is cleared once
read, and that the context still computes the block correctly afterwards.
"""
import time

import pytest
import torch

import mixture_experts_ffn_05_b200 as mf
import synth
from tests import cases
from tests.gpu_util import bf16_np, config, device_layer, oracle_block, run_block

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    mf.lib()


def test_wait_timeout_is_reported_cleared_and_recoverable():
    c = cases.make_case(synth.TINY, seed=1234)
    cfg = config(c.shape)
    ws = mf.workspace(cfg, c.shape.T)
    assert mf.moe_check_device_status(ws) == mf.MOE_OK

    t0 = time.perf_counter()
    mf.moe_wait_selftest(ws, 2_000_000)  # 2 ms bound
    st = mf.moe_check_device_status(ws)  # waits for the stream
    dt = time.perf_counter() - t0
    assert st == mf.MOE_ERR_DEVICE_TIMEOUT
    assert 0.002 <= dt < 5.0, dt
    assert mf.moe_check_device_status(ws) == mf.MOE_OK  # read once, then cleared

    # the context is still usable and the workspace still serves the block
    out, moe = run_block(cfg, c, device_layer(c), ws=ws)
    o = oracle_block(c)
    cases.check_bar(bf16_np(out), o["out"], cases.FRAC_BF16, "out after a timeout")
    cases.check_bar(bf16_np(moe), o["moe"], cases.FRAC_BF16, "moe_out after a timeout")
