"""moe_permute_noalloc, the permutation entry point that needs no workspace.

Some callers cannot give the library any scratch memory: plugin hosts that hand a custom
operation only its input and output buffers, or processes whose device memory is
already held by another framework's caching allocator.  For them the library sorts with
its own fixed device array.  These tests check, through the C interface, that it
returns exactly what the oracle's permutation and moe_permute (with a workspace) return,
on two calls in a row with different routing, so nothing left in the shared array by
one call leaks into the next.
This file is collected last so that a run stopping at the first failure has already run
every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_ffn_05_b200 as mf
import oracle
from tests.gpu_util import run_permute, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    mf.lib()


def _ids(T, k, E, seed):
    rng = np.random.default_rng(seed)
    return (rng.zipf(1.3, size=(T, k)) % E).astype(np.int32)


def _noalloc(cfg, idx):
    T, k = idx.shape
    n = T * k
    out = {
        "offsets": torch.full((cfg.num_experts + 1,), -7, dtype=torch.int32, device="cuda"),
        "sorted_src": torch.full((n,), -7, dtype=torch.int32, device="cuda"),
        "inv_pos": torch.full((n,), -7, dtype=torch.int32, device="cuda"),
    }
    mf.moe_permute_noalloc(cfg, idx, out["offsets"], out["sorted_src"], out["inv_pos"])
    torch.cuda.synchronize()
    return out


# More than 2048 pairs take the multi-block sort, which uses the scratch array: 2049
# pairs is the first such size, (2048, 8) and (40000, 16) larger ones; (8, 8) takes the
# single-block sort.
@pytest.mark.parametrize("T,k,E", [(2048, 8, 128), (8, 8, 128), (2049, 1, 16), (40000, 16, 256)])
def test_noalloc_equals_oracle_and_workspace_permutation_twice(T, k, E):
    cfg = mf.Config(512, E, k, 128, 128)
    for seed in (1, 2):  # two calls in a row, different routing
        ids = _ids(T, k, E, seed)
        idx = to_dev(ids, torch.int32)
        got = _noalloc(cfg, idx)
        want = dict(zip(("offsets", "sorted_src", "inv_pos"), oracle.permute(ids, E)))
        ref = run_permute(cfg, idx)
        for name in ("offsets", "sorted_src", "inv_pos"):
            assert np.array_equal(got[name].cpu().numpy(), want[name]), (name, seed, "oracle")
            assert torch.equal(got[name], ref[name][: got[name].numel()]), (name, seed)


def test_noalloc_rejects_batches_beyond_its_scratch():
    cfg = mf.Config(512, 128, 8, 128, 128)
    T = mf.PERMUTE_NOALLOC_MAX_PAIRS // 8 + 1
    fake = 1 << 20  # never dereferenced: the size check comes first
    st = mf.lib().moe_permute_noalloc(ctypes.byref(cfg.c()), T, fake, fake, fake, fake, None)
    assert st == mf.MOE_ERR_UNSUPPORTED
