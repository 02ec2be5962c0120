"""GPU check of calibatt_block_energy_noalloc, the block-energy entry point for
callers that may not allocate device memory (its scratch is built into the
library).  Its energies must equal, bit for bit, those of
calibatt_block_energy, which runs the same kernels with a caller workspace,
on two calls in a row (the built-in scratch is reused and keeps the previous
call's contents).  Collected last on purpose."""

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C(calibatt_lib):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return calibatt_lib


def _with_workspace(C, q, k, block):
    b, n, h, _ = q.shape
    nb = -(-n // block)
    e = torch.full((b, h, nb, nb), float("nan"), device=q.device)
    ws = torch.empty(C.calibatt_block_energy_workspace_size(q) // 4, device=q.device)
    C.calibatt_block_energy(q, k, e, ws, block)
    return e


def _no_alloc(C, q, k, block):
    b, n, h, _ = q.shape
    nb = -(-n // block)
    e = torch.full((b, h, nb, nb), float("nan"), device=q.device)
    C.calibatt_block_energy_noalloc(q, k, e, block)
    return e


def test_noalloc_energy_matches_workspace_entry_point_twice(C):
    cases = [(30, 1, 300, 2, 128, "bf16", 128), (31, 2, 256, 3, 64, "fp32", 64)]
    for seed, b, n, h, d, dtype, block in cases:   # two calls in a row, different shapes
        q, k, _ = W.make_qkv(seed, b, n, h, d, dtype, 1.0, "cuda")
        ref = _with_workspace(C, q, k, block)
        got = _no_alloc(C, q, k, block)
        torch.cuda.synchronize()
        assert C.device_status() == 0
        assert torch.isfinite(got).all()
        # the same kernels on the same inputs: only the scratch differs, so any
        # difference at all is a scratch fault
        assert torch.equal(got, ref)
        np.testing.assert_allclose(got.sum(-1).cpu().numpy(), 1.0, atol=1e-5)


def test_noalloc_energy_rejects_problems_beyond_its_scratch(C):
    q = torch.zeros((1, 1 << 17, 9, 64), dtype=torch.bfloat16, device="cuda")   # 9 * 2^17 rows > 2^20
    e = torch.zeros(1, device="cuda")
    with pytest.raises(C.CalibattError) as err:
        C.calibatt_block_energy_noalloc(q, q, e, 128)
    assert err.value.status == C.ERR_INVALID_ARG
    assert "exceeds the built-in scratch" in str(err.value)
