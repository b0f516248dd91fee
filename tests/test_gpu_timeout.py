"""A bounded device-side wait that runs out, without a fault or a hang.

Every wait of the tensor-core kernels on an mbarrier gives up after about two seconds of SM
clock, raises the CTA's abort flag and lets the other warps leave their waits; the CTA then
returns with its TMEM freed, and the launch records SPARSEPR_ERR_TIMEOUT in the handle's device
status word. The test-only flag SPARSEPR_FLAG_TEST_STALL makes the dense-attention kernel's
producer issue no load at all, so the MMA warp's first wait (for the query tile) can never
complete: no copy and no MMA is in flight when the CTAs give up. The host must read the timeout
from the status word, and the next call on a fresh handle must run clean and correct.
"""
import time

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import free_block_sparse_sparsepr_b200 as spr  # noqa: E402
from synthetic import Workload  # noqa: E402
from gpu_helpers import assert_close, bf16_to_f64, inputs  # noqa: E402

pytestmark = pytest.mark.gpu

W = Workload("stall_n640", B=1, Hq=2, Hkv=2, T=2, Hg=16, Wg=20, d=128, Gk=8, Gq=8, block=128, rho=0.3, M=32,
             r=8)


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    spr.load_library()


def test_bounded_wait_runs_out_and_reports_timeout():
    (Q, K, V), (q, k, v) = inputs(W)
    with spr.SparsePR.from_workload(W, flags=spr.FLAG_TEST_STALL) as h:
        O = torch.full_like(q, float("nan"))
        t0 = time.perf_counter()
        h.dense_attn(q, k, v, O)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
        assert h.device_status() == 5, "the run-out wait must be reported as SPARSEPR_ERR_TIMEOUT"
        assert h.device_status() == 0, "reading the status clears it"
    assert elapsed < 60.0, elapsed
    # a CTA that gave up writes its rows as zeros; one that started after the status word was set
    # returns at once and leaves its rows untouched (NaN here): never anything else
    Of = O.float()
    assert torch.all((Of == 0) | torch.isnan(Of)), "rows of CTAs that gave up must be zero or untouched"
    # a fresh handle runs clean and correct afterwards
    with spr.SparsePR.from_workload(W) as h:
        Od = h.dense_attn(q, k, v)
        O2 = h.attention(q, k, v)
        torch.cuda.synchronize()
        assert h.device_status() == 0
    assert_close(bf16_to_f64(Od), oracle.dense_attention(Q, K, V), "dense attention after the timeout")
    assert torch.isfinite(O2.float()).all()
