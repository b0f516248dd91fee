"""Full-size parity on the 720p (N=118800, 24 heads) and GQA world-model (N=75600, 32 query
heads on 8 KV heads) calls, in the launch configuration bench.py times.

The whole call runs on the GPU once through `sparsepr_attention` and once stage by stage (the
same kernels; the outputs must agree bit for bit), and its intermediates are read back. The
oracle then checks, on two KV heads each, what it can afford at this size:
  - response features at sampled keys (brute-force dot products) and key-group means at sampled
    groups (means of the raw keys);
  - the group-major orders and offsets (bit-exact against a stable sort of the GPU's labels);
  - the cell scores (the oracle's formula on the GPU's partition) and the selected cells (the
    oracle's selection rule on the GPU's scores: identical cells);
  - the sparse output O_s and the final corrected output O at sampled query rows and at every
    probe row, with the GPU's partition and route handed to the oracle (its own dense probe
    rows, residuals, ridge fit and subspace): max-abs 2e-2, mean-abs 2e-3;
  - probe rows of O equal the GPU's dense rows (rounded to bf16) exactly.
"""
import pytest

torch = pytest.importorskip("torch")

import free_block_sparse_sparsepr_b200 as spr  # noqa: E402
from synthetic import get_workload, video_qkv  # noqa: E402
from gpu_helpers import sampled_call_parity  # noqa: E402

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    spr.load_library()


@pytest.mark.parametrize("name", ["hunyuan720p_n118800", "worldmodel_gqa_n75600"])
def test_full_size_sampled(name):
    w = get_workload(name)
    sampled_call_parity(w, *video_qkv(w))
