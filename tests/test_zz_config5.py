"""Parity on the denoising-step configuration: the density x length sweep and one stack layer.

The sweep covers target densities rho in {10, 15, 22, 30, 50, 100}% and lengths N in {8192,
32760, 75600, 118800} at 24 heads, d=128 (grids 8x32x32, 13x45x56, 21x45x80, 33x45x80). The
low end (rho = 10%, where the route budget rho - M/N is smallest) and rho = 100% (every cell, no
budget) are routing corners the other configurations do not reach ([execution]: rho_exec = route
density + M/N, whole cells indivisible). The stack's layers draw their locality from U[0.4, 1.2];
the layer at 0.4 has the densest rows.

  - N = 8192 at every rho, on a subset of two heads: the oracle runs the whole call; the GPU runs
    steps 3-7 with the oracle's partition handed in (its route on the GPU's scores must be the
    oracle's selection rule applied to them, identical cells) and steps 4-7 with the oracle's
    partition and route handed in: O_s and O element by element within max-abs 2e-2, mean-abs
    2e-3;
  - N = 32760 at rho = 10% and 100%, and one 720p stack layer at locality 0.4, all 24 heads in
    the launch configuration the benchmark times: the oracle checks sampled rows and every probe
    row of two KV heads with the GPU's partition and route handed to it.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import free_block_sparse_sparsepr_b200 as spr  # noqa: E402
from synthetic import bf16_bits_to_f64, get_workload, video_qkv  # noqa: E402
from synthetic.workloads import SWEEP_RHOS, sweep_workload  # noqa: E402
from gpu_helpers import (assert_close, bf16_to_f64, partition_tensors, route_tensors,  # noqa: E402
                         sampled_call_parity, selected_from_csr, to_group_major)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    spr.load_library()


@pytest.mark.parametrize("rho", SWEEP_RHOS)
def test_sweep_n8192_every_density(rho):
    w = sweep_workload(8192, rho).replace(Hq=2, Hkv=2)
    Qb, Kb, Vb = video_qkv(w)
    Q, K, V = (bf16_bits_to_f64(x) for x in (Qb, Kb, Vb))
    q, k, v = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda() for x in (Qb, Kb, Vb))
    res = oracle.sparsepr_attention(Q, K, V, w)
    pt = partition_tensors(res, w)
    part = spr.partition_from_tensors(pt)
    with spr.SparsePR.from_workload(w) as h:
        # (3) routing on the oracle's partition: the oracle's rule on the GPU's scores
        route_gpu = h.route(q, part)
        torch.cuda.synchronize()
        rv = {n: t.cpu().numpy() for n, t in h.route_views(route_gpu).items()}
        for z in range(w.B * w.Hkv):
            po = res["partitions"][(z // w.Hkv, z % w.Hkv)]
            ro = res["routes"][(z // w.Hkv, z % w.Hkv)]
            S = rv["scores"][z]
            nz = ro.scores > 0
            assert (np.abs(S - ro.scores) / np.maximum(ro.scores, 1e-30))[nz].max() < 2e-4
            sel_ref, _, pairs_ref = oracle.select_cells(S, np.diff(po.qoff), np.diff(po.koff), w.N, w.M, w.rho)
            sel = selected_from_csr(rv["rowptr"][z], rv["kg"][z], w.Gq, w.Gk)
            assert np.array_equal(sel, sel_ref)
            assert int(rv["pairs"][z]) == int(pairs_ref)
            if rho >= 1.0:
                assert sel.sum() == ((np.diff(po.qoff)[:, None] > 0) & (np.diff(po.koff)[None, :] > 0)).sum()
        # (4-7) with the oracle's partition and route handed in
        route = spr.route_from_tensors(route_tensors(res, w))
        Qp, Kp, Vp, Osp, O = (torch.empty_like(t) for t in (q, k, v, q, q))
        h.permute(q, k, v, part, Qp, Kp, Vp)
        h.blocksparse_attn(Qp, Kp, Vp, part, route, Osp)
        fit = h.probe_fit(q, k, v, part, Osp)
        h.writeback(part, Osp, fit, O)
        torch.cuda.synchronize()
        assert h.device_status() == 0
    assert_close(bf16_to_f64(Osp), to_group_major(res["O_sparse"], res, w), f"sparse output rho={rho}")
    assert_close(bf16_to_f64(O), res["O"], f"corrected output rho={rho}")
    if rho >= 1.0:
        D = oracle.dense_attention(Q, K, V, rows=np.arange(0, w.N, 7))
        assert_close(bf16_to_f64(O)[:, :, ::7], D, "rho=1 output vs dense attention")


@pytest.mark.slow
@pytest.mark.parametrize("rho", [0.10, 1.00])
def test_sweep_n32760_extremes_sampled(rho):
    w = sweep_workload(32760, rho)
    sampled_call_parity(w, *video_qkv(w))


@pytest.mark.slow
def test_stack_layer_locality_0p4_sampled():
    w = get_workload("hunyuan720p_n118800")
    sampled_call_parity(w, *video_qkv(w, layer=1, locality=0.4))
