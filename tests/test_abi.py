"""The C ABI library loads, exports every entry point its header declares, and
rejects bad arguments before touching the GPU (runs without a GPU)."""
import ctypes
import os

import pytest

import free_block_sparse_sparsepr_b200 as spr


def test_library_exists_and_loads():
    assert os.path.exists(spr.LIB_PATH), "build the library first (python -m free_block_sparse_sparsepr_b200.build)"
    lib = spr.load_library()
    assert lib.sparsepr_version() >= 100


def test_every_declared_symbol_is_exported():
    lib = spr.load_library()
    names = spr.header_functions()
    assert len(names) >= 17
    for n in ["sparsepr_create", "sparsepr_partition", "sparsepr_route", "sparsepr_blocksparse_attn",
              "sparsepr_probe_fit", "sparsepr_attention", "sparsepr_dense_attn", "sparsepr_writeback",
              "sparsepr_permute"]:
        assert n in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/sparsepr.h but not exported"


def test_status_strings():
    lib = spr.load_library()
    for code, text in spr.STATUS.items():
        assert lib.sparsepr_status_string(code).decode() == text
    assert lib.sparsepr_status_string(99).decode() == "unknown status"


def _cfg(**kw):
    base = dict(B=1, Hq=2, Hkv=2, N=1024, d=64, block=64, Gk=16, Gq=16, rK=48, rQ=64, M=64, r=16,
                kmeans_iters=10, lam=0.1, rho_exec=0.25, flags=0, seed=0)
    base.update(kw)
    return spr.Config(*[base[f] for f, _ in spr.Config._fields_])


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=3, Hkv=2), 1), (dict(N=0), 1), (dict(d=96), 2), (dict(block=32), 1),
    (dict(Gk=0), 1), (dict(Gq=2000), 1), (dict(Gk=1025, N=4096), 2), (dict(rK=65), 1), (dict(rQ=0), 1),
    (dict(M=0), 1), (dict(M=65), 2), (dict(r=0), 1), (dict(r=65), 1), (dict(lam=0.0), 1),
    (dict(rho_exec=0.0), 1), (dict(rho_exec=float("nan")), 1), (dict(kmeans_iters=-1), 1),
    (dict(flags=1 << 20), 1),
    (dict(flags=spr.FLAG_PROBES_UNIFORM | spr.FLAG_PROBES_RANDOM), 1),      # one probe sampler at most
    (dict(flags=spr.FLAG_SEMANTIC_PARTITION | spr.FLAG_TOPMASS), 1),        # no sampled responses to measure
])
def test_create_rejects_bad_configs_without_gpu(kw, code):
    lib = spr.load_library()
    h = ctypes.c_void_p()
    assert lib.sparsepr_create(ctypes.byref(_cfg(**kw)), ctypes.byref(h)) == code
    assert not h.value


def test_diagnostic_entry_points_reject_null_arguments():
    lib = spr.load_library()
    n = ctypes.c_size_t()
    assert lib.sparsepr_shared_support_workspace(None, ctypes.byref(n), None) == 1
    assert lib.sparsepr_shared_support(None, None, None, None, None, None, None, 0, None) == 1
    assert lib.sparsepr_affine_diagnostics_workspace(None, ctypes.byref(n)) == 1
    assert lib.sparsepr_affine_diagnostics(None, None, None, None, None, 0, None) == 1
    assert lib.sparsepr_attention_host(None, None, None, None, None, None) == 1


def test_null_handle_and_pointer_checks():
    lib = spr.load_library()
    assert lib.sparsepr_create(None, None) == 1
    assert lib.sparsepr_destroy(None) == 0
    assert lib.sparsepr_attention(None, None, None, None, None, None) == 1
    assert lib.sparsepr_dense_attn(None, None, None, None, None, None) == 1
    assert lib.sparsepr_get_stats(None, None) == 1
    p = spr.Partition()
    r = spr.Route()
    assert lib.sparsepr_route(None, None, ctypes.byref(p), ctypes.byref(r), None) == 1
    assert lib.sparsepr_blocksparse_attn(None, None, None, None, ctypes.byref(p), ctypes.byref(r), None, None,
                                         None) == 1
