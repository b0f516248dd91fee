"""Python binding of the SparsePR attention library (libsparsepr.so, sm_100a).

Argument marshalling only: every step of the call runs in the CUDA kernels
behind the C ABI declared in include/sparsepr.h. PyTorch provides device
memory and streams. There is no CPU fallback: if the shared library is
missing, importing the binding's entry points raises.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libsparsepr.so")
HEADER_PATH = os.path.join(os.path.dirname(PKG_DIR), "include", "sparsepr.h")

FLAG_HARD_DROP_ONLY = 1 << 0
FLAG_RIDGE_ONLY = 1 << 1
FLAG_RBAR_UNPROJECTED = 1 << 2
FLAG_UNIFORM_WEIGHTS = 1 << 3
FLAG_TOPMASS = 1 << 4
FLAG_PROBES_UNIFORM = 1 << 5     # ablation: probes on a uniform grid of the original token order
FLAG_PROBES_RANDOM = 1 << 6      # ablation: probes drawn at random (seeded SplitMix64)
FLAG_SEMANTIC_PARTITION = 1 << 7  # ablation: k-means on the raw keys and the raw mean query
FLAG_STAGE_TIMING = 1 << 8
FLAG_TEST_STALL = 1 << 9          # test only: the dense kernel's first bounded wait runs out

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "workspace allocation failed",
          4: "CUDA error", 5: "device wait timed out", 6: "device-side check failed"}

_p = ctypes.c_void_p


class Config(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("N", ctypes.c_int),
                ("d", ctypes.c_int), ("block", ctypes.c_int), ("Gk", ctypes.c_int), ("Gq", ctypes.c_int),
                ("rK", ctypes.c_int), ("rQ", ctypes.c_int), ("M", ctypes.c_int), ("r", ctypes.c_int),
                ("kmeans_iters", ctypes.c_int), ("lam", ctypes.c_float), ("rho_exec", ctypes.c_float),
                ("flags", ctypes.c_uint), ("seed", ctypes.c_ulonglong)]


class Partition(ctypes.Structure):
    _fields_ = [(n, _p) for n in ("kgroup", "qgroup", "kperm", "koff", "qperm", "qoff", "kcent", "radial",
                                  "probe", "probe_pos", "weights", "features", "topmass")]


class Route(ctypes.Structure):
    _fields_ = [(n, _p) for n in ("rowptr", "kg", "scores", "pairs")]


class Fit(ctypes.Structure):
    _fields_ = [(n, _p) for n in ("obar", "Rbar", "A", "U", "Bm", "c0", "rank", "R", "Odense", "Osp")]


class Stats(ctypes.Structure):
    _fields_ = [("route_density", ctypes.c_double), ("rho_exec", ctypes.c_double),
                ("useful_pairs", ctypes.c_double), ("stage_ms", ctypes.c_float * 8),
                ("device_status", ctypes.c_int)]


class SparsePRError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({code})")
        self.code = code


SHARED_ROWS = 8   # rows per query group in the shared-support diagnostic (SPARSEPR_SHARED_ROWS)

_lib = None


def header_functions() -> list[str]:
    """Names of the entry points that include/sparsepr.h declares."""
    txt = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+(sparsepr_\w+)\s*\(", txt, re.M)))


def load_library() -> ctypes.CDLL:
    """Load libsparsepr.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m free_block_sparse_sparsepr_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    st = ctypes.c_int
    H = _p
    sig = {
        "sparsepr_status_string": (ctypes.c_char_p, [st]),
        "sparsepr_version": (ctypes.c_int, []),
        "sparsepr_create": (st, [ctypes.POINTER(Config), ctypes.POINTER(_p)]),
        "sparsepr_destroy": (st, [H]),
        "sparsepr_workspace_bytes": (st, [H, ctypes.POINTER(ctypes.c_size_t)]),
        "sparsepr_partition": (st, [H, _p, _p, ctypes.POINTER(Partition), _p]),
        "sparsepr_route": (st, [H, _p, ctypes.POINTER(Partition), ctypes.POINTER(Route), _p]),
        "sparsepr_permute": (st, [H, _p, _p, _p, ctypes.POINTER(Partition), _p, _p, _p, _p]),
        "sparsepr_blocksparse_attn": (st, [H, _p, _p, _p, ctypes.POINTER(Partition), ctypes.POINTER(Route),
                                           _p, _p, _p]),
        "sparsepr_probe_fit": (st, [H, _p, _p, _p, ctypes.POINTER(Partition), _p, ctypes.POINTER(Fit), _p]),
        "sparsepr_writeback": (st, [H, ctypes.POINTER(Partition), _p, ctypes.POINTER(Fit), _p, _p]),
        "sparsepr_attention": (st, [H, _p, _p, _p, _p, _p]),
        "sparsepr_attention_host": (st, [H, _p, _p, _p, _p, _p]),
        "sparsepr_dense_attn": (st, [H, _p, _p, _p, _p, _p]),
        "sparsepr_get_stats": (st, [H, ctypes.POINTER(Stats)]),
        "sparsepr_device_status": (st, [H, ctypes.POINTER(ctypes.c_int)]),
        "sparsepr_last_launch_count": (st, [H, ctypes.POINTER(ctypes.c_int)]),
        "sparsepr_set_stage_events": (st, [H, ctypes.c_void_p]),
        "sparsepr_shared_support_workspace": (st, [H, ctypes.POINTER(ctypes.c_size_t),
                                                   ctypes.POINTER(ctypes.c_size_t)]),
        "sparsepr_shared_support": (st, [H, _p, _p, ctypes.POINTER(Partition), _p, _p, _p, ctypes.c_size_t, _p]),
        "sparsepr_affine_diagnostics_workspace": (st, [H, ctypes.POINTER(ctypes.c_size_t)]),
        "sparsepr_affine_diagnostics": (st, [H, _p, _p, _p, _p, ctypes.c_size_t, _p]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _check(fn: str, code: int):
    if code != 0:
        raise SparsePRError(fn, code)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class _DevArray:
    """Zero-copy __cuda_array_interface__ view of handle-owned device memory."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"data": (ptr, False), "shape": tuple(shape), "typestr": typestr,
                                         "version": 3, "strides": None}


def device_view(ptr: int, shape, dtype):
    """torch tensor viewing `ptr` (valid until the handle overwrites or frees it)."""
    import torch

    typestr = {torch.float32: "<f4", torch.int32: "<i4", torch.int64: "<i8", torch.int16: "<i2"}[dtype]
    return torch.as_tensor(_DevArray(ptr, shape, typestr), device="cuda")


class SparsePR:
    """One configured SparsePR call on the current CUDA device (owns the workspace)."""

    def __init__(self, B, Hq, Hkv, N, d, Gk, Gq, block=128, rK=48, rQ=64, M=64, r=16, kmeans_iters=10,
                 lam=0.1, rho_exec=0.22, flags=0, seed=0):
        self.lib = load_library()
        self.cfg = Config(B, Hq, Hkv, N, d, block, Gk, Gq, rK, rQ, M, r, kmeans_iters, lam, rho_exec, flags,
                          seed)
        h = _p()
        _check("sparsepr_create", self.lib.sparsepr_create(ctypes.byref(self.cfg), ctypes.byref(h)))
        self.h = h

    @classmethod
    def from_workload(cls, w, flags=0, **kw):
        args = dict(B=w.B, Hq=w.Hq, Hkv=w.Hkv, N=w.N, d=w.d, Gk=w.Gk, Gq=w.Gq, block=w.block, rK=w.rK,
                    rQ=w.rQ, M=w.M, r=w.r, kmeans_iters=w.kmeans_iters, lam=w.lam, rho_exec=w.rho,
                    flags=flags, seed=w.seed)
        args.update(kw)
        return cls(**args)

    # ------------------------------------------------------------------ lifetime
    def close(self):
        if getattr(self, "h", None):
            self.lib.sparsepr_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    @property
    def P(self):
        return self.cfg.B * self.cfg.Hkv

    @property
    def Hp(self):
        return self.cfg.B * self.cfg.Hq

    def workspace_bytes(self) -> int:
        n = ctypes.c_size_t()
        _check("sparsepr_workspace_bytes", self.lib.sparsepr_workspace_bytes(self.h, ctypes.byref(n)))
        return n.value

    # ------------------------------------------------------------------ steps
    def partition(self, Q, K, stream=None) -> Partition:
        out = Partition()
        _check("sparsepr_partition", self.lib.sparsepr_partition(self.h, _ptr(Q), _ptr(K), ctypes.byref(out),
                                                                 _stream(stream)))
        return out

    def route(self, Q, part: Partition, stream=None) -> Route:
        out = Route()
        _check("sparsepr_route", self.lib.sparsepr_route(self.h, _ptr(Q), ctypes.byref(part), ctypes.byref(out),
                                                         _stream(stream)))
        return out

    def permute(self, Q, K, V, part: Partition, Qp=None, Kp=None, Vp=None, stream=None):
        _check("sparsepr_permute", self.lib.sparsepr_permute(self.h, _ptr(Q), _ptr(K), _ptr(V), ctypes.byref(part),
                                                             _ptr(Qp), _ptr(Kp), _ptr(Vp), _stream(stream)))

    def blocksparse_attn(self, Qp, Kp, Vp, part: Partition, route: Route, Osp, lse=None, stream=None):
        _check("sparsepr_blocksparse_attn",
               self.lib.sparsepr_blocksparse_attn(self.h, _ptr(Qp), _ptr(Kp), _ptr(Vp), ctypes.byref(part),
                                                  ctypes.byref(route), _ptr(Osp), _ptr(lse), _stream(stream)))

    def probe_fit(self, Q, K, V, part: Partition, Osp, stream=None) -> Fit:
        out = Fit()
        _check("sparsepr_probe_fit", self.lib.sparsepr_probe_fit(self.h, _ptr(Q), _ptr(K), _ptr(V),
                                                                 ctypes.byref(part), _ptr(Osp), ctypes.byref(out),
                                                                 _stream(stream)))
        return out

    def shared_support(self, Q, K, part: Partition, max_workspace_bytes: int = 8 << 30, stream=None):
        """Shared-route support diagnostic: (row_frac [B*Hkv, Gq, SHARED_ROWS], union_frac
        [B*Hkv, Gq]) as fp32 device tensors; the workspace (device memory through torch) holds
        as many KV heads' logits per pass as max_workspace_bytes allows (at least one)."""
        import torch

        lo, hi = ctypes.c_size_t(), ctypes.c_size_t()
        _check("sparsepr_shared_support_workspace",
               self.lib.sparsepr_shared_support_workspace(self.h, ctypes.byref(lo), ctypes.byref(hi)))
        nbytes = max(lo.value, min(hi.value, max_workspace_bytes))
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        P = self.cfg.B * self.cfg.Hkv
        row_frac = torch.empty((P, self.cfg.Gq, SHARED_ROWS), dtype=torch.float32, device="cuda")
        union_frac = torch.empty((P, self.cfg.Gq), dtype=torch.float32, device="cuda")
        _check("sparsepr_shared_support",
               self.lib.sparsepr_shared_support(self.h, _ptr(Q), _ptr(K), ctypes.byref(part), _ptr(row_frac),
                                                _ptr(union_frac), _ptr(ws), nbytes, _stream(stream)))
        return row_frac, union_frac

    def affine_diagnostics(self, Q, K, V, stream=None):
        """Affine-explainable fraction and affine-orthogonal energy of each query head's hard-drop
        residual (dense output minus the uncorrected sparse output), as a [B*Hq, 2] fp64 device
        tensor; runs the partition, routing, sparse attention and the dense baseline."""
        import torch

        part = self.partition(Q, K, stream)
        route = self.route(Q, part, stream)
        Qp, Kp, Vp, Osp = (torch.empty_like(t) for t in (Q, K, V, Q))
        self.permute(Q, K, V, part, Qp, Kp, Vp, stream)
        self.blocksparse_attn(Qp, Kp, Vp, part, route, Osp, None, stream)
        Os, Od = torch.empty_like(Q), torch.empty_like(Q)
        self.writeback(part, Osp, None, Os, stream)
        self.dense_attn(Q, K, V, Od, stream)
        n = ctypes.c_size_t()
        _check("sparsepr_affine_diagnostics_workspace",
               self.lib.sparsepr_affine_diagnostics_workspace(self.h, ctypes.byref(n)))
        ws = torch.empty(n.value, dtype=torch.uint8, device="cuda")
        out = torch.empty((self.cfg.B * self.cfg.Hq, 2), dtype=torch.float64, device="cuda")
        _check("sparsepr_affine_diagnostics",
               self.lib.sparsepr_affine_diagnostics(self.h, _ptr(Os), _ptr(Od), _ptr(out), _ptr(ws), n.value,
                                                    _stream(stream)))
        return out, Os, Od

    def writeback(self, part: Partition, Osp, fit: Fit | None, O, stream=None):
        _check("sparsepr_writeback", self.lib.sparsepr_writeback(self.h, ctypes.byref(part), _ptr(Osp),
                                                                 ctypes.byref(fit) if fit is not None else None,
                                                                 _ptr(O), _stream(stream)))

    def attention(self, Q, K, V, O=None, stream=None):
        if O is None:
            import torch

            O = torch.empty_like(Q)
        _check("sparsepr_attention", self.lib.sparsepr_attention(self.h, _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                                                 _stream(stream)))
        return O

    def attention_host(self, Q, K, V, O, stream=None):
        """Whole call on HOST tensors (pinned for full copy speed); synchronises the stream."""
        _check("sparsepr_attention_host", self.lib.sparsepr_attention_host(self.h, _ptr(Q), _ptr(K), _ptr(V),
                                                                           _ptr(O), _stream(stream)))
        return O

    def dense_attn(self, Q, K, V, O=None, stream=None):
        if O is None:
            import torch

            O = torch.empty_like(Q)
        _check("sparsepr_dense_attn", self.lib.sparsepr_dense_attn(self.h, _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                                                   _stream(stream)))
        return O

    # ------------------------------------------------------------------ introspection
    def stats(self) -> dict:
        s = Stats()
        _check("sparsepr_get_stats", self.lib.sparsepr_get_stats(self.h, ctypes.byref(s)))
        names = ["partition", "route", "permute", "attention", "probe_fit", "writeback", "unused", "total"]
        return {"route_density": s.route_density, "rho_exec": s.rho_exec, "useful_pairs": s.useful_pairs,
                "stage_ms": {n: s.stage_ms[i] for i, n in enumerate(names) if n != "unused"},
                "device_status": s.device_status}

    def device_status(self) -> int:
        v = ctypes.c_int()
        _check("sparsepr_device_status", self.lib.sparsepr_device_status(self.h, ctypes.byref(v)))
        return v.value

    def set_stage_events(self, events):
        """Record the next calls' 7 stage boundaries into these torch.cuda.Event objects (None: stop)."""
        if events is None:
            _check("sparsepr_set_stage_events", self.lib.sparsepr_set_stage_events(self.h, None))
            return
        assert len(events) == 7
        arr = (ctypes.c_void_p * 7)(*[e.cuda_event for e in events])
        self._events_keepalive = (events, arr)
        _check("sparsepr_set_stage_events", self.lib.sparsepr_set_stage_events(self.h, ctypes.cast(arr, ctypes.c_void_p)))

    def last_launch_count(self) -> int:
        v = ctypes.c_int()
        _check("sparsepr_last_launch_count", self.lib.sparsepr_last_launch_count(self.h, ctypes.byref(v)))
        return v.value

    # ------------------------------------------------------------------ views of handle-owned buffers
    def partition_views(self, part: Partition) -> dict:
        import torch

        c, P, N = self.cfg, self.P, self.cfg.N
        M = 0 if (c.flags & FLAG_HARD_DROP_ONLY) else c.M
        v = {"kperm": device_view(part.kperm, (P, N), torch.int32), "koff": device_view(part.koff, (P, c.Gk + 1), torch.int32),
             "qperm": device_view(part.qperm, (P, N), torch.int32), "qoff": device_view(part.qoff, (P, c.Gq + 1), torch.int32),
             "kgroup": device_view(part.kgroup, (P, N), torch.int32), "qgroup": device_view(part.qgroup, (P, N), torch.int32),
             "kcent": device_view(part.kcent, (P, c.Gk, c.d), torch.float32),
             "radial": device_view(part.radial, (P, N), torch.float32)}
        if part.features:
            DP = c.d if c.flags & FLAG_SEMANTIC_PARTITION else (c.rK + 15) // 16 * 16
            v["features"] = device_view(part.features, (P, N, DP), torch.float32)
        if part.topmass:
            v["topmass"] = device_view(part.topmass, (P, c.rK), torch.float32)
        if M:
            v["probe"] = device_view(part.probe, (P, M), torch.int32)
            v["probe_pos"] = device_view(part.probe_pos, (P, M), torch.int32)
            v["weights"] = device_view(part.weights, (P, M), torch.float32)
        return v

    def route_views(self, route: Route) -> dict:
        import torch

        c, P = self.cfg, self.P
        return {"rowptr": device_view(route.rowptr, (P, c.Gq + 1), torch.int32),
                "kg": device_view(route.kg, (P, c.Gq * c.Gk), torch.int32),
                "scores": device_view(route.scores, (P, c.Gq, c.Gk), torch.float32),
                "pairs": device_view(route.pairs, (P,), torch.int64)}

    def fit_views(self, fit: Fit) -> dict:
        import torch

        c, Hp = self.cfg, self.Hp
        return {"obar": device_view(fit.obar, (Hp, c.d), torch.float32),
                "Rbar": device_view(fit.Rbar, (Hp, c.d), torch.float32),
                "A": device_view(fit.A, (Hp, c.d, c.d), torch.float32),
                "U": device_view(fit.U, (Hp, c.d, c.r), torch.float32),
                "Bm": device_view(fit.Bm, (Hp, c.r, c.d), torch.float32),
                "c0": device_view(fit.c0, (Hp, c.r), torch.float32),
                "rank": device_view(fit.rank, (Hp,), torch.int32),
                "R": device_view(fit.R, (Hp, c.M, c.d), torch.float32),
                "Odense": device_view(fit.Odense, (Hp, c.M, c.d), torch.float32),
                "Osp": device_view(fit.Osp, (Hp, c.M, c.d), torch.float32)}


def partition_from_tensors(t: dict) -> Partition:
    """Partition struct pointing at caller-owned device tensors (for handing a partition in)."""
    p = Partition()
    for name in ("kgroup", "qgroup", "kperm", "koff", "qperm", "qoff", "kcent", "radial", "probe", "probe_pos",
                 "weights", "features"):
        if name in t and t[name] is not None:
            setattr(p, name, t[name].data_ptr())
    return p


def route_from_tensors(t: dict) -> Route:
    r = Route()
    for name in ("rowptr", "kg", "scores", "pairs"):
        if name in t and t[name] is not None:
            setattr(r, name, t[name].data_ptr())
    return r


__all__ = ["SparsePR", "SparsePRError", "Config", "Partition", "Route", "Fit", "Stats", "load_library",
           "header_functions", "partition_from_tensors", "route_from_tensors", "device_view", "LIB_PATH",
           "FLAG_HARD_DROP_ONLY", "FLAG_RIDGE_ONLY", "FLAG_RBAR_UNPROJECTED", "FLAG_UNIFORM_WEIGHTS", "FLAG_TOPMASS",
           "FLAG_PROBES_UNIFORM", "FLAG_PROBES_RANDOM", "FLAG_SEMANTIC_PARTITION", "SHARED_ROWS",
           "FLAG_STAGE_TIMING"]
