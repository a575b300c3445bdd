"""Python face of the fp64 CPU oracle for dynamic bifocal RoPE attention.

TEST INFRASTRUCTURE ONLY: the checker the CUDA library is compared against.
Only tests/, ``__graft_entry__.smoke()`` and bench.py's CPU-baseline leg may
import this package.  The library (``long_context_attention_bifocal_b200``)
never imports it and has no CPU fallback.

Every function here marshals numpy arrays into ``libjloracle.so`` (built from
``jl_oracle.c``), which evaluates the per-pair definition in double precision;
that file's header states the definition and the passages it follows.
"""
import ctypes

import numpy as np

from . import build as _build

F32, BF16, F64 = 0, 1, 2


def _as_input(x):
    """(contiguous array, dtype code) for fp32, bf16-bits (uint16) or fp64."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    if x.dtype == np.float64:
        return x, F64
    raise TypeError("oracle inputs must be float32, uint16 (bf16 bits) or "
                    f"float64, got {x.dtype}")


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """The oracle functions bound to one build of jl_oracle.c."""

    def __init__(self, path: str):
        L = ctypes.CDLL(path)
        i, d, p, ll = ctypes.c_int, ctypes.c_double, ctypes.c_void_p, ctypes.c_longlong
        L.jlo_group_size.restype = ll
        L.jlo_group_size.argtypes = [ll, ll]
        L.jlo_remap.restype = ll
        L.jlo_remap.argtypes = [ll, ll]
        L.jlo_theta.restype = d
        L.jlo_theta.argtypes = [i, i, d]
        L.jlo_rope.restype = None
        L.jlo_rope.argtypes = [p, p, i, d, d]
        L.jlo_bifocal_rows.restype = i
        L.jlo_bifocal_rows.argtypes = [p, p, p, i, i, i, i, i, i, i, i, d, d,
                                       i, p, p, p, p, p]
        L.jlo_bifocal_decode.restype = i
        L.jlo_bifocal_decode.argtypes = [p, p, p, i, i, i, i, i, i, i, i, i,
                                         d, d, p, p]
        L.jlo_num_threads.restype = i
        L.jlo_num_threads.argtypes = []
        self.lib = L
        self.path = path

    def group_size(self, L: int, w_pretrained: int) -> int:
        return int(self.lib.jlo_group_size(L, w_pretrained))

    def remap(self, x: int, G: int) -> int:
        return int(self.lib.jlo_remap(x, G))

    def theta(self, i: int, D: int, base: float) -> float:
        return float(self.lib.jlo_theta(i, D, base))

    def rope(self, x, pos: float, base: float) -> np.ndarray:
        """R(pos) x for one vector of even length D (rotate-half pairs)."""
        x = np.ascontiguousarray(x, dtype=np.float64)
        y = np.empty_like(x)
        self.lib.jlo_rope(_ptr(x), _ptr(y), x.shape[-1], float(pos), float(base))
        return y

    def num_threads(self) -> int:
        return int(self.lib.jlo_num_threads())

    def bifocal_rows(self, q, k, v, rows_b, rows_q, rows_h, *, w_local,
                     w_pretrained, rope_base, scale=0.0):
        """Per-pair bifocal attention for selected rows.

        q [B,L,Hq,D], k/v [B,L,Hkv,D] (one dtype: float32, bf16 bits as uint16,
        or float64).  Returns (out [n,D] fp64, lse [n] fp64) for the rows
        (rows_b[i], rows_q[i], rows_h[i]).
        """
        q, dt = _as_input(q)
        k, dk = _as_input(k)
        v, dv = _as_input(v)
        if not (dt == dk == dv):
            raise TypeError("q, k, v must share a dtype")
        B, L, Hq, D = q.shape
        Hkv = k.shape[2]
        rb = np.ascontiguousarray(rows_b, dtype=np.int32)
        rq = np.ascontiguousarray(rows_q, dtype=np.int32)
        rh = np.ascontiguousarray(rows_h, dtype=np.int32)
        n = rb.shape[0]
        out = np.empty((n, D), dtype=np.float64)
        lse = np.empty((n,), dtype=np.float64)
        rc = self.lib.jlo_bifocal_rows(
            _ptr(q), _ptr(k), _ptr(v), dt, B, L, Hq, Hkv, D, int(w_local),
            int(w_pretrained), float(rope_base), float(scale), n, _ptr(rb),
            _ptr(rq), _ptr(rh), _ptr(out), _ptr(lse))
        if rc != 0:
            raise ValueError(f"jlo_bifocal_rows rejected its arguments (code {rc})")
        return out, lse

    def bifocal_all_rows(self, q, k, v, **kw):
        """Every (b, q, h) row; returns out [B,L,Hq,D] and lse [B,Hq,L]."""
        B, L, Hq, D = q.shape
        bb, qq, hh = np.meshgrid(np.arange(B), np.arange(L), np.arange(Hq),
                                 indexing="ij")
        out, lse = self.bifocal_rows(q, k, v, bb.ravel(), qq.ravel(), hh.ravel(), **kw)
        return (out.reshape(B, L, Hq, D),
                lse.reshape(B, L, Hq).transpose(0, 2, 1).copy())

    def bifocal_decode(self, q_new, k_cache, v_cache, pos, *, w_local,
                       w_pretrained, rope_base, scale=0.0):
        """Decode at position pos over caches [B,S,Hkv,D] holding keys rotated
        at their original positions.  Returns (out [B,Hq,D], lse [B,Hq])."""
        q_new, dt = _as_input(q_new)
        k_cache, dk = _as_input(k_cache)
        v_cache, dv = _as_input(v_cache)
        if not (dt == dk == dv):
            raise TypeError("q_new, k_cache, v_cache must share a dtype")
        B, Hq, D = q_new.shape
        S, Hkv = k_cache.shape[1], k_cache.shape[2]
        out = np.empty((B, Hq, D), dtype=np.float64)
        lse = np.empty((B, Hq), dtype=np.float64)
        rc = self.lib.jlo_bifocal_decode(
            _ptr(q_new), _ptr(k_cache), _ptr(v_cache), dt, B, Hq, Hkv, D,
            int(pos), S, int(w_local), int(w_pretrained), float(rope_base),
            float(scale), _ptr(out), _ptr(lse))
        if rc != 0:
            raise ValueError(f"jlo_bifocal_decode rejected its arguments (code {rc})")
        return out, lse


_default = None


def default() -> Oracle:
    """The oracle built from oracle/jl_oracle.c (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def __getattr__(name):
    # Module-level access (oracle.bifocal_rows, ...) goes to the default build.
    if name in ("group_size", "remap", "theta", "rope", "num_threads",
                "bifocal_rows", "bifocal_all_rows", "bifocal_decode"):
        return getattr(default(), name)
    raise AttributeError(name)
