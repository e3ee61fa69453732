"""PaTH attention oracle: plain fp64 CPU reference (test infrastructure only).

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA library never calls it, and it
shares no code with the CUDA library: the arithmetic lives in
``path_oracle.c`` (built here with gcc + OpenMP); this file only marshals
arrays into fp64 and calls it.

Definitions it follows (all from the pages' problem statement):
- logit ``z_ij = scale * q_i^T H_i ... H_{j+1} k_j + c_i - c_j`` for j <= i
  ("PaTH Attention", gist.science summary section 2, logit equation;
  Paper-Notes "整体框架" / "PaTH-FoX 扩展");
- ``H_s = I - beta_s w_s w_s^T`` (gist.science section 2; Paper-Notes "关键设计");
- forward by the in-place key-cache update (Paper-Notes "训练策略",
  inference paragraph), backward by the per-query adjoint chain;
- decode (optionally with the gate's per-key bias carried in place) and the
  cache a prefill leaves behind, by the same in-place update.

Parity is pinned by ``tests/test_oracle_pins.py`` against explicit matrix
products, a library attention routine, closed forms, finite differences and
autograd of an explicit-matrix formulation.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "path_oracle.c")
_LIB = os.path.join(_HERE, "libpath_oracle.so")
_lock = threading.Lock()
_default = None


def compile_source(src: str, out: str) -> str:
    """gcc -O2 -fopenmp build of one oracle source file into a shared library."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(
        ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", src, "-o", tmp, "-lm"]
    )
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile path_oracle.c into libpath_oracle.so if it is missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(SOURCE):
        compile_source(SOURCE, _LIB)
    return _LIB


def _f64(x):
    """Any array-like (numpy, torch CPU tensor of any float dtype) -> C-contiguous fp64."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: upcast exactly (bf16/fp32 -> fp64)
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _dims(q):
    if q.ndim != 4:
        raise ValueError("q must be [B,H,L,d]")
    return q.shape


class Oracle:
    """ctypes handle on one build of the oracle library."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        dp = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        d = ctypes.c_double
        lib.path_oracle_fwd.argtypes = [dp, dp, dp, dp, dp, dp, d, i, i, i, i, dp, dp]
        lib.path_oracle_scores.argtypes = [dp, dp, dp, dp, dp, d, i, i, i, i, dp]
        lib.path_oracle_bwd.argtypes = [dp, dp, dp, dp, dp, dp, d, i, i, i, i,
                                        dp, dp, dp, dp, dp, dp, dp]
        lib.path_oracle_decode_step.argtypes = [dp, dp, dp, dp, dp, d, i, i, i, i, i, i,
                                                dp, dp, dp]
        lib.path_oracle_decode_step_gated.argtypes = [dp, dp, dp, dp, dp, dp, d, i, i, i, i, i,
                                                      i, dp, dp, dp, dp]
        lib.path_oracle_prefill_cache.argtypes = [dp, dp, dp, dp, dp, i, i, i, i, i, dp, dp, dp]
        lib.path_oracle_round_bf16.argtypes = [d]
        lib.path_oracle_round_bf16.restype = d
        for f in (lib.path_oracle_fwd, lib.path_oracle_scores, lib.path_oracle_bwd,
                  lib.path_oracle_decode_step, lib.path_oracle_decode_step_gated,
                  lib.path_oracle_prefill_cache):
            f.restype = ctypes.c_int
        self.lib = lib
        self.path = lib_path

    def fwd(self, q, k, v, w, beta, log_f=None, scale=None):
        """Returns (out [B,H,L,d], lse [B,H,L]) in fp64."""
        q, k, v, w, beta, log_f = map(_f64, (q, k, v, w, beta, log_f))
        B, H, L, d = _dims(q)
        if scale is None:
            scale = d ** -0.5
        out = np.empty((B, H, L, d))
        lse = np.empty((B, H, L))
        rc = self.lib.path_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(w), _ptr(beta),
                                      _ptr(log_f), float(scale), B, H, L, d, _ptr(out), _ptr(lse))
        if rc:
            raise ValueError("oracle fwd: invalid arguments")
        return out, lse

    def scores(self, q, k, w, beta, log_f=None, scale=None):
        """Full logit matrices z [B,H,L,L] (-inf above the diagonal); tiny sizes only."""
        q, k, w, beta, log_f = map(_f64, (q, k, w, beta, log_f))
        B, H, L, d = _dims(q)
        if scale is None:
            scale = d ** -0.5
        z = np.empty((B, H, L, L))
        rc = self.lib.path_oracle_scores(_ptr(q), _ptr(k), _ptr(w), _ptr(beta), _ptr(log_f),
                                         float(scale), B, H, L, d, _ptr(z))
        if rc:
            raise ValueError("oracle scores: invalid arguments")
        return z

    def bwd(self, q, k, v, w, beta, dout, log_f=None, scale=None):
        """Gradients of sum(out * dout): dict dq, dk, dv, dw, dbeta[, dlog_f] (fp64)."""
        q, k, v, w, beta, log_f, dout = map(_f64, (q, k, v, w, beta, log_f, dout))
        B, H, L, d = _dims(q)
        if scale is None:
            scale = d ** -0.5
        g = {n: np.empty((B, H, L, d)) for n in ("dq", "dk", "dv", "dw")}
        g["dbeta"] = np.empty((B, H, L))
        dlf = np.empty((B, H, L)) if log_f is not None else None
        rc = self.lib.path_oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(w), _ptr(beta),
                                      _ptr(log_f), float(scale), B, H, L, d, _ptr(dout),
                                      _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dw"]),
                                      _ptr(g["dbeta"]), _ptr(dlf))
        if rc:
            raise ValueError("oracle bwd: invalid arguments")
        if dlf is not None:
            g["dlog_f"] = dlf
        return g

    def decode_step(self, q, k_new, v_new, w, beta, k_cache, v_cache, n_cached, scale=None,
                    round_bf16=False, log_f=None, g_cache=None):
        """One decode step; k_cache/v_cache (fp64 numpy [B,H,cap,d]) are updated IN PLACE.

        With the forget gate, log_f [B,H] is log f of the new position and
        g_cache (fp64 numpy [B,H,cap]) the cached gate biases, also updated in
        place. Returns out [B,H,d] (fp64)."""
        q, k_new, v_new, w, beta, log_f = map(_f64, (q, k_new, v_new, w, beta, log_f))
        caches = (k_cache, v_cache) + ((g_cache,) if log_f is not None else ())
        for c in caches:
            if not (isinstance(c, np.ndarray) and c.dtype == np.float64 and c.flags.c_contiguous):
                raise TypeError("caches must be C-contiguous fp64 numpy arrays")
        B, H, cap, d = k_cache.shape
        if scale is None:
            scale = d ** -0.5
        out = np.empty((B, H, d))
        if log_f is None:
            rc = self.lib.path_oracle_decode_step(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(w),
                                                  _ptr(beta), float(scale), B, H, d,
                                                  int(n_cached), cap, int(bool(round_bf16)),
                                                  _ptr(k_cache), _ptr(v_cache), _ptr(out))
        else:
            rc = self.lib.path_oracle_decode_step_gated(
                _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(w), _ptr(beta), _ptr(log_f),
                float(scale), B, H, d, int(n_cached), cap, int(bool(round_bf16)), _ptr(k_cache),
                _ptr(v_cache), _ptr(g_cache), _ptr(out))
        if rc:
            raise ValueError("oracle decode_step: invalid arguments")
        return out

    def prefill_cache(self, k, v, w, beta, log_f=None, capacity=None):
        """The decode cache after positions 0..L-1: (k_cache, v_cache, g_cache), fp64
        [B,H,cap,d], [B,H,cap,d], [B,H,cap] (g_cache None without the gate); rows past L
        are zero."""
        k, v, w, beta, log_f = map(_f64, (k, v, w, beta, log_f))
        B, H, L, d = _dims(k)
        cap = L if capacity is None else int(capacity)
        kc = np.zeros((B, H, cap, d))
        vc = np.zeros((B, H, cap, d))
        gc = np.zeros((B, H, cap)) if log_f is not None else None
        rc = self.lib.path_oracle_prefill_cache(_ptr(k), _ptr(v), _ptr(w), _ptr(beta),
                                                _ptr(log_f), B, H, L, d, cap, _ptr(kc),
                                                _ptr(vc), _ptr(gc))
        if rc:
            raise ValueError("oracle prefill_cache: invalid arguments")
        return kc, vc, gc

    def round_bf16(self, x: float) -> float:
        """The oracle's double -> bfloat16 rounding (nearest, ties to even)."""
        return self.lib.path_oracle_round_bf16(float(x))


def default() -> Oracle:
    """The oracle built from path_oracle.c (compiled on first use)."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle(build())
    return _default


def fwd(*a, **kw):
    return default().fwd(*a, **kw)


def scores(*a, **kw):
    return default().scores(*a, **kw)


def bwd(*a, **kw):
    return default().bwd(*a, **kw)


def decode_step(*a, **kw):
    return default().decode_step(*a, **kw)


def prefill_cache(*a, **kw):
    return default().prefill_cache(*a, **kw)


def round_bf16(x):
    return default().round_bf16(x)
