"""PaTH attention on B200 (sm_100a): thin Python binding of libpath_attn.so.

The binding only marshals arguments: it checks dtypes, shapes and
contiguity, allocates outputs and workspace with torch when the caller does
not pass them, and calls the C ABI declared in ``include/path_attn.h`` on the
current torch CUDA stream. Every step of the computation runs in the
library's CUDA kernels; there is no CPU path. If the library is missing or no
CUDA device is present, the calls raise.

Entry points (same names as the C ABI):
- ``path_attn_fwd(q, k, v, w, beta, log_f=None, scale=None) -> (out, lse)``
- ``path_attn_bwd(q, k, v, w, beta, out, lse, dout, log_f=None, scale=None) -> dict``
- ``path_decode_step(q, k_new, v_new, w, beta, k_cache, v_cache, n_cached, scale=None,
  log_f=None, g_cache=None) -> out`` (with ``log_f``: ``path_decode_step_gated``)
- ``path_attn_prefill(q, k, v, w, beta, capacity, log_f=None, scale=None)
  -> (out, lse, k_cache, v_cache, g_cache)``
- ``path_decode_step_gated(q, k_new, v_new, w, beta, log_f, k_cache, v_cache, g_cache,
  n_cached, scale=None) -> out``
- ``path_decode_step_noalloc(q, k_new, v_new, w, beta, k_cache, v_cache, n_cached, scale=None)
  -> out``
- ``path_attn_wait_status(workspace) -> int`` (0 = no bounded wait gave up)
- ``path_attn_workspace_bytes``, ``path_decode_workspace_bytes``, ``path_status_string``
- diagnostics: ``path_kernel_launch_count()``, ``path_profile_enable(on)``,
  ``path_profile_read() -> {stage: (total_ms, count)}``
- the w / beta prologue: ``path_wbeta_fwd(x, A, Bw, f, U, b, H, beta_max=2.0) -> (w, beta)``,
  ``path_wbeta_bwd(x, A, Bw, f, U, b, H, dw, dbeta, beta_max=2.0) -> dict``,
  ``path_wbeta_workspace_bytes``
- test hook: ``path_test_withhold_kv_load(on)`` (makes the forward's bounded waits give up)
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpath_attn.so")

PATH_F32, PATH_BF16, PATH_BF16_F32OUT = 0, 1, 2
_DT = {torch.float32: PATH_F32, torch.bfloat16: PATH_BF16}


def _mode(in_dtype, out_dtype):
    """path_dtype of a call from the input and output element types."""
    if in_dtype == torch.float32 and out_dtype == torch.float32:
        return PATH_F32
    if in_dtype == torch.bfloat16 and out_dtype == torch.bfloat16:
        return PATH_BF16
    if in_dtype == torch.bfloat16 and out_dtype == torch.float32:
        return PATH_BF16_F32OUT
    raise ValueError(f"unsupported dtypes: inputs {in_dtype}, outputs {out_dtype}")
_lib = None


class _StageTime(ctypes.Structure):
    """path_stage_time of the C header."""
    _fields_ = [("name", ctypes.c_char * 32), ("total_ms", ctypes.c_double),
                ("count", ctypes.c_int)]


class PathError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {path_status_string(status)} (status {status})")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m softmax_attention_block_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, fp, i, f, sz = (ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float,
                            ctypes.c_size_t)
        L.path_status_string.argtypes = [i]
        L.path_status_string.restype = ctypes.c_char_p
        L.path_attn_workspace_bytes.argtypes = [i, i, i, i, i, i]
        L.path_attn_workspace_bytes.restype = sz
        L.path_decode_workspace_bytes.argtypes = [i, i, i, i, i]
        L.path_decode_workspace_bytes.restype = sz
        L.path_attn_fwd.argtypes = [vp, vp, vp, vp, fp, fp, f, i, i, i, i, i, vp, fp, vp, sz, vp]
        L.path_attn_bwd.argtypes = [vp, vp, vp, vp, fp, fp, f, i, i, i, i, i, vp, fp, vp,
                                    vp, vp, vp, vp, fp, fp, ctypes.c_uint, vp, sz, vp]
        L.path_decode_step.argtypes = [vp, vp, vp, vp, fp, f, i, i, i, i, i, i, vp, vp, vp, vp,
                                       sz, vp]
        L.path_decode_step_gated.argtypes = [vp, vp, vp, vp, fp, fp, f, i, i, i, i, i, i, vp,
                                             vp, fp, vp, vp, sz, vp]
        L.path_attn_prefill.argtypes = [vp, vp, vp, vp, fp, fp, f, i, i, i, i, i, vp, fp, vp, vp,
                                        fp, i, vp, sz, vp]
        L.path_decode_step_noalloc.argtypes = [vp, vp, vp, vp, fp, f, i, i, i, i, i, i, vp, vp,
                                               vp, vp]
        L.path_attn_wait_status.argtypes = [vp, vp]
        L.path_wbeta_workspace_bytes.argtypes = [i, i, i, i, i, i, i, i]
        L.path_wbeta_workspace_bytes.restype = sz
        L.path_wbeta_fwd.argtypes = [vp, vp, vp, fp, vp, fp, f, i, i, i, i, i, i, i, vp, fp, vp, sz,
                                     vp]
        L.path_wbeta_bwd.argtypes = [vp, vp, vp, fp, vp, fp, f, i, i, i, i, i, i, i, vp, fp, vp, fp,
                                     fp, fp, fp, fp, ctypes.c_uint, vp, sz, vp]
        L.path_wbeta_fwd.restype = i
        L.path_wbeta_bwd.restype = i
        L.path_test_withhold_kv_load.argtypes = [i]
        L.path_test_withhold_kv_load.restype = i
        L.path_kernel_launch_count.restype = ctypes.c_ulonglong
        L.path_profile_enable.argtypes = [i]
        L.path_profile_enable.restype = i
        L.path_profile_read.argtypes = [ctypes.POINTER(_StageTime), i]
        L.path_profile_read.restype = i
        for fn in (L.path_attn_fwd, L.path_attn_bwd, L.path_decode_step,
                   L.path_decode_step_gated, L.path_decode_step_noalloc, L.path_attn_prefill,
                   L.path_attn_wait_status):
            fn.restype = i
        _lib = L
    return _lib


def path_status_string(status: int) -> str:
    return lib().path_status_string(int(status)).decode()


def path_attn_workspace_bytes(B, H, L, d, dtype, for_bwd=False, out_dtype=None) -> int:
    mode = _mode(dtype, out_dtype or dtype)
    return int(lib().path_attn_workspace_bytes(B, H, L, d, mode, int(bool(for_bwd))))


def path_decode_workspace_bytes(B, H, capacity, d, dtype) -> int:
    return int(lib().path_decode_workspace_bytes(B, H, capacity, d, _DT[dtype]))


def _ptr(t):
    return None if t is None else t.data_ptr()


def _expect(name, t, shape, dtype):
    """The library reads and writes these buffers by size alone: check what it will assume."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")


def _check_dev(*ts):
    """All tensors contiguous, on one CUDA device, and that device the current one: the
    library launches on the current device's stream and resolves its own per-device
    state (the allocation-free decode's scratch array) through the current device."""
    ts = [t for t in ts if t is not None]
    for t in ts:
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")
        if t.device != ts[0].device:
            raise ValueError("all tensors must be on one device")
    if ts and ts[0].device.index != torch.cuda.current_device():
        raise ValueError(f"tensors are on {ts[0].device} but the current CUDA device is "
                         f"cuda:{torch.cuda.current_device()}: call under "
                         f"torch.cuda.device({ts[0].device})")


def _check_attn_inputs(q, k, v, w, beta, log_f):
    if q.dim() != 4:
        raise ValueError("q must be [B,H,L,d]")
    if q.dtype not in _DT:
        raise ValueError(f"q: dtype {q.dtype}, expected float32 or bfloat16")
    B, H, L, d = q.shape
    for n, t in (("k", k), ("v", v), ("w", w)):
        _expect(n, t, q.shape, q.dtype)
    _expect("beta", beta, (B, H, L), torch.float32)
    _expect("log_f", log_f, (B, H, L), torch.float32)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _workspace(nbytes, device, ws):
    if ws is None:
        return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)
    if ws.numel() * ws.element_size() < nbytes:
        raise ValueError("workspace too small")
    return ws


def _scale(scale, d):
    return float(d ** -0.5 if scale is None else scale)


def path_attn_fwd(q, k, v, w, beta, log_f=None, scale=None, out=None, lse=None, workspace=None,
                  out_dtype=None):
    """Forward pass. q, k, v, w: [B,H,L,d] (fp32 or bf16); beta, log_f: [B,H,L] fp32.
    out_dtype (default: q's dtype) may be torch.float32 with bf16 inputs.
    Returns (out [B,H,L,d], lse [B,H,L] fp32)."""
    _check_attn_inputs(q, k, v, w, beta, log_f)
    B, H, L, d = q.shape
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    dt = _mode(q.dtype, out.dtype)
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    _expect("out", out, q.shape, out.dtype)
    _expect("lse", lse, (B, H, L), torch.float32)
    _check_dev(q, k, v, w, beta, log_f, out, lse, workspace)
    nbytes = path_attn_workspace_bytes(B, H, L, d, q.dtype, False, out.dtype)
    ws = _workspace(nbytes, q.device, workspace)
    # the buffer's whole size: a backward-sized workspace also receives what a
    # backward that reuses it reads
    st = lib().path_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(w), _ptr(beta), _ptr(log_f),
                             _scale(scale, d), B, H, L, d, dt, _ptr(out), _ptr(lse), _ptr(ws),
                             ws.numel() * ws.element_size(), _stream())
    if st:
        raise PathError(st, "path_attn_fwd")
    return out, lse


PATH_BWD_REUSE_FWD_WORKSPACE = 1


def path_attn_bwd(q, k, v, w, beta, out, lse, dout, log_f=None, scale=None, grads=None,
                  workspace=None, reuse_fwd_workspace=False):
    """Backward of sum(out * dout). out, dout and the returned dq, dk, dv, dw share
    out's dtype. Returns dict dq, dk, dv, dw, dbeta[, dlog_f].

    reuse_fwd_workspace: `workspace` is the buffer the matching path_attn_fwd call
    used (allocated with the backward size), inputs unchanged since; the backward
    then reuses the forward's block transforms and transported keys."""
    if reuse_fwd_workspace and workspace is None:
        raise ValueError("reuse_fwd_workspace needs the forward's workspace")
    _check_attn_inputs(q, k, v, w, beta, log_f)
    B, H, L, d = q.shape
    dt = _mode(q.dtype, out.dtype)
    if dout.dtype != out.dtype:
        raise ValueError("dout must have out's dtype")
    _expect("out", out, q.shape, out.dtype)
    _expect("dout", dout, q.shape, out.dtype)
    _expect("lse", lse, (B, H, L), torch.float32)
    if grads is None:
        grads = {n: torch.empty(q.shape, dtype=out.dtype, device=q.device)
                 for n in ("dq", "dk", "dv", "dw")}
        grads["dbeta"] = torch.empty_like(beta)
        if log_f is not None:
            grads["dlog_f"] = torch.empty_like(log_f)
    for n in ("dq", "dk", "dv", "dw"):
        _expect(n, grads[n], q.shape, out.dtype)
    _expect("dbeta", grads["dbeta"], (B, H, L), torch.float32)
    dlf = grads.get("dlog_f") if log_f is not None else None
    if log_f is not None and dlf is None:
        raise ValueError("grads needs dlog_f when log_f is given")
    _expect("dlog_f", dlf, (B, H, L), torch.float32)
    _check_dev(q, k, v, w, beta, log_f, out, lse, dout, workspace, *grads.values())
    nbytes = path_attn_workspace_bytes(B, H, L, d, q.dtype, True, out.dtype)
    ws = _workspace(nbytes, q.device, workspace)
    st = lib().path_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(w), _ptr(beta), _ptr(log_f),
                             _scale(scale, d), B, H, L, d, dt, _ptr(out), _ptr(lse), _ptr(dout),
                             _ptr(grads["dq"]), _ptr(grads["dk"]), _ptr(grads["dv"]),
                             _ptr(grads["dw"]), _ptr(grads["dbeta"]), _ptr(dlf),
                             PATH_BWD_REUSE_FWD_WORKSPACE if reuse_fwd_workspace else 0, _ptr(ws),
                             nbytes, _stream())
    if st:
        raise PathError(st, "path_attn_bwd")
    return grads


def _check_decode(q, k_new, v_new, w, beta, k_cache, v_cache, out, log_f, g_cache):
    if k_cache.dim() != 4 or k_cache.dtype not in _DT:
        raise ValueError("k_cache must be [B,H,capacity,d], float32 or bfloat16")
    B, H, cap, d = k_cache.shape
    if (log_f is None) != (g_cache is None):
        raise ValueError("log_f and g_cache go together")
    _expect("v_cache", v_cache, k_cache.shape, k_cache.dtype)
    for n, t in (("q", q), ("k_new", k_new), ("v_new", v_new), ("w", w), ("out", out)):
        _expect(n, t, (B, H, d), k_cache.dtype)
    _expect("beta", beta, (B, H), torch.float32)
    _expect("log_f", log_f, (B, H), torch.float32)
    _expect("g_cache", g_cache, (B, H, cap), torch.float32)
    return B, H, cap, d


def path_decode_step(q, k_new, v_new, w, beta, k_cache, v_cache, n_cached, scale=None, out=None,
                     workspace=None, log_f=None, g_cache=None):
    """One decode step; updates k_cache / v_cache ([B,H,cap,d]) in place. Returns out [B,H,d].

    With the forget gate, log_f [B,H] fp32 is log f of the new position and g_cache
    [B,H,cap] fp32 the cached keys' gate biases, also updated in place
    (path_decode_step_gated)."""
    if out is None:
        out = torch.empty_like(q)
    B, H, cap, d = _check_decode(q, k_new, v_new, w, beta, k_cache, v_cache, out, log_f, g_cache)
    dt = _DT[k_cache.dtype]
    _check_dev(q, k_new, v_new, w, beta, k_cache, v_cache, out, log_f, g_cache, workspace)
    nbytes = path_decode_workspace_bytes(B, H, cap, d, k_cache.dtype)
    ws = _workspace(nbytes, q.device, workspace)
    if log_f is None:
        st = lib().path_decode_step(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(w), _ptr(beta),
                                    _scale(scale, d), B, H, d, int(n_cached), cap, dt,
                                    _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(ws), nbytes,
                                    _stream())
        where = "path_decode_step"
    else:
        st = lib().path_decode_step_gated(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(w), _ptr(beta),
                                          _ptr(log_f), _scale(scale, d), B, H, d, int(n_cached),
                                          cap, dt, _ptr(k_cache), _ptr(v_cache), _ptr(g_cache),
                                          _ptr(out), _ptr(ws), nbytes, _stream())
        where = "path_decode_step_gated"
    if st:
        raise PathError(st, where)
    return out


def path_decode_step_gated(q, k_new, v_new, w, beta, log_f, k_cache, v_cache, g_cache, n_cached,
                           scale=None, out=None, workspace=None):
    """PaTH-FoX decode step: path_decode_step with the forget gate (log_f [B,H] fp32 of the
    new position; g_cache [B,H,cap] fp32, the cached keys' gate biases, updated in place)."""
    if log_f is None or g_cache is None:
        raise ValueError("path_decode_step_gated needs log_f and g_cache")
    return path_decode_step(q, k_new, v_new, w, beta, k_cache, v_cache, n_cached, scale=scale,
                            out=out, workspace=workspace, log_f=log_f, g_cache=g_cache)


def path_decode_step_noalloc(q, k_new, v_new, w, beta, k_cache, v_cache, n_cached, scale=None,
                             out=None):
    """path_decode_step without a workspace (the library's fixed 4 MiB device scratch; see
    the C header for its limit and its sharing between calls on one device)."""
    if out is None:
        out = torch.empty_like(q)
    B, H, cap, d = _check_decode(q, k_new, v_new, w, beta, k_cache, v_cache, out, None, None)
    _check_dev(q, k_new, v_new, w, beta, k_cache, v_cache, out)
    st = lib().path_decode_step_noalloc(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(w), _ptr(beta),
                                        _scale(scale, d), B, H, d, int(n_cached), cap,
                                        _DT[k_cache.dtype], _ptr(k_cache), _ptr(v_cache),
                                        _ptr(out), _stream())
    if st:
        raise PathError(st, "path_decode_step_noalloc")
    return out


def path_attn_wait_status(workspace) -> int:
    """Waits for the current stream, then returns 0, or PATH_ERR_TIMEOUT (5) if the last
    path_attn_fwd / path_attn_bwd that used `workspace` had a bounded wait give up."""
    _check_dev(workspace)
    return int(lib().path_attn_wait_status(_ptr(workspace), _stream()))


def path_kernel_launch_count() -> int:
    """Kernels this library has launched in this process so far."""
    return int(lib().path_kernel_launch_count())


def path_profile_enable(on: bool) -> bool:
    """Per-stage event timing on or off; returns the previous setting."""
    return bool(lib().path_profile_enable(int(bool(on))))


def path_profile_read(max_entries: int = 64) -> dict:
    """Stage name -> (total ms, launches) of the stages timed since the last read."""
    buf = (_StageTime * max_entries)()
    n = lib().path_profile_read(buf, max_entries)
    return {buf[i].name.decode(): (buf[i].total_ms, buf[i].count) for i in range(n)}


def path_attn_prefill(q, k, v, w, beta, capacity, log_f=None, scale=None, out=None, lse=None,
                      k_cache=None, v_cache=None, g_cache=None, workspace=None, out_dtype=None):
    """Forward over positions 0..L-1 plus the decode cache it leaves.

    Returns (out, lse, k_cache, v_cache, g_cache): out / lse as path_attn_fwd; the
    caches [B,H,capacity,d] in q's dtype with rows 0..L-1 written (k_cache row j =
    H_{L-1} ... H_{j+1} k_j, v_cache row j = v_j); g_cache [B,H,capacity] fp32 (row j =
    c_{L-1} - c_j) with the forget gate, else None. Caches the call allocates are
    zero past row L-1."""
    _check_attn_inputs(q, k, v, w, beta, log_f)
    B, H, L, d = q.shape
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    dt = _mode(q.dtype, out.dtype)
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    _expect("out", out, q.shape, out.dtype)
    _expect("lse", lse, (B, H, L), torch.float32)
    _expect("k_cache", k_cache, (B, H, capacity, d), q.dtype)
    _expect("v_cache", v_cache, (B, H, capacity, d), q.dtype)
    if log_f is not None:
        _expect("g_cache", g_cache, (B, H, capacity), torch.float32)
    if k_cache is None:
        k_cache = torch.zeros((B, H, capacity, d), dtype=q.dtype, device=q.device)
    if v_cache is None:
        v_cache = torch.zeros((B, H, capacity, d), dtype=q.dtype, device=q.device)
    if log_f is not None and g_cache is None:
        g_cache = torch.zeros((B, H, capacity), dtype=torch.float32, device=q.device)
    if log_f is None:
        g_cache = None
    _check_dev(q, k, v, w, beta, log_f, out, lse, k_cache, v_cache, g_cache, workspace)
    nbytes = path_attn_workspace_bytes(B, H, L, d, q.dtype, False, out.dtype)
    ws = _workspace(nbytes, q.device, workspace)
    st = lib().path_attn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(w), _ptr(beta), _ptr(log_f),
                                 _scale(scale, d), B, H, L, d, dt, _ptr(out), _ptr(lse),
                                 _ptr(k_cache), _ptr(v_cache), _ptr(g_cache), int(capacity),
                                 _ptr(ws), nbytes, _stream())
    if st:
        raise PathError(st, "path_attn_prefill")
    return out, lse, k_cache, v_cache, g_cache


def path_test_withhold_kv_load(on: bool) -> None:
    """Test hook of the bounded waits (include/path_attn.h): while on, the tensor-core
    forward's last query tile never receives one key/value block and reports a timeout."""
    st = lib().path_test_withhold_kv_load(1 if on else 0)
    if st:
        raise PathError(st, "path_test_withhold_kv_load")


# ---------------------------------------------------------------- the w / beta prologue
def path_wbeta_workspace_bytes(B, L, D, r, H, d, dtype, for_bwd=False, out_dtype=None) -> int:
    mode = _mode(dtype, out_dtype or dtype)
    return int(lib().path_wbeta_workspace_bytes(B, L, D, r, H, d, mode, int(bool(for_bwd))))


def _check_wbeta(x, A, Bw, f, U, b, H):
    if x.dim() != 3 or x.dtype not in _DT:
        raise ValueError("x must be [B,L,D], float32 or bfloat16")
    B, L, D = x.shape
    if A.dim() != 2 or A.shape[0] != D:
        raise ValueError(f"A: shape {tuple(A.shape)}, expected ({D}, r)")
    r = A.shape[1]
    if Bw.dim() != 2 or Bw.shape[0] != r or Bw.shape[1] % H:
        raise ValueError(f"Bw: shape {tuple(Bw.shape)}, expected ({r}, H*d) with H={H}")
    d = Bw.shape[1] // H
    _expect("A", A, (D, r), x.dtype)
    _expect("Bw", Bw, (r, H * d), x.dtype)
    _expect("U", U, (D, H), x.dtype)
    _expect("f", f, (H * d, 3), torch.float32)
    _expect("b", b, (H,), torch.float32)
    return B, L, D, r, d


def path_wbeta_fwd(x, A, Bw, f, U, b, H, beta_max=2.0, w=None, beta=None, workspace=None,
                   out_dtype=None):
    """w [B,H,L,d] (out_dtype, default x's dtype) and beta [B,H,L] fp32 from x [B,L,D]:
    w = per-head L2 normalisation of the 3-tap causal convolution (filter f [H*d,3]) of
    (x A) Bw; beta = min(2 sigmoid(x U + b), beta_max)."""
    B, L, D, r, d = _check_wbeta(x, A, Bw, f, U, b, H)
    od = out_dtype or x.dtype
    if w is None:
        w = torch.empty((B, H, L, d), dtype=od, device=x.device)
    if beta is None:
        beta = torch.empty((B, H, L), dtype=torch.float32, device=x.device)
    _expect("w", w, (B, H, L, d), od)
    _expect("beta", beta, (B, H, L), torch.float32)
    mode = _mode(x.dtype, od)
    _check_dev(x, A, Bw, f, U, b, w, beta, workspace)
    nbytes = path_wbeta_workspace_bytes(B, L, D, r, H, d, x.dtype, False, od)
    ws = _workspace(nbytes, x.device, workspace)
    st = lib().path_wbeta_fwd(_ptr(x), _ptr(A), _ptr(Bw), _ptr(f), _ptr(U), _ptr(b), float(beta_max),
                              B, L, D, r, H, d, mode, _ptr(w), _ptr(beta), _ptr(ws), nbytes,
                              _stream())
    if st:
        raise PathError(st, "path_wbeta_fwd")
    return w, beta


def path_wbeta_bwd(x, A, Bw, f, U, b, H, dw, dbeta, beta_max=2.0, grads=None, workspace=None,
                   reuse_fwd_workspace=False):
    """Gradients of sum(w * dw) + sum(beta * dbeta): dict dx (dw's dtype), dA, dBw, df, dU,
    db (fp32)."""
    if reuse_fwd_workspace and workspace is None:
        raise ValueError("reuse_fwd_workspace needs the forward's workspace")
    B, L, D, r, d = _check_wbeta(x, A, Bw, f, U, b, H)
    od = dw.dtype
    _expect("dw", dw, (B, H, L, d), od)
    _expect("dbeta", dbeta, (B, H, L), torch.float32)
    if grads is None:
        dev = x.device
        grads = dict(dx=torch.empty((B, L, D), dtype=od, device=dev),
                     dA=torch.empty((D, r), dtype=torch.float32, device=dev),
                     dBw=torch.empty((r, H * d), dtype=torch.float32, device=dev),
                     df=torch.empty((H * d, 3), dtype=torch.float32, device=dev),
                     dU=torch.empty((D, H), dtype=torch.float32, device=dev),
                     db=torch.empty((H,), dtype=torch.float32, device=dev))
    _expect("dx", grads["dx"], (B, L, D), od)
    for n, shp in (("dA", (D, r)), ("dBw", (r, H * d)), ("df", (H * d, 3)), ("dU", (D, H)),
                   ("db", (H,))):
        _expect(n, grads[n], shp, torch.float32)
    mode = _mode(x.dtype, od)
    _check_dev(x, A, Bw, f, U, b, dw, dbeta, workspace, *grads.values())
    nbytes = path_wbeta_workspace_bytes(B, L, D, r, H, d, x.dtype, True, od)
    ws = _workspace(nbytes, x.device, workspace)
    st = lib().path_wbeta_bwd(_ptr(x), _ptr(A), _ptr(Bw), _ptr(f), _ptr(U), _ptr(b), float(beta_max),
                              B, L, D, r, H, d, mode, _ptr(dw), _ptr(dbeta), _ptr(grads["dx"]),
                              _ptr(grads["dA"]), _ptr(grads["dBw"]), _ptr(grads["df"]),
                              _ptr(grads["dU"]), _ptr(grads["db"]),
                              PATH_BWD_REUSE_FWD_WORKSPACE if reuse_fwd_workspace else 0, _ptr(ws),
                              nbytes, _stream())
    if st:
        raise PathError(st, "path_wbeta_bwd")
    return grads
