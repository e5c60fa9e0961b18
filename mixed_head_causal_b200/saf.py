"""Python binding of libsaf.so (include/saf.h): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; this module only
allocates outputs and workspace with torch, passes raw device pointers and
the current CUDA stream through ctypes, and turns status codes into
exceptions.  It raises when the library is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import functools
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsaf.so")

SAF_OK, SAF_ERR_INVALID_ARG, SAF_ERR_UNSUPPORTED, SAF_ERR_WORKSPACE, SAF_ERR_CUDA, SAF_ERR_TIMEOUT = range(6)
HEAD_DIM = 64

# Every symbol include/saf.h declares, with its ctypes signature.
_vp, _sz, _i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
SIGNATURES = {
    "saf_status_string": ([_i], ctypes.c_char_p),
    "saf_version": ([], _i),
    "saf_workspace_size": ([_i, _i, _i, _i, _i], _sz),
    "saf_workspace_size_gqa": ([_i, _i, _i, _i, _i, _i], _sz),
    "saf_replaced_lognorm": ([_vp, _vp, _vp, _i, _i, _vp, _vp], _i),
    "saf_mixed_attn_fwd": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _sz, _vp], _i),
    "saf_mixed_attn_bwd": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                            _vp, _vp, _vp, _i, _vp, _sz, _vp], _i),
    "saf_mixed_attn_fwd_gqa": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _sz, _vp],
                               _i),
    "saf_mixed_attn_bwd_gqa": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                                _vp, _vp, _vp, _i, _vp, _sz, _vp], _i),
    "saf_device_status": ([_vp, _sz, _vp], _i),
    "saf_selftest_wait_timeout": ([_vp, _sz, ctypes.c_longlong, _vp], _i),
    "saf_replaced_pattern_grad": ([_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _sz, _vp], _i),
    "saf_calibration_workspace_size": ([_i, _i, _i], _sz),
    "saf_fit_workspace_size": ([_i, _i], _sz),
    "saf_fit_pattern": ([_vp, _i, _i, _i, ctypes.c_float, _vp, _vp, _vp, _vp, _sz, _vp], _i),
    "saf_attn_calibration": ([_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _sz, _vp], _i),
    "saf_mixed_attn_bwd_noalloc": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                    _vp, _vp, _vp, _i, _vp], _i),
    "saf_launch_count": ([], ctypes.c_uint64),
    "saf_profile_enable": ([_i], _i),
    "saf_profile_read": ([ctypes.POINTER(_i), ctypes.POINTER(ctypes.c_float), _i], _i),
    "saf_kernel_name": ([_i], ctypes.c_char_p),
}

_lib = None


def _annotated(fn):
    """With SAF_NVTX=1 in the environment, each call is an NVTX range named
    saf.<function> (a profiler can then select one call, e.g. ncu --nvtx
    --nvtx-include); otherwise the call is unchanged."""
    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        if os.environ.get("SAF_NVTX", "") in ("", "0"):
            return fn(*args, **kwargs)
        torch.cuda.nvtx.range_push("saf." + fn.__name__)
        try:
            return fn(*args, **kwargs)
        finally:
            torch.cuda.nvtx.range_pop()
    return wrapper


class SafError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Loads libsaf.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"libsaf.so not found at {p}: build it with "
                           "`python -m mixed_head_causal_b200.build` (no fallback exists)")
    lib = ctypes.CDLL(p)
    for name, (args, res) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    if path is None:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().saf_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != SAF_OK:
        raise SafError(status, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _mask_buffer(mask) -> Tuple[ctypes.Array, int]:
    m = torch.as_tensor(mask).to("cpu", torch.uint8).contiguous()
    buf = (ctypes.c_uint8 * max(1, m.numel())).from_buffer_copy(m.numpy().tobytes() or b"\0")
    return buf, m.numel()


def workspace_size(B: int, H: int, T: int, d_h: int = HEAD_DIM, backward: bool = False,
                   h_kv: Optional[int] = None) -> int:
    """Workspace bytes; h_kv (default H) K/V heads shared by groups of H / h_kv query heads."""
    if h_kv is None or h_kv == H:
        n = load().saf_workspace_size(B, H, T, d_h, 1 if backward else 0)
    else:
        n = load().saf_workspace_size_gqa(B, H, h_kv, T, d_h, 1 if backward else 0)
    if n == ctypes.c_size_t(-1).value:
        raise SafError(SAF_ERR_INVALID_ARG, "saf_workspace_size")
    return int(n)


def new_workspace(B: int, H: int, T: int, device, backward: bool = False, h_kv: Optional[int] = None) -> torch.Tensor:
    """A zero-initialised uint8 workspace (its 256-byte header must start at 0)."""
    n = max(256, workspace_size(B, H, T, HEAD_DIM, backward, h_kv))
    return torch.zeros(n, dtype=torch.uint8, device=device)


def _check_layer_tensor(name: str, t: torch.Tensor, shape, dtype=torch.bfloat16) -> None:
    if t.dtype != dtype or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} of shape {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)} on {t.device}")


@_annotated
def replaced_lognorm(alpha: torch.Tensor, rho: torch.Tensor, mask, out: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """log Z [H, T] of the replaced heads (other rows left as in `out`)."""
    H, T = alpha.shape
    if out is None:
        out = torch.zeros(H, T, dtype=torch.float32, device=alpha.device)
    mbuf, mh = _mask_buffer(mask)
    if mh != H:
        raise ValueError("mask length != H")
    _check(load().saf_replaced_lognorm(_ptr(alpha), _ptr(rho), ctypes.addressof(mbuf), H, T,
                                       _ptr(out), _stream_ptr(stream)), "saf_replaced_lognorm")
    return out


@_annotated
def mixed_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, alpha: torch.Tensor,
                   rho: torch.Tensor, mask, logz: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None):
    """Forward of one mixed-head layer.  Returns (O [B,H,T,64] bf16, lse [B,H,T] fp32).

    k, v may hold fewer heads than q (H_kv dividing H): query head h then reads
    K/V head h // (H // H_kv) (grouped-query attention)."""
    B, H, T, d = q.shape
    Hkv = k.shape[1]
    _check_layer_tensor("q", q, (B, H, T, d))
    for n, t in (("k", k), ("v", v)):
        _check_layer_tensor(n, t, (B, Hkv, T, d))
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, H, T, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = new_workspace(B, H, T, q.device, backward=False, h_kv=Hkv)
    mbuf, mh = _mask_buffer(mask)
    if mh != H:
        raise ValueError("mask length != H")
    wsb = workspace.numel() * workspace.element_size()
    if Hkv == H:
        st = load().saf_mixed_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(alpha), _ptr(rho),
                                       _ptr(logz), ctypes.addressof(mbuf), B, H, T, d, _ptr(workspace), wsb,
                                       _stream_ptr(stream))
    else:
        st = load().saf_mixed_attn_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(alpha),
                                           _ptr(rho), _ptr(logz), ctypes.addressof(mbuf), B, H, Hkv, T, d,
                                           _ptr(workspace), wsb, _stream_ptr(stream))
    _check(st, "saf_mixed_attn_fwd")
    return out, lse


@_annotated
def mixed_attn_bwd(q, k, v, o, dout, lse, alpha, rho, mask, logz=None, grad_dtype=torch.bfloat16,
                   dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Backward of one mixed-head layer.  Returns (dQ, dK, dV) in grad_dtype (bf16 or fp32).

    With shared K/V (k, v holding H_kv < H heads) dK and dV have H_kv heads, each
    the sum over the query heads of its group."""
    B, H, T, d = q.shape
    Hkv = k.shape[1]
    for n, t in (("q", q), ("o", o), ("dout", dout)):
        _check_layer_tensor(n, t, (B, H, T, d))
    for n, t in (("k", k), ("v", v)):
        _check_layer_tensor(n, t, (B, Hkv, T, d))
    if grad_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("grad_dtype must be bf16 or fp32")
    gd = 1 if grad_dtype == torch.float32 else 0
    dq = torch.empty(B, H, T, d, dtype=grad_dtype, device=q.device) if dq is None else dq
    dk = torch.empty(B, Hkv, T, d, dtype=grad_dtype, device=q.device) if dk is None else dk
    dv = torch.empty(B, Hkv, T, d, dtype=grad_dtype, device=q.device) if dv is None else dv
    if workspace is None:
        workspace = new_workspace(B, H, T, q.device, backward=True, h_kv=Hkv)
    mbuf, mh = _mask_buffer(mask)
    if mh != H:
        raise ValueError("mask length != H")
    wsb = workspace.numel() * workspace.element_size()
    if Hkv == H:
        st = load().saf_mixed_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(alpha),
                                       _ptr(rho), _ptr(logz), ctypes.addressof(mbuf), B, H, T, d,
                                       _ptr(dq), _ptr(dk), _ptr(dv), gd, _ptr(workspace), wsb, _stream_ptr(stream))
    else:
        st = load().saf_mixed_attn_bwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                                           _ptr(alpha), _ptr(rho), _ptr(logz), ctypes.addressof(mbuf), B, H, Hkv,
                                           T, d, _ptr(dq), _ptr(dk), _ptr(dv), gd, _ptr(workspace), wsb,
                                           _stream_ptr(stream))
    _check(st, "saf_mixed_attn_bwd")
    return dq, dk, dv


@_annotated
def replaced_pattern_grad(v, dout, alpha, rho, mask, logz=None, da=None, dr=None, workspace=None, stream=None):
    """Trainable pattern: (dalpha, drho) [H, T] fp32 of the replaced heads
    (rows of ordinary heads zero) for the output gradient dout."""
    B, H, T, d = v.shape
    for n, t in (("v", v), ("dout", dout)):
        _check_layer_tensor(n, t, (B, H, T, d))
    da = torch.empty(H, T, dtype=torch.float32, device=v.device) if da is None else da
    dr = torch.empty(H, T, dtype=torch.float32, device=v.device) if dr is None else dr
    if workspace is None and logz is None:
        workspace = new_workspace(B, H, T, v.device, backward=False)
    mbuf, mh = _mask_buffer(mask)
    if mh != H:
        raise ValueError("mask length != H")
    wsb = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().saf_replaced_pattern_grad(_ptr(v), _ptr(dout), _ptr(alpha), _ptr(rho), _ptr(logz),
                                            ctypes.addressof(mbuf), B, H, T, d, _ptr(da), _ptr(dr),
                                            _ptr(workspace), wsb, _stream_ptr(stream)),
           "saf_replaced_pattern_grad")
    return da, dr


@_annotated
def fit_pattern(target, steps: int = 400, lr: float = 0.1, stream=None):
    """Fits a, r of Eq. (3) to target patterns [n, T, T] (fp32, causal, unit
    row sums).  Returns (a [n, T], r [n, T], mean row KL [n])."""
    if target.dim() == 2:
        target = target[None]
    n, T, T2 = target.shape
    if T != T2 or target.dtype != torch.float32 or not target.is_cuda or not target.is_contiguous():
        raise ValueError("target: expected a contiguous CUDA fp32 [n, T, T] tensor")
    a = torch.empty(n, T, dtype=torch.float32, device=target.device)
    r = torch.empty_like(a)
    kl = torch.empty(n, dtype=torch.float32, device=target.device)
    nbytes = load().saf_fit_workspace_size(n, T)
    if nbytes == ctypes.c_size_t(-1).value:
        raise SafError(SAF_ERR_INVALID_ARG, "saf_fit_workspace_size")
    ws = torch.zeros(max(256, int(nbytes)), dtype=torch.uint8, device=target.device)
    _check(load().saf_fit_pattern(_ptr(target), n, T, steps, lr, _ptr(a), _ptr(r), _ptr(kl), _ptr(ws),
                                  ws.numel(), _stream_ptr(stream)), "saf_fit_pattern")
    return a, r, kl


@_annotated
def attn_calibration(q, k, lse, a_hat=None, svar=None, workspace=None, stream=None):
    """Calibration statistics over the N samples of q, k [N,H,T,64] (lse from
    the forward of the same inputs): (A_hat [H,T,T] fp32, s_var [H] fp32), Eq. (1)."""
    N, H, T, d = q.shape
    for n, t in (("q", q), ("k", k)):
        _check_layer_tensor(n, t, (N, H, T, d))
    a_hat = torch.empty(H, T, T, dtype=torch.float32, device=q.device) if a_hat is None else a_hat
    svar = torch.empty(H, dtype=torch.float32, device=q.device) if svar is None else svar
    if workspace is None:
        nbytes = load().saf_calibration_workspace_size(H, T, d)
        if nbytes == ctypes.c_size_t(-1).value:
            raise SafError(SAF_ERR_INVALID_ARG, "saf_calibration_workspace_size")
        workspace = torch.empty(max(16, int(nbytes)), dtype=torch.uint8, device=q.device)
    _check(load().saf_attn_calibration(_ptr(q), _ptr(k), _ptr(lse), N, H, T, d, _ptr(a_hat), _ptr(svar),
                                       _ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _stream_ptr(stream)), "saf_attn_calibration")
    return a_hat, svar


@_annotated
def mixed_attn_bwd_noalloc(q, k, v, o, dout, lse, alpha, rho, mask, logz=None, grad_dtype=torch.bfloat16,
                           dq=None, dk=None, dv=None, stream=None):
    """Backward without a workspace (the library's own fixed scratch, see
    include/saf.h): for callers that cannot allocate device memory.  Output
    tensors are still the caller's; pass them in to allocate nothing here."""
    B, H, T, d = v.shape
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_layer_tensor(n, t, (B, H, T, d))
    gd = 1 if grad_dtype == torch.float32 else 0
    dq = torch.empty(B, H, T, d, dtype=grad_dtype, device=v.device) if dq is None else dq
    dk = torch.empty(B, H, T, d, dtype=grad_dtype, device=v.device) if dk is None else dk
    dv = torch.empty(B, H, T, d, dtype=grad_dtype, device=v.device) if dv is None else dv
    mbuf, mh = _mask_buffer(mask)
    if mh != H:
        raise ValueError("mask length != H")
    _check(load().saf_mixed_attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                                             _ptr(alpha), _ptr(rho), _ptr(logz), ctypes.addressof(mbuf),
                                             B, H, T, d, _ptr(dq), _ptr(dk), _ptr(dv), gd, _stream_ptr(stream)),
           "saf_mixed_attn_bwd_noalloc")
    return dq, dk, dv


def device_status(workspace: torch.Tensor, stream=None) -> int:
    """Reads and clears the device error word of `workspace` (synchronous)."""
    return int(load().saf_device_status(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                        _stream_ptr(stream)))


def selftest_wait_timeout(workspace: torch.Tensor, limit_cycles: int = 1 << 20, stream=None) -> None:
    """Enqueues a bounded device wait that nothing completes (it sets the
    workspace's error word when it gives up; see device_status)."""
    _check(load().saf_selftest_wait_timeout(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                            int(limit_cycles), _stream_ptr(stream)), "saf_selftest_wait_timeout")


def launch_count() -> int:
    """Kernels the library has enqueued since it was loaded."""
    return int(load().saf_launch_count())


def profile_enable(max_launches: int) -> None:
    """Start (max_launches > 0) or stop (0) per-kernel event timing."""
    _check(load().saf_profile_enable(int(max_launches)), "saf_profile_enable")


def profile_read(n: int = 1 << 16):
    """[(kernel_name, milliseconds)] of the current profiling session."""
    lib = load()
    ids = (ctypes.c_int * n)()
    ms = (ctypes.c_float * n)()
    got = lib.saf_profile_read(ids, ms, n)
    if got < 0:
        raise SafError(SAF_ERR_CUDA, "saf_profile_read")
    return [(lib.saf_kernel_name(ids[i]).decode(), float(ms[i])) for i in range(min(got, n))]
