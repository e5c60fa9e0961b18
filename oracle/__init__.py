"""fp64 CPU oracle for the mixed-head causal attention layer.

TEST INFRASTRUCTURE ONLY: imported by the test suite, by the smoke check and
by the benchmark's CPU-baseline leg, never by the GPU product path.  It shares
no code with the CUDA library.

The arithmetic lives in ``saf_oracle.c`` (plain loops, double precision, one
(batch, head) slice per task); this module only marshals torch/numpy arrays
into it.  See that file's header for the definitions it follows (the causal
softmax attention of section 一 and the compact fixed pattern of Eq. (3) in
"When Can Attention Heads Be Statically Defined?", with the V-only backward of
replaced heads from section 二.4).

Every function here is pinned by tests/test_oracle_pins.py (closed forms,
library routines, finite differences, invariants and planted mutations).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "saf_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")


def compile_library(src: str, out: str) -> str:
    """gcc -O2 (no fast-math) of an oracle source into a shared library."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-std=c11",
                           "-fno-fast-math", "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(SOURCE):
        compile_library(SOURCE, _LIB_PATH)
    return _LIB_PATH


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _f64(x) -> np.ndarray:
    """Exact widening of a torch / numpy array to a contiguous float64 array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _u8(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))


class Oracle:
    """The oracle bound to one compiled library (the real one, or a planted
    mutant that the pin tests must reject)."""

    def __init__(self, lib_path: Optional[str] = None):
        lib = ctypes.CDLL(lib_path or build())
        dp = ctypes.POINTER(ctypes.c_double)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        i = ctypes.c_int
        lib.oracle_lognorm.argtypes = [i, dp, dp, dp]
        lib.oracle_lognorm.restype = None
        lib.oracle_fwd_slices.argtypes = [i, i, i, u8p, dp, dp, dp, dp, dp, dp, dp, i]
        lib.oracle_fwd_slices.restype = i
        lib.oracle_bwd_slices.argtypes = [i, i, i, u8p, dp, dp, dp, dp, dp, dp, dp, dp, dp, i]
        lib.oracle_bwd_slices.restype = i
        lib.oracle_pattern_grad_slice.argtypes = [i, i, dp, dp, dp, dp, dp, dp]
        lib.oracle_pattern_grad_slice.restype = i
        lib.oracle_calibration_head.argtypes = [i, i, i, dp, dp, dp, dp]
        lib.oracle_calibration_head.restype = i
        lib.oracle_fit_pattern.argtypes = [i, dp, i, ctypes.c_double, dp, dp, dp]
        lib.oracle_fit_pattern.restype = i
        self.lib = lib

    def lognorm(self, a, r) -> np.ndarray:
        """log Z(i) of Eq. (3) for one head ([T]) or several ([H, T])."""
        a64, r64 = _f64(a), _f64(r)
        out = np.empty_like(a64)
        if a64.ndim == 1:
            self.lib.oracle_lognorm(a64.shape[0], _p(a64), _p(r64), _p(out))
            return out
        for h in range(a64.shape[0]):
            ah, rh, oh = (np.ascontiguousarray(x) for x in (a64[h], r64[h], out[h]))
            self.lib.oracle_lognorm(a64.shape[1], _p(ah), _p(rh), _p(oh))
            out[h] = oh
        return out

    def fwd_slices(self, q, k, v, a_rows, r_rows, replaced: Sequence[int],
                   n_threads: Optional[int] = None) -> Tuple[np.ndarray, np.ndarray]:
        """Forward of n independent slices: q,k,v [n,T,d]; a_rows,r_rows [n,T]
        (the pattern row of each slice's head); replaced[n] flags.
        Returns (O [n,T,d], lse [n,T])."""
        q64, k64, v64 = _f64(q), _f64(k), _f64(v)
        n, T, d = v64.shape
        rep = np.ascontiguousarray(np.asarray(replaced, dtype=np.uint8).reshape(n))
        a64, r64 = _f64(a_rows).reshape(n, T), _f64(r_rows).reshape(n, T)
        a64, r64 = np.ascontiguousarray(a64), np.ascontiguousarray(r64)
        o = np.empty_like(v64)
        lse = np.empty((n, T), dtype=np.float64)
        rc = self.lib.oracle_fwd_slices(n, T, d, _u8(rep), _p(q64), _p(k64), _p(v64),
                                        _p(a64), _p(r64), _p(o), _p(lse),
                                        n_threads or default_threads())
        if rc != 0:
            raise MemoryError("oracle forward failed")
        return o, lse

    def bwd_slices(self, q, k, v, dout, a_rows, r_rows, replaced: Sequence[int],
                   n_threads: Optional[int] = None):
        """Backward of n independent slices (layout as fwd_slices).
        Returns (dQ, dK, dV), each [n,T,d]."""
        q64, k64, v64, do64 = _f64(q), _f64(k), _f64(v), _f64(dout)
        n, T, d = v64.shape
        rep = np.ascontiguousarray(np.asarray(replaced, dtype=np.uint8).reshape(n))
        a64, r64 = _f64(a_rows).reshape(n, T), _f64(r_rows).reshape(n, T)
        a64, r64 = np.ascontiguousarray(a64), np.ascontiguousarray(r64)
        dq, dk, dv = np.empty_like(v64), np.empty_like(v64), np.empty_like(v64)
        rc = self.lib.oracle_bwd_slices(n, T, d, _u8(rep), _p(q64), _p(k64), _p(v64), _p(do64),
                                        _p(a64), _p(r64), _p(dq), _p(dk), _p(dv),
                                        n_threads or default_threads())
        if rc != 0:
            raise MemoryError("oracle backward failed")
        return dq, dk, dv

    def _expand(self, x, a, r, mask):
        B, H, T, d = x.shape
        heads = np.tile(np.arange(H), B)
        m = (_f64(mask) != 0).astype(np.uint8)
        return heads, m[heads], _f64(a)[heads], _f64(r)[heads]

    def fwd(self, q, k, v, a, r, mask, n_threads: Optional[int] = None):
        """Layer forward on [B,H,T,d] inputs; a, r [H,T]; mask [H].
        Returns (O [B,H,T,d], lse [B,H,T]) in fp64."""
        B, H, T, d = v.shape
        _, rep, ar, rr = self._expand(v, a, r, mask)
        o, lse = self.fwd_slices(_f64(q).reshape(B * H, T, d), _f64(k).reshape(B * H, T, d),
                                 _f64(v).reshape(B * H, T, d), ar, rr, rep, n_threads)
        return o.reshape(B, H, T, d), lse.reshape(B, H, T)

    def bwd(self, q, k, v, dout, a, r, mask, n_threads: Optional[int] = None):
        """Layer backward on [B,H,T,d] inputs.  Returns (dQ, dK, dV) in fp64."""
        B, H, T, d = v.shape
        _, rep, ar, rr = self._expand(v, a, r, mask)
        sh = (B * H, T, d)
        dq, dk, dv = self.bwd_slices(_f64(q).reshape(sh), _f64(k).reshape(sh), _f64(v).reshape(sh),
                                     _f64(dout).reshape(sh), ar, rr, rep, n_threads)
        return dq.reshape(v.shape), dk.reshape(v.shape), dv.reshape(v.shape)

    def fit_pattern(self, target, steps: int = 400, lr: float = 0.1):
        """Fits (alpha, rho) of one head to a target pattern [T,T] by Adam on
        the row-wise cross-entropy.  Returns (alpha [T], rho [T], mean row KL)."""
        t64 = np.ascontiguousarray(_f64(target))
        T = t64.shape[0]
        a, r = np.zeros(T), np.zeros(T)
        kl = ctypes.c_double(0.0)
        if self.lib.oracle_fit_pattern(T, _p(t64), steps, lr, _p(a), _p(r), ctypes.byref(kl)):
            raise MemoryError("oracle pattern fit failed")
        return a, r, kl.value

    def calibration(self, q, k):
        """Calibration statistics of every head over the N samples of q, k
        [N,H,T,d]: (A_hat [H,T,T], s_var [H]) per Eq. (1); N >= 2."""
        q64, k64 = _f64(q), _f64(k)
        N, H, T, d = q64.shape
        if N < 2:
            raise ValueError("Eq. (1) needs N >= 2 samples")
        a_hat = np.zeros((H, T, T))
        svar = np.zeros(H)
        for h in range(H):
            qh, kh = np.ascontiguousarray(q64[:, h]), np.ascontiguousarray(k64[:, h])
            ah = np.zeros((T, T))
            sv = ctypes.c_double(0.0)
            if self.lib.oracle_calibration_head(N, T, d, _p(qh), _p(kh), _p(ah), ctypes.byref(sv)):
                raise MemoryError("oracle calibration failed")
            a_hat[h] = ah
            svar[h] = sv.value
        return a_hat, svar

    def pattern_grad(self, v, dout, a, r, mask):
        """Trainable pattern: (dalpha, drho) [H,T] of a loss with output
        gradient dout through the replaced heads (rows of ordinary heads 0).
        v, dout [B,H,T,d]; sums over the batch (alpha, rho are per head)."""
        v64, do64 = _f64(v), _f64(dout)
        B, H, T, d = v64.shape
        a64, r64 = _f64(a), _f64(r)
        m = _f64(mask) != 0
        da = np.zeros((H, T))
        dr = np.zeros((H, T))
        for h in range(H):
            if not m[h]:
                continue
            ah, rh = np.ascontiguousarray(a64[h]), np.ascontiguousarray(r64[h])
            for b in range(B):
                vb, db = np.ascontiguousarray(v64[b, h]), np.ascontiguousarray(do64[b, h])
                dah, drh = np.zeros(T), np.zeros(T)
                if self.lib.oracle_pattern_grad_slice(T, d, _p(ah), _p(rh), _p(vb), _p(db), _p(dah), _p(drh)):
                    raise MemoryError("oracle pattern gradient failed")
                da[h] += dah
                dr[h] += drh
        return da, dr

    # ---- shared K/V (grouped-query attention): the plain layer with K and V
    # repeated over each group of H / H_kv consecutive query heads; the
    # gradient of a shared head is the sum over its group (each use of an
    # input adds to its gradient).
    @staticmethod
    def _repeat_kv(x, H):
        x64 = _f64(x)
        B, Hkv, T, d = x64.shape
        if H % Hkv:
            raise ValueError("H_kv must divide H")
        return np.ascontiguousarray(np.repeat(x64, H // Hkv, axis=1))

    def fwd_gqa(self, q, k, v, a, r, mask, n_threads: Optional[int] = None):
        """Forward with k, v [B,H_kv,T,d] shared by groups of H / H_kv query heads."""
        H = _f64(q).shape[1]
        return self.fwd(q, self._repeat_kv(k, H), self._repeat_kv(v, H), a, r, mask, n_threads)

    def bwd_gqa(self, q, k, v, dout, a, r, mask, n_threads: Optional[int] = None):
        """Backward with shared K/V.  Returns (dQ [B,H,T,d], dK, dV [B,H_kv,T,d])."""
        q64 = _f64(q)
        B, H, T, d = q64.shape
        Hkv = _f64(k).shape[1]
        dq, dk, dv = self.bwd(q64, self._repeat_kv(k, H), self._repeat_kv(v, H), dout, a, r, mask, n_threads)
        G = H // Hkv
        return dq, dk.reshape(B, Hkv, G, T, d).sum(axis=2), dv.reshape(B, Hkv, G, T, d).sum(axis=2)


_default: Optional[Oracle] = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def lognorm(a, r):
    return default().lognorm(a, r)


def fwd(q, k, v, a, r, mask, n_threads=None):
    return default().fwd(q, k, v, a, r, mask, n_threads)


def bwd(q, k, v, dout, a, r, mask, n_threads=None):
    return default().bwd(q, k, v, dout, a, r, mask, n_threads)


def pattern_grad(v, dout, a, r, mask):
    return default().pattern_grad(v, dout, a, r, mask)


def calibration(q, k):
    return default().calibration(q, k)


def fit_pattern(target, steps=400, lr=0.1):
    return default().fit_pattern(target, steps, lr)


def fwd_gqa(q, k, v, a, r, mask, n_threads=None):
    return default().fwd_gqa(q, k, v, a, r, mask, n_threads)


def bwd_gqa(q, k, v, dout, a, r, mask, n_threads=None):
    return default().bwd_gqa(q, k, v, dout, a, r, mask, n_threads)


def fwd_slices(q, k, v, a_rows, r_rows, replaced, n_threads=None):
    return default().fwd_slices(q, k, v, a_rows, r_rows, replaced, n_threads)


def bwd_slices(q, k, v, dout, a_rows, r_rows, replaced, n_threads=None):
    return default().bwd_slices(q, k, v, dout, a_rows, r_rows, replaced, n_threads)
