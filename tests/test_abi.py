"""The C-ABI library without a GPU: it loads, exports every symbol that
include/saf.h declares, and rejects bad arguments on the host before any CUDA
call (no compute call is made here)."""
import ctypes
import os
import re

import pytest

from mixed_head_causal_b200 import build as saf_build
from mixed_head_causal_b200 import saf

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "saf.h")


@pytest.fixture(scope="module")
def lib():
    saf_build.build()
    return saf.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SAF_API\s+[\w\s\*]*?\b(saf_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for want in ("saf_mixed_attn_fwd", "saf_mixed_attn_bwd", "saf_replaced_lognorm",
                 "saf_workspace_size", "saf_status_string", "saf_device_status"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert name in saf.SIGNATURES, f"binding lacks {name}"


def test_status_strings(lib):
    assert saf.status_string(0) == "SAF_OK"
    assert saf.status_string(5) == "SAF_ERR_TIMEOUT"
    assert saf.status_string(99) == "SAF_ERR_UNKNOWN"
    assert lib.saf_version() >= 100


def test_workspace_size(lib):
    assert lib.saf_workspace_size(0, 12, 4096, 64, 0) == 0
    n_f = lib.saf_workspace_size(8, 12, 4096, 64, 0)
    n_b = lib.saf_workspace_size(8, 12, 4096, 64, 1)
    assert 0 < n_f <= n_b
    assert n_b >= 8 * 12 * 4096 * 4  # the backward's per-row fp32 term
    assert lib.saf_workspace_size(1, 1, 1, 32, 0) == ctypes.c_size_t(-1).value
    assert lib.saf_workspace_size(-1, 1, 1, 64, 0) == ctypes.c_size_t(-1).value


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails validation first


def _mask(h, val=0):
    return (ctypes.c_uint8 * h)(*([val] * h))


def _fwd(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, a=FAKE, r=FAKE, logz=None, mask="x", B=1, H=2,
         T=16, d=64, ws=FAKE, wsb=None):
    m = _mask(H, 1) if mask == "x" else mask
    if wsb is None:
        wsb = lib.saf_workspace_size(B, H, T, 64, 0)
    return lib.saf_mixed_attn_fwd(q, k, v, o, lse, a, r, logz, m, B, H, T, d, ws, wsb, None)


def test_fwd_argument_errors(lib):
    assert _fwd(lib, d=128) == saf.SAF_ERR_UNSUPPORTED
    assert _fwd(lib, q=None) == saf.SAF_ERR_INVALID_ARG
    assert _fwd(lib, o=FAKE + 2) == saf.SAF_ERR_INVALID_ARG
    assert _fwd(lib, a=None) == saf.SAF_ERR_INVALID_ARG          # replaced heads need a
    assert _fwd(lib, mask=None) == saf.SAF_ERR_INVALID_ARG
    assert _fwd(lib, ws=None) == saf.SAF_ERR_WORKSPACE
    assert _fwd(lib, wsb=16) == saf.SAF_ERR_WORKSPACE
    assert _fwd(lib, ws=FAKE + 16) == saf.SAF_ERR_INVALID_ARG    # workspace must be 256-aligned
    assert _fwd(lib, B=-1) == saf.SAF_ERR_INVALID_ARG
    assert _fwd(lib, T=1 << 30) == saf.SAF_ERR_INVALID_ARG
    assert _fwd(lib, H=100000, mask=_mask(1)) == saf.SAF_ERR_UNSUPPORTED


def test_empty_problem_enqueues_nothing(lib):
    # nothing is dereferenced or launched for an empty problem
    assert _fwd(lib, B=0, q=None, k=None, v=None, o=None, lse=None, ws=None) == saf.SAF_OK
    assert _fwd(lib, T=0, q=None, k=None, v=None, o=None, lse=None, ws=None) == saf.SAF_OK
    assert lib.saf_mixed_attn_bwd(None, None, None, None, None, None, None, None, None, _mask(2), 3, 2, 0, 64,
                                  None, None, None, 0, None, 0, None) == saf.SAF_OK


def test_bwd_argument_errors(lib):
    B, H, T = 1, 2, 16
    wsb = lib.saf_workspace_size(B, H, T, 64, 1)

    def call(**kw):
        args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, do=FAKE, lse=FAKE, a=FAKE, r=FAKE, logz=None,
                    mask=_mask(H, 1), dq=FAKE, dk=FAKE, dv=FAKE, gd=0, ws=FAKE, wsb=wsb, d=64)
        args.update(kw)
        return lib.saf_mixed_attn_bwd(args["q"], args["k"], args["v"], args["o"], args["do"], args["lse"],
                                      args["a"], args["r"], args["logz"], args["mask"], B, H, T, args["d"],
                                      args["dq"], args["dk"], args["dv"], args["gd"], args["ws"],
                                      args["wsb"], None)

    assert call(gd=2) == saf.SAF_ERR_UNSUPPORTED
    assert call(d=32) == saf.SAF_ERR_UNSUPPORTED
    assert call(do=None) == saf.SAF_ERR_INVALID_ARG
    assert call(dv=FAKE + 4) == saf.SAF_ERR_INVALID_ARG
    assert call(r=None) == saf.SAF_ERR_INVALID_ARG
    assert call(wsb=wsb - 1) == saf.SAF_ERR_WORKSPACE


def test_lognorm_argument_errors(lib):
    assert lib.saf_replaced_lognorm(None, FAKE, _mask(2, 1), 2, 8, FAKE, None) == saf.SAF_ERR_INVALID_ARG
    assert lib.saf_replaced_lognorm(FAKE, FAKE, None, 2, 8, FAKE, None) == saf.SAF_ERR_INVALID_ARG
    # no replaced head: nothing to do, nothing read
    assert lib.saf_replaced_lognorm(None, None, _mask(2, 0), 2, 8, None, None) == saf.SAF_OK


def test_device_status_argument_errors(lib):
    assert lib.saf_device_status(None, 256, None) == saf.SAF_ERR_WORKSPACE
    assert lib.saf_device_status(FAKE, 4, None) == saf.SAF_ERR_WORKSPACE


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(RuntimeError, match="no fallback"):
        saf.load(str(tmp_path / "missing.so"))


def test_selftest_argument_errors(lib):
    assert lib.saf_selftest_wait_timeout(None, 256, 1000, None) == saf.SAF_ERR_WORKSPACE
    assert lib.saf_selftest_wait_timeout(FAKE, 16, 1000, None) == saf.SAF_ERR_WORKSPACE
    assert lib.saf_selftest_wait_timeout(FAKE, 256, 0, None) == saf.SAF_ERR_INVALID_ARG
    assert lib.saf_selftest_wait_timeout(FAKE, 256, 1 << 40, None) == saf.SAF_ERR_INVALID_ARG


def test_nvtx_ranges_are_opt_in(monkeypatch):
    """With SAF_NVTX=1 each binding call is one NVTX range (pushed and popped
    even when the call raises); without it no NVTX call is made."""
    import torch

    calls = []
    monkeypatch.setattr(torch.cuda.nvtx, "range_push", lambda name: calls.append(("push", name)))
    monkeypatch.setattr(torch.cuda.nvtx, "range_pop", lambda: calls.append(("pop",)))
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    k_bad = torch.zeros(1, 2, 9, 64, dtype=torch.bfloat16)  # T mismatch: rejected before the library
    a = torch.zeros(2, 8)
    monkeypatch.delenv("SAF_NVTX", raising=False)
    with pytest.raises(ValueError):
        saf.mixed_attn_fwd(q, k_bad, k_bad, a, a, [0, 1])
    assert calls == []
    monkeypatch.setenv("SAF_NVTX", "1")
    with pytest.raises(ValueError):
        saf.mixed_attn_fwd(q, k_bad, k_bad, a, a, [0, 1])
    assert calls == [("push", "saf.mixed_attn_fwd"), ("pop",)]
