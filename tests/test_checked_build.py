"""The index-checked build of the library (libsaf_checked.so: the kernels'
SAF_CHECKED_OK checks compiled in, each recording a failed check in the
workspace error word and skipping the access it guards).  On the GPU it runs
the layer on ragged, multi-tile and all-replaced shapes with both error words
clear afterwards and results that match the oracle; on the CPU it must build
and export the same entry points as the regular library."""
import pytest
import torch

from mixed_head_causal_b200 import build as saf_build
from mixed_head_causal_b200 import inputs as I
from mixed_head_causal_b200 import saf
from tests import parity as P


@pytest.fixture(scope="module")
def checked_lib():
    return saf.load(saf_build.build(checked=True))


def test_checked_library_exports_the_boundary(checked_lib):
    for name in saf.SIGNATURES:
        assert hasattr(checked_lib, name), name


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,T,replaced,grad", [
    (1, 3, 300, [1], torch.float32),
    (2, 4, 1000, [0, 3], torch.bfloat16),
    (1, 2, 129, [0, 1], torch.float32),
    (2, 2, 2100, [1], torch.bfloat16),
    (3, 3, 640, [], torch.float32),
], ids=["t300", "t1000_bf16", "t129_all_replaced", "t2100_bf16", "t640_no_replaced"])
def test_checked_build_runs_clean(checked_lib, monkeypatch, B, H, T, replaced, grad):
    monkeypatch.setattr(saf, "_lib", checked_lib)
    w = I.custom(B, H, T, replaced)
    x = I.make_inputs(w, 77)
    g = P.to_gpu(x)
    wsf = saf.new_workspace(B, H, T, "cuda")
    wsb = saf.new_workspace(B, H, T, "cuda", backward=True)
    o, lse = saf.mixed_attn_fwd(g["q"], g["k"], g["v"], g["alpha"], g["rho"], x["mask"], workspace=wsf)
    dq, dk, dv = saf.mixed_attn_bwd(g["q"], g["k"], g["v"], o, g["do"], lse, g["alpha"], g["rho"], x["mask"],
                                    grad_dtype=grad, workspace=wsb)
    torch.cuda.synchronize()
    for ws in (wsf, wsb):
        err = ws[:8].view(torch.int32).cpu()
        assert int(err[0]) == 0 and int(err[1]) == 0, (hex(int(err[0])), hex(int(err[1])))
    got = {"o": o.cpu(), "lse": lse.cpu(), "dq": dq.cpu(), "dk": dk.cpu(), "dv": dv.cpu()}
    P.check_slices(w, x, got, [(b, h) for b in range(B) for h in range(H)], grad_dtype=grad)
