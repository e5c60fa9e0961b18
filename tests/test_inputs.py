"""The seeded input generator: determinism and the stated recipe (no GPU)."""
import torch

from mixed_head_causal_b200 import inputs as I


def test_workloads_present():
    assert set(I.PREFILL_SWEEP) == {n for n in I.WORKLOADS if n.startswith("prefill_")}
    assert len(I.PREFILL_SWEEP) == 10
    w = I.WORKLOADS["124m_b8_t4096_r25"]
    assert (w.B, w.H, w.T, w.d, w.n_replaced) == (8, 12, 4096, 64, 3)


def test_slices_deterministic_and_distinct():
    w = I.custom(2, 3, 40, [1])
    a = I.make_tensor(w, 0, "q")
    b = I.make_tensor(w, 0, "q")
    assert torch.equal(a, b) and a.dtype == torch.bfloat16
    assert torch.equal(a[1, 2], I.make_slice(w, 0, "q", 1, 2))
    assert not torch.equal(a[0, 0], a[0, 1])
    assert not torch.equal(I.make_tensor(w, 0, "k"), a)
    assert not torch.equal(I.make_tensor(w, 1, "q"), a)


def test_pattern_recipe():
    w = I.WORKLOADS["124m_b8_t4096_r25"]
    heads = I.replaced_heads(w, 0)
    assert len(heads) == 3 and heads == sorted(heads)
    a, r = I.make_pattern(w, 0)
    for h in range(w.H):
        if h in heads:
            assert torch.isfinite(a[h]).all() and torch.isfinite(r[h]).all()
            # sink at a[0]; r decays by 0.05 per step with a +2 bump at distance 0
            assert a[h, 0] > a[h, 1:].max()
            assert abs(float(a[h, 1:].std()) - 0.5) < 0.03
            resid = r[h, 1:] + 0.05 * torch.arange(1, w.T)
            assert abs(float(resid.std()) - 0.3) < 0.02
        else:
            assert torch.isnan(a[h]).all() and torch.isnan(r[h]).all()
    assert I.replaced_heads(I.WORKLOADS["tiny_b1_h4_t256"]) == [2]


def test_flops_convention():
    w = I.WORKLOADS["124m_b8_t4096_r25"]
    f = I.flops(w)
    assert abs(f["total"] - 8 * (9 * 7 + 3 * 2) * 64 * 4096 ** 2) < 1
    # the strict count drops the backward's recompute of Q K^T: ordinary 6 units, replaced 2
    s = I.flops(w, strict=True)
    assert abs(s["total"] - 8 * (9 * 6 + 3 * 2) * 64 * 4096 ** 2) < 1
    assert s["fwd"] == f["fwd"]
    fo = I.flops(I.WORKLOADS["prefill_124m_b64_t4096"], strict=True)
    assert fo["bwd"] == 0.0 and fo["total"] == I.flops(I.WORKLOADS["prefill_124m_b64_t4096"])["total"]
