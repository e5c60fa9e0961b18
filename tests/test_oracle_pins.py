"""The oracle against what the pages and the mathematics fix (no GPU).

Each pin is a check in ``oracle_pins``; the mutation test below plants
plausible mistakes in a copy of the oracle's C source (on the CPU) and
requires that some pin rejects every one of them.
"""
import json
import os
import shutil
import tempfile

import numpy as np
import pytest

import oracle
from tests import oracle_pins as pins

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def orc():
    return oracle.default()


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(orc, check):
    check(orc)


# (description, exact snippet in saf_oracle.c, replacement, occurrence index)
MUTANTS = [
    ("replaced: diagonal dropped",
     "for (int j = 0; j <= i; ++j) {\n            double p = exp(a[j] + r[i - j] - logz[i]);\n            const double *vj",
     "for (int j = 0; j < i; ++j) {\n            double p = exp(a[j] + r[i - j] - logz[i]);\n            const double *vj", 0),
    ("replaced: a and r roles swapped",
     "double p = exp(a[j] + r[i - j] - logz[i]);\n            const double *vj",
     "double p = exp(a[i - j] + r[j] - logz[i]);\n            const double *vj", 0),
    ("lognorm: distance index wrong",
     "s += exp(a[k] + r[i - k] - L);", "s += exp(a[k] + r[k] - L);", 0),
    ("lognorm: max shift not added back",
     "logz[i] = L + log(s);", "logz[i] = log(s);", 0),
    ("ordinary fwd: scale dropped",
     "srow[j] = scale * dot;", "srow[j] = dot;", 0),
    ("ordinary fwd: lse misses the max",
     "lse[i] = m + log(l);", "lse[i] = log(l);", 0),
    ("ordinary fwd: causal bound off by one",
     "for (int j = 0; j <= i; ++j) {\n            const double *kj = k + (size_t)j * d;\n            double dot = 0.0;\n            for (int c = 0; c < d; ++c) dot += qi[c] * kj[c];\n            srow[j]",
     "for (int j = 0; j <= i && j < T - 1; ++j) {\n            const double *kj = k + (size_t)j * d;\n            double dot = 0.0;\n            for (int c = 0; c < d; ++c) dot += qi[c] * kj[c];\n            srow[j]", 0),
    ("ordinary bwd: D term dropped",
     "double ds = prow[j] * (dprow[j] - D);", "double ds = prow[j] * dprow[j];", 0),
    ("ordinary bwd: dK uses K instead of Q",
     "dkj[c] += scale * ds * qi[c];", "dkj[c] += scale * ds * kj[c];", 0),
    ("ordinary bwd: dQ sign flipped",
     "dqi[c] += scale * ds * kj[c];", "dqi[c] -= scale * ds * kj[c];", 0),
    ("ordinary bwd: dV uses Q instead of dO",
     "dvj[c] += prow[j] * doi[c];", "dvj[c] += prow[j] * qi[c];", 0),
    ("ordinary bwd: scale dropped in dQ",
     "dqi[c] += scale * ds * kj[c];", "dqi[c] += ds * kj[c];", 0),
    ("replaced bwd: normaliser of the wrong row",
     "double p = exp(a[j] + r[i - j] - logz[i]);\n            double *dvj",
     "double p = exp(a[j] + r[i - j] - logz[j]);\n            double *dvj", 0),
    ("pattern grad: distance bin of the key",
     "dr[i - j] += ds;", "dr[j] += ds;", 0),
    ("pattern grad: row term D dropped",
     "const double ds = prow[j] * (dprow[j] - Di);", "const double ds = prow[j] * dprow[j];", 0),
    ("pattern grad: dP from the wrong row of V",
     "const double *vj = v + (size_t)j * d;\n            double dp = 0.0;",
     "const double *vj = v + (size_t)i * d;\n            double dp = 0.0;", 0),
    ("calibration: mean over N - 1",
     "a_hat[e] = sum / N;", "a_hat[e] = sum / (N - 1);", 0),
    ("calibration: Eq. (1) normalised by N",
     "*svar = err / ((double)(N - 1) * (double)T * (double)T);", "*svar = err / ((double)N * (double)T * (double)T);", 0),
    ("calibration: scores not scaled",
     "srow[j] = scale * dot;\n                if (srow[j] > m) m = srow[j];\n            }\n            double l = 0.0;\n            for (int j = 0; j <= i; ++j) l += exp(srow[j] - m);\n            for (int j = 0; j < T; ++j) an",
     "srow[j] = dot;\n                if (srow[j] > m) m = srow[j];\n            }\n            double l = 0.0;\n            for (int j = 0; j <= i; ++j) l += exp(srow[j] - m);\n            for (int j = 0; j < T; ++j) an", 0),
    ("fit: distance statistic of the key",
     "nd[i - j] += x;", "nd[j] += x;", 0),
    ("fit: gradient sign flipped",
     "const double g = e < T ? -(m[e] - cs[e]) / T : -(nd[e - T] - ds[e - T]) / T;",
     "const double g = e < T ? (m[e] - cs[e]) / T : (nd[e - T] - ds[e - T]) / T;", 0),
    ("fit: KL without the entropy term",
     "*kl = (-loss + ent) / T;", "*kl = -loss / T;", 0),
    ("replaced bwd: dQ not cleared",
     "memset(dq, 0, sizeof(double) * (size_t)T * d);\n    memset(dk, 0, sizeof(double) * (size_t)T * d);\n    memset(dv, 0, sizeof(double) * (size_t)T * d);\n    for (int i = 0; i < T; ++i) {\n        if (logz",
     "for (int c = 0; c < T * d; ++c) dq[c] = 1e-3 * c;\n    memset(dk, 0, sizeof(double) * (size_t)T * d);\n    memset(dv, 0, sizeof(double) * (size_t)T * d);\n    for (int i = 0; i < T; ++i) {\n        if (logz", 0),
]


def _replace_nth(text, old, new, n):
    start = -1
    for _ in range(n + 1):
        start = text.find(old, start + 1)
        assert start >= 0, f"snippet not found: {old!r}"
    return text[:start] + new + text[start + len(old):]


@pytest.mark.parametrize("desc,old,new,nth", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(desc, old, new, nth):
    src = open(oracle.SOURCE).read()
    mutated = _replace_nth(src, old, new, nth)
    assert mutated != src
    tmp = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        csrc = os.path.join(tmp, "m.c")
        with open(csrc, "w") as f:
            f.write(mutated)
        mut = oracle.Oracle(oracle.compile_library(csrc, os.path.join(tmp, "m.so")))
        caught = []
        for check in pins.ALL_CHECKS:
            try:
                check(mut)
            except AssertionError:
                caught.append(check.__name__)
        assert caught, f"no pin rejects the planted mistake: {desc}"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)


@pytest.mark.parametrize("mistake", ["groups interleaved", "first head of the group only"])
def test_planted_grouped_kv_mistake_is_caught(mistake, monkeypatch):
    """Plausible mistakes in the shared-K/V marshalling (query head h reading
    K/V head h % H_kv, or a shared head's gradient taken from one query head
    instead of the group sum) are rejected by the grouped-K/V pin."""
    orc = oracle.Oracle()
    if mistake == "groups interleaved":
        def bad_repeat(x, H):
            x64 = np.asarray(x, dtype=np.float64)
            return np.ascontiguousarray(np.tile(x64, (1, H // x64.shape[1], 1, 1)))
        monkeypatch.setattr(oracle.Oracle, "_repeat_kv", staticmethod(bad_repeat))
    else:
        good_bwd = oracle.Oracle.bwd_gqa

        def bad_bwd(self, q, k, v, dout, a, r, mask, n_threads=None):
            dq, dk, dv = good_bwd(self, q, k, v, dout, a, r, mask, n_threads)
            B, H, T, d = np.asarray(q).shape
            Hkv = np.asarray(k).shape[1]
            full = self.bwd(q, self._repeat_kv(k, H), self._repeat_kv(v, H), dout, a, r, mask, n_threads)
            G = H // Hkv
            return dq, full[1][:, ::G], full[2][:, ::G]
        monkeypatch.setattr(oracle.Oracle, "bwd_gqa", bad_bwd)
    with pytest.raises(AssertionError):
        pins.check_grouped_kv_matches_autograd(orc)


def test_golden_regression(orc):
    """Frozen oracle outputs on a tiny mixed case (tests/golden/make_golden.py)."""
    path = os.path.join(HERE, "golden", "tiny_mixed_layer.json")
    with open(path) as f:
        g = json.load(f)
    arr = {k: np.asarray(v, dtype=np.float64) for k, v in g["inputs"].items()}
    o, lse = orc.fwd(arr["q"], arr["k"], arr["v"], arr["alpha"], arr["rho"], arr["mask"].astype(np.uint8))
    dq, dk, dv = orc.bwd(arr["q"], arr["k"], arr["v"], arr["do"], arr["alpha"], arr["rho"],
                         arr["mask"].astype(np.uint8))
    for name, got in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
        np.testing.assert_allclose(got, np.asarray(g["outputs"][name]), rtol=1e-12, atol=1e-13, err_msg=name)
