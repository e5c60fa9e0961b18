"""Pins for the fp64 oracle, written as plain check functions so that the same
checks can be run against planted mutants of the oracle source.

Every check ties the oracle to something other than itself:
  * closed forms of Eq. (3) of "When Can Attention Heads Be Statically
    Defined?" (reading notes, section 二.3) for special a / r,
  * invariants the same equation fixes (row sums, causality, shift
    invariance, T = 1),
  * library routines (torch's scaled_dot_product_attention and autograd in
    fp64, numpy's convolution, scipy's logsumexp),
  * central finite differences of the oracle's own forward.
"""
from __future__ import annotations

import numpy as np
import torch
from scipy.special import logsumexp

NEG_INF = -np.inf


def _rng(seed):
    return np.random.default_rng(seed)


def _pattern(T, rng):
    a = rng.normal(0.0, 0.5, T)
    a[0] += 4.0
    r = -0.05 * np.arange(T) + rng.normal(0.0, 0.3, T)
    r[0] += 2.0
    return a, r


def _pattern_matrix(orc, a, r):
    """P of one replaced head, read off the oracle by feeding V = identity."""
    T = a.shape[0]
    eye = np.eye(T)[None]
    zeros = np.zeros_like(eye)
    o, lse = orc.fwd_slices(zeros, zeros, eye, a[None], r[None], [1])
    return o[0], lse[0]


def _dense_pattern(a, r):
    """Brute force: the T x T masked logit matrix, row-normalised with scipy."""
    T = a.shape[0]
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    logits = np.where(j <= i, a[None, :] + r[np.clip(i - j, 0, T - 1)], NEG_INF)
    lz = logsumexp(logits, axis=1)
    return np.exp(logits - lz[:, None]), lz


# ------------------------------------------------------------- replaced heads

def check_pattern_is_causal_distribution(orc):
    rng = _rng(1)
    for T in (1, 2, 17, 48):
        a, r = _pattern(T, rng)
        P, lse = _pattern_matrix(orc, a, r)
        assert np.all(P >= 0)
        assert np.all(np.triu(P, 1) == 0.0), "weight on a future position"
        np.testing.assert_allclose(P.sum(1), 1.0, rtol=0, atol=1e-13)
        assert P[0, 0] == 1.0
        Pd, lz = _dense_pattern(a, r)
        np.testing.assert_allclose(P, Pd, rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse, lz, rtol=1e-14, atol=1e-13)


def check_uniform_pattern_is_running_mean(orc):
    rng = _rng(2)
    T, d = 37, 8
    v = rng.normal(size=(1, T, d))
    z = np.zeros((1, T))
    o, lse = orc.fwd_slices(np.zeros_like(v), np.zeros_like(v), v, z, z, [1])
    mean = np.cumsum(v[0], axis=0) / np.arange(1, T + 1)[:, None]
    np.testing.assert_allclose(o[0], mean, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[0], np.log(np.arange(1, T + 1)), rtol=0, atol=1e-13)


def check_identity_pattern(orc):
    """r one-hot at distance 0 (r[0] = 0, r[d > 0] = -inf): P = I for any a."""
    rng = _rng(3)
    T, d = 29, 8
    a = rng.normal(size=(1, T)) * 3
    r = np.full((1, T), NEG_INF)
    r[0, 0] = 0.0
    v = rng.normal(size=(1, T, d))
    do = rng.normal(size=(1, T, d))
    q = rng.normal(size=(1, T, d))
    o, lse = orc.fwd_slices(q, q, v, a, r, [1])
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0], a[0], rtol=0, atol=1e-14)
    dq, dk, dv = orc.bwd_slices(q, q, v, do, a, r, [1])
    np.testing.assert_allclose(dv, do, rtol=0, atol=1e-14)
    assert np.all(dq == 0) and np.all(dk == 0)


def check_sink_pattern(orc):
    """a one-hot at j = 0: every row puts all mass on key 0, so O[i] = V[0]
    and dV[0] = sum_i dO[i], dV[j > 0] = 0."""
    rng = _rng(4)
    T, d = 23, 8
    a = np.full((1, T), NEG_INF)
    a[0, 0] = 0.0
    r = rng.normal(size=(1, T))
    v = rng.normal(size=(1, T, d))
    do = rng.normal(size=(1, T, d))
    z = np.zeros_like(v)
    o, lse = orc.fwd_slices(z, z, v, a, r, [1])
    np.testing.assert_allclose(o[0], np.broadcast_to(v[0, 0], (T, d)), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0], r[0], rtol=0, atol=1e-14)
    _, _, dv = orc.bwd_slices(z, z, v, do, a, r, [1])
    np.testing.assert_allclose(dv[0, 0], do[0].sum(0), rtol=0, atol=1e-12)
    assert np.all(dv[0, 1:] == 0)


def check_shift_invariance(orc):
    rng = _rng(5)
    T, d = 40, 8
    a, r = _pattern(T, rng)
    v = rng.normal(size=(1, T, d))
    do = rng.normal(size=(1, T, d))
    z = np.zeros_like(v)
    o0, l0 = orc.fwd_slices(z, z, v, a[None], r[None], [1])
    _, _, dv0 = orc.bwd_slices(z, z, v, do, a[None], r[None], [1])
    for ca, cr in ((1000.0, 0.0), (0.0, -1000.0), (-1000.0, 1000.0)):
        o1, l1 = orc.fwd_slices(z, z, v, (a + ca)[None], (r + cr)[None], [1])
        _, _, dv1 = orc.bwd_slices(z, z, v, do, (a + ca)[None], (r + cr)[None], [1])
        np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-10)
        np.testing.assert_allclose(dv1, dv0, rtol=0, atol=1e-10)
        np.testing.assert_allclose(l1 - (ca + cr), l0, rtol=0, atol=1e-9)


def check_geometric_closed_form(orc):
    """a = 0, r[d] = -lam d: P(i,j) = e^{-lam(i-j)} (1 - e^{-lam}) / (1 - e^{-lam(i+1)})."""
    T = 33
    for lam in (0.05, 0.7, 3.0):
        a = np.zeros(T)
        r = -lam * np.arange(T)
        P, _ = _pattern_matrix(orc, a, r)
        i = np.arange(T)[:, None]
        j = np.arange(T)[None, :]
        ref = np.where(j <= i, np.exp(-lam * (i - j)) * (1 - np.exp(-lam)) / (1 - np.exp(-lam * (i + 1))), 0.0)
        np.testing.assert_allclose(P, ref, rtol=1e-12, atol=1e-15)


def check_lognorm_is_causal_convolution(orc):
    """Z(i) = sum_k e^{a[k]} e^{r[i-k]}: a causal convolution (numpy.convolve)."""
    rng = _rng(6)
    T = 200
    a, r = _pattern(T, rng)
    lz = orc.lognorm(a, r)
    ref = np.log(np.convolve(np.exp(a), np.exp(r))[:T])
    np.testing.assert_allclose(lz, ref, rtol=1e-13, atol=1e-12)
    # [H, T] form, one row per head
    A = np.stack([a, a[::-1].copy()])
    R = np.stack([r, r + 1.0])
    lz2 = orc.lognorm(A, R)
    np.testing.assert_allclose(lz2[0], ref, rtol=1e-13, atol=1e-12)
    ref2 = np.log(np.convolve(np.exp(A[1]), np.exp(R[1]))[:T])
    np.testing.assert_allclose(lz2[1], ref2, rtol=1e-13, atol=1e-12)


def check_replaced_backward_is_pattern_transpose(orc):
    rng = _rng(7)
    T, d = 31, 8
    a, r = _pattern(T, rng)
    P, _ = _pattern_matrix(orc, a, r)
    do = rng.normal(size=(1, T, d))
    v = rng.normal(size=(1, T, d))
    q = rng.normal(size=(1, T, d))
    dq, dk, dv = orc.bwd_slices(q, q, v, do, a[None], r[None], [1])
    np.testing.assert_allclose(dv[0], P.T @ do[0], rtol=0, atol=1e-13)
    assert np.all(dq == 0) and np.all(dk == 0)
    o, _ = orc.fwd_slices(q, q, v, a[None], r[None], [1])
    np.testing.assert_allclose(o[0], P @ v[0], rtol=0, atol=1e-13)


def check_replaced_finite_differences(orc):
    """dV of loss = sum(O * dO) against central differences of the forward;
    the forward must not depend on Q or K at all."""
    rng = _rng(8)
    T, d = 7, 3
    a, r = _pattern(T, rng)
    q, k, v, do = (rng.normal(size=(1, T, d)) for _ in range(4))
    A, R = a[None], r[None]

    def loss(vv, qq=q, kk=k):
        o, _ = orc.fwd_slices(qq, kk, vv, A, R, [1])
        return float((o * do).sum())

    _, _, dv = orc.bwd_slices(q, k, v, do, A, R, [1])
    h = 1e-6
    num = np.zeros_like(v)
    for idx in np.ndindex(v.shape):
        vp, vm = v.copy(), v.copy()
        vp[idx] += h
        vm[idx] -= h
        num[idx] = (loss(vp) - loss(vm)) / (2 * h)
    np.testing.assert_allclose(dv, num, rtol=0, atol=1e-7)
    assert loss(v, q * 3.0 + 1.0, -k) == loss(v)


# ------------------------------------------------------------- ordinary heads

def _sdpa(q, k, v):
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)


def check_ordinary_matches_sdpa(orc):
    g = torch.Generator().manual_seed(9)
    for T, d in ((1, 8), (19, 8), (64, 64), (130, 16)):
        q, k, v = (torch.randn(1, T, d, generator=g, dtype=torch.float64) * 1.5 for _ in range(3))
        nan = np.full((1, T), np.nan)
        o, lse = orc.fwd_slices(q, k, v, nan, nan, [0])
        ref = _sdpa(q[None], k[None], v[None])[0]
        np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)
        s = (q[0] @ k[0].T) / np.sqrt(d)
        s = s.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), 1), float("-inf"))
        np.testing.assert_allclose(lse[0], torch.logsumexp(s, dim=1).numpy(), rtol=0, atol=1e-12)


def check_ordinary_grads_match_autograd(orc):
    g = torch.Generator().manual_seed(10)
    for T, d in ((1, 4), (13, 8), (70, 16)):
        q, k, v, do = (torch.randn(1, T, d, generator=g, dtype=torch.float64) for _ in range(4))
        qq, kk, vv = (x.clone().requires_grad_(True) for x in (q, k, v))
        (_sdpa(qq[None], kk[None], vv[None])[0] * do).sum().backward()
        nan = np.full((1, T), np.nan)
        dq, dk, dv = orc.bwd_slices(q, k, v, do, nan, nan, [0])
        np.testing.assert_allclose(dq, qq.grad.numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dk, kk.grad.numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dv, vv.grad.numpy(), rtol=0, atol=1e-11)


def check_ordinary_finite_differences(orc):
    rng = _rng(11)
    T, d = 6, 4
    q, k, v, do = (rng.normal(size=(1, T, d)) for _ in range(4))
    nan = np.full((1, T), np.nan)

    def loss(qq, kk, vv):
        o, _ = orc.fwd_slices(qq, kk, vv, nan, nan, [0])
        return float((o * do).sum())

    grads = orc.bwd_slices(q, k, v, do, nan, nan, [0])
    h = 1e-6
    for which, g in enumerate(grads):
        num = np.zeros_like(q)
        for idx in np.ndindex(q.shape):
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=0, atol=1e-7)


def check_zero_query_is_running_mean(orc):
    rng = _rng(12)
    T, d = 21, 8
    v = rng.normal(size=(1, T, d))
    k = rng.normal(size=(1, T, d))
    nan = np.full((1, T), np.nan)
    o, lse = orc.fwd_slices(np.zeros_like(v), k, v, nan, nan, [0])
    mean = np.cumsum(v[0], axis=0) / np.arange(1, T + 1)[:, None]
    np.testing.assert_allclose(o[0], mean, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[0], np.log(np.arange(1, T + 1)), rtol=0, atol=1e-13)


# ------------------------------------------------------------- whole layer

def check_layer_mixes_head_kinds(orc):
    """[B, H] marshalling: each head uses its own pattern row; ordinary heads
    never read theirs (NaN rows); equals the dense brute force head by head."""
    g = torch.Generator().manual_seed(13)
    B, H, T, d = 2, 3, 24, 8
    q, k, v, do = (torch.randn(B, H, T, d, generator=g, dtype=torch.float64) for _ in range(4))
    rng = _rng(13)
    a = np.full((H, T), np.nan)
    r = np.full((H, T), np.nan)
    mask = np.array([0, 1, 1], dtype=np.uint8)
    for h in (1, 2):
        a[h], r[h] = _pattern(T, rng)
        r[h] *= h  # distinct rows
    o, lse = orc.fwd(q, k, v, a, r, mask)
    dq, dk, dv = orc.bwd(q, k, v, do, a, r, mask)
    assert np.isfinite(o).all() and np.isfinite(dq).all() and np.isfinite(dv).all()
    for b in range(B):
        qq, kk, vv = (x[b, 0].clone().requires_grad_(True) for x in (q, k, v))
        ref = _sdpa(qq[None, None], kk[None, None], vv[None, None])[0, 0]
        (ref * do[b, 0]).sum().backward()
        np.testing.assert_allclose(o[b, 0], ref.detach().numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(dq[b, 0], qq.grad.numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dk[b, 0], kk.grad.numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dv[b, 0], vv.grad.numpy(), rtol=0, atol=1e-11)
        for h in (1, 2):
            P, lz = _dense_pattern(a[h], r[h])
            np.testing.assert_allclose(o[b, h], P @ v[b, h].numpy(), rtol=0, atol=1e-13)
            np.testing.assert_allclose(lse[b, h], lz, rtol=1e-14, atol=1e-13)
            np.testing.assert_allclose(dv[b, h], P.T @ do[b, h].numpy(), rtol=0, atol=1e-13)
            assert np.all(dq[b, h] == 0) and np.all(dk[b, h] == 0)


def check_grouped_kv_matches_autograd(orc):
    """Shared K/V (H_kv = 2 heads, groups of 2 query heads, one replaced head in
    each group): forward and backward against fp64 torch autograd of a dense
    layer that indexes the shared K/V per query head (autograd sums the
    gradient of each shared head over its uses by itself)."""
    g = torch.Generator().manual_seed(14)
    B, H, Hkv, T, d = 2, 4, 2, 20, 8
    G = H // Hkv
    q, do = (torch.randn(B, H, T, d, generator=g, dtype=torch.float64) for _ in range(2))
    k, v = (torch.randn(B, Hkv, T, d, generator=g, dtype=torch.float64) for _ in range(2))
    rng = _rng(14)
    a = np.full((H, T), np.nan)
    r = np.full((H, T), np.nan)
    mask = np.array([0, 1, 0, 1], dtype=np.uint8)
    for h in (1, 3):
        a[h], r[h] = _pattern(T, rng)
        r[h] *= 0.5 * h
    o, lse = orc.fwd_gqa(q, k, v, a, r, mask)
    dq, dk, dv = orc.bwd_gqa(q, k, v, do, a, r, mask)
    assert dk.shape == (B, Hkv, T, d) and dv.shape == (B, Hkv, T, d)
    qq, kk, vv = (x.clone().requires_grad_(True) for x in (q, k, v))
    outs = []
    for b in range(B):
        for h in range(H):
            kv = h // G
            if mask[h]:
                P, _ = _dense_pattern(a[h], r[h])
                outs.append(torch.from_numpy(P) @ vv[b, kv])
            else:
                outs.append(_sdpa(qq[b, h][None, None], kk[b, kv][None, None], vv[b, kv][None, None])[0, 0])
    ref = torch.stack(outs).reshape(B, H, T, d)
    (ref * do).sum().backward()
    np.testing.assert_allclose(o, ref.detach().numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dq, qq.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dk, kk.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dv, vv.grad.numpy(), rtol=0, atol=1e-11)
    for h in (1, 3):
        assert np.all(dq[:, h] == 0)


def _dense_pattern_torch_grads(a, r, v, do):
    """fp64 torch autograd of L = sum(O o dO), O = P V, P the row softmax of the
    masked logits a[j] + r[i-j] (a library routine differentiates Eq. (3))."""
    T = a.shape[0]
    at = torch.tensor(a, dtype=torch.float64, requires_grad=True)
    rt = torch.tensor(r, dtype=torch.float64, requires_grad=True)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    logits = at[j.expand(T, T)] + rt[(i - j).clamp(min=0)]
    logits = logits.masked_fill(j > i, float("-inf"))
    P = torch.softmax(logits, dim=1)
    loss = sum(((P @ torch.as_tensor(vb)) * torch.as_tensor(db)).sum() for vb, db in zip(v, do))
    loss.backward()
    return at.grad.numpy(), rt.grad.numpy()


def check_pattern_grad_matches_autograd(orc):
    """Trainable pattern: dalpha, drho summed over the batch, per head, against
    torch autograd of the dense definition; ordinary heads' rows stay 0."""
    rng = _rng(15)
    B, H, T, d = 2, 3, 21, 6
    v, do = rng.normal(size=(B, H, T, d)), rng.normal(size=(B, H, T, d))
    a = np.full((H, T), np.nan)
    r = np.full((H, T), np.nan)
    mask = np.array([1, 0, 1], dtype=np.uint8)
    for h in (0, 2):
        a[h], r[h] = _pattern(T, rng)
        r[h] *= 1 + h
    da, dr = orc.pattern_grad(v, do, a, r, mask)
    assert np.all(da[1] == 0) and np.all(dr[1] == 0)
    for h in (0, 2):
        ga, gr = _dense_pattern_torch_grads(a[h], r[h], v[:, h], do[:, h])
        np.testing.assert_allclose(da[h], ga, rtol=0, atol=1e-12)
        np.testing.assert_allclose(dr[h], gr, rtol=0, atol=1e-12)


def check_pattern_grad_finite_differences(orc):
    """Central differences of L = sum(O o dO) through the oracle's own forward."""
    rng = _rng(16)
    T, d = 7, 3
    a, r = _pattern(T, rng)
    v, do = rng.normal(size=(1, 1, T, d)), rng.normal(size=(1, 1, T, d))
    da, dr = orc.pattern_grad(v, do, a[None], r[None], np.array([1], dtype=np.uint8))
    z = np.zeros((1, T, d))

    def loss(aa, rr):
        o, _ = orc.fwd_slices(z, z, v[0], aa[None], rr[None], [1])
        return float((o[0] * do[0, 0]).sum())
    eps = 1e-6
    for idx in range(T):
        e = np.zeros(T)
        e[idx] = eps
        np.testing.assert_allclose(da[0, idx], (loss(a + e, r) - loss(a - e, r)) / (2 * eps), rtol=0, atol=1e-7)
        np.testing.assert_allclose(dr[0, idx], (loss(a, r + e) - loss(a, r - e)) / (2 * eps), rtol=0, atol=1e-7)


def check_pattern_grad_sums_vanish(orc):
    """Each row of dS sums to zero (softmax rows are normalised), so the
    dalpha and drho vectors of every head sum to zero; a constant shift of
    a or r leaves both gradients unchanged."""
    rng = _rng(17)
    B, T, d = 2, 33, 5
    a, r = _pattern(T, rng)
    v, do = rng.normal(size=(B, 1, T, d)), rng.normal(size=(B, 1, T, d))
    m = np.array([1], dtype=np.uint8)
    da, dr = orc.pattern_grad(v, do, a[None], r[None], m)
    assert abs(da.sum()) < 1e-11 and abs(dr.sum()) < 1e-11
    da2, dr2 = orc.pattern_grad(v, do, a[None] + 7.0, r[None] - 3.0, m)
    np.testing.assert_allclose(da2, da, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dr2, dr, rtol=0, atol=1e-11)


def _read_attention(orc, q, k):
    """A = softmax_causal(q k^T / sqrt(d)) of one slice, read off the oracle's
    forward with V = identity (an independent code path)."""
    T, d = q.shape
    # the forward takes one width for q, k and v: pad q, k to width T, with q
    # scaled so that the forward's 1/sqrt(T) becomes 1/sqrt(d)
    qp, kp = np.zeros((T, T)), np.zeros((T, T))
    qp[:, :d] = np.asarray(q) * np.sqrt(T / d)
    kp[:, :d] = np.asarray(k)
    nan = np.full((1, T), np.nan)
    o, _ = orc.fwd_slices(qp[None], kp[None], np.eye(T)[None], nan, nan, [0])
    return o[0]


def check_calibration_closed_forms(orc):
    """Eq. (1) and the sample mean: identical samples give s_var = 0 and the
    mean equal to the (forward-read) attention matrix; two samples give
    s_var = ||A1 - A2||_F^2 / (2 T^2); the mean is row-stochastic and causal."""
    rng = _rng(18)
    T, d = 17, 8
    q, k = rng.normal(size=(T, d)) * 1.3, rng.normal(size=(T, d)) * 1.3
    Q = np.stack([q, q, q])[:, None]
    K = np.stack([k, k, k])[:, None]
    a_hat, sv = orc.calibration(Q, K)
    A = _read_attention(orc, q, k)
    np.testing.assert_allclose(a_hat[0], A, rtol=0, atol=1e-13)
    assert sv[0] < 1e-28
    q2, k2 = rng.normal(size=(T, d)), rng.normal(size=(T, d))
    a_hat, sv = orc.calibration(np.stack([q, q2])[:, None], np.stack([k, k2])[:, None])
    A2 = _read_attention(orc, q2, k2)
    np.testing.assert_allclose(a_hat[0], 0.5 * (A + A2), rtol=0, atol=1e-13)
    np.testing.assert_allclose(sv[0], ((A - A2) ** 2).sum() / (2 * T * T), rtol=1e-9, atol=0)
    np.testing.assert_allclose(a_hat[0].sum(axis=1), np.ones(T), rtol=0, atol=1e-13)
    assert np.all(np.triu(a_hat[0], 1) == 0)


def check_calibration_mean_is_linear(orc):
    """A_hat V equals the mean of the oracle's forward outputs A_n V (same V
    for every sample), head by head; s_var does not depend on sample order."""
    rng = _rng(19)
    N, H, T, d = 4, 2, 12, 4
    q, k = rng.normal(size=(N, H, T, d)), rng.normal(size=(N, H, T, d))
    v = rng.normal(size=(T, d))
    a_hat, sv = orc.calibration(q, k)
    nan = np.full((1, T), np.nan)
    for h in range(H):
        outs = [orc.fwd_slices(q[n, h][None], k[n, h][None], v[None], nan, nan, [0])[0][0] for n in range(N)]
        np.testing.assert_allclose(a_hat[h] @ v, np.mean(outs, axis=0), rtol=0, atol=1e-13)
    _, sv2 = orc.calibration(q[::-1], k[::-1])
    np.testing.assert_allclose(sv2, sv, rtol=1e-13, atol=0)


def _pattern_of(orc, a, r):
    return _pattern_matrix(orc, np.asarray(a, dtype=np.float64), np.asarray(r, dtype=np.float64))[0]


def check_fit_recovers_a_pattern(orc):
    """A target that is itself a compact pattern (Eq. (3)) is fitted back: the
    fitted pattern equals it (a and r up to their shift freedom) and the KL is
    zero."""
    rng = _rng(20)
    T = 40
    a, r = _pattern(T, rng)
    target = _pattern_of(orc, a, r)
    fa, fr, kl = orc.fit_pattern(target, 400, 0.1)
    np.testing.assert_allclose(_pattern_of(orc, fa, fr), target, rtol=0, atol=1e-6)
    assert abs(kl) < 1e-9


def check_fit_matches_moments_and_kl(orc):
    """A target outside the family (a random row-stochastic causal matrix):
    at the optimum of the cross-entropy the fitted pattern's column sums and
    distance sums equal the target's (the sufficient statistics of Eq. (4));
    the returned KL equals the mean row KL computed directly."""
    rng = _rng(21)
    T = 24
    logits = rng.normal(size=(T, T)) * 1.5
    logits[np.triu_indices(T, 1)] = NEG_INF
    target = np.exp(logits - logsumexp(logits, axis=1)[:, None])
    fa, fr, kl = orc.fit_pattern(target, 3000, 0.01)
    P = _pattern_of(orc, fa, fr)
    np.testing.assert_allclose(P.sum(axis=0), target.sum(axis=0), rtol=0, atol=2e-4)
    diag = lambda M: np.array([np.trace(M, offset=-d) for d in range(T)])  # noqa: E731
    np.testing.assert_allclose(diag(P), diag(target), rtol=0, atol=2e-4)
    mask = np.tril(np.ones((T, T), dtype=bool))
    direct = np.sum(target[mask] * (np.log(target[mask]) - np.log(P[mask]))) / T
    np.testing.assert_allclose(kl, direct, rtol=0, atol=1e-10)
    assert kl > 0.05  # the random target is far from the family


def check_all_masked_row(orc):
    """Every logit -inf (a = -inf): output 0 and lse = -inf, no NaN."""
    T, d = 5, 4
    a = np.full((1, T), NEG_INF)
    r = np.zeros((1, T))
    v = np.ones((1, T, d))
    o, lse = orc.fwd_slices(v, v, v, a, r, [1])
    assert np.all(o == 0) and np.all(lse == NEG_INF)
    _, _, dv = orc.bwd_slices(v, v, v, v, a, r, [1])
    assert np.all(dv == 0)


ALL_CHECKS = [
    check_pattern_is_causal_distribution,
    check_uniform_pattern_is_running_mean,
    check_identity_pattern,
    check_sink_pattern,
    check_shift_invariance,
    check_geometric_closed_form,
    check_lognorm_is_causal_convolution,
    check_replaced_backward_is_pattern_transpose,
    check_replaced_finite_differences,
    check_ordinary_matches_sdpa,
    check_ordinary_grads_match_autograd,
    check_ordinary_finite_differences,
    check_zero_query_is_running_mean,
    check_layer_mixes_head_kinds,
    check_grouped_kv_matches_autograd,
    check_pattern_grad_matches_autograd,
    check_pattern_grad_finite_differences,
    check_pattern_grad_sums_vanish,
    check_calibration_closed_forms,
    check_calibration_mean_is_linear,
    check_fit_recovers_a_pattern,
    check_fit_matches_moments_and_kl,
    check_all_masked_row,
]
