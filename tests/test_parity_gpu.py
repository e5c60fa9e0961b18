"""GPU path (through the C ABI) against the fp64 oracle, element by element.

Tolerances are stated in tests/parity.py.  Small shapes are compared in
full (several tiles plus ragged tails, both head kinds, degenerate patterns);
the full-size workloads are compared on sampled (batch, head) slices that the
oracle recomputes one by one, plus properties checked on every slice.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from mixed_head_causal_b200 import inputs as I
from mixed_head_causal_b200 import saf
from tests import parity as P

pytestmark = pytest.mark.gpu

THREADS = min(16, os.cpu_count() or 1)


def _all_slices(w):
    return [(b, h) for b in range(w.B) for h in range(w.H)]


@pytest.fixture(params=["tensor_core", "mma_sync"])
def path(request, monkeypatch):
    """Runs a test on the default tcgen05 path and on the warp-level path."""
    if request.param == "mma_sync":
        monkeypatch.setenv("SAF_FORCE_MMA", "1")
    else:
        monkeypatch.delenv("SAF_FORCE_MMA", raising=False)
    return request.param


@pytest.mark.parametrize("grad_dtype", [torch.float32, torch.bfloat16], ids=["grad_fp32", "grad_bf16"])
def test_tiny_layer_full(grad_dtype, path):
    w = I.WORKLOADS["tiny_b1_h4_t256"]
    x = I.make_inputs(w, 0)
    got = P.run_layer(w, x, grad_dtype)
    stats = P.check_slices(w, x, got, _all_slices(w), grad_dtype=grad_dtype)
    print(w.name, stats)


@pytest.mark.parametrize("T", [1, 2, 7, 63, 64, 65, 127, 128, 129, 200, 255, 257, 383])
@pytest.mark.parametrize("kind", ["mixed", "ordinary", "replaced"])
def test_ragged_lengths(T, kind, path):
    heads = {"mixed": [0, 2], "ordinary": [], "replaced": [0, 1, 2]}[kind]
    w = I.custom(2, 3, T, heads)
    x = I.make_inputs(w, 3)
    got = P.run_layer(w, x, torch.float32)
    P.check_slices(w, x, got, _all_slices(w))


@pytest.mark.parametrize("grad_dtype", [torch.float32, torch.bfloat16], ids=["grad_fp32", "grad_bf16"])
def test_several_tiles_full(grad_dtype, path):
    w = I.custom(2, 4, 1000, [1, 2])
    x = I.make_inputs(w, 5)
    got = P.run_layer(w, x, grad_dtype)
    stats = P.check_slices(w, x, got, _all_slices(w), grad_dtype=grad_dtype)
    print(w.name, stats)


def _special(T, a_fn, r_fn):
    """Head 1 of a (1, 2, T) layer replaced with pattern vectors a_fn(T),
    r_fn(T); their draws are seeded by T (the global generator is restored)."""
    w = I.custom(1, 2, T, [1])
    x = I.make_inputs(w, 7)
    with torch.random.fork_rng(devices=[]):
        torch.manual_seed(1000 + T)
        x["alpha"][1] = a_fn(T)
        x["rho"][1] = r_fn(T)
    return w, x


def test_uniform_pattern_is_running_mean():
    w, x = _special(300, lambda T: torch.zeros(T), lambda T: torch.zeros(T))
    got = P.run_layer(w, x)
    P.check_slices(w, x, got, _all_slices(w))
    v = x["v"][0, 1].double()
    mean = torch.cumsum(v, 0) / torch.arange(1, 301, dtype=torch.float64)[:, None]
    assert (got["o"][0, 1].double() - mean).abs().max() < 1e-2


def test_identity_pattern_gives_v():
    def r_fn(T):
        r = torch.full((T,), float("-inf"))
        r[0] = 0.0
        return r
    w, x = _special(257, lambda T: torch.randn(T), r_fn)
    got = P.run_layer(w, x)
    P.check_slices(w, x, got, _all_slices(w))
    # P = I: O = V and dV = dO up to the rounding of one bf16 factor
    v, do = x["v"][0, 1].double(), x["do"][0, 1].double()
    assert ((got["o"][0, 1].double() - v).abs() <= 2.0 ** -7 * v.abs()).all()
    assert ((got["dv"][0, 1].double() - do).abs() <= 2.0 ** -7 * do.abs()).all()


def test_sink_pattern_gives_first_value():
    def a_fn(T):
        a = torch.full((T,), float("-inf"))
        a[0] = 0.0
        return a
    w, x = _special(190, a_fn, lambda T: torch.randn(T))
    got = P.run_layer(w, x)
    v0 = x["v"][0, 1][:1].double().expand(190, 64)
    assert ((got["o"][0, 1].double() - v0).abs() <= 2.0 ** -7 * v0.abs()).all()
    P.check_slices(w, x, got, _all_slices(w))


def test_extreme_pattern_ranges(path):
    """Long linear decay (terms far below fp32 range) and a +-60 shift."""
    w, x = _special(2048, lambda T: torch.randn(T) * 3 + 60.0, lambda T: -0.5 * torch.arange(T, dtype=torch.float32) - 60.0)
    got = P.run_layer(w, x)
    P.check_slices(w, x, got, _all_slices(w))


def test_lognorm_entry_point_and_explicit_logz():
    w = I.custom(2, 4, 777, [0, 3])
    x = I.make_inputs(w, 11)
    g = P.to_gpu(x)
    lz = saf.replaced_lognorm(g["alpha"], g["rho"], x["mask"])
    ref = oracle.lognorm(x["alpha"][[0, 3]], x["rho"][[0, 3]])
    err = np.abs(lz[[0, 3]].cpu().double().numpy() - ref)
    assert err.max() < 1e-4 * max(1.0, np.abs(ref).max())
    o1, l1 = saf.mixed_attn_fwd(g["q"], g["k"], g["v"], g["alpha"], g["rho"], x["mask"])
    o2, l2 = saf.mixed_attn_fwd(g["q"], g["k"], g["v"], g["alpha"], g["rho"], x["mask"], logz=lz)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    d1 = saf.mixed_attn_bwd(g["q"], g["k"], g["v"], o1, g["do"], l1, g["alpha"], g["rho"], x["mask"])
    d2 = saf.mixed_attn_bwd(g["q"], g["k"], g["v"], o1, g["do"], l1, g["alpha"], g["rho"], x["mask"], logz=lz)
    # dK, dV bit-exact; dQ up to the order of its fp32 reduce-adds across CTAs
    assert torch.equal(d1[1], d2[1]) and torch.equal(d1[2], d2[2])
    scale = max(1.0, d1[0].abs().max().item())
    assert (d1[0].float() - d2[0].float()).abs().max().item() <= 1e-5 * scale


@pytest.mark.parametrize("T", [1, 31, 32, 257, 545, 4101])
def test_lognorm_tiles_and_special_values(T):
    """log Z over ragged row tiles and several k chunks, with -inf terms
    (a masked key, a forbidden distance) and offsets of +-50."""
    gen = torch.Generator().manual_seed(T)
    a = torch.randn(3, T, generator=gen) * 4
    r = torch.randn(3, T, generator=gen) * 4
    a[1] += 50.0
    r[2] -= 50.0
    a[0, ::7] = float("-inf")
    r[0, 1::5] = float("-inf")
    if T > 3:
        a[2, :3] = float("-inf")  # rows 0..2 of head 2 have no term: log Z = -inf
        r[2, 0] = float("-inf")
    mask = torch.ones(3, dtype=torch.bool)
    lz = saf.replaced_lognorm(a.cuda(), r.cuda(), mask).cpu().double().numpy()
    ref = oracle.lognorm(a, r)
    fin = np.isfinite(ref)
    assert (np.isfinite(lz) == fin).all()
    assert (lz[~fin] == -np.inf).all()
    err = np.abs(lz[fin] - ref[fin])
    assert err.max() < 1e-4 * max(1.0, np.abs(ref[fin]).max())


def test_repeatable():
    """Two calls on the same inputs: O, lse, dK and dV are bit-identical (each
    is produced by one CTA in a fixed order); dQ is the sum of fp32 reduce-adds
    from several CTAs, whose order is not fixed, so it repeats to within the
    rounding of that sum."""
    w = I.custom(1, 3, 700, [1])
    x = I.make_inputs(w, 2)
    a = P.run_layer(w, x)
    b = P.run_layer(w, x)
    for k in a:
        if k == "dq":
            scale = max(1.0, a[k].abs().max().item())
            assert (a[k] - b[k]).abs().max().item() <= 1e-5 * scale, k
        else:
            assert torch.equal(a[k], b[k]), k


def test_dq_repeats_across_many_calls():
    """dQ boxes are written by the last of their contributions: eight calls on a
    layer with many contributions per box (T = 3000, 24 key blocks) and several
    items per CTA give the same dQ up to the order of the fp32 reduce-adds, and
    every call matches the oracle on a sampled slice."""
    w = I.custom(4, 6, 3000, [2, 5])
    x = I.make_inputs(w, 66)
    g = P.to_gpu(x)
    o, lse = saf.mixed_attn_fwd(g["q"], g["k"], g["v"], g["alpha"], g["rho"], x["mask"])
    ref = None
    for _ in range(8):
        dq, dk, dv = saf.mixed_attn_bwd(g["q"], g["k"], g["v"], o, g["do"], lse, g["alpha"], g["rho"], x["mask"],
                                        grad_dtype=torch.float32)
        torch.cuda.synchronize()
        if ref is None:
            ref = (dq.clone(), dk.clone(), dv.clone())
            got = {"o": o.cpu(), "lse": lse.cpu(), "dq": dq.cpu(), "dk": dk.cpu(), "dv": dv.cpu()}
            P.check_slices(w, x, got, [(3, 0), (1, 5)])
            continue
        scale = max(1.0, ref[0].abs().max().item())
        assert (dq - ref[0]).abs().max().item() <= 1e-5 * scale
        assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])


def _full_size(name, grad_dtype=torch.float32, per_kind=2):
    w = I.WORKLOADS[name]
    x = I.make_inputs(w, 0, threads=THREADS)
    got = P.run_layer(w, x, grad_dtype, backward=w.backward)
    mask = x["mask"]
    # properties on every slice
    for key in got:
        assert torch.isfinite(got[key].float()).all(), key
    if w.backward:
        rep = mask.bool()
        assert torch.count_nonzero(got["dq"][:, rep]) == 0
        assert torch.count_nonzero(got["dk"][:, rep]) == 0
    slices = P.sample_slices(w, mask.numpy(), per_kind=per_kind)
    stats = P.check_slices(w, x, got, slices, grad_dtype=grad_dtype)
    print(name, slices, stats)


@pytest.mark.parametrize("name", ["124m_b8_t4096_r25", "124m_b4_t8192_r50", "1b_b4_h32_t8192_r25"])
def test_full_size_fwd_bwd_sampled(name):
    _full_size(name, torch.float32)


def test_full_size_bf16_grads_sampled():
    _full_size("124m_b8_t4096_r25", torch.bfloat16)


@pytest.mark.parametrize("name", I.PREFILL_SWEEP)
def test_prefill_sweep_sampled(name):
    _full_size(name, per_kind=2)


def test_factored_range_guard_falls_back(path):
    """a spanning far more than fp32's range: the factored form is refused for
    that head, which then runs the per-element exp path; results unchanged."""
    w, x = _special(777, lambda T: torch.randn(T) * 40.0, lambda T: -0.05 * torch.arange(T, dtype=torch.float32))
    got = P.run_layer(w, x)
    P.check_slices(w, x, got, _all_slices(w))


def test_rows_far_below_the_pattern_maxima(path):
    """Rows whose log Z sits far below max a + max r: a sink a[0] = 25 that
    rows past 200 cannot see (r = -1000 beyond distance 200) and every other
    key near -50, so max a + max r - log Z(i) is about 70 for those rows,
    above the factored form's limit of 50 while max a - min a stays under 80:
    the log Z limit alone sends the head to the per-element path.  Every
    slice against the oracle."""
    def a_fn(T):
        a = torch.randn(T) * 0.5 - 50.0
        a[0] = 25.0
        return a

    def r_fn(T):
        r = torch.zeros(T)
        r[200:] = -1000.0
        return r
    w, x = _special(900, a_fn, r_fn)
    got = P.run_layer(w, x)
    P.check_slices(w, x, got, _all_slices(w))


def test_guarded_and_factored_heads_in_one_call():
    """Two batches, heads 0 and 2 replaced: head 0 with a far beyond fp32
    range (per-element exps), head 2 ordinary-range (factored form), a ragged
    T spanning several tiles; every slice against the oracle."""
    w = I.custom(2, 4, 650, [0, 2])
    x = I.make_inputs(w, 13)
    gen = torch.Generator().manual_seed(13)
    x["alpha"][0] = torch.randn(650, generator=gen) * 40.0
    x["rho"][0] = -0.02 * torch.arange(650, dtype=torch.float32) + torch.randn(650, generator=gen) * 30.0
    got = P.run_layer(w, x)
    P.check_slices(w, x, got, _all_slices(w))


@pytest.mark.parametrize("B,H,Hkv,T,replaced", [(2, 8, 2, 650, [1, 5]), (1, 4, 1, 300, [0, 3]),
                                                (2, 6, 3, 1000, [2]), (1, 4, 2, 129, []),
                                                (2, 8, 2, 2000, [1, 5])],
                         ids=["gqa4_t650", "mqa_t300", "gqa2_t1000", "gqa2_t129_no_replaced",
                              "gqa4_t2000_several_items_per_cta"])
@pytest.mark.parametrize("grad_dtype", [torch.float32, torch.bfloat16], ids=["grad_fp32", "grad_bf16"])
def test_grouped_kv_layer(B, H, Hkv, T, replaced, grad_dtype):
    """Shared K/V heads (H / Hkv query heads per K/V head, replaced heads mixed
    in): O, lse, dQ and the group-summed dK, dV against the oracle."""
    w = I.custom(B, H, T, replaced)
    x = I.make_inputs(w, 21)
    k = x["k"][:, :Hkv].contiguous()
    v = x["v"][:, :Hkv].contiguous()
    g = P.to_gpu(x)
    kg, vg = k.cuda(), v.cuda()
    o, lse = saf.mixed_attn_fwd(g["q"], kg, vg, g["alpha"], g["rho"], x["mask"])
    dq, dk, dv = saf.mixed_attn_bwd(g["q"], kg, vg, o, g["do"], lse, g["alpha"], g["rho"], x["mask"],
                                    grad_dtype=grad_dtype)
    torch.cuda.synchronize()
    assert tuple(dk.shape) == (B, Hkv, T, 64) and tuple(dv.shape) == (B, Hkv, T, 64)
    o_ref, lse_ref = oracle.fwd_gqa(x["q"], k, v, x["alpha"], x["rho"], x["mask"])
    dq_ref, dk_ref, dv_ref = oracle.bwd_gqa(x["q"], k, v, x["do"], x["alpha"], x["rho"], x["mask"])
    P.compare("O", o.cpu(), o_ref, stored_bf16=True, gradient=False)
    lse_fin = np.isfinite(lse_ref)
    assert np.abs(lse.cpu().double().numpy()[lse_fin] - lse_ref[lse_fin]).max() <= P.TOL_LSE
    bf = grad_dtype == torch.bfloat16
    P.compare("dQ", dq.cpu(), dq_ref, bf)
    P.compare("dK", dk.cpu(), dk_ref, bf)
    P.compare("dV", dv.cpu(), dv_ref, bf)


def test_grouped_kv_argument_errors():
    """H_kv must divide H; the warp-level path has no shared K/V."""
    w = I.custom(1, 4, 64, [1])
    x = I.make_inputs(w, 3)
    g = P.to_gpu(x)
    k3 = g["k"][:, :3].contiguous()
    with pytest.raises(saf.SafError):
        saf.mixed_attn_fwd(g["q"], k3, k3, g["alpha"], g["rho"], x["mask"])


@pytest.mark.parametrize("B,H,T,replaced", [(2, 3, 300, [0, 2]), (1, 2, 1000, [1]), (3, 4, 129, [0, 1, 2, 3]),
                                            (1, 2, 64, [0])],
                         ids=["b2_t300", "b1_t1000", "b3_t129_all_replaced", "b1_t64"])
def test_pattern_grad(B, H, T, replaced):
    """Trainable pattern: dalpha, drho against the oracle.  The kernel works in
    fp32 (exact bf16 products, fp32 sums and exps); its error relative to the
    largest gradient entry of a head stays far below 2e-4 (the fp32 rounding
    of sums over about B*T terms), which is the bound used here; rows of
    ordinary heads must be exactly zero."""
    w = I.custom(B, H, T, replaced)
    x = I.make_inputs(w, 31)
    g = P.to_gpu(x)
    da, dr = saf.replaced_pattern_grad(g["v"], g["do"], g["alpha"], g["rho"], x["mask"])
    torch.cuda.synchronize()
    da_ref, dr_ref = oracle.pattern_grad(x["v"], x["do"], x["alpha"], x["rho"], x["mask"])
    da, dr = da.cpu().double().numpy(), dr.cpu().double().numpy()
    for h in range(H):
        if h not in replaced:
            assert np.all(da[h] == 0) and np.all(dr[h] == 0)
            continue
        for got, ref in ((da[h], da_ref[h]), (dr[h], dr_ref[h])):
            scale = max(1.0, np.abs(ref).max())
            assert np.abs(got - ref).max() <= 2e-4 * scale, (h, np.abs(got - ref).max(), scale)


def _pattern_grad_noise(x, h):
    """Expected fp32 rounding noise of dalpha, drho of head h.

    The kernel's log P(i,j) = a[j] + r[i-j] - log Z(i) carries an error of
    about one unit of fp32 rounding of the largest logit magnitude L (log Z(i)
    is itself an fp32 number of that size), shared by a row and by every
    batch.  A relative error eps_i of row i moves dS(i,j) by eps_i (dS(i,j) -
    P(i,j) D(i)), so dalpha[j] and drho[d] collect sums of such terms of
    random sign: noise = 2^-23 L sqrt(sum_i (sum_b |dS| + P |D|)^2) over the
    entries (i, j) that reach the output."""
    a = x["alpha"][h].double().numpy()
    r = x["rho"][h].double().numpy()
    T = a.shape[0]
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    causal = j <= i
    logit = np.where(causal, a[None, :] + r[np.clip(i - j, 0, T - 1)], -np.inf)
    top = logit.max(1, keepdims=True)
    lz = top + np.log(np.exp(logit - top).sum(1, keepdims=True))
    p = np.exp(logit - lz)
    wsum = np.zeros((T, T))
    for b in range(x["v"].shape[0]):
        dp = x["do"][b, h].double().numpy() @ x["v"][b, h].double().numpy().T
        dvec = (p * dp).sum(1, keepdims=True)
        wsum += np.abs(p * (dp - dvec)) + p * np.abs(dvec)
    big = max(np.abs(a).max(), np.abs(r[np.isfinite(r)]).max(), np.abs(lz).max())
    delta = 2.0 ** -23 * (big + 1.0)
    w2 = wsum ** 2
    noise_a = delta * np.sqrt(w2.sum(0))
    noise_r = delta * np.sqrt(np.array([np.trace(w2, -d) for d in range(T)]))
    return noise_a, noise_r


def test_pattern_grad_extreme_range_and_explicit_logz():
    """Pattern vectors far beyond the factored form's range (logits of size
    ~150) and a log Z passed in: dalpha, drho against the oracle within 2e-4
    of the largest entry plus four times the expected fp32 noise of logits
    that large (_pattern_grad_noise)."""
    w, x = _special(500, lambda T: torch.randn(T) * 40.0, lambda T: -0.05 * torch.arange(T, dtype=torch.float32))
    g = P.to_gpu(x)
    lz = saf.replaced_lognorm(g["alpha"], g["rho"], x["mask"])
    da, dr = saf.replaced_pattern_grad(g["v"], g["do"], g["alpha"], g["rho"], x["mask"], logz=lz)
    torch.cuda.synchronize()
    da_ref, dr_ref = oracle.pattern_grad(x["v"], x["do"], x["alpha"], x["rho"], x["mask"])
    noise_a, noise_r = _pattern_grad_noise(x, 1)
    for got, ref, noise in ((da[1].cpu().double().numpy(), da_ref[1], noise_a),
                            (dr[1].cpu().double().numpy(), dr_ref[1], noise_r)):
        tol = 2e-4 * max(1.0, np.abs(ref).max()) + 4.0 * noise
        assert np.all(np.abs(got - ref) <= tol), (np.abs(got - ref).max(), tol.max())


@pytest.mark.parametrize("N,H,T", [(3, 2, 300), (2, 3, 64), (4, 1, 650)], ids=["n3_t300", "n2_t64", "n4_t650"])
def test_calibration(N, H, T):
    """Calibration statistics (sample-mean attention, Eq. (1)) against the
    oracle: every element of A_hat within 1e-4 (probabilities; the kernel's
    fp32 exps and the forward's lse are good to ~1e-6), s_var within 1e-3
    relative; A_hat zero above the diagonal."""
    w = I.custom(N, H, T, [])
    x = I.make_inputs(w, 41)
    g = P.to_gpu(x)
    _, lse = saf.mixed_attn_fwd(g["q"], g["k"], g["v"], g["alpha"], g["rho"], x["mask"])
    a_hat, svar = saf.attn_calibration(g["q"], g["k"], lse)
    torch.cuda.synchronize()
    a_ref, sv_ref = oracle.calibration(x["q"], x["k"])
    a_hat = a_hat.cpu().double().numpy()
    assert np.abs(a_hat - a_ref).max() <= 1e-4
    assert np.all(np.triu(a_hat, 1) == 0)
    np.testing.assert_allclose(svar.cpu().double().numpy(), sv_ref, rtol=1e-3, atol=0)


def test_calibration_needs_two_samples():
    w = I.custom(1, 2, 64, [])
    x = I.make_inputs(w, 42)
    g = P.to_gpu(x)
    _, lse = saf.mixed_attn_fwd(g["q"], g["k"], g["v"], g["alpha"], g["rho"], x["mask"])
    with pytest.raises(saf.SafError):
        saf.attn_calibration(g["q"], g["k"], lse)


def _oracle_pattern(a, r):
    """P of Eq. (3) for one head, read off the oracle's forward with V = I."""
    T = a.shape[0]
    z = np.zeros((1, T, T))
    p, _ = oracle.fwd_slices(z, z, np.eye(T)[None], np.asarray(a, np.float64)[None], np.asarray(r, np.float64)[None],
                             [1])
    return p[0]


def test_fit_recovers_compact_targets():
    """Targets that are compact patterns themselves are fitted back (fp32 Adam,
    400 steps): the fitted pattern matches the target and the KL is ~0."""
    T = 200
    gen = torch.Generator().manual_seed(51)
    targets = []
    for h in range(2):
        a = torch.randn(T, generator=gen) * 0.5
        a[0] += 3.0
        r = -0.05 * (h + 1) * torch.arange(T, dtype=torch.float32) + torch.randn(T, generator=gen) * 0.3
        r[0] += 1.0
        targets.append(_oracle_pattern(a.double().numpy(), r.double().numpy()))
    tg = torch.tensor(np.stack(targets), dtype=torch.float32, device="cuda")
    fa, fr, kl = saf.fit_pattern(tg, steps=400, lr=0.1)
    torch.cuda.synchronize()
    for h in range(2):
        P = _oracle_pattern(fa[h].cpu().double().numpy(), fr[h].cpu().double().numpy())
        assert np.abs(P - targets[h]).max() <= 2e-3
        assert abs(float(kl[h])) <= 1e-3


def test_fit_matches_the_oracle_on_a_calibration_target():
    """A calibration-mean target (the mean of 4 causal softmax matrices): the
    GPU fit and the oracle's fp64 fit (same Adam schedule) reach the same KL
    and the same pattern."""
    N, T = 4, 96
    gen = torch.Generator().manual_seed(52)
    q = torch.randn(N, 1, T, 64, generator=gen)
    k = torch.randn(N, 1, T, 64, generator=gen)
    a_hat, _ = oracle.calibration(q, k)
    target = a_hat[0]
    fa, fr, kl = saf.fit_pattern(torch.tensor(target, dtype=torch.float32, device="cuda")[None], steps=400, lr=0.1)
    torch.cuda.synchronize()
    oa, orr, okl = oracle.fit_pattern(target, 400, 0.1)
    assert abs(float(kl[0]) - okl) <= 2e-3
    P = _oracle_pattern(fa[0].cpu().double().numpy(), fr[0].cpu().double().numpy())
    assert np.abs(P - _oracle_pattern(oa, orr)).max() <= 1e-2
    mask = np.tril(np.ones((T, T), dtype=bool))
    direct = np.sum(target[mask] * (np.log(target[mask]) - np.log(P[mask]))) / T
    assert abs(float(kl[0]) - direct) <= 2e-3


def test_device_wait_timeout_is_reported_and_cleared():
    """A bounded device wait that nothing completes (no copy or MMA in flight)
    sets the workspace error word; saf_device_status reports the time-out once
    and clears it, and the layer still runs on the same context."""
    w = I.custom(1, 2, 200, [1])
    x = I.make_inputs(w, 61)
    g = P.to_gpu(x)
    ws = saf.new_workspace(w.B, w.H, w.T, "cuda")
    saf.selftest_wait_timeout(ws, 1 << 20)
    assert saf.device_status(ws) == saf.SAF_ERR_TIMEOUT
    assert saf.device_status(ws) == saf.SAF_OK
    o, lse = saf.mixed_attn_fwd(g["q"], g["k"], g["v"], g["alpha"], g["rho"], x["mask"], workspace=ws)
    assert saf.device_status(ws) == saf.SAF_OK
    P.check_slices(w, x, {"o": o.cpu(), "lse": lse.cpu()}, _all_slices(w))


def test_persistent_forward_leaves_its_counters_zero():
    """The persistent forward's work counters in the workspace header are zero
    after each call (the last CTA resets them), so the workspace can be reused
    and calls repeat exactly."""
    w = I.custom(2, 3, 520, [0])
    x = I.make_inputs(w, 62)
    g = P.to_gpu(x)
    ws = saf.new_workspace(w.B, w.H, w.T, "cuda")
    outs = []
    for _ in range(3):
        o, lse = saf.mixed_attn_fwd(g["q"], g["k"], g["v"], g["alpha"], g["rho"], x["mask"], workspace=ws)
        torch.cuda.synchronize()
        header = ws[:64].view(torch.int32).cpu()
        assert int(header[2]) == 0 and int(header[3]) == 0
        outs.append((o.clone(), lse.clone()))
    for o, lse in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(lse, outs[0][1])


def test_persistent_backward_leaves_its_counters_zero():
    """The persistent backward's work counters in the workspace header are zero
    after each call, and repeated calls give the same dK, dV (one CTA owns a key
    block) and dQ up to the order of its fp32 reduce-adds."""
    w = I.custom(2, 3, 520, [0])
    x = I.make_inputs(w, 63)
    g = P.to_gpu(x)
    o, lse = saf.mixed_attn_fwd(g["q"], g["k"], g["v"], g["alpha"], g["rho"], x["mask"])
    ws = saf.new_workspace(w.B, w.H, w.T, "cuda", backward=True)
    outs = []
    for _ in range(3):
        dq, dk, dv = saf.mixed_attn_bwd(g["q"], g["k"], g["v"], o, g["do"], lse, g["alpha"], g["rho"], x["mask"],
                                        grad_dtype=torch.float32, workspace=ws)
        torch.cuda.synchronize()
        header = ws[:64].view(torch.int32).cpu()
        assert int(header[0]) == 0 and int(header[4]) == 0 and int(header[5]) == 0
        outs.append((dq.clone(), dk.clone(), dv.clone()))
    for dq, dk, dv in outs[1:]:
        assert torch.equal(dk, outs[0][1]) and torch.equal(dv, outs[0][2])
        assert (dq - outs[0][0]).abs().max().item() <= 1e-5 * max(1.0, outs[0][0].abs().max().item())


def test_persistent_backward_many_items_per_cta():
    """More key-block items than SMs (512 items of 1 to 16 tiles, ordinary and
    replaced heads interleaved in the longest-first order, a ragged T), so every
    CTA runs several items back to back: every slice against the oracle."""
    w = I.custom(4, 8, 2000, [1, 4, 6])
    x = I.make_inputs(w, 64)
    got = P.run_layer(w, x, torch.float32)
    P.check_slices(w, x, got, _all_slices(w))
