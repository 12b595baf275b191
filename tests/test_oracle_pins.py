"""Pins for the float64 oracle, against things other than the oracle itself.

Each test names the invariant it checks (I1..I11) and the statement it rests
on.  Between them they fail on a dropped term, a wrong sign, a wrong index or
a transposed operand anywhere in the oracle.  CPU only.
"""
import math

import numpy as np
import pytest
import torch

from oracle import rope_attn_naive as naive
from oracle import rope_attn_ref as ref


def rand_problem(seed, B, H, n, d, alpha_scale=0.4, base=10000.0, qscale=1.0):
    rng = np.random.default_rng(seed)
    q = qscale * rng.standard_normal((B, H, n, d))
    k = qscale * rng.standard_normal((B, H, n, d))
    v = rng.standard_normal((B, H, n, d))
    e = rng.standard_normal((B, H, n, d))
    alpha = alpha_scale * rng.standard_normal(d // 2)
    return q, k, v, e, alpha, base


def total_loss(q, k, v, e, alpha, base, causal, **kw):
    o, _ = ref.forward(q, k, v, alpha, base, causal, **kw)
    return ref.loss(o, e)[0]


# ---------------------------------------------------------------- naive vs blocked
@pytest.mark.parametrize("causal", [False, True])
def test_naive_matches_blocked(causal):
    q, k, v, e, alpha, base = rand_problem(1, 1, 2, 11, 8, base=100.0)
    r = ref.forward_backward(q, k, v, e, alpha, base, causal, block=4)
    acc = np.zeros(4)
    Ltot = 0.0
    for h in range(2):
        nv = naive.head(q[0, h].tolist(), k[0, h].tolist(), v[0, h].tolist(), e[0, h].tolist(),
                        alpha.tolist(), base, causal)
        for key in ("o", "dq", "dk", "dv"):
            np.testing.assert_allclose(np.array(nv[key]), r[key][0, h], rtol=0, atol=1e-12)
        np.testing.assert_allclose(np.array(nv["lse"]), r["lse"][0, h], rtol=0, atol=1e-12)
        acc += np.array(nv["dalpha"])
        Ltot += nv["L"]
    np.testing.assert_allclose(acc, r["dalpha"], rtol=1e-12, atol=1e-12)
    assert abs(Ltot - r["L"]) < 1e-12 * max(1.0, abs(Ltot))


# ---------------------------------------------------------------- I4 finite differences
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [4, 8])
def test_I4_finite_differences(causal, d):
    """Central differences of L (fp64, h = 1e-6) on every entry of Q, K, V and alpha."""
    n = 6 if d == 8 else 7
    q, k, v, e, alpha, base = rand_problem(7 + d, 1, 2, n, d, alpha_scale=0.5, base=20.0)
    r = ref.forward_backward(q, k, v, e, alpha, base, causal)
    h = 1e-6
    for name, arr, grad in (("q", q, r["dq"]), ("k", k, r["dk"]), ("v", v, r["dv"])):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + h
            lp = total_loss(q, k, v, e, alpha, base, causal)
            arr[idx] = old - h
            lm = total_loss(q, k, v, e, alpha, base, causal)
            arr[idx] = old
            fd[idx] = (lp - lm) / (2 * h)
        err = np.max(np.abs(fd - grad)) / np.max(np.abs(grad))
        assert err < 1e-7, (name, err)
    fd = np.zeros_like(alpha)
    for m in range(len(alpha)):
        old = alpha[m]
        alpha[m] = old + h
        lp = total_loss(q, k, v, e, alpha, base, causal)
        alpha[m] = old - h
        lm = total_loss(q, k, v, e, alpha, base, causal)
        alpha[m] = old
        fd[m] = (lp - lm) / (2 * h)
    err = np.max(np.abs(fd - r["dalpha"])) / np.max(np.abs(r["dalpha"]))
    assert err < 1e-7, ("alpha", err)


# ---------------------------------------------------------------- I4b autograd route
def _torch_rope_complex(x, pos, theta_hat):
    """Textbook complex-number RoPE: pair (2m, 2m+1) -> z, z * exp(i p theta)."""
    z = torch.view_as_complex(x.reshape(*x.shape[:-1], -1, 2).contiguous())
    rot = torch.polar(torch.ones_like(pos[:, None] * theta_hat[None, :]),
                      pos[:, None] * theta_hat[None, :])
    return torch.view_as_real(z * rot).reshape(x.shape)


@pytest.mark.parametrize("causal", [False, True])
def test_I4b_autograd_of_independent_forward(causal):
    """A forward written with complex multiplication and torch's own softmax, differentiated
    by autograd, gives the same dQ, dK, dV, dalpha as the oracle's hand-written backward."""
    B, H, n, d = 2, 3, 33, 16
    q, k, v, e, alpha, base = rand_problem(3, B, H, n, d, alpha_scale=0.7, base=500.0)
    r = ref.forward_backward(q, k, v, e, alpha, base, causal, block=8)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    ta = torch.tensor(alpha, requires_grad=True)
    m = torch.arange(d // 2, dtype=torch.float64)
    th = torch.exp(ta) * base ** (-2.0 * m / d)
    pos = torch.arange(n, dtype=torch.float64)
    qr, kr = _torch_rope_complex(tq, pos, th), _torch_rope_complex(tk, pos, th)
    s = qr @ kr.transpose(-1, -2) / math.sqrt(d)
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), float("-inf"))
    o = torch.softmax(s, dim=-1) @ tv
    L = 0.5 * ((o - torch.tensor(e)) ** 2).sum()
    L.backward()
    np.testing.assert_allclose(o.detach().numpy(), r["o"], atol=1e-12)
    assert abs(L.item() - r["L"]) < 1e-10 * abs(r["L"])
    for g, key in ((tq.grad, "dq"), (tk.grad, "dk"), (tv.grad, "dv")):
        np.testing.assert_allclose(g.numpy(), r[key], atol=1e-11)
    np.testing.assert_allclose(ta.grad.numpy(), r["dalpha"], rtol=1e-10, atol=1e-11)


# ---------------------------------------------------------------- I1 alpha = 0 is standard RoPE
def test_I1_alpha_zero_is_textbook_rope():
    """alpha = 0 reduces LeRoPE to standard RoPE ("LeRoPE", Escolhas de Design Principais:
    initialisation at 0).  Textbook rotate_half RoPE over the half-split layout."""
    n, d, base = 40, 16, 10000.0
    rng = np.random.default_rng(5)
    x = rng.standard_normal((n, d))
    inv = 1.0 / (base ** (np.arange(0, d, 2) / d))
    freqs = np.outer(np.arange(n), inv)
    emb = np.concatenate([freqs, freqs], axis=1)
    rot_half = np.concatenate([-x[:, d // 2:], x[:, :d // 2]], axis=1)
    textbook = x * np.cos(emb) + rot_half * np.sin(emb)
    _, th = ref.frequencies(d, base, np.zeros(d // 2))
    ours = ref.rotate(x, ref.angles(n, th), pairing="halfsplit")
    np.testing.assert_allclose(ours, textbook, atol=1e-13)


def test_pairing_is_a_permutation():
    """Interleaved and half-split pairings differ by a fixed column permutation: O, L and
    dalpha agree; dQ, dK are the same numbers permuted."""
    B, H, n, d = 1, 2, 13, 8
    q, k, v, e, alpha, base = rand_problem(9, B, H, n, d)
    perm = np.concatenate([np.arange(0, d, 2), np.arange(1, d, 2)])  # interleaved -> halfsplit
    a = ref.forward_backward(q, k, v, e, alpha, base, True)
    b = ref.forward_backward(q[..., perm], k[..., perm], v, e, alpha, base, True, pairing="halfsplit")
    np.testing.assert_allclose(a["o"], b["o"], atol=1e-13)
    np.testing.assert_allclose(a["dalpha"], b["dalpha"], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(a["dq"][..., perm], b["dq"], atol=1e-13)
    np.testing.assert_allclose(a["dk"][..., perm], b["dk"], atol=1e-13)


# ---------------------------------------------------------------- I2 relative position
def test_I2_scores_depend_on_offset_only():
    n, d = 25, 8
    q, k, v, e, alpha, base = rand_problem(11, 1, 1, n, d, base=50.0)
    _, th = ref.frequencies(d, base, alpha)
    S = {}
    for shift in (0, 1000):
        phi = ref.angles(n, th, offset=shift)
        S[shift] = ref.rotate(q[0, 0], phi) @ ref.rotate(k[0, 0], phi).T
    np.testing.assert_allclose(S[1000], S[0], atol=1e-11)
    o0, _ = ref.forward(q, k, v, alpha, base, True)
    o1, _ = ref.forward(q, k, v, alpha, base, True, offset=1000)
    np.testing.assert_allclose(o1, o0, atol=1e-11)


# ---------------------------------------------------------------- I3 norms
def test_I3_rotation_preserves_band_norms():
    n, d = 30, 12
    rng = np.random.default_rng(2)
    x = rng.standard_normal((n, d))
    _, th = ref.frequencies(d, 10000.0, rng.standard_normal(d // 2))
    y = ref.rotate(x, ref.angles(n, th))
    nb = lambda z: z[:, 0::2] ** 2 + z[:, 1::2] ** 2
    np.testing.assert_allclose(nb(y), nb(x), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(ref.rotate(y, ref.angles(n, th), sign=-1.0), x, atol=1e-14)


# ---------------------------------------------------------------- I5 DTFT surrogate
@pytest.mark.parametrize("causal", [False, True])
def test_I5_dalpha_equals_dtft_surrogate_derivative(causal):
    q, k, v, e, alpha, base = rand_problem(13, 2, 2, 17, 8, alpha_scale=0.8, base=30.0)
    r = ref.forward_backward(q, k, v, e, alpha, base, causal)
    alt = ref.dalpha_offset_dtft(q, k, v, r["do"], alpha, base, causal)
    np.testing.assert_allclose(alt, r["dalpha"], rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------- I6 global rotation
@pytest.mark.parametrize("causal", [False, True])
def test_I6_global_rotation_invariance(causal):
    q, k, v, e, alpha, base = rand_problem(17, 1, 3, 21, 8, base=40.0)
    o, _ = ref.forward(q, k, v, alpha, base, causal)
    _, do = ref.loss(o, e)
    *_, extra = ref.backward(q, k, v, do, alpha, base, causal, return_rotated=True)
    for qt, kt, dqt, dkt in extra:
        tot = ref.band_torque(dqt, qt).sum(0) + ref.band_torque(dkt, kt).sum(0)
        scale = np.abs(ref.band_torque(dqt, qt)).sum(0)
        assert np.all(np.abs(tot) < 1e-12 * np.maximum(scale, 1.0))


# ---------------------------------------------------------------- I7 zero frequency
def test_I7_zero_frequency_is_plain_attention():
    B, H, n, d = 1, 2, 19, 8
    q, k, v, e, _, base = rand_problem(19, B, H, n, d)
    alpha = np.full(d // 2, -80.0)   # exp(-80) ~ 1.8e-35: no band rotates
    o, _ = ref.forward(q, k, v, alpha, base, True)
    sd = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q), torch.tensor(k), torch.tensor(v), is_causal=True).numpy()
    np.testing.assert_allclose(o, sd, atol=1e-13)
    # dalpha_m is linear in theta_hat_m as theta_hat_m -> 0: lowering alpha by 1 divides by e
    _, do = ref.loss(o, e)
    d1 = ref.backward(q, k, v, do, np.full(d // 2, -30.0), base, True)[3]
    d2 = ref.backward(q, k, v, do, np.full(d // 2, -31.0), base, True)[3]
    np.testing.assert_allclose(d1 / d2, np.e, rtol=1e-9)


# ---------------------------------------------------------------- I8, I9 causal row 0, softmax rows
def test_I8_I9_rows():
    q, k, v, e, alpha, base = rand_problem(23, 1, 1, 15, 8)
    o, _ = ref.forward(q, k, v, alpha, base, True)
    assert np.array_equal(o[0, 0, 0], v[0, 0, 0])
    _, th = ref.frequencies(8, base, alpha)
    phi = ref.angles(15, th)
    qt, kt = ref.rotate(q[0, 0], phi), ref.rotate(k[0, 0], phi)
    p, ds = ref.head_matrices(qt, kt, v[0, 0], o[0, 0] - e[0, 0], True)
    assert np.all(ds[0] == 0.0)
    np.testing.assert_allclose(p.sum(1), 1.0, atol=1e-15)
    np.testing.assert_allclose(ds.sum(1), 0.0, atol=1e-14)
    assert np.all(np.triu(p, 1) == 0.0)


# ---------------------------------------------------------------- I10 Q = 0
@pytest.mark.parametrize("causal", [False, True])
def test_I10_zero_queries(causal):
    B, H, n, d = 1, 2, 12, 8
    _, k, v, e, alpha, base = rand_problem(29, B, H, n, d)
    q = np.zeros((B, H, n, d))
    r = ref.forward_backward(q, k, v, e, alpha, base, causal)
    for h in range(H):
        for i in range(n):
            hi = i + 1 if causal else n
            np.testing.assert_allclose(r["o"][0, h, i], v[0, h, :hi].mean(0), atol=1e-14)
    assert np.max(np.abs(r["dk"])) < 1e-15
    assert np.max(np.abs(r["dalpha"])) < 1e-14


# ---------------------------------------------------------------- I11 d = 2 closed form
def test_I11_single_band_closed_form():
    """One band: S_ij = |q_i| |k_j| cos(arg q_i - arg k_j + (i - j) theta_hat) / sqrt(2)."""
    n, theta_hat, alpha, base = 3, None, np.array([0.3]), 7.0
    rng = np.random.default_rng(31)
    q = rng.standard_normal((1, 1, n, 2))
    k = rng.standard_normal((1, 1, n, 2))
    v = rng.standard_normal((1, 1, n, 2))
    theta_hat = math.exp(0.3) * 1.0   # m = 0: base^0 = 1
    S = np.zeros((n, n))
    for i in range(n):
        for j in range(n):
            a = math.atan2(q[0, 0, i, 1], q[0, 0, i, 0])
            b = math.atan2(k[0, 0, j, 1], k[0, 0, j, 0])
            S[i, j] = (np.hypot(*q[0, 0, i]) * np.hypot(*k[0, 0, j])
                       * math.cos(a - b + (i - j) * theta_hat) / math.sqrt(2))
    P = np.exp(S) / np.exp(S).sum(1, keepdims=True)
    o, lse = ref.forward(q, k, v, alpha, base, False)
    np.testing.assert_allclose(o[0, 0], P @ v[0, 0], atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], np.log(np.exp(S).sum(1)), atol=1e-14)


# ---------------------------------------------------------------- loss special case
def test_loss_zero_when_target_is_output():
    q, k, v, _, alpha, base = rand_problem(37, 1, 2, 9, 8)
    o, _ = ref.forward(q, k, v, alpha, base, False)
    r = ref.forward_backward(q, k, v, o.copy(), alpha, base, False)
    assert r["L"] == 0.0
    for key in ("dq", "dk", "dv", "dalpha"):
        assert np.max(np.abs(r[key])) == 0.0


# ---------------------------------------------------------------- regression fixture
def test_oracle_regression_fixture():
    """The oracle still produces what tests/golden/make_golden.py recorded."""
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_small.json")
    g = json.load(open(path))
    arr = lambda key: np.array(g[key], dtype=np.float64)
    r = ref.forward_backward(arr("q"), arr("k"), arr("v"), arr("e"), arr("alpha"), g["base"],
                             g["causal"])
    for key in ("o", "lse", "dq", "dk", "dv", "dalpha"):
        np.testing.assert_allclose(r[key], arr(key), rtol=1e-13, atol=1e-14)
    assert abs(r["L"] - g["L"]) <= 1e-13 * abs(g["L"])


# ---------------------------------------------------------------- row / column restrictions
@pytest.mark.parametrize("causal", [False, True])
def test_row_and_column_restricted_backward(causal):
    """head_backward_rows / _cols (used at full sizes on sampled rows) equal the rows of the
    full blocked backward; Delta taken as rowsum(dO o O)."""
    n, d = 37, 8
    q, k, v, e, alpha, base = rand_problem(41, 1, 1, n, d, base=300.0)
    _, th = ref.frequencies(d, base, alpha)
    phi = ref.angles(n, th)
    qt, kt = ref.rotate(q[0, 0], phi), ref.rotate(k[0, 0], phi)
    o, lse = ref.head_forward(qt, kt, v[0, 0], causal)
    do = o - e[0, 0]
    delta = np.sum(do * o, axis=1)
    dqt, dkt, dv = ref.head_backward(qt, kt, v[0, 0], do, causal, block=5)
    rows = np.array([0, 3, 17, 36])
    np.testing.assert_allclose(
        ref.head_backward_rows(qt, kt, v[0, 0], do[rows], lse[rows], delta[rows], rows, causal),
        dqt[rows], atol=1e-13)
    ck, cv = ref.head_backward_cols(qt, kt, v[0, 0], do, lse, delta, rows, causal)
    np.testing.assert_allclose(ck, dkt[rows], atol=1e-13)
    np.testing.assert_allclose(cv, dv[rows], atol=1e-13)


# ---------------------------------------------------------------- variants: p-RoPE fixed bands
def test_fixed_bands_all_is_plain_attention():
    """Every band fixed (no rotation at all) is plain softmax attention: torch's
    scaled_dot_product_attention on the unrotated q, k; and dalpha is exactly 0."""
    B, H, n, d = 1, 2, 21, 8
    q, k, v, e, alpha, base = rand_problem(41, B, H, n, d, alpha_scale=0.5)
    o, _ = ref.forward(q, k, v, alpha, base, True, fixed_bands=d // 2)
    sd = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q), torch.tensor(k), torch.tensor(v), is_causal=True).numpy()
    np.testing.assert_allclose(o, sd, atol=1e-13)
    _, do = ref.loss(o, e)
    assert np.all(ref.backward(q, k, v, do, alpha, base, True, fixed_bands=d // 2)[3] == 0.0)


@pytest.mark.parametrize("causal", [False, True])
def test_fixed_bands_autograd(causal):
    """p-RoPE (the slowest f bands unrotated) against an independent complex-multiplication
    forward with those bands' frequency set to zero, differentiated by autograd: the fixed
    bands get dalpha = 0 (their frequency does not depend on alpha), the others agree."""
    B, H, n, d, f = 1, 2, 29, 16, 2
    q, k, v, e, alpha, base = rand_problem(43, B, H, n, d, alpha_scale=0.6, base=300.0)
    r = ref.forward_backward(q, k, v, e, alpha, base, causal, block=8, fixed_bands=f)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    ta = torch.tensor(alpha, requires_grad=True)
    m = torch.arange(d // 2, dtype=torch.float64)
    keep = (m < d // 2 - f).to(torch.float64)
    th = torch.exp(ta) * base ** (-2.0 * m / d) * keep
    pos = torch.arange(n, dtype=torch.float64)
    qr, kr = _torch_rope_complex(tq, pos, th), _torch_rope_complex(tk, pos, th)
    s = qr @ kr.transpose(-1, -2) / math.sqrt(d)
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), float("-inf"))
    o = torch.softmax(s, dim=-1) @ tv
    L = 0.5 * ((o - torch.tensor(e)) ** 2).sum()
    L.backward()
    np.testing.assert_allclose(o.detach().numpy(), r["o"], atol=1e-12)
    for g, key in ((tq.grad, "dq"), (tk.grad, "dk"), (tv.grad, "dv")):
        np.testing.assert_allclose(g.numpy(), r[key], atol=1e-11)
    np.testing.assert_allclose(ta.grad.numpy(), r["dalpha"], rtol=1e-10, atol=1e-11)
    assert np.all(r["dalpha"][d // 2 - f:] == 0.0)


def test_fixed_bands_limit_of_vanishing_frequency():
    """Fixing a band equals sending its alpha to -inf: O and the other bands' dalpha match
    alpha_m = -80 (theta_hat ~ 1.8e-35) to rounding."""
    B, H, n, d, f = 1, 1, 24, 16, 3
    q, k, v, e, alpha, base = rand_problem(47, B, H, n, d, alpha_scale=0.5)
    a2 = alpha.copy()
    a2[d // 2 - f:] = -80.0
    r1 = ref.forward_backward(q, k, v, e, alpha, base, True, fixed_bands=f)
    r2 = ref.forward_backward(q, k, v, e, a2, base, True)
    for key in ("o", "dq", "dk", "dv"):
        np.testing.assert_allclose(r1[key], r2[key], atol=1e-13)
    np.testing.assert_allclose(r1["dalpha"][: d // 2 - f], r2["dalpha"][: d // 2 - f],
                               rtol=1e-10)


# ---------------------------------------------------------------- variants: the alpha optimiser step
def test_alpha_adam_matches_torch_adam_with_own_clipping():
    """Three steps of the oracle's alpha update against torch.optim.Adam (weight_decay=0)
    fed the gradient clipped by torch.nn.utils.clip_grad_norm_.  torch clips by
    max_norm / (norm + 1e-6), the oracle to exactly max_norm; that moves alpha by ~1e-11
    here, while a wrong moment, sign or bias correction moves it by ~1e-3 (lr = 3e-3)."""
    M = 32
    rng = np.random.default_rng(53)
    alpha = 0.2 * rng.standard_normal(M)
    p = torch.nn.Parameter(torch.tensor(alpha))
    opt = torch.optim.Adam([p], lr=3e-3, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.0)
    m1 = np.zeros(M)
    m2 = np.zeros(M)
    a = alpha.copy()
    for t in (1, 2, 3):
        g = (2.0 ** t) * rng.standard_normal(M)   # norms above and below the clip
        a, m1, m2 = ref.alpha_adam_step(a, g, m1, m2, t, 3e-3, 0.9, 0.95, 1e-8, clip_norm=4.0)
        opt.zero_grad()
        p.grad = torch.tensor(g)
        torch.nn.utils.clip_grad_norm_([p], 4.0)
        opt.step()
        np.testing.assert_allclose(a, p.detach().numpy(), rtol=0, atol=1e-9)


def test_alpha_adam_closed_forms():
    """First step: the bias-corrected moments are g and g^2, so each alpha_m moves by
    -lr g_m / (|g_m| + eps); the first moment after clipping is (1 - beta1) g clip / |g|."""
    M = 16
    rng = np.random.default_rng(59)
    g = rng.standard_normal(M) * 10.0
    a, m1, _ = ref.alpha_adam_step(np.zeros(M), g, np.zeros(M), np.zeros(M), 1, 0.01,
                                   clip_norm=0.0)
    np.testing.assert_allclose(a, -0.01 * g / (np.abs(g) + 1e-8), rtol=1e-12)
    nrm = np.linalg.norm(g)
    _, m1, _ = ref.alpha_adam_step(np.zeros(M), g, np.zeros(M), np.zeros(M), 1, 0.01,
                                   clip_norm=1.0)
    np.testing.assert_allclose(m1, 0.1 * g / nrm, rtol=1e-12)


# ---------------------------------------------------------------- the projections (Lemma 4.1)
def test_projection_gradients_match_autograd_of_the_layer():
    """X -> (Q, K, V) = X W -> LeRoPE attention -> L, differentiated by autograd (the
    complex-multiplication forward of I4b), against the oracle's chain: forward_backward on
    the projected q, k, v, then proj_backward for dW_Q, dW_K, dW_V and dX."""
    B, H, n, d, dm = 2, 2, 17, 8, 12
    rng = np.random.default_rng(61)
    x = rng.standard_normal((B, n, dm))
    wq, wk, wv = (0.3 * rng.standard_normal((dm, H * d)) for _ in range(3))
    e = rng.standard_normal((B, H, n, d))
    alpha = 0.4 * rng.standard_normal(d // 2)
    base = 200.0
    q, k, v = ref.proj_forward(x, wq, wk, wv, H)
    r = ref.forward_backward(q, k, v, e, alpha, base, True, block=8)
    dwq, dwk, dwv, dx = ref.proj_backward(x, wq, wk, wv, r["dq"], r["dk"], r["dv"])
    tx = torch.tensor(x, requires_grad=True)
    tw = [torch.tensor(w, requires_grad=True) for w in (wq, wk, wv)]
    m = torch.arange(d // 2, dtype=torch.float64)
    th = torch.exp(torch.tensor(alpha)) * base ** (-2.0 * m / d)
    pos = torch.arange(n, dtype=torch.float64)
    def heads(y):
        return y.reshape(B, n, H, d).transpose(1, 2)
    tq, tk, tv = (heads(tx @ w) for w in tw)
    qr, kr = _torch_rope_complex(tq, pos, th), _torch_rope_complex(tk, pos, th)
    s = (qr @ kr.transpose(-1, -2) / math.sqrt(d)).masked_fill(
        torch.triu(torch.ones(n, n, dtype=torch.bool), 1), float("-inf"))
    o = torch.softmax(s, dim=-1) @ tv
    (0.5 * ((o - torch.tensor(e)) ** 2).sum()).backward()
    for g, want in zip(tw, (dwq, dwk, dwv)):
        np.testing.assert_allclose(g.grad.numpy(), want, atol=1e-11)
    np.testing.assert_allclose(tx.grad.numpy(), dx, atol=1e-11)


# ---------------------------------------------------------------- the spectrum of the gradient signal
@pytest.mark.parametrize("causal", [False, True])
def test_offset_signal_surrogate_equals_score_inner_product(causal):
    """sum over bands of P_m(theta_hat_m) = sum_ij dS_ij S_ij: the surrogate evaluated at the
    model's own frequencies gives back each band's share of the scores (S from the rotated
    vectors, dS from the backward's matrices, per head)."""
    B, H, n, d = 1, 2, 14, 8
    q, k, v, e, alpha, base = rand_problem(67, B, H, n, d, alpha_scale=0.5, base=50.0)
    r = ref.forward_backward(q, k, v, e, alpha, base, causal)
    g = ref.offset_signal(q, k, v, r["do"], alpha, base, causal)
    _, th = ref.frequencies(d, base, alpha)
    offs = np.arange(-(n - 1), n)
    surrogate = np.sum(np.real(g * np.exp(1j * np.outer(th, offs))))
    phi = ref.angles(n, th)
    want = 0.0
    for h in range(H):
        qt, kt = ref.rotate(q[0, h], phi), ref.rotate(k[0, h], phi)
        _, ds = ref.head_matrices(qt, kt, v[0, h], r["do"][0, h], causal)
        s = qt @ kt.T / np.sqrt(d)
        want += np.sum(np.where(np.isfinite(ds), ds, 0.0) * s)
    np.testing.assert_allclose(surrogate, want, rtol=1e-11, atol=1e-12)
    if causal:
        assert np.all(g[:, : n - 1] == 0)   # no key after its query: no negative offset
