"""Float64 CPU oracle for exact RoPE / LeRoPE softmax attention, forward and backward.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it.  It shares no code with the CUDA path.

What it computes, per (batch b, head h), with positions p = 0..n-1 and
M = d/2 frequency bands:

1.  theta_m = base^(-2m/d), theta_hat_m = exp(alpha_m) * theta_m.
    ("LeRoPE: learnable RoPE frequencies", Metodologia: LeRoPE / Mecanismo
    Central -- the effective frequency is the standard RoPE frequency rescaled
    by a learned exponential; the standard frequencies form a geometric
    sequence set by the base b, Declaracao do Problema.  The exponent -2m/d is
    the standard RoPE choice; the page leaves it open.)
2.  Band m of each query/key is rotated in its 2-D plane by the angle
    p * theta_hat_m ("LeRoPE", Declaracao do Problema: RoPE rotates queries and
    keys in two-dimensional frequency bands).  Band m is the pair of
    coordinates (2m, 2m+1) ("interleaved", the default) or (m, m+M)
    ("halfsplit"); the choice is a fixed column permutation.
3.  S = Q~ K~^T / sqrt(d); causal: S_ij = -inf for j > i.
4.  P = D^-1 exp(S) with D the diagonal of row sums -- the normalised softmax
    s(x) of "RoPE attention can be trained in almost-linear time",
    Metodologia 1 (closed-form gradient); O = P V; lse_i = log sum_j exp(S_ij).
5.  L = 1/2 ||O - E||_F^2 and dO = O - E: the error term l(x), the difference
    between the attention output and the target (same page, Metodologia 1).
6.  dV = P^T dO; beta = dP = dO V^T (the error combined with the value matrix);
    gamma = diag(s) beta - s s^T beta row by row, i.e. dS = P o (dP - rowsum(P o dP))
    (same page, Metodologia 1 and 2, gamma_1 - gamma_2).
7.  dQ~ = dS K~ / sqrt(d), dK~ = dS^T Q~ / sqrt(d); dQ, dK = band-wise rotation
    by -p * theta_hat_m of dQ~, dK~ (the transpose of step 2).
8.  dalpha_m = theta_hat_m * sum_{b,h,p} p * (<dQ~_pm, J q~_pm> + <dK~_pm, J k~_pm>),
    J = [[0, -1], [1, 0]] (the derivative of a 2-D rotation), with alpha shared
    by every head ("LeRoPE", Escolhas de Design Principais: one set of d/2
    frequencies shared across all layers and heads; log-space parametrisation).

Variants ("LeRoPE", Configuracao Experimental and Ablacao):
- fixed_bands = f: the f slowest bands (m >= M - f) keep theta_hat_m = 0, i.e. are not
  rotated -- partial RoPE, the p-RoPE baseline with p = 1 - f/M (p = 0.75 drops the
  slowest 25% of bands).  Their dalpha is 0: theta_hat_m does not depend on alpha_m.
- frozen frequencies: alpha given, no dalpha (the backward's step 8 skipped).
- the optimiser step for alpha ("LeRoPE", Escolhas de Design Principais: no weight decay
  on the LeRoPE parameters, their gradient clipped separately): :func:`alpha_adam_step`.

A second, independent formula for dalpha -- the derivative of the real part of
the DTFT of the offset-aggregated gradient signal ("LeRoPE", Analise Teorica)
-- is :func:`dalpha_offset_dtft`.

Everything is float64.  Inputs are the values the GPU sees (already rounded
to the storage dtype), widened exactly.  Query rows are processed in blocks of
full rows, so each row's softmax is the plain definition.
"""
import numpy as np


# --------------------------------------------------------------------------
# step 1-2: frequencies, angles, band rotation
# --------------------------------------------------------------------------
def frequencies(d, base, alpha, fixed_bands=0):
    """theta_m = base^(-2m/d) and theta_hat_m = exp(alpha_m) theta_m, m < d/2; the
    fixed_bands slowest bands (m >= d/2 - fixed_bands) get theta_hat_m = 0."""
    M = d // 2
    m = np.arange(M, dtype=np.float64)
    theta = np.power(float(base), -2.0 * m / d)
    theta_hat = np.exp(np.asarray(alpha, dtype=np.float64)) * theta
    if fixed_bands:
        theta_hat = np.where(m >= M - fixed_bands, 0.0, theta_hat)
    return theta, theta_hat


def angles(n, theta_hat, offset=0):
    """phi[p, m] = (p + offset) * theta_hat_m for positions p = 0..n-1."""
    p = np.arange(n, dtype=np.float64) + offset
    return p[:, None] * np.asarray(theta_hat, dtype=np.float64)[None, :]


def band_index(d, pairing="interleaved"):
    """Column indices (first, second) of each band's 2-D plane."""
    M = d // 2
    if pairing == "interleaved":
        return np.arange(0, d, 2), np.arange(1, d, 2)
    if pairing == "halfsplit":
        return np.arange(M), np.arange(M, d)
    raise ValueError(pairing)


def rotate(x, phi, pairing="interleaved", sign=1.0):
    """Rotate band m of row p of x ([..., n, d]) by sign * phi[p, m]."""
    i0, i1 = band_index(x.shape[-1], pairing)
    c, s = np.cos(phi), sign * np.sin(phi)
    y = np.empty_like(x, dtype=np.float64)
    x0, x1 = x[..., i0], x[..., i1]
    y[..., i0] = c * x0 - s * x1
    y[..., i1] = s * x0 + c * x1
    return y


# --------------------------------------------------------------------------
# steps 3-7 for one head, in blocks of full query rows
# --------------------------------------------------------------------------
def _scores(qt_rows, kt, rows, causal, scale):
    s = (qt_rows @ kt.T) * scale
    if causal:
        cols = np.arange(kt.shape[0])
        s = np.where(cols[None, :] > rows[:, None], -np.inf, s)
    return s


def _softmax_rows(s):
    mx = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - mx)
    z = np.sum(e, axis=1, keepdims=True)
    return e / z, (mx + np.log(z))[:, 0]


def head_forward(qt, kt, v, causal, rows=None, block=512):
    """O and lse of the given query rows (default all) for rotated q~, k~ of one head."""
    n, d = qt.shape
    scale = 1.0 / np.sqrt(d)
    rows = np.arange(n) if rows is None else np.asarray(rows)
    o = np.empty((len(rows), v.shape[1]))
    lse = np.empty(len(rows))
    for a in range(0, len(rows), block):
        r = rows[a:a + block]
        p, l = _softmax_rows(_scores(qt[r], kt, r, causal, scale))
        o[a:a + block] = p @ v
        lse[a:a + block] = l
    return o, lse


def head_backward(qt, kt, v, do, causal, block=512):
    """dQ~, dK~, dV of one head from the upstream gradient dO (= l(x))."""
    n, d = qt.shape
    scale = 1.0 / np.sqrt(d)
    dqt = np.empty_like(qt)
    dkt = np.zeros_like(kt)
    dv = np.zeros_like(v)
    for a in range(0, n, block):
        r = np.arange(a, min(n, a + block))
        p, _ = _softmax_rows(_scores(qt[r], kt, r, causal, scale))   # s(x)
        beta = do[r] @ v.T                                           # beta(x)
        gamma1 = p * beta                                            # diag(s) beta
        gamma2 = p * np.sum(p * beta, axis=1, keepdims=True)         # s s^T beta
        ds = gamma1 - gamma2                                         # gamma(x)
        dv += p.T @ do[r]
        dqt[r] = (ds @ kt) * scale
        dkt += (ds.T @ qt[r]) * scale
    return dqt, dkt, dv


def head_backward_rows(qt, kt, v, do_rows, lse_rows, delta_rows, rows, causal):
    """dQ~ of the given query rows only (row i needs its own lse_i and Delta_i)."""
    n, d = qt.shape
    scale = 1.0 / np.sqrt(d)
    rows = np.asarray(rows)
    s = _scores(qt[rows], kt, rows, causal, scale)
    p = np.exp(s - lse_rows[:, None])                                # s(x), rows
    beta = do_rows @ v.T
    ds = p * beta - p * delta_rows[:, None]                          # gamma(x), rows
    return (ds @ kt) * scale


def head_backward_cols(qt, kt, v, do, lse, delta, cols, causal):
    """dK~ and dV of the given key rows only; needs every query's lse and Delta."""
    n, d = qt.shape
    scale = 1.0 / np.sqrt(d)
    cols = np.asarray(cols)
    s = (qt @ kt[cols].T) * scale                                    # n x |cols|
    if causal:
        s = np.where(cols[None, :] > np.arange(n)[:, None], -np.inf, s)
    p = np.exp(s - lse[:, None])
    beta = do @ v[cols].T
    ds = p * beta - p * delta[:, None]
    return (ds.T @ qt) * scale, p.T @ do


def head_matrices(qt, kt, v, do, causal):
    """Full n x n P and dS of one head (small n only): for pins and the DTFT form."""
    n, d = qt.shape
    r = np.arange(n)
    p, _ = _softmax_rows(_scores(qt, kt, r, causal, 1.0 / np.sqrt(d)))
    beta = do @ v.T
    ds = p * beta - p * np.sum(p * beta, axis=1, keepdims=True)
    return p, ds


# --------------------------------------------------------------------------
# public API over [B, H, n, d]
# --------------------------------------------------------------------------
def forward(q, k, v, alpha, base, causal, pairing="interleaved", offset=0, block=512,
            fixed_bands=0):
    """O [B,H,n,d] and lse [B,H,n] (natural log) in float64."""
    B, H, n, d = q.shape
    _, th = frequencies(d, base, alpha, fixed_bands)
    phi = angles(n, th, offset)
    o = np.empty((B, H, n, d))
    lse = np.empty((B, H, n))
    for b in range(B):
        for h in range(H):
            qt = rotate(q[b, h], phi, pairing)
            kt = rotate(k[b, h], phi, pairing)
            o[b, h], lse[b, h] = head_forward(qt, kt, v[b, h], causal, block=block)
    return o, lse


def loss(o, e):
    """L = 1/2 ||O - E||_F^2 summed over every element, and dO = O - E."""
    do = np.asarray(o, dtype=np.float64) - np.asarray(e, dtype=np.float64)
    return 0.5 * float(np.sum(do * do)), do


def band_torque(g, x, pairing="interleaved"):
    """<g_pm, J x_pm> for every row p and band m: g1*x0 - g0*x1."""
    i0, i1 = band_index(x.shape[-1], pairing)
    return g[..., i1] * x[..., i0] - g[..., i0] * x[..., i1]


def backward(q, k, v, do, alpha, base, causal, pairing="interleaved", offset=0, block=512,
             return_rotated=False, fixed_bands=0):
    """dQ, dK, dV [B,H,n,d] and dalpha [d/2] in float64 for upstream gradient dO."""
    B, H, n, d = q.shape
    _, th = frequencies(d, base, alpha, fixed_bands)
    phi = angles(n, th, offset)
    pos = np.arange(n, dtype=np.float64) + offset
    dq = np.empty((B, H, n, d))
    dk = np.empty((B, H, n, d))
    dv = np.empty((B, H, n, d))
    acc = np.zeros(d // 2)
    extra = []
    for b in range(B):
        for h in range(H):
            qt = rotate(q[b, h], phi, pairing)
            kt = rotate(k[b, h], phi, pairing)
            dqt, dkt, dv[b, h] = head_backward(qt, kt, v[b, h], do[b, h], causal, block)
            dq[b, h] = rotate(dqt, phi, pairing, sign=-1.0)
            dk[b, h] = rotate(dkt, phi, pairing, sign=-1.0)
            tq = band_torque(dqt, qt, pairing)
            tk = band_torque(dkt, kt, pairing)
            acc += pos @ (tq + tk)
            if return_rotated:
                extra.append((qt, kt, dqt, dkt))
    dalpha = th * acc
    if return_rotated:
        return dq, dk, dv, dalpha, extra
    return dq, dk, dv, dalpha


def forward_backward(q, k, v, e, alpha, base, causal, **kw):
    """The whole path: O, lse, L, dO, dQ, dK, dV, dalpha."""
    o, lse = forward(q, k, v, alpha, base, causal, **kw)
    L, do = loss(o, e)
    dq, dk, dv, dalpha = backward(q, k, v, do, alpha, base, causal, **kw)
    return dict(o=o, lse=lse, L=L, do=do, dq=dq, dk=dk, dv=dv, dalpha=dalpha)


# --------------------------------------------------------------------------
# second formula for dalpha: derivative of the DTFT surrogate
# --------------------------------------------------------------------------
def offset_signal(q, k, v, do, alpha, base, causal, pairing="interleaved", fixed_bands=0):
    """The offset-aggregated gradient signal ("LeRoPE", Analise Teorica), summed over every
    batch and head: g[m, D + n - 1] = sum_{i - j = D} dS_ij z_q,i conj(z_k,j) / sqrt(d) for
    offsets D = -(n-1)..n-1, with band m of a row read as z = x0 + i x1 of the UNROTATED
    q, k (a rotation by psi is multiplication by exp(i psi)).  Then the band's share of the
    scores is S_ij^(m) = Re(exp(i (i-j) theta_hat_m) z_q,i conj(z_k,j)) / sqrt(d), and
    P_m(theta) = Re sum_D g_m(D) exp(i D theta), the real part of the DTFT of g_m, is the
    surrogate whose derivative at theta_hat_m is dL/dtheta_hat_m.  Small n only (n x n)."""
    B, H, n, d = q.shape
    _, th = frequencies(d, base, alpha, fixed_bands)
    phi = angles(n, th)
    i0, i1 = band_index(d, pairing)
    D = np.arange(n)[:, None] - np.arange(n)[None, :]
    g = np.zeros((d // 2, 2 * n - 1), dtype=complex)
    for b in range(B):
        for h in range(H):
            qt = rotate(q[b, h], phi, pairing)
            kt = rotate(k[b, h], phi, pairing)
            _, ds = head_matrices(qt, kt, v[b, h], do[b, h], causal)
            zq = q[b, h][:, i0] + 1j * q[b, h][:, i1]
            zk = k[b, h][:, i0] + 1j * k[b, h][:, i1]
            for m in range(d // 2):
                w = ds * np.outer(zq[:, m], np.conj(zk[:, m])) / np.sqrt(d)
                np.add.at(g[m], (D + n - 1).ravel(), w.ravel())
    return g


def dtft_derivative(g, theta):
    """P_m'(theta_m) = d/dtheta Re sum_D g_m(D) exp(i D theta) at theta = theta_m, for the
    signal g [M, 2n - 1] of offsets D = -(n-1)..n-1."""
    n = (g.shape[1] + 1) // 2
    offs = np.arange(-(n - 1), n)
    ph = np.exp(1j * np.outer(np.asarray(theta, dtype=np.float64), offs))
    return np.real(np.sum(1j * offs[None, :] * g * ph, axis=1))


def dalpha_offset_dtft(q, k, v, do, alpha, base, causal, pairing="interleaved", fixed_bands=0):
    """dalpha via the offset-aggregated gradient signal ("LeRoPE", Analise Teorica):
    dalpha_m = theta_hat_m P_m'(theta_hat_m) with g_m from :func:`offset_signal`."""
    d = q.shape[3]
    _, th = frequencies(d, base, alpha, fixed_bands)
    g = offset_signal(q, k, v, do, alpha, base, causal, pairing, fixed_bands)
    return th * dtft_derivative(g, th)


# --------------------------------------------------------------------------
# the optimiser step for alpha
# --------------------------------------------------------------------------
def alpha_adam_step(alpha, dalpha, m1, m2, step, lr, beta1=0.9, beta2=0.999, eps=1e-8,
                    clip_norm=1.0):
    """One Adam step for the LeRoPE log-frequencies with their own gradient clipping and no
    weight decay ("LeRoPE", Escolhas de Design Principais: Otimizacao).  The page names
    neither the optimiser nor the clipping rule; this is the plainest reading: dalpha is
    scaled to L2 norm clip_norm when its norm exceeds it (clip_norm <= 0: no clipping),
    then the Adam update (first and second moments m1, m2 with bias correction at the
    1-based step t) is applied with weight decay 0.  Returns (alpha, m1, m2)."""
    g = np.asarray(dalpha, dtype=np.float64)
    if clip_norm > 0:
        nrm = float(np.sqrt(np.sum(g * g)))
        if nrm > clip_norm:
            g = g * (clip_norm / nrm)
    m1 = beta1 * np.asarray(m1, dtype=np.float64) + (1.0 - beta1) * g
    m2 = beta2 * np.asarray(m2, dtype=np.float64) + (1.0 - beta2) * g * g
    m_hat = m1 / (1.0 - beta1 ** step)
    v_hat = m2 / (1.0 - beta2 ** step)
    alpha = np.asarray(alpha, dtype=np.float64) - lr * m_hat / (np.sqrt(v_hat) + eps)
    return alpha, m1, m2


# --------------------------------------------------------------------------
# the projections around the path (Lemma 4.1's gradient with respect to the weights)
# --------------------------------------------------------------------------
def proj_forward(x, wq, wk, wv, H):
    """q, k, v [B, H, n, d] = x [B, n, d_model] W [d_model, H d] split into heads."""
    B, n, _ = x.shape
    d = wq.shape[1] // H
    def split(y):
        return y.reshape(B, n, H, d).transpose(0, 2, 1, 3)
    x = np.asarray(x, dtype=np.float64)
    return tuple(split(x @ np.asarray(w, dtype=np.float64)) for w in (wq, wk, wv))


def proj_backward(x, wq, wk, wv, dq, dk, dv):
    """dW = sum_b x_b^T dY_b with dY_b = dq[b] merged to [n, H d] (likewise dW_K, dW_V) and
    dx = sum over q, k, v of dY W^T ("RoPE attention can be trained in almost-linear time",
    Lemma 4.1: the gradient with respect to the weights; the chain rule through Y = X W)."""
    x = np.asarray(x, dtype=np.float64)
    B, n, dm = x.shape
    out, dx = [], np.zeros((B, n, dm))
    for w, g in ((wq, dq), (wk, dk), (wv, dv)):
        g = np.asarray(g, dtype=np.float64)
        gm = g.transpose(0, 2, 1, 3).reshape(B, n, -1)          # [B, n, H d]
        out.append(np.einsum("bnm,bnc->mc", x, gm))
        dx += gm @ np.asarray(w, dtype=np.float64).T
    return out[0], out[1], out[2], dx
