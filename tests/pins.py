"""Pins: facts fixed by the pages or by mathematics, used to check the oracle.

Each ``pin_*`` function takes the oracle module (or a deliberately broken
copy of it) and raises ``AssertionError`` when the implementation disagrees
with the fact.  ``tests/test_oracle_pins.py`` runs them on the real oracle and
shows that plausible mistakes planted in a copy of the oracle fail at least
one of them.

None of the expected values below is obtained by calling the function under
test: they come from a scalar recurrence, an independent Jacobi SVD, exact
rational arithmetic, or an algebraic identity.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

EPS = 1e-7   # blog "Muon 核心" listing: G / (G.norm() + 1e-7)


# ----------------------------------------------------------------- helpers
def cubic_map(s: float, k: int) -> float:
    """f^k(s) for f(s) = 1.5 s - 0.5 s^3: the action of one cubic step on a
    single singular value (blog, "Muon 核心" G_{t+1} equation applied to
    G = U diag(s) V^T)."""
    for _ in range(k):
        s = 1.5 * s - 0.5 * s * s * s
    return s


def jacobi_svd(G: np.ndarray, tol: float = 1e-15, max_sweeps: int = 60):
    """One-sided (Hestenes) Jacobi SVD written out by hand.

    Returns U (p x r), sigma (r), V (q x r) with G = U diag(sigma) V^T, where
    r = min(p, q).  Rotations orthogonalise the columns of the tall
    orientation until every pair is orthogonal to ``tol``.
    """
    G = np.asarray(G, dtype=np.float64)
    flip = G.shape[0] < G.shape[1]
    A = (G.T if flip else G).copy()
    q = A.shape[1]
    V = np.eye(q)
    for _ in range(max_sweeps):
        rotated = False
        for i in range(q - 1):
            for j in range(i + 1, q):
                a = float(A[:, i] @ A[:, i])
                b = float(A[:, j] @ A[:, j])
                c = float(A[:, i] @ A[:, j])
                if abs(c) <= tol * math.sqrt(a * b) or c == 0.0:
                    continue
                rotated = True
                zeta = (b - a) / (2.0 * c)
                t = math.copysign(1.0, zeta) / (abs(zeta) + math.sqrt(1.0 + zeta * zeta))
                cs = 1.0 / math.sqrt(1.0 + t * t)
                sn = cs * t
                ai, aj = A[:, i].copy(), A[:, j].copy()
                A[:, i] = cs * ai - sn * aj
                A[:, j] = sn * ai + cs * aj
                vi, vj = V[:, i].copy(), V[:, j].copy()
                V[:, i] = cs * vi - sn * vj
                V[:, j] = sn * vi + cs * vj
        if not rotated:
            break
    sigma = np.sqrt(np.sum(A * A, axis=0))
    U = np.zeros_like(A)
    nz = sigma > 0
    U[:, nz] = A[:, nz] / sigma[nz]
    if flip:
        return V, sigma, U
    return U, sigma, V


def _rel(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    d = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (d if d > 0 else 1.0))


def _semi_orthogonal(rng, m: int, n: int) -> np.ndarray:
    """An m x n matrix with orthonormal rows (m <= n)."""
    Q, _ = np.linalg.qr(rng.standard_normal((n, m)))
    return Q.T.copy()


def exact_f32_round(x: Fraction) -> np.float32:
    """Round an exact rational to the nearest float32, ties to even."""
    guess = np.float32(float(x))
    cands = {float(guess), float(np.nextafter(guess, np.float32(np.inf))),
             float(np.nextafter(guess, np.float32(-np.inf)))}
    best = None
    for c in sorted(cands):
        err = abs(Fraction(c) - x)
        if best is None or err < best[0]:
            best = (err, c)
        elif err == best[0]:
            # tie: keep the one with an even last mantissa bit
            bits = np.array([c], dtype=np.float32).view(np.uint32)[0]
            if bits & 1 == 0:
                best = (err, c)
    return np.float32(best[1])


def exact_bf16_round(x: Fraction) -> float:
    """Round an exact rational in the normal range to the nearest bfloat16
    (8 significant bits), ties to even, worked out on the rational itself."""
    if x == 0:
        return 0.0
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = math.floor(math.log2(a))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 7)
    q = a / ulp                      # in [128, 256)
    lo = math.floor(q)
    rem = q - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return float(sign * lo * ulp)


# -------------------------------------------------------------------- pins
def pin_scalar_closed_form(o) -> None:
    """A 1x1 input reduces to s0 = x / (|x| + 1e-7), s <- 1.5 s - 0.5 s^3."""
    for x in (3.0, -2.5, 1e-6, -1e-7, 0.37, 0.0):
        for k in (0, 1, 2, 5, 9):
            got = o.newton_schulz(np.array([[x]]), k)[0, 0]
            want = cubic_map(x / (abs(x) + EPS), k)
            assert abs(got - want) <= 1e-15 * max(1.0, abs(want)), (x, k, got, want)


def pin_spectral_map(o, seed: int = 11) -> None:
    """For small random matrices (both orientations) the output equals
    U diag(f^k(sigma / (||G||_F + 1e-7))) V^T, with U, sigma, V from a
    hand-written Jacobi SVD: cubic NS is an odd matrix polynomial and acts on
    each singular value independently."""
    rng = np.random.default_rng(seed)
    for (p, q) in ((1, 7), (5, 5), (7, 3), (12, 30), (30, 12), (48, 96), (17, 17)):
        G = rng.standard_normal((p, q))
        if p == q == 17:
            G = np.triu(G) + 0.3 * np.eye(p)   # non-normal square input
        U, sig, V = jacobi_svd(G)
        nrm = math.sqrt(float(np.sum(G * G)))
        for k in (1, 3, 5):
            fs = np.array([cubic_map(s / (nrm + EPS), k) for s in sig])
            want = (U * fs) @ V.T
            got = o.newton_schulz(G, k)
            assert got.shape == G.shape
            assert _rel(got, want) <= 1e-12, (p, q, k, _rel(got, want))


def pin_orthogonal_input(o, seed: int = 12) -> None:
    """Orthogonal rows are a fixed point of the inner cubic step (f(1) = 1);
    the full function maps c*Q to f^k(c / (c sqrt(m) + 1e-7)) * Q."""
    rng = np.random.default_rng(seed)
    for (m, n) in ((8, 8), (16, 40), (33, 64)):
        Q = _semi_orthogonal(rng, m, n)
        assert _rel(o.ns_iteration(Q), Q) <= 1e-14
        for c in (1.0, 0.01, 50.0):
            for k in (0, 1, 5):
                s0 = c / (c * math.sqrt(m) + EPS)
                want = cubic_map(s0, k) * Q
                assert _rel(o.newton_schulz(c * Q, k), want) <= 1e-13
                assert _rel(o.newton_schulz((c * Q).T, k), want.T) <= 1e-13


def pin_monotone_error(o, seed: int = 13) -> None:
    """||X X^T - I||_F does not increase with the step count: after
    normalisation every singular value lies in [0, 1], where f is increasing
    and f(s) >= s, so each value moves monotonically toward 1."""
    rng = np.random.default_rng(seed)
    cases = [rng.standard_normal((64, 128)),
             _semi_orthogonal(rng, 32, 48) * rng.uniform(0.5, 1.0, size=(32, 1)),
             rng.standard_normal((96, 40))]
    for G in cases:
        errs = []
        for k in range(0, 12):
            X = o.newton_schulz(G, k)
            errs.append(o.orthogonality_error(X))
        for a, b in zip(errs, errs[1:]):
            assert b <= a + 1e-12, errs


def pin_symmetries(o, seed: int = 14) -> None:
    """NS(G^T) = NS(G)^T; NS(cG) = NS(G) for c > 0 far above the epsilon;
    zero maps to zero; a rank-8 input with equal singular values follows the
    scalar map from 1/sqrt(8)."""
    rng = np.random.default_rng(seed)
    G = rng.standard_normal((24, 56))
    G *= 1e3 / np.linalg.norm(G)          # eps / ||G|| = 1e-10: far below the bound
    assert _rel(o.newton_schulz(G.T, 5), o.newton_schulz(G, 5).T) <= 1e-13
    assert _rel(o.newton_schulz(1000.0 * G, 5), o.newton_schulz(G, 5)) <= 1e-9
    Z = o.newton_schulz(np.zeros((6, 9)), 5)
    assert np.all(Z == 0.0)
    U = _semi_orthogonal(rng, 8, 64).T           # 64 x 8, orthonormal columns
    V = _semi_orthogonal(rng, 8, 96).T           # 96 x 8
    R = U @ V.T                                   # rank 8, singular values 1
    X = o.newton_schulz(R, 5)
    want = cubic_map(1.0 / (math.sqrt(8.0) + EPS), 5) * R   # ||R||_F = sqrt(8)
    assert _rel(X, want) <= 1e-13


def pin_momentum_bitwise(o, seed: int = 15) -> None:
    """buf' = fl32(fl32(mu * buf) + g): each value checked against exact
    rational arithmetic rounded once per operation (blog, Vanilla Muon:
    ``mul_(momentum)`` then ``add_(grad)``)."""
    rng = np.random.default_rng(seed)
    buf = (rng.standard_normal(300) * 10.0 ** rng.integers(-8, 4, 300)).astype(np.float32)
    g = (rng.standard_normal(300) * 10.0 ** rng.integers(-8, 4, 300)).astype(np.float32)
    buf[:3] = [0.0, -0.0, 1.0]
    g[:3] = [0.0, 0.0, -0.95]
    for mu in (0.95, 0.9, 0.5):
        got = o.momentum_update(buf, g, mu)
        assert got.dtype == np.float32
        mu32 = Fraction(float(np.float32(mu)))
        for i in range(buf.size):
            p = exact_f32_round(mu32 * Fraction(float(buf[i])))
            want = exact_f32_round(Fraction(float(p)) + Fraction(float(g[i])))
            assert got[i].tobytes() == want.tobytes() or (got[i] == 0 and want == 0), (i, got[i], want)


def pin_nesterov_post_update(o) -> None:
    """Nesterov input uses the updated buffer: with mu = 0.5 and buf = -2 g
    the updated buffer is exactly 0, so the input is g itself (it would be 0
    with the pre-update buffer, and 2g - ... with no Nesterov)."""
    rng = np.random.default_rng(16)
    g = (rng.standard_normal((8, 12))).astype(np.float32)
    buf = (-2.0 * g).astype(np.float32)
    buf_new, X, _ = o.muon_step(np.zeros((8, 12), np.float32), g, buf, lr=0.1,
                                momentum=0.5, nesterov=True, weight_decay=0.0, ns_steps=3)
    assert np.all(buf_new == 0.0)
    U, sig, V = jacobi_svd(g.astype(np.float64))
    nrm = math.sqrt(float(np.sum(g.astype(np.float64) ** 2)))
    want = (U * np.array([cubic_map(s / (nrm + EPS), 3) for s in sig])) @ V.T
    assert _rel(X, want) <= 1e-12


def _hadamard(n: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order n (a power of two)."""
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def pin_update_closed_form(o, seed: int = 17) -> None:
    """With g = c Q where Q has orthonormal rows made of +-1/4 entries (rows of
    a 16x16 Hadamard matrix over 4, exact in float32), a zero buffer and
    Nesterov, the input is (1 + mu) g, so X = f^k(sigma0) Q with
    sigma0 = ||M|| / sqrt(m) / (||M|| + 1e-7), and W' = W (1 - lr wd) - lr X,
    for wide, square and tall (transposed) matrices."""
    rng = np.random.default_rng(seed)
    H = _hadamard(16) / 4.0
    for (m, tall) in ((8, False), (8, True), (16, False)):
        Q = H[:m].copy()
        c = 2.0 ** -9
        g = (c * Q).astype(np.float32)
        if tall:
            g, Q = g.T.copy(), Q.T.copy()
        W = (rng.standard_normal(g.shape) * 0.02).astype(np.float32)
        lr, mu, wd, k = 0.02, 0.95, 0.01, 5
        buf_new, X, Wn = o.muon_step(W, g, np.zeros_like(g), lr=lr, momentum=mu,
                                     nesterov=True, weight_decay=wd, ns_steps=k)
        assert np.array_equal(buf_new, g)
        mu64 = float(np.float32(mu))
        alpha = c + mu64 * c                  # every |M_ij| / |Q_ij| (one fp64 rounding)
        nrm = alpha * math.sqrt(m)            # ||M||_F: m orthonormal rows scaled by alpha
        sig0 = alpha / (nrm + EPS)
        Xw = cubic_map(sig0, k) * Q
        assert _rel(X, Xw) <= 1e-13, _rel(X, Xw)
        lr64, wd64 = float(np.float32(lr)), float(np.float32(wd))
        Ww = W.astype(np.float64) * (1.0 - lr64 * wd64) - lr64 * Xw
        assert np.max(np.abs(Wn - Ww)) <= 1e-15


def pin_custom_coefficients(o, seed: int = 18) -> None:
    """Custom cubic coefficients (a, b): a 1x1 input follows s <- a s + b s^3
    and the spectral map holds with f(s) = a s + b s^3 (float32 a, b)."""
    rng = np.random.default_rng(seed)
    for (a, b) in ((1.875, -0.875), (2.0, -1.0)):
        a32, b32 = float(np.float32(a)), float(np.float32(b))
        for x in (0.8, -3.0, 1e-6):
            s_ = x / (abs(x) + EPS)
            for _ in range(4):
                s_ = a32 * s_ + b32 * s_ ** 3
            got = o.newton_schulz(np.array([[x]]), 4, (a, b))[0, 0]
            assert abs(got - s_) <= 1e-14 * max(1.0, abs(s_)), (a, b, x, got, s_)
        G = rng.standard_normal((9, 21))
        U, sig, V = jacobi_svd(G)
        nrm = math.sqrt(float(np.sum(G * G)))
        fs = []
        for sv in sig:
            t = sv / (nrm + EPS)
            for _ in range(3):
                t = a32 * t + b32 * t ** 3
            fs.append(t)
        want = (U * np.array(fs)) @ V.T
        assert _rel(o.newton_schulz(G, 3, (a, b)), want) <= 1e-12
        assert _rel(o.newton_schulz(G.T, 3, (a, b)), want.T) <= 1e-12


def pin_lr_scale(o, seed: int = 19) -> None:
    """lr scaled by 0.2 sqrt(max(rows, cols)) in the whole update: with the
    Hadamard input of pin_update_closed_form, W' = W (1 - lr_s wd) - lr_s c_k Q
    where lr_s = fl32(lr * fl32(0.2 * 4)) for 16 columns."""
    rng = np.random.default_rng(seed)
    H = _hadamard(16) / 4.0
    Q = H[:8].copy()
    c = 2.0 ** -9
    g = (c * Q).astype(np.float32)
    W = (rng.standard_normal(g.shape) * 0.02).astype(np.float32)
    lr, mu, wd, k = 0.02, 0.95, 0.01, 5
    _, X, Wn = o.muon_step(W, g, np.zeros_like(g), lr=lr, momentum=mu, nesterov=True,
                           weight_decay=wd, ns_steps=k, lr_scale=True)
    alpha = c + float(np.float32(mu)) * c
    Xw = cubic_map(alpha / (alpha * math.sqrt(8.0) + EPS), k) * Q
    assert _rel(X, Xw) <= 1e-13
    lr_s = float(np.float32(np.float32(lr) * np.float32(0.2 * 4.0)))
    Ww = W.astype(np.float64) * (1.0 - lr_s * float(np.float32(wd))) - lr_s * Xw
    assert np.max(np.abs(Wn - Ww)) <= 1e-15
    assert abs(o.lr_scale_factor(14336, 4096) - 0.2 * math.sqrt(14336.0)) < 1e-6


def pin_gradient_clipping(o) -> None:
    """Global-norm clipping before the momentum update: two matrices of +-1/4
    entries (Hadamard rows) have ||g|| = sqrt(64/16 + 256/16) = sqrt(20) ...
    here chosen as 4 x 16 and 16 x 16 blocks, ||g||^2 = 4 + 16 = 20.  With
    max_norm = 1 the coefficient is fl32(1 / (sqrt(20) + 1e-6)), and the new
    buffer is fl32(fl32(mu buf) + fl32(g c)), checked with exact arithmetic
    (a nonzero buffer distinguishes clipping before from after momentum)."""
    H = _hadamard(16) / 4.0
    g1 = H[:4].astype(np.float32)
    g2 = H.astype(np.float32)
    c32, norm = o.clip_coefficient([g1, g2], 1.0)
    assert abs(norm - math.sqrt(20.0)) <= 1e-15
    want_c = exact_f32_round(Fraction(1) / (Fraction(math.sqrt(20.0)) + Fraction(1e-6)))
    assert c32 == want_c
    assert o.clip_coefficient([g1], 100.0)[0] == np.float32(1.0)       # no clipping below the bound
    buf = (np.arange(64, dtype=np.float32).reshape(4, 16) - 31.0) * np.float32(0.01)
    mu = 0.9
    buf_new, _, _ = o.muon_step(np.zeros_like(g1), g1, buf, lr=0.0, momentum=mu, nesterov=False,
                                weight_decay=0.0, ns_steps=0, grad_scale=c32)
    mu32 = Fraction(float(np.float32(mu)))
    for i in range(4):
        for j in range(16):
            gc = exact_f32_round(Fraction(float(g1[i, j])) * Fraction(float(c32)))
            p = exact_f32_round(mu32 * Fraction(float(buf[i, j])))
            want = exact_f32_round(Fraction(float(p)) + Fraction(float(gc)))
            assert buf_new[i, j] == want, (i, j)


def pin_adamw(o, seed: int = 20) -> None:
    """AdamW (decoupled decay, bias-corrected moments):
    * first step from zero moments moves each element by lr g / (|g| + eps)
      (the bias corrections cancel 1 - beta exactly), i.e. lr sign(g) far
      above eps and lr / 2 at |g| = eps;
    * a constant gradient keeps that step size at every later step;
    * a zero gradient leaves the moments at zero and only decays p;
    * the moments follow fl(fl(beta m) + fl((1 - beta) g)) exactly."""
    rng = np.random.default_rng(seed)
    lr, b1, b2, wd = 1e-3, 0.9, 0.999, 0.0
    eps = 1e-8
    g = np.array([3.0, -0.25, 1e-8, -1e-8, 7e-3], dtype=np.float32)
    p0 = rng.standard_normal(5).astype(np.float32)
    m = np.zeros(5, np.float32)
    v = np.zeros(5, np.float32)
    p = p0.astype(np.float64)
    for t in range(1, 4):
        m, v, p = o.adamw_step(p, g, m, v, lr=lr, beta1=b1, beta2=b2, eps=eps, weight_decay=wd, step=t)
        g64 = g.astype(np.float64)
        step_want = float(np.float32(lr)) * g64 / (np.abs(g64) + float(np.float32(eps)))
        moved = p0.astype(np.float64) - p
        assert np.allclose(moved, t * step_want, rtol=2e-6, atol=0), (t, moved, t * step_want)
    # zero gradient: moments stay zero, p decays only
    w = rng.standard_normal(6).astype(np.float32)
    m1, v1, p1 = o.adamw_step(w, np.zeros(6, np.float32), np.zeros(6, np.float32),
                              np.zeros(6, np.float32), lr=0.1, beta1=b1, beta2=b2, eps=eps,
                              weight_decay=0.05, step=4)
    assert not m1.any() and not v1.any()
    assert np.array_equal(p1, w.astype(np.float64) * (1.0 - float(np.float32(0.1)) * float(np.float32(0.05))))
    # exact moment rounding
    gm = (rng.standard_normal(40) * 10.0 ** rng.integers(-6, 2, 40)).astype(np.float32)
    mm = (rng.standard_normal(40) * 1e-3).astype(np.float32)
    vv = (rng.random(40) * 1e-5).astype(np.float32)
    m2, v2, _ = o.adamw_step(np.zeros(40), gm, mm, vv, lr=lr, beta1=b1, beta2=b2, eps=eps,
                             weight_decay=0.0, step=2)
    B1, B2 = Fraction(float(np.float32(b1))), Fraction(float(np.float32(b2)))
    C1 = exact_f32_round(Fraction(1) - B1)
    C2 = exact_f32_round(Fraction(1) - B2)
    for i in range(40):
        G = Fraction(float(gm[i]))
        want_m = exact_f32_round(Fraction(float(exact_f32_round(B1 * Fraction(float(mm[i]))))) +
                                 Fraction(float(exact_f32_round(Fraction(float(C1)) * G))))
        cg = exact_f32_round(Fraction(float(C2)) * G)
        want_v = exact_f32_round(Fraction(float(exact_f32_round(B2 * Fraction(float(vv[i]))))) +
                                 Fraction(float(exact_f32_round(Fraction(float(cg)) * G))))
        assert m2[i] == want_m and v2[i] == want_v, i


def pin_rank_mean(o) -> None:
    """Mean of the ranks' gradients for the owner's fused reduction:
    * one rank: the gradient itself, bit for bit;
    * exactly summable values: the exact mean;
    * the float32 sum runs in rank order: 1 + 2^-24 + 2^-24 rounds to 1 each
      time (ties to even), while any other order or a wider sum keeps 2^-23;
    * the division is one correctly rounded float32 division, checked
      against exact rational rounding of S / 3 for S = 1 .. 200."""
    g = np.array([0.1, -3.0, 7e-9], dtype=np.float32)
    assert np.array_equal(o.rank_mean([g]).view(np.uint32), g.view(np.uint32))
    ranks = [np.array([v], dtype=np.float32) for v in (1.0, 2.0, 3.0, 6.0)]
    assert o.rank_mean(ranks)[0] == np.float32(3.0)
    t = np.float32(2.0 ** -24)
    got = o.rank_mean([np.array([1.0], np.float32), np.array([t]), np.array([t])])[0]
    assert got == exact_f32_round(Fraction(1, 3)), got
    S = np.arange(1, 201, dtype=np.float32)
    got = o.rank_mean([S, np.zeros_like(S), np.zeros_like(S)])
    for k in range(S.size):
        assert got[k] == exact_f32_round(Fraction(int(S[k]), 3)), (k, got[k])


def pin_relative_frobenius(o) -> None:
    """||a - b||_F / ||b||_F against values worked out by hand:
    * b = [[3, 4]] (norm 5), a = b + 0.5 e_11: 0.5 / 5 = 0.1 (the
      denominator is b's norm, not a's, which is sqrt(28.25));
    * b = [[1, 2], [2, 4]] (norm 5), a - b = diag(0.3, 0.4): the difference
      norm adds every element, sqrt(0.09 + 0.16) = 0.5, so again 0.1 (the
      largest element alone would give 0.08);
    * both zero gives 0, a nonzero a against a zero b gives inf, a == b gives 0;
    * scaling both arguments by the same c > 0 leaves the value unchanged."""
    b = np.array([[3.0, 4.0]])
    a = b + np.array([[0.5, 0.0]])
    assert abs(o.relative_frobenius(a, b) - 0.1) <= 1e-16, o.relative_frobenius(a, b)
    b2 = np.array([[1.0, 2.0], [2.0, 4.0]])
    a2 = b2 + np.diag([0.3, 0.4])
    assert abs(o.relative_frobenius(a2, b2) - 0.1) <= 1e-15, o.relative_frobenius(a2, b2)
    assert abs(o.relative_frobenius(7.0 * a2, 7.0 * b2) - 0.1) <= 1e-15
    assert o.relative_frobenius(np.zeros((2, 3)), np.zeros((2, 3))) == 0.0
    assert o.relative_frobenius(np.ones((2, 3)), np.zeros((2, 3))) == float("inf")
    assert o.relative_frobenius(b2, b2) == 0.0


def pin_orthogonality_error(o, seed: int = 21) -> None:
    """||X X^T - I||_F on the short side of X, against closed forms:
    * hand-worked: [[1, 1]] gives |2 - 1| = 1; diag(2, 1) gives 3;
      [[1, 1], [0, 1]] gives ||[[1, 1], [1, 0]]||_F = sqrt(3);
    * c Q with orthonormal rows (m x n, m < n) and its transpose (tall) both
      give sqrt(m) |c^2 - 1|: the tall one must use the m x m column Gram, the
      n x n row Gram would add n - m to the squared value;
    * a tall 96 x 40 random matrix gives sqrt(sum_i (sigma_i^2 - 1)^2) over
      its 40 singular values from the hand-written Jacobi SVD."""
    assert abs(o.orthogonality_error(np.array([[1.0, 1.0]])) - 1.0) <= 1e-15
    assert abs(o.orthogonality_error(np.diag([2.0, 1.0])) - 3.0) <= 1e-15
    assert abs(o.orthogonality_error(np.array([[1.0, 1.0], [0.0, 1.0]])) - math.sqrt(3.0)) <= 1e-15
    rng = np.random.default_rng(seed)
    for (m, n) in ((16, 40), (5, 64)):
        Q = _semi_orthogonal(rng, m, n)
        for c in (0.5, 1.0, 1.7):
            want = math.sqrt(m) * abs(c * c - 1.0)
            assert abs(o.orthogonality_error(c * Q) - want) <= 1e-12, (m, n, c)
            assert abs(o.orthogonality_error((c * Q).T) - want) <= 1e-12, (m, n, c, "tall")
    G = rng.standard_normal((96, 40))
    _, sig, _ = jacobi_svd(G)
    want = math.sqrt(float(np.sum((sig * sig - 1.0) ** 2)))
    got = o.orthogonality_error(G)
    assert abs(got - want) <= 1e-10 * want, (got, want)


def pin_round_to_bf16(o, seed: int = 22) -> None:
    """float32 -> bfloat16 rounding against exact rational rounding to 8
    significant bits: random values over many binades, the exact halfway
    points between neighbours (ties to even, both parities), values that are
    already bfloat16, signs, and overflow past the largest bfloat16."""
    rng = np.random.default_rng(seed)
    vals = (rng.standard_normal(400) * 10.0 ** rng.integers(-30, 30, 400)).astype(np.float32)
    ties = []
    for k in range(128, 140):
        for e in (-3, 0, 5):
            ties.append(np.float32((k + 0.5) * 2.0 ** (e - 7)))     # halfway, both parities of k
            ties.append(np.float32(k * 2.0 ** (e - 7)))             # already bfloat16
    vals = np.concatenate([vals, np.array(ties, np.float32), -np.array(ties, np.float32)])
    got = o.round_to_bf16(vals)
    for v, r in zip(vals, got):
        want = exact_bf16_round(Fraction(float(v)))
        assert float(r) == want, (float(v), float(r), want)
    big = o.round_to_bf16(np.array([3.4e38, -3.4e38, 3.38e38], np.float32))
    assert big[0] == np.inf and big[1] == -np.inf and np.isfinite(big[2])
    assert np.isnan(o.round_to_bf16(np.array([np.nan], np.float32))[0])


def pin_clip_buckets(o) -> None:
    """Per-segment clipping: three segments of +-1/4 Hadamard rows with
    exactly known norms, sqrt(4) = 2, sqrt(16) = 4 and sqrt(1) = 1, and
    max_norm 1.5 for each.  Segment 0 is scaled by
    c0 = fl32(1.5 / (2 + 1e-6)), segment 1 by c1 = fl32(1.5 / (4 + 1e-6)),
    segment 2 is below its bound and stays bit for bit (c2 = 1).  One global
    norm (sqrt(21)) would give every segment the same coefficient.  Every
    element must equal the exact product g * c rounded once to float32 and,
    for bfloat16 storage, once more to bfloat16."""
    H = _hadamard(16) / 4.0
    seg0 = [(H[:4].astype(np.float32), True)]                      # norm 2 (bf16)
    seg1 = [(H[:10].astype(np.float32), False), (H[10:].astype(np.float32), True)]   # norm 4
    seg2 = [(H[:1].astype(np.float32), True)]                      # norm 1: no clipping
    out, norms, coefs = o.clip_grad_norm_buckets([seg0, seg1, seg2], [1.5, 1.5, 1.5])
    assert [abs(n - w) <= 1e-15 for n, w in zip(norms, (2.0, 4.0, 1.0))] == [True] * 3, norms
    for c, nrm in zip(coefs[:2], (2.0, 4.0)):
        assert c == exact_f32_round(Fraction(1.5) / (Fraction(nrm) + Fraction(1e-6))), (c, nrm)
    assert coefs[2] == np.float32(1.0)
    for seg, new, c in zip((seg0, seg1, seg2), out, coefs):
        for (v, is_bf16), y in zip(seg, new):
            assert y.dtype == np.float32 and y.shape == v.shape
            for a, b in zip(v.ravel(), y.ravel()):
                prod = exact_f32_round(Fraction(float(a)) * Fraction(float(c)))
                want = exact_bf16_round(Fraction(float(prod))) if is_bf16 else float(prod)
                assert float(b) == want, (float(a), float(c), float(b), want)
    # random values: bfloat16 ones built from integer significands, float32
    # ones from a generator; the norm comes from the exact sum of squares and
    # an integer square root with 100 fractional bits
    rng = np.random.default_rng(23)
    vb = (rng.integers(128, 256, (8, 8)) * 2.0 ** rng.integers(-12, -6, (8, 8))
          * rng.choice([-1.0, 1.0], (8, 8))).astype(np.float32)
    vf = (rng.standard_normal((5, 3)) * 0.01).astype(np.float32)
    S = sum(Fraction(float(x)) ** 2 for x in np.concatenate([vb.ravel(), vf.ravel()]))
    root = Fraction(math.isqrt(int(S * 2 ** 200)), 2 ** 100)
    mx = 0.3 * float(root)
    out3, norms3, coefs3 = o.clip_grad_norm_buckets([[(vb, True), (vf, False)]], [mx])
    assert abs(norms3[0] - float(root)) <= 1e-15 * float(root)
    c = coefs3[0]
    assert c == exact_f32_round(Fraction(float(np.float32(mx))) / (root + Fraction(1e-6))), c
    for (v, is_bf16), y in zip(((vb, True), (vf, False)), out3[0]):
        for a, b in zip(v.ravel(), y.ravel()):
            prod = exact_f32_round(Fraction(float(a)) * Fraction(float(c)))
            want = exact_bf16_round(Fraction(float(prod))) if is_bf16 else float(prod)
            assert float(b) == want, (float(a), float(c), float(b), want)
    # a NaN norm leaves its segment unchanged; an empty segment has norm 0
    nan_seg = [(np.array([1.0, np.nan], np.float32), False)]
    out2, norms2, coefs2 = o.clip_grad_norm_buckets([nan_seg, []], [1.0, 1.0])
    assert np.isnan(norms2[0]) and coefs2[0] == np.float32(1.0) and out2[0][0][0] == 1.0
    assert norms2[1] == 0.0 and coefs2[1] == np.float32(1.0) and out2[1] == []


def pin_quintic_coefficients(o, seed: int = 24) -> None:
    """Quintic custom coefficients (a, b, c): X <- a X + b A X + c A^2 X,
    A = X X^T, acts on each singular value as f(s) = a s + b s^3 + c s^5
    (float32 a, b, c):
    * a 1x1 input follows that scalar recurrence;
    * random wide and tall inputs match U diag(f^k(sigma / (||G|| + 1e-7))) V^T
      from the hand-written Jacobi SVD;
    * the textbook quintic Newton-Schulz polynomial (15 s - 10 s^3 + 3 s^5) / 8
      has f(1) = 1, so orthonormal rows are a fixed point of its inner step;
    * c = 0 gives the cubic step with the same (a, b)."""
    rng = np.random.default_rng(seed)
    for coeffs in ((3.4445, -4.7750, 2.0315), (15.0 / 8.0, -10.0 / 8.0, 3.0 / 8.0)):
        a, b, c = (float(np.float32(x)) for x in coeffs)
        f = lambda t: a * t + b * t ** 3 + c * t ** 5
        for x in (0.8, -3.0, 1e-6):
            t = x / (abs(x) + EPS)
            for _ in range(4):
                t = f(t)
            got = o.newton_schulz(np.array([[x]]), 4, coeffs)[0, 0]
            assert abs(got - t) <= 1e-13 * max(1.0, abs(t)), (coeffs, x, got, t)
        G = rng.standard_normal((9, 21))
        U, sig, V = jacobi_svd(G)
        nrm = math.sqrt(float(np.sum(G * G)))
        fs = []
        for sv in sig:
            t = sv / (nrm + EPS)
            for _ in range(3):
                t = f(t)
            fs.append(t)
        want = (U * np.array(fs)) @ V.T
        assert _rel(o.newton_schulz(G, 3, coeffs), want) <= 1e-12
        assert _rel(o.newton_schulz(G.T, 3, coeffs), want.T) <= 1e-12
    Q = _semi_orthogonal(rng, 12, 30)
    assert _rel(o.ns_iteration(Q, 15.0 / 8.0, -10.0 / 8.0, 3.0 / 8.0), Q) <= 1e-14
    G = rng.standard_normal((7, 16))
    assert _rel(o.newton_schulz(G, 4, (1.875, -0.875, 0.0)), o.newton_schulz(G, 4, (1.875, -0.875))) <= 1e-15


def pin_ns_flops(o) -> None:
    """Useful Newton-Schulz FLOPs as the metric counts them: per step m^2 n for
    the symmetric product X X^T (half of the dense 2 m^2 n) and 2 m^2 n for
    (X X^T) X, with m the short side and n the long one; the quintic form adds
    m^3 for the symmetric square A A (half of the dense 2 m^3).  Hand-counted:
    * 2 x 3, one step: 4 * 3 + 2 * 4 * 3 = 36; its transpose 3 x 2 too;
    * five steps: 180; quintic, one step: 36 + 2^3 = 44;
    * 1024 x 4096, one step: 3 * 2^20 * 2^12 = 12 884 901 888;
    * 4096 x 4096, five steps: 15 * 2^36 = 1 030 792 151 040."""
    assert o.ns_flops(2, 3, 1) == 36.0, o.ns_flops(2, 3, 1)
    assert o.ns_flops(3, 2, 1) == 36.0, o.ns_flops(3, 2, 1)
    assert o.ns_flops(2, 3, 5) == 180.0
    assert o.ns_flops(2, 3, 1, quintic=True) == 44.0, o.ns_flops(2, 3, 1, quintic=True)
    assert o.ns_flops(1024, 4096, 1) == 12884901888.0
    assert o.ns_flops(4096, 4096, 5) == 1030792151040.0


ALL_PINS = (pin_scalar_closed_form, pin_spectral_map, pin_orthogonal_input,
            pin_monotone_error, pin_symmetries, pin_momentum_bitwise,
            pin_nesterov_post_update, pin_update_closed_form, pin_custom_coefficients,
            pin_lr_scale, pin_gradient_clipping, pin_adamw, pin_rank_mean,
            pin_relative_frobenius, pin_orthogonality_error, pin_round_to_bf16,
            pin_clip_buckets, pin_quintic_coefficients, pin_ns_flops)
