"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each ``pin_*`` takes an oracle ``fwd(form, q, k, v, log_w, e1, e2, S0)`` that
returns ``(o [B,T,H,dv], S_T [B,H,dk,dv])`` and raises AssertionError when the
oracle disagrees with an independent statement of the same result.  None of them
re-types the oracle's loop: each uses another formulation from the pages (closed
form, a special case that reduces to a textbook rule, a spectrum, the chunkwise
algebra) or a printed value.  ``test_oracle_pins.py`` runs them on the real
oracle; ``test_oracle_mutants.py`` runs them on copies of the oracle with planted
mistakes and checks each mutant fails at least one of them.

All pins use d_k == d_v (the mutants include a transposed-index mistake).
State orientation: the oracle returns the storage layout [.., d_k, d_v]; the
column form of the pages' chapter 13 is its transpose.
"""
from __future__ import annotations

import json
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


# ---------------------------------------------------------------------------
# 1. GLA (u = 0): brute-force O(T^2) unrolling with decays as direct products.
#    "Muir ...", section 2.1 (channel-wise decayed linear attention) and the
#    unrolled form behind section 2.2's S_C and O.
# ---------------------------------------------------------------------------
def pin_gla_unrolled(fwd, seed=0):
    rng = np.random.default_rng(seed)
    B, T, H, d = 2, 11, 2, 5
    q, k, v = (rng.standard_normal((B, T, H, d)) for _ in range(3))
    log_w = -np.exp(rng.normal(-1.0, 0.5, (B, T, H, d)))
    S0 = rng.standard_normal((B, H, d, d))
    o, S_T = fwd("gla", q, k, v, log_w, None, None, S0)
    w = np.exp(log_w)
    err = 0.0
    for b in range(B):
        for h in range(H):
            Sc0 = S0[b, h].T                       # column form, d_v x d_k
            for t in range(T):
                pi_t = np.prod(w[b, : t + 1, h], axis=0)
                ref = Sc0 @ (pi_t * q[b, t, h])
                for s in range(t + 1):
                    pi_ts = np.prod(w[b, s + 1: t + 1, h], axis=0)   # empty product = 1
                    ref = ref + v[b, s, h] * np.dot(k[b, s, h] * pi_ts, q[b, t, h])
                err = max(err, _rel(o[b, t, h], ref))
            ST = Sc0 * np.prod(w[b, :, h], axis=0)[None, :]
            for s in range(T):
                pi_Ts = np.prod(w[b, s + 1:, h], axis=0)
                ST = ST + np.outer(v[b, s, h], k[b, s, h] * pi_Ts)
            err = max(err, _rel(S_T[b, h].T, ST))
    assert err < 1e-12, f"GLA unrolled mismatch {err:.3e}"
    return err


# ---------------------------------------------------------------------------
# 2. Delta rule (w = 1, u = beta k, z = k, written value beta v): the LMS step
#    S <- S - beta (S k - v) k^T, one step of gradient descent on the key-value
#    reconstruction loss ("Muir ...", section 2.1; "Exponential gates ...",
#    solution to Exercise 13.5, plain DeltaNet).
# ---------------------------------------------------------------------------
def pin_delta_rule_lms(fwd, seed=1):
    rng = np.random.default_rng(seed)
    B, T, H, d = 1, 17, 2, 6
    q, v = (rng.standard_normal((B, T, H, d)) for _ in range(2))
    k = _unit(rng.standard_normal((B, T, H, d)))
    beta = rng.uniform(0.1, 1.2, (B, T, H, 1))
    S0 = rng.standard_normal((B, H, d, d))
    o, S_T = fwd("general", q, k, beta * v, np.zeros((B, T, H, d)), beta * k, k, S0)
    err = 0.0
    for b in range(B):
        for h in range(H):
            S = S0[b, h].T.copy()
            for t in range(T):
                kk, bt = k[b, t, h], beta[b, t, h, 0]
                S = S - bt * np.outer(S @ kk - v[b, t, h], kk)
                err = max(err, _rel(o[b, t, h], S @ q[b, t, h]))
            err = max(err, _rel(S_T[b, h].T, S))
    assert err < 1e-12, f"delta-rule (LMS) mismatch {err:.3e}"
    return err


# ---------------------------------------------------------------------------
# 3. Proposition 13.2: the generalized rule with w = gamma 1, a = k/|k|,
#    c = gamma beta |k|^2 and write beta v k^T equals gated DeltaNet
#    S <- gamma S (I - beta k k^T) + beta v k^T ("Exponential gates ...", 13.3).
# ---------------------------------------------------------------------------
def pin_prop_13_2(fwd, seed=2):
    rng = np.random.default_rng(seed)
    B, T, H, d = 1, 15, 1, 7
    q, v, k = (rng.standard_normal((B, T, H, d)) for _ in range(3))
    gamma = rng.uniform(0.6, 0.99, (B, T, H))
    beta = rng.uniform(0.1, 1.5, (B, T, H))
    kn2 = np.sum(k * k, axis=-1)
    a = k / np.sqrt(kn2)[..., None]
    c = gamma * beta * kn2
    log_w = np.repeat(np.log(gamma)[..., None], d, axis=-1)
    o, S_T = fwd("rwkv7", q, k, beta[..., None] * v, log_w, a, c, None)
    S = np.zeros((d, d))
    err = 0.0
    for t in range(T):
        kk = k[0, t, 0]
        S = gamma[0, t, 0] * S @ (np.eye(d) - beta[0, t, 0] * np.outer(kk, kk)) \
            + beta[0, t, 0] * np.outer(v[0, t, 0], kk)
        err = max(err, _rel(o[0, t, 0], S @ q[0, t, 0]))
    err = max(err, _rel(S_T[0, 0].T, S))
    assert err < 1e-12, f"Prop 13.2 reduction mismatch {err:.3e}"
    return err


# ---------------------------------------------------------------------------
# 4. Proposition 13.1: spectrum of the transition the oracle applies.  One RWKV-7
#    step from S0 = I with a zero write returns I A = A.  Scalar diagonal w0:
#    spectrum {w0 - c} and w0 (multiplicity d - 1).  General diagonal: roots of
#    the secular equation f(l) = 1 - c sum a_i^2 / (w_i - l), interlacing, and
#    spectrum inside [min w - c, max w].  Exercise 13.1 values from the golden file.
# ---------------------------------------------------------------------------
def _transition(fwd, w, a, c):
    d = w.size
    z = np.zeros((1, 1, 1, d))
    S0 = np.eye(d)[None, None]
    _, S_T = fwd("rwkv7", z + 1.0, z, z, np.log(w)[None, None, None], a[None, None, None],
                 np.array([[[c]]]), S0)
    return S_T[0, 0].T        # column form: S_1 = I A


def pin_prop_13_1(fwd, seed=3):
    rng = np.random.default_rng(seed)
    d = 8
    err = 0.0
    with open(os.path.join(GOLDEN, "spectrum_ch13.json")) as f:
        gold = json.load(f)
    # scalar diagonal, including the exercise's cases at w0 = 1
    cases = [(gold["w0"], cs["c"], cs["rho"]) for cs in gold["cases"]] + [(0.7, 0.4, None),
                                                                          (0.9, 1.7, None)]
    for w0, c, rho_gold in cases:
        a = _unit(rng.standard_normal(d))
        A = _transition(fwd, np.full(d, w0), a, c)
        assert np.allclose(A, A.T, atol=1e-14), "transition not symmetric"
        lam = np.linalg.eigvalsh(A)
        closed = np.sort(np.array([w0 - c] + [w0] * (d - 1)))
        err = max(err, float(np.max(np.abs(lam - closed))))
        rho = float(np.max(np.abs(lam)))
        assert abs(rho - max(abs(w0), abs(w0 - c))) < 1e-12
        if rho_gold is not None:
            assert abs(rho - rho_gold) < 1e-12, f"rho {rho} vs printed {rho_gold}"
    assert err < 1e-13, f"scalar-diagonal spectrum mismatch {err:.3e}"
    # general diagonal: secular equation, interlacing, bounds
    for _ in range(3):
        w = np.sort(rng.uniform(0.2, 1.0, d))
        a = _unit(rng.standard_normal(d))
        c = float(rng.uniform(0.1, 2.0))
        lam = np.sort(np.linalg.eigvalsh(_transition(fwd, w, a, c)))
        f = 1.0 - c * np.sum(a[None, :] ** 2 / (w[None, :] - lam[:, None]), axis=1)
        scale = c * np.sum(a[None, :] ** 2 / np.abs(w[None, :] - lam[:, None]), axis=1)
        res = float(np.max(np.abs(f) / np.maximum(scale, 1.0)))
        assert res < 1e-9, f"secular residual {res:.3e}"
        assert lam[0] >= w.min() - c - 1e-12 and lam[-1] <= w.max() + 1e-12
        for i in range(d - 1):           # one root per gap, at or below its w
            assert w[i] - 1e-12 <= lam[i + 1] <= w[i + 1] + 1e-12
        err = max(err, res)
    return err


# ---------------------------------------------------------------------------
# 5. Decoupled eviction ("Exponential gates ...", section 13.3): targeted removal
#    gives |S_T k_A| = (1 - c)^T |v_A|; removal locked to orthogonal write keys
#    leaves |v_A|.  Printed values in the golden file (c = 0.1, T = 30).
# ---------------------------------------------------------------------------
def pin_eviction(fwd, seed=4):
    with open(os.path.join(GOLDEN, "eviction_ch13_3.json")) as f:
        gold = json.load(f)
    c, T = gold["c"], gold["T"]
    rng = np.random.default_rng(seed)
    d = 8
    kA = _unit(rng.standard_normal(d))
    vA = rng.standard_normal(d)
    P = np.eye(d) - np.outer(kA, kA)
    ratios = []
    for targeted in (True, False):
        n = T + 1
        q = np.ones((1, n, 1, d))
        k = np.zeros((1, n, 1, d))
        v = np.zeros((1, n, 1, d))
        a = np.zeros((1, n, 1, d))
        cc = np.zeros((1, n, 1))
        k[0, 0, 0], v[0, 0, 0], a[0, 0, 0] = kA, vA, kA       # store (k_A, v_A), no removal
        for t in range(1, n):
            b = _unit(P @ rng.standard_normal(d))             # write key orthogonal to k_A
            k[0, t, 0], v[0, t, 0] = b, rng.standard_normal(d)
            a[0, t, 0] = kA if targeted else b
            cc[0, t, 0] = c
        _, S_T = fwd("rwkv7", q, k, v, np.zeros((1, n, 1, d)), a, cc, None)
        ratios.append(np.linalg.norm(S_T[0, 0].T @ kA) / np.linalg.norm(vA))
    printed = gold["printed_targeted_norm"] / gold["printed_locked_norm"]
    assert abs(ratios[0] - (1 - c) ** T) < 1e-13, f"targeted ratio {ratios[0]!r}"
    assert abs(ratios[0] - printed) < 1e-6, f"targeted ratio vs printed {printed!r}"
    assert abs(ratios[1] - 1.0) < 1e-13, f"locked ratio {ratios[1]!r}"
    return abs(ratios[0] - (1 - c) ** T)


# ---------------------------------------------------------------------------
# 6. Boundedness: with every transition contractive (c < 1 + min w, so by
#    Prop. 13.1 rho(A_t) <= max(max w, |min w - c|) < 1), the triangle inequality
#    gives |S_t| <= prod rho |S_0| + sum_s prod_{r>s} rho |v_s||k_s|.
# ---------------------------------------------------------------------------
def pin_bounded(fwd, seed=5):
    rng = np.random.default_rng(seed)
    d, T = 6, 120
    S = rng.standard_normal((1, 1, d, d))
    bound = np.linalg.norm(S)
    worst = 0.0
    for t in range(T):
        w = rng.uniform(0.5, 0.95, d)
        c = float(rng.uniform(0.0, 1.0 + w.min() - 0.05))
        rho = max(w.max(), abs(w.min() - c))
        a = _unit(rng.standard_normal(d))
        k, v, q = rng.standard_normal(d), rng.standard_normal(d), rng.standard_normal(d)
        _, S = fwd("rwkv7", q[None, None, None], k[None, None, None], v[None, None, None],
                   np.log(w)[None, None, None], a[None, None, None], np.array([[[c]]]), S)
        bound = rho * bound + np.linalg.norm(v) * np.linalg.norm(k)
        worst = max(worst, np.linalg.norm(S) / bound)
    assert worst <= 1.0 + 1e-12, f"state norm exceeds the contraction bound ({worst:.4f})"
    return worst


# ---------------------------------------------------------------------------
# 7. GDN-2 eq. (1) in the page's own row form: S <- (I - k^T (b.k)) Diag(alpha) S
#    + k^T (w.v), o = q S ("Muir ...", section 2.1; eq. (8) with q_hat).
# ---------------------------------------------------------------------------
def pin_gdn2_row_form(fwd, seed=6):
    rng = np.random.default_rng(seed)
    B, T, H, d = 1, 13, 2, 6
    q, v = (rng.standard_normal((B, T, H, d)) for _ in range(2))
    k = _unit(rng.standard_normal((B, T, H, d)))
    alpha = rng.uniform(0.5, 0.999, (B, T, H, d))
    bg = rng.uniform(0.0, 2.0, (B, T, H, d))
    wg = rng.uniform(0.0, 1.0, (B, T, H, d))
    S0 = rng.standard_normal((B, H, d, d))
    o, S_T = fwd("gdn2", q, k, v, np.log(alpha), bg, wg, S0)
    err = 0.0
    for h in range(H):
        S = S0[0, h].copy()                         # row form: d_k x d_v
        for t in range(T):
            kk = k[0, t, h]
            S = (np.eye(d) - np.outer(kk, bg[0, t, h] * kk)) @ np.diag(alpha[0, t, h]) @ S \
                + np.outer(kk, wg[0, t, h] * v[0, t, h])
            err = max(err, _rel(o[0, t, h], q[0, t, h] @ S))
        err = max(err, _rel(S_T[0, h], S))
    assert err < 1e-12, f"GDN-2 row-form mismatch {err:.3e}"
    return err


# ---------------------------------------------------------------------------
# 8. GDN-2 chunkwise algebra ("Muir ...", section 2.2 and section 4.2 eqs.
#    (10)-(12)), fp64, in the page's row orientation: cumulative log-decay,
#    L_strict, T = I + L_strict, [U Y] = T^-1 [V^ K^_pi], V~ = U - Y S0,
#    S_C = Diag(pi_C) S0 + K~^T V~, O = Q_pi S0 + M V~; the affine form (10);
#    the Neumann-product leaf inverse (12) and the 2x2 block inverse (11).
# ---------------------------------------------------------------------------
def gdn2_chunked_reference(q, k, v, log_w, bg, wg, S0, C):
    """Chunkwise evaluation of GDN-2 for one (b, h): inputs [T, d], S0 [dk, dv]."""
    T, dk = k.shape
    S = S0.copy()
    O = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        sl = slice(c0, min(c0 + C, T))
        n = sl.stop - sl.start
        Lam = np.cumsum(log_w[sl], axis=0)                       # Lambda_t <= 0
        pi = np.exp(Lam)
        rel = np.exp(Lam[:, None, :] - Lam[None, :, :])          # pi_{t,s}, used for t >= s
        kh = bg[sl] * k[sl]
        vh = wg[sl] * v[sl]
        L = np.tril(np.einsum("tj,tsj,sj->ts", kh, rel, k[sl]), -1)
        M = np.tril(np.einsum("tj,tsj,sj->ts", q[sl], rel, k[sl]))
        Tm = np.eye(n) + L
        UY = np.linalg.solve(Tm, np.concatenate([vh, pi * kh], axis=1))
        U, Y = UY[:, : v.shape[1]], UY[:, v.shape[1]:]
        Vt = U - Y @ S
        Kt = np.exp(Lam[-1][None, :] - Lam) * k[sl]
        O_direct = (pi * q[sl]) @ S + M @ Vt
        S_direct = pi[-1][:, None] * S + Kt.T @ Vt
        O_affine = ((pi * q[sl]) - M @ Y) @ S + M @ U                      # eq. (10)
        S_affine = (np.diag(pi[-1]) - Kt.T @ Y) @ S + Kt.T @ U
        assert _rel(O_affine, O_direct) < 1e-12 and _rel(S_affine, S_direct) < 1e-12
        O[sl] = O_direct
        S = S_direct
    return O, S


def pin_gdn2_chunk_algebra(fwd, seed=7):
    rng = np.random.default_rng(seed)
    B, T, H, d = 1, 22, 2, 6          # 22 = 5 chunks of 4 and a ragged tail of 2
    q, v = (rng.standard_normal((B, T, H, d)) for _ in range(2))
    k = _unit(rng.standard_normal((B, T, H, d)))
    log_w = np.log(rng.uniform(0.3, 0.999, (B, T, H, d)))
    bg = rng.uniform(0.0, 2.0, (B, T, H, d))
    wg = rng.uniform(0.0, 1.0, (B, T, H, d))
    S0 = rng.standard_normal((B, H, d, d))
    o, S_T = fwd("gdn2", q, k, v, log_w, bg, wg, S0)
    err = 0.0
    for C in (4, 8, 22):
        for h in range(H):
            O, S = gdn2_chunked_reference(q[0, :, h], k[0, :, h], v[0, :, h], log_w[0, :, h],
                                          bg[0, :, h], wg[0, :, h], S0[0, h], C)
            err = max(err, _rel(o[0, :, h], O), _rel(S_T[0, h], S))
    assert err < 1e-11, f"GDN-2 chunkwise algebra mismatch {err:.3e}"
    return err


def check_block_inverses(seed=8):
    """Eq. (12) leaf Neumann product and eq. (11) block inverse equal inv(T)."""
    rng = np.random.default_rng(seed)
    n0 = 8
    L = np.tril(rng.standard_normal((n0, n0)) * 0.5, -1)
    T = np.eye(n0) + L
    prod = np.eye(n0)
    for j in range(int(np.log2(n0))):
        prod = prod @ (np.eye(n0) + np.linalg.matrix_power(-L, 2 ** j))
    e12 = _rel(prod, np.linalg.inv(T))
    C = 16
    L = np.tril(rng.standard_normal((C, C)) * 0.3, -1)
    T = np.eye(C) + L
    h = C // 2
    TLi, TRi = np.linalg.inv(T[:h, :h]), np.linalg.inv(T[h:, h:])
    X21 = -TRi @ T[h:, :h] @ TLi
    blk = np.block([[TLi, np.zeros((h, h))], [X21, TRi]])
    e11 = _rel(blk, np.linalg.inv(T))
    return e12, e11


# ---------------------------------------------------------------------------
# 9. General form (separate erase key z) in chunkwise form: the unrolled
#    e_t = S0(pi_{t-1}.u_t) + sum_{s<t}[v_s<k_s.pi_{t-1,s},u_t> - e_s<z_s.pi_{t-1,s},u_t>]
#    solved as a unit lower-triangular system, then O and S_C as sums of rank-one
#    terms (the section 2.2 derivation with two write streams).
# ---------------------------------------------------------------------------
def pin_general_chunk_algebra(fwd, seed=9):
    rng = np.random.default_rng(seed)
    B, T, H, d = 1, 19, 1, 5
    q, v, u, z, k = (rng.standard_normal((B, T, H, d)) for _ in range(5))
    u *= 0.3
    log_w = np.log(rng.uniform(0.3, 1.0, (B, T, H, d)))
    S0 = rng.standard_normal((B, H, d, d))
    o, S_T = fwd("general", q, k, v, log_w, u, z, S0)
    C = 7
    S = S0[0, 0].T.copy()                  # column form
    O = np.zeros((T, d))
    for c0 in range(0, T, C):
        idx = range(c0, min(c0 + C, T))
        n = len(idx)
        lw = log_w[0, c0:c0 + n, 0]
        Lam = np.concatenate([np.zeros((1, d)), np.cumsum(lw, axis=0)])   # Lam[t], t = 0..n
        Q, K, V, Uu, Z = (x[0, c0:c0 + n, 0] for x in (q, k, v, u, z))
        A = np.zeros((n, n))
        Bm = np.zeros((n, n))
        for t in range(n):
            for s in range(t):
                p = np.exp(Lam[t] - Lam[s + 1])          # pi_{t-1,s} over tokens s+1..t-1
                A[t, s] = np.dot(Uu[t] * p, Z[s])
                Bm[t, s] = np.dot(Uu[t] * p, K[s])
        P = np.stack([S @ (np.exp(Lam[t]) * Uu[t]) for t in range(n)])
        E = np.linalg.solve(np.eye(n) + A, P + Bm @ V)
        for t in range(n):
            ot = S @ (np.exp(Lam[t + 1]) * Q[t])
            for s in range(t + 1):
                p = np.exp(Lam[t + 1] - Lam[s + 1])
                ot = ot + V[s] * np.dot(K[s] * p, Q[t]) - E[s] * np.dot(Z[s] * p, Q[t])
            O[c0 + t] = ot
        Sn = S * np.exp(Lam[n])[None, :]
        for s in range(n):
            p = np.exp(Lam[n] - Lam[s + 1])
            Sn = Sn + np.outer(V[s], K[s] * p) - np.outer(E[s], Z[s] * p)
        S = Sn
    err = max(_rel(o[0, :, 0], O), _rel(S_T[0, 0].T, S))
    assert err < 1e-11, f"general chunkwise algebra mismatch {err:.3e}"
    return err


ALL_PINS = [pin_gla_unrolled, pin_delta_rule_lms, pin_prop_13_2, pin_prop_13_1, pin_eviction,
            pin_bounded, pin_gdn2_row_form, pin_gdn2_chunk_algebra, pin_general_chunk_algebra]
