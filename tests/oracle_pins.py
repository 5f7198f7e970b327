"""Pins that tie the fp64 oracle to what the pages and the mathematics fix.

Each ``pin_*`` function takes an oracle object (``forward``, ``decode_step``,
``backward``) and raises AssertionError when the oracle disagrees with an
independent statement of the result. None of them re-types the oracle's own
rank-1 update: each uses a different formula (a reduction to an older rule in
that rule's own form and orientation, a closed form, a dense product of
transition matrices, the optimality condition of the objective, finite
differences). The mutation test runs the same pins against deliberately broken
copies of the oracle.

Sources (page titles and sections):
  GDN2  "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
        (graygoo.forestry.md note): sec. 1 summary (gate ranges, reductions),
        sec. 2 theory (fast-weight objective, reductions to KDA and Gated
        DeltaNet), sec. 3 architecture (forward steps, asymmetric factor
        (I - k e^T), gate-aware backward).
  GDN2-HF  the Hugging Face daily-papers abstract of the same paper
        (reductions, asymmetric erase factor).
  VIS   blog.vllbc.top visual reading of Gated DeltaNet: the one-hot
        "memory simulation" and "alpha = 0 clears the memory".
  GDN   "Gated Delta Net" survey (hebangwen.github.io), sec. 1.1: the DeltaNet
        and Gated DeltaNet update equations with S in R^{dv x dk}.
"""
from __future__ import annotations

import numpy as np


def _rand_case(rng, B, T, H, dk, dv, beta_gates=False, decay="softplus", normalise=True):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if normalise:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    if decay == "softplus":
        la = -np.log1p(np.exp(rng.standard_normal((B, T, H, dk))))
    elif decay == "zero":
        la = np.zeros((B, T, H, dk))
    else:
        raise ValueError(decay)
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H, dk))))
    w = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H, dv))))
    return q, k, v, la, b, w


def _close(a, b, tol, what):
    err = np.max(np.abs(np.asarray(a) - np.asarray(b)))
    scale = max(1.0, float(np.max(np.abs(b))))
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} (scale {scale:.3e}, tol {tol:.1e})"


# ---------------------------------------------------------------------------
# P1  Reduction to KDA (GDN2 sec. 2 last paragraph; GDN2-HF abstract):
#     b_t = w_t = beta_t * 1  =>  S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
# ---------------------------------------------------------------------------
def pin_kda(orc, seed=1):
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 1, 12, 2, 5, 3
    q, k, v, la, _, _ = _rand_case(rng, B, T, H, dk, dv)
    beta = rng.random((B, T, H))
    b = np.repeat(beta[..., None], dk, axis=-1)
    w = np.repeat(beta[..., None], dv, axis=-1)
    S0 = rng.standard_normal((B, H, dk, dv)) * 0.3
    o, ST = orc.forward(q, k, v, la, b, w, S0=S0)
    for h in range(H):
        S = S0[0, h].copy()
        for t in range(T):
            kt, vt, bt = k[0, t, h], v[0, t, h], beta[0, t, h]
            S = (np.eye(dk) - bt * np.outer(kt, kt)) @ np.diag(np.exp(la[0, t, h])) @ S + bt * np.outer(kt, vt)
            _close(o[0, t, h], S.T @ q[0, t, h], 1e-12, f"KDA o[t={t},h={h}]")
        _close(ST[0, h], S, 1e-12, f"KDA S_T[h={h}]")


# ---------------------------------------------------------------------------
# P2  Reduction to Gated DeltaNet (GDN2 sec. 2; GDN sec. 1.1 equation, whose
#     state is M = S^T in R^{dv x dk}):
#     alpha_t = a_t * 1, b = w = beta*1  =>  M_t = a_t M_{t-1} (I - beta_t k k^T) + beta_t v k^T
# P3  Reduction to DeltaNet (GDN sec. 1.1, both printed forms):
#     a_t = 1  =>  M_t = M_{t-1}(I - beta k k^T) + beta v k^T = M_{t-1} + beta (v - M_{t-1} k) k^T
# ---------------------------------------------------------------------------
def pin_gated_deltanet(orc, seed=2, deltanet=False):
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 2, 10, 1, 4, 6
    q, k, v, _, _, _ = _rand_case(rng, B, T, H, dk, dv)
    beta = rng.random((B, T, H))
    a = np.ones((B, T, H)) if deltanet else np.exp(-rng.random((B, T, H)) * 2.0)
    la = np.repeat(np.log(a)[..., None], dk, axis=-1)
    b = np.repeat(beta[..., None], dk, axis=-1)
    w = np.repeat(beta[..., None], dv, axis=-1)
    M0 = rng.standard_normal((B, H, dv, dk)) * 0.5
    o, ST = orc.forward(q, k, v, la, b, w, S0=np.swapaxes(M0, -1, -2))
    for bb in range(B):
        M = M0[bb, 0].copy()
        for t in range(T):
            kt, vt, bt, at = k[bb, t, 0], v[bb, t, 0], beta[bb, t, 0], a[bb, t, 0]
            if deltanet:
                M_alt = M + bt * np.outer(vt - M @ kt, kt)
                M = M @ (np.eye(dk) - bt * np.outer(kt, kt)) + bt * np.outer(vt, kt)
                _close(M, M_alt, 1e-12, "DeltaNet printed forms agree")
            else:
                M = at * M @ (np.eye(dk) - bt * np.outer(kt, kt)) + bt * np.outer(vt, kt)
            _close(o[bb, t, 0], M @ q[bb, t, 0], 1e-12, f"GDN o[b={bb},t={t}]")
        _close(ST[bb, 0], M.T, 1e-12, f"GDN S_T[b={bb}]")


def pin_deltanet(orc, seed=3):
    pin_gated_deltanet(orc, seed=seed, deltanet=True)


# ---------------------------------------------------------------------------
# P4  Full reset (VIS: "alpha = 0 clears the memory"; GDN sec. 1.1 alpha -> 0):
#     log alpha_t = -inf  =>  S_t = k_t z_t^T exactly, o_t = (k_t . q_t) z_t
# ---------------------------------------------------------------------------
def pin_full_reset(orc, seed=4):
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 1, 9, 2, 6, 5
    q, k, v, la, b, w = _rand_case(rng, B, T, H, dk, dv)
    t_reset = 6
    la[0, t_reset] = -np.inf
    o_full, _ = orc.forward(q, k, v, la, b, w, S0=rng.standard_normal((B, H, dk, dv)))
    _, S_at = orc.forward(q[:, :t_reset + 1], k[:, :t_reset + 1], v[:, :t_reset + 1],
                          la[:, :t_reset + 1], b[:, :t_reset + 1], w[:, :t_reset + 1],
                          S0=rng.standard_normal((B, H, dk, dv)))
    for h in range(H):
        z = w[0, t_reset, h] * v[0, t_reset, h]
        assert np.array_equal(S_at[0, h], np.outer(k[0, t_reset, h], z)), "reset state is k z^T"
        _close(o_full[0, t_reset, h], np.dot(k[0, t_reset, h], q[0, t_reset, h]) * z, 1e-14, "reset output")


# ---------------------------------------------------------------------------
# P5  No erase (b = 0): the rule is channel-decay plus add (the Mamba-2 rule of
#     GDN sec. 1.1 with the decay made channel-wise, GDN2 sec. 3 with e = 0):
#     S_t = Diag(exp G_t) S_0 + sum_{i<=t} Diag(exp(G_t - G_i)) k_i z_i^T,
#     G_t = sum_{s<=t} log alpha_s
# ---------------------------------------------------------------------------
def pin_no_erase_closed_form(orc, seed=5):
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 1, 16, 3, 7, 4
    q, k, v, la, _, w = _rand_case(rng, B, T, H, dk, dv)
    b = np.zeros((B, T, H, dk))
    S0 = rng.standard_normal((B, H, dk, dv))
    o, ST = orc.forward(q, k, v, la, b, w, S0=S0)
    G = np.cumsum(la, axis=1)
    for h in range(H):
        for t in range(T):
            S = np.exp(G[0, t, h])[:, None] * S0[0, h]
            for i in range(t + 1):
                S = S + np.outer(np.exp(G[0, t, h] - G[0, i, h]) * k[0, i, h], w[0, i, h] * v[0, i, h])
            _close(o[0, t, h], S.T @ q[0, t, h], 1e-12, f"b=0 o[t={t}]")
        _close(ST[0, h], S, 1e-12, "b=0 S_T")


# ---------------------------------------------------------------------------
# P6  One-hot keys (VIS memory simulation: four slots, two-dimensional values,
#     orthogonal one-hot keys, erase touches only the addressed slot):
#     k_t = e_j  =>  row j: S_j <- (1 - b_j) alpha_j S_j + z;  row c != j: S_c <- alpha_c S_c
#     Dyadic gates keep every product short; exp(log alpha) rounds, so the
#     comparison allows a few ulps.
# ---------------------------------------------------------------------------
def pin_one_hot_slots(orc):
    dk, dv, T = 4, 2, 8
    slots = [0, 2, 1, 2, 3, 0, 2, 2]
    k = np.zeros((1, T, 1, dk))
    for t, j in enumerate(slots):
        k[0, t, 0, j] = 1.0
    q = np.zeros((1, T, 1, dk))
    for t in range(T):
        q[0, t, 0, (slots[t] + 1) % dk] = 1.0  # read a neighbouring slot
    alpha = np.array([1.0, 0.5, 0.75, 0.25])
    la = np.broadcast_to(np.log(alpha), (1, T, 1, dk)).copy()
    b = np.broadcast_to(np.array([0.5, 1.0, 0.25, 0.0]), (1, T, 1, dk)).copy()
    v = np.arange(T * dv, dtype=np.float64).reshape(1, T, 1, dv) - 5.0
    w = np.broadcast_to(np.array([1.0, 0.5]), (1, T, 1, dv)).copy()
    S0 = np.array([[1.0, -2.0], [0.5, 4.0], [-8.0, 0.25], [2.0, 2.0]])[None, None]
    o, ST = orc.forward(q, k, v, la, b, w, S0=S0)
    S = S0[0, 0].copy()
    for t, j in enumerate(slots):
        S = alpha[:, None] * S
        S[j] = (1.0 - b[0, t, 0, j]) * S[j] + w[0, t, 0] * v[0, t, 0]
        _close(o[0, t, 0], S[(j + 1) % dk], 1e-15, f"one-hot read t={t}")
    _close(ST[0, 0], S, 1e-15, "one-hot final state")


# ---------------------------------------------------------------------------
# P7  Fast-weight objective (GDN2 sec. 2): S_t is the minimiser of
#     L(S) = ||S - Sb||_F^2 - 2 <S^T k_t, z_t - Sb^T e_t>,  Sb = Diag(alpha_t) S_{t-1}.
#     L is strictly convex (Hessian 2I): the gradient vanishes at S_t and L rises
#     along every perturbation.
# ---------------------------------------------------------------------------
def pin_objective_stationarity(orc, seed=7):
    rng = np.random.default_rng(seed)
    N, H, dk, dv = 3, 2, 6, 5
    S_prev = rng.standard_normal((N, H, dk, dv))
    q, k, v, la, b, w = (x[:, 0] for x in _rand_case(rng, N, 1, H, dk, dv))
    b = b * 2.0  # the erase-range ablation of GDN2 sec. 4 (b in [0, 2]) keeps the objective form
    _, S_new = orc.decode_step(q, k, v, la, b, w, S_prev)
    for n in range(N):
        for h in range(H):
            Sb = np.exp(la[n, h])[:, None] * S_prev[n, h]
            e, z, kk = b[n, h] * k[n, h], w[n, h] * v[n, h], k[n, h]

            def L(S):
                return np.sum((S - Sb) ** 2) - 2.0 * np.dot(S.T @ kk, z - Sb.T @ e)

            St = S_new[n, h]
            grad = 2.0 * (St - Sb) - 2.0 * np.outer(kk, z - Sb.T @ e)
            assert np.max(np.abs(grad)) < 1e-12, f"objective gradient at S_t: {np.max(np.abs(grad)):.2e}"
            for _ in range(4):
                D = rng.standard_normal((dk, dv)) * 1e-3
                assert L(St + D) > L(St) and L(St - D) > L(St), "S_t is not the minimiser"


# ---------------------------------------------------------------------------
# P8  Exact write (GDN2 sec. 2: "predict the target residual along k"):
#     ||k|| = 1  =>  S_t^T k_t = Sb^T ((1 - b_t) (.) k_t) + z_t,  and with b = 1: S_t^T k_t = z_t.
# ---------------------------------------------------------------------------
def pin_exact_write(orc, seed=8):
    rng = np.random.default_rng(seed)
    N, H, dk, dv = 2, 3, 8, 5
    S_prev = rng.standard_normal((N, H, dk, dv))
    q, k, v, la, b, w = (x[:, 0] for x in _rand_case(rng, N, 1, H, dk, dv))
    _, S_new = orc.decode_step(q, k, v, la, b, w, S_prev)
    _, S_one = orc.decode_step(q, k, v, la, np.ones_like(b), w, S_prev)
    for n in range(N):
        for h in range(H):
            Sb = np.exp(la[n, h])[:, None] * S_prev[n, h]
            z = w[n, h] * v[n, h]
            _close(S_new[n, h].T @ k[n, h], Sb.T @ ((1.0 - b[n, h]) * k[n, h]) + z, 1e-13, "read-back")
            _close(S_one[n, h].T @ k[n, h], z, 1e-13, "exact write with b = 1")


# ---------------------------------------------------------------------------
# P9  Dense transition product (GDN2 sec. 3: per-token factor (I - k_t e_t^T)):
#     with A_t = (I - k_t e_t^T) Diag(alpha_t):  S_T = A_T...A_1 S_0 + sum_t A_T...A_{t+1} k_t z_t^T
#     evaluated as explicit matrix products at tiny sizes (brute force).
# ---------------------------------------------------------------------------
def pin_dense_product(orc, seed=9):
    rng = np.random.default_rng(seed)
    for (dk, dv, T) in [(1, 1, 5), (2, 3, 8), (4, 4, 8), (3, 2, 7)]:
        q, k, v, la, b, w = _rand_case(rng, 1, T, 1, dk, dv, normalise=False)
        b = b * 2.0
        S0 = rng.standard_normal((1, 1, dk, dv))
        _, ST = orc.forward(q, k, v, la, b, w, S0=S0)
        A = [(np.eye(dk) - np.outer(k[0, t, 0], b[0, t, 0] * k[0, t, 0])) @ np.diag(np.exp(la[0, t, 0]))
             for t in range(T)]
        total = np.eye(dk)
        for t in range(T):
            total = A[t] @ total
        expect = total @ S0[0, 0]
        for t in range(T):
            P = np.eye(dk)
            for s in range(t + 1, T):
                P = A[s] @ P
            expect = expect + P @ np.outer(k[0, t, 0], w[0, t, 0] * v[0, t, 0])
        _close(ST[0, 0], expect, 1e-12, f"dense product dk={dk} dv={dv}")


# ---------------------------------------------------------------------------
# P10 Structure: (a) the recurrence splits at any token (resume from S_T);
#     (b) for fixed q, k, alpha, b, w the map (S0, v) -> (o, S_T) is linear.
# ---------------------------------------------------------------------------
def pin_split_and_linearity(orc, seed=10):
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 2, 21, 2, 5, 4
    q, k, v, la, b, w = _rand_case(rng, B, T, H, dk, dv)
    S0 = rng.standard_normal((B, H, dk, dv))
    o, ST = orc.forward(q, k, v, la, b, w, S0=S0)
    for cut in (0, 1, 7, 20, 21):
        o1, S1 = orc.forward(q[:, :cut], k[:, :cut], v[:, :cut], la[:, :cut], b[:, :cut], w[:, :cut], S0=S0)
        o2, S2 = orc.forward(q[:, cut:], k[:, cut:], v[:, cut:], la[:, cut:], b[:, cut:], w[:, cut:], S0=S1)
        _close(np.concatenate([o1, o2], axis=1), o, 1e-13, f"split at {cut}: o")
        _close(S2, ST, 1e-13, f"split at {cut}: S_T")
    v2 = rng.standard_normal(v.shape)
    S02 = rng.standard_normal(S0.shape)
    oa, Sa = orc.forward(q, k, v2, la, b, w, S0=S02)
    os_, Ss = orc.forward(q, k, 2.0 * v + 3.0 * v2, la, b, w, S0=2.0 * S0 + 3.0 * S02)
    _close(os_, 2.0 * o + 3.0 * oa, 1e-12, "linearity o")
    _close(Ss, 2.0 * ST + 3.0 * Sa, 1e-12, "linearity S_T")


# ---------------------------------------------------------------------------
# P11 Gate-aware backward (GDN2 sec. 3) checked by central finite differences
#     of L = <o, dO> + <S_T, dS_T> in fp64.
# ---------------------------------------------------------------------------
def _loss(orc, x, dO, dST):
    o, ST = orc.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], S0=x["S0"])
    return float(np.sum(o * dO) + np.sum(ST * dST))


def pin_backward_fd(orc, seed=11, B=1, T=6, H=2, dk=3, dv=4, full=True, n_dirs=3):
    rng = np.random.default_rng(seed)
    q, k, v, la, b, w = _rand_case(rng, B, T, H, dk, dv)
    x = dict(q=q, k=k, v=v, log_alpha=la, b=b * 1.5, w=w, S0=rng.standard_normal((B, H, dk, dv)) * 0.5)
    dO = rng.standard_normal((B, T, H, dv))
    dST = rng.standard_normal((B, H, dk, dv))
    g = orc.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], dO, S0=x["S0"], dS_T=dST)
    names = {"q": "dq", "k": "dk", "v": "dv", "log_alpha": "dlog_alpha", "b": "db", "w": "dw", "S0": "dS0"}
    eps = 1e-6
    for name, gname in names.items():
        G = g[gname]
        if full:
            num = np.zeros_like(G)
            it = np.nditer(x[name], flags=["multi_index"])
            for _ in it:
                idx = it.multi_index
                xp = {kk: vv.copy() for kk, vv in x.items()}
                xm = {kk: vv.copy() for kk, vv in x.items()}
                xp[name][idx] += eps
                xm[name][idx] -= eps
                num[idx] = (_loss(orc, xp, dO, dST) - _loss(orc, xm, dO, dST)) / (2 * eps)
            _close(G, num, 1e-7, f"FD {gname}")
        for _ in range(n_dirs):
            D = rng.standard_normal(x[name].shape)
            xp = {kk: vv.copy() for kk, vv in x.items()}
            xm = {kk: vv.copy() for kk, vv in x.items()}
            xp[name] += eps * D
            xm[name] -= eps * D
            num = (_loss(orc, xp, dO, dST) - _loss(orc, xm, dO, dST)) / (2 * eps)
            ana = float(np.sum(G * D))
            assert abs(num - ana) <= 1e-6 * max(1.0, abs(ana)), f"directional FD {gname}: {num} vs {ana}"


def pin_backward_fd_t32_d16(orc, seed=12):
    """Directional central differences at T = 32, d = 16 (the backward check instance)."""
    pin_backward_fd(orc, seed=seed, B=1, T=32, H=2, dk=16, dv=16, full=False, n_dirs=4)


# ---------------------------------------------------------------------------
# Self-consistency (not a pin, but part of the suite): the decode step is the
# forward's token update, and T = 0 returns S0.
# ---------------------------------------------------------------------------
def check_decode_matches_forward(orc, seed=13):
    rng = np.random.default_rng(seed)
    B, T, H, dk, dv = 2, 5, 3, 4, 6
    q, k, v, la, b, w = _rand_case(rng, B, T, H, dk, dv)
    S0 = rng.standard_normal((B, H, dk, dv))
    o, ST = orc.forward(q, k, v, la, b, w, S0=S0)
    S = S0.copy()
    for t in range(T):
        ot, S = orc.decode_step(q[:, t], k[:, t], v[:, t], la[:, t], b[:, t], w[:, t], S)
        _close(ot, o[:, t], 1e-14, "decode o")
    _close(S, ST, 1e-14, "decode S")
    o0, S00 = orc.forward(q[:, :0], k[:, :0], v[:, :0], la[:, :0], b[:, :0], w[:, :0], S0=S0)
    assert o0.shape == (B, 0, H, dv) and np.array_equal(S00, S0)


# ---------------------------------------------------------------------------
# P12  Block epilogue, y = RMSNorm(o) weight (.) silu(g) (GDN2 sec. 3, block data flow):
#      closed forms and invariants of the norm and of the gate
# ---------------------------------------------------------------------------
def pin_output_norm_gate(orc=None, seed=14, OB=None):
    if OB is None:
        from oracle import block as OB

    rng = np.random.default_rng(seed)
    n, dv, eps = 7, 16, 1e-6
    o = rng.standard_normal((n, dv))
    wgt = rng.uniform(0.5, 1.5, dv)
    g = rng.standard_normal((n, dv))
    # silu: silu(x) - silu(-x) = x; silu(0) = 0; silu(x) ~ x for large x, ~ 0 for very negative x
    x = rng.standard_normal(50) * 3
    _close(OB.silu(x) - OB.silu(-x), x, 1e-14, "silu odd part")
    assert OB.silu(0.0) == 0.0 and abs(OB.silu(40.0) - 40.0) < 1e-12 and abs(OB.silu(-40.0)) < 1e-15
    # a constant row c 1 normalises to sign(c) |c| / sqrt(c^2 + eps)
    c = -2.5
    y = OB.output_norm_gate(np.full((1, dv), c), weight=wgt, eps=eps)
    _close(y, np.sign(c) * abs(c) / np.sqrt(c * c + eps) * wgt[None], 1e-14, "constant row")
    # the normalised row (unit weight, no gate) has mean square ms / (ms + eps) and scale invariance
    y1 = OB.output_norm_gate(o, weight=np.ones(dv), eps=eps)
    ms = np.mean(o * o, axis=-1)
    _close(np.mean(y1 * y1, axis=-1), ms / (ms + eps), 1e-13, "rms of the output")
    _close(OB.output_norm_gate(37.0 * o, weight=wgt, eps=0.0), OB.output_norm_gate(o, weight=wgt, eps=0.0), 1e-13,
           "scale invariance")
    # a zero gate closes the output; the gate factor is the same with or without the norm
    assert np.all(OB.output_norm_gate(o, g=np.zeros_like(o), weight=wgt) == 0.0)
    _close(OB.output_norm_gate(o, g=g, weight=wgt) / OB.output_norm_gate(o, weight=wgt),
           OB.output_norm_gate(np.ones_like(o), g=g), 1e-12, "gate factor")
    # an open gate (g large and positive) passes the normalised output through, scaled by g
    _close(OB.output_norm_gate(o, g=np.full_like(o, 40.0), weight=wgt), 40.0 * OB.output_norm_gate(o, weight=wgt),
           1e-12, "open gate")
    # absent factors: identity
    assert np.array_equal(OB.output_norm_gate(o), o)


# ---------------------------------------------------------------------------
# P13  Block prologue (GDN2 sec. 3, block data flow): the causal depthwise convolution
#      against numpy's convolution, its state and causality, packed sequences, the L2
#      norm per head, the decay and gate activations against their direct formulas
# ---------------------------------------------------------------------------
def pin_block_prologue(orc=None, seed=15, OB=None):
    if OB is None:
        from oracle import block as OB

    rng = np.random.default_rng(seed)
    W, T, C = 4, 11, 5
    x = rng.standard_normal((1, T, C))
    wgt = rng.standard_normal((C, W))
    st = rng.standard_normal((1, W - 1, C))
    # the convolution is numpy's ("valid" over [state; x], taps reversed: tap W-1 on the current token)
    for state in (None, st):
        y = OB.causal_conv(x, wgt, state)
        pad = np.zeros((W - 1, C)) if state is None else state[0]
        z = np.concatenate([pad, x[0]], axis=0)
        for c in range(C):
            _close(y[0, :, c], np.convolve(z[:, c], wgt[c, ::-1], mode="valid"), 1e-13, "conv vs numpy")
    # delta taps: the identity and a one-token delay
    delta = np.zeros((C, W))
    delta[:, W - 1] = 1.0
    _close(OB.causal_conv(x, delta, st), x, 0, "delta taps")
    delay = np.zeros((C, W))
    delay[:, W - 2] = 1.0
    _close(OB.causal_conv(x, delay, st), np.concatenate([st[:, -1:], x[:, :-1]], axis=1), 0, "one-token delay")
    # conv then SiLU: with delta taps the prologue of v is silu(x)
    yv, _ = OB.short_conv_silu(x, delta, st)
    _close(yv, OB.silu(x), 1e-15, "delta taps then silu")
    # causality and reach: a change at t0 moves outputs t0 .. t0 + W - 1 only
    x2 = x.copy()
    x2[0, 4] += 1.0
    dy = np.abs(OB.causal_conv(x2, wgt, st) - OB.causal_conv(x, wgt, st))[0].max(axis=1)
    assert np.all(dy[:4] == 0) and np.all(dy[4 + W:] == 0) and np.all(dy[4:4 + W] > 0), "causality"
    # continuing from the state: one call over [x1; x2] equals two calls, also when the second
    # part is shorter than the state
    for cut in (6, T - 2):
        y_all, s_all = OB.short_conv_silu(x, wgt, st)
        y1, s1 = OB.short_conv_silu(x[:, :cut], wgt, st)
        y2, s2 = OB.short_conv_silu(x[:, cut:], wgt, s1)
        _close(np.concatenate([y1, y2], axis=1), y_all, 1e-14, "split outputs")
        _close(s2, s_all, 0, "split state")
    _close(s_all[0], np.concatenate([st[0], x[0]])[-(W - 1):], 0, "state = last W - 1 inputs")
    # packed sequences convolve on their own, each from its own state (empty ones keep it)
    lens = [3, 0, 1, 7]
    cu = np.concatenate([[0], np.cumsum(lens)])
    xs = rng.standard_normal((1, int(cu[-1]), C))
    sts = rng.standard_normal((len(lens), W - 1, C))
    yp, sp = OB.short_conv_silu(xs, wgt, cu_seqlens=cu, states=sts)
    for i in range(len(lens)):
        yi, si = OB.short_conv_silu(xs[:, cu[i]:cu[i + 1]], wgt, sts[i][None])
        if lens[i]:
            _close(yp[:, cu[i]:cu[i + 1]], yi, 0, f"packed seq {i}")
        _close(sp[i], si[0], 0, f"packed state {i}")
    _close(sp[1], sts[1], 0, "empty sequence keeps its state")
    # L2 norm per head: |y| = sqrt(s / (s + eps)); scale invariance at eps = 0; heads apart
    v = rng.standard_normal((6, 8))
    v[0] *= 1e-4  # a row whose squared norm is comparable to eps
    for eps in (0.0, 1e-6):
        s = np.sum(v * v, axis=-1)
        _close(np.linalg.norm(OB.l2_normalize(v, eps), axis=-1), np.sqrt(s / (s + eps)), 1e-13, "l2 norms")
    _close(OB.l2_normalize(3.7 * v, 0.0), OB.l2_normalize(v, 0.0), 1e-14, "l2 scale invariance")
    xh = rng.standard_normal((1, T, 2 * C))
    wh = rng.standard_normal((2 * C, W))
    yh, _ = OB.short_conv_silu(xh, wh, l2norm=True, eps=0.0, heads=2)
    _close(np.linalg.norm(yh.reshape(1, T, 2, C), axis=-1), np.ones((1, T, 2)), 1e-13, "unit norm per head")
    xh2 = xh.copy()
    xh2[..., C:] *= 5.0  # head 1's input only
    yh2, _ = OB.short_conv_silu(xh2, wh, l2norm=True, eps=0.0, heads=2)
    _close(yh2[..., :C], yh[..., :C], 0, "head 0 independent of head 1")
    # activations against their direct formulas
    a = rng.standard_normal(40) * 4
    _close(np.exp(OB.neg_softplus(a)), 1.0 / (1.0 + np.exp(a)), 1e-14, "alpha = 1 / (1 + e^a)")
    _close(np.exp(OB.neg_softplus(a)) + OB.sigmoid(a), np.ones_like(a), 1e-14, "alpha + sigmoid(a) = 1")
    _close(OB.sigmoid(a), 1.0 / (1.0 + np.exp(-a)), 1e-14, "sigmoid")
    assert abs(OB.neg_softplus(40.0) + 40.0) < 1e-15 and abs(OB.neg_softplus(-40.0) + np.exp(-40.0)) < 1e-30
    assert OB.sigmoid(0.0) == 0.5


ALL_PINS = [pin_kda, pin_gated_deltanet, pin_deltanet, pin_full_reset, pin_no_erase_closed_form,
            pin_one_hot_slots, pin_objective_stationarity, pin_exact_write, pin_dense_product,
            pin_split_and_linearity, pin_backward_fd, pin_backward_fd_t32_d16, pin_output_norm_gate,
            pin_block_prologue]
