"""The chunk-form equations, restated in float64 numpy, against the oracle.

The CUDA path computes the forward in chunks (a chunk-parallel preparation and
a sequential carry over chunks), and the planned backward does the same in
reverse.  This CPU test pins both sets of equations, with a per-channel decay
(KDA; a scalar decay and DeltaNet are its special cases), to the token-by-token
oracle on a ragged sequence with an initial state and a q scale:

forward, per chunk with the chunk-local cumulative log decay gamma (C x d_k):
    A = tril(Diag(beta) (K o e^gamma)(K o e^-gamma)^T, -1),  T = (I + A)^-1
    W = T Diag(beta) (K o e^gamma),  U' = T Diag(beta) V,  E = U' - W S0
    P = tril(scale (Q o e^gamma)(K o e^-gamma)^T)
    O = scale (Q o e^gamma) S0 + P E
    S_C = Diag(e^gamma_C) S0 + Kt^T E,  Kt = K o e^(gamma_C - gamma)
backward, chunks in reverse, dS the gradient of the chunk's end state:
    dE = Kt dS + P^T dO
    dS0 = Diag(e^gamma_C) dS + scale (Q o e^gamma)^T dO - W^T dE
so the sequential part of the backward is the forward carry's mirror on the
same per-chunk operands (Kt, P, Q o e^gamma, W); every other gradient is local
to a chunk given S0, dS and dO.  GDN-2's chunk form (its own test below) and
a carry step over two records (the 128-token step) are pinned the same way.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_forward_b200.inputs import make_inputs

C = 8


def chunk_forward(q, k, v, beta, lg, s0, scale):
    """One sequence: q, k [T, dk], v [T, dv], beta [T], lg [T, dk] (log decay)."""
    T = k.shape[0]
    o = np.zeros((T, v.shape[1]))
    S = s0.copy()
    saved = []
    for c0 in range(0, T, C):
        sl = slice(c0, min(T, c0 + C))
        K, Q, V, b = k[sl], q[sl], v[sl], beta[sl]
        gam = np.cumsum(lg[sl], axis=0)
        Kg, Ki, Qg = K * np.exp(gam), K * np.exp(-gam), Q * np.exp(gam)
        n = K.shape[0]
        A = np.tril(b[:, None] * (Kg @ Ki.T), -1)
        Tm = np.linalg.inv(np.eye(n) + A)
        W = Tm @ (b[:, None] * Kg)
        Up = Tm @ (b[:, None] * V)
        E = Up - W @ S
        P = np.tril(scale * (Qg @ Ki.T))
        Kt = K * np.exp(gam[-1] - gam)
        o[sl] = scale * Qg @ S + P @ E
        saved.append(dict(sl=sl, S0=S.copy(), K=K, Q=Q, V=V, b=b, gam=gam, Kg=Kg, Ki=Ki, Qg=Qg,
                          T=Tm, W=W, E=E, P=P, Kt=Kt))
        S = np.exp(gam[-1])[:, None] * S + Kt.T @ E
    return o, S, saved


def chunk_backward(saved, dO, dS_final, scale):
    T = saved[-1]["sl"].stop
    dk, dv = saved[0]["K"].shape[1], saved[0]["V"].shape[1]
    g = {"q": np.zeros((T, dk)), "k": np.zeros((T, dk)), "v": np.zeros((T, dv)),
         "beta": np.zeros(T), "log_g": np.zeros((T, dk))}
    dS = dS_final.copy()
    for sv in reversed(saved):
        sl, S0, K, Q, V, b, gam = (sv[x] for x in ("sl", "S0", "K", "Q", "V", "b", "gam"))
        Kg, Ki, Qg, Tm, W, E, P, Kt = (sv[x] for x in ("Kg", "Ki", "Qg", "T", "W", "E", "P", "Kt"))
        dOc = dO[sl]
        gC = np.exp(gam[-1])
        # the reverse carry: end-state gradient -> start-state gradient
        dE = Kt @ dS + P.T @ dOc
        dS0 = gC[:, None] * dS + scale * Qg.T @ dOc - W.T @ dE
        # chunk-local gradients
        dgam = np.zeros_like(gam)
        dgam[-1] += np.sum(dS * S0, 1) * gC
        dKt = E @ dS.T
        dQg = scale * dOc @ S0.T
        dP = np.tril(dOc @ E.T)
        dW = -dE @ S0.T
        tU, tW = Tm.T @ dE, Tm.T @ dW
        dV = b[:, None] * tU
        dKg = b[:, None] * tW
        db = np.sum(V * tU, 1) + np.sum(Kg * tW, 1)
        dT = dE @ (b[:, None] * V).T + dW @ (b[:, None] * Kg).T
        dA = np.tril(-Tm.T @ dT @ Tm.T, -1)
        db += np.sum(dA * (Kg @ Ki.T), 1)
        M = b[:, None] * dA
        dKg += M @ Ki
        dKi = M.T @ Kg + scale * dP.T @ Qg
        dQg += scale * dP @ Ki
        fac = np.exp(gam[-1] - gam)
        dK = dKt * fac + dKg * np.exp(gam) + dKi * np.exp(-gam)
        dgam += -dKt * Kt + dKg * Kg - dKi * Ki + dQg * Qg
        dgam[-1] += np.sum(dKt * Kt, 0)
        g["q"][sl] = dQg * np.exp(gam)
        g["k"][sl] = dK
        g["v"][sl] = dV
        g["beta"][sl] = db
        g["log_g"][sl] = np.cumsum(dgam[::-1], axis=0)[::-1]
        dS = dS0
    g["initial_state"] = dS
    return g


@pytest.mark.parametrize("variant", ["deltanet", "gdn", "kda"])
def test_chunk_equations_match_the_oracle(variant):
    B, T, H, dk, dv, scale = 1, 29, 1, 6, 5, 0.7
    d = make_inputs(variant, B, T, H, dk, dv, dtype=torch.float32, seed=7)
    d = {k: (None if v is None else v.double().numpy()) for k, v in d.items()}
    rng = np.random.default_rng(7)
    s0 = rng.standard_normal((B, H, dk, dv))
    dO = rng.standard_normal((B, T, H, dv))
    dS = rng.standard_normal((B, H, dk, dv))
    o_ref, S_ref = oracle.forward(variant, **d, initial_state=s0, scale=scale)
    g_ref = oracle.backward(variant, d_o=dO, d_final=dS, initial_state=s0, scale=scale, **d)

    if variant == "deltanet":
        lg = np.zeros((T, dk))
    elif variant == "gdn":
        lg = np.repeat(d["log_g"][0, :, 0][:, None], dk, axis=1)
    else:
        lg = d["log_g"][0, :, 0]
    o, S, saved = chunk_forward(d["q"][0, :, 0], d["k"][0, :, 0], d["v"][0, :, 0], d["beta"][0, :, 0],
                                lg, s0[0, 0], scale)
    np.testing.assert_allclose(o, o_ref[0, :, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(S, S_ref[0, 0], rtol=0, atol=1e-12)

    g = chunk_backward(saved, dO[0, :, 0], dS[0, 0], scale)
    for name in ("q", "k", "v", "beta"):
        np.testing.assert_allclose(g[name], g_ref[name][0, :, 0], rtol=0, atol=1e-10)
    np.testing.assert_allclose(g["initial_state"], g_ref["initial_state"][0, 0], rtol=0, atol=1e-10)
    if variant == "gdn":      # one decay per token: its gradient sums over the channels
        np.testing.assert_allclose(g["log_g"].sum(1), g_ref["log_g"][0, :, 0], rtol=0, atol=1e-10)
    elif variant == "kda":
        np.testing.assert_allclose(g["log_g"], g_ref["log_g"][0, :, 0], rtol=0, atol=1e-10)


@pytest.mark.parametrize("variant", ["deltanet", "gdn", "kda"])
def test_segmented_carry_with_finer_parts_matches_the_oracle(variant):
    """The segmented carry as the library plans it for B=1, H=17, T=7041 on 148
    SMs (111 chunks, the last of one token): phase 1 runs segment 0 from S0 and
    the other segments but the last from zero (offsets D_g) and from the
    identity without values (maps M_g), leaving snapshots of both at every
    multiple of the part length inside a segment; the chain forms the segment
    starts S[g+1] = M_g S[g] + D_g and, in the same pass, each part start inside
    segment g as M_g(j) S[g] + D_g(j) (D_0(j) itself in segment 0); phase 2 runs
    the parts from their starts.  Here with chunks of 8 tokens and small d_k,
    d_v, against the token-by-token oracle.  beta and the decay are weakened
    (x 0.05, x 0.01) so that a segment's start state still shows at its end:
    with the recipe's gates the maps M_g(j) fall below 1e-20 and the test
    would not see their products."""
    import gated_delta_rule_forward_b200 as gdr
    plan = gdr.forward_plan(variant, 1, 7041, 17, 128, 148)
    G, L, P, Lp = plan["segments"], plan["segment_chunks"], plan["parts"], plan["part_chunks"]
    assert P > G and Lp < L
    NC = 111
    B, T, H, dk, dv, scale = 1, (NC - 1) * C + 1, 1, 6, 5, 0.7
    d = make_inputs(variant, B, T, H, dk, dv, dtype=torch.float32, seed=17)
    d = {k: (None if v is None else v.double().numpy()) for k, v in d.items()}
    d["beta"] = 0.05 * d["beta"]
    if d["log_g"] is not None:
        d["log_g"] = 0.01 * d["log_g"]
    s0 = np.random.default_rng(17).standard_normal((dk, dv))
    o_ref, S_ref = oracle.forward(variant, **d, initial_state=s0[None, None], scale=scale)
    lg = (np.zeros((T, dk)) if variant == "deltanet" else
          np.repeat(d["log_g"][0, :, 0][:, None], dk, axis=1) if variant == "gdn" else d["log_g"][0, :, 0])
    # per-chunk quantities (none depends on the state) and each chunk's affine map S -> A S + Bc
    _, _, saved = chunk_forward(d["q"][0, :, 0], d["k"][0, :, 0], d["v"][0, :, 0], d["beta"][0, :, 0], lg, s0,
                                scale)
    assert len(saved) == NC
    for sv in saved:
        sv["U"] = sv["T"] @ (sv["b"][:, None] * sv["V"])
        sv["A"] = np.diag(np.exp(sv["gam"][-1])) - sv["Kt"].T @ sv["W"]
        sv["Bc"] = sv["Kt"].T @ sv["U"]

    def sweep(x, c0, c1, values=True, snaps=None):
        for c in range(c0, c1):
            if snaps is not None and c > c0 and c % Lp == 0:
                snaps[c // Lp] = x.copy()
            x = saved[c]["A"] @ x + (saved[c]["Bc"] if values else 0)
        return x

    # phase 1
    Dend, Mend, snapD, snapM = {}, {}, {}, {}
    for g in range(G - 1):
        Dend[g] = sweep(s0 if g == 0 else np.zeros((dk, dv)), g * L, min(NC, (g + 1) * L), snaps=snapD)
    for g in range(1, G - 1):
        Mend[g] = sweep(np.eye(dk), g * L, min(NC, (g + 1) * L), values=False, snaps=snapM)
    # the chain, in the kernel's order: part starts inside segment g, then segment start g + 1
    starts, Sg, p = {0: s0}, s0, 1
    for g in range(G - 1):
        while p < P and p * Lp < (g + 1) * L:
            starts[p] = snapD[p] if g == 0 else snapM[p] @ Sg + snapD[p]
            p += 1
        Sg = Dend[0] if g == 0 else Mend[g] @ Sg + Dend[g]
        if p < P and p * Lp == (g + 1) * L:
            starts[p] = Sg
            p += 1
    assert p == P and sorted(starts) == list(range(P))
    # phase 2: every part from its start, with outputs
    o = np.zeros((T, dv))
    for q in range(P):
        x = starts[q]
        for c in range(q * Lp, min(NC, (q + 1) * Lp)):
            sv = saved[c]
            o[sv["sl"]] = scale * sv["Qg"] @ x + sv["P"] @ (sv["U"] - sv["W"] @ x)
            x = sv["A"] @ x + sv["Bc"]
    np.testing.assert_allclose(o, o_ref[0, :, 0], rtol=0, atol=1e-10)
    np.testing.assert_allclose(x, S_ref[0, 0], rtol=0, atol=1e-10)
    # the maps matter: the last part's start moves by more than 1e-3 without its M S[g] term
    g_last = ((P - 1) * Lp - 1) // L
    assert np.abs(Mend[g_last] @ Dend[g_last - 1]).max() > 1e-3 if g_last >= 2 else True


@pytest.mark.parametrize("variant", ["gdn", "kda"])
def test_two_record_carry_step_matches_the_oracle(variant):
    """One carry step over two records (c, c+1), from their single-chunk quantities
    only, with G_c = Diag(e^gamma_C) of chunk c (the chunk's decay per channel):
        M    = W_{c+1} Kt_c^T                     (cross term, local to the pair)
        What = [W_c ; W_{c+1} G_c - M W_c],  Uhat = [U'_c ; U'_{c+1} - M U'_c]
        [E_c ; E_{c+1}] = Uhat - What S
        S''  = G_{c+1} G_c S + [Kt_c G_{c+1} ; Kt_{c+1}]^T [E_c ; E_{c+1}]
        O_c  = Qg_c S + P_c E_c
        O_c+1 = Qg_{c+1} G_c S + [Qg_{c+1} Kt_c^T , P_{c+1}] [E_c ; E_{c+1}]
    (Qg = scale Q o e^gamma).  Half the sequential steps of the 64-token carry."""
    B, T, H, dk, dv, scale = 1, 2 * C, 1, 6, 5, 0.7
    d = make_inputs(variant, B, T, H, dk, dv, dtype=torch.float32, seed=9)
    d = {k: (None if v is None else v.double().numpy()) for k, v in d.items()}
    rng = np.random.default_rng(9)
    S = rng.standard_normal((dk, dv))
    o_ref, S_ref = oracle.forward(variant, **d, initial_state=S[None, None], scale=scale)
    lg = (np.zeros((T, dk)) if variant == "deltanet" else
          np.repeat(d["log_g"][0, :, 0][:, None], dk, axis=1) if variant == "gdn" else d["log_g"][0, :, 0])
    _, _, sv = chunk_forward(d["q"][0, :, 0], d["k"][0, :, 0], d["v"][0, :, 0], d["beta"][0, :, 0], lg, S, scale)
    a, b = sv
    ga, gb = np.exp(a["gam"][-1]), np.exp(b["gam"][-1])      # per-channel end decays
    Upa, Upb = a["T"] @ (a["b"][:, None] * a["V"]), b["T"] @ (b["b"][:, None] * b["V"])
    Qga, Qgb = scale * a["Qg"], scale * b["Qg"]
    M = b["W"] @ a["Kt"].T
    What = np.vstack([a["W"], b["W"] * ga[None, :] - M @ a["W"]])
    Uhat = np.vstack([Upa, Upb - M @ Upa])
    E = Uhat - What @ S
    S2 = (gb * ga)[:, None] * S + np.vstack([a["Kt"] * gb[None, :], b["Kt"]]).T @ E
    Oa = Qga @ S + a["P"] @ E[:C]
    Ob = (Qgb * ga[None, :]) @ S + np.hstack([Qgb @ a["Kt"].T, b["P"]]) @ E
    np.testing.assert_allclose(np.vstack([Oa, Ob]), o_ref[0, :, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(S2, S_ref[0, 0], rtol=0, atol=1e-12)


def test_gdn2_chunk_equations_match_the_oracle():
    """GDN-2's chunk form, with a = b o k (erase) and d = (w - b) o k:
        A = tril(Gram(K, a), -1),  A^d = tril(Gram(K, d), -1),  P^a, P^d = tril(Gram(scale Q, a or d))
        T = (I + A)^-1,  W = T (K o e^gamma),  U' = T (I - A^d) V,  E = U' - W S0
        O = scale (Q o e^gamma) S0 + P^a E + P^d V
        S_C = Diag(e^gamma_C) S0 + (a o e^(gamma_C - gamma))^T E + (d o e^(gamma_C - gamma))^T V
    where Gram(X, Y)_tr = sum_i x_t[i] y_r[i] e^(gamma_t[i] - gamma_r[i]): the residual
    form of the other variants with the write split off ("Gated DeltaNet-2", technical
    core, read as erase on the key side and write weighted per channel)."""
    B, T, H, dk, dv, scale = 1, 29, 1, 6, 5, 0.7
    d = make_inputs("gdn2", B, T, H, dk, dv, dtype=torch.float32, seed=11)
    d = {k: (None if v is None else v.double().numpy()) for k, v in d.items()}
    S = np.random.default_rng(11).standard_normal((dk, dv))
    o_ref, S_ref = oracle.forward("gdn2", **d, initial_state=S[None, None], scale=scale)
    q, k, v = d["q"][0, :, 0], d["k"][0, :, 0], d["v"][0, :, 0]
    lg, eb, ww = d["log_g"][0, :, 0], d["erase_b"][0, :, 0], d["write_w"][0, :, 0]
    o = np.zeros((T, dv))
    for c0 in range(0, T, C):
        sl = slice(c0, min(T, c0 + C))
        K, Q, V = k[sl], scale * q[sl], v[sl]
        gam = np.cumsum(lg[sl], axis=0)
        a, dd = eb[sl] * K, (ww[sl] - eb[sl]) * K
        n = K.shape[0]

        def gram(X, Y):
            return (X * np.exp(gam)) @ (Y * np.exp(-gam)).T

        A, Ad = np.tril(gram(K, a), -1), np.tril(gram(K, dd), -1)
        Pa, Pd = np.tril(gram(Q, a)), np.tril(gram(Q, dd))
        Tm = np.linalg.inv(np.eye(n) + A)
        W = Tm @ (K * np.exp(gam))
        E = Tm @ (np.eye(n) - Ad) @ V - W @ S
        o[sl] = (Q * np.exp(gam)) @ S + Pa @ E + Pd @ V
        fac = np.exp(gam[-1] - gam)
        S = np.exp(gam[-1])[:, None] * S + (a * fac).T @ E + (dd * fac).T @ V
    np.testing.assert_allclose(o, o_ref[0, :, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(S, S_ref[0, 0], rtol=0, atol=1e-12)


def test_kla_chunk_form_is_gdn_with_the_kaczmarz_step():
    """"Kaczmarz Linear Attention" (implementation): the chunked solver changes only
    Diag(beta), with beta_t = eta_t / (||k_t||^2 + eps) computed from the loaded keys."""
    B, T, H, dk, dv, scale, eps = 1, 29, 1, 6, 5, 0.7, 1e-6
    d = make_inputs("kla", B, T, H, dk, dv, dtype=torch.float32, seed=13)
    d = {k: (None if v is None else v.double().numpy()) for k, v in d.items()}
    s0 = np.random.default_rng(13).standard_normal((dk, dv))
    o_ref, S_ref = oracle.forward("kla", **d, initial_state=s0[None, None], scale=scale, eps=eps)
    k = d["k"][0, :, 0]
    beta = d["beta"][0, :, 0] / (np.sum(k * k, 1) + eps)
    lg = np.repeat(d["log_g"][0, :, 0][:, None], dk, axis=1)
    o, S, _ = chunk_forward(d["q"][0, :, 0], k, d["v"][0, :, 0], beta, lg, s0, scale)
    np.testing.assert_allclose(o, o_ref[0, :, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(S, S_ref[0, 0], rtol=0, atol=1e-12)


def test_fp16_carry_operands_fit_the_bf16_budget():
    """The carry's precision choice: with the per-chunk products exact and every
    carry operand (S, E, W, U', Kt, P, Qg) rounded to fp16 with fp32 accumulation,
    as the tensor cores see them, a 2048-token GDN sequence at d = 128 stays well
    inside the bf16 parity budget (2e-2 of RMS); bf16 operands would not."""
    T, d, C64 = 2048, 128, 64
    dd = make_inputs("gdn", 1, T, 1, d, d, dtype=torch.bfloat16, seed=2)
    dd = {k: (None if v is None else v.double().numpy()) for k, v in dd.items()}
    o_ref, S_ref = oracle.forward("gdn", **dd)
    q, k, v = dd["q"][0, :, 0], dd["k"][0, :, 0], dd["v"][0, :, 0]
    beta, lg = dd["beta"][0, :, 0], dd["log_g"][0, :, 0]

    def run(rnd):
        S = np.zeros((d, d))
        out = []
        for c0 in range(0, T, C64):
            sl = slice(c0, c0 + C64)
            K, Q, V, b = k[sl], q[sl], v[sl], beta[sl]
            gam = np.cumsum(lg[sl])
            R = np.exp(gam[:, None] - gam[None, :])
            Tm = np.linalg.inv(np.eye(C64) + np.tril(b[:, None] * R * (K @ K.T), -1))
            W = Tm @ ((b * np.exp(gam))[:, None] * K)
            Up = Tm @ (b[:, None] * V)
            P = np.tril(R * (Q @ K.T))
            Kt = np.exp(gam[-1] - gam)[:, None] * K
            Qg = np.exp(gam)[:, None] * Q
            Sh = rnd(S)
            E = (rnd(Up) - rnd(W) @ Sh).astype(np.float32).astype(np.float64)
            out.append(rnd(Qg) @ Sh + rnd(P) @ rnd(E))
            S = (np.exp(gam[-1]) * S + rnd(Kt).T @ rnd(E)).astype(np.float32).astype(np.float64)
        o = np.vstack(out)
        rms = np.sqrt(np.mean(o_ref[0, :, 0] ** 2))
        return np.abs(o - o_ref[0, :, 0]).max() / rms

    f16 = lambda x: x.astype(np.float16).astype(np.float64)
    bf16 = lambda x: torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    assert run(f16) < 2e-2 / 2          # measured 6.4e-3
    assert run(bf16) > 2e-2             # measured 4.0e-2: bf16 operands break the budget


def _round_tf32(x):
    """Round to the tf32 format (8-bit exponent, 10 stored mantissa bits), to
    nearest with ties to even, from the float32 bit pattern."""
    u = np.asarray(x, np.float32).copy().view(np.uint32)
    u = (u + np.uint32(0xFFF) + ((u >> np.uint32(13)) & np.uint32(1))) & np.uint32(0xFFFFE000)
    return u.view(np.float32).astype(np.float64)


def test_channel_decay_gram_needs_tf32_operands():
    """KDA's Gram / attention product [K o G; Q o G](K o G^-1)^T, with the decay
    factored around the chunk's middle token (G = e^(gamma - gamma_m)): with every
    other product exact, tf32 operands keep a 2048-token sequence at d = 128 inside
    the bf16 budget (2e-2 of RMS); bf16 operands, one rounding of G, do not."""
    T, d, C64 = 2048, 128, 64
    dd = make_inputs("kda", 1, T, 1, d, d, dtype=torch.bfloat16, seed=4)
    dd = {k: (None if v is None else v.double().numpy()) for k, v in dd.items()}
    o_ref, _ = oracle.forward("kda", **dd)
    q, k, v, beta, lg = (dd[n][0, :, 0] for n in ("q", "k", "v", "beta", "log_g"))
    assert _round_tf32(np.array([1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11]))[0] == 1.0   # tie to even
    assert _round_tf32(np.array([1.0 + 3 * 2.0 ** -11]))[0] == 1.0 + 2.0 ** -9

    def run(rnd):
        S = np.zeros((d, d))
        out = []
        for c0 in range(0, T, C64):
            sl = slice(c0, c0 + C64)
            K, Q, V, b = k[sl], q[sl], v[sl], beta[sl]
            gam = np.cumsum(lg[sl], axis=0)
            G = np.exp(gam - gam[31])
            GQ = rnd(np.vstack([K * G, Q * G])) @ rnd(K / G).T
            A = np.tril(b[:, None] * GQ[:C64], -1)
            P = np.tril(GQ[C64:])
            Tm = np.linalg.inv(np.eye(C64) + A)
            W = Tm @ (b[:, None] * K * np.exp(gam))
            E = Tm @ (b[:, None] * V) - W @ S
            out.append((Q * np.exp(gam)) @ S + P @ E)
            S = np.exp(gam[-1])[:, None] * S + (K * np.exp(gam[-1] - gam)).T @ E
        o = np.vstack(out)
        return np.abs(o - o_ref[0, :, 0]).max() / np.sqrt(np.mean(o_ref[0, :, 0] ** 2))

    bf16 = lambda x: torch.from_numpy(np.asarray(x, np.float64)).to(torch.bfloat16).double().numpy()
    assert run(lambda x: x) < 1e-12          # the factored product is exact algebra
    assert run(_round_tf32) < 2e-2 / 2       # measured 2.8e-3
    assert run(bf16) > 2e-2                  # measured 3.4e-2


def test_gdn2_preparation_products_need_fp16_operands():
    """GDN-2's preparation products after the Gram product (R = T (I - A^d), W,
    U' = R V, P^d V, Dt^T V) pass more roundings into the state than the other
    variants'.  With the carry operands in fp16 throughout, a 4096-token sequence
    at d = 128 keeps its final state within a quarter of the bf16 budget
    (2e-2 of RMS) when those products take fp16 operands.  With bf16 operands the
    state error triples, to three quarters of the budget on this one sequence;
    across the 64 sequences of the 1.3B layer it left the budget on the GPU."""
    T, d, C64 = 4096, 128, 64
    dd = make_inputs("gdn2", 1, T, 1, d, d, dtype=torch.bfloat16, seed=6)
    dd = {k: (None if v is None else v.double().numpy()) for k, v in dd.items()}
    o_ref, S_ref = oracle.forward("gdn2", **dd)
    q, k, v, lg, eb, ww = (dd[n][0, :, 0] for n in ("q", "k", "v", "log_g", "erase_b", "write_w"))
    f16 = lambda x: np.asarray(x).astype(np.float16).astype(np.float64)
    f32 = lambda x: np.asarray(x).astype(np.float32).astype(np.float64)
    bf16 = lambda x: torch.from_numpy(np.asarray(x, np.float64)).to(torch.bfloat16).double().numpy()

    def state_error(rp):
        S = np.zeros((d, d))
        for c0 in range(0, T, C64):
            sl = slice(c0, c0 + C64)
            K, V = k[sl], v[sl]
            gam = np.cumsum(lg[sl], axis=0)
            a, dw = eb[sl] * K, (ww[sl] - eb[sl]) * K
            Ad = np.tril((K * np.exp(gam)) @ (dw * np.exp(-gam)).T, -1)
            Tm = np.linalg.inv(np.eye(C64) + np.tril((K * np.exp(gam)) @ (a * np.exp(-gam)).T, -1))
            W = rp(Tm) @ rp(K * np.exp(gam))
            Up = rp(rp(Tm) @ rp(np.eye(C64) - Ad)) @ rp(V)
            fac = np.exp(gam[-1] - gam)
            DtV = rp(dw * fac).T @ rp(V)
            E = f32(f16(Up) - f16(W) @ f16(S))
            S = f32(np.exp(gam[-1])[:, None] * S + f16(a * fac).T @ f16(E) + f16(DtV))
        return np.abs(S - S_ref[0, 0]).max() / np.sqrt(np.mean(S_ref[0, 0] ** 2))

    e16, eb16 = state_error(f16), state_error(bf16)
    assert e16 < 2e-2 / 4                    # measured 4.9e-3
    assert eb16 > 2.5 * e16                  # measured 1.5e-2


def scalar_backward_as_built(q, k, v, beta, lg, s0, dO, dS_final, scale):
    """The scalar-decay backward in the form the CUDA path computes it (one
    sequence; q, k [T, dk], v [T, dv], beta and lg [T]).  Three passes:

    1. the forward carry, keeping each chunk's start state S0_c;
    2. the reverse carry, run as a forward carry over the chunks in reverse with
       the state X = dS (gradient of the chunk's end state) and per chunk
           Y = Kt X (the forward's -W S0 slot),  dE = R + Y with R = P^T dO,
           X <- Gamma_C X + F + (-W)^T dE  with F = Qg^T dO (scale included),
       the forward carry's steps with Kt in the -W operand, -W in the Kt operand,
       R in the U' slot and F as the extra state term;
    3. per chunk, from S0_c, dS_c, dE_c and the inputs, with D_tr = e^(g_t - g_r)
       (r <= t, g the chunk-local cumulative log decay), e = e^g, f = e^(g_C - g):
           G = K K^T, A = tril(Diag(beta) (D o G), -1), T = (I + A)^-1
           E = T Diag(beta) V - T Diag(beta e) K S0
           dk  = Diag(f) E dS^T + Diag(beta e) T^T dW + N1 K + N1^T K + N2^T Q
           dq  = scale Diag(e) dO S0^T + N2 K
           dv  = Diag(beta) T^T dE
           dW  = -dE S0^T,  dP = tril(dO E^T),  N2 = scale (dP o D)
           dT  = dE V^T Diag(beta) + dW K^T Diag(beta e)
           dA  = tril(-T^T dT T^T, -1),  N1 = Diag(beta) (dA o D)
           dbeta = rowsum(V o T^T dE) + rowsum(Diag(e) K o T^T dW) + rowsum(dA o D o G)
           dg_t  = sum_i [dq o Q + (Diag(beta e) T^T dW + N1 K) o K - Diag(f) E dS^T o K
                          - (N1^T K + N2^T Q) o K]_ti,  plus at the chunk's last token
                   sum(Diag(f) E dS^T o K) + e^(g_C) sum(dS o S0)
           dlog_g_t = sum_{s >= t in the chunk} dg_s."""
    T, dk = k.shape
    dv = v.shape[1]
    chunks = [slice(c0, min(T, c0 + C)) for c0 in range(0, T, C)]
    # 1. forward carry with chunk-start states
    S, S0s, per = s0.copy(), [], []
    for sl in chunks:
        K, Q, V, b = k[sl], q[sl], v[sl], beta[sl]
        n = K.shape[0]
        g = np.cumsum(lg[sl])
        D = np.tril(np.exp(g[:, None] - g[None, :]))
        e, f = np.exp(g), np.exp(g[-1] - g)
        A = np.tril(b[:, None] * D * (K @ K.T), -1)
        Tm = np.linalg.inv(np.eye(n) + A)
        W = Tm @ ((b * e)[:, None] * K)
        Up = Tm @ (b[:, None] * V)
        P = scale * D * (Q @ K.T)
        Qg = scale * e[:, None] * Q
        Kt = f[:, None] * K
        S0s.append(S.copy())
        per.append(dict(K=K, Q=Q, V=V, b=b, g=g, D=D, e=e, f=f, T=Tm, W=W, P=P, Qg=Qg, Kt=Kt))
        S = np.exp(g[-1]) * S + Kt.T @ (Up - W @ S)
    # 2. reverse carry
    X, dSs, dEs = dS_final.copy(), [None] * len(chunks), [None] * len(chunks)
    for c in reversed(range(len(chunks))):
        r, dOc = per[c], dO[chunks[c]]
        dSs[c] = X.copy()
        dE = r["P"].T @ dOc + r["Kt"] @ X
        dEs[c] = dE
        X = np.exp(r["g"][-1]) * X + r["Qg"].T @ dOc + (-r["W"]).T @ dE
    g_all = {"q": np.zeros_like(q), "k": np.zeros_like(k), "v": np.zeros_like(v),
             "beta": np.zeros(T), "log_g": np.zeros(T), "initial_state": X}
    # 3. chunk-local gradients
    for c, sl in enumerate(chunks):
        r, S0, dS, dE, dOc = per[c], S0s[c], dSs[c], dEs[c], dO[sl]
        K, Q, V, b, D, e, f, Tm = (r[x] for x in ("K", "Q", "V", "b", "D", "e", "f", "T"))
        n = K.shape[0]
        E = Tm @ (b[:, None] * V) - Tm @ ((b * e)[:, None] * K) @ S0
        X1 = f[:, None] * (E @ dS.T)
        dW = -dE @ S0.T
        tU, tW = Tm.T @ dE, Tm.T @ dW
        dP = np.tril(dOc @ E.T)
        dT = (dE @ V.T) * b[None, :] + (dW @ K.T) * (b * e)[None, :]
        dA = np.tril(-Tm.T @ dT @ Tm.T, -1)
        G = K @ K.T
        N1 = b[:, None] * dA * D
        N2 = scale * dP * D
        Y1 = (b * e)[:, None] * tW + N1 @ K
        Y2 = N1.T @ K + N2.T @ Q
        dq = scale * e[:, None] * (dOc @ S0.T) + N2 @ K
        g_all["q"][sl] = dq
        g_all["k"][sl] = X1 + Y1 + Y2
        g_all["v"][sl] = b[:, None] * tU
        g_all["beta"][sl] = (np.sum(V * tU, 1) + e * np.sum(K * tW, 1) + np.sum(dA * D * G, 1))
        dg = np.sum(dq * Q + (Y1 - X1 - Y2) * K, 1)
        dg[n - 1] += np.sum(X1 * K) + np.exp(r["g"][-1]) * np.sum(dS * S0)
        g_all["log_g"][sl] = np.cumsum(dg[::-1])[::-1]
    return g_all


@pytest.mark.parametrize("variant", ["deltanet", "gdn", "kla"])
def test_scalar_backward_as_built_matches_the_oracle(variant):
    B, T, H, dk, dv, scale = 1, 29, 1, 6, 5, 0.7
    d = make_inputs(variant, B, T, H, dk, dv, dtype=torch.float32, seed=11)
    d = {k: (None if v is None else v.double().numpy()) for k, v in d.items()}
    rng = np.random.default_rng(11)
    s0 = rng.standard_normal((B, H, dk, dv))
    dO = rng.standard_normal((B, T, H, dv))
    dS = rng.standard_normal((B, H, dk, dv))
    eps = 1e-6
    g_ref = oracle.backward(variant, d_o=dO, d_final=dS, initial_state=s0, scale=scale, eps=eps, **d)
    q, k, v = d["q"][0, :, 0], d["k"][0, :, 0], d["v"][0, :, 0]
    lg = np.zeros(T) if variant == "deltanet" else d["log_g"][0, :, 0]
    beta = d["beta"][0, :, 0]
    if variant == "kla":                       # the Kaczmarz step from eta and ||k||^2
        nk = np.sum(k * k, 1)
        beta = beta / (nk + eps)
    g = scalar_backward_as_built(q, k, v, beta, lg, s0[0, 0], dO[0, :, 0], dS[0, 0], scale)
    if variant == "kla":                       # chain rule through beta = eta / (||k||^2 + eps)
        dbeta = g["beta"]
        g["beta"] = dbeta / (nk + eps)
        g["k"] = g["k"] - (2 * dbeta * beta / (nk + eps))[:, None] * k
    for name in ("q", "k", "v", "beta"):
        np.testing.assert_allclose(g[name], g_ref[name][0, :, 0], rtol=0, atol=1e-10)
    np.testing.assert_allclose(g["initial_state"], g_ref["initial_state"][0, 0], rtol=0, atol=1e-10)
    if variant != "deltanet":
        np.testing.assert_allclose(g["log_g"], g_ref["log_g"][0, :, 0], rtol=0, atol=1e-10)


def channel_local_as_built(K, Q, V, b, lg, S0, dS, dO, scale):
    """KDA's chunk-local gradients in the form the CUDA path computes them (one
    chunk, lg [n, dk] the per-channel log decay, S0 the chunk's start state, dS
    its end-state gradient).  With g the chunk-local cumulative log decay per
    channel and a middle token m, the decay enters only through per-element
    factors on the K and Q operands and on the results:
        a = e^(g - g_m), bb = e^(g_m - g) (K o a)(K o bb)^T = the decayed Gram,
        e = e^g, f = e^(g_C - g) (both at most 1)
        A = tril(Diag(beta) (K o a)(K o bb)^T, -1),  T = (I + A)^-1
        W = T Diag(beta) (K o e),  E = T Diag(beta) V - W S0
        P = scale tril((Q o a)(K o bb)^T),  dE = (K o f) dS + P^T dO
        dW = -dE S0^T,  dP = tril(dO E^T),  dT = dE V^T Diag(beta) + dW (K o e)^T Diag(beta)
        dA = tril(-T^T dT T^T, -1),  N1 = Diag(beta) dA,  N2 = scale dP
        dk = f o E dS^T + e o Diag(beta) T^T dW + a o N1 (K o bb) + bb o N1^T (K o a) + bb o N2^T (Q o a)
        dq = e o scale dO S0^T + a o N2 (K o bb),  dv = Diag(beta) T^T dE
        dbeta = rowsum(V o T^T dE) + rowsum((K o e) o T^T dW) + rowsum(dA o (K o a)(K o bb)^T)
        dg = dq o Q + (e o Diag(beta) T^T dW + a o N1 (K o bb) - f o E dS^T
             - bb o N1^T (K o a) - bb o N2^T (Q o a)) o K,
             plus at the chunk's last token colsum(f o E dS^T o K) + e^(g_C) o rowsum(dS o S0)
        dlog_g_t = sum over s >= t of dg_s (per channel)."""
    n = K.shape[0]
    g = np.cumsum(lg, axis=0)
    # the token the CUDA path factors around: the middle one of a full chunk, the
    # last one of a shorter chunk (past which the padded decay stays flat)
    m = min(C // 2 - 1, n - 1)
    a, bb = np.exp(g - g[m]), np.exp(g[m] - g)
    e, f = np.exp(g), np.exp(g[-1] - g)
    Ka, Kb, Qa, Ke, Kf = K * a, K * bb, Q * a, K * e, K * f
    Gd = Ka @ Kb.T
    A = np.tril(b[:, None] * Gd, -1)
    Tm = np.linalg.inv(np.eye(n) + A)
    W = Tm @ (b[:, None] * Ke)
    E = Tm @ (b[:, None] * V) - W @ S0
    P = np.tril(scale * (Qa @ Kb.T))
    dE = Kf @ dS + P.T @ dO
    dW = -dE @ S0.T
    dP = np.tril(dO @ E.T)
    dT = (dE @ V.T) * b[None, :] + (dW @ Ke.T) * b[None, :]
    dA = np.tril(-Tm.T @ dT @ Tm.T, -1)
    N1 = b[:, None] * dA
    N2 = scale * dP
    tU, tW = Tm.T @ dE, Tm.T @ dW
    X1 = f * (E @ dS.T)
    Y1 = e * (b[:, None] * tW) + a * (N1 @ Kb)
    Y2 = bb * (N1.T @ Ka) + bb * (N2.T @ Qa)
    dq = e * (scale * dO @ S0.T) + a * (N2 @ Kb)
    dk = X1 + Y1 + Y2
    dv = b[:, None] * tU
    dbeta = np.sum(V * tU, 1) + np.sum(Ke * tW, 1) + np.sum(dA * Gd, 1)
    dg = dq * Q + (Y1 - X1 - Y2) * K
    dg[n - 1] += np.sum(X1 * K, 0) + np.exp(g[-1]) * np.sum(dS * S0, 1)
    return dq, dk, dv, dbeta, np.cumsum(dg[::-1], axis=0)[::-1]


@pytest.mark.parametrize("T", [27, 29])
def test_channel_backward_as_built_matches_the_oracle(T):
    """KDA: the forward and reverse carries in chunk form (as for the scalar
    decay, with Gamma_C a vector) and the channel-resolved local gradients,
    against the reverse-mode oracle (a last chunk of 3 or 5 tokens: factored
    around its last token or the full chunks' middle one)."""
    B, H, dk, dv, scale = 1, 1, 6, 5, 0.7
    d = make_inputs("kda", B, T, H, dk, dv, dtype=torch.float32, seed=13)
    d = {k: (None if v is None else v.double().numpy()) for k, v in d.items()}
    rng = np.random.default_rng(13)
    s0 = rng.standard_normal((B, H, dk, dv))
    dO = rng.standard_normal((B, T, H, dv))
    dSf = rng.standard_normal((B, H, dk, dv))
    g_ref = oracle.backward("kda", d_o=dO, d_final=dSf, initial_state=s0, scale=scale, **d)
    q, k, v, beta, lg = (d[x][0, :, 0] for x in ("q", "k", "v", "beta", "log_g"))
    dOn = dO[0, :, 0]
    chunks = [slice(c0, min(T, c0 + C)) for c0 in range(0, T, C)]
    # forward carry: chunk start states
    S, S0s = s0[0, 0].copy(), []
    for sl in chunks:
        K, V, bt = k[sl], v[sl], beta[sl]
        gam = np.cumsum(lg[sl], axis=0)
        n = K.shape[0]
        A = np.tril(bt[:, None] * ((K * np.exp(gam)) @ (K * np.exp(-gam)).T), -1)
        Tm = np.linalg.inv(np.eye(n) + A)
        E = Tm @ (bt[:, None] * V) - Tm @ (bt[:, None] * K * np.exp(gam)) @ S
        S0s.append(S.copy())
        S = np.exp(gam[-1])[:, None] * S + (K * np.exp(gam[-1] - gam)).T @ E
    # reverse carry: end-state gradients
    X, dSs = dSf[0, 0].copy(), [None] * len(chunks)
    for c in reversed(range(len(chunks))):
        sl = chunks[c]
        K, Q, bt = k[sl], q[sl], beta[sl]
        gam = np.cumsum(lg[sl], axis=0)
        n = K.shape[0]
        dSs[c] = X.copy()
        A = np.tril(bt[:, None] * ((K * np.exp(gam)) @ (K * np.exp(-gam)).T), -1)
        Tm = np.linalg.inv(np.eye(n) + A)
        W = Tm @ (bt[:, None] * K * np.exp(gam))
        P = np.tril(scale * ((Q * np.exp(gam)) @ (K * np.exp(-gam)).T))
        dE = (K * np.exp(gam[-1] - gam)) @ X + P.T @ dOn[sl]
        X = np.exp(gam[-1])[:, None] * X + scale * (Q * np.exp(gam)).T @ dOn[sl] - W.T @ dE
    np.testing.assert_allclose(X, g_ref["initial_state"][0, 0], rtol=0, atol=1e-10)
    for c, sl in enumerate(chunks):
        dq, dkk, dvv, db, dlg = channel_local_as_built(k[sl], q[sl], v[sl], beta[sl], lg[sl], S0s[c], dSs[c],
                                                       dOn[sl], scale)
        for name, x in (("q", dq), ("k", dkk), ("v", dvv), ("beta", db), ("log_g", dlg)):
            np.testing.assert_allclose(x, g_ref[name][0, sl, 0], rtol=0, atol=1e-10, err_msg=name)


def gdn2_local_as_built(K, Q, V, eb, ww, lg, S0, dS, dO, scale):
    """GDN-2's chunk-local gradients in the form a chunk-parallel kernel computes
    them (one chunk; eb, ww, lg [n, dk] the erase gate, write gate and log decay;
    S0 the chunk's start state, dS its end-state gradient).  With a = eb o k,
    d = (ww - eb) o k, the factors a_ = e^(g - g_m), bb = e^(g_m - g), e = e^g,
    f = e^(g_C - g) (middle token m as for KDA), and the factored operands
    Ka = K o a_, Qa = Q o a_, Ab = a o bb, Db = d o bb, Ke = K o e, Af = a o f,
    Df = d o f:
        A = tril(Ka Ab^T, -1),  A^d = tril(Ka Db^T, -1),  T = (I + A)^-1
        Y = V - A^d V,  W = T Ke,  E = T Y - W S0
        P^a = scale tril(Qa Ab^T),  P^d = scale tril(Qa Db^T)
        dE = Af dS + P^a^T dO,  dW = -dE S0^T,  tU = T^T dE,  tW = T^T dW
        dT = dE Y^T + dW Ke^T,  dA = tril(-T^T dT T^T, -1),  dA^d = -tril(tU V^T, -1)
        N2a = scale tril(dO E^T),  N2d = scale tril(dO V^T)
        dv = tU - A^d^T tU + P^d^T dO + Df dS
        dKa = dA Ab + dA^d Db,  dAb = dA^T Ka + N2a^T Qa,  dDb = dA^d^T Ka + N2d^T Qa
        dQa = N2a Ab + N2d Db,  dKe = tW,  dQe = scale dO S0^T,  dAf = E dS^T,  dDf = V dS^T
        dq = a_ o dQa + e o dQe,  da = bb o dAb + f o dAf,  dd = bb o dDb + f o dDf
        dk = a_ o dKa + e o dKe + eb o da + (ww - eb) o dd
        d eb = k o (da - dd),  d ww = k o dd
        dg = dKa o Ka + dQa o Qa - dAb o Ab - dDb o Db + dKe o Ke + dQe o (Q o e)
             - dAf o Af - dDf o Df, plus colsum(dAf o Af + dDf o Df) + e^(g_C) o rowsum(dS o S0)
             at the chunk's last token; d log g = per-channel suffix sums of dg."""
    n = K.shape[0]
    g = np.cumsum(lg, axis=0)
    m = min(C // 2 - 1, n - 1)
    a_, bb = np.exp(g - g[m]), np.exp(g[m] - g)
    e, f = np.exp(g), np.exp(g[-1] - g)
    a, d = eb * K, (ww - eb) * K
    Ka, Qa, Ab, Db, Ke, Af, Df = K * a_, Q * a_, a * bb, d * bb, K * e, a * f, d * f
    A = np.tril(Ka @ Ab.T, -1)
    Ad = np.tril(Ka @ Db.T, -1)
    Tm = np.linalg.inv(np.eye(n) + A)
    Y = V - Ad @ V
    W = Tm @ Ke
    E = Tm @ Y - W @ S0
    Pa = scale * np.tril(Qa @ Ab.T)
    Pd = scale * np.tril(Qa @ Db.T)
    dE = Af @ dS + Pa.T @ dO
    dW = -dE @ S0.T
    tU, tW = Tm.T @ dE, Tm.T @ dW
    dT = dE @ Y.T + dW @ Ke.T
    dA = np.tril(-Tm.T @ dT @ Tm.T, -1)
    dAd = -np.tril(tU @ V.T, -1)
    N2a, N2d = scale * np.tril(dO @ E.T), scale * np.tril(dO @ V.T)
    dv = tU - Ad.T @ tU + Pd.T @ dO + Df @ dS
    dKa = dA @ Ab + dAd @ Db
    dAb = dA.T @ Ka + N2a.T @ Qa
    dDb = dAd.T @ Ka + N2d.T @ Qa
    dQa = N2a @ Ab + N2d @ Db
    dKe, dQe, dAf, dDf = tW, scale * dO @ S0.T, E @ dS.T, V @ dS.T
    dq = a_ * dQa + e * dQe
    da, dd = bb * dAb + f * dAf, bb * dDb + f * dDf
    dk = a_ * dKa + e * dKe + eb * da + (ww - eb) * dd
    deb, dww = K * (da - dd), K * dd
    dg = (dKa * Ka + dQa * Qa - dAb * Ab - dDb * Db + dKe * Ke + dQe * (Q * e) - dAf * Af - dDf * Df)
    dg[n - 1] += np.sum(dAf * Af + dDf * Df, 0) + np.exp(g[-1]) * np.sum(dS * S0, 1)
    return dq, dk, dv, deb, dww, np.cumsum(dg[::-1], axis=0)[::-1]


@pytest.mark.parametrize("T", [27, 29])
def test_gdn2_backward_as_built_matches_the_oracle(T):
    """GDN-2: the forward carry in chunk form (E the residual, the record's Ã = a o f),
    the reverse carry dE = Ã dS + P^a^T dO, dS0 = Diag(e^g_C) dS + scale (Q o e)^T dO - W^T dE
    (the state-free terms P^d V and D̃^T V do not enter it), and the chunk-local
    gradients above, against the reverse-mode oracle."""
    B, H, dk, dv, scale = 1, 1, 6, 5, 0.7
    d = make_inputs("gdn2", B, T, H, dk, dv, dtype=torch.float32, seed=17)
    d = {k: (None if v is None else v.double().numpy()) for k, v in d.items()}
    rng = np.random.default_rng(17)
    s0 = rng.standard_normal((B, H, dk, dv))
    dO = rng.standard_normal((B, T, H, dv))
    dSf = rng.standard_normal((B, H, dk, dv))
    g_ref = oracle.backward("gdn2", d_o=dO, d_final=dSf, initial_state=s0, scale=scale, **d)
    q, k, v, lg, eb, ww = (d[x][0, :, 0] for x in ("q", "k", "v", "log_g", "erase_b", "write_w"))
    dOn = dO[0, :, 0]
    chunks = [slice(c0, min(T, c0 + C)) for c0 in range(0, T, C)]

    def chunk_ops(sl):
        K, Q = k[sl], q[sl]
        gam = np.cumsum(lg[sl], axis=0)
        a, dd = eb[sl] * K, (ww[sl] - eb[sl]) * K
        n = K.shape[0]
        G = lambda X, Y: (X * np.exp(gam)) @ (Y * np.exp(-gam)).T
        A, Ad = np.tril(G(K, a), -1), np.tril(G(K, dd), -1)
        Tm = np.linalg.inv(np.eye(n) + A)
        W = Tm @ (K * np.exp(gam))
        Pa = scale * np.tril(G(Q, a))
        fac = np.exp(gam[-1] - gam)
        return gam, a, dd, Ad, Tm, W, Pa, fac

    S, S0s = s0[0, 0].copy(), []
    for sl in chunks:   # forward carry: chunk start states
        gam, a, dd, Ad, Tm, W, Pa, fac = chunk_ops(sl)
        E = Tm @ (v[sl] - Ad @ v[sl]) - W @ S
        S0s.append(S.copy())
        S = np.exp(gam[-1])[:, None] * S + (a * fac).T @ E + (dd * fac).T @ v[sl]
    X, dSs = dSf[0, 0].copy(), [None] * len(chunks)
    for c in reversed(range(len(chunks))):   # reverse carry: end-state gradients
        sl = chunks[c]
        gam, a, dd, Ad, Tm, W, Pa, fac = chunk_ops(sl)
        dSs[c] = X.copy()
        dE = (a * fac) @ X + Pa.T @ dOn[sl]
        X = np.exp(gam[-1])[:, None] * X + scale * (q[sl] * np.exp(gam)).T @ dOn[sl] - W.T @ dE
    np.testing.assert_allclose(X, g_ref["initial_state"][0, 0], rtol=0, atol=1e-10)
    names = ("q", "k", "v", "erase_b", "write_w", "log_g")
    for c, sl in enumerate(chunks):
        got = gdn2_local_as_built(k[sl], q[sl], v[sl], eb[sl], ww[sl], lg[sl], S0s[c], dSs[c], dOn[sl], scale)
        for name, x in zip(names, got):
            np.testing.assert_allclose(x, g_ref[name][0, sl, 0], rtol=0, atol=1e-10, err_msg=f"{name} chunk {c}")
