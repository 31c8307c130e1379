"""Pins for the fp64 oracle, checked against facts the pages and the mathematics fix.

None of these re-types the oracle's recurrence.  Each pin is an independent
statement:

* brute force: the closed form of the linear recurrence, built from explicit
  d_k x d_k transition matrices M_t = (I - a_t k_t^T) Diag(g_t) and their
  products, on T <= 8;
* the Kaczmarz projection ("Kaczmarz Linear Attention", theoretical derivation
  and key properties): with eta = 1, eps = 0 the new state satisfies
  S_t^T k_t = v_t, and the change S_t - S~ is the minimum-Frobenius-norm
  solution of that constraint (checked with numpy's least-squares routine);
* the reductions of "Gated DeltaNet-2" (what is new): tied erase/write gates
  give KDA, and a channel-constant decay gives Gated DeltaNet;
* beta = 0 leaves only the decay (closed form with cumulative products);
* the delta rule with one-hot keys and beta = 1 is a key -> value table
  (subtract the readout, then write: an overwrite);
* resume, decode = forward, linearity in v, column independence, q scale.

``test_mutants_are_caught`` rebuilds the oracle with planted mistakes and
checks that some pin fails for each.
"""
import numpy as np
import pytest

import oracle

VARS = ["deltanet", "gdn", "kda", "gdn2", "kla"]


# --------------------------------------------------------------------------- helpers
def rand_inputs(variant, B, T, H, dk, dv, seed, unit_keys=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    beta = rng.uniform(0.05, 1.0, (B, T, H))
    if variant in ("kda", "gdn2"):
        log_g = -rng.uniform(0.0, 0.7, (B, T, H, dk))
    elif variant in ("gdn", "kla"):
        log_g = -rng.uniform(0.0, 0.7, (B, T, H))
    else:
        log_g = None
    erase_b = write_w = None
    if variant == "gdn2":
        erase_b = rng.uniform(0.0, 1.0, (B, T, H, dk))
        write_w = rng.uniform(0.0, 1.0, (B, T, H, dk))
        beta = None
    S0 = rng.standard_normal((B, H, dk, dv))
    return dict(q=q, k=k, v=v, beta=beta, log_g=log_g, erase_b=erase_b, write_w=write_w), S0


def brute_force(variant, q, k, v, beta, log_g, erase_b, write_w, S0, eps=1e-6, scale=1.0):
    """Closed form S_t = M_t..M_1 S0 + sum_s M_t..M_{s+1} c_s v_s^T with explicit matrices."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    S_T = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            Ms, Cs = [], []
            for t in range(T):
                kt = k[b, t, h]
                if variant in ("kda", "gdn2"):
                    g = np.exp(log_g[b, t, h])
                elif variant in ("gdn", "kla"):
                    g = np.full(dk, np.exp(log_g[b, t, h]))
                else:
                    g = np.ones(dk)
                if variant == "gdn2":
                    a, c = erase_b[b, t, h] * kt, write_w[b, t, h] * kt
                elif variant == "kla":
                    step = beta[b, t, h] / (kt @ kt + eps)
                    a = c = step * kt
                else:
                    a = c = beta[b, t, h] * kt
                Ms.append((np.eye(dk) - np.outer(a, kt)) @ np.diag(g))
                Cs.append(np.outer(c, v[b, t, h]))
            for t in range(T):
                P = np.eye(dk)
                for r in range(t, -1, -1):
                    P = P @ Ms[r]
                St = P @ S0[b, h]
                for s in range(t + 1):
                    Pt = np.eye(dk)
                    for r in range(t, s, -1):
                        Pt = Pt @ Ms[r]
                    St = St + Pt @ Cs[s]
                o[b, t, h] = St.T @ (scale * q[b, t, h])
                if t == T - 1:
                    S_T[b, h] = St
    return o, S_T


def rel(a, b):
    return np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300)


# --------------------------------------------------------------------------- pins
def pin_brute_force(variant, mutant=0, dk=5, dv=3, T=7):
    inp, S0 = rand_inputs(variant, 2, T, 2, dk, dv, seed=11 + T)
    o, S = oracle.forward(variant, **inp, initial_state=S0, eps=1e-6, scale=0.8, mutant=mutant)
    ob, Sb = brute_force(variant, **inp, S0=S0, eps=1e-6, scale=0.8)
    assert rel(o, ob) < 1e-12, rel(o, ob)
    assert rel(S, Sb) < 1e-12, rel(S, Sb)


def pin_kla_projection(mutant=0, decay=True, dk=6, dv=4):
    """eta = 1, eps = 0: the new state reproduces v_t at k_t (q_t = k_t reads it)."""
    inp, S0 = rand_inputs("kla", 1, 9, 3, dk, dv, seed=5)
    inp["beta"][:] = 1.0
    if not decay:
        inp["log_g"][:] = 0.0
    inp["q"] = inp["k"].copy()
    o, _ = oracle.forward("kla", **inp, initial_state=S0, eps=0.0, scale=1.0, mutant=mutant)
    assert rel(o, inp["v"]) < 1e-11, rel(o, inp["v"])


def pin_kla_min_norm(mutant=0, dk=6, dv=4):
    """S_t - S~ is the minimum-norm solution of (S~ + D)^T k_t = v_t (lstsq)."""
    inp, S0 = rand_inputs("kla", 1, 4, 1, dk, dv, seed=9)
    inp["beta"][:] = 1.0
    t = 3
    head = {n: (None if a is None else a[:, :t]) for n, a in inp.items()}
    _, S_prev = oracle.forward("kla", **head, initial_state=S0, eps=0.0, mutant=mutant)
    full = {n: (None if a is None else a[:, :t + 1]) for n, a in inp.items()}
    _, S_t = oracle.forward("kla", **full, initial_state=S0, eps=0.0, mutant=mutant)
    S_tilde = np.exp(inp["log_g"][0, t, 0]) * S_prev[0, 0]
    kt, vt = inp["k"][0, t, 0], inp["v"][0, t, 0]
    rhs = vt - S_tilde.T @ kt
    D_min, *_ = np.linalg.lstsq(kt[None, :], rhs[None, :], rcond=None)
    assert rel(S_t[0, 0] - S_tilde, D_min) < 1e-11


def pin_kda_equals_gdn(mutant=0, dk=5, dv=4):
    inp, S0 = rand_inputs("gdn", 2, 8, 2, dk, dv, seed=3)
    o1, S1 = oracle.forward("gdn", **inp, initial_state=S0, mutant=mutant)
    inp_c = dict(inp, log_g=np.repeat(inp["log_g"][..., None], dk, axis=-1))
    o2, S2 = oracle.forward("kda", **inp_c, initial_state=S0, mutant=mutant)
    assert rel(o2, o1) < 1e-13 and rel(S2, S1) < 1e-13


def pin_gdn2_tied_equals_kda(mutant=0, dk=5, dv=4):
    inp, S0 = rand_inputs("kda", 2, 8, 2, dk, dv, seed=4)
    o1, S1 = oracle.forward("kda", **inp, initial_state=S0, mutant=mutant)
    tied = np.repeat(inp["beta"][..., None], dk, axis=-1)
    inp2 = dict(inp, beta=None, erase_b=tied, write_w=tied.copy())
    o2, S2 = oracle.forward("gdn2", **inp2, initial_state=S0, mutant=mutant)
    assert rel(o2, o1) < 1e-12 and rel(S2, S1) < 1e-12


def pin_beta_zero_decay_only(variant, mutant=0, dk=4, dv=4):
    inp, S0 = rand_inputs(variant, 1, 6, 2, dk, dv, seed=8)
    if variant == "gdn2":
        inp["erase_b"][:] = 0.0
        inp["write_w"][:] = 0.0
    else:
        inp["beta"][:] = 0.0
    o, S = oracle.forward(variant, **inp, initial_state=S0, mutant=mutant)
    T, H = 6, 2
    if variant in ("kda", "gdn2"):
        cum = np.cumprod(np.exp(inp["log_g"][0]), axis=0)            # [T,H,dk]
    elif variant in ("gdn", "kla"):
        cum = np.repeat(np.cumprod(np.exp(inp["log_g"][0]), axis=0)[..., None], dk, -1)
    else:
        cum = np.ones((T, H, dk))
    for t in range(T):
        for h in range(H):
            St = cum[t, h][:, None] * S0[0, h]
            assert rel(o[0, t, h], St.T @ inp["q"][0, t, h]) < 1e-12
    assert rel(S[0], cum[-1][:, :, None] * S0[0]) < 1e-12


def pin_delta_key_value_table(mutant=0, dk=6, dv=3):
    """One-hot keys, beta = 1, no decay: the state is a key -> value table."""
    rng = np.random.default_rng(21)
    keys = [2, 0, 2, 5, 1, 0, 2, 4, 5, 5]
    T = len(keys)
    k = np.zeros((1, T, 1, dk))
    for t, j in enumerate(keys):
        k[0, t, 0, j] = 1.0
    v = rng.standard_normal((1, T, 1, dv))
    beta = np.ones((1, T, 1))
    q = k.copy()                               # read back the key just written
    o, S = oracle.forward("deltanet", q, k, v, beta=beta, mutant=mutant)
    assert rel(o, v) < 1e-14
    table = np.zeros((dk, dv))
    for t, j in enumerate(keys):
        table[j] = v[0, t, 0]
    assert np.max(np.abs(S[0, 0] - table)) < 1e-14


def pin_resume(variant, mutant=0, dk=4, dv=4):
    inp, S0 = rand_inputs(variant, 2, 9, 2, dk, dv, seed=13)
    o, S = oracle.forward(variant, **inp, initial_state=S0, mutant=mutant)
    a = {n: (None if x is None else x[:, :4]) for n, x in inp.items()}
    b = {n: (None if x is None else x[:, 4:]) for n, x in inp.items()}
    oa, Sa = oracle.forward(variant, **a, initial_state=S0, mutant=mutant)
    ob, Sb = oracle.forward(variant, **b, initial_state=Sa, mutant=mutant)
    assert np.array_equal(np.concatenate([oa, ob], axis=1), o)
    assert np.array_equal(Sb, S)


def pin_decode_equals_forward(variant, mutant=0, dk=4, dv=4):
    inp, S0 = rand_inputs(variant, 3, 5, 2, dk, dv, seed=17)
    o, S = oracle.forward(variant, **inp, initial_state=S0, mutant=mutant)
    state = S0.copy()
    for t in range(5):
        step = {n: (None if x is None else x[:, t]) for n, x in inp.items()}
        ot, state = oracle.decode_step(variant, step["q"], step["k"], step["v"], state,
                                       beta=step["beta"], log_g=step["log_g"],
                                       erase_b=step["erase_b"], write_w=step["write_w"],
                                       mutant=mutant)
        assert np.array_equal(ot, o[:, t])
    assert np.array_equal(state, S)


# --------------------------------------------------------------------------- tests
@pytest.mark.parametrize("variant", VARS)
@pytest.mark.parametrize("T", [1, 5, 8])
def test_brute_force(variant, T):
    pin_brute_force(variant, T=T)


@pytest.mark.parametrize("decay", [True, False])
def test_kla_projection(decay):
    pin_kla_projection(decay=decay)


def test_kla_min_norm():
    pin_kla_min_norm()


def test_kla_relaxation_scales_the_step():
    """The relaxation gate eta scales the projection step linearly (eps = 0)."""
    inp, S0 = rand_inputs("kla", 1, 1, 1, 6, 4, seed=31)
    _, S_prev = oracle.forward("kla", **{n: (None if a is None else a[:, :0]) for n, a in inp.items()},
                               initial_state=S0, eps=0.0)
    inp1 = dict(inp, beta=np.ones_like(inp["beta"]))
    inp2 = dict(inp, beta=np.full_like(inp["beta"], 0.3))
    _, S1 = oracle.forward("kla", **inp1, initial_state=S0, eps=0.0)
    _, S2 = oracle.forward("kla", **inp2, initial_state=S0, eps=0.0)
    S_tilde = np.exp(inp["log_g"][0, 0, 0]) * S0[0, 0]
    assert rel(S2[0, 0] - S_tilde, 0.3 * (S1[0, 0] - S_tilde)) < 1e-12


def test_kda_channel_constant_equals_gdn():
    pin_kda_equals_gdn()


def test_gdn2_tied_gates_equal_kda():
    pin_gdn2_tied_equals_kda()


def test_gdn2_tied_channel_constant_equals_gdn():
    inp, S0 = rand_inputs("gdn", 1, 8, 2, 5, 3, seed=6)
    o1, S1 = oracle.forward("gdn", **inp, initial_state=S0)
    tied = np.repeat(inp["beta"][..., None], 5, axis=-1)
    lg = np.repeat(inp["log_g"][..., None], 5, axis=-1)
    o2, S2 = oracle.forward("gdn2", inp["q"], inp["k"], inp["v"], log_g=lg, erase_b=tied,
                            write_w=tied.copy(), initial_state=S0)
    assert rel(o2, o1) < 1e-12 and rel(S2, S1) < 1e-12


def test_deltanet_is_gdn_without_decay():
    inp, S0 = rand_inputs("gdn", 1, 8, 2, 4, 4, seed=7)
    o1, S1 = oracle.forward("deltanet", **dict(inp, log_g=None), initial_state=S0)
    o2, S2 = oracle.forward("gdn", **dict(inp, log_g=np.zeros_like(inp["log_g"])), initial_state=S0)
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


@pytest.mark.parametrize("variant", VARS)
def test_beta_zero_decay_only(variant):
    pin_beta_zero_decay_only(variant)


def test_delta_rule_key_value_table():
    pin_delta_key_value_table()


@pytest.mark.parametrize("variant", VARS)
def test_resume(variant):
    pin_resume(variant)


@pytest.mark.parametrize("variant", VARS)
def test_decode_equals_forward(variant):
    pin_decode_equals_forward(variant)


@pytest.mark.parametrize("variant", VARS)
def test_linear_in_v_from_zero_state(variant):
    inp, _ = rand_inputs(variant, 1, 7, 2, 4, 3, seed=19)
    v2 = np.random.default_rng(1).standard_normal(inp["v"].shape)
    oa, Sa = oracle.forward(variant, **inp)
    ob, Sb = oracle.forward(variant, **dict(inp, v=v2))
    oc, Sc = oracle.forward(variant, **dict(inp, v=inp["v"] + 2.0 * v2))
    assert rel(oc, oa + 2.0 * ob) < 1e-12 and rel(Sc, Sa + 2.0 * Sb) < 1e-12


@pytest.mark.parametrize("variant", VARS)
def test_columns_independent(variant):
    inp, S0 = rand_inputs(variant, 1, 6, 2, 4, 6, seed=23)
    o, S = oracle.forward(variant, **inp, initial_state=S0)
    for lo, hi in ((0, 2), (2, 6)):
        part = dict(inp, v=np.ascontiguousarray(inp["v"][..., lo:hi]))
        op, Sp = oracle.forward(variant, **part, initial_state=np.ascontiguousarray(S0[..., lo:hi]))
        assert np.array_equal(op, o[..., lo:hi]) and np.array_equal(Sp, S[..., lo:hi])


def test_q_scale_is_linear():
    inp, S0 = rand_inputs("kda", 1, 6, 2, 4, 4, seed=29)
    o1, S1 = oracle.forward("kda", **inp, initial_state=S0, scale=1.0)
    o2, S2 = oracle.forward("kda", **inp, initial_state=S0, scale=0.125)
    assert rel(o2, 0.125 * o1) < 1e-15 and np.array_equal(S1, S2)


def test_bad_arguments_rejected():
    inp, _ = rand_inputs("gdn", 1, 2, 1, 4, 4, seed=1)
    with pytest.raises(ValueError):
        oracle.forward("gdn", **dict(inp, log_g=None))
    with pytest.raises(ValueError):
        oracle.forward("nope", **inp)


MUTANTS = {
    1: "readout added instead of subtracted",
    2: "readout taken before the decay",
    3: "state transposed in the key readout",
    4: "output read before the write",
    5: "Kaczmarz step divides by the norm, not its square",
    6: "GDN-2 erase and write gates swapped",
    7: "decay applied after the write",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_mutants_are_caught(mutant):
    """Each planted mistake must make at least one pin fail (dk == dv keeps mutant 3 in bounds)."""
    pins = []
    for var in VARS:
        pins.append(lambda var=var: pin_brute_force(var, mutant, dk=4, dv=4, T=6))
        pins.append(lambda var=var: pin_beta_zero_decay_only(var, mutant))
    pins += [
        lambda: pin_kla_projection(mutant, dk=4, dv=4),
        lambda: pin_kla_min_norm(mutant, dk=4, dv=4),
        lambda: pin_kda_equals_gdn(mutant, dk=4, dv=4),
        lambda: pin_gdn2_tied_equals_kda(mutant, dk=4, dv=4),
        lambda: pin_delta_key_value_table(mutant, dk=6, dv=6),
    ]
    failures = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failures += 1
    assert failures > 0, f"no pin caught mutant {mutant}: {MUTANTS[mutant]}"


def test_raw_inputs_follow_the_recipe():
    """inputs.make_raw_inputs draws what make_inputs draws, and transform_raw
    applies the recipe's transforms: the two agree up to the I/O rounding."""
    import torch

    from gated_delta_rule_forward_b200.inputs import make_inputs, make_raw_inputs, transform_raw
    for variant in ("deltanet", "gdn", "kda", "gdn2", "kla"):
        ref = make_inputs(variant, 2, 9, 3, 128, 64, dtype=torch.float32, seed=5)
        got = transform_raw(variant, make_raw_inputs(variant, 2, 9, 3, 128, 64, dtype=torch.float32, seed=5))
        for name, x in ref.items():
            if x is None:
                assert got[name] is None, name
                continue
            assert torch.allclose(got[name].float(), x, rtol=1e-5, atol=1e-6), (variant, name)
