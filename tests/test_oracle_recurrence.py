"""Pins of the oracle's recurrence (quantization disabled, 32-bit state).

The recurrence is "Preserving Updates in Low-Bit Recurrent State
Quantization", Table 1:  S_t = A_t S_{t-1} + B_t,  o_t = S_t^T q_t.
Each kind is checked against something other than the recurrence itself:

- RetNet / Mamba2 / GLA: the closed form S_T = sum_t (prod_{s>t} A_s) k_t v_t^T
  evaluated in fp64, within the forward-error bound of the fp32 recursion;
- GDN: the delta-rule identities S_t^T k_t = (1-beta) alpha S_{t-1}^T k_t + beta v_t
  for unit keys, the Hebbian closed form for orthonormal keys, pure decay
  at beta = 0;
- GLA with a constant alpha vector reduces bit-exactly to Mamba2;
- the canonical summation order, by hand-worked cancellation examples.
"""
import numpy as np
import pytest

U32 = 2.0 ** -24


def _run(orc, kind, T, dk, dv, q, k, v, alpha=None, beta=None, gamma=1 - 2 ** -5):
    cfg = orc.Config(dk, dv, kind, 0, gamma=gamma)
    st = orc.State(cfg, [32])
    outs = []
    states = []
    for t in range(T):
        o = st.step(q[t], k[t], v[t],
                    None if alpha is None else alpha[t],
                    None if beta is None else np.array([beta[t]], np.float32))
        outs.append(o[0].copy())
        states.append(st.S[0].copy())
    return np.array(outs), np.array(states)


def _inputs(rng, T, dk, dv):
    q = (rng.standard_normal((T, dk)) / 8).astype(np.float32)
    k = (rng.standard_normal((T, dk)) / 8).astype(np.float32)
    v = rng.standard_normal((T, dv)).astype(np.float32)
    return q, k, v


def _check_closed_form(S32, S64, decay_weights, k, v, T):
    # |fl(S_T) - S_T| <= 3 T u sum_t w_t |k_t| |v_t|^T   (elementwise)
    bound = 3 * T * U32 * np.einsum("t,ti,tj->ij", decay_weights, np.abs(k.astype(np.float64)),
                                    np.abs(v.astype(np.float64)))
    err = np.abs(S32.astype(np.float64) - S64)
    assert np.all(err <= bound + 1e-30), (err / (bound + 1e-30)).max()
    # and the match is not vacuous: the state is far larger than the bound
    assert np.abs(S64).max() > 1e3 * bound.max()


def test_retnet_closed_form(orc):
    rng = np.random.default_rng(10)
    T, dk, dv = 256, 64, 64
    gamma = np.float32(1 - 2 ** -5)
    q, k, v = _inputs(rng, T, dk, dv)
    outs, states = _run(orc, orc.RETNET, T, dk, dv, q, k, v, gamma=gamma)
    w = float(gamma) ** (T - 1 - np.arange(T))            # gamma^(T-t)
    S64 = np.einsum("t,ti,tj->ij", w, k.astype(np.float64), v.astype(np.float64))
    _check_closed_form(states[-1], S64, w, k, v, T)
    o64 = S64.T @ q[-1].astype(np.float64)
    assert np.allclose(outs[-1], o64, rtol=1e-4, atol=1e-5 * np.abs(o64).max())


def test_mamba2_closed_form(orc):
    rng = np.random.default_rng(11)
    T, dk, dv = 200, 128, 64
    q, k, v = _inputs(rng, T, dk, dv)
    alpha = (1 / (1 + np.exp(rng.standard_normal(T)))).astype(np.float32)[:, None]
    outs, states = _run(orc, orc.MAMBA2, T, dk, dv, q, k, v, alpha=alpha)
    a64 = alpha[:, 0].astype(np.float64)
    w = np.array([np.prod(a64[t + 1:]) for t in range(T)])
    S64 = np.einsum("t,ti,tj->ij", w, k.astype(np.float64), v.astype(np.float64))
    _check_closed_form(states[-1], S64, w, k, v, T)


def test_gla_closed_form(orc):
    rng = np.random.default_rng(12)
    T, dk, dv = 200, 64, 128
    q, k, v = _inputs(rng, T, dk, dv)
    alpha = ((1 / (1 + np.exp(-(2 + rng.standard_normal((T, dk)))))) ** (1 / 16)).astype(np.float32)
    outs, states = _run(orc, orc.GLA, T, dk, dv, q, k, v, alpha=alpha)
    a64 = alpha.astype(np.float64)
    # row-wise decay: W[t, i] = prod_{s>t} alpha_{s,i}
    W = np.array([np.prod(a64[t + 1:], axis=0) for t in range(T)])
    S64 = np.einsum("ti,ti,tj->ij", W, k.astype(np.float64), v.astype(np.float64))
    bound = 3 * T * U32 * np.einsum("ti,ti,tj->ij", W, np.abs(k.astype(np.float64)),
                                    np.abs(v.astype(np.float64)))
    err = np.abs(states[-1].astype(np.float64) - S64)
    assert np.all(err <= bound)
    assert np.abs(S64).max() > 1e3 * bound.max()
    o64 = states[-1].astype(np.float64).T @ q[-1].astype(np.float64)
    assert np.allclose(outs[-1], o64, rtol=1e-4, atol=1e-5 * np.abs(o64).max())


def test_gla_constant_alpha_equals_mamba2(orc):
    rng = np.random.default_rng(13)
    T, dk, dv = 20, 64, 64
    q, k, v = _inputs(rng, T, dk, dv)
    al = rng.uniform(0.5, 1.0, T).astype(np.float32)
    o1, s1 = _run(orc, orc.MAMBA2, T, dk, dv, q, k, v, alpha=al[:, None])
    o2, s2 = _run(orc, orc.GLA, T, dk, dv, q, k, v, alpha=np.repeat(al[:, None], dk, 1))
    assert np.array_equal(s1.view(np.uint32), s2.view(np.uint32))
    assert np.array_equal(o1.view(np.uint32), o2.view(np.uint32))


def _unit(x):
    x = x.astype(np.float64)
    return (x / np.linalg.norm(x, axis=-1, keepdims=True)).astype(np.float32)


def test_gdn_delta_rule_identity(orc):
    # With |k_t| = 1:  S_t^T k_t = (1 - beta) (alpha S_{t-1})^T k_t + beta v_t.
    # beta = 1 is the overwrite case S_t^T k_t = v_t.
    rng = np.random.default_rng(14)
    T, dk, dv = 60, 128, 128
    q = _unit(rng.standard_normal((T, dk)))
    k = _unit(rng.standard_normal((T, dk)))
    v = rng.standard_normal((T, dv)).astype(np.float32)
    alpha = (1 / (1 + np.exp(-(3 + rng.standard_normal(T))))).astype(np.float32)[:, None]
    beta = (1 / (1 + np.exp(-rng.standard_normal(T)))).astype(np.float32)
    beta[::7] = 1.0
    outs, states = _run(orc, orc.GDN, T, dk, dv, q, k, v, alpha=alpha, beta=beta)
    prev = np.zeros((dk, dv))
    for t in range(T):
        S = states[t].astype(np.float64)
        kt = k[t].astype(np.float64)
        kk = kt @ kt
        lhs = S.T @ kt
        rhs = (1 - beta[t] * kk) * float(alpha[t, 0]) * (prev.T @ kt) + beta[t] * kk * v[t]
        assert np.allclose(lhs, rhs, rtol=0, atol=2e-5 * (1 + np.abs(rhs).max())), t
        o64 = S.T @ q[t].astype(np.float64)
        assert np.allclose(outs[t], o64, rtol=0, atol=1e-5 * (1 + np.abs(o64).max()))
        prev = S


def test_gdn_orthonormal_keys_closed_form(orc):
    # Orthonormal keys make (alpha S_{t-1})^T k_t vanish, so the delta rule
    # reduces to S_T = sum_t (prod_{s>t} alpha_s) beta_t k_t v_t^T.
    rng = np.random.default_rng(15)
    dk, dv, T = 64, 64, 48
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm.T[:T].astype(np.float32)
    q = _unit(rng.standard_normal((T, dk)))
    v = rng.standard_normal((T, dv)).astype(np.float32)
    alpha = rng.uniform(0.9, 1.0, T).astype(np.float32)[:, None]
    beta = rng.uniform(0.1, 1.0, T).astype(np.float32)
    _, states = _run(orc, orc.GDN, T, dk, dv, q, k, v, alpha=alpha, beta=beta)
    a64 = alpha[:, 0].astype(np.float64)
    w = np.array([np.prod(a64[t + 1:]) for t in range(T)]) * beta.astype(np.float64)
    S64 = np.einsum("t,ti,tj->ij", w, k.astype(np.float64), v.astype(np.float64))
    # the float32 keys are orthonormal only to ~1e-7, hence a loose bound
    assert np.allclose(states[-1], S64, rtol=0, atol=1e-5 * np.abs(S64).max())


def test_gdn_beta_zero_is_pure_decay(orc):
    rng = np.random.default_rng(16)
    dk, dv, T = 64, 64, 12
    q = _unit(rng.standard_normal((T, dk)))
    k = _unit(rng.standard_normal((T, dk)))
    v = rng.standard_normal((T, dv)).astype(np.float32)
    alpha = rng.uniform(0.8, 1.0, T).astype(np.float32)[:, None]
    beta = np.ones(T, np.float32)
    beta[6:] = 0.0
    _, states = _run(orc, orc.GDN, T, dk, dv, q, k, v, alpha=alpha, beta=beta)
    S = states[5].copy()
    for t in range(6, T):
        S = S * alpha[t, 0]                  # one fp32 product per element
        assert np.array_equal(states[t], S)


# -------------------------------------------------------------- canonical order
def test_canon_dot_integers_exact(orc):
    rng = np.random.default_rng(17)
    for n in (8, 16, 64, 128, 256):
        a = rng.integers(-1000, 1000, n)
        b = rng.integers(-1000, 1000, n)
        assert orc.canon_dot(a, b) == float(np.dot(a, b))


def test_canon_dot_block_is_ascending_fma_chain(orc):
    # Block of 8 rows: 2^24 first, then seven 1s.  Ascending: 2^24 + 1 is a
    # tie that rounds to even (2^24), and so on, so the block sums to 2^24.
    # Any order that adds the 1s first would give 2^24 + 8.
    a = np.array([2.0 ** 24] + [1.0] * 7, np.float32)
    assert orc.canon_dot(a, np.ones(8)) == 2.0 ** 24
    assert orc.canon_dot(a[::-1], np.ones(8)) == 2.0 ** 24 + 8


def test_canon_dot_pairwise_adjacent_tree(orc):
    # Four blocks with sums P = (2^25, 3, -2^25, 3) (blocks 1 and 3 hold three
    # 1s).  Adjacent pairs first: 2^25 + 3 -> 2^25 + 4 (spacing 4 at 2^25) and
    # -2^25 + 3 -> -2^25 + 4, total 8.  Pairing blocks (0,2),(1,3) would give
    # 0 + 6 = 6, and a left-to-right sum of the blocks 7.
    a = np.zeros(32, np.float32)
    a[0] = 2.0 ** 25
    a[8:11] = 1.0
    a[16] = -(2.0 ** 25)
    a[24:27] = 1.0
    assert orc.canon_dot(a, np.ones(32)) == 8.0
    # 2 blocks, P = (2^25, 3): tree gives 2^25 + 4
    assert orc.canon_dot(a[:16], np.ones(16)) == 2.0 ** 25 + 4
    # 8 blocks: ((P0+P1)+(P2+P3)) + ((P4+P5)+(P6+P7)) with the same 4 sums in
    # both halves but the second half negated: exactly 0.
    b = np.concatenate([a, -a])
    assert orc.canon_dot(b, np.ones(64)) == 0.0


def test_canon_dot_accuracy_random(orc):
    import math
    rng = np.random.default_rng(18)
    for n in (64, 128):
        for _ in range(50):
            a = rng.standard_normal(n).astype(np.float32)
            b = rng.standard_normal(n).astype(np.float32)
            exact = math.fsum(float(x) * float(y) for x, y in zip(a, b))
            bound = (8 + np.log2(n / 8) + 2) * U32 * float(np.sum(np.abs(a * b.astype(np.float64))))
            assert abs(orc.canon_dot(a, b) - exact) <= bound
