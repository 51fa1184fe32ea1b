"""Pins for the CPU oracle, each against something other than the oracle itself.

* the chunk dual form printed on page "Modular TTT: Rethinking Test-Time
  Training as Composable Modules", section "方法步骤详情"
  (O = Q W_start - Tril(Q Khat^T) dVhat, W_end = W_start - Khat^T dVhat),
  evaluated by brute force with explicit masks and decay weights;
* C = 1 closed forms: the delta rule (MSE, identity) and decayed Hebbian
  linear attention (inner product, identity);
* chunk-size invariance of the inner-product/identity case;
* eta = 0 and the affine state transition (I - K^T diag(eta) K) W0 + K^T diag(eta) V
  (section "内部学习规则与学习率参数化", the update matrix whose eigenvalues
  govern stability);
* streaming and column independence;
* hand-worked golden values (tests/golden/: a scalar chunk, a vector-decay chunk, a TTT-MLP
  chunk, In-Place with and without a document reset, and the NTP target), forward and
  backward;
* central finite differences for every backward output;
* TTT-MLP (two-layer fast weight): its own brute-force chunk dual form, the
  decay-only case without learning, and finite differences of its backward;
* per-feature (vector) decay: its own brute-force dual form, the scalar decay
  when all features share one factor, a zero factor clearing exactly one row
  of W, and finite differences including the per-feature decay gradient;
* In-Place TTT (page "In-Place Test-Time Training", section "核心方法和技术细节"):
  associativity of the update, plain GEMM when C = T or eta = 0, and the
  dual form with Z_i Z_j^T corrections; its backward against finite
  differences, the single-chunk closed form, and the row-subset and
  sampled-token evaluations against the full one; document resets against
  independent per-document calls and finite differences; the NTP-aligned target
  against shifted copies (one-hot taps) and a plain matmul (one tap), and
  its backward against finite differences.
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "scalar_chunk_worked.txt")


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def act_np(act, z):
    return z * sigmoid(z) if act == "silu" else z


def dact_np(act, z):
    if act != "silu":
        return np.ones_like(z)
    s = sigmoid(z)
    return s * (1 + z * (1 - s))


def rand_inputs(rng, B, H, T, dk, dv, decay=True, w0_scale=0.3):
    Q = rng.standard_normal((B, H, T, dk)) / math.sqrt(dk)
    K = rng.standard_normal((B, H, T, dk)) / math.sqrt(dk)
    V = rng.standard_normal((B, H, T, dv))
    beta = rng.standard_normal((B, H, T))
    gamma = sigmoid(2.0 + rng.standard_normal((B, H, T))) if decay else None
    W0 = w0_scale * rng.standard_normal((B, H, dk, dv))
    return Q, K, V, beta, gamma, W0


def dual_form(Q, K, V, beta, gamma, W0, C, loss, act, b):
    """The page's chunk dual form, by brute force, one head at a time."""
    B, H, T, dk = Q.shape
    dv = V.shape[-1]
    O = np.zeros((B, H, T, dv))
    WF = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for hi in range(H):
            W = W0[bi, hi].copy()
            for c in range(T // C):
                sl = slice(c * C, (c + 1) * C)
                q, k, v = Q[bi, hi, sl], K[bi, hi, sl], V[bi, hi, sl]
                eta = 2 * sigmoid(beta[bi, hi, sl] + b)
                lg = np.log(gamma[bi, hi, sl]) if gamma is not None else np.zeros(C)
                L = np.cumsum(lg)
                Z = k @ W
                Vh = act_np(act, Z)
                A = Vh - v if loss == "mse" else -v
                G = A * dact_np(act, Z)
                Zq = np.zeros((C, dv))
                for s in range(C):
                    acc = math.exp(L[s]) * (q[s] @ W)
                    for r in range(s + 1):  # Tril: r <= s, the diagonal included
                        acc = acc - eta[r] * math.exp(L[s] - L[r]) * float(q[s] @ k[r]) * G[r]
                    Zq[s] = acc
                O[bi, hi, sl] = act_np(act, Zq)
                u = eta * np.exp(L[-1] - L)
                W = math.exp(L[-1]) * W - k.T @ (u[:, None] * G)
            WF[bi, hi] = W
    return O, WF


COMBOS = [(l, a) for l in ("mse", "ip") for a in ("id", "silu")]


@pytest.mark.parametrize("loss,act", COMBOS)
@pytest.mark.parametrize("C", [1, 2, 4, 8])
@pytest.mark.parametrize("decay", [False, True])
def test_oracle_matches_chunk_dual_form(loss, act, C, decay):
    rng = np.random.default_rng(100 + C)
    Q, K, V, beta, gamma, W0 = rand_inputs(rng, 1, 2, 16, 5, 3, decay=decay)
    b = -0.7
    O, WF, WC, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, C=C, loss=loss, act=act, lr_bias=b)
    O2, WF2 = dual_form(Q, K, V, beta, gamma, W0, C, loss, act, b)
    np.testing.assert_allclose(O, O2, rtol=0, atol=1e-12 * max(1, np.abs(O2).max()))
    np.testing.assert_allclose(WF, WF2, rtol=0, atol=1e-12 * max(1, np.abs(WF2).max()))
    # saved chunk-start weights: first is W0, each later one equals the state after the previous chunk
    np.testing.assert_array_equal(WC[:, :, 0], W0)


@pytest.mark.parametrize("decay", [False, True])
def test_c1_is_the_delta_rule(decay):
    rng = np.random.default_rng(7)
    Q, K, V, beta, gamma, W0 = rand_inputs(rng, 1, 1, 24, 4, 3, decay=decay)
    b = 0.3
    O, WF, _, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, C=1, loss="mse", act="id", lr_bias=b)
    W = W0[0, 0].copy()
    for t in range(24):
        k, v, q = K[0, 0, t], V[0, 0, t], Q[0, 0, t]
        eta = 2 * sigmoid(beta[0, 0, t] + b)
        g = 1.0 if gamma is None else gamma[0, 0, t]
        W = g * W - eta * np.outer(k, k @ W - v)     # textbook delta rule with decay
        np.testing.assert_allclose(O[0, 0, t], q @ W, atol=1e-12)
    np.testing.assert_allclose(WF[0, 0], W, atol=1e-12)


def test_c1_inner_product_is_decayed_hebbian_attention():
    rng = np.random.default_rng(8)
    T = 20
    Q, K, V, beta, gamma, W0 = rand_inputs(rng, 1, 1, T, 4, 3, decay=True)
    b = -1.1
    O, _, _, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, C=1, loss="ip", act="id", lr_bias=b)
    eta = 2 * sigmoid(beta[0, 0] + b)
    cum = np.cumprod(gamma[0, 0])
    for t in range(T):
        want = cum[t] * (Q[0, 0, t] @ W0[0, 0])
        for r in range(t + 1):
            want = want + (cum[t] / cum[r]) * eta[r] * (Q[0, 0, t] @ K[0, 0, r]) * V[0, 0, r]
        np.testing.assert_allclose(O[0, 0, t], want, atol=1e-12)


def test_inner_product_identity_is_chunk_invariant():
    rng = np.random.default_rng(9)
    Q, K, V, beta, gamma, W0 = rand_inputs(rng, 2, 1, 32, 4, 4, decay=True)
    ref = None
    for C in (1, 2, 4, 8, 16, 32):
        O, WF, _, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, C=C, loss="ip", act="id", lr_bias=0.2)
        if ref is None:
            ref = (O, WF)
        else:
            np.testing.assert_allclose(O, ref[0], atol=1e-12)
            np.testing.assert_allclose(WF, ref[1], atol=1e-12)


def test_mse_depends_on_chunk_size():
    rng = np.random.default_rng(10)
    Q, K, V, beta, gamma, W0 = rand_inputs(rng, 1, 1, 16, 4, 4)
    O1, _, _, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, C=1, loss="mse", act="id", lr_bias=0.5)
    O4, _, _, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, C=4, loss="mse", act="id", lr_bias=0.5)
    assert np.abs(O1 - O4).max() > 1e-3


@pytest.mark.parametrize("loss,act", COMBOS)
def test_eta_zero_only_decays(loss, act):
    rng = np.random.default_rng(11)
    Q, K, V, beta, gamma, W0 = rand_inputs(rng, 1, 2, 16, 4, 3)
    O, WF, _, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, C=4, loss=loss, act=act, lr_bias=-1e4)
    cum = np.cumprod(gamma, axis=-1)
    want = act_np(act, cum[..., None] * np.einsum("bhtk,bhkv->bhtv", Q, W0))
    np.testing.assert_allclose(O, want, atol=1e-12)
    np.testing.assert_allclose(WF, cum[..., -1, None, None] * W0, atol=1e-12)


def test_affine_state_transition():
    """No decay, identity, MSE: W_end = (I - K^T diag(eta) K) W0 + K^T diag(eta) V."""
    rng = np.random.default_rng(12)
    C = 8
    Q, K, V, beta, _, W0 = rand_inputs(rng, 1, 1, C, 5, 3, decay=False)
    b = 0.1
    _, WF, _, _ = oracle.ttt_fwd(Q, K, V, beta, None, W0, C=C, loss="mse", act="id", lr_bias=b)
    k, v = K[0, 0], V[0, 0]
    D = np.diag(2 * sigmoid(beta[0, 0] + b))
    want = (np.eye(5) - k.T @ D @ k) @ W0[0, 0] + k.T @ D @ v
    np.testing.assert_allclose(WF[0, 0], want, atol=1e-12)


def test_streaming_equals_one_call():
    rng = np.random.default_rng(13)
    Q, K, V, beta, gamma, W0 = rand_inputs(rng, 1, 2, 32, 4, 4)
    kw = dict(C=8, loss="mse", act="silu", lr_bias=-0.5)
    O, WF, _, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, **kw)
    a = slice(0, 16)
    b_ = slice(16, 32)
    O1, W1, _, _ = oracle.ttt_fwd(Q[:, :, a], K[:, :, a], V[:, :, a], beta[..., a], gamma[..., a], W0, **kw)
    O2, W2, _, _ = oracle.ttt_fwd(Q[:, :, b_], K[:, :, b_], V[:, :, b_], beta[..., b_], gamma[..., b_], W1, **kw)
    np.testing.assert_allclose(np.concatenate([O1, O2], axis=2), O, atol=1e-13)
    np.testing.assert_allclose(W2, WF, atol=1e-13)


def test_value_columns_are_independent():
    rng = np.random.default_rng(14)
    Q, K, V, beta, gamma, W0 = rand_inputs(rng, 1, 1, 16, 4, 6)
    kw = dict(C=4, loss="mse", act="silu", lr_bias=0.0)
    O, WF, _, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, **kw)
    cols = [1, 4, 5]
    Os, WFs, _, _ = oracle.ttt_fwd(Q, K, V[..., cols], beta, gamma, W0[..., cols], **kw)
    np.testing.assert_allclose(Os, O[..., cols], atol=1e-14)
    np.testing.assert_allclose(WFs, WF[..., cols], atol=1e-14)


def _golden():
    cases, grads = {}, {}
    with open(GOLDEN) as f:
        for line in f:
            if line.startswith("case "):
                lhs, rhs = line[5:].split("|")
                name, loss, act, C, g1, g2 = lhs.split()
                cases[name] = (loss, act, int(C), float(g1), float(g2), [float(x) for x in rhs.split()])
            elif line.startswith("grad "):
                lhs, rhs = line[5:].split("|")
                grads[lhs.strip()] = [float(x) for x in rhs.split()]
    return cases, grads


def _golden_inputs():
    Q = np.array([1.0, 3.0]).reshape(1, 1, 2, 1)
    K = np.array([1.0, 2.0]).reshape(1, 1, 2, 1)
    V = np.array([2.0, -1.0]).reshape(1, 1, 2, 1)
    beta = np.zeros((1, 1, 2))
    W0 = np.full((1, 1, 1, 1), 0.5)
    return Q, K, V, beta, W0


def test_golden_scalar_worked_examples():
    cases, _ = _golden()
    assert len(cases) == 4
    Q, K, V, beta, W0 = _golden_inputs()
    for name, (loss, act, C, g1, g2, (o1, o2, wf)) in cases.items():
        gamma = None if g1 == 1 and g2 == 1 else np.array([g1, g2]).reshape(1, 1, 2)
        O, WF, _, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, C=C, loss=loss, act=act, lr_bias=0.0)
        np.testing.assert_allclose(O.ravel(), [o1, o2], atol=1e-14, err_msg=name)
        np.testing.assert_allclose(WF.ravel(), [wf], atol=1e-14, err_msg=name)


def test_golden_scalar_backward():
    _, grads = _golden()
    Q, K, V, beta, W0 = _golden_inputs()
    dO = np.array([0.0, 1.0]).reshape(1, 1, 2, 1)
    g = oracle.ttt_bwd(Q, K, V, beta, None, W0, dO, None, C=2, loss="mse", act="id", lr_bias=0.0)
    got = np.concatenate([g["dQ"].ravel(), g["dK"].ravel(), g["dV"].ravel(), g["dbeta"].ravel(),
                          g["dW0"].ravel()])
    np.testing.assert_allclose(got, grads["mse_c2"], atol=1e-14)


def _objective(Q, K, V, beta, gamma, W0, dO, dWT, kw):
    O, WF, _, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, **kw)
    return float((O * dO).sum() + (WF * dWT).sum())


@pytest.mark.parametrize("loss,act", COMBOS)
def test_backward_matches_finite_differences(loss, act):
    rng = np.random.default_rng(20 + 2 * list(dict.fromkeys(COMBOS)).index((loss, act)))
    B, H, T, dk, dv, C = 1, 2, 16, 4, 3, 4
    Q, K, V, beta, gamma, W0 = rand_inputs(rng, B, H, T, dk, dv, decay=True, w0_scale=0.5)
    dO = rng.standard_normal((B, H, T, dv))
    dWT = rng.standard_normal((B, H, dk, dv))
    kw = dict(C=C, loss=loss, act=act, lr_bias=-0.4)
    g = oracle.ttt_bwd(Q, K, V, beta, gamma, W0, dO, dWT, **kw)
    h = 1e-6
    args = dict(Q=Q, K=K, V=V, beta=beta, gamma=gamma, W0=W0)
    names = dict(Q="dQ", K="dK", V="dV", beta="dbeta", gamma="dgamma", W0="dW0")
    for name, x in args.items():
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            jp = _objective(Q, K, V, beta, gamma, W0, dO, dWT, kw)
            x[idx] = old - h
            jm = _objective(Q, K, V, beta, gamma, W0, dO, dWT, kw)
            x[idx] = old
            fd[idx] = (jp - jm) / (2 * h)
        an = g[names[name]]
        err = np.abs(an - fd).max() / max(1e-12, np.abs(fd).max())
        assert err < 1e-7, (name, err)


# ------------------------------------------------------------ per-feature (vector) decay
# Page "Modular TTT: Rethinking Test-Time Training as Composable Modules", section "权重衰减":
# vector decay is a per-feature forgetting factor. Reading: gamma_t has one factor per key
# feature and scales that row of W, W_t = diag(gamma_t) W_{t-1} - eta_t k_t^T g_t.


def vector_gamma(rng, B, H, T, dk):
    return sigmoid(2.0 + rng.standard_normal((B, H, T, dk)))


def dual_form_vector(Q, K, V, beta, gamma, W0, C, loss, act, b):
    """Chunk dual form with a per-feature decay, by brute force: with L_s the chunk-local
    cumulative log-decay of every feature,
        Zq_s  = (q_s * exp(L_s)) W0 - sum_{r<=s} eta_r (sum_i q_si k_ri exp(L_si - L_ri)) g_r
        W_end = diag(exp(L_C)) W0 - sum_r eta_r (k_r * exp(L_C - L_r))^T g_r."""
    B, H, T, dk = Q.shape
    dv = V.shape[-1]
    O = np.zeros((B, H, T, dv))
    WF = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for hi in range(H):
            W = W0[bi, hi].copy()
            for c in range(T // C):
                sl = slice(c * C, (c + 1) * C)
                q, k, v = Q[bi, hi, sl], K[bi, hi, sl], V[bi, hi, sl]
                eta = 2 * sigmoid(beta[bi, hi, sl] + b)
                L = np.cumsum(np.log(gamma[bi, hi, sl]), axis=0)  # [C, dk]
                Z = k @ W
                A = act_np(act, Z) - v if loss == "mse" else -v
                G = A * dact_np(act, Z)
                Zq = np.zeros((C, dv))
                for s in range(C):
                    acc = (q[s] * np.exp(L[s])) @ W
                    for r in range(s + 1):
                        p = float(np.sum(q[s] * k[r] * np.exp(L[s] - L[r])))
                        acc = acc - eta[r] * p * G[r]
                    Zq[s] = acc
                O[bi, hi, sl] = act_np(act, Zq)
                Wn = np.exp(L[-1])[:, None] * W
                for r in range(C):
                    Wn = Wn - eta[r] * np.outer(k[r] * np.exp(L[-1] - L[r]), G[r])
                W = Wn
            WF[bi, hi] = W
    return O, WF


@pytest.mark.parametrize("loss,act", COMBOS)
@pytest.mark.parametrize("C", [1, 2, 4, 8])
def test_vector_decay_matches_its_dual_form(loss, act, C):
    rng = np.random.default_rng(300 + C)
    Q, K, V, beta, _, W0 = rand_inputs(rng, 1, 2, 16, 5, 3, decay=False)
    gamma = vector_gamma(rng, 1, 2, 16, 5)
    b = -0.7
    O, WF, _, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, C=C, loss=loss, act=act, lr_bias=b)
    O2, WF2 = dual_form_vector(Q, K, V, beta, gamma, W0, C, loss, act, b)
    np.testing.assert_allclose(O, O2, rtol=0, atol=1e-12 * max(1, np.abs(O2).max()))
    np.testing.assert_allclose(WF, WF2, rtol=0, atol=1e-12 * max(1, np.abs(WF2).max()))


VECTOR_GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "vector_decay_worked.txt")


def test_golden_vector_decay_worked_example():
    """Hand-worked rationals of tests/golden/vector_decay_worked.txt, forward and backward."""
    want = {}
    with open(VECTOR_GOLDEN) as f:
        for line in f:
            if "|" in line and not line.startswith("#"):
                name, vals = line.split("|")
                want[name.strip()] = [float(x) for x in vals.split()]
    assert len(want) == 8
    Q = np.array([[1.0, 1.0], [1.0, 1.0]]).reshape(1, 1, 2, 2)
    K = np.array([[1.0, 0.0], [0.0, 1.0]]).reshape(1, 1, 2, 2)
    V = np.array([0.0, 1.0]).reshape(1, 1, 2, 1)
    beta = np.zeros((1, 1, 2))
    gamma = np.array([[0.5, 1.0], [1.0, 0.5]]).reshape(1, 1, 2, 2)
    W0 = np.array([1.0, 0.0]).reshape(1, 1, 2, 1)
    kw = dict(C=2, loss="mse", act="id", lr_bias=0.0)
    O, WF, _, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, **kw)
    g = oracle.ttt_bwd(Q, K, V, beta, gamma, W0, np.array([0.0, 1.0]).reshape(1, 1, 2, 1), None,
                       **kw)
    got = dict(O=O, W_final=WF, **g)
    for name, vals in want.items():
        np.testing.assert_allclose(got[name].ravel(), vals, atol=1e-14, err_msg=name)


def test_vector_decay_with_equal_features_is_the_scalar_decay():
    rng = np.random.default_rng(310)
    B, H, T, dk, dv = 1, 2, 16, 4, 3
    Q, K, V, beta, gamma, W0 = rand_inputs(rng, B, H, T, dk, dv, decay=True)
    gv = np.repeat(gamma[..., None], dk, axis=-1)
    dO = rng.standard_normal((B, H, T, dv))
    dWT = rng.standard_normal((B, H, dk, dv))
    kw = dict(C=4, loss="mse", act="silu", lr_bias=-0.5)
    O, WF, _, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, **kw)
    Ov, WFv, _, _ = oracle.ttt_fwd(Q, K, V, beta, gv, W0, **kw)
    np.testing.assert_allclose(Ov, O, rtol=0, atol=1e-13)
    np.testing.assert_allclose(WFv, WF, rtol=0, atol=1e-13)
    g = oracle.ttt_bwd(Q, K, V, beta, gamma, W0, dO, dWT, **kw)
    gv_ = oracle.ttt_bwd(Q, K, V, beta, gv, W0, dO, dWT, **kw)
    for k in ("dQ", "dK", "dV", "dbeta", "dW0"):
        np.testing.assert_allclose(gv_[k], g[k], rtol=0, atol=1e-12)
    # the scalar factor multiplies every row, so its gradient is the sum of the rows'
    np.testing.assert_allclose(gv_["dgamma"].sum(-1), g["dgamma"], rtol=0, atol=1e-12)


def test_vector_decay_zero_clears_exactly_one_row():
    # gamma = 0 on key feature i0 at the last token: row i0 of W_final is that token's write
    # alone, -eta k_{i0} g with g = k W0c - v (MSE, identity) at the last chunk's start state
    rng = np.random.default_rng(320)
    B, H, T, dk, dv, C, i0 = 1, 1, 12, 5, 3, 4, 2
    Q, K, V, beta, _, W0 = rand_inputs(rng, B, H, T, dk, dv, decay=False)
    gamma = vector_gamma(rng, B, H, T, dk)
    gamma[0, 0, T - 1, i0] = 0.0
    b = 0.2
    _, WF, WC, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, C=C, loss="mse", act="id", lr_bias=b)
    k, v = K[0, 0, T - 1], V[0, 0, T - 1]
    eta = 2 * sigmoid(beta[0, 0, T - 1] + b)
    g = k @ WC[0, 0, -1] - v
    np.testing.assert_allclose(WF[0, 0, i0], -eta * k[i0] * g, rtol=0, atol=1e-13)
    # with gamma = 1 there instead, the row keeps its history and differs
    gamma[0, 0, T - 1, i0] = 1.0
    _, WF1, _, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, C=C, loss="mse", act="id", lr_bias=b)
    assert np.abs(WF1[0, 0, i0] - WF[0, 0, i0]).max() > 1e-3
    others = [i for i in range(dk) if i != i0]
    np.testing.assert_allclose(WF1[0, 0, others], WF[0, 0, others], rtol=0, atol=1e-13)


@pytest.mark.parametrize("loss,act", COMBOS)
def test_vector_decay_backward_matches_finite_differences(loss, act):
    rng = np.random.default_rng(330 + 2 * list(dict.fromkeys(COMBOS)).index((loss, act)))
    B, H, T, dk, dv, C = 1, 1, 12, 4, 3, 4
    Q, K, V, beta, _, W0 = rand_inputs(rng, B, H, T, dk, dv, decay=False, w0_scale=0.5)
    gamma = vector_gamma(rng, B, H, T, dk)
    dO = rng.standard_normal((B, H, T, dv))
    dWT = rng.standard_normal((B, H, dk, dv))
    kw = dict(C=C, loss=loss, act=act, lr_bias=-0.4)
    g = oracle.ttt_bwd(Q, K, V, beta, gamma, W0, dO, dWT, **kw)
    assert g["dgamma"].shape == gamma.shape
    h = 1e-6
    args = dict(Q=Q, K=K, V=V, beta=beta, gamma=gamma, W0=W0)
    names = dict(Q="dQ", K="dK", V="dV", beta="dbeta", gamma="dgamma", W0="dW0")
    for name, x in args.items():
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            jp = _objective(Q, K, V, beta, gamma, W0, dO, dWT, kw)
            x[idx] = old - h
            jm = _objective(Q, K, V, beta, gamma, W0, dO, dWT, kw)
            x[idx] = old
            fd[idx] = (jp - jm) / (2 * h)
        err = np.abs(g[names[name]] - fd).max() / max(1e-12, np.abs(fd).max())
        assert err < 1e-7, (name, err)


def test_f32_state_build_tracks_f64():
    rng = np.random.default_rng(30)
    Q, K, V, beta, gamma, W0 = rand_inputs(rng, 1, 2, 64, 16, 16)
    kw = dict(C=16, loss="mse", act="silu", lr_bias=-2.0)
    O64, W64, _, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, **kw)
    O32, W32, _, _ = oracle.ttt_fwd(Q, K, V, beta, gamma, W0, state="f32", **kw)
    assert np.abs(O32 - O64).max() / np.abs(O64).max() < 1e-5
    assert np.abs(W32 - W64).max() / np.abs(W64).max() < 1e-5


# --------------------------------------------------------------------------- In-Place TTT


def _inplace_rand(rng, T, d_ff, d_model):
    Z = rng.standard_normal((T, d_ff))
    Vh = 0.1 * rng.standard_normal((T, d_model))
    W = 0.1 * rng.standard_normal((d_model, d_ff))
    return Z, Vh, W


def test_inplace_final_state_is_associative():
    rng = np.random.default_rng(40)
    Z, Vh, W = _inplace_rand(rng, 32, 12, 5)
    for C in (1, 4, 8, 32):
        _, WF = oracle.inplace_fwd(Z, Vh, W, C=C, lr=0.05)
        np.testing.assert_allclose(WF, W + 0.05 * Vh.T @ Z, atol=1e-12)


def test_inplace_single_chunk_and_zero_lr_are_plain_gemm():
    rng = np.random.default_rng(41)
    Z, Vh, W = _inplace_rand(rng, 32, 12, 5)
    O, _ = oracle.inplace_fwd(Z, Vh, W, C=32, lr=0.05)
    np.testing.assert_allclose(O, Z @ W.T, atol=1e-12)
    O0, _ = oracle.inplace_fwd(Z, Vh, W, C=4, lr=0.0)
    np.testing.assert_allclose(O0, Z @ W.T, atol=1e-12)


def test_inplace_dual_form():
    """O_i = Z_i W_0^T + eta * sum_{j<i} (Z_i Z_j^T) Vhat_j  (apply-then-update, no intra-chunk term)."""
    rng = np.random.default_rng(42)
    T, C, eta = 24, 4, 0.03
    Z, Vh, W = _inplace_rand(rng, T, 7, 6)
    O, _ = oracle.inplace_fwd(Z, Vh, W, C=C, lr=eta)
    for i in range(T // C):
        zi = Z[i * C:(i + 1) * C]
        want = zi @ W.T
        for j in range(i):
            want = want + eta * (zi @ Z[j * C:(j + 1) * C].T) @ Vh[j * C:(j + 1) * C]
        np.testing.assert_allclose(O[i * C:(i + 1) * C], want, atol=1e-12)


def test_inplace_row_subset_is_exact():
    rng = np.random.default_rng(43)
    Z, Vh, W = _inplace_rand(rng, 16, 9, 8)
    O, WF = oracle.inplace_fwd(Z, Vh, W, C=4, lr=0.1)
    rows = np.array([0, 3, 7])
    Os, WFs = oracle.inplace_fwd(Z, Vh, W, C=4, lr=0.1, rows=rows)
    np.testing.assert_array_equal(Os, O[:, rows])
    np.testing.assert_array_equal(WFs, WF[rows])


def _inplace_objective(Z, Vh, W, dO, dWf, C, lr):
    O, WF = oracle.inplace_fwd(Z, Vh, W, C=C, lr=lr)
    return float((O * dO).sum() + (WF * dWf).sum())


def test_inplace_backward_matches_finite_differences():
    rng = np.random.default_rng(44)
    T, d_ff, d_model, C, lr = 8, 5, 3, 2, 0.3
    Z, Vh, W = _inplace_rand(rng, T, d_ff, d_model)
    dO = rng.standard_normal((T, d_model))
    dWf = rng.standard_normal((d_model, d_ff))
    g = oracle.inplace_bwd(Z, Vh, W, dO, dWf, C=C, lr=lr)
    h = 1e-6
    for name, x, key in (("Z", Z, "dZ"), ("Vhat", Vh, "dVhat"), ("W", W, "dW")):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            jp = _inplace_objective(Z, Vh, W, dO, dWf, C, lr)
            x[idx] = old - h
            jm = _inplace_objective(Z, Vh, W, dO, dWf, C, lr)
            x[idx] = old
            fd[idx] = (jp - jm) / (2 * h)
        err = np.abs(g[key] - fd).max() / np.abs(fd).max()
        assert err < 1e-8, (name, err)


def test_inplace_backward_single_chunk_closed_form():
    # C = T: O = Z W^T, W_final = W + lr Vhat^T Z, so dZ = dO W + lr Vhat dWf,
    # dVhat = lr Z dWf^T and dW = dWf + dO^T Z
    rng = np.random.default_rng(45)
    T, lr = 16, 0.07
    Z, Vh, W = _inplace_rand(rng, T, 6, 4)
    dO = rng.standard_normal((T, 4))
    dWf = rng.standard_normal((4, 6))
    g = oracle.inplace_bwd(Z, Vh, W, dO, dWf, C=T, lr=lr)
    np.testing.assert_allclose(g["dZ"], dO @ W + lr * Vh @ dWf, atol=1e-12)
    np.testing.assert_allclose(g["dVhat"], lr * Z @ dWf.T, atol=1e-12)
    np.testing.assert_allclose(g["dW"], dWf + dO.T @ Z, atol=1e-12)


def test_inplace_backward_row_subset_and_sampled_tokens_are_exact():
    rng = np.random.default_rng(46)
    T, d_ff, d_model, C, lr = 24, 7, 6, 4, 0.05
    Z, Vh, W = _inplace_rand(rng, T, d_ff, d_model)
    dO = rng.standard_normal((T, d_model))
    dWf = rng.standard_normal((d_model, d_ff))
    g = oracle.inplace_bwd(Z, Vh, W, dO, dWf, C=C, lr=lr)
    rows = np.array([1, 4, 5])
    gs = oracle.inplace_bwd(Z, Vh, W, dO, dWf, C=C, lr=lr, rows=rows)
    assert gs["dZ"] is None
    np.testing.assert_allclose(gs["dVhat"], g["dVhat"][:, rows], atol=1e-13)
    np.testing.assert_allclose(gs["dW"], g["dW"][rows], atol=1e-13)
    tokens = [0, 5, 13, 23]
    dz = oracle.inplace_bwd_dz_tokens(Z, Vh, W, dO, dWf, C=C, lr=lr, tokens=tokens)
    np.testing.assert_allclose(dz, g["dZ"][tokens], atol=1e-12)
    dz0 = oracle.inplace_bwd_dz_tokens(Z, Vh, W, dO, None, C=C, lr=lr, tokens=tokens)
    g0 = oracle.inplace_bwd(Z, Vh, W, dO, None, C=C, lr=lr)
    np.testing.assert_allclose(dz0, g0["dZ"][tokens], atol=1e-12)


def test_inplace_target_special_cases():
    # one tap at offset j with weight 1 and W_target = I: Vhat is X0 shifted j tokens up
    rng = np.random.default_rng(47)
    T, d, k = 12, 5, 4
    X0 = rng.standard_normal((T, d))
    for j in range(k):
        w = np.zeros((k, d))
        w[j] = 1.0
        V, _ = oracle.inplace_target(X0, w, np.eye(d))
        want = np.zeros_like(X0)
        want[: T - j] = X0[j:]
        np.testing.assert_array_equal(V, want)
    # a single tap (k = 1) makes it a per-channel scale followed by a plain matmul
    w1 = rng.standard_normal((1, d))
    Wt = rng.standard_normal((d, 3))
    V, _ = oracle.inplace_target(X0, w1, Wt)
    np.testing.assert_allclose(V, (X0 * w1[0]) @ Wt, atol=1e-12)


def test_inplace_target_backward_matches_finite_differences():
    rng = np.random.default_rng(48)
    T, d, k, d_out = 7, 3, 3, 2
    X0 = rng.standard_normal((T, d))
    w = rng.standard_normal((k, d))
    Wt = rng.standard_normal((d, d_out))
    dV = rng.standard_normal((T, d_out))
    g = oracle.inplace_target_bwd(X0, w, Wt, dV)
    h = 1e-6
    for name, x, key in (("X0", X0, "dX0"), ("w", w, "dconv_w"), ("Wt", Wt, "dW_target")):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            jp = float((oracle.inplace_target(X0, w, Wt)[0] * dV).sum())
            x[idx] = old - h
            jm = float((oracle.inplace_target(X0, w, Wt)[0] * dV).sum())
            x[idx] = old
            fd[idx] = (jp - jm) / (2 * h)
        err = np.abs(g[key] - fd).max() / np.abs(fd).max()
        assert err < 1e-8, (name, err)


def test_inplace_target_backward_channel_subset_is_exact():
    rng = np.random.default_rng(49)
    T, d, k = 10, 6, 3
    X0 = rng.standard_normal((T, d))
    w = rng.standard_normal((k, d))
    Wt = rng.standard_normal((d, 4))
    dV = rng.standard_normal((T, 4))
    g = oracle.inplace_target_bwd(X0, w, Wt, dV)
    ch = np.array([0, 2, 5])
    gs = oracle.inplace_target_bwd(X0, w, Wt, dV, channels=ch)
    np.testing.assert_allclose(gs["dX0"], g["dX0"][:, ch], atol=1e-13)
    np.testing.assert_allclose(gs["dconv_w"], g["dconv_w"][:, ch], atol=1e-13)
    np.testing.assert_allclose(gs["dW_target"], g["dW_target"][ch], atol=1e-13)


# ------------------------------------------------------------------------------- TTT-MLP


def _mlp_rand(rng, B, H, T, dk, dv, hd, decay=True):
    Q, K, V, beta, gamma, _ = rand_inputs(rng, B, H, T, dk, dv, decay=decay)
    W1 = 0.4 * rng.standard_normal((B, H, dk, hd))
    W2 = 0.4 * rng.standard_normal((B, H, hd, dv))
    return Q, K, V, beta, gamma, W1, W2


def mlp_dual_form(Q, K, V, beta, gamma, W1, W2, C, loss, act, b):
    """Chunk dual form of the two-layer learner, by brute force: with A1 = act(K W1_0),
    G2 = dl/dvhat, G1 = (G2 W2_0^T) * act'(K W1_0) and w_sr = eta_r exp(L_s - L_r), r <= s,
        Zq1_s = Gamma_s q_s W1_0 - sum_r w_sr (q_s . k_r) G1_r,   Aq_s = act(Zq1_s),
        o_s   = Gamma_s Aq_s W2_0 - sum_r w_sr (Aq_s . A1_r) G2_r,
        W1_end = Gamma_C W1_0 - K^T diag(u) G1,  W2_end = Gamma_C W2_0 - A1^T diag(u) G2."""
    B, H, T, dk = Q.shape
    dv = V.shape[-1]
    O = np.zeros((B, H, T, dv))
    W1F, W2F = np.zeros_like(W1), np.zeros_like(W2)
    for bi in range(B):
        for hi in range(H):
            A, Bw = W1[bi, hi].copy(), W2[bi, hi].copy()
            for c in range(T // C):
                sl = slice(c * C, (c + 1) * C)
                q, k, v = Q[bi, hi, sl], K[bi, hi, sl], V[bi, hi, sl]
                eta = 2 * sigmoid(beta[bi, hi, sl] + b)
                L = np.cumsum(np.log(gamma[bi, hi, sl])) if gamma is not None else np.zeros(C)
                Z1 = k @ A
                A1 = act_np(act, Z1)
                G2 = A1 @ Bw - v if loss == "mse" else -v
                G1 = (G2 @ Bw.T) * dact_np(act, Z1)
                for s_ in range(C):
                    zq = math.exp(L[s_]) * (q[s_] @ A)
                    for r in range(s_ + 1):
                        zq = zq - eta[r] * math.exp(L[s_] - L[r]) * float(q[s_] @ k[r]) * G1[r]
                    aq = act_np(act, zq)
                    o = math.exp(L[s_]) * (aq @ Bw)
                    for r in range(s_ + 1):
                        o = o - eta[r] * math.exp(L[s_] - L[r]) * float(aq @ A1[r]) * G2[r]
                    O[bi, hi, c * C + s_] = o
                u = eta * np.exp(L[-1] - L)
                A = math.exp(L[-1]) * A - k.T @ (u[:, None] * G1)
                Bw = math.exp(L[-1]) * Bw - A1.T @ (u[:, None] * G2)
            W1F[bi, hi], W2F[bi, hi] = A, Bw
    return O, W1F, W2F


@pytest.mark.parametrize("loss,act", COMBOS)
@pytest.mark.parametrize("C", [1, 2, 4])
def test_ttt_mlp_matches_its_dual_form(loss, act, C):
    rng = np.random.default_rng(500 + C)
    Q, K, V, beta, gamma, W1, W2 = _mlp_rand(rng, 1, 2, 8, 3, 2, 5)
    b = -0.6
    O, W1F, W2F = oracle.ttt_mlp_fwd(Q, K, V, beta, gamma, W1, W2, C=C, loss=loss, act=act,
                                     lr_bias=b)
    O2, W1F2, W2F2 = mlp_dual_form(Q, K, V, beta, gamma, W1, W2, C, loss, act, b)
    np.testing.assert_allclose(O.numpy(), O2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(W1F.numpy(), W1F2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(W2F.numpy(), W2F2, rtol=0, atol=1e-12)


def test_ttt_mlp_without_learning_only_decays():
    # eta = 2 sigmoid(beta + b) -> 0: both layers only decay, o_t = act(c_t q_t W1) c_t W2 with
    # c_t the product of every gamma up to t
    rng = np.random.default_rng(510)
    Q, K, V, beta, gamma, W1, W2 = _mlp_rand(rng, 1, 1, 8, 3, 2, 4)
    O, W1F, W2F = oracle.ttt_mlp_fwd(Q, K, V, beta, gamma, W1, W2, C=4, loss="mse", act="silu",
                                     lr_bias=-80.0)
    cum = np.cumprod(gamma[0, 0])
    for t in range(8):
        want = act_np("silu", cum[t] * (Q[0, 0, t] @ W1[0, 0])) @ (cum[t] * W2[0, 0])
        np.testing.assert_allclose(O[0, 0, t].numpy(), want, atol=1e-12)
    np.testing.assert_allclose(W2F[0, 0].numpy(), cum[-1] * W2[0, 0], atol=1e-12)


@pytest.mark.parametrize("loss,act", COMBOS)
def test_ttt_mlp_backward_matches_finite_differences(loss, act):
    rng = np.random.default_rng(520 + 2 * list(dict.fromkeys(COMBOS)).index((loss, act)))
    B, H, T, dk, dv, hd, C = 1, 1, 6, 2, 2, 3, 3
    Q, K, V, beta, gamma, W1, W2 = _mlp_rand(rng, B, H, T, dk, dv, hd)
    dO = rng.standard_normal((B, H, T, dv))
    dW1 = rng.standard_normal(W1.shape)
    dW2 = rng.standard_normal(W2.shape)
    kw = dict(C=C, loss=loss, act=act, lr_bias=-0.3)
    g = oracle.ttt_mlp_bwd(Q, K, V, beta, gamma, W1, W2, dO, dW1, dW2, **kw)

    def J():
        O, A, Bw = oracle.ttt_mlp_fwd(Q, K, V, beta, gamma, W1, W2, **kw)
        return float((O.numpy() * dO).sum() + (A.numpy() * dW1).sum() + (Bw.numpy() * dW2).sum())

    h = 1e-6
    for name, x, key in (("Q", Q, "dQ"), ("K", K, "dK"), ("V", V, "dV"), ("beta", beta, "dbeta"),
                         ("gamma", gamma, "dgamma"), ("W1", W1, "dW1"), ("W2", W2, "dW2")):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            jp = J()
            x[idx] = old - h
            jm = J()
            x[idx] = old
            fd[idx] = (jp - jm) / (2 * h)
        err = np.abs(g[key] - fd).max() / np.abs(fd).max()
        assert err < 1e-7, (name, err)


def test_inplace_document_resets():
    rng = np.random.default_rng(50)
    T, d_ff, d_model, C, lr = 24, 7, 5, 4, 0.05
    Z, Vh, W = _inplace_rand(rng, T, d_ff, d_model)
    # a reset at every chunk: each chunk applies the initial W; the final state holds the last
    # chunk's update only
    every = list(range(1, T // C))
    O, WF = oracle.inplace_fwd(Z, Vh, W, C=C, lr=lr, doc_starts=every)
    np.testing.assert_allclose(O, Z @ W.T, atol=1e-12)
    np.testing.assert_allclose(WF, W + lr * Vh[-C:].T @ Z[-C:], atol=1e-12)
    # a reset at chunk 3 == two independent calls, one per document
    O2, WF2 = oracle.inplace_fwd(Z, Vh, W, C=C, lr=lr, doc_starts=[3])
    Oa, _ = oracle.inplace_fwd(Z[:12], Vh[:12], W, C=C, lr=lr)
    Ob, WFb = oracle.inplace_fwd(Z[12:], Vh[12:], W, C=C, lr=lr)
    np.testing.assert_allclose(O2, np.concatenate([Oa, Ob]), atol=1e-12)
    np.testing.assert_allclose(WF2, WFb, atol=1e-12)
    # and the gradients: the initial W gets both documents' adjoints, each part its own
    dO = rng.standard_normal((T, d_model))
    dWf = rng.standard_normal((d_model, d_ff))
    g = oracle.inplace_bwd(Z, Vh, W, dO, dWf, C=C, lr=lr, doc_starts=[3])
    ga = oracle.inplace_bwd(Z[:12], Vh[:12], W, dO[:12], None, C=C, lr=lr)
    gb = oracle.inplace_bwd(Z[12:], Vh[12:], W, dO[12:], dWf, C=C, lr=lr)
    np.testing.assert_allclose(g["dZ"], np.concatenate([ga["dZ"], gb["dZ"]]), atol=1e-12)
    np.testing.assert_allclose(g["dVhat"], np.concatenate([ga["dVhat"], gb["dVhat"]]), atol=1e-12)
    np.testing.assert_allclose(g["dW"], ga["dW"] + gb["dW"], atol=1e-12)


def test_inplace_backward_with_resets_matches_finite_differences():
    rng = np.random.default_rng(51)
    T, d_ff, d_model, C, lr = 8, 4, 3, 2, 0.3
    Z, Vh, W = _inplace_rand(rng, T, d_ff, d_model)
    dO = rng.standard_normal((T, d_model))
    dWf = rng.standard_normal((d_model, d_ff))
    starts = [2]
    g = oracle.inplace_bwd(Z, Vh, W, dO, dWf, C=C, lr=lr, doc_starts=starts)

    def J():
        O, WF = oracle.inplace_fwd(Z, Vh, W, C=C, lr=lr, doc_starts=starts)
        return float((O * dO).sum() + (WF * dWf).sum())

    h = 1e-6
    for x, key in ((Z, "dZ"), (Vh, "dVhat"), (W, "dW")):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            jp = J()
            x[idx] = old - h
            jm = J()
            x[idx] = old
            fd[idx] = (jp - jm) / (2 * h)
        assert np.abs(g[key] - fd).max() / np.abs(fd).max() < 1e-8, key


# ------------------------------------------------------------------ hand-worked fixtures
def _worked_values(name):
    want = {}
    with open(os.path.join(os.path.dirname(__file__), "golden", name)) as f:
        for line in f:
            if "|" in line and not line.startswith("#"):
                key, vals = line.split("|")
                want[key.strip()] = [float(x) for x in vals.split()]
    return want


def test_golden_ttt_mlp_worked_example():
    """Hand-worked integers of tests/golden/ttt_mlp_worked.txt, forward and backward."""
    want = _worked_values("ttt_mlp_worked.txt")
    assert len(want) == 9
    col = lambda *v: np.array(v, dtype=float).reshape(1, 1, len(v), 1)
    Q, K, V = col(1, 2), col(1, 1), col(1, 0)
    beta = np.zeros((1, 1, 2))
    W1, W2 = np.ones((1, 1, 1, 1)), np.full((1, 1, 1, 1), 2.0)
    kw = dict(C=2, loss="mse", act="id", lr_bias=0.0)
    O, W1f, W2f = oracle.ttt_mlp_fwd(Q, K, V, beta, None, W1, W2, **kw)
    got = dict(O=O.numpy(), W1_final=W1f.numpy(), W2_final=W2f.numpy())
    for key in got:
        np.testing.assert_allclose(got[key].ravel(), want[key], atol=1e-12, err_msg=key)
    g = oracle.ttt_mlp_bwd(Q, K, V, beta, None, W1, W2, col(0, 1), **kw)
    for key in ("dQ", "dK", "dV", "dbeta", "dW1", "dW2"):
        np.testing.assert_allclose(g[key].ravel(), want[key], atol=1e-12, err_msg=key)


def test_golden_inplace_and_target_worked_examples():
    """Hand-worked rationals of tests/golden/inplace_worked.txt: In-Place forward and backward
    without and with a document reset, and the NTP target with its backward."""
    want = _worked_values("inplace_worked.txt")
    assert len(want) == 15
    Z = np.array([[1.0, 0.0], [1.0, 1.0]])
    Vh = np.array([[2.0], [4.0]])
    W = np.array([[1.0, 2.0]])
    dO = np.array([[0.0], [1.0]])
    for tag, starts in (("inplace", ()), ("reset", (1,))):
        O, Wf = oracle.inplace_fwd(Z, Vh, W, C=1, lr=0.5, doc_starts=starts)
        g = oracle.inplace_bwd(Z, Vh, W, dO, None, C=1, lr=0.5, doc_starts=starts)
        got = dict(O=O, W_final=Wf, **g)
        for key in ("O", "W_final", "dZ", "dVhat", "dW"):
            np.testing.assert_allclose(got[key].ravel(), want[f"{tag} {key}"], atol=1e-14,
                                       err_msg=f"{tag} {key}")
    X0 = np.array([[1.0], [2.0], [3.0]])
    taps = np.array([[1.0], [2.0]])
    Wt = np.array([[3.0]])
    Vt, Y = oracle.inplace_target(X0, taps, Wt)
    g = oracle.inplace_target_bwd(X0, taps, Wt, np.array([[1.0], [0.0], [1.0]]))
    got = dict(Vhat=Vt, Y=Y, **g)
    for key in ("Vhat", "Y", "dX0", "dconv_w", "dW_target"):
        np.testing.assert_allclose(got[key].ravel(), want[f"target {key}"], atol=1e-14,
                                   err_msg=f"target {key}")
