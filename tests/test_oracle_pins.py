"""Pins of the fp64 oracle to facts fixed by the pages and by the mathematics.

The oracle (oracle/kda_oracle.c) is the token-by-token recurrence of the Kimi
Linear feature page (chapter 4, state-update equation). Each check below ties
it to something other than itself:

* the DPLR expansion equals the delta rule applied to the decayed state
  (chapter 4 equation vs chapter 3 delta-rule equation);
* an explicit-matrix recurrence in the factored form (I - b k k^T) Diag(a);
* closed forms: beta = 0 (pure per-channel decay), one token, two tokens;
* special cases: alpha = 1 is DeltaNet (chapter 3), a channel-constant gate is
  Gated DeltaNet (Kimi Delta Attention review page, "KDA" section);
* invariants: delta-rule overwrite, the norm bound of a contraction;
* an independent chunkwise evaluation (the pages' chunkwise DPLR claim) that
  must agree with the recurrence to rounding;
* split calls and packed varlen batches against single calls;
* a hand-worked golden fixture (tests/golden/two_token_d2.txt).

``test_mutants_are_caught`` builds the oracle with planted mistakes and checks
that these pins reject every one of them.
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "two_token_d2.txt")


def rel_err(a, b):
    a = np.asarray(a, dtype=np.float64); b = np.asarray(b, dtype=np.float64)
    den = max(np.abs(b).max(), 1e-300)
    return float(np.abs(a - b).max() / den)


def f32(x):
    return np.asarray(x, dtype=np.float32)


def rand_case(rng, T, H, Dk, Dv, knorm=True, g_mu=3.0, with_h0=True):
    q = rng.standard_normal((T, H, Dk)); k = rng.standard_normal((T, H, Dk))
    if knorm:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, Dv))
    x = rng.standard_normal((T, H, Dk)) + g_mu
    g = -np.log1p(np.exp(-x))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    h0 = 0.1 * rng.standard_normal((1, H, Dk, Dv)) if with_h0 else None
    return f32(q), f32(k), f32(v), f32(g), f32(beta), h0


# --------------------------------------------------------------------------
# reference forms written independently of the oracle's loop
# --------------------------------------------------------------------------

def explicit_matrix_recurrence(q, k, v, g, beta, scale, h0):
    """S_t = (I - b k k^T) Diag(alpha) S_{t-1} + b k v^T with the Dk x Dk
    transition formed explicitly (single sequence, single head)."""
    q, k, v, g, beta = (np.asarray(x, np.float64) for x in (q, k, v, g, beta))
    T, Dk = k.shape
    S = np.zeros((Dk, v.shape[1])) if h0 is None else np.array(h0, np.float64)
    out = np.zeros((T, v.shape[1]))
    I = np.eye(Dk)
    for t in range(T):
        M = (I - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(g[t]))
        S = M @ S + beta[t] * np.outer(k[t], v[t])
        out[t] = scale * S.T @ q[t]
    return out, S


def chunkwise(q, k, v, g, beta, scale, h0, C):
    """Chunk-parallel evaluation (single sequence, single head), fp64.

    With G the in-chunk running sum of g, K^ = K e^G, K_ = K e^-G, Q^ = Q e^G,
    K~ = K e^(G_last - G):  A = strict_tril(diag(beta) K^ K_^T),
    Tm = (I + A)^-1, W = Tm diag(beta) K^, U = Tm diag(beta) V,
    D = U - W S, O = scale (Q^ S + tril(Q^ K_^T) D),
    S <- diag(e^G_last) S + K~^T D.
    """
    q, k, v, g, beta = (np.asarray(x, np.float64) for x in (q, k, v, g, beta))
    T, Dk = k.shape
    S = np.zeros((Dk, v.shape[1])) if h0 is None else np.array(h0, np.float64)
    out = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        sl = slice(c0, min(T, c0 + C))
        n = sl.stop - sl.start
        G = np.cumsum(g[sl], axis=0)
        Kh, Kc, Qh = k[sl] * np.exp(G), k[sl] * np.exp(-G), q[sl] * np.exp(G)
        Kt = k[sl] * np.exp(G[-1] - G)
        b = beta[sl][:, None]
        A = np.tril(b * (Kh @ Kc.T), -1)
        Tm = np.linalg.inv(np.eye(n) + A)
        W, U = Tm @ (b * Kh), Tm @ (b * v[sl])
        D = U - W @ S
        out[sl] = scale * (Qh @ S + np.tril(Qh @ Kc.T) @ D)
        S = np.exp(G[-1])[:, None] * S + Kt.T @ D
    return out, S


# --------------------------------------------------------------------------
# pin checks; each takes an optional library path so the mutation test can
# run the same checks against a deliberately broken build
# --------------------------------------------------------------------------

def check_dplr_identity(lib_path=None):
    rng = np.random.default_rng(10)
    Dk, Dv = 7, 5
    for _ in range(5):
        a = np.exp(-rng.random(Dk)); b = rng.random()
        k = rng.standard_normal(Dk); S = rng.standard_normal((Dk, Dv))
        lhs = (np.diag(a) - b * np.outer(k, k * a)) @ S
        rhs = (np.eye(Dk) - b * np.outer(k, k)) @ np.diag(a) @ S
        assert rel_err(lhs, rhs) < 1e-14


def check_explicit_matrix(lib_path=None):
    rng = np.random.default_rng(11)
    q, k, v, g, beta, h0 = rand_case(rng, 37, 2, 8, 8)
    out, hT = oracle.kda_oracle(q, k, v, g, beta, 0.3, h0=h0, lib_path=lib_path)
    for h in range(2):
        eo, eS = explicit_matrix_recurrence(q[:, h], k[:, h], v[:, h], g[:, h], beta[:, h],
                                            np.float64(0.3), h0[0, h])
        assert rel_err(out[:, h], eo) < 1e-12
        assert rel_err(hT[0, h], eS) < 1e-12


def check_beta_zero(lib_path=None):
    rng = np.random.default_rng(12)
    q, k, v, g, beta, h0 = rand_case(rng, 29, 1, 6, 4, g_mu=0.5)
    beta = np.zeros_like(beta)
    out, hT = oracle.kda_oracle(q, k, v, g, beta, 1.0, h0=h0, lib_path=lib_path)
    Gam = np.cumsum(g[:, 0].astype(np.float64), axis=0)
    S0 = h0[0, 0]
    exp_out = np.stack([S0.T @ (np.exp(Gam[t]) * q[t, 0]) for t in range(29)])
    assert rel_err(out[:, 0], exp_out) < 1e-13
    assert rel_err(hT[0, 0], np.exp(Gam[-1])[:, None] * S0) < 1e-13


def check_alpha_one_is_deltanet(lib_path=None):
    rng = np.random.default_rng(13)
    q, k, v, g, beta, h0 = rand_case(rng, 31, 1, 8, 6)
    g = np.zeros_like(g)
    out, hT = oracle.kda_oracle(q, k, v, g, beta, 0.5, h0=h0, lib_path=lib_path)
    S = np.array(h0[0, 0])
    for t in range(31):
        kt, vt = k[t, 0].astype(np.float64), v[t, 0].astype(np.float64)
        S = S + beta[t, 0] * np.outer(kt, vt - S.T @ kt)      # delta rule, chapter 3
        assert rel_err(out[t, 0], 0.5 * S.T @ q[t, 0].astype(np.float64)) < 1e-12
    assert rel_err(hT[0, 0], S) < 1e-12
    # with beta = 0 as well the state never moves: o_t = scale S0^T q_t exactly
    out0, hT0 = oracle.kda_oracle(q, k, v, g, np.zeros_like(beta), 0.5, h0=h0, lib_path=lib_path)
    assert np.array_equal(hT0[0, 0], h0[0, 0])
    exp0 = np.stack([0.5 * (h0[0, 0].T @ q[t, 0].astype(np.float64)) for t in range(31)])
    assert rel_err(out0[:, 0], exp0) < 1e-15


def check_scalar_gate_is_gated_deltanet(lib_path=None):
    rng = np.random.default_rng(14)
    q, k, v, g, beta, h0 = rand_case(rng, 33, 1, 8, 8)
    gs = g[:, :, :1].repeat(8, axis=2)                         # same decay on every channel
    out, hT = oracle.kda_oracle(q, k, v, gs, beta, 1.0, h0=h0, lib_path=lib_path)
    S = np.array(h0[0, 0])
    for t in range(33):
        a = math.exp(float(gs[t, 0, 0]))
        kt, vt = k[t, 0].astype(np.float64), v[t, 0].astype(np.float64)
        S = a * S
        S = S + beta[t, 0] * np.outer(kt, vt - S.T @ kt)
        assert rel_err(out[t, 0], S.T @ q[t, 0].astype(np.float64)) < 1e-12
    assert rel_err(hT[0, 0], S) < 1e-12


def check_one_token(lib_path=None):
    rng = np.random.default_rng(15)
    q, k, v, g, beta, _ = rand_case(rng, 1, 1, 5, 3, with_h0=False)
    out, hT = oracle.kda_oracle(q, k, v, g, beta, 0.25, lib_path=lib_path)
    k1, v1, q1 = (x[0, 0].astype(np.float64) for x in (k, v, q))
    b = float(beta[0, 0])
    assert rel_err(hT[0, 0], b * np.outer(k1, v1)) < 1e-15
    assert rel_err(out[0, 0], 0.25 * b * (k1 @ q1) * v1) < 1e-15


def check_two_tokens_closed_form(lib_path=None):
    rng = np.random.default_rng(16)
    q, k, v, g, beta, _ = rand_case(rng, 2, 1, 4, 3, g_mu=0.0, with_h0=False)
    out, hT = oracle.kda_oracle(q, k, v, g, beta, 0.7, lib_path=lib_path)
    q1, q2 = q[:, 0].astype(np.float64); k1, k2 = k[:, 0].astype(np.float64)
    v1, v2 = v[:, 0].astype(np.float64); b1, b2 = beta[:, 0].astype(np.float64)
    a2 = np.exp(g[1, 0].astype(np.float64))
    ak1 = a2 * k1
    o2 = 0.7 * (b1 * (ak1 @ q2 - b2 * (k2 @ q2) * (k2 @ ak1)) * v1 + b2 * (k2 @ q2) * v2)
    assert rel_err(out[1, 0], o2) < 1e-13
    S2 = b1 * np.outer(ak1, v1) + b2 * np.outer(k2, v2 - b1 * (k2 @ ak1) * v1)
    assert rel_err(hT[0, 0], S2) < 1e-13


def check_overwrite(lib_path=None):
    """Delta-rule overwrite (chapter 3): with alpha = 1, beta = 1 and a unit key,
    writing v under key k makes S^T k read back exactly v, whatever S held."""
    rng = np.random.default_rng(17)
    D = 4
    kk = np.tile(f32([0.5, -0.5, 0.5, 0.5]), (2, 1))[:, None, :]   # |k| = 1 exactly
    v = f32(rng.standard_normal((2, 1, D)))
    q = f32(rng.standard_normal((2, 1, D)))
    h0 = rng.standard_normal((1, 1, D, D))
    z = np.zeros((2, 1, D), np.float32); one = np.ones((2, 1), np.float32)
    kn = kk[0, 0].astype(np.float64)
    for t in (1, 2):
        _, hT = oracle.kda_oracle(q[:t], kk[:t], v[:t], z[:t], one[:t], 1.0, h0=h0,
                                  lib_path=lib_path)
        assert rel_err(hT[0, 0].T @ kn, v[t - 1, 0].astype(np.float64)) < 1e-14


def check_contraction_bound(lib_path=None):
    rng = np.random.default_rng(18)
    T, D = 40, 8
    q, k, v, g, beta, h0 = rand_case(rng, T, 1, D, D)
    prev = np.linalg.norm(h0[0, 0], 2)
    for t in range(1, T + 1):
        _, hT = oracle.kda_oracle(q[:t], k[:t], v[:t], g[:t], beta[:t], 1.0, h0=h0,
                                  lib_path=lib_path)
        cur = np.linalg.norm(hT[0, 0], 2)
        bound = prev + float(beta[t - 1, 0]) * np.linalg.norm(k[t - 1, 0]) * np.linalg.norm(v[t - 1, 0])
        assert cur <= bound * (1 + 1e-12)
        prev = cur


def check_chunkwise_agrees(lib_path=None):
    rng = np.random.default_rng(19)
    for (T, D, C) in [(150, 16, 64), (150, 16, 16), (37, 8, 1), (200, 128, 64)]:
        q, k, v, g, beta, h0 = rand_case(rng, T, 1, D, D)
        out, hT = oracle.kda_oracle(q, k, v, g, beta, 0.125, h0=h0, lib_path=lib_path)
        eo, eS = chunkwise(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0], 0.125, h0[0, 0], C)
        assert rel_err(out[:, 0], eo) < 1e-11, (T, D, C)
        assert rel_err(hT[0, 0], eS) < 1e-11, (T, D, C)


def check_split_and_varlen(lib_path=None):
    rng = np.random.default_rng(20)
    T, H, D = 90, 2, 8
    q, k, v, g, beta, h0 = rand_case(rng, T, H, D, D)
    out, hT = oracle.kda_oracle(q, k, v, g, beta, 1.0, h0=h0, lib_path=lib_path)
    t0 = 41
    o1, h1 = oracle.kda_oracle(q[:t0], k[:t0], v[:t0], g[:t0], beta[:t0], 1.0, h0=h0,
                               lib_path=lib_path)
    o2, h2 = oracle.kda_oracle(q[t0:], k[t0:], v[t0:], g[t0:], beta[t0:], 1.0, h0=h1,
                               lib_path=lib_path)
    assert rel_err(np.concatenate([o1, o2]), out) < 1e-13
    assert rel_err(h2, hT) < 1e-13
    # a packed batch of three sequences equals three separate calls
    cu = [0, 13, 13, 90]                      # includes an empty sequence
    h0s = 0.1 * rng.standard_normal((3, H, D, D))
    ov, hv = oracle.kda_oracle(q, k, v, g, beta, 1.0, cu_seqlens=cu, h0=h0s, lib_path=lib_path)
    for s in range(3):
        a, b = cu[s], cu[s + 1]
        if b == a:
            assert np.array_equal(hv[s], h0s[s])
            continue
        os_, hs = oracle.kda_oracle(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], 1.0,
                                    h0=h0s[s:s + 1], lib_path=lib_path)
        assert rel_err(ov[a:b], os_) < 1e-15
        assert rel_err(hv[s], hs[0]) < 1e-15


def check_golden(lib_path=None):
    fx = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, *vals = line.split()
        fx[name] = np.array([float(x) for x in vals])
    q = f32(fx["q"].reshape(2, 1, 2)); k = f32(fx["k"].reshape(2, 1, 2))
    v = f32(fx["v"].reshape(2, 1, 2)); g = f32(fx["g"].reshape(2, 1, 2))
    beta = f32(fx["beta"].reshape(2, 1))
    out, hT = oracle.kda_oracle(q, k, v, g, beta, fx["scale"][0], lib_path=lib_path)
    assert np.array_equal(out.reshape(-1), fx["expect_out"])
    assert np.array_equal(hT.reshape(-1), fx["expect_state"])


PINS = [check_dplr_identity, check_explicit_matrix, check_beta_zero, check_alpha_one_is_deltanet,
        check_scalar_gate_is_gated_deltanet, check_one_token, check_two_tokens_closed_form,
        check_overwrite, check_contraction_bound, check_chunkwise_agrees, check_split_and_varlen,
        check_golden]


@pytest.mark.parametrize("check", PINS, ids=[c.__name__ for c in PINS])
def test_pin(check, oracle_mod):
    check()


def test_thread_count_invariance(oracle_mod):
    rng = np.random.default_rng(21)
    q, k, v, g, beta, _ = rand_case(rng, 64, 5, 16, 16)
    cu = [0, 10, 30, 64]
    h0 = 0.1 * rng.standard_normal((3, 5, 16, 16))
    a = oracle.kda_oracle(q, k, v, g, beta, 1.0, cu_seqlens=cu, h0=h0, nthreads=1)
    b = oracle.kda_oracle(q, k, v, g, beta, 1.0, cu_seqlens=cu, h0=h0, nthreads=7)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_rejects_malformed(oracle_mod):
    rng = np.random.default_rng(22)
    q, k, v, g, beta, _ = rand_case(rng, 8, 1, 4, 4)
    with pytest.raises(ValueError):
        oracle.kda_oracle(q, k, v, g, beta, 1.0, cu_seqlens=[0, 5, 3, 8])
    with pytest.raises(ValueError):
        oracle.kda_oracle(q, k, v, g, beta, 1.0, cu_seqlens=[1, 8])


@pytest.mark.parametrize("mutant", [1, 2, 3, 4, 5])
def test_mutants_are_caught(mutant, tmp_path, oracle_mod):
    path = oracle.build(mutant=mutant, out_path=str(tmp_path / f"mut{mutant}.so"))
    failed = []
    for check in PINS:
        try:
            check(lib_path=path)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"planted mistake {mutant} passed every pin"


def test_segments_compose_through_their_affine_maps():
    """The state-update equation is affine in the state, so a segment maps S_in to M S_in + B,
    with M the final state of a run from the identity with v = 0 and B the final state of a run
    from zero. Scanning (M, B) over segments and re-running each from the scanned state must
    reproduce one run over the whole sequence (the construction of a segment-parallel scan)."""
    rng = np.random.default_rng(21)
    T, H, D = 300, 2, 16
    f = lambda *s: rng.normal(size=s).astype(np.float32)
    q, v = f(1, T, H, D), f(1, T, H, D)
    k = (f(1, T, H, D) / 4).astype(np.float32)
    g = (-np.abs(f(1, T, H, D)) * 0.1).astype(np.float32)
    beta = rng.uniform(0, 1, size=(1, T, H)).astype(np.float32)
    h0 = rng.normal(size=(1, H, D, D)) * 0.3
    ref_out, ref_hT = oracle.kda_oracle(q, k, v, g, beta, 0.5, h0=h0)
    eye = np.broadcast_to(np.eye(D), (1, H, D, D)).copy()
    S, outs = h0.copy(), []
    for a, b in ((0, 100), (100, 230), (230, 300)):
        sl = lambda x: np.ascontiguousarray(x[:, a:b])
        _, M = oracle.kda_oracle(sl(q), sl(k), np.zeros_like(sl(v)), sl(g), sl(beta), 0.5, h0=eye)
        _, B = oracle.kda_oracle(sl(q), sl(k), sl(v), sl(g), sl(beta), 0.5)
        o, _ = oracle.kda_oracle(sl(q), sl(k), sl(v), sl(g), sl(beta), 0.5, h0=S)
        outs.append(o)
        S = np.einsum("hij,hjk->hik", M[0], S[0])[None] + B
    out = np.concatenate(outs, axis=1)
    assert np.abs(out - ref_out).max() <= 1e-12 * np.abs(ref_out).max()
    assert np.abs(S - ref_hT).max() <= 1e-12 * np.abs(ref_hT).max()
