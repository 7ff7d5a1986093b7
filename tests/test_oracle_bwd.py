"""Pins of the oracle's backward pass (kda_oracle_bwd), on the CPU.

The backward walks the tokens in reverse through the delta-rule form of the
state-update equation. It is pinned to derivatives of an fp64 forward written
here in the other, DPLR matrix form of the same equation (Kimi Linear feature
page, chapter 4: S_t = (Diag(alpha_t) - beta_t k_t (k_t (.) alpha_t)^T) S_{t-1}
+ beta_t k_t v_t^T, o_t = scale S_t^T q_t). That forward is itself checked
against the pinned C forward oracle. Central finite differences, element by
element on tiny cases and along random directions on a case that crosses the
backward's 64-token checkpoints, must match the analytic gradients; so must
a handful of exact special cases. A chunkwise backward of the chunk form the
kernels use (the algebra a backward kernel would follow) must agree with it for
chunk sizes 1 to 64 and ragged sequences.
"""
import numpy as np
import pytest

import oracle


def forward_dplr(q, k, v, g, beta, scale, cu, h0=None):
    """fp64 forward in the DPLR matrix form, token by token. q, k, g: [Ttot, H, Dk];
    v: [Ttot, H, Dv]; beta: [Ttot, H]. Returns (out [Ttot, H, Dv], hT [N, H, Dk, Dv])."""
    Ttot, H, Dk = q.shape
    Dv = v.shape[-1]
    N = len(cu) - 1
    out = np.zeros((Ttot, H, Dv))
    hT = np.zeros((N, H, Dk, Dv))
    for s in range(N):
        for h in range(H):
            S = np.zeros((Dk, Dv)) if h0 is None else h0[s, h].copy()
            for t in range(cu[s], cu[s + 1]):
                a = np.exp(g[t, h])
                M = np.diag(a) - beta[t, h] * np.outer(k[t, h], k[t, h] * a)
                S = M @ S + beta[t, h] * np.outer(k[t, h], v[t, h])
                out[t, h] = scale * S.T @ q[t, h]
            hT[s, h] = S
    return out, hT


def case(seed, lens, H, Dk, Dv, with_h0=True):
    rng = np.random.default_rng(seed)
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    q = rng.normal(size=(T, H, Dk))
    k = rng.normal(size=(T, H, Dk)) / np.sqrt(Dk)
    v = rng.normal(size=(T, H, Dv))
    g = -np.abs(rng.normal(size=(T, H, Dk))) * 0.2   # log-decays below 0
    beta = rng.uniform(0.1, 0.9, size=(T, H))
    h0 = rng.normal(size=(len(lens), H, Dk, Dv)) * 0.3 if with_h0 else None
    dout = rng.normal(size=(T, H, Dv))
    dhT = rng.normal(size=(len(lens), H, Dk, Dv))
    return dict(q=q, k=k, v=v, g=g, beta=beta, h0=h0, cu=cu, dout=dout, dhT=dhT, scale=0.7)


def loss(c, **over):
    x = dict(c, **over)
    out, hT = forward_dplr(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["cu"], x["h0"])
    return float((out * c["dout"]).sum() + (hT * c["dhT"]).sum())


def grads(c, **over):
    x = dict(c, **over)
    return oracle.kda_oracle_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["scale"], x["dout"],
                                 cu_seqlens=x["cu"], h0=x["h0"], dhT=x["dhT"], nthreads=2)


NAMES = ("q", "k", "v", "g", "beta", "h0")


def test_dplr_forward_matches_the_c_oracle():
    c = case(1, [5, 9], H=2, Dk=8, Dv=6)
    f32 = {n: c[n].astype(np.float32) for n in ("q", "k", "v", "g", "beta")}
    ref_out, ref_hT = oracle.kda_oracle(f32["q"], f32["k"], f32["v"], f32["g"], f32["beta"], c["scale"],
                                        cu_seqlens=c["cu"], h0=c["h0"])
    out, hT = forward_dplr(*(f32[n].astype(np.float64) for n in ("q", "k", "v", "g", "beta")), c["scale"],
                           c["cu"], c["h0"])
    assert np.abs(out - ref_out).max() <= 1e-12 * max(1.0, np.abs(ref_out).max())
    assert np.abs(hT - ref_hT).max() <= 1e-12 * max(1.0, np.abs(ref_hT).max())


@pytest.mark.parametrize("lens,Dk,Dv", [([3], 2, 2), ([2, 0, 3], 3, 2), ([4], 2, 3)])
def test_gradients_match_elementwise_finite_differences(lens, Dk, Dv):
    c = case(2 + Dk, lens, H=2, Dk=Dk, Dv=Dv)
    gr = grads(c)
    eps = 1e-6
    for name in NAMES:
        x = c[name]
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            num[idx] = (loss(c, **{name: xp}) - loss(c, **{name: xm})) / (2 * eps)
        ana = gr["d" + name]
        err = np.abs(ana - num).max() / max(1.0, np.abs(num).max())
        assert err <= 1e-7, f"d{name}: {err:.2e}"


def test_gradients_match_directional_derivatives_across_checkpoints():
    # two sequences, one of them longer than two checkpoint blocks (64 tokens)
    c = case(7, [150, 37], H=2, Dk=5, Dv=4)
    gr = grads(c)
    rng = np.random.default_rng(8)
    eps = 1e-6
    for name in NAMES:
        for _ in range(2):
            d = rng.normal(size=c[name].shape)
            num = (loss(c, **{name: c[name] + eps * d}) - loss(c, **{name: c[name] - eps * d})) / (2 * eps)
            ana = float((gr["d" + name] * d).sum())
            assert abs(ana - num) <= 1e-7 * max(1.0, abs(num)), f"d{name}: {ana} vs {num}"


def test_zero_beta_leaves_keys_and_values_without_gradient():
    c = case(3, [6, 4], H=1, Dk=4, Dv=3)
    gr = grads(c, beta=np.zeros_like(c["beta"]))
    assert np.all(gr["dk"] == 0.0) and np.all(gr["dv"] == 0.0)
    assert np.any(gr["dbeta"] != 0.0)   # beta itself still matters


def test_zero_cotangents_give_zero_gradients():
    c = case(4, [5], H=2, Dk=3, Dv=3)
    gr = grads(c, dout=np.zeros_like(c["dout"]), dhT=np.zeros_like(c["dhT"]))
    for n in ("dq", "dk", "dv", "dg", "dbeta", "dh0"):
        assert np.all(gr[n] == 0.0), n


def test_empty_sequence_passes_the_final_state_gradient_to_the_initial_state():
    c = case(5, [3, 0], H=1, Dk=3, Dv=2)
    gr = grads(c)
    assert np.array_equal(gr["dh0"][1], c["dhT"][1])


def test_gradients_are_linear_in_the_cotangents():
    c = case(6, [7], H=1, Dk=4, Dv=4)
    rng = np.random.default_rng(9)
    d2o, d2s = rng.normal(size=c["dout"].shape), rng.normal(size=c["dhT"].shape)
    g1 = grads(c)
    g2 = grads(c, dout=d2o, dhT=d2s)
    g12 = grads(c, dout=c["dout"] + d2o, dhT=c["dhT"] + d2s)
    for n in ("dq", "dk", "dv", "dg", "dbeta", "dh0"):
        assert np.allclose(g12[n], g1[n] + g2[n], rtol=1e-12, atol=1e-12), n


def chunkwise_backward(c, C):
    """fp64 chunkwise backward of the chunk form the kernels use (per chunk, Gam the in-chunk
    running log-decay, Kd = K e^Gam, Qd = Q e^Gam, Kn = K e^-Gam, Kt = K e^(Gam_last - Gam)):

        A_kk = strict_lower(Diag(beta) Kd Kn^T),  A_qk = lower(Qd Kn^T),  T = (I + A_kk)^-1
        X = V - Kd S0,  D = T Diag(beta) X,  O = scale (Qd S0 + A_qk D)
        S1 = Diag(e^Gam_last) S0 + Kt^T D

    written backwards chunk by chunk from dO and the final-state gradient. The blueprint of a
    chunkwise backward kernel; here it pins, and is pinned by, the token-by-token backward."""
    q, k, v, g, beta, cu, scale = c["q"], c["k"], c["v"], c["g"], c["beta"], c["cu"], c["scale"]
    Ttot, H, Dk = q.shape
    Dv = v.shape[-1]
    N = len(cu) - 1
    res = {n: np.zeros_like(c[n]) for n in ("q", "k", "v", "g", "beta")}
    dh0 = np.zeros((N, H, Dk, Dv))
    for s in range(N):
        for h in range(H):
            bounds = [(t0, min(t0 + C, cu[s + 1])) for t0 in range(cu[s], cu[s + 1], C)]
            # forward: the state at every chunk start
            S = np.zeros((Dk, Dv)) if c["h0"] is None else c["h0"][s, h].copy()
            starts, parts = [], []
            for t0, t1 in bounds:
                K, Q, V = k[t0:t1, h], q[t0:t1, h], v[t0:t1, h]
                Gam = np.cumsum(g[t0:t1, h], axis=0)
                b = beta[t0:t1, h]
                Kd, Qd, Kn = K * np.exp(Gam), Q * np.exp(Gam), K * np.exp(-Gam)
                Kt = K * np.exp(Gam[-1] - Gam)
                B = Kd @ Kn.T
                Akk = np.tril(b[:, None] * B, -1)
                Aqk = np.tril(Qd @ Kn.T, 0)
                T = np.linalg.inv(np.eye(len(b)) + Akk)
                X = V - Kd @ S
                Dl = T @ (b[:, None] * X)
                starts.append(S.copy())
                parts.append((K, Q, Gam, b, Kd, Qd, Kn, Kt, B, Aqk, T, X, Dl))
                S = np.exp(Gam[-1])[:, None] * S + Kt.T @ Dl
            # backward, last chunk first
            dS = c["dhT"][s, h].copy()
            for (t0, t1), S0, (K, Q, Gam, b, Kd, Qd, Kn, Kt, B, Aqk, T, X, Dl) in \
                    reversed(list(zip(bounds, starts, parts))):
                dO = c["dout"][t0:t1, h]
                eC = np.exp(Gam[-1])
                # O = scale (Qd S0 + Aqk D)
                dQd = scale * dO @ S0.T
                dS0 = scale * Qd.T @ dO
                dAqk = np.tril(scale * dO @ Dl.T, 0)
                dD = scale * Aqk.T @ dO
                # S1 = Diag(e^Gam_last) S0 + Kt^T D
                dS0 += eC[:, None] * dS
                dGlast = eC * (dS * S0).sum(axis=1)
                dKt = Dl @ dS.T
                dD += Kt @ dS
                # D = T Diag(beta) X
                Tp = T * b[None, :]
                dTp = dD @ X.T
                dX = Tp.T @ dD
                dV = dX
                dKd = -dX @ S0.T
                dS0 -= Kd.T @ dX
                db = (dTp * T).sum(axis=0)
                dT = dTp * b[None, :]
                # T = (I + Akk)^-1 ; Akk = strict_lower(Diag(beta) B)
                dAkk = np.tril(-T.T @ dT @ T.T, -1)
                db += (dAkk * B).sum(axis=1)
                dB = b[:, None] * dAkk
                dKd += dB @ Kn
                dKn = dB.T @ Kd
                # Aqk = lower(Qd Kn^T)
                dQd += dAqk @ Kn
                dKn += dAqk.T @ Qd
                # the decayed factors back to K, Q and the running log-decay
                dK = dKd * np.exp(Gam) + dKn * np.exp(-Gam) + dKt * np.exp(Gam[-1] - Gam)
                dQ = dQd * np.exp(Gam)
                dGam = dKd * Kd + dQd * Qd - dKn * Kn - dKt * Kt
                dGam[-1] += dGlast + (dKt * Kt).sum(axis=0)
                res["k"][t0:t1, h] = dK
                res["q"][t0:t1, h] = dQ
                res["v"][t0:t1, h] = dV
                res["beta"][t0:t1, h] = db
                res["g"][t0:t1, h] = np.cumsum(dGam[::-1], axis=0)[::-1]   # Gam = cumsum(g)
                dS = dS0
            dh0[s, h] = dS
    return {"d" + n: a for n, a in res.items()} | {"dh0": dh0}


@pytest.mark.parametrize("C", [1, 4, 16, 64])
def test_chunkwise_backward_equals_the_token_by_token_backward(C):
    c = case(11, [70, 5, 0, 33], H=2, Dk=6, Dv=5)
    ref = grads(c)
    got = chunkwise_backward(c, C)
    for n in ("dq", "dk", "dv", "dg", "dbeta", "dh0"):
        err = np.abs(got[n] - ref[n]).max() / max(1.0, np.abs(ref[n]).max())
        assert err <= 1e-10, f"C={C} {n}: {err:.2e}"
