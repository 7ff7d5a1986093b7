"""Pins of the oracle's backward pass (kda_oracle_bwd), on the CPU.

The backward walks the tokens in reverse through the delta-rule form of the
state-update equation. It is pinned to derivatives of an fp64 forward written
here in the other, DPLR matrix form of the same equation (Kimi Linear feature
page, chapter 4: S_t = (Diag(alpha_t) - beta_t k_t (k_t (.) alpha_t)^T) S_{t-1}
+ beta_t k_t v_t^T, o_t = scale S_t^T q_t). That forward is itself checked
against the pinned C forward oracle. Central finite differences, element by
element on tiny cases and along random directions on a case that crosses the
backward's 64-token checkpoints, must match the analytic gradients; so must
a handful of exact special cases.
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
