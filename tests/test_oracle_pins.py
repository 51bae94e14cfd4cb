"""Pins of the float64 oracle against facts the pages and the mathematics fix.

Every check here is independent of the oracle's own formulas: closed forms, the
first-order optimality condition of the frame objective, brute-force least
squares, a hand-derived worked example, set statements about the frame ranges,
and an independent library convolution. None of these tests needs a GPU.
"""
import json
import os
from types import SimpleNamespace

import numpy as np
import pytest
import torch

from oracle import vda_oracle as vo

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _frame_update(S_prev, K, V, beta, alpha):
    A, B = vo.frame_stats(K, V, beta)
    M, C = vo.frame_solve(A, B, alpha)
    return S_prev @ M + C


def _lstsq_frame(S_bar, K, V, beta):
    """argmin_S 1/2|S - S_bar|^2 + 1/2 sum_u beta_u |S k_u - v_u|^2, row by row.

    Row i of S solves the stacked least-squares system
    [I; Diag(sqrt(beta)) K] s_i = [s_bar_i; sqrt(beta) * V[:, i]].
    """
    d_v, d_k = S_bar.shape
    sb = np.sqrt(beta)
    Amat = np.vstack([np.eye(d_k), sb[:, None] * K])
    S = np.zeros_like(S_bar)
    for i in range(d_v):
        rhs = np.concatenate([S_bar[i], sb * V[:, i]])
        S[i] = np.linalg.lstsq(Amat, rhs, rcond=None)[0]
    return S


# ---------------------------------------------------------------- (a) U = 1
@pytest.mark.parametrize("seed", range(6))
def test_single_token_reduces_to_token_delta_rule(seed):
    """U = 1, |k| = 1: Sherman-Morrison turns the frame solve into the token rule
    S = Sbar + beta/(1+beta) (v - Sbar k) k^T (the token rule of the pages with an
    effective write strength beta/(1+beta))."""
    r = _rng(seed)
    d_k, d_v = 5, 4
    S_prev = r.normal(size=(d_v, d_k))
    k = _unit(r.normal(size=d_k))
    v = r.normal(size=d_v)
    beta = float(r.uniform(0.05, 3.0))
    alpha = r.uniform(0.0, 1.0, size=d_k)
    got = _frame_update(S_prev, k[None, :], v[None, :], np.array([beta]), alpha)
    S_bar = S_prev * alpha[None, :]
    b_eff = beta / (1.0 + beta)
    want = S_bar + b_eff * np.outer(v - S_bar @ k, k)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


# ------------------------------------------------- (b) optimality condition
@pytest.mark.parametrize("seed", range(6))
def test_gradient_of_frame_objective_vanishes(seed):
    r = _rng(100 + seed)
    d_k, d_v, U = 6, 5, 9
    S_prev = r.normal(size=(d_v, d_k))
    K = _unit(r.normal(size=(U, d_k)))
    V = r.normal(size=(U, d_v))
    beta = _sigmoid(r.normal(size=U))
    alpha = _sigmoid(r.normal(size=d_k) + 3)
    S = _frame_update(S_prev, K, V, beta, alpha)
    S_bar = S_prev * alpha[None, :]
    grad = S - S_bar
    for u in range(U):  # token by token
        grad = grad + beta[u] * np.outer(S @ K[u] - V[u], K[u])
    assert np.abs(grad).max() <= 1e-12 * max(1.0, np.abs(S).max())


# ------------------------------------------------------- (c) non-expansion
@pytest.mark.parametrize("case", ["random", "alpha_one", "alpha_zero", "beta_zero", "big_beta"])
def test_transition_is_non_expansive(case):
    r = _rng(7)
    d, U = 8, 12
    for _ in range(20):
        K = r.normal(size=(U, d))  # not normalised: the bound holds for any keys
        beta = r.uniform(0, 2, size=U)
        alpha = r.uniform(0, 1, size=d)
        if case == "alpha_one":
            alpha[:] = 1.0
        elif case == "alpha_zero":
            alpha[: d // 2] = 0.0
        elif case == "beta_zero":
            beta[:] = 0.0
        elif case == "big_beta":
            beta *= 1e3
        A, _ = vo.frame_stats(K, np.zeros((U, d)), beta)
        M, _ = vo.frame_solve(A, np.zeros((d, d)), alpha)
        assert np.linalg.svd(M, compute_uv=False).max() <= 1.0 + 1e-12
        lam = np.linalg.eigvalsh(np.eye(d) + A)
        assert lam.min() >= 1.0 - 1e-12
        assert lam.max() <= 1.0 + np.sum(beta * np.sum(K * K, axis=1)) + 1e-9
        if case == "alpha_one" and np.all(beta == 0):
            np.testing.assert_allclose(M, np.eye(d), atol=1e-15)


def test_beta_zero_frame_is_pure_decay():
    r = _rng(8)
    d, U = 5, 7
    S_prev = r.normal(size=(d, d))
    K, V = r.normal(size=(U, d)), r.normal(size=(U, d))
    alpha = r.uniform(0, 1, size=d)
    got = _frame_update(S_prev, K, V, np.zeros(U), alpha)
    np.testing.assert_allclose(got, S_prev * alpha[None, :], atol=1e-14)


# ------------------------------------------------- (d) brute-force lstsq
@pytest.mark.parametrize("seed", range(8))
def test_frame_solve_matches_bruteforce_least_squares(seed):
    r = _rng(200 + seed)
    d_k = int(r.integers(1, 9))
    d_v = int(r.integers(1, 9))
    U = int(r.integers(1, 7))
    S_prev = r.normal(size=(d_v, d_k))
    K = r.normal(size=(U, d_k))
    V = r.normal(size=(U, d_v))
    beta = r.uniform(0, 2, size=U)
    alpha = r.uniform(0, 1, size=d_k)
    got = _frame_update(S_prev, K, V, beta, alpha)
    want = _lstsq_frame(S_prev * alpha[None, :], K, V, beta)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-10)


def test_text_state_is_least_squares_from_zero():
    r = _rng(9)
    d_k, d_v, L = 6, 4, 5
    K = r.normal(size=(L, d_k))
    V = r.normal(size=(L, d_v))
    beta = r.uniform(0.1, 1.5, size=L)
    A, B = vo.frame_stats(K, V, beta)
    got = vo.text_state(A, B)
    want = _lstsq_frame(np.zeros((d_v, d_k)), K, V, beta)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------- (e) partition
@pytest.mark.parametrize("T,c", [(12, 2), (20, 5), (40, 5), (120, 5), (7, 1), (9, 3), (13, 5), (6, 4), (3, 1)])
def test_frame_ranges_partition_the_clip(T, c):
    anchors = set(vo.anchor_frames(T))
    for t in range(T):
        j = vo.chunk_of(t, c)
        fwd = set(vo.forward_frames(j, c))
        rev = set(vo.reverse_frames(j, c, T))
        win = set(vo.window_frames(j, c, T))
        assert fwd | rev | win | anchors == set(range(T))
        assert not fwd & rev
        assert not fwd & (win | anchors)
        assert not rev & (win | anchors)
        assert t in win
        # The window is the chunks j-1..j+1 restricted to the clip.
        assert win == {f for f in range(T) if j - 1 <= f // c <= j + 1}


# --------------------------------------------------- worked example (golden)
def _scalar_inputs(T=7, c=1):
    d, U, L = 1, 1, 1
    cfg = SimpleNamespace(B=1, H=1, d=d, T=T, grid_h=1, grid_w=1, chunk=c, L=L,
                          prep_conv=False, norm_gate=False)
    Q = np.ones((1, T * U, 1, d))
    K = np.ones((1, T * U, 1, d))
    V = np.arange(T, dtype=np.float64).reshape(1, T, 1, 1)
    inp = dict(Q=Q, K=K, V=V, K_txt=np.ones((1, L, 1, d)), V_txt=np.full((1, L, 1, d), 2.0),
               alpha=np.full((1, 1, T, d), 0.5), beta=np.ones((1, 1, T, U)),
               beta_txt=np.ones((1, 1, L)))
    return cfg, inp


def test_hand_derived_scalar_example():
    with open(os.path.join(GOLDEN, "hand_scalar_d1.json")) as f:
        gold = json.load(f)
    cfg, inp = _scalar_inputs()
    res = vo.vda_reference(inp, cfg)
    o = res["O"][0, :, 0, 0]
    for t, val in gold["o_over_q"].items():
        assert o[int(t)] == pytest.approx(val, abs=1e-14)
    it = res["inter"][(0, 0)]
    for t, val in gold["forward_states"].items():
        assert it["F"][int(t)][0, 0] == pytest.approx(val, abs=1e-14)
    for t, val in gold["reverse_states"].items():
        assert it["R"][int(t)][0, 0] == pytest.approx(val, abs=1e-14)


# ------------------------------------------------- whole-branch brute force
def _random_case(seed, B=1, H=2, d=3, T=8, gh=1, gw=3, c=2, L=2, prep=False, gate=False):
    r = _rng(seed)
    U = gh * gw
    cfg = SimpleNamespace(B=B, H=H, d=d, T=T, grid_h=gh, grid_w=gw, chunk=c, L=L,
                          prep_conv=prep, norm_gate=gate)
    inp = dict(
        Q=r.normal(size=(B, T * U, H, d)), K=r.normal(size=(B, T * U, H, d)) * 0.7,
        V=r.normal(size=(B, T * U, H, d)), K_txt=r.normal(size=(B, L, H, d)) * 0.7,
        V_txt=r.normal(size=(B, L, H, d)), alpha=_sigmoid(r.normal(size=(B, H, T, d)) + 1.0),
        beta=_sigmoid(r.normal(size=(B, H, T, U))), beta_txt=_sigmoid(r.normal(size=(B, H, L))))
    if prep:
        inp["conv_w"] = r.normal(size=(H * d * 60,)) * 0.3
    if gate:
        inp["gate"] = r.normal(size=(B, T * U, H, d))
    return cfg, inp


def _bruteforce_branch(cfg, inp):
    """The whole linear branch from its statement, independent of the oracle:
    per query frame, re-run the frame objective by least squares over exactly the
    frames outside the chunk window [j-1, j+1] that are not anchors."""
    B, H, d, T, c = cfg.B, cfg.H, cfg.d, cfg.T, cfg.chunk
    U = cfg.grid_h * cfg.grid_w
    O = np.zeros((B, T * U, H, d))
    for b in range(B):
        for h in range(H):
            Kt, Vt = inp["K_txt"][b, :, h], inp["V_txt"][b, :, h]
            S_T = _lstsq_frame(np.zeros((d, d)), Kt, Vt, inp["beta_txt"][b, h])
            for t in range(1, T - 1):
                j = t // c
                before = [f for f in range(1, T - 1) if f < c * (j - 1)]
                after = [f for f in range(1, T - 1) if f >= c * (j + 2)]
                S_sum = np.zeros((d, d))
                for frames in (before, after[::-1]):
                    S = S_T / 2
                    for f in frames:
                        Kf = inp["K"][b, f * U:(f + 1) * U, h]
                        Vf = inp["V"][b, f * U:(f + 1) * U, h]
                        S = _lstsq_frame(S * inp["alpha"][b, h, f][None, :], Kf, Vf,
                                         inp["beta"][b, h, f])
                    S_sum = S_sum + S
                for u in range(U):
                    q = inp["Q"][b, t * U + u, h]
                    O[b, t * U + u, h] = [sum(S_sum[i, k] * q[k] for k in range(d)) for i in range(d)]
    return O


@pytest.mark.parametrize("seed,T,c", [(0, 8, 2), (1, 9, 3), (2, 7, 1), (3, 12, 2), (4, 11, 3)])
def test_whole_branch_matches_bruteforce(seed, T, c):
    cfg, inp = _random_case(seed, T=T, c=c)
    got = vo.vda_reference(inp, cfg)["O"]
    want = _bruteforce_branch(cfg, inp)
    np.testing.assert_allclose(got, want, rtol=1e-9, atol=1e-11)


def test_boundary_states_equal_set_based_recurrence():
    cfg, inp = _random_case(11, H=1, d=4, T=20, gw=2, c=3)
    it = vo.vda_reference(inp, cfg)["inter"][(0, 0)]
    M, C, S_T = it["M"], it["C"], it["S_T"]
    for j in range(-(-cfg.T // cfg.chunk)):
        S = S_T / 2
        for f in [f for f in range(1, cfg.T - 1) if f // cfg.chunk < j - 1]:
            S = S @ M[f] + C[f]
        np.testing.assert_allclose(it["S_fwd"][j], S, atol=1e-13)
        S = S_T / 2
        for f in sorted([f for f in range(1, cfg.T - 1) if f // cfg.chunk > j + 1], reverse=True):
            S = S @ M[f] + C[f]
        np.testing.assert_allclose(it["S_rev"][j], S, atol=1e-13)


# ------------------------------------------------------ global properties
def test_text_counted_once():
    """beta = 0 on video and alpha = 1 make every frame the identity map, so every
    non-anchor query reads exactly S_T q (S_T/2 from each direction)."""
    cfg, inp = _random_case(12, H=1, d=4, T=10, gw=2, c=2, L=5)
    inp["beta"][:] = 0.0
    inp["alpha"][:] = 1.0
    got = vo.vda_reference(inp, cfg)["O"]
    S_T = _lstsq_frame(np.zeros((4, 4)), inp["K_txt"][0, :, 0], inp["V_txt"][0, :, 0],
                       inp["beta_txt"][0, 0])
    U = 2
    for t in range(cfg.T):
        for u in range(U):
            q = inp["Q"][0, t * U + u, 0]
            want = S_T @ q if 0 < t < cfg.T - 1 else np.zeros(4)
            np.testing.assert_allclose(got[0, t * U + u, 0], want, atol=1e-12)


def test_flip_symmetry():
    """With T a multiple of c, reversing the frame order maps O[t] to O[T-1-t]."""
    cfg, inp = _random_case(13, T=12, c=3, gw=2)
    U = 2
    flip = dict(inp)
    for key in ("Q", "K", "V"):
        x = inp[key].reshape(1, cfg.T, U, cfg.H, cfg.d)
        flip[key] = x[:, ::-1].reshape(inp[key].shape).copy()
    flip["alpha"] = inp["alpha"][:, :, ::-1].copy()
    flip["beta"] = inp["beta"][:, :, ::-1].copy()
    O = vo.vda_reference(inp, cfg)["O"].reshape(1, cfg.T, U, cfg.H, cfg.d)
    Of = vo.vda_reference(flip, cfg)["O"].reshape(1, cfg.T, U, cfg.H, cfg.d)
    np.testing.assert_allclose(Of[:, ::-1], O, atol=1e-12)


def test_linear_in_values():
    cfg, inp = _random_case(14, T=10, c=2)
    _, other = _random_case(15, T=10, c=2)
    both = dict(inp, V=inp["V"] + other["V"], V_txt=inp["V_txt"] + other["V_txt"])
    o2 = dict(inp, V=other["V"], V_txt=other["V_txt"])
    Oa = vo.vda_reference(inp, cfg)["O"]
    Ob = vo.vda_reference(o2, cfg)["O"]
    Oab = vo.vda_reference(both, cfg)["O"]
    np.testing.assert_allclose(Oab, Oa + Ob, atol=1e-12)
    scaled = dict(inp, V=inp["V"] * -2.5, V_txt=inp["V_txt"] * -2.5)
    np.testing.assert_allclose(vo.vda_reference(scaled, cfg)["O"], -2.5 * Oa, atol=1e-12)


def test_permuting_tokens_inside_a_frame_leaves_states_unchanged():
    cfg, inp = _random_case(16, T=8, c=2, gw=4)
    U = 4
    perm = dict(inp)
    r = _rng(17)
    for key in ("K", "V"):
        perm[key] = inp[key].copy()
    perm["beta"] = inp["beta"].copy()
    for t in range(cfg.T):
        p = r.permutation(U)
        for key in ("K", "V"):
            perm[key][:, t * U:(t + 1) * U] = inp[key][:, t * U + p]
        perm["beta"][:, :, t] = inp["beta"][:, :, t][:, :, p]
    a = vo.vda_reference(inp, cfg)
    b = vo.vda_reference(perm, cfg)
    np.testing.assert_allclose(a["O"], b["O"], atol=1e-12)


def test_anchor_frames_read_zero():
    cfg, inp = _random_case(18, T=9, c=3, gw=2, gate=True)
    cfg.norm_gate = True
    O = vo.vda_reference(inp, cfg)["O"]
    U = 2
    assert np.all(O[:, :U] == 0) and np.all(O[:, (cfg.T - 1) * U:] == 0)
    assert np.all(np.abs(O[:, U:(cfg.T - 1) * U]) > 0)


# ------------------------------------------------------------ feature prep
def test_separable_conv_matches_torch_conv3d():
    """Spatial 5x5 then temporal 5-tap depthwise cross-correlation equals one
    depthwise 3-D cross-correlation whose kernel is the outer product of the two
    filters (zero 'same' padding), computed by torch's conv3d in float64."""
    r = _rng(19)
    T, gh, gw, d = 7, 6, 9, 3
    x = r.normal(size=(T, gh, gw, d))
    ws = r.normal(size=(d, 5, 5))
    wt = r.normal(size=(d, 5))
    got = vo.depthwise_temporal_5(vo.depthwise_spatial_5x5(x, ws), wt)
    xt = torch.from_numpy(x).permute(3, 0, 1, 2)[None]  # [1, d, T, gh, gw]
    w3 = torch.from_numpy(np.einsum("ct,cab->ctab", wt, ws))[:, None]  # [d,1,5,5,5]
    want = torch.nn.functional.conv3d(xt, w3, padding=2, groups=d)[0].permute(1, 2, 3, 0).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_conv_with_delta_filters_is_identity_then_silu():
    r = _rng(20)
    T, gh, gw, d = 5, 4, 6, 2
    X = r.normal(size=(T, gh * gw, d))
    ws = np.zeros((d, 5, 5))
    ws[:, 2, 2] = 1.0
    wt = np.zeros((d, 5))
    wt[:, 2] = 1.0
    got = vo.prep_video_kv(X, ws, wt, gh, gw)
    np.testing.assert_allclose(got, X * _sigmoid(X), atol=1e-14)
    # A shifted delta moves the grid by one column (zero fill at the edge).
    ws2 = np.zeros((d, 5, 5))
    ws2[:, 2, 3] = 1.0  # out[y, x] = in[y, x + 1]
    got2 = vo.depthwise_spatial_5x5(X.reshape(T, gh, gw, d), ws2)
    want2 = np.zeros((T, gh, gw, d))
    want2[:, :, :-1] = X.reshape(T, gh, gw, d)[:, :, 1:]
    np.testing.assert_allclose(got2, want2, atol=1e-15)
    wt2 = np.zeros((d, 5))
    wt2[:, 0] = 1.0  # out[t] = in[t - 2]
    got3 = vo.depthwise_temporal_5(X, wt2)
    want3 = np.zeros_like(X)
    want3[2:] = X[:-2]
    np.testing.assert_allclose(got3, want3, atol=1e-15)


def test_norms_closed_forms():
    x = np.array([[3.0, 4.0], [0.0, 0.0]])
    n = vo.l2_normalize(x, 1e-6)
    np.testing.assert_allclose(n[0], [3 / np.sqrt(25 + 1e-6), 4 / np.sqrt(25 + 1e-6)], rtol=1e-15)
    assert np.all(n[1] == 0)
    o = np.full((1, 8), -2.0)
    y = vo.rms_norm_gate(o, np.zeros((1, 8)), 1e-6)
    np.testing.assert_allclose(y, -0.5 * 2 / np.sqrt(4 + 1e-6), rtol=1e-15)
    o2 = np.array([[1.0, -1.0, 2.0, 0.0]])
    g2 = np.array([[10.0, 0.0, -1.0, 3.0]])
    rms = np.sqrt((1 + 1 + 4 + 0) / 4 + 1e-6)
    np.testing.assert_allclose(vo.rms_norm_gate(o2, g2, 1e-6), o2 / rms * _sigmoid(g2), rtol=1e-15)


def test_prep_branch_matches_bruteforce():
    """Conv workloads: the oracle's prep (conv, SiLU, L2 on K and Q, SiLU/L2 on text)
    followed by the branch equals the brute-force branch on features prepared with
    torch's conv3d."""
    cfg, inp = _random_case(21, H=2, d=3, T=7, gh=3, gw=4, c=2, L=3, prep=True, gate=True)
    got = vo.vda_reference(inp, cfg)["O"]
    B, H, d, T = cfg.B, cfg.H, cfg.d, cfg.T
    gh, gw = cfg.grid_h, cfg.grid_w
    U = gh * gw
    w = inp["conv_w"]
    hd = H * d
    parts = [w[:hd * 25].reshape(H, d, 5, 5), w[hd * 25:hd * 30].reshape(H, d, 5),
             w[hd * 30:hd * 55].reshape(H, d, 5, 5), w[hd * 55:].reshape(H, d, 5)]

    def conv(x, ws, wt):  # x: [T*U, d] one head
        xt = torch.from_numpy(x.reshape(T, gh, gw, d)).permute(3, 0, 1, 2)[None]
        w3 = torch.from_numpy(np.einsum("ct,cab->ctab", wt, ws))[:, None]
        y = torch.nn.functional.conv3d(xt, w3, padding=2, groups=d)[0].permute(1, 2, 3, 0)
        return y.reshape(T * U, d).numpy()

    prep = dict(inp)
    for key in ("Q", "K", "V", "K_txt", "V_txt"):
        prep[key] = inp[key].copy()
    for h in range(H):
        k = conv(inp["K"][0, :, h], parts[0][h], parts[1][h])
        k = k * _sigmoid(k)
        prep["K"][0, :, h] = k / np.sqrt((k * k).sum(-1, keepdims=True) + 1e-6)
        v = conv(inp["V"][0, :, h], parts[2][h], parts[3][h])
        prep["V"][0, :, h] = v * _sigmoid(v)
        q = inp["Q"][0, :, h]
        prep["Q"][0, :, h] = q / np.sqrt((q * q).sum(-1, keepdims=True) + 1e-6)
        kt = inp["K_txt"][0, :, h] * _sigmoid(inp["K_txt"][0, :, h])
        prep["K_txt"][0, :, h] = kt / np.sqrt((kt * kt).sum(-1, keepdims=True) + 1e-6)
        prep["V_txt"][0, :, h] = inp["V_txt"][0, :, h] * _sigmoid(inp["V_txt"][0, :, h])
    lin = _bruteforce_branch(cfg, prep)
    g = inp["gate"]
    want = lin / np.sqrt((lin * lin).mean(-1, keepdims=True) + 1e-6) * _sigmoid(g)
    want[:, :U] = 0
    want[:, (T - 1) * U:] = 0
    np.testing.assert_allclose(got, want, rtol=1e-8, atol=1e-10)
