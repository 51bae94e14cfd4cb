"""Pins of the softmax-branch and hybrid-merge oracle (oracle/hybrid_oracle.py).

Each check rests on something other than the oracle's own code:
  * the density that the four-way anchors add, as printed in "VDN-H3: a hybrid
    attention model that generates MiniMax H3 video faster than playback",
    section "hybrid attention structure" (3.57%), at the H3 workload of
    102 latent frames in chunks of five;
  * a token-pair mask built from the chunk-distance statement of the window
    (|chunk(query) - chunk(key)| <= 1, or either frame an anchor), evaluated as a
    dense masked softmax;
  * the reduction to plain dense attention when the window spans the clip;
  * properties of any softmax attention (convex combinations of the visible
    values, invariance to the order of keys within a frame);
  * closed forms of the gate and the merge.
Planted mistakes in a copy of the oracle must fail these pins.
"""
import inspect
import types

import numpy as np
import pytest

from oracle import hybrid_oracle as ho


def _dense_masked(Q, K, V, mask, scale):
    logits = (Q @ K.T) * scale
    logits = np.where(mask, logits, -np.inf)
    logits = logits - logits.max(axis=1, keepdims=True)
    w = np.exp(logits)
    w = w / w.sum(axis=1, keepdims=True)
    return w @ V


def _pair_mask(T, U, c):
    frame = np.repeat(np.arange(T), U)
    chunk = frame // c
    near = np.abs(chunk[:, None] - chunk[None, :]) <= 1
    anchor_key = (frame[None, :] == 0) | (frame[None, :] == T - 1)
    anchor_query = (frame[:, None] == 0) | (frame[:, None] == T - 1)
    return near | anchor_key | anchor_query


def _rand(seed, T, U, d):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((T * U, d)), rng.standard_normal((T * U, d)), rng.standard_normal((T * U, d)))


def test_anchor_density_matches_the_printed_figure(mod=ho):
    added = mod.attention_density(102, 5, anchors=True) - mod.attention_density(102, 5, anchors=False)
    assert abs(added - 0.0357) <= 1e-4, added


@pytest.mark.parametrize("T,U,c,d", [(9, 3, 2, 4), (13, 2, 3, 5), (7, 4, 1, 3), (20, 1, 5, 2)])
def test_window_softmax_matches_token_pair_mask(T, U, c, d, mod=ho):
    Q, K, V = _rand(T * 100 + U, T, U, d)
    got = mod.window_softmax_head(Q, K, V, T, U, c)
    want = _dense_masked(Q, K, V, _pair_mask(T, U, c), 1.0 / np.sqrt(d))
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("T,U,c,d", [(9, 3, 2, 4), (13, 2, 3, 5), (20, 1, 5, 2)])
def test_sampled_rows_match_the_token_pair_mask(T, U, c, d, mod=ho):
    """The spot-check form (selected query tokens) against the dense masked
    softmax over the token-pair mask, on every row and on a shuffled subset."""
    Q, K, V = _rand(T * 7 + U, T, U, d)
    want = _dense_masked(Q, K, V, _pair_mask(T, U, c), 1.0 / np.sqrt(d))
    rows = np.random.default_rng(3).permutation(T * U)[: max(3, T * U // 3)]
    np.testing.assert_allclose(mod.window_softmax_rows(Q, K, V, T, U, c, rows), want[rows], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(mod.window_softmax_rows(Q, K, V, T, U, c, range(T * U)), want, rtol=1e-12,
                               atol=1e-12)


def test_window_spanning_the_clip_is_dense_attention(mod=ho):
    T, U, c, d = 6, 3, 3, 4  # two chunks: every window covers both
    Q, K, V = _rand(7, T, U, d)
    got = mod.window_softmax_head(Q, K, V, T, U, c)
    logits = Q @ K.T / np.sqrt(d)
    w = np.exp(logits - logits.max(axis=1, keepdims=True))
    want = (w / w.sum(axis=1, keepdims=True)) @ V
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_outputs_are_convex_combinations_of_visible_values(mod=ho):
    T, U, c, d = 15, 2, 3, 3
    Q, K, V = _rand(11, T, U, d)
    got = mod.window_softmax_head(Q, K, V, T, U, c)
    mask = _pair_mask(T, U, c)
    for i in range(T * U):
        vis = V[mask[i]]
        assert np.all(got[i] <= vis.max(axis=0) + 1e-12) and np.all(got[i] >= vis.min(axis=0) - 1e-12)
    # equal visible values are returned exactly (weights sum to one)
    Vc = np.tile(np.arange(1.0, d + 1.0), (T * U, 1))
    np.testing.assert_allclose(mod.window_softmax_head(Q, K, Vc, T, U, c), Vc, rtol=1e-13)
    # a far key with a huge value but outside the window leaves a middle query untouched
    Vf = V.copy()
    far = 12 * U  # frame 12: chunk 4, not visible from frame 4 (chunk 1), not an anchor
    Vf[far] += 1e6
    a = mod.window_softmax_head(Q, K, V, T, U, c)
    b = mod.window_softmax_head(Q, K, Vf, T, U, c)
    np.testing.assert_array_equal(a[4 * U:5 * U], b[4 * U:5 * U])
    assert not np.allclose(a[0:U], b[0:U])  # the first frame sees it


def test_key_order_within_a_frame_does_not_matter(mod=ho):
    T, U, c, d = 9, 4, 2, 3
    Q, K, V = _rand(5, T, U, d)
    perm = np.arange(T * U)
    rng = np.random.default_rng(0)
    for t in range(T):
        perm[t * U:(t + 1) * U] = t * U + rng.permutation(U)
    a = mod.window_softmax_head(Q, K, V, T, U, c)
    b = mod.window_softmax_head(Q, K[perm], V[perm], T, U, c)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_gate_and_merge_closed_forms(mod=ho):
    rng = np.random.default_rng(3)
    O = rng.standard_normal((5, 2, 3))
    np.testing.assert_allclose(mod.softmax_gate(O, np.zeros_like(O)), 0.5 * O)
    g = rng.standard_normal(O.shape)
    np.testing.assert_allclose(mod.softmax_gate(O, g), O / (1.0 + np.exp(-g)))
    np.testing.assert_allclose(mod.softmax_gate(O, np.full(O.shape, 40.0)), O, rtol=1e-15)
    OL = rng.standard_normal(O.shape)
    W_S, W_L = rng.standard_normal((6, 4)), rng.standard_normal((6, 4))
    Y = mod.hybrid_output(O, OL, W_S, W_L)
    # token 2, output column 1, written as the sum over heads and channels
    want = sum(O[2, h, k] * W_S[3 * h + k, 1] + OL[2, h, k] * W_L[3 * h + k, 1] for h in range(2) for k in range(3))
    assert Y.shape == (5, 4) and abs(Y[2, 1] - want) < 1e-12
    np.testing.assert_allclose(mod.hybrid_output(O, OL, W_S, np.zeros_like(W_L)), O.reshape(5, 6) @ W_S)


def test_layer_runs_every_head_and_gates(mod=ho):
    rng = np.random.default_rng(4)
    B, T, U, H, d, c = 2, 7, 2, 3, 4, 2
    Q, K, V, g = (rng.standard_normal((B, T * U, H, d)) for _ in range(4))
    out = mod.window_softmax_layer(Q, K, V, g, T, U, c)
    for b in range(B):
        for h in range(H):
            want = _dense_masked(Q[b, :, h], K[b, :, h], V[b, :, h], _pair_mask(T, U, c), 1.0 / np.sqrt(d))
            np.testing.assert_allclose(out[b, :, h], want / (1.0 + np.exp(-g[b, :, h])), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# Planted mistakes
# ---------------------------------------------------------------------------
MUTATIONS = {
    "window_forward_only": ("return sorted(set(window_frames(chunk_of(t, c), c, T)) | set(anchor_frames(T)))",
                            "return sorted(set(window_frames(chunk_of(t, c) + 1, c, T)) | set(anchor_frames(T)))"),
    "no_anchor_keys": ("return sorted(set(window_frames(chunk_of(t, c), c, T)) | set(anchor_frames(T)))",
                       "return sorted(set(window_frames(chunk_of(t, c), c, T)))"),
    "anchor_rows_windowed": ("    if t in anchor_frames(T):\n        return list(range(T))\n", ""),
    "scale_one_over_d": ("scale = 1.0 / np.sqrt(d_k)", "scale = 1.0 / d_k"),
    "softmax_over_queries": ("w = w / w.sum(axis=1, keepdims=True)", "w = w / w.sum(axis=0, keepdims=True)"),
    "rows_keys_of_wrong_frame": ("    frames = rows // U\n", "    frames = rows // U + 1\n"),
    "gate_sign": ("return O * (1.0 / (1.0 + np.exp(-g)))", "return O * (1.0 / (1.0 + np.exp(g)))"),
    "merge_drops_linear": ("return Ot_S.reshape(N, -1) @ W_S + Ot_L.reshape(N, -1) @ W_L",
                           "return Ot_S.reshape(N, -1) @ W_S"),
    "merge_transposed_heads": ("return Ot_S.reshape(N, -1) @ W_S + Ot_L.reshape(N, -1) @ W_L",
                               "return Ot_S.transpose(0, 2, 1).reshape(N, -1) @ W_S + Ot_L.reshape(N, -1) @ W_L"),
    "density_window_only": ("            pairs += len(visible_frames(t, c, T))",
                            "            pairs += len(window_frames(chunk_of(t, c), c, T))"),
}


def _mutant(name):
    src = inspect.getsource(ho)
    old, new = MUTATIONS[name]
    assert src.count(old) >= 1, name  # a systematic mistake: planted wherever the text occurs
    mod = types.ModuleType("hybrid_oracle_mutant_" + name)
    exec(compile(src.replace(old, new), mod.__name__, "exec"), mod.__dict__)
    return mod


def _checks(mod):
    ok = True
    for fn, args in [
        (test_anchor_density_matches_the_printed_figure, ()),
        (test_window_softmax_matches_token_pair_mask, (9, 3, 2, 4)),
        (test_window_softmax_matches_token_pair_mask, (13, 2, 3, 5)),
        (test_sampled_rows_match_the_token_pair_mask, (13, 2, 3, 5)),
        (test_window_spanning_the_clip_is_dense_attention, ()),
        (test_outputs_are_convex_combinations_of_visible_values, ()),
        (test_key_order_within_a_frame_does_not_matter, ()),
        (test_gate_and_merge_closed_forms, ()),
        (test_layer_runs_every_head_and_gates, ()),
    ]:
        try:
            fn(*args, mod=mod)
        except (AssertionError, IndexError, ValueError):
            ok = False
    return ok


def test_unmutated_copy_passes():
    src = inspect.getsource(ho)
    mod = types.ModuleType("hybrid_oracle_copy")
    exec(compile(src, mod.__name__, "exec"), mod.__dict__)
    assert _checks(mod)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    assert not _checks(_mutant(name)), f"mutation {name} slipped through the pins"
