"""Parity of the softmax branch (vda_window_attention, tcgen05) with the float64
oracle in oracle/hybrid_oracle.py, element by element.

Bound: relative Frobenius error <= 2e-2 over the output (bf16 storage), per
(head, frame) and per token (|o_gpu - o_ref| <= 2e-2 max(|o_ref|, 5% of the
head's RMS token norm)). Sources of error: bf16 rounding of the probabilities
fed to the P V product (2^-9 relative per weight) and of the output; the logits
and the running sums are fp32. Small clips are compared on every token; the
H3-like clip at full size on sampled query tokens of every group (first and last
token of every tile, both anchor frames, random tokens), which the oracle can
compute one by one.
"""
import numpy as np
import pytest
import torch

from frame_level_delta_b200 import vda as V
from frame_level_delta_b200.inputs import CONFIGS, make_attention_inputs, make_merge_inputs
from oracle import hybrid_oracle as ho
from tests.parity import TOL_O, local_output_errors, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    V.lib()


def _oracle(cfg, inp, gate: bool):
    Q, K, Vv = (inp[k].double().numpy() for k in ("Q", "K", "V"))
    if gate:
        return ho.window_softmax_layer(Q, K, Vv, inp["gate"].double().numpy(), cfg.T, cfg.U, cfg.chunk)
    out = np.zeros(Vv.shape)
    for b in range(cfg.B):
        for h in range(cfg.H):
            out[b, :, h] = ho.window_softmax_head(Q[b, :, h], K[b, :, h], Vv[b, :, h], cfg.T, cfg.U, cfg.chunk)
    return out


def _run(cfg, inp, gate: bool, heads=None):
    dev = torch.device("cuda:0")
    d = {k: v.to(dev) for k, v in inp.items()}
    ctx = V.VDA(cfg, device=dev, heads=heads)
    O = ctx.window_attention(d["Q"], d["K"], d["V"], d["gate"] if gate else None)
    torch.cuda.synchronize()
    assert ctx.poll_device_status() == 0
    return O.double().cpu().numpy()


def _check(cfg, got, want):
    tol = TOL_O["bf16"]
    err = rel_fro(got, want)
    assert err <= tol, err
    # Every frame's queries are outputs here, anchors included: a local view of
    # the whole clip (the linear branch's helper skips the anchors).
    pairs = [(b, h) for b in range(cfg.B) for h in range(cfg.H)]
    pad = np.zeros((cfg.B, cfg.U, cfg.H, cfg.d))
    wide = cfg.with_(T=cfg.T + 2)
    loc = local_output_errors(wide, np.concatenate([pad, got, pad], axis=1),
                              np.concatenate([pad, want, pad], axis=1), pairs)
    assert loc["frame"] <= tol and loc["token_ratio"] <= 1.0, loc
    return err


CASES = [
    # name, overrides of the small bf16 workload, logit spread, gate
    ("d64_flat", dict(H=2, d=64, T=10, grid_h=6, grid_w=7, chunk=2), 1.0, True),
    ("d64_peaked", dict(H=2, d=64, T=10, grid_h=6, grid_w=7, chunk=2), 4.0, True),
    ("d128_peaked_ragged", dict(H=2, d=128, T=11, grid_h=5, grid_w=9, chunk=3), 4.0, True),
    ("d128_very_peaked", dict(H=1, d=128, T=9, grid_h=8, grid_w=8, chunk=2), 30.0, True),
    ("d128_no_gate", dict(H=2, d=128, T=8, grid_h=4, grid_w=16, chunk=2), 2.0, False),
    ("d128_chunk_one", dict(H=1, d=128, T=7, grid_h=3, grid_w=5, chunk=1), 3.0, True),
    ("d128_window_spans_clip", dict(H=1, d=128, T=6, grid_h=6, grid_w=6, chunk=5), 3.0, True),
    ("d128_T_not_multiple_of_c", dict(H=1, d=128, T=13, grid_h=4, grid_w=10, chunk=5), 3.0, True),
    ("d128_single_token_frames", dict(H=2, d=128, T=12, grid_h=1, grid_w=1, chunk=2), 3.0, True),
    ("d128_batch_two", dict(B=2, H=2, d=128, T=8, grid_h=5, grid_w=5, chunk=2), 3.0, True),
    ("d128_three_frames", dict(H=1, d=128, T=3, grid_h=7, grid_w=7, chunk=1), 3.0, True),
]


@pytest.mark.parametrize("name,kw,spread,gate", CASES, ids=[c[0] for c in CASES])
def test_window_attention_matches_oracle(name, kw, spread, gate):
    cfg = CONFIGS["small"].with_(name=name, **kw)
    inp = make_attention_inputs(cfg, logit_std=spread, gate=gate)
    _check(cfg, _run(cfg, inp, gate), _oracle(cfg, inp, gate))


def test_window_attention_head_slices():
    """Three contexts over head slices of one batch write exactly their heads."""
    cfg = CONFIGS["small"].with_(H=5, d=128, T=9, grid_h=5, grid_w=8, chunk=2)
    inp = make_attention_inputs(cfg, logit_std=3.0)
    whole = _run(cfg, inp, True)
    dev = torch.device("cuda:0")
    d = {k: v.to(dev) for k, v in inp.items()}
    O = torch.full_like(d["Q"], float("nan"))
    for h0, n in ((0, 2), (2, 1), (3, 2)):
        V.VDA(cfg, device=dev, heads=(h0, n)).window_attention(d["Q"], d["K"], d["V"], d["gate"], O)
        torch.cuda.synchronize()
        assert torch.isnan(O[:, :, h0 + n:]).all()
    assert np.array_equal(O.double().cpu().numpy(), whole)


def test_window_attention_rejects_unsupported_storage():
    cfg = CONFIGS["tiny"]  # fp32, d = 16: no tensor-core form
    inp = make_attention_inputs(cfg)
    d = {k: v.cuda() for k, v in inp.items()}
    with pytest.raises(V.VDAError):
        V.VDA(cfg).window_attention(d["Q"], d["K"], d["V"], d["gate"])


def _sample_rows(cfg, rng):
    U, T, c = cfg.U, cfg.T, cfg.chunk
    rows = set(range(0, U, 97)) | set(range((T - 1) * U, T * U, 97)) | {U - 1, T * U - 1}
    for j in range(cfg.J):
        lo, hi = max(c * j, 1) * U, min(c * (j + 1), T - 1) * U
        for a in range(lo, hi, 128):
            rows |= {a, min(a + 127, hi - 1)}
    rows |= set(int(x) for x in rng.integers(0, T * U, 200))
    return sorted(rows)


@pytest.mark.parametrize("spread", [1.0, 4.0])
def test_window_attention_h3_full_size_sampled_rows(spread):
    """The H3-like clip at full size (24 heads, 40 frames of 1560 tokens, chunks
    of 5): sampled query tokens of three heads against the oracle's rows."""
    cfg = CONFIGS["h3"]
    inp = make_attention_inputs(cfg, logit_std=spread)
    got = _run(cfg, inp, True)
    assert np.isfinite(got).all()
    rng = np.random.default_rng(0)
    rows = _sample_rows(cfg, rng)
    tol = TOL_O["bf16"]
    for h in (0, 11, 23):
        Q, K, Vv = (inp[k][0, :, h].double().numpy() for k in ("Q", "K", "V"))
        want = ho.window_softmax_rows(Q, K, Vv, cfg.T, cfg.U, cfg.chunk, rows)
        want = ho.softmax_gate(want, inp["gate"][0, rows, h].double().numpy())
        g = got[0, rows, h]
        assert rel_fro(g, want) <= tol
        en = np.linalg.norm(g - want, axis=1)
        rn = np.linalg.norm(want, axis=1)
        floor = 0.05 * np.sqrt(np.mean(rn * rn))
        assert (en <= tol * np.maximum(rn, floor)).all(), float((en / np.maximum(rn, floor)).max())


# ---------------------------------------------------------------------------
# Hybrid merge Y = O~S W_S^T + O~L W_L^T (vda_hybrid_merge)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M,N,K", [(300, 136, 200), (128, 256, 64), (1000, 520, 1032), (7, 8, 8)])
def test_hybrid_merge_matches_oracle(M, N, K):
    x = make_merge_inputs(M, N, K, seed=M + N + K)
    Os, Ol, Ws, Wl = x["O_soft"], x["O_lin"], x["W_soft"], x["W_lin"]
    Y = V.hybrid_merge(*(t.cuda() for t in (Os, Ws, Ol, Wl)))
    torch.cuda.synchronize()
    want = ho.hybrid_output(Os.double().numpy()[:, None, :], Ol.double().numpy()[:, None, :],
                            Ws.double().numpy().T, Wl.double().numpy().T)
    got = Y.double().cpu().numpy()
    assert rel_fro(got, want) <= 5e-3
    en, rn = np.linalg.norm(got - want, axis=1), np.linalg.norm(want, axis=1)
    assert (en <= 1e-2 * np.maximum(rn, 0.05 * np.sqrt(np.mean(rn * rn)))).all()


def test_hybrid_merge_h3_projection_sampled_rows():
    """The H3-like clip's merge: 62400 tokens, 24 heads x 128 channels per branch,
    a 3072-wide model dimension; sampled output rows against the oracle."""
    cfg = CONFIGS["h3"]
    M, K, N = cfg.B * cfg.T * cfg.U, cfg.H * cfg.d, cfg.H * cfg.d
    x = make_merge_inputs(M, N, K, seed=5)
    Os, Ol, Ws, Wl = x["O_soft"], x["O_lin"], x["W_soft"], x["W_lin"]
    Y = V.hybrid_merge(*(t.cuda() for t in (Os, Ws, Ol, Wl))).cpu()
    rows = np.random.default_rng(1).integers(0, M, 300)
    rows = np.unique(np.concatenate([rows, [0, 127, 128, M - 1]]))
    want = ho.hybrid_output(Os[rows].double().numpy()[:, None, :], Ol[rows].double().numpy()[:, None, :],
                            Ws.double().numpy().T, Wl.double().numpy().T)
    assert rel_fro(Y[rows].double().numpy(), want) <= 5e-3


def test_hybrid_layer_end_to_end():
    """Both branches of one attention layer on the same Q, K, V through the C ABI
    (the softmax branch with its gate, the linear branch with conv prep, RMSNorm
    and its gate), merged by the two output projections, against the oracles."""
    from oracle.vda_oracle import vda_reference
    from frame_level_delta_b200.inputs import make_inputs
    cfg = CONFIGS["hires"].with_(H=2, T=9, grid_h=6, grid_w=10, L=5, chunk=2)
    inp = make_inputs(cfg)
    ga = make_attention_inputs(cfg)["gate"]  # the softmax branch's own gate logits
    dev = torch.device("cuda:0")
    d = {k: v.to(dev) for k, v in inp.items()}
    ctx = V.VDA(cfg, device=dev)
    O_lin = ctx.run(d)
    O_soft = ctx.window_attention(d["Q"], d["K"], d["V"], ga.to(dev))
    K = cfg.H * cfg.d
    w = make_merge_inputs(1, 96, K, seed=9)
    Ws, Wl = w["W_soft"], w["W_lin"]
    Y = V.hybrid_merge(O_soft, Ws.to(dev), O_lin, Wl.to(dev))
    torch.cuda.synchronize()
    assert ctx.poll_device_status() == 0
    Q, Kk, Vv = (inp[k].double().numpy() for k in ("Q", "K", "V"))
    o_soft = ho.window_softmax_layer(Q, Kk, Vv, ga.double().numpy(), cfg.T, cfg.U, cfg.chunk)
    o_lin = vda_reference(inp, cfg, keep=False)["O"]
    N = cfg.B * cfg.T * cfg.U
    want = ho.hybrid_output(o_soft.reshape(N, cfg.H, cfg.d), o_lin.reshape(N, cfg.H, cfg.d),
                            Ws.double().numpy().T, Wl.double().numpy().T)
    assert rel_fro(Y.double().cpu().numpy(), want) <= TOL_O["bf16"]
