"""Parity of the frame-step backward (vda_frame_solve_backward) with the float64
oracle's frame_step_backward, which finite differences of the forward frame step
pin (tests/test_oracle_backward.py).

Bounds, relative Frobenius per output and per (head, frame): fp32 storage on the
CUDA-core kernels 1e-4 x cond-free slack (1e-3); bf16 storage 2e-2, the method's
bf16 target: the statistics kernel rounds beta K to bf16 (2^-9 relative) and dK,
dV are stored in bf16.
"""
import numpy as np
import pytest
import torch

from frame_level_delta_b200 import vda as V
from frame_level_delta_b200.inputs import CONFIGS, make_backward_inputs, make_inputs
from oracle import vda_oracle as vo
from tests.parity import rel_fro

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-3, "bf16": 2e-2}


@pytest.fixture(autouse=True, scope="module")
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    V.lib()


def _run(cfg, inp, bw, heads=None):
    dev = torch.device("cuda:0")
    ctx = V.VDA(cfg, device=dev, heads=heads)
    h0, n = heads if heads else (0, cfg.H)
    out = ctx.frame_solve_backward(inp["K"].to(dev), inp["V"].to(dev), inp["alpha"].to(dev), inp["beta"].to(dev),
                                   bw["S_prev"][:, h0:h0 + n].contiguous().to(dev),
                                   bw["dS"][:, h0:h0 + n].contiguous().to(dev))
    torch.cuda.synchronize()
    assert ctx.poll_device_status() == 0
    return {k: v.double().cpu().numpy() for k, v in out.items()}, V.describe(ctx.c)


def _check(cfg, inp, bw, got, pairs, frames, h0=0):
    tol = TOL[cfg.dtype]
    U = cfg.U
    worst = {}
    for (b, h) in pairs:
        for t in frames:
            Kf = inp["K"][b, t * U:(t + 1) * U, h].double().numpy()
            Vf = inp["V"][b, t * U:(t + 1) * U, h].double().numpy()
            ref = vo.frame_step_backward(bw["S_prev"][b, h, t].double().numpy(), Kf, Vf,
                                         inp["beta"][b, h, t].double().numpy(),
                                         inp["alpha"][b, h, t].double().numpy(), bw["dS"][b, h, t].double().numpy())
            hl = h - h0
            mine = {"dK": got["dK"][b, t * U:(t + 1) * U, h], "dV": got["dV"][b, t * U:(t + 1) * U, h],
                    "dS_prev": got["dS_prev"][b, hl, t], "dalpha": got["dalpha"][b, hl, t],
                    "dbeta": got["dbeta"][b, hl, t]}
            for k, v in mine.items():
                e = rel_fro(v, ref[k])
                worst[k] = max(worst.get(k, 0.0), e)
    for k, e in worst.items():
        assert e <= tol, (k, e, worst)
    return worst


CASES = [
    ("tiny_fp32", CONFIGS["tiny"]),
    ("small_d64", CONFIGS["small"].with_(H=2, T=8, grid_h=8, grid_w=8)),
    ("d128_ragged", CONFIGS["h3"].with_(H=2, T=7, grid_h=5, grid_w=9, L=4)),
    ("d32_batch_two", CONFIGS["small"].with_(B=2, H=2, d=32, T=6, grid_h=3, grid_w=7)),
]


@pytest.mark.parametrize("name,cfg", CASES, ids=[c[0] for c in CASES])
def test_frame_backward_matches_oracle(name, cfg):
    inp, bw = make_inputs(cfg), make_backward_inputs(cfg)
    got, desc = _run(cfg, inp, bw)
    pairs = [(b, h) for b in range(cfg.B) for h in range(cfg.H)]
    _check(cfg, inp, bw, got, pairs, range(1, cfg.T - 1))
    # Anchor frames are left as they were (zero here).
    U, T = cfg.U, cfg.T
    assert np.all(got["dK"][:, :U] == 0) and np.all(got["dK"][:, (T - 1) * U:] == 0)
    assert np.all(got["dbeta"][:, :, 0] == 0) and np.all(got["dS_prev"][:, :, T - 1] == 0)


def test_frame_backward_head_slice():
    cfg = CONFIGS["small"].with_(H=4, T=6, grid_h=6, grid_w=6)
    inp, bw = make_inputs(cfg), make_backward_inputs(cfg)
    got, _ = _run(cfg, inp, bw, heads=(1, 2))
    _check(cfg, inp, bw, got, [(0, 1), (0, 2)], range(1, cfg.T - 1), h0=1)
    assert np.all(got["dK"][:, :, [0, 3]] == 0)


def test_frame_backward_h3_full_size_sampled():
    """The H3-like clip at full size (24 heads, 38 scanned frames of 1560 tokens):
    every head and frame runs; three heads x four frames are compared."""
    cfg = CONFIGS["h3"]
    inp, bw = make_inputs(cfg), make_backward_inputs(cfg)
    got, desc = _run(cfg, inp, bw)
    assert "gram=tcgen05" in desc
    for k, v in got.items():
        assert np.isfinite(v).all(), k
    _check(cfg, inp, bw, got, [(0, 0), (0, 12), (0, 23)], [1, 2, 19, cfg.T - 2])
