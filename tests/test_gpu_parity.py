"""Parity of the CUDA path (through the C ABI) with the float64 oracle.

Bounds: relative Frobenius error of the whole output <= 1e-4 (fp32 storage) and
<= 2e-2 (bf16 storage); staged bounds on every intermediate (see tests/parity.py).
Full-size workloads compare sampled heads (heads are independent) plus
properties that hold at any size on every head.
"""
import numpy as np
import pytest
import torch

from frame_level_delta_b200 import vda as V
from frame_level_delta_b200.inputs import CONFIGS, VDAConfig, make_inputs
from oracle import vda_oracle as vo
from tests.parity import TOL_O, check_config, rel_fro, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    V.lib()  # fail loudly if the library is missing


@pytest.mark.parametrize("force_simt", [False, True])
def test_tiny_fp32(force_simt):
    err, st = check_config(CONFIGS["tiny"], force_simt=force_simt)
    assert err <= 1e-4


@pytest.mark.parametrize("force_simt", [False, True])
def test_small_bf16(force_simt):
    check_config(CONFIGS["small"], force_simt=force_simt)


def test_h3_full_size_all_heads():
    """The H3-like clip at full size, every one of its 24 heads against the
    oracle: whole-output, per-(head, frame) and per-token bounds, and the staged
    intermediates of every slot and chunk of every head."""
    check_config(CONFIGS["h3"])


def test_h3_full_size_cholesky_solve():
    check_config(CONFIGS["h3"], heads=[(0, 3), (0, 20)], cholesky=True)


def test_h3_full_size_chunked_scan():
    check_config(CONFIGS["h3"], heads=[(0, 7), (0, 16)], chunked=True)


# Six heads spread over the head range (first, last and four between).
SPREAD_HEADS = [(0, 0), (0, 5), (0, 10), (0, 14), (0, 19), (0, 23)]


def test_long_full_size_spread_heads():
    check_config(CONFIGS["long"], heads=SPREAD_HEADS)


def test_hires_full_size_spread_heads():
    """The high-res clip with conv prep and the gated readout at full size, on six
    heads: output bounds (whole, per frame, per token), every staged
    intermediate, and the prepared keys and values against the oracle's prep."""
    cfg = CONFIGS["hires"]
    inp = make_inputs(cfg)
    _, _, regions = check_config(cfg, heads=SPREAD_HEADS, inp=inp, return_regions=True)
    w = inp["conv_w"].double().numpy()
    hd = cfg.H * cfg.d
    for (_, h) in SPREAD_HEADS:
        for which, off in (("K", 0), ("V", hd * 30)):
            X = inp[which][0, :, h].double().numpy().reshape(cfg.T, cfg.U, cfg.d)
            want = vo.prep_video_kv(X, w[off:off + hd * 25].reshape(cfg.H, cfg.d, 5, 5)[h],
                                    w[off + hd * 25:off + hd * 30].reshape(cfg.H, cfg.d, 5)[h],
                                    cfg.grid_h, cfg.grid_w)
            if which == "K":
                want = vo.l2_normalize(want, 1e-6)
            got = regions[which + "_prep"][0, h, 1:cfg.T - 1].numpy()
            assert rel_fro(got, want[1:cfg.T - 1]) <= 5e-3, (which, h)


def test_low_write_long_memory_diagnostic():
    """beta = sigmoid(N(-4, 1)) makes the state remember many frames, so errors in
    the text init or in far frames cannot hide below the output bound."""
    cfg = CONFIGS["h3"].with_(beta_mu=-4.0, T=20)
    check_config(cfg, heads=[(0, 3)])


def test_text_counted_once_on_gpu():
    cfg = CONFIGS["small"].with_(H=2, T=12, grid_h=4, grid_w=4)
    inp = make_inputs(cfg)
    inp["beta"].zero_()
    inp["alpha"].fill_(1.0)
    O_gpu, regions, _ = run_gpu(cfg, inp)
    S_T = regions["C"][:, :, 0]  # [B, H, d, d]
    U = cfg.U
    Q = inp["Q"].float()
    for h in range(cfg.H):
        want = Q[0, U:(cfg.T - 1) * U, h] @ S_T[0, h].T
        assert rel_fro(O_gpu[0, U:(cfg.T - 1) * U, h].numpy(), want.numpy()) <= 1e-2
        np.testing.assert_allclose(regions["S_fwd"][0, h].numpy(),
                                   np.broadcast_to(0.5 * S_T[0, h].numpy(), regions["S_fwd"][0, h].shape),
                                   rtol=1e-5, atol=1e-6)


EDGE = [
    # name, overrides
    ("ragged_tokens_d64", dict(d=64, grid_h=5, grid_w=7, T=9, chunk=2, L=3, H=3)),
    ("ragged_tokens_d128", dict(d=128, grid_h=13, grid_w=11, T=8, chunk=3, L=130, H=2)),
    ("T_not_multiple_of_c", dict(d=64, T=13, chunk=5, grid_h=8, grid_w=8, H=2)),
    ("single_scanned_frame", dict(d=32, T=3, chunk=1, grid_h=2, grid_w=3, L=1, H=2)),
    ("one_chunk_covers_clip", dict(d=64, T=7, chunk=8, grid_h=4, grid_w=4, H=1)),
    ("chunk_one", dict(d=16, T=9, chunk=1, grid_h=3, grid_w=3, L=2, H=2)),
    ("single_token_frames", dict(d=64, T=10, chunk=2, grid_h=1, grid_w=1, L=1, H=2)),
    ("batch_two", dict(B=2, d=64, T=8, chunk=2, grid_h=6, grid_w=6, H=2)),
    ("d32_bf16", dict(d=32, T=10, chunk=3, grid_h=6, grid_w=5, H=2)),
    ("d16_bf16", dict(d=16, T=10, chunk=3, grid_h=6, grid_w=5, H=2)),
]


@pytest.mark.parametrize("name,kw", EDGE, ids=[e[0] for e in EDGE])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_edge_cases(name, kw, dtype):
    cfg = CONFIGS["small"].with_(name=name, dtype=dtype, **kw)
    check_config(cfg)


# Chunk structures of the tensor-core scan (d = 128, bf16): composed chunk maps
# with one frame (a copy), none (the identity), a ragged last chunk, the
# smallest clip that has a composed chunk, and single-frame chunks (no
# composition: the scan steps over frames).
EDGE_CHUNKS = [
    ("d128_ragged_last_chunk", dict(T=23, chunk=5)),
    ("d128_last_chunk_anchor_only", dict(T=13, chunk=4)),
    ("d128_two_frame_chunks", dict(T=12, chunk=2)),
    ("d128_three_chunks", dict(T=8, chunk=3)),
    ("d128_chunk_one", dict(T=9, chunk=1)),
    ("d128_wide_chunks", dict(T=20, chunk=8)),
    ("d128_batch_two", dict(B=2, T=11, chunk=3)),
    # No scanned step in either direction, and one step in each.
    ("d128_no_scan_step", dict(T=3, chunk=1)),
    ("d128_one_scan_step", dict(T=4, chunk=1)),
]


@pytest.mark.parametrize("name,kw", EDGE_CHUNKS, ids=[e[0] for e in EDGE_CHUNKS])
def test_edge_chunk_structures_tensor_core_scan(name, kw):
    cfg = CONFIGS["small"].with_(name=name, d=128, H=2, grid_h=4, grid_w=5, L=9, **kw)
    check_config(cfg)
    check_config(cfg, split_scan=True)  # the frame scan on two-CTA clusters
    check_config(cfg, chunked=True)
    if name in ("d128_ragged_last_chunk", "d128_batch_two"):
        check_config(cfg, cholesky=True)


def test_edge_conv_gate_small():
    cfg = CONFIGS["hires"].with_(H=2, d=64, T=9, grid_h=6, grid_w=7, L=5, chunk=2)
    check_config(cfg)
    check_config(cfg.with_(dtype="f32"))


# Conv prep at every head dimension and storage type, on grids whose width is
# not a multiple of the 16-column block (a ragged last block) and with a single
# grid row; the prepared keys and values are compared with the oracle's prep.
CONV_EDGE = [
    ("conv_d16", dict(d=16, grid_h=5, grid_w=9)),
    ("conv_d32", dict(d=32, grid_h=3, grid_w=17)),
    ("conv_d64", dict(d=64, grid_h=4, grid_w=35)),
    ("conv_d128", dict(d=128, grid_h=7, grid_w=21)),
    ("conv_d128_single_row", dict(d=128, grid_h=1, grid_w=33)),
    # d = 128 bf16 runs persistent CTAs over tiles of two grid rows and a frame
    # loop unrolled by five: a single scanned frame, a loop that ends on each
    # unrolled position, a second batch, and more tiles than SMs (each CTA
    # walks several tiles across planes).
    ("conv_d128_T3", dict(d=128, grid_h=3, grid_w=18, T=3, chunk=1)),
    ("conv_d128_T6_batch_two", dict(d=128, B=2, grid_h=4, grid_w=16, T=6)),
    ("conv_d128_T7", dict(d=128, grid_h=2, grid_w=47, T=7)),
    ("conv_d128_T8", dict(d=128, grid_h=5, grid_w=3, T=8)),
    ("conv_d128_many_tiles", dict(d=128, H=4, grid_h=15, grid_w=64, T=5)),
]


@pytest.mark.parametrize("name,kw", CONV_EDGE, ids=[e[0] for e in CONV_EDGE])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_edge_conv_dims(name, kw, dtype):
    cfg = CONFIGS["hires"].with_(name=name, **{**dict(H=2, T=9, L=5, chunk=2, dtype=dtype), **kw})
    inp = make_inputs(cfg)
    check_config(cfg, inp=inp)
    _, regions, _ = run_gpu(cfg, inp)
    w = inp["conv_w"].double().numpy()
    hd = cfg.H * cfg.d
    tol = 5e-3 if dtype == "bf16" else 1e-5
    for h in range(cfg.H):
        for which, off in (("K", 0), ("V", hd * 30)):
            X = inp[which][0, :, h].double().numpy().reshape(cfg.T, cfg.U, cfg.d)
            ws = w[off:off + hd * 25].reshape(cfg.H, cfg.d, 5, 5)[h]
            wt = w[off + hd * 25:off + hd * 30].reshape(cfg.H, cfg.d, 5)[h]
            want = vo.prep_video_kv(X, ws, wt, cfg.grid_h, cfg.grid_w)
            if which == "K":
                want = vo.l2_normalize(want, 1e-6)
            got = regions[which + "_prep"][0, h, 1:cfg.T - 1].numpy()
            assert rel_fro(got, want[1:cfg.T - 1]) <= tol, (which, h)


def test_degenerate_gates():
    cfg = CONFIGS["small"].with_(H=2, T=10, grid_h=4, grid_w=4)
    inp = make_inputs(cfg)
    inp["alpha"][:, 0].zero_()  # head 0 forgets everything each frame
    inp["beta"][:, 1, :, ::2] = 0  # head 1 skips every other token
    check_config(cfg, inp=inp)


def test_split_scan_matches_one_cta_scan():
    """The two-CTA cluster scan (each CTA half of every state's columns, the
    halves of the next left factor exchanged between the CTAs' shared memories)
    against the single-CTA scan on an H3-shaped clip: the same readout states up
    to fp32 accumulation order over 29 steps."""
    cfg = CONFIGS["h3"].with_(H=4)
    inp = make_inputs(cfg)
    _, r_split, lib = run_gpu(cfg, inp, split_scan=True)
    assert "scan=tcgen05-split" in V.describe(lib.c)
    _, r_one, _ = run_gpu(cfg, inp)
    for k in ("S_fwd", "S_rev"):
        assert rel_fro(r_split[k].numpy(), r_one[k].numpy()) <= 1e-5, k


def test_repeated_runs_are_bitwise_identical():
    cfg = CONFIGS["small"]
    inp = {k: v.cuda() for k, v in make_inputs(cfg).items()}
    lib = V.VDA(cfg)
    O1 = lib.run(inp).clone()
    O2 = lib.run(inp)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2)


@pytest.mark.parametrize("chunked", [False, True])
def test_interleaved_calls_on_overlapped_path(chunked):
    """The d = 128 path runs the solve and the frame scan as overlapping kernels
    that hand slots over through per-slot ready words (cleared by vda_prepare).
    Repeated and interleaved calls - a second scan and readout after one
    prepare, two prepares in a row, a readout on another stream after a
    synchronise - must give the same output bit for bit and report no timeout."""
    cfg = CONFIGS["h3"].with_(H=3, T=12, grid_h=6, grid_w=9, L=20)
    inp = {k: v.cuda() for k, v in make_inputs(cfg).items()}
    lib = V.VDA(cfg, chunked=chunked)
    ref = lib.run(inp).clone()
    O = lib.new_output()
    lib.scan_bidir()
    lib.readout(O)
    torch.cuda.synchronize()
    assert torch.equal(O, ref)
    lib.prepare(inp)
    lib.prepare(inp)
    lib.scan_bidir()
    lib.scan_bidir()
    O.zero_()
    side = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(side):
        lib.readout(O, stream=side)
    side.synchronize()
    assert torch.equal(O, ref)
    assert lib.poll_device_status() == 0


def test_bounded_wait_reports_timeout_without_faulting():
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    assert V.selftest_bounded_wait(status, 2000) == 0
    torch.cuda.synchronize()
    assert int(status[0]) == 6  # VDA_ERR_TIMEOUT
    # The context is still usable afterwards.
    check_config(CONFIGS["tiny"])


def test_launch_accounting_and_profiling():
    cfg = CONFIGS["small"]
    inp = {k: v.cuda() for k, v in make_inputs(cfg).items()}
    lib = V.VDA(cfg)
    lib.profile_enable(True)
    n0 = lib.launch_count()
    for _ in range(3):
        lib.run(inp)
    torch.cuda.synchronize()
    n = lib.launch_count() - n0
    prof = lib.profile_read()
    assert sum(v[0] for v in prof.values()) == n
    assert all(v[1] > 0 for v in prof.values())


def test_pivot_reciprocal_error_bound():
    """The sweep solve's pivot reciprocal (hardware approximation plus one
    Newton-Raphson step) against the correctly rounded 1/x, over the pivot range
    x in [1, 1e4]: log-spaced values, powers of two and random draws. Every
    result must lie within two ulps (2^-22 relative) of the exact reciprocal,
    and its rounding error against CUDA's correctly rounded 1.0f/x is at most
    one ulp."""
    g = torch.Generator().manual_seed(0)
    xs = torch.cat([torch.logspace(0, 4, 200001, dtype=torch.float64).float(),
                    torch.tensor([2.0 ** k for k in range(14)]),
                    1 + torch.rand(100000, generator=g) * 9999]).contiguous()
    y = V.selftest_recip(xs.cuda()).cpu()
    exact = 1.0 / xs.double()
    rel = ((y.double() - exact).abs() / exact).max().item()
    assert rel <= 2.0 ** -22, rel
    cr = exact.float()  # the correctly rounded reciprocal (what IEEE 1.0f / x returns)
    ulp = torch.nextafter(cr, torch.full_like(cr, float("inf"))) - cr
    assert ((y - cr).abs() <= ulp).all()
    dev_div = (1.0 / xs.cuda()).cpu()  # CUDA's own division, for the record
    assert ((dev_div - cr).abs() <= ulp).all()
