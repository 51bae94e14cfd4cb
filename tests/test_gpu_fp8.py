"""FP8 readout (vda_readout_fp8): queries stored as e4m3 with one float32 scale
per (token, head). Parity is against the float64 oracle run on the exact stored
values (q = scale * q8, upcast exactly), at the bf16 bound 2e-2, whole-output,
per (head, frame) and per token. The error of the FP8 storage itself (q8 * scale
against the bf16 queries, about 2^-4 per value) is a property of the input
format, recorded here but not bounded by 2e-2."""
import numpy as np
import pytest
import torch

from frame_level_delta_b200 import vda as V
from frame_level_delta_b200.inputs import CONFIGS, make_inputs, quantize_e4m3
from oracle import vda_oracle as vo
from tests.parity import TOL_O, local_output_errors, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    V.lib()


def _run(cfg, heads=None):
    inp = make_inputs(cfg)
    Q8, qs = quantize_e4m3(inp["Q"])
    dev = torch.device("cuda:0")
    d = {k: v.to(dev) for k, v in inp.items()}
    ctx = V.VDA(cfg, device=dev)
    ctx.prepare(d)
    ctx.scan_bidir()
    O = ctx.readout_fp8(Q8.to(dev), qs.to(dev))
    ref_bf16 = ctx.new_output()
    ctx.readout(ref_bf16)
    torch.cuda.synchronize()
    assert ctx.poll_device_status() == 0
    deq = dict(inp)
    deq["Q"] = Q8.double() * qs.double().unsqueeze(-1)  # the exact stored values
    want = vo.vda_reference(deq, cfg, heads=heads, keep=False)["O"]
    return O.double().cpu().numpy(), want, ref_bf16.double().cpu().numpy()


CASES = [
    ("h3_shaped", CONFIGS["h3"].with_(H=2, T=10, grid_h=8, grid_w=8, L=16)),
    ("ragged_tiles", CONFIGS["h3"].with_(H=3, T=11, grid_h=7, grid_w=9, L=5, chunk=3)),
    ("batch_two", CONFIGS["h3"].with_(B=2, H=2, T=8, grid_h=5, grid_w=6, L=4, chunk=2)),
]


@pytest.mark.parametrize("name,cfg", CASES, ids=[c[0] for c in CASES])
def test_fp8_readout_matches_oracle_on_stored_values(name, cfg):
    got, want, _ = _run(cfg)
    tol = TOL_O["bf16"]
    assert rel_fro(got, want) <= tol
    pairs = [(b, h) for b in range(cfg.B) for h in range(cfg.H)]
    loc = local_output_errors(cfg, got, want, pairs)
    assert loc["frame"] <= tol and loc["token_ratio"] <= 1.0, loc
    U, T = cfg.U, cfg.T
    assert np.all(got[:, :U] == 0) and np.all(got[:, (T - 1) * U:] == 0)


def test_fp8_readout_h3_full_size_spread_heads():
    cfg = CONFIGS["h3"]
    heads = [(0, 0), (0, 7), (0, 15), (0, 23)]
    got, want, bf16 = _run(cfg, heads)
    hs = [h for _, h in heads]
    assert rel_fro(got[:, :, hs], want[:, :, hs]) <= TOL_O["bf16"]
    loc = local_output_errors(cfg, got, want, heads)
    assert loc["frame"] <= TOL_O["bf16"] and loc["token_ratio"] <= 1.0, loc
    # For the record: FP8 against the bf16-query readout of the same states.
    print("fp8 vs bf16 queries, rel Frobenius:", rel_fro(got, bf16))


# ---------------------------------------------------------------------------
# The whole path in FP8: vda_prepare_fp8 (statistics from e4m3 K, V) + scan +
# vda_readout_fp8, against the oracle on the exact stored values.
# ---------------------------------------------------------------------------
FP8_PATH = [
    ("h3_shaped", CONFIGS["h3"].with_(H=2, T=10, grid_h=8, grid_w=8, L=16)),
    ("ragged", CONFIGS["h3"].with_(H=3, T=11, grid_h=7, grid_w=9, L=70, chunk=3)),
    # More heads than the exponent pre-pass takes in one pass over a slot's tokens.
    ("many_heads", CONFIGS["h3"].with_(H=34, T=6, grid_h=4, grid_w=5, L=9, chunk=2)),
]


def _run_fp8_path(cfg, heads=None):
    from frame_level_delta_b200.inputs import make_fp8_inputs
    x = make_fp8_inputs(cfg)
    dev = torch.device("cuda:0")
    keys8 = ("K8", "V8", "Kt8", "Vt8", "kv_scale", "kvt_scale", "alpha", "beta", "beta_txt")
    d = {k: x[k].to(dev) for k in keys8}
    ctx = V.VDA(cfg, device=dev)
    ctx.prepare_fp8(d)
    ctx.scan_bidir()
    O = ctx.readout_fp8(x["Q8"].to(dev), x["q_scale"].to(dev))
    torch.cuda.synchronize()
    assert ctx.poll_device_status() == 0
    regions = {k: ctx.region(k).detach().cpu().clone() for k in ("A", "B", "S_fwd", "S_rev")}
    ref = vo.vda_reference({k: x[k] for k in ("Q", "K", "V", "K_txt", "V_txt", "alpha", "beta", "beta_txt")},
                           cfg, heads=heads)
    return O.double().cpu().numpy(), ref, regions


@pytest.mark.parametrize("name,cfg", FP8_PATH, ids=[c[0] for c in FP8_PATH])
def test_fp8_path_matches_oracle_on_stored_values(name, cfg):
    got, ref, regions = _run_fp8_path(cfg)
    tol = TOL_O["bf16"]
    assert rel_fro(got, ref["O"]) <= tol
    loc = local_output_errors(cfg, got, ref["O"], ref["heads"])
    assert loc["frame"] <= tol and loc["token_ratio"] <= 1.0, loc
    # Staged: the statistics from e4m3 operands (write operand split in two e4m3
    # parts, ~2^-8), bounded like one bf16 rounding level.
    for (b, h), it in ref["inter"].items():
        for s in range(cfg.T - 1):
            assert rel_fro(regions["A"][b, h, s], it["A"][s]) <= 4e-3, ("A", b, h, s)
            assert rel_fro(regions["B"][b, h, s], it["B"][s]) <= 4e-3, ("B", b, h, s)


def test_fp8_path_long_clip_three_heads():
    """The long clip's per-head workload at full size (120 frames of 30 x 52
    tokens, chunks of 5, L = 512) with three heads: heads are independent, so
    this is config 4's per-head computation, with the host-side float64 copies
    of the inputs kept to a few GB."""
    cfg = CONFIGS["long"].with_(H=3)
    got, ref, _ = _run_fp8_path(cfg)
    assert rel_fro(got, ref["O"]) <= TOL_O["bf16"]
    loc = local_output_errors(cfg, got, ref["O"], ref["heads"])
    assert loc["frame"] <= TOL_O["bf16"] and loc["token_ratio"] <= 1.0, loc


def test_fp8_path_h3_full_size_spread_heads():
    cfg = CONFIGS["h3"]
    heads = [(0, 0), (0, 11), (0, 23)]
    got, ref, _ = _run_fp8_path(cfg, heads)
    hs = [h for _, h in heads]
    assert rel_fro(got[:, :, hs], ref["O"][:, :, hs]) <= TOL_O["bf16"]
    loc = local_output_errors(cfg, got, ref["O"], heads)
    assert loc["frame"] <= TOL_O["bf16"] and loc["token_ratio"] <= 1.0, loc
