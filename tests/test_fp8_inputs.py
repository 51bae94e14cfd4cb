"""The FP8 storage form of the inputs (frame_level_delta_b200/inputs.py), on the
CPU: the e4m3 codes, their per-row scales and the exact stored values the
oracle receives. These pin the input recipe, not the method."""
import torch

from frame_level_delta_b200.inputs import CONFIGS, make_fp8_inputs, quantize_e4m3, quantize_e4m3_pair


def _rows(n=64, d=128, seed=0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(n, d, generator=g) * torch.exp(torch.randn(n, 1, generator=g))
    x[3] = 0.0  # an all-zero row
    return x


def test_row_maximum_maps_to_the_largest_e4m3_value_and_errors_stay_within_half_a_step():
    x = _rows()
    x8, s = quantize_e4m3(x)
    assert x8.dtype == torch.float8_e4m3fn and s.dtype == torch.float32
    q = x8.float()
    assert q.abs().max() <= 448.0
    nz = x.abs().amax(dim=1) > 0
    assert torch.all(q[nz].abs().amax(dim=1) == 448.0)
    assert s[3] == 1.0 and torch.all(q[3] == 0)
    # e4m3 keeps 3 mantissa bits: normal values round to within 2^-4 relative.
    back = q * s[:, None]
    normal = (x / s[:, None]).abs() >= 2.0 ** -6
    rel = ((back - x).abs() / x.abs())[normal]
    assert rel.max() <= 2.0 ** -4 + 1e-7


def test_pair_shares_one_scale_from_the_larger_row():
    k, v = _rows(seed=1), _rows(seed=2) * 3.0
    k8, v8, s = quantize_e4m3_pair(k, v)
    amax = torch.maximum(k.abs().amax(dim=1), v.abs().amax(dim=1))
    nz = amax > 0
    assert torch.allclose(s[nz], amax[nz] / 448.0)
    both = torch.maximum(k8.float().abs().amax(dim=1), v8.float().abs().amax(dim=1))
    assert torch.all(both[nz] == 448.0)


def test_fp8_inputs_give_the_oracle_the_exact_stored_values():
    cfg = CONFIGS["h3"].with_(H=2, T=5, grid_h=3, grid_w=4, L=6)
    x = make_fp8_inputs(cfg)
    assert torch.equal(x["Q"], x["Q8"].double() * x["q_scale"].double().unsqueeze(-1))
    assert torch.equal(x["K"], x["K8"].double() * x["kv_scale"].double().unsqueeze(-1))
    assert torch.equal(x["V"], x["V8"].double() * x["kv_scale"].double().unsqueeze(-1))
    assert x["Q8"].shape == (cfg.B, cfg.T * cfg.U, cfg.H, cfg.d)
    assert x["kv_scale"].shape == (cfg.B, cfg.T * cfg.U, cfg.H)
    # Same seed, same draw: the generator is deterministic.
    y = make_fp8_inputs(cfg)
    assert torch.equal(x["K8"].view(torch.uint8), y["K8"].view(torch.uint8))
