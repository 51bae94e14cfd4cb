"""The local output bounds of tests/parity.py catch what the whole-tensor norm
misses (CPU only: arrays stand in for the GPU's output)."""
import numpy as np

from frame_level_delta_b200.inputs import CONFIGS
from tests.parity import TOL_O, local_output_errors, readout_tiles, rel_fro


def test_readout_tiles_cover_each_chunk_once():
    cfg = CONFIGS["h3"]
    seen = []
    for j in range(cfg.J):
        tiles = readout_tiles(cfg, j)
        for a, e in tiles:
            assert 0 < e - a <= 128
        seen += tiles
    flat = [x for a, e in seen for x in (a, e)]
    assert flat[0] == cfg.U and flat[-1] == (cfg.T - 1) * cfg.U
    assert all(seen[i][1] == seen[i + 1][0] for i in range(len(seen) - 1))
    # Chunk 0 holds frames 1..4 (6240 tokens: 48 full tiles and a 96-token tail),
    # the others five frames (7800 tokens: 60 full tiles and a 120-token tail).
    assert readout_tiles(cfg, 0)[-1][1] - readout_tiles(cfg, 0)[-1][0] == 96
    assert readout_tiles(cfg, 3)[-1][1] - readout_tiles(cfg, 3)[-1][0] == 120


def test_local_bounds_catch_an_error_confined_to_ragged_tiles():
    cfg = CONFIGS["small"].with_(H=2, T=10, grid_h=10, grid_w=10)
    rng = np.random.default_rng(0)
    ref = rng.standard_normal((1, cfg.T * cfg.U, cfg.H, cfg.d))
    ref[:, :cfg.U] = 0
    ref[:, (cfg.T - 1) * cfg.U:] = 0
    got = ref * (1 + 1e-3 * rng.standard_normal(ref.shape))
    pairs = [(0, 0), (0, 1)]
    ok = local_output_errors(cfg, got, ref, pairs)
    assert ok["frame"] <= TOL_O["bf16"] and ok["token_ratio"] <= 1.0
    # 15% error on every token of each chunk's last tile only.
    bad = got.copy()
    for j in range(cfg.J):
        tiles = readout_tiles(cfg, j)
        if tiles:
            a, e = tiles[-1]
            bad[0, a:e, 0] = ref[0, a:e, 0] * 1.15
    assert rel_fro(bad, ref) <= TOL_O["bf16"] * 3  # the whole norm barely notices
    loc = local_output_errors(cfg, bad, ref, pairs)
    assert loc["token_ratio"] > 1.0 and loc["tail_tile_ratio"] > 1.0


def test_local_bounds_catch_one_wrong_frame():
    cfg = CONFIGS["small"].with_(H=1, T=40, grid_h=8, grid_w=8)
    rng = np.random.default_rng(1)
    ref = rng.standard_normal((1, cfg.T * cfg.U, 1, cfg.d))
    got = ref.copy()
    t = 17
    got[0, t * cfg.U:(t + 1) * cfg.U] *= 1.05
    assert rel_fro(got, ref) < TOL_O["bf16"]
    assert local_output_errors(cfg, got, ref, [(0, 0)])["frame"] > TOL_O["bf16"]


def test_gated_allowance_grows_for_tokens_with_a_small_pre_norm_readout():
    cfg = CONFIGS["small"].with_(H=1, T=6, grid_h=4, grid_w=4, norm_gate=True)
    rng = np.random.default_rng(2)
    ref = rng.standard_normal((1, cfg.T * cfg.U, 1, cfg.d))
    got = ref.copy()
    u = 2 * cfg.U + 3
    got[0, u, 0] *= 1.05  # 5% off on one token
    pre = np.ones(cfg.T * cfg.U)
    assert local_output_errors(cfg, got, ref, [(0, 0)], {(0, 0): pre})["token_ratio"] > 1.0
    pre[u] = 0.1  # its pre-norm readout is a tenth of the head's: RMSNorm scaled its error up 10x
    assert local_output_errors(cfg, got, ref, [(0, 0)], {(0, 0): pre})["token_ratio"] <= 1.0
