"""Head slices (vda_config.H_total, h0): several contexts, each serving a share
of the heads of one batch in place, as the ranks of a head-sharded multi-GPU
run do. On one GPU the ranks run one after the other on the same tensors; their
outputs together must equal a single context's output bit for bit (heads are
independent and per-head arithmetic does not depend on the grid), and no
context may write another's heads."""
import pytest
import torch

from frame_level_delta_b200 import vda as V
from frame_level_delta_b200.inputs import CONFIGS, make_inputs
from frame_level_delta_b200.shard import head_partition

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    V.lib()


CASES = [
    # name, config, partition weights (None: even)
    ("small_d64_two_ranks", CONFIGS["small"], 2, None),
    ("small_d64_uneven_5_3", CONFIGS["small"], 2, (5, 3)),
    ("h3_shaped_d128_three_ranks", CONFIGS["h3"].with_(H=7, T=12, grid_h=6, grid_w=10, L=20), 3, None),
    ("conv_gate_d128_two_ranks", CONFIGS["hires"].with_(H=4, T=9, grid_h=6, grid_w=20, L=5), 2, None),
    ("fp32_simt_two_ranks", CONFIGS["small"].with_(H=4, d=32, T=10, grid_h=5, grid_w=6, dtype="f32"), 2, None),
]


@pytest.mark.parametrize("name,cfg,world,weights", CASES, ids=[c[0] for c in CASES])
def test_head_slices_reassemble_the_whole_output(name, cfg, world, weights):
    inp = {k: v.cuda() for k, v in make_inputs(cfg).items()}
    whole = V.VDA(cfg).run(inp)
    torch.cuda.synchronize()
    O = torch.full_like(whole, float("nan"))
    parts = head_partition(cfg.H, world, weights)
    for rank, (h0, n) in enumerate(parts):
        ctx = V.VDA(cfg, heads=(h0, n))
        ctx.run(inp, O)
        torch.cuda.synchronize()
        assert ctx.poll_device_status() == 0
        # This rank's heads are written; the heads of later ranks are untouched.
        assert torch.equal(O[:, :, h0:h0 + n], whole[:, :, h0:h0 + n]), rank
        assert torch.isnan(O[:, :, h0 + n:]).all()
    assert torch.equal(O, whole)


def test_head_slice_config_checks():
    cfg = CONFIGS["small"]
    with pytest.raises(V.VDAError):
        V.VDA(cfg, heads=(6, 3))  # h0 + n > H
