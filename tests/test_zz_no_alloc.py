"""The entry point with library-owned scratch (vda_run_static_workspace).

It serves callers that cannot allocate device memory, e.g. a plugin handed only
its input and output buffers. Its output must match the regular path (caller
workspace) and the float64 oracle within the output tolerance of the parity
tests, on two calls in a row through the same static scratch array, with the
static array's status word reporting no timeout after each call. This file is collected last so that
a failure here cannot hide any other test's result.
"""
import numpy as np
import pytest
import torch

from frame_level_delta_b200 import vda as V
from frame_level_delta_b200.inputs import CONFIGS, make_inputs
from oracle import vda_oracle as vo
from tests.parity import TOL_O, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    V.lib()


# The fp32 CUDA-core path (tiny), the d = 64 path (small), and the d = 128
# tensor-core path of the H3-like clip's shape (statistics, sweep solve, frame
# scan and readout on tcgen05, with the solve -> scan slot-ready words living
# in the shared static array), plus the conv prep with the gated readout.
CASES = {
    "tiny": CONFIGS["tiny"],
    "small": CONFIGS["small"],
    "h3_shaped_d128": CONFIGS["h3"].with_(name="h3-shaped", H=2, T=10, grid_h=8, grid_w=8, L=16),
    "conv_gate_d128": CONFIGS["hires"].with_(name="conv+gate", H=2, T=9, grid_h=6, grid_w=20, L=5),
}


@pytest.mark.parametrize("name", list(CASES))
def test_static_workspace_matches_caller_workspace(name):
    cfg = CASES[name]
    need = V.workspace_size(V.make_config(cfg))
    assert need <= V.lib().vda_static_workspace_capacity()
    inp_cpu = make_inputs(cfg)
    inp = {k: v.cuda() for k, v in inp_cpu.items()}
    ref = V.VDA(cfg).run(inp)
    torch.cuda.synchronize()
    want = vo.vda_reference(inp_cpu, cfg, keep=False)["O"]
    for call in range(2):
        O = torch.full_like(ref, float("nan"))
        assert V.run_static_workspace(cfg, inp, O) == 0
        assert V.static_workspace_poll() == 0  # synchronises; no device-side wait gave up
        err = rel_fro(O.float().cpu().numpy(), ref.float().cpu().numpy())
        assert err <= TOL_O[cfg.dtype], (call, err)
        assert torch.isfinite(O).all()
        err_oracle = rel_fro(O.double().cpu().numpy(), want)
        assert err_oracle <= TOL_O[cfg.dtype], (call, err_oracle)


def test_static_workspace_rejects_configs_beyond_capacity():
    cfg = CONFIGS["h3"]
    assert V.workspace_size(V.make_config(cfg)) > V.lib().vda_static_workspace_capacity()
    O = torch.empty(16, device="cuda")  # never written: the call fails before any launch
    assert V.run_static_workspace(cfg, {k: O for k in ("Q", "K", "V", "K_txt", "V_txt", "alpha", "beta",
                                                       "beta_txt")}, O) == 4  # VDA_ERR_WORKSPACE_TOO_SMALL
