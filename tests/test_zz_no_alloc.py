"""The entry point with library-owned scratch (vda_run_static_workspace).

It serves callers that cannot allocate device memory, e.g. a plugin handed only
its input and output buffers. Its output must match the regular path (caller
workspace) within the output tolerance of the parity tests, on two calls in a
row through the same static scratch array. This file is collected last so that
a failure here cannot hide any other test's result.
"""
import numpy as np
import pytest
import torch

from frame_level_delta_b200 import vda as V
from frame_level_delta_b200.inputs import CONFIGS, make_inputs
from tests.parity import TOL_O, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    V.lib()


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_static_workspace_matches_caller_workspace(name):
    cfg = CONFIGS[name]
    need = V.workspace_size(V.make_config(cfg))
    assert need <= V.lib().vda_static_workspace_capacity()
    inp = {k: v.cuda() for k, v in make_inputs(cfg).items()}
    ref = V.VDA(cfg).run(inp)
    torch.cuda.synchronize()
    for call in range(2):
        O = torch.full_like(ref, float("nan"))
        assert V.run_static_workspace(cfg, inp, O) == 0
        torch.cuda.synchronize()
        err = rel_fro(O.float().cpu().numpy(), ref.float().cpu().numpy())
        assert err <= TOL_O[cfg.dtype], (call, err)
        assert torch.isfinite(O).all()


def test_static_workspace_rejects_configs_beyond_capacity():
    cfg = CONFIGS["h3"]
    assert V.workspace_size(V.make_config(cfg)) > V.lib().vda_static_workspace_capacity()
    O = torch.empty(16, device="cuda")  # never written: the call fails before any launch
    assert V.run_static_workspace(cfg, {k: O for k in ("Q", "K", "V", "K_txt", "V_txt", "alpha", "beta",
                                                       "beta_txt")}, O) == 4  # VDA_ERR_WORKSPACE_TOO_SMALL
