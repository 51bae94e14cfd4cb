"""Host-side checks of the C ABI: the library loads and exports every symbol the
header declares, and argument errors come back as status codes before any launch.
No test here needs a GPU; no test passes pointers that could reach a kernel."""
import ctypes
import os
import re

import pytest

from frame_level_delta_b200 import vda as V
from frame_level_delta_b200.inputs import CONFIGS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "vda.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(vda_\w+)\s*\(", text, flags=re.M)))


def test_header_matches_binding_list():
    assert _declared_symbols() == sorted(V.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = V.lib()
    for name in _declared_symbols():
        assert hasattr(L, name), name


def _cfg(**kw):
    c = V.make_config(CONFIGS["small"])
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def _create(c):
    ctx = ctypes.c_void_p()
    st = V.lib().vda_create(ctypes.byref(c), ctypes.byref(ctx))
    return st, ctx


@pytest.mark.parametrize("field,value,want", [
    ("T", 2, 1), ("U", 255, 1), ("L", 0, 1), ("chunk", 0, 1), ("B", 0, 1), ("dtype", 7, 1),
    ("d_k", 48, 2), ("d_v", 32, 2), ("flags", 0x80, 1),
])
def test_create_rejects_bad_configs(field, value, want):
    c = _cfg(**{field: value})
    if field == "d_k":
        c.d_v = value
    st, ctx = _create(c)
    assert st == want and not ctx.value
    n = ctypes.c_size_t(0)
    assert V.lib().vda_workspace_size(ctypes.byref(c), ctypes.byref(n)) == want


@pytest.mark.parametrize("kw,want", [
    (dict(grid_h=65536, grid_w=1, U=65536), 2),   # conv prep: grid rows on grid.y
    (dict(B=1, H=32768), 2),                       # conv prep: 2 B H on grid.z
    (dict(B=1, H=32767), 0),
    (dict(grid_h=2, grid_w=4096, U=8192, d_k=128, d_v=128), 0),  # wide grids tile in 16-column blocks
])
def test_conv_prep_launch_limits_are_checked_at_create(kw, want):
    c = _cfg(flags=V.VDA_PREP_CONV, **kw)
    st, ctx = _create(c)
    assert st == want
    if ctx.value:
        assert V.lib().vda_destroy(ctx) == 0


def test_chunked_scan_launch_limit_is_checked_at_create():
    c = _cfg(flags=V.VDA_SCAN_CHUNKED, B=2, H=32768)
    st, ctx = _create(c)
    assert st == 2 and not ctx.value


def test_workspace_regions_are_disjoint_and_aligned():
    for name in ("tiny", "small", "h3", "long", "hires"):
        c = V.make_config(CONFIGS[name])
        total = V.workspace_size(c)
        spans = []
        for r in V.REGIONS:
            off, nb = V.workspace_region(c, r)
            assert off % 1024 == 0
            assert off + nb <= total
            if nb:
                spans.append((off, off + nb))
        spans.sort()
        for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
            assert a1 <= b0
        cfg = CONFIGS[name]
        D = cfg.d
        assert V.workspace_region(c, "A")[1] == cfg.B * cfg.H * (cfg.T - 1) * D * D * 4
        assert V.workspace_region(c, "S_fwd")[1] == cfg.B * cfg.H * cfg.J * D * D * 4
        assert (V.workspace_region(c, "K_prep")[1] > 0) == cfg.prep_conv


def test_calls_out_of_order_and_bad_pointers_are_rejected_before_launch():
    c = _cfg()
    st, ctx = _create(c)
    assert st == 0
    L = V.lib()
    try:
        assert L.vda_scan_bidir(ctx, None) == 7
        assert L.vda_readout(ctx, None, ctypes.c_void_p(0x10000), None) == 7
        assert L.vda_poll_device_status(ctx, None) == 7
        good = [ctypes.c_void_p(0x100000 * (i + 1)) for i in range(9)]
        ws = ctypes.c_void_p(0x7000000)
        big = V.workspace_size(c)
        # NULL input
        args = list(good)
        args[2] = None
        assert L.vda_prepare(ctx, *args, ws, big, None) == 1
        # misaligned token tensor
        args = list(good)
        args[1] = ctypes.c_void_p(0x100008)
        assert L.vda_prepare(ctx, *args, ws, big, None) == 3
        # misaligned workspace
        assert L.vda_prepare(ctx, *good, ctypes.c_void_p(0x7000080), big, None) == 3
        # workspace too small
        assert L.vda_prepare(ctx, *good, ws, big - 1, None) == 4
        assert b"workspace" in L.vda_last_error(ctx)
        # still not prepared
        assert L.vda_scan_bidir(ctx, None) == 7
    finally:
        assert L.vda_destroy(ctx) == 0


def test_fp8_prepare_rejects_conv_and_non_tensor_core_configs():
    """vda_prepare_fp8 needs d = 128, bf16 outputs and no conv prep; it refuses
    the others with VDA_ERR_UNSUPPORTED before touching any pointer."""
    L = V.lib()
    fake = [ctypes.c_void_p(0x100000 * (i + 1)) for i in range(9)]  # K8 .. beta_txt
    for cfg in (CONFIGS["hires"], CONFIGS["small"], CONFIGS["tiny"]):
        c = V.make_config(cfg)
        st, ctx = _create(c)
        assert st == 0
        try:
            got = L.vda_prepare_fp8(ctx, *fake, ctypes.c_void_p(0x7000000), ctypes.c_size_t(V.workspace_size(c)), None)
            assert V.STATUS_NAMES[got] == "VDA_ERR_UNSUPPORTED", (cfg.name, got)
        finally:
            L.vda_destroy(ctx)


def test_conv_and_gate_requirements():
    c = V.make_config(CONFIGS["hires"])
    st, ctx = _create(c)
    assert st == 0
    L = V.lib()
    try:
        good = [ctypes.c_void_p(0x100000 * (i + 1)) for i in range(8)]
        # conv_w is required with the conv flag
        assert L.vda_prepare(ctx, *good, None, ctypes.c_void_p(0x7000000), V.workspace_size(c), None) == 1
    finally:
        L.vda_destroy(ctx)


def test_status_strings_and_describe():
    L = V.lib()
    for code, name in V.STATUS_NAMES.items():
        assert L.vda_status_string(code).decode() == name
    assert L.vda_num_kernels() >= 8
    text = V.describe(V.make_config(CONFIGS["tiny"]))
    assert "gram=" in text and "readout=" in text
    assert "tcgen05" not in text  # fp32 storage always takes the CUDA-core path
    assert "tcgen05" not in V.describe(V.make_config(CONFIGS["h3"], force_simt=True))
    # The frame scan forms the injections (S Diag(alpha) + B) P itself after the
    # sweep solve; the chunked scan and the Cholesky solve keep M_t and C_t.
    assert "inject=scan" in V.describe(V.make_config(CONFIGS["h3"]))
    assert "inject=scan" not in V.describe(V.make_config(CONFIGS["h3"], chunked=True))
    assert "inject=scan" not in V.describe(V.make_config(CONFIGS["h3"], cholesky=True))
    assert "inject=scan" not in V.describe(V.make_config(CONFIGS["small"]))  # d = 64: CUDA-core solve
    # The two-CTA cluster scan only on request, and only where the scan forms the injections.
    assert "scan=tcgen05 " in V.describe(V.make_config(CONFIGS["h3"]))
    assert "scan=tcgen05-split" in V.describe(V.make_config(CONFIGS["h3"], split_scan=True))
    assert "scan=tcgen05-split" not in V.describe(V.make_config(CONFIGS["h3"], split_scan=True, chunked=True))


def test_region_view_undoes_column_quad_layout():
    """Workspace matrices are stored in column quads: element (i, j) at float
    ((j // 4) * d + i) * 4 + j % 4. The region view must return row-major."""
    import torch
    from frame_level_delta_b200.vda import _from_quads
    D = 16
    raw = torch.arange(2 * D * D, dtype=torch.float32).view(torch.uint8)
    m = _from_quads(raw, (2,), D)
    for s in range(2):
        for i in range(D):
            for j in range(D):
                assert m[s, i, j] == s * D * D + ((j // 4) * D + i) * 4 + j % 4


def test_region_view_decodes_operand_images():
    """M_t's hi/lo images use the swizzled operand layout the header states:
    element (i, j) at byte (j//64)*D*128 + i*128 + (((j%64)//8) ^ (i%8))*16 + (j%8)*2."""
    import torch
    from frame_level_delta_b200.vda import _from_images
    D = 128
    vals = torch.randn(D, D)
    img = torch.zeros(D * D, dtype=torch.bfloat16)
    for i in range(D):
        for j in range(D):
            byte = (j // 64) * D * 128 + i * 128 + (((j % 64) // 8) ^ (i % 8)) * 16 + (j % 8) * 2
            img[byte // 2] = vals[i, j]
    out = _from_images(img.view(torch.uint8), (1,), D)[0]
    assert torch.equal(out, vals.bfloat16().float())


def test_binding_checks_tensors_before_calling_the_library():
    """The Python binding rejects inputs the C ABI would misread (wrong device,
    shape, dtype or layout) before any call that could reach a kernel."""
    import torch
    from frame_level_delta_b200.inputs import make_inputs

    cfg = CONFIGS["hires"].with_(H=2, T=5, grid_h=3, grid_w=4, L=3)
    inp = make_inputs(cfg)
    O = torch.empty(cfg.B, cfg.T * cfg.U, cfg.H, cfg.d, dtype=inp["Q"].dtype)
    host = V.VDA(cfg, device="cpu")  # checks only: a CPU context never calls the library
    host.check_inputs(inp)
    host.check_output(O, inp["gate"])
    with pytest.raises(ValueError, match="CUDA devices"):
        host.run(inp, O)

    def bad(mutate, match):
        x = dict(inp)
        mutate(x)
        with pytest.raises(ValueError, match=match):
            host.check_inputs(x)

    bad(lambda x: x.pop("beta"), "missing input beta")
    bad(lambda x: x.update(Q=inp["Q"][:, :-1]), "shape")
    bad(lambda x: x.update(alpha=inp["alpha"].double()), "dtype")
    bad(lambda x: x.update(K=inp["K"].transpose(2, 3).contiguous().transpose(2, 3)), "contiguous")
    bad(lambda x: x.update(conv_w=inp["conv_w"][:-1]), "shape")
    with pytest.raises(ValueError, match="gate is required"):
        host.check_output(O, None)
    with pytest.raises(ValueError, match="shape"):
        host.check_output(O[:, :-1], inp["gate"])
    # a CUDA context handed host tensors refuses them before any library call
    dev = V.VDA(cfg, device="cuda")
    with pytest.raises(ValueError, match="is on cpu"):
        dev.prepare(inp)
    with pytest.raises(ValueError, match="is on cpu"):
        dev.run(inp, O)


@pytest.mark.parametrize("kw,want", [
    (dict(H_total=8, h0=0, H=8), 0),
    (dict(H_total=8, h0=5, H=3), 0),
    (dict(H_total=8, h0=6, H=3), 1),   # slice runs past the last head
    (dict(H_total=0, h0=1, H=8), 1),   # h0 without H_total
    (dict(H_total=-1, h0=0, H=8), 1),
    (dict(H_total=8, h0=-1, H=2), 1),
])
def test_head_slice_fields_are_checked(kw, want):
    c = _cfg(**kw)
    st, ctx = _create(c)
    assert st == want
    if ctx.value:
        assert V.lib().vda_destroy(ctx) == 0


def test_head_slice_workspace_is_sized_by_the_slice():
    whole = V.workspace_size(V.make_config(CONFIGS["small"].with_(H=3)))
    part = V.workspace_size(V.make_config(CONFIGS["small"], heads=(5, 3)))
    assert part == whole
