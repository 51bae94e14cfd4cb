"""Thin ctypes binding of libvda.so (the C ABI in include/vda.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. PyTorch supplies device memory and streams. Loading fails loudly if the
library has not been built; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Tuple

import torch

from .inputs import VDAConfig

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvda.so")

VDA_OK = 0
STATUS_NAMES = {0: "VDA_OK", 1: "VDA_ERR_INVALID_ARG", 2: "VDA_ERR_UNSUPPORTED", 3: "VDA_ERR_ALIGNMENT",
                4: "VDA_ERR_WORKSPACE_TOO_SMALL", 5: "VDA_ERR_CUDA", 6: "VDA_ERR_TIMEOUT", 7: "VDA_ERR_STATE"}
VDA_F32, VDA_BF16 = 0, 1
VDA_PREP_CONV = 0x1
VDA_READOUT_NORM_GATE = 0x2
VDA_SOLVE_CHOLESKY = 0x4
VDA_SCAN_CHUNKED = 0x8
VDA_SCAN_SPLIT = 0x10
VDA_FORCE_SIMT = 0x100
REGIONS = {"status": 0, "A": 1, "B": 2, "M": 3, "C": 4, "S_fwd": 5, "S_rev": 6,
           "K_prep": 7, "V_prep": 8, "Kt_prep": 9, "Vt_prep": 10, "M_split": 11,
           "chunk_M": 12, "chunk_C": 13}

# Exported symbols, in the order include/vda.h declares them.
EXPORTS = ["vda_create", "vda_destroy", "vda_workspace_size", "vda_prepare", "vda_scan_bidir",
           "vda_readout", "vda_prepare_fp8", "vda_readout_fp8", "vda_poll_device_status", "vda_window_attention",
           "vda_frame_solve_backward",
           "vda_hybrid_merge",
           "vda_workspace_region", "vda_status_string",
           "vda_last_error", "vda_profile_enable", "vda_num_kernels", "vda_profile_read",
           "vda_launch_count", "vda_describe", "vda_selftest_bounded_wait",
           "vda_selftest_recip", "vda_static_workspace_capacity", "vda_run_static_workspace",
           "vda_static_workspace_poll"]


class VDAError(RuntimeError):
    def __init__(self, status: int, msg: str = ""):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class vda_config(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int), ("U", ctypes.c_int),
                ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int), ("L", ctypes.c_int),
                ("d_k", ctypes.c_int), ("d_v", ctypes.c_int), ("chunk", ctypes.c_int),
                ("dtype", ctypes.c_int), ("flags", ctypes.c_uint), ("l2_eps", ctypes.c_float),
                ("rms_eps", ctypes.c_float), ("H_total", ctypes.c_int), ("h0", ctypes.c_int)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libvda.so once; raise if it is missing (no fallback path exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m frame_level_delta_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(_LIB_PATH)
        vp, sz, i, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_int
        cfgp = ctypes.POINTER(vda_config)
        L.vda_create.argtypes = [cfgp, ctypes.POINTER(vp)]
        L.vda_destroy.argtypes = [vp]
        L.vda_workspace_size.argtypes = [cfgp, ctypes.POINTER(sz)]
        L.vda_prepare.argtypes = [vp] + [vp] * 9 + [vp, sz, vp]
        L.vda_scan_bidir.argtypes = [vp, vp]
        L.vda_readout.argtypes = [vp, vp, vp, vp]
        L.vda_poll_device_status.argtypes = [vp, vp]
        L.vda_window_attention.argtypes = [vp] * 7 + [sz, vp]
        L.vda_hybrid_merge.argtypes = [vp] * 5 + [i, i, i, vp, sz, vp]
        L.vda_readout_fp8.argtypes = [vp] * 5
        L.vda_prepare_fp8.argtypes = [vp] * 11 + [sz, vp]
        L.vda_frame_solve_backward.argtypes = [vp] * 13 + [sz, vp]
        L.vda_workspace_region.argtypes = [cfgp, i, ctypes.POINTER(sz), ctypes.POINTER(sz)]
        L.vda_status_string.argtypes = [st]
        L.vda_status_string.restype = ctypes.c_char_p
        L.vda_last_error.argtypes = [vp]
        L.vda_last_error.restype = ctypes.c_char_p
        L.vda_profile_enable.argtypes = [vp, i]
        L.vda_num_kernels.argtypes = []
        L.vda_profile_read.argtypes = [vp, i, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(i),
                                       ctypes.POINTER(ctypes.c_double)]
        L.vda_launch_count.argtypes = [vp, ctypes.POINTER(ctypes.c_uint64)]
        L.vda_describe.argtypes = [cfgp, ctypes.POINTER(ctypes.c_char_p)]
        L.vda_selftest_bounded_wait.argtypes = [vp, ctypes.c_uint64, vp]
        L.vda_selftest_recip.argtypes = [vp, vp, i, vp]
        L.vda_static_workspace_poll.argtypes = [vp]
        L.vda_static_workspace_capacity.argtypes = []
        L.vda_static_workspace_capacity.restype = ctypes.c_size_t
        L.vda_run_static_workspace.argtypes = [cfgp] + [vp] * 11 + [vp]
        for name in EXPORTS:
            if name not in ("vda_status_string", "vda_last_error", "vda_static_workspace_capacity"):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def make_config(cfg: VDAConfig, force_simt: bool = False, l2_eps: float = 1e-6,
                rms_eps: float = 1e-6, cholesky: bool = False, chunked: bool = False,
                heads: Optional[Tuple[int, int]] = None, split_scan: bool = False) -> vda_config:
    """The C config of a workload. ``heads = (h0, n)`` makes a context for heads
    h0 .. h0+n-1 of the workload's cfg.H heads (token tensors keep all cfg.H)."""
    flags = (VDA_PREP_CONV if cfg.prep_conv else 0) | (VDA_READOUT_NORM_GATE if cfg.norm_gate else 0)
    if force_simt:
        flags |= VDA_FORCE_SIMT
    if cholesky:
        flags |= VDA_SOLVE_CHOLESKY
    if chunked:
        flags |= VDA_SCAN_CHUNKED
    if split_scan:
        flags |= VDA_SCAN_SPLIT
    h0, n = heads if heads is not None else (0, cfg.H)
    return vda_config(B=cfg.B, H=n, T=cfg.T, U=cfg.U, grid_h=cfg.grid_h, grid_w=cfg.grid_w, L=cfg.L,
                      d_k=cfg.d, d_v=cfg.d, chunk=cfg.chunk,
                      dtype=VDA_F32 if cfg.dtype == "f32" else VDA_BF16, flags=flags,
                      l2_eps=l2_eps, rms_eps=rms_eps, H_total=cfg.H if heads is not None else 0, h0=h0)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def workspace_size(c: vda_config) -> int:
    n = ctypes.c_size_t(0)
    st = lib().vda_workspace_size(ctypes.byref(c), ctypes.byref(n))
    if st != VDA_OK:
        raise VDAError(st, "vda_workspace_size")
    return n.value


def workspace_region(c: vda_config, name: str):
    off, nb = ctypes.c_size_t(0), ctypes.c_size_t(0)
    st = lib().vda_workspace_region(ctypes.byref(c), REGIONS[name], ctypes.byref(off), ctypes.byref(nb))
    if st != VDA_OK:
        raise VDAError(st, "vda_workspace_region")
    return off.value, nb.value


def describe(c: vda_config) -> str:
    t = ctypes.c_char_p()
    st = lib().vda_describe(ctypes.byref(c), ctypes.byref(t))
    if st != VDA_OK:
        raise VDAError(st, "vda_describe")
    return t.value.decode()


class VDA:
    """One context of the library: prepare -> scan_bidir -> readout on a stream.

    With ``heads = (h0, n)`` the context serves heads h0 .. h0+n-1 of the
    workload: the token tensors (Q, K, V, K_txt, V_txt, gate, O) keep all cfg.H
    heads and are read and written in place, and the per-head parameters
    (alpha, beta, beta_txt, conv_w) are passed for all cfg.H heads and sliced to
    the context's heads here."""

    def __init__(self, cfg: VDAConfig, force_simt: bool = False, device="cuda", cholesky: bool = False,
                 chunked: bool = False, heads: Optional[Tuple[int, int]] = None, split_scan: bool = False):
        self.cfg = cfg
        self.heads = heads
        self.c = make_config(cfg, force_simt=force_simt, cholesky=cholesky, chunked=chunked, heads=heads,
                             split_scan=split_scan)
        self._ctx = ctypes.c_void_p()
        st = lib().vda_create(ctypes.byref(self.c), ctypes.byref(self._ctx))
        if st != VDA_OK:
            raise VDAError(st, "vda_create")
        self.ws_bytes = workspace_size(self.c)
        self.device = torch.device(device)
        self.workspace: Optional[torch.Tensor] = None
        self._attn_ws: Optional[torch.Tensor] = None
        self._keep = None

    def __del__(self):
        if getattr(self, "_ctx", None) and self._ctx.value and _lib is not None:
            _lib.vda_destroy(self._ctx)
            self._ctx = ctypes.c_void_p()

    def _check(self, st: int, what: str):
        if st != VDA_OK:
            raise VDAError(st, f"{what}: {lib().vda_last_error(self._ctx).decode()}")

    def ensure_workspace(self) -> torch.Tensor:
        if self.workspace is None:
            self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.device)
        return self.workspace

    # -- argument checks (before any call into the library) -----------------------
    def _expect(self, name: str, t, shape, dtype):
        if not isinstance(t, torch.Tensor):
            raise ValueError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
        if t.device.type != self.device.type or (self.device.index is not None and t.device.index != self.device.index):
            raise ValueError(f"{name} is on {t.device}; this context runs on {self.device}")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}; expected {tuple(shape)}")
        if t.dtype != dtype:
            raise ValueError(f"{name} has dtype {t.dtype}; expected {dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")

    def check_inputs(self, inp: Dict[str, torch.Tensor]):
        """Raise ValueError unless every input of vda_prepare has the device,
        shape, dtype and contiguous layout the C ABI takes."""
        cfg = self.cfg
        B, H, d, T, U, L = cfg.B, cfg.H, cfg.d, cfg.T, cfg.U, cfg.L
        sd = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
        f32 = torch.float32
        spec = {"Q": ((B, T * U, H, d), sd), "K": ((B, T * U, H, d), sd), "V": ((B, T * U, H, d), sd),
                "K_txt": ((B, L, H, d), sd), "V_txt": ((B, L, H, d), sd), "alpha": ((B, H, T, d), f32),
                "beta": ((B, H, T, U), f32), "beta_txt": ((B, H, L), f32)}
        if cfg.prep_conv:
            spec["conv_w"] = ((H * d * 60,), f32)
        for name, (shape, dt) in spec.items():
            if name not in inp:
                raise ValueError(f"missing input {name}")
            self._expect(name, inp[name], shape, dt)

    def check_output(self, O: torch.Tensor, gate: Optional[torch.Tensor] = None):
        """Raise ValueError unless O (and the gate, when given) match the C ABI."""
        cfg = self.cfg
        sd = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
        shape = (cfg.B, cfg.T * cfg.U, cfg.H, cfg.d)
        self._expect("O", O, shape, sd)
        if gate is not None:
            self._expect("gate", gate, shape, sd)
        elif cfg.norm_gate:
            raise ValueError("gate is required by the normalised, gated readout")

    def _on_device(self):
        if self.device.type != "cuda":
            raise ValueError(f"the library runs on CUDA devices; this context is on {self.device}")
        return torch.cuda.device(self.device)

    def prepare(self, inp: Dict[str, torch.Tensor], stream=None):
        self.check_inputs(inp)
        with self._on_device():
            self._prepare(inp, stream)

    def _head_params(self, inp: Dict[str, torch.Tensor]) -> Dict[str, torch.Tensor]:
        """The per-head parameters of this context's heads (views for B = 1)."""
        if self.heads is None:
            return inp
        h0, n = self.heads
        cfg = self.cfg
        out = dict(inp)
        for k in ("alpha", "beta", "beta_txt"):
            t = inp[k][:, h0:h0 + n]
            if not t.is_contiguous() or t.data_ptr() % 16:
                t = t.clone(memory_format=torch.contiguous_format)  # the C ABI takes 16-byte aligned rows
            out[k] = t
        if cfg.prep_conv:
            hd, d = cfg.H * cfg.d, cfg.d
            w = inp["conv_w"]
            parts = []
            for off, taps in ((0, 25), (hd * 25, 5), (hd * 30, 25), (hd * 55, 5)):
                parts.append(w[off + h0 * d * taps: off + (h0 + n) * d * taps])
            out["conv_w"] = torch.cat(parts).contiguous()
        return out

    def _prepare(self, inp: Dict[str, torch.Tensor], stream=None):
        ws = self.ensure_workspace()
        inp = self._head_params(inp)
        self._keep = inp  # inputs must outlive the readout
        st = lib().vda_prepare(self._ctx, _ptr(inp["Q"]), _ptr(inp["K"]), _ptr(inp["V"]), _ptr(inp["K_txt"]),
                               _ptr(inp["V_txt"]), _ptr(inp["alpha"]), _ptr(inp["beta"]), _ptr(inp["beta_txt"]),
                               _ptr(inp.get("conv_w")), _ptr(ws), ws.numel(), _stream_handle(stream))
        self._check(st, "vda_prepare")

    def scan_bidir(self, stream=None):
        with self._on_device():
            self._check(lib().vda_scan_bidir(self._ctx, _stream_handle(stream)), "vda_scan_bidir")

    def readout(self, O: torch.Tensor, gate: Optional[torch.Tensor] = None, stream=None):
        self.check_output(O, gate)
        with self._on_device():
            self._check(lib().vda_readout(self._ctx, _ptr(gate), _ptr(O), _stream_handle(stream)), "vda_readout")

    def prepare_fp8(self, inp8: Dict[str, torch.Tensor], stream=None):
        """Statistics and solve from e4m3 keys and values (vda_prepare_fp8). inp8
        holds K8, V8 [B, T*U, H, d] and Kt8, Vt8 [B, L, H, d] (float8_e4m3fn),
        kv_scale [B, T*U, H], kvt_scale [B, L, H] (float32), and alpha, beta,
        beta_txt as for prepare."""
        cfg = self.cfg
        f8, f32 = torch.float8_e4m3fn, torch.float32
        B, H, T, U, L, d = cfg.B, cfg.H, cfg.T, cfg.U, cfg.L, cfg.d
        spec = {"K8": ((B, T * U, H, d), f8), "V8": ((B, T * U, H, d), f8), "Kt8": ((B, L, H, d), f8),
                "Vt8": ((B, L, H, d), f8), "kv_scale": ((B, T * U, H), f32), "kvt_scale": ((B, L, H), f32),
                "alpha": ((B, H, T, d), f32), "beta": ((B, H, T, U), f32), "beta_txt": ((B, H, L), f32)}
        for name, (shape, dt) in spec.items():
            if name not in inp8:
                raise ValueError(f"missing input {name}")
            self._expect(name, inp8[name], shape, dt)
        par = self._head_params(inp8)
        ws = self.ensure_workspace()
        self._keep = (inp8, par)
        with self._on_device():
            self._check(lib().vda_prepare_fp8(
                self._ctx, _ptr(inp8["K8"]), _ptr(inp8["V8"]), _ptr(inp8["kv_scale"]), _ptr(inp8["Kt8"]),
                _ptr(inp8["Vt8"]), _ptr(inp8["kvt_scale"]), _ptr(par["alpha"]), _ptr(par["beta"]),
                _ptr(par["beta_txt"]), _ptr(ws), ws.numel(), _stream_handle(stream)), "vda_prepare_fp8")

    def readout_fp8(self, Q8: torch.Tensor, q_scale: torch.Tensor, O: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
        """The readout from e4m3 queries with per-(token, head) float32 scales
        (vda_readout_fp8), after prepare and scan_bidir."""
        cfg = self.cfg
        self._expect("Q8", Q8, (cfg.B, cfg.T * cfg.U, cfg.H, cfg.d), torch.float8_e4m3fn)
        self._expect("q_scale", q_scale, (cfg.B, cfg.T * cfg.U, cfg.H), torch.float32)
        if O is None:
            O = self.new_output()
        self._expect("O", O, (cfg.B, cfg.T * cfg.U, cfg.H, cfg.d), torch.bfloat16)
        with self._on_device():
            self._check(lib().vda_readout_fp8(self._ctx, _ptr(Q8), _ptr(q_scale), _ptr(O), _stream_handle(stream)),
                        "vda_readout_fp8")
        return O

    def new_output(self) -> torch.Tensor:
        cfg = self.cfg
        dt = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
        return torch.empty(cfg.B, cfg.T * cfg.U, cfg.H, cfg.d, dtype=dt, device=self.device)

    def run(self, inp: Dict[str, torch.Tensor], O: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """One pass of the whole path: prepare, bidirectional scan, readout."""
        if O is None:
            O = self.new_output()
        gate = inp.get("gate")
        self.check_inputs(inp)
        self.check_output(O, gate)
        with self._on_device():
            self._prepare(inp, stream)
            self._check(lib().vda_scan_bidir(self._ctx, _stream_handle(stream)), "vda_scan_bidir")
            self._check(lib().vda_readout(self._ctx, _ptr(gate), _ptr(O), _stream_handle(stream)), "vda_readout")
        return O

    def window_attention(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                         gate: Optional[torch.Tensor] = None, O: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
        """The softmax branch (window + anchor attention, optional sigmoid gate)
        over the same token tensors as the linear branch."""
        cfg = self.cfg
        sd = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
        shape = (cfg.B, cfg.T * cfg.U, cfg.H, cfg.d)
        for name, t in (("Q", Q), ("K", K), ("V", V)):
            self._expect(name, t, shape, sd)
        if gate is not None:
            self._expect("gate", gate, shape, sd)
        if O is None:
            O = self.new_output()
        self._expect("O", O, shape, sd)
        if self._attn_ws is None:
            self._attn_ws = torch.zeros(256, dtype=torch.uint8, device=self.device)
        with self._on_device():
            self._check(lib().vda_window_attention(self._ctx, _ptr(Q), _ptr(K), _ptr(V), _ptr(gate), _ptr(O),
                                                   _ptr(self._attn_ws), 256, _stream_handle(stream)),
                        "vda_window_attention")
        return O

    def frame_solve_backward(self, K: torch.Tensor, V: torch.Tensor, alpha: torch.Tensor, beta: torch.Tensor,
                             S_prev: torch.Tensor, dS: torch.Tensor, stream=None,
                             out: Optional[Dict[str, torch.Tensor]] = None) -> Dict[str, torch.Tensor]:
        """Backward of the frame step for frames 1..T-2 (vda_frame_solve_backward).
        Returns dK, dV (storage dtype) and dS_prev, dalpha, dbeta (float32), zero
        on the anchor frames (``out``, from an earlier call, is written again)."""
        cfg = self.cfg
        sd = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
        B, H, T, U, d = cfg.B, self.c.H, cfg.T, cfg.U, cfg.d
        tok = (cfg.B, T * U, cfg.H, d)
        self._expect("K", K, tok, sd)
        self._expect("V", V, tok, sd)
        p = self._head_params({"alpha": alpha, "beta": beta, "beta_txt": beta[:, :, 0]}) if self.heads else \
            {"alpha": alpha, "beta": beta}
        self._expect("alpha", p["alpha"], (B, H, T, d), torch.float32)
        self._expect("beta", p["beta"], (B, H, T, U), torch.float32)
        self._expect("S_prev", S_prev, (B, H, T, d, d), torch.float32)
        self._expect("dS", dS, (B, H, T, d, d), torch.float32)
        if out is None:
            out = {"dK": torch.zeros(tok, dtype=sd, device=self.device),
                   "dV": torch.zeros(tok, dtype=sd, device=self.device),
                   "dS_prev": torch.zeros_like(S_prev), "dalpha": torch.zeros_like(p["alpha"]),
                   "dbeta": torch.zeros_like(p["beta"])}
        ws = self.ensure_workspace()
        with self._on_device():
            self._check(lib().vda_frame_solve_backward(
                self._ctx, _ptr(K), _ptr(V), _ptr(p["alpha"]), _ptr(p["beta"]), _ptr(S_prev), _ptr(dS),
                _ptr(out["dK"]), _ptr(out["dV"]), _ptr(out["dalpha"]), _ptr(out["dbeta"]), _ptr(out["dS_prev"]),
                _ptr(ws), ws.numel(), _stream_handle(stream)), "vda_frame_solve_backward")
        return out

    def poll_device_status(self, stream=None) -> int:
        with self._on_device():
            return lib().vda_poll_device_status(self._ctx, _stream_handle(stream))

    def region(self, name: str) -> torch.Tensor:
        """A view of one workspace region (float32 unless it is a prepared token copy)."""
        off, nb = workspace_region(self.c, name)
        raw = self.ensure_workspace()[off:off + nb]
        cfg = self.cfg.with_(H=self.c.H)  # the context's heads (all of them unless sliced)
        D = cfg.d
        if name in ("A", "B", "M", "C"):
            return _from_quads(raw, (cfg.B, cfg.H, cfg.T - 1), D)
        if name in ("S_fwd", "S_rev"):
            return _from_quads(raw, (cfg.B, cfg.H, cfg.J), D)
        if name == "status":
            return raw.view(torch.int32)
        if name == "chunk_C":
            return _from_quads(raw, (cfg.B, cfg.H, 2, cfg.J), D)
        if name == "M_split":  # decoded: float32 [B, H, T-1, 2 (hi, lo), D, D]
            return _from_images(raw, (cfg.B, cfg.H, cfg.T - 1, 2), D)
        if name == "chunk_M":
            return _from_images(raw, (cfg.B, cfg.H, 2, cfg.J, 2), D)
        dt = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
        if name in ("K_prep", "V_prep"):
            return raw.view(dt).view(cfg.B, cfg.H, cfg.T, cfg.U, D)
        return raw.view(dt).view(cfg.B, cfg.H, cfg.L, D)

    # -- profiling ---------------------------------------------------------------
    def profile_enable(self, on: bool = True):
        self._check(lib().vda_profile_enable(self._ctx, int(on)), "vda_profile_enable")

    def profile_read(self) -> Dict[str, tuple]:
        out = {}
        for k in range(lib().vda_num_kernels()):
            name, n, ms = ctypes.c_char_p(), ctypes.c_int(0), ctypes.c_double(0)
            self._check(lib().vda_profile_read(self._ctx, k, ctypes.byref(name), ctypes.byref(n),
                                               ctypes.byref(ms)), "vda_profile_read")
            if n.value:
                out[name.value.decode()] = (n.value, ms.value)
        return out

    def launch_count(self) -> int:
        n = ctypes.c_uint64(0)
        self._check(lib().vda_launch_count(self._ctx, ctypes.byref(n)), "vda_launch_count")
        return n.value


def _from_quads(raw: torch.Tensor, lead: tuple, D: int) -> torch.Tensor:
    """Row-major (..., D, D) copy of fp32 d x d matrices stored in column quads
    (element (i, j) at float ((j // 4) * D + i) * 4 + j % 4)."""
    q = raw.view(torch.float32).view(*lead, D // 4, D, 4)
    return q.movedim(-3, -2).reshape(*lead, D, D)


def _image_index(D: int) -> torch.Tensor:
    """Element offset of (i, j) in a bf16 D x D operand image (128-byte rows of
    64 elements, 16-byte chunks XOR-swizzled by i % 8, 64-column atoms)."""
    i = torch.arange(D).view(D, 1)
    j = torch.arange(D).view(1, D)
    byte = (j // 64) * D * 128 + i * 128 + (((j % 64) // 8) ^ (i % 8)) * 16 + (j % 8) * 2
    return byte // 2


def _from_images(raw: torch.Tensor, lead: tuple, D: int) -> torch.Tensor:
    """Row-major float32 copies of bf16 operand images."""
    flat = raw.view(torch.bfloat16).view(*lead, D * D)
    idx = _image_index(D).to(flat.device).view(-1)
    return flat.index_select(-1, idx).view(*lead, D, D).float()


def run_static_workspace(cfg: VDAConfig, inp: Dict[str, torch.Tensor], O: torch.Tensor, stream=None) -> int:
    """The whole path through vda_run_static_workspace (library-owned scratch)."""
    c = make_config(cfg)
    return lib().vda_run_static_workspace(
        ctypes.byref(c), _ptr(inp["Q"]), _ptr(inp["K"]), _ptr(inp["V"]), _ptr(inp["K_txt"]), _ptr(inp["V_txt"]),
        _ptr(inp["alpha"]), _ptr(inp["beta"]), _ptr(inp["beta_txt"]), _ptr(inp.get("conv_w")),
        _ptr(inp.get("gate")), _ptr(O), _stream_handle(stream))


def hybrid_merge(O_soft: torch.Tensor, W_soft: torch.Tensor, O_lin: torch.Tensor, W_lin: torch.Tensor,
                 Y: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """Y = O_soft W_soft^T + O_lin W_lin^T through vda_hybrid_merge. The branch
    outputs may be [B, T*U, H, d] (viewed as [B*T*U, H*d]); the projections are
    [N, H*d] bf16. ``status`` (256 device bytes) receives the call's status word."""
    M = O_soft.numel() // O_soft.shape[-1] // (O_soft.shape[-2] if O_soft.dim() == 4 else 1)
    K = W_soft.shape[1]
    N = W_soft.shape[0]
    for name, t in (("O_soft", O_soft), ("O_lin", O_lin), ("W_soft", W_soft), ("W_lin", W_lin)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    if O_soft.numel() != M * K or O_lin.numel() != M * K or tuple(W_lin.shape) != (N, K):
        raise ValueError("O_soft, O_lin must hold M x K values and W_soft, W_lin be N x K")
    if Y is None:
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=O_soft.device)
    if status is None:
        status = torch.zeros(256, dtype=torch.uint8, device=O_soft.device)
    st = lib().vda_hybrid_merge(_ptr(O_soft), _ptr(W_soft), _ptr(O_lin), _ptr(W_lin), _ptr(Y), M, N, K,
                                _ptr(status), status.numel(), _stream_handle(stream))
    if st != VDA_OK:
        raise VDAError(st, "vda_hybrid_merge")
    return Y


def static_workspace_poll(stream=None) -> int:
    """Status of the last vda_run_static_workspace call on the current device
    (synchronises the stream; VDA_ERR_TIMEOUT if a device-side wait gave up)."""
    return lib().vda_static_workspace_poll(_stream_handle(stream))


def selftest_recip(x: torch.Tensor, stream=None) -> torch.Tensor:
    """The sweep solve's pivot reciprocal applied to a float32 CUDA tensor."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 CUDA tensor")
    y = torch.empty_like(x)
    st = lib().vda_selftest_recip(_ptr(x), _ptr(y), x.numel(), _stream_handle(stream))
    if st != VDA_OK:
        raise VDAError(st, "vda_selftest_recip")
    return y


def selftest_bounded_wait(status: torch.Tensor, spins: int, stream=None) -> int:
    return lib().vda_selftest_bounded_wait(_ptr(status), spins, _stream_handle(stream))


def to_device(inp: Dict[str, torch.Tensor], device="cuda") -> Dict[str, torch.Tensor]:
    return {k: v.to(device, non_blocking=True) for k, v in inp.items()}
