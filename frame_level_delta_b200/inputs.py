"""Seeded synthetic inputs for the Video Delta Attention (VDA) linear branch.

This module is shared by the CUDA path's tests and benchmark and by the tests of
the float64 oracle. It draws random numbers and rounds them to their storage
dtype; it holds none of the method's arithmetic (no statistics, solves, scans or
readouts).

Workloads (sizes follow the Video DeltaNet summary, onedev.kr/papers/80, section
"how it works": chunks of 5 latent frames, a +-1-chunk softmax window, boundary
anchors at the first and last frame, text tokens summarised into the state):

=====  ======================================================================
name   shapes
=====  ======================================================================
tiny   B=1 H=1  d=16  T=12  U=16   (4x4)   c=2 L=8   fp32
small  B=1 H=8  d=64  T=20  U=256  (16x16) c=5 L=64  bf16
h3     B=1 H=24 d=128 T=40  U=1560 (30x52) c=5 L=512 bf16   (H3-like clip)
long   B=1 H=24 d=128 T=120 U=1560 (30x52) c=5 L=512 bf16   slow decay
hires  B=1 H=24 d=128 T=40  U=3600 (45x80) c=5 L=512 bf16   conv prep + RMSNorm/gate
=====  ======================================================================

Draw order (one CPU ``torch.Generator`` seeded once, fp32 draws):
  1. Q, K, V              [B, T*U, H, d]      N(0, 1)
  2. K_txt, V_txt         [B, L, H, d]        N(0, 1)
  3. beta logits          [B, H, T, U]        N(0, 1)     -> beta = sigmoid
  4. beta_txt logits      [B, H, L]           N(0, 1)     -> sigmoid
  5. alpha logits         [B, H, T, d_k]      N(mu_a, 1)  -> alpha = sigmoid
  6. (hires only) conv weights K-spatial [H*d,5,5], K-temporal [H*d,5],
     V-spatial [H*d,5,5], V-temporal [H*d,5], each N(0,1)*0.05, then
     gate logits [B, T*U, H, d_v] N(0, 1).

For every workload except ``hires`` the features arrive already prepared: Q, K
and K_txt are divided by their per-token Euclidean norm (in fp32) as part of the
input distribution. Rounding to the storage dtype (round-to-nearest-even for
bf16) is the last step, so both the oracle and the GPU see identical values.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class VDAConfig:
    """One synthetic workload. ``d`` is both d_k and d_v."""

    name: str
    B: int
    H: int
    d: int
    T: int
    grid_h: int
    grid_w: int
    chunk: int
    L: int
    dtype: str  # "f32" or "bf16": storage of Q, K, V, K_txt, V_txt, gate, O
    alpha_mu: float = 3.0
    beta_mu: float = 0.0
    prep_conv: bool = False  # depthwise 5x5 spatial + 5-tap temporal conv + SiLU on K, V; L2 on Q, K
    norm_gate: bool = False  # RMSNorm then sigmoid gate on the linear readout
    seed: int = 0

    @property
    def U(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def J(self) -> int:
        return -(-self.T // self.chunk)

    @property
    def head_tokens(self) -> int:
        return self.B * self.H * self.T * self.U

    def with_(self, **kw) -> "VDAConfig":
        return dataclasses.replace(self, **kw)


CONFIGS: Dict[str, VDAConfig] = {
    "tiny": VDAConfig("tiny", B=1, H=1, d=16, T=12, grid_h=4, grid_w=4, chunk=2, L=8, dtype="f32"),
    "small": VDAConfig("small", B=1, H=8, d=64, T=20, grid_h=16, grid_w=16, chunk=5, L=64, dtype="bf16"),
    "h3": VDAConfig("h3", B=1, H=24, d=128, T=40, grid_h=30, grid_w=52, chunk=5, L=512, dtype="bf16"),
    "long": VDAConfig("long", B=1, H=24, d=128, T=120, grid_h=30, grid_w=52, chunk=5, L=512,
                      dtype="bf16", alpha_mu=4.0),
    "hires": VDAConfig("hires", B=1, H=24, d=128, T=40, grid_h=45, grid_w=80, chunk=5, L=512,
                       dtype="bf16", prep_conv=True, norm_gate=True),
}
# The five workloads in their published order (1-based numbering used in docs).
CONFIG_ORDER = ["tiny", "small", "h3", "long", "hires"]


def storage_dtype(cfg: VDAConfig) -> torch.dtype:
    return torch.float32 if cfg.dtype == "f32" else torch.bfloat16


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    # Part of the input distribution ("Q, K L2-normalised per token"), not of the
    # method: the prepared-feature workloads hand the library unit-norm keys.
    return x / x.norm(dim=-1, keepdim=True)


def make_inputs(cfg: VDAConfig, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Draw one seeded batch of CPU tensors in the layouts the C ABI takes.

    Returns a dict with Q, K, V, K_txt, V_txt (storage dtype), alpha, beta,
    beta_txt (fp32), and for ``prep_conv`` workloads ``conv_w`` (fp32, the four
    filters concatenated: K-spatial, K-temporal, V-spatial, V-temporal) and
    ``gate`` (storage dtype) when ``norm_gate`` is set.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(cfg.seed if seed is None else seed)
    B, H, d, T, U, L = cfg.B, cfg.H, cfg.d, cfg.T, cfg.U, cfg.L
    sd = storage_dtype(cfg)

    def randn(*shape):
        return torch.randn(*shape, generator=g, dtype=torch.float32)

    Q = randn(B, T * U, H, d)
    K = randn(B, T * U, H, d)
    V = randn(B, T * U, H, d)
    Kt = randn(B, L, H, d)
    Vt = randn(B, L, H, d)
    beta = torch.sigmoid(randn(B, H, T, U) + cfg.beta_mu)
    beta_txt = torch.sigmoid(randn(B, H, L) + cfg.beta_mu)
    alpha = torch.sigmoid(randn(B, H, T, d) + cfg.alpha_mu)
    out = {}
    if cfg.prep_conv:
        hd = H * d
        w = [randn(hd, 5, 5) * 0.05, randn(hd, 5) * 0.05, randn(hd, 5, 5) * 0.05, randn(hd, 5) * 0.05]
        out["conv_w"] = torch.cat([x.reshape(-1) for x in w]).contiguous()
    else:
        Q, K, Kt = _unit_rows(Q), _unit_rows(K), _unit_rows(Kt)
    if cfg.norm_gate:
        out["gate"] = randn(B, T * U, H, d).to(sd).contiguous()
    out.update(
        Q=Q.to(sd).contiguous(), K=K.to(sd).contiguous(), V=V.to(sd).contiguous(),
        K_txt=Kt.to(sd).contiguous(), V_txt=Vt.to(sd).contiguous(),
        alpha=alpha.contiguous(), beta=beta.contiguous(), beta_txt=beta_txt.contiguous(),
    )
    return out


def split_conv_w(conv_w: torch.Tensor, H: int, d: int):
    """View the concatenated filter buffer as its four [H, d, ...] parts."""
    hd = H * d
    sizes = [hd * 25, hd * 5, hd * 25, hd * 5]
    parts = torch.split(conv_w, sizes)
    return (parts[0].reshape(H, d, 5, 5), parts[1].reshape(H, d, 5),
            parts[2].reshape(H, d, 5, 5), parts[3].reshape(H, d, 5))


def make_attention_inputs(cfg: VDAConfig, logit_std: float = 1.0, seed: Optional[int] = None,
                          gate: bool = True) -> Dict[str, torch.Tensor]:
    """Seeded inputs of the softmax branch in the layouts the C ABI takes: Q, K,
    V [B, T*U, H, d] and the branch's gate logits g [B, T*U, H, d] (storage dtype).

    K rows are unit vectors and Q rows have N(0, logit_std^2 d) entries, so the
    logits q.k / sqrt(d) are roughly N(0, logit_std^2): 1 gives the nearly flat
    weights of normalised features, larger values sharply peaked ones. V ~ N(0, 1),
    gate logits ~ N(0, 1). Draw order: Q, K, V, gate.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed((cfg.seed if seed is None else seed) + 1000)
    B, H, d, T, U = cfg.B, cfg.H, cfg.d, cfg.T, cfg.U
    sd = storage_dtype(cfg)

    def randn(*shape):
        return torch.randn(*shape, generator=g, dtype=torch.float32)

    Q = randn(B, T * U, H, d) * (logit_std * d ** 0.5)
    K = _unit_rows(randn(B, T * U, H, d))
    V = randn(B, T * U, H, d)
    out = {"Q": Q.to(sd).contiguous(), "K": K.to(sd).contiguous(),
           "V": V.to(sd).contiguous()}
    if gate:
        out["gate"] = randn(B, T * U, H, d).to(sd).contiguous()
    return out


def make_merge_inputs(M: int, N: int, K: int, seed: int = 0) -> Dict[str, torch.Tensor]:
    """Seeded inputs of the hybrid merge: the two gated branch outputs O_soft, O_lin
    [M, K] ~ N(0, 1) and the output projections W_soft, W_lin [N, K] ~ N(0, 1/K)
    (the [out, in] layout of a linear layer), all bf16. Draw order: O_soft, O_lin,
    W_soft, W_lin."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed + 2000)

    def randn(*shape, scale=1.0):
        return (torch.randn(*shape, generator=g, dtype=torch.float32) * scale).to(torch.bfloat16).contiguous()

    return {"O_soft": randn(M, K), "O_lin": randn(M, K), "W_soft": randn(N, K, scale=K ** -0.5),
            "W_lin": randn(N, K, scale=K ** -0.5)}


def make_backward_inputs(cfg: VDAConfig, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Seeded inputs of the frame-step backward on top of make_inputs(cfg): the
    state before each frame S_prev and the upstream gradient dS, both
    [B, H, T, d, d] float32 ~ N(0, 1) (row-major d_v x d_k per frame). Draw order:
    S_prev, dS."""
    g = torch.Generator(device="cpu")
    g.manual_seed((cfg.seed if seed is None else seed) + 3000)
    shape = (cfg.B, cfg.H, cfg.T, cfg.d, cfg.d)
    return {"S_prev": torch.randn(*shape, generator=g).contiguous(),
            "dS": torch.randn(*shape, generator=g).contiguous()}


def quantize_e4m3(x: torch.Tensor):
    """Per-row e4m3 quantisation of [..., d] values: scale = max|row| / 448 (1 for
    an all-zero row), x8 = round-to-nearest e4m3 of x / scale. Returns (x8, scale
    [...] float32); x8 * scale is what a consumer of the FP8 form sees. A storage
    format of the inputs, not part of the method."""
    xf = x.float()
    amax = xf.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    x8 = (xf / scale.unsqueeze(-1)).to(torch.float8_e4m3fn)
    return x8.contiguous(), scale.contiguous()


def quantize_e4m3_pair(k: torch.Tensor, v: torch.Tensor):
    """e4m3 form of a key and a value sharing one scale per row:
    scale = max(max|k_row|, max|v_row|) / 448. Returns (k8, v8, scale)."""
    kf, vf = k.float(), v.float()
    amax = torch.maximum(kf.abs().amax(dim=-1), vf.abs().amax(dim=-1))
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    s = scale.unsqueeze(-1)
    return ((kf / s).to(torch.float8_e4m3fn).contiguous(), (vf / s).to(torch.float8_e4m3fn).contiguous(),
            scale.contiguous())


def make_fp8_inputs(cfg: VDAConfig, seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """The FP8 storage form of make_inputs(cfg): Q8 with q_scale (per token and
    head), K8 and V8 sharing kv_scale, Kt8 and Vt8 sharing kvt_scale; alpha,
    beta, beta_txt as drawn by make_inputs. Also returns the exact stored values
    in float64 under Q, K, V, K_txt, V_txt (scale times e4m3 value), for the
    oracle."""
    inp = make_inputs(cfg, seed)
    Q8, qs = quantize_e4m3(inp["Q"])
    K8, V8, kvs = quantize_e4m3_pair(inp["K"], inp["V"])
    Kt8, Vt8, kvts = quantize_e4m3_pair(inp["K_txt"], inp["V_txt"])
    out = {"Q8": Q8, "q_scale": qs, "K8": K8, "V8": V8, "kv_scale": kvs, "Kt8": Kt8, "Vt8": Vt8,
           "kvt_scale": kvts, "alpha": inp["alpha"], "beta": inp["beta"], "beta_txt": inp["beta_txt"]}
    out["Q"] = Q8.double() * qs.double().unsqueeze(-1)
    out["K"] = K8.double() * kvs.double().unsqueeze(-1)
    out["V"] = V8.double() * kvs.double().unsqueeze(-1)
    out["K_txt"] = Kt8.double() * kvts.double().unsqueeze(-1)
    out["V_txt"] = Vt8.double() * kvts.double().unsqueeze(-1)
    return out
