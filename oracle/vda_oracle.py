"""Float64 CPU oracle for Video Delta Attention (VDA) -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module. The CUDA library never calls it and shares
no code with it; the product path fails loudly when its CUDA extension is missing.

Sources (web pages on Video DeltaNet, cited by title and section):
  [P1] "Video DeltaNet: removing the attention bottleneck of video diffusion
       with a frame-level delta rule and bidirectional linear memory"
       (onedev.kr/papers/80), sections "how it works" (어떻게 동작하나),
       "how it differs" (무엇과 다른가), "how to use" (어떻게 쓰나) and
       "assumptions and limits" (전제와 한계).
  [P3] "VDN-H3: a hybrid attention model that generates MiniMax H3 video faster
       than playback" (discuss.pytorch.kr), section "hybrid attention structure".

Every function is a plain statement of the definition: library primitives
(matrix products, ``numpy.linalg.solve``) serve as single steps, with no
blocking, fusion or reordering beyond what the definition states.

Readings taken where the pages are silent (each listed in the design notes):
  * S is d_v x d_k, a query reads o = S q, Diag(alpha) multiplies on the right.
  * The text state is S_T = B_txt (I + A_txt)^-1, the frame solve from S = 0.
  * The reverse scan absorbs frame t with the same M_t, C_t as the forward scan.
  * Chunk j = floor(t / c); the forward readout state is the forward state after
    frame c(j-1)-1 (S_T/2 if that is < 1); the reverse readout state is the
    reverse state after frame c(j+2) (S_T/2 if that is > T-2). Anchor frames 0
    and T-1 are absorbed by neither scan and read out exactly zero.
  * Feature prep (conv workloads): depthwise 5x5 spatial and centred 5-tap
    temporal cross-correlation, zero "same" padding, no bias, then SiLU; K and Q
    divided by sqrt(|x|^2 + eps); text K, V get SiLU and L2(K) only.
  * RMSNorm weight 1, eps inside the square root; eps = 1e-6 for both norms.

Parity status: every function below is pinned by the CPU tests (closed forms,
invariants, brute-force least squares, a hand-derived worked example and an
independent library routine for the convolution). No function is unpinned.
"""
from __future__ import annotations

from typing import Dict, Iterable, List, Optional, Tuple

import numpy as np

# ----------------------------------------------------------------------------
# Index sets  [P1 "how it works": chunk +-1 window, boundary anchors; P1
# "assumptions and limits": anchors excluded from the linear state]
# ----------------------------------------------------------------------------


def chunk_of(t: int, c: int) -> int:
    """Chunk index of latent frame t for chunks of c frames starting at frame 0."""
    return t // c


def forward_frames(j: int, c: int) -> List[int]:
    """Frames absorbed by the forward readout state of query chunk j: 1 .. c(j-1)-1."""
    return list(range(1, c * (j - 1)))


def reverse_frames(j: int, c: int, T: int) -> List[int]:
    """Frames absorbed by the reverse readout state of query chunk j: c(j+2) .. T-2."""
    return list(range(c * (j + 2), T - 1))


def window_frames(j: int, c: int, T: int) -> List[int]:
    """Softmax window of query chunk j: chunks j-1 .. j+1, truncated at the clip ends."""
    return list(range(max(0, c * (j - 1)), min(T - 1, c * (j + 2) - 1) + 1))


def anchor_frames(T: int) -> List[int]:
    return [0, T - 1]


# ----------------------------------------------------------------------------
# Feature prep  [P1 "how it differs": separable short conv on K and V (depthwise
# 5x5 spatial + 5-tap temporal), then SiLU; L2 norm on Q and K; no rotary]
# ----------------------------------------------------------------------------


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def l2_normalize(x: np.ndarray, eps: float) -> np.ndarray:
    """x / sqrt(|x|^2 + eps) over the last axis."""
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def depthwise_spatial_5x5(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Per-channel 5x5 cross-correlation with zero 'same' padding.

    x: [T, gh, gw, d]; w: [d, 5, 5]. out[t,y,x,ch] = sum_{a,b} w[ch,a,b] x[t,y+a-2,x+b-2,ch].
    """
    T, gh, gw, d = x.shape
    xp = np.zeros((T, gh + 4, gw + 4, d), dtype=np.float64)
    xp[:, 2:2 + gh, 2:2 + gw, :] = x
    out = np.zeros_like(x, dtype=np.float64)
    for a in range(5):
        for b in range(5):
            out += xp[:, a:a + gh, b:b + gw, :] * w[:, a, b]
    return out


def depthwise_temporal_5(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Per-channel centred 5-tap cross-correlation over frames with zero padding.

    x: [T, ...spatial..., d]; w: [d, 5]. out[t] = sum_s w[:, s] x[t+s-2].
    """
    T = x.shape[0]
    xp = np.zeros((T + 4,) + x.shape[1:], dtype=np.float64)
    xp[2:2 + T] = x
    out = np.zeros_like(x, dtype=np.float64)
    for s in range(5):
        out += xp[s:s + T] * w[:, s]
    return out


def prep_video_kv(X: np.ndarray, w_spatial: np.ndarray, w_temporal: np.ndarray,
                  grid_h: int, grid_w: int) -> np.ndarray:
    """Conv (spatial then temporal; the two commute under zero padding) then SiLU.

    X: [T, U, d] for one head, tokens row-major over the gh x gw latent grid.
    """
    T, U, d = X.shape
    x = X.reshape(T, grid_h, grid_w, d)
    x = depthwise_spatial_5x5(x, w_spatial)
    x = depthwise_temporal_5(x, w_temporal)
    return silu(x).reshape(T, U, d)


# ----------------------------------------------------------------------------
# Frame statistics and frame solve  [P1 "how to use": A_t = K^T Diag(beta) K,
# B_t = V^T Diag(beta) K, objective argmin_S 1/2|S - Sbar|_F^2 +
# 1/2 sum_u beta_u |S k_u - v_u|^2  =>  S (I + A) = Sbar + B; M_t =
# Diag(alpha)(I + A)^-1; inverse taken in the d_k x d_k key space]
# ----------------------------------------------------------------------------


def frame_stats(Kf: np.ndarray, Vf: np.ndarray, beta: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """A = K^T Diag(beta) K  (d_k x d_k),  B = V^T Diag(beta) K  (d_v x d_k).

    Kf: [U, d_k], Vf: [U, d_v], beta: [U].
    """
    bK = Kf * beta[:, None]
    return Kf.T @ bK, Vf.T @ bK


def frame_solve(A: np.ndarray, B: np.ndarray, alpha: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """M = Diag(alpha) (I + A)^-1 and C = B (I + A)^-1, so that S_t = S_{t-1} M + C.

    Since S_t = (S_{t-1} Diag(alpha) + B)(I + A)^-1, the transition is
    Diag(alpha)(I+A)^-1 and the injection is B (I+A)^-1.
    """
    d_k = A.shape[0]
    P = np.linalg.solve(np.eye(d_k) + A, np.eye(d_k))
    return alpha[:, None] * P, B @ P


def text_state(A_txt: np.ndarray, B_txt: np.ndarray) -> np.ndarray:
    """S_T: the frame solve from S = 0 over the text tokens, B_txt (I + A_txt)^-1.

    [P1 "how it works": all text tokens are summarised into S_T before the video
    scan; P1 "assumptions and limits" (notes on the inference kernels): the
    prompt enters as a leading virtual frame.]
    (I + A) is symmetric, so S (I + A) = B is the transpose of (I + A) S^T = B^T.
    """
    d_k = A_txt.shape[0]
    return np.linalg.solve(np.eye(d_k) + A_txt, B_txt.T).T


# ----------------------------------------------------------------------------
# Bidirectional scan and readout  [P1 "how it works": forward state summarises
# frames before the window, reverse state frames after it, disjoint, o = S-> q +
# S<- q, each direction starts at S_T/2 so the prompt counts once]
# ----------------------------------------------------------------------------


def forward_scan(M: Dict[int, np.ndarray], C: Dict[int, np.ndarray], S0: np.ndarray,
                 frames: Iterable[int]) -> Dict[int, np.ndarray]:
    """F(0) = S0; F(t) = F(t-1) M_t + C_t over the given increasing frames."""
    states = {0: S0}
    S = S0
    for t in frames:
        S = S @ M[t] + C[t]
        states[t] = S
    return states


def reverse_scan(M: Dict[int, np.ndarray], C: Dict[int, np.ndarray], S0: np.ndarray,
                 frames: Iterable[int], T: int) -> Dict[int, np.ndarray]:
    """R(T-1) = S0; R(t) = R(t+1) M_t + C_t over the given decreasing frames."""
    states = {T - 1: S0}
    S = S0
    for t in frames:
        S = S @ M[t] + C[t]
        states[t] = S
    return states


def rms_norm_gate(o: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """y = o / sqrt(mean(o^2) + eps) * sigmoid(g) over the last axis (weight 1).

    [P1 "how it differs": the linear readout passes RMS normalisation and then its
    own sigmoid output gate; P3 "hybrid attention structure": RMSNorm then an
    elementwise sigmoid gate.]
    """
    r = o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    return r * (1.0 / (1.0 + np.exp(-g)))


# ----------------------------------------------------------------------------
# Whole linear branch
# ----------------------------------------------------------------------------


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor; upcast its exact stored values
        x = x.detach().to("cpu")
        import torch  # local: only to read tensors handed in by tests
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def vda_reference(inp: Dict, cfg, heads: Optional[Iterable[Tuple[int, int]]] = None,
                  keep: bool = True) -> Dict[str, object]:
    """Run the linear branch for the (b, h) pairs in ``heads`` (default: all).

    ``inp`` holds Q, K, V [B, T*U, H, d], K_txt, V_txt [B, L, H, d], alpha
    [B, H, T, d], beta [B, H, T, U], beta_txt [B, H, L] and, when used,
    conv_w (four concatenated filters) and gate [B, T*U, H, d]. ``cfg`` has
    B, H, d, T, grid_h, grid_w, chunk, L, prep_conv, norm_gate.

    Returns ``O`` ([B, T*U, H, d] float64, zero for heads not computed) and, when
    ``keep``, per-(b, h) intermediates: A, B (slot 0 = text, slot t = frame t),
    M, C, S_T, all forward and reverse states, the per-chunk readout states, and
    the Euclidean norm of every token's readout before RMSNorm and the gate
    (o_pre_norm, [T*U], zero on anchor frames).
    """
    B_, H, d, T, c = cfg.B, cfg.H, cfg.d, cfg.T, cfg.chunk
    gh, gw = cfg.grid_h, cfg.grid_w
    U = gh * gw
    J = -(-T // c)
    eps = 1e-6
    if heads is None:
        heads = [(b, h) for b in range(B_) for h in range(H)]
    heads = list(heads)

    O = np.zeros((B_, T * U, H, d), dtype=np.float64)
    inter: Dict[Tuple[int, int], Dict[str, object]] = {}
    conv = None
    if cfg.prep_conv:
        w = _f64(inp["conv_w"])
        hd = H * d
        conv = (w[:hd * 25].reshape(H, d, 5, 5), w[hd * 25:hd * 30].reshape(H, d, 5),
                w[hd * 30:hd * 55].reshape(H, d, 5, 5), w[hd * 55:hd * 60].reshape(H, d, 5))

    for (b, h) in heads:
        Qh = _f64(inp["Q"][b, :, h, :]).reshape(T, U, d)
        Kh = _f64(inp["K"][b, :, h, :]).reshape(T, U, d)
        Vh = _f64(inp["V"][b, :, h, :]).reshape(T, U, d)
        Kt = _f64(inp["K_txt"][b, :, h, :])
        Vt = _f64(inp["V_txt"][b, :, h, :])
        alpha = _f64(inp["alpha"][b, h])
        beta = _f64(inp["beta"][b, h])
        beta_t = _f64(inp["beta_txt"][b, h])
        if cfg.prep_conv:
            Kh = l2_normalize(prep_video_kv(Kh, conv[0][h], conv[1][h], gh, gw), eps)
            Vh = prep_video_kv(Vh, conv[2][h], conv[3][h], gh, gw)
            Kt = l2_normalize(silu(Kt), eps)
            Vt = silu(Vt)
            Qh = l2_normalize(Qh, eps)

        # Text: the frame solve from S = 0.
        A_txt, B_txt = frame_stats(Kt, Vt, beta_t)
        S_T = text_state(A_txt, B_txt)

        # Frames 1..T-2 (anchors 0 and T-1 are never absorbed).
        A, Bm, M, C = {0: A_txt}, {0: B_txt}, {}, {}
        for t in range(1, T - 1):
            A[t], Bm[t] = frame_stats(Kh[t], Vh[t], beta[t])
            M[t], C[t] = frame_solve(A[t], Bm[t], alpha[t])

        F = forward_scan(M, C, S_T / 2.0, range(1, T - 1))
        R = reverse_scan(M, C, S_T / 2.0, range(T - 2, 0, -1), T)

        S_fwd, S_rev = [], []
        for j in range(J):
            S_fwd.append(F[max(0, c * (j - 1) - 1)])
            S_rev.append(R[min(T - 1, c * (j + 2))])

        o_pre_norm = np.zeros(T * U)
        for t in range(1, T - 1):
            j = chunk_of(t, c)
            S = S_fwd[j] + S_rev[j]
            o = Qh[t] @ S.T  # row u is S q_u
            o_pre_norm[t * U:(t + 1) * U] = np.linalg.norm(o, axis=1)
            if cfg.norm_gate:
                g = _f64(inp["gate"][b, t * U:(t + 1) * U, h, :])
                o = rms_norm_gate(o, g, eps)
            O[b, t * U:(t + 1) * U, h, :] = o

        if keep:
            inter[(b, h)] = dict(A=A, B=Bm, M=M, C=C, S_T=S_T, F=F, R=R,
                                 S_fwd=S_fwd, S_rev=S_rev, o_pre_norm=o_pre_norm)
    return {"O": O, "inter": inter, "heads": heads}


# ----------------------------------------------------------------------------
# Backward of one frame step (for training)  [P1 "assumptions and limits": the
# frame-level update is trained end to end (stages A1/A2/B); the pages print no
# backward, so this is the plain chain rule of the forward step above]
# ----------------------------------------------------------------------------


def frame_step(S_prev: np.ndarray, Kf: np.ndarray, Vf: np.ndarray, beta: np.ndarray,
               alpha: np.ndarray) -> np.ndarray:
    """One frame of the scan: S_t = S_{t-1} M_t + C_t with M_t, C_t from frame_solve."""
    A, B = frame_stats(Kf, Vf, beta)
    M, C = frame_solve(A, B, alpha)
    return S_prev @ M + C


def frame_step_backward(S_prev: np.ndarray, Kf: np.ndarray, Vf: np.ndarray, beta: np.ndarray,
                        alpha: np.ndarray, dS: np.ndarray) -> Dict[str, np.ndarray]:
    """Vector-Jacobian product of frame_step: given dS = dL/dS_t, the gradients of
    L with respect to S_{t-1}, K_t, V_t, beta_t and alpha_t.

    With P = (I + A)^-1 (symmetric), X = S_{t-1} Diag(alpha) + B and S_t = X P:
      dL/dX = dS P^T = dS P =: Gx           (so dL/dB = Gx, dL/dS_{t-1} = Gx Diag(alpha))
      dL/dP = X^T dS,  dL/dA = -P^T (X^T dS) P^T = -S_t^T Gx =: GA
      dL/dalpha_k = sum_i S_{t-1}[i, k] Gx[i, k]
    and through A = sum_u beta_u k_u k_u^T, B = sum_u beta_u v_u k_u^T:
      dL/dk_u = beta_u ((GA + GA^T) k_u + Gx^T v_u)
      dL/dv_u = beta_u Gx k_u
      dL/dbeta_u = k_u^T GA k_u + v_u^T Gx k_u.
    """
    A, B = frame_stats(Kf, Vf, beta)
    d_k = A.shape[0]
    P = np.linalg.solve(np.eye(d_k) + A, np.eye(d_k))
    X = S_prev * alpha[None, :] + B
    S = X @ P
    Gx = dS @ P.T
    GA = -(S.T @ Gx)
    out = {
        "dS_prev": Gx * alpha[None, :],
        "dalpha": np.sum(S_prev * Gx, axis=0),
        "dK": beta[:, None] * (Kf @ (GA + GA.T).T + Vf @ Gx),
        "dV": beta[:, None] * (Kf @ Gx.T),
        "dbeta": np.einsum("uk,kl,ul->u", Kf, GA, Kf) + np.einsum("uv,vk,uk->u", Vf, Gx, Kf),
    }
    return out
