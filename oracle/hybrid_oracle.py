"""Float64 CPU oracle for the softmax half of the VDN attention layer and the
hybrid merge -- TEST INFRASTRUCTURE ONLY.

Only the tests may import this module. It extends the linear-branch oracle in
``oracle/vda_oracle.py`` (whose index sets it reuses) with the other branch of
the same layer. No CUDA kernel implements it yet.

Sources (cited by title and section):
  [P1] "Video DeltaNet: removing the attention bottleneck of video diffusion
       with a frame-level delta rule and bidirectional linear memory"
       (onedev.kr/papers/80), sections "how it works" (the +-1 chunk window and
       the two boundary anchors) and "how it differs" (shared QKV, the sigmoid
       gate on the softmax readout, separate output projections summed).
  [P3] "VDN-H3: a hybrid attention model that generates MiniMax H3 video faster
       than playback" (discuss.pytorch.kr), section "hybrid attention structure"
       (chunks of five latent frames, the window, the four-way anchors and the
       3.57% density they add).

Readings taken where the pages are silent (each listed in the design notes):
  * A query of frame t (not an anchor) sees every token of the frames in chunks
    j-1 .. j+1 (j = floor(t / c), truncated at the clip ends) and every token of
    frames 0 and T-1; a query of frame 0 or T-1 sees every video token.
  * Scaled dot-product logits q.k / sqrt(d); the softmax branch's Q and K arrive
    with the backbone's own QK normalisation and rotary embedding applied.
  * The branch is video-to-video: text keys are not part of it.
  * The softmax gate is elementwise: O~S = O^S * sigmoid(g^S), with the gate
    logits g^S an input of the layer (the model computes them from the token).
  * Y = O~S W_S + O~L W_L with W_S, W_L of shape [H d, D_model], the heads
    concatenated in order.

Parity status: pinned by the CPU tests (the anchor density printed in [P3], a
token-pair mask built from the chunk-distance rule, the reduction to dense
attention, convex-combination and permutation properties, closed forms of the
gate and the merge). No function is unpinned.
"""
from __future__ import annotations

from typing import List

import numpy as np

from oracle.vda_oracle import anchor_frames, chunk_of, window_frames


def visible_frames(t: int, c: int, T: int) -> List[int]:
    """Frames whose tokens a query token of frame t attends to."""
    if t in anchor_frames(T):
        return list(range(T))
    return sorted(set(window_frames(chunk_of(t, c), c, T)) | set(anchor_frames(T)))


def attention_density(T: int, c: int, anchors: bool = True) -> float:
    """Fraction of (query frame, key frame) pairs that are visible. Every frame
    holds the same number of tokens, so this is also the token-pair density."""
    pairs = 0
    for t in range(T):
        if anchors:
            pairs += len(visible_frames(t, c, T))
        else:
            pairs += len(window_frames(chunk_of(t, c), c, T))
    return pairs / float(T * T)


def window_softmax_head(Q: np.ndarray, K: np.ndarray, V: np.ndarray, T: int, U: int, c: int,
                        scale: float = None) -> np.ndarray:
    """Softmax attention of one (b, h) over the window + anchor pattern.

    Q, K: [T U, d_k]; V: [T U, d_v]; tokens frame-major. Returns O^S [T U, d_v].
    """
    d_k = Q.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d_k)
    O = np.zeros((T * U, V.shape[1]))
    for t in range(T):
        keys = np.concatenate([np.arange(f * U, (f + 1) * U) for f in visible_frames(t, c, T)])
        logits = (Q[t * U:(t + 1) * U] @ K[keys].T) * scale
        logits = logits - logits.max(axis=1, keepdims=True)
        w = np.exp(logits)
        w = w / w.sum(axis=1, keepdims=True)
        O[t * U:(t + 1) * U] = w @ V[keys]
    return O


def window_softmax_rows(Q: np.ndarray, K: np.ndarray, V: np.ndarray, T: int, U: int, c: int,
                        rows, scale: float = None) -> np.ndarray:
    """The same attention as window_softmax_head for selected query tokens only
    (token indices into the frame-major [T U] axis), for spot checks of large
    clips. Returns [len(rows), d_v]."""
    d_k = Q.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d_k)
    rows = np.asarray(list(rows), dtype=np.int64)
    out = np.zeros((len(rows), V.shape[1]))
    frames = rows // U
    for t in np.unique(frames):  # the rows of one frame share their visible keys
        sel = np.nonzero(frames == t)[0]
        keys = np.concatenate([np.arange(f * U, (f + 1) * U) for f in visible_frames(int(t), c, T)])
        logits = (Q[rows[sel]] @ K[keys].T) * scale
        logits = logits - logits.max(axis=1, keepdims=True)
        w = np.exp(logits)
        w = w / w.sum(axis=1, keepdims=True)
        out[sel] = w @ V[keys]
    return out


def softmax_gate(O: np.ndarray, g: np.ndarray) -> np.ndarray:
    """O~S = O^S * sigmoid(g^S), elementwise."""
    return O * (1.0 / (1.0 + np.exp(-g)))


def hybrid_output(Ot_S: np.ndarray, Ot_L: np.ndarray, W_S: np.ndarray, W_L: np.ndarray) -> np.ndarray:
    """Y = O~S W_S + O~L W_L for token-major [N, H, d] branch outputs and
    projections [H d, D_model]; returns [N, D_model]."""
    N = Ot_S.shape[0]
    return Ot_S.reshape(N, -1) @ W_S + Ot_L.reshape(N, -1) @ W_L


def window_softmax_layer(Q: np.ndarray, K: np.ndarray, V: np.ndarray, g: np.ndarray, T: int, U: int,
                         c: int) -> np.ndarray:
    """Gated softmax branch for token-major [B, T U, H, d] inputs (float64)."""
    B, _, H, _ = Q.shape
    out = np.zeros(V.shape)
    for b in range(B):
        for h in range(H):
            out[b, :, h] = window_softmax_head(Q[b, :, h], K[b, :, h], V[b, :, h], T, U, c)
    return softmax_gate(out, g)
