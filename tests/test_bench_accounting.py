"""The algorithmic work bench.py divides by its timings, against hand counts.

Per head: the statistics take 4 d^2 flop per token (two rank-one d x d updates)
over the text and non-anchor frames; the readout 2 d^2 flop per non-anchor
query token. The whole step reads Q, K, V and beta and writes O once on
non-anchor frames, (4 d esz + 4) bytes per head-token, plus the small text,
alpha and anchor terms (a few per cent). The figures below are those counts
evaluated by hand for each workload, rounded to three digits.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from frame_level_delta_b200.inputs import CONFIGS  # noqa: E402

HAND = [
    # workload, statistics flop, readout flop, step bytes
    ("small", 0.612e9, 0.302e9, 19.2e6),
    ("h3", 94.0e9, 46.6e9, 1.47e9),
    ("long", 290e9, 145e9, 4.55e9),
    ("hires", 216e9, 108e9, 4.31e9),
]


@pytest.mark.parametrize("name,gram,readout,step_bytes", HAND, ids=[h[0] for h in HAND])
def test_flops_and_bytes_match_hand_counts(name, gram, readout, step_bytes):
    cfg = CONFIGS[name]
    assert bench.kernel_flops("gram_tc", cfg) == pytest.approx(gram, rel=5e-3)
    assert bench.kernel_flops("readout_tc", cfg) == pytest.approx(readout, rel=5e-3)
    # the hand count leaves out the text, alpha and anchor terms: within 3%
    assert step_bytes <= bench.path_bytes(cfg) <= 1.03 * step_bytes


def test_h3_statistics_bytes_by_parts():
    cfg = CONFIGS["h3"]
    heads, d, U, T, L = 24, 128, 1560, 40, 512
    tokens = (T - 2) * U + L                      # text and non-anchor frames
    reads = tokens * (2 * d * 2 + 4)              # K, V bf16 and beta
    writes = 2 * (T - 1) * d * d * 4              # A and B, fp32, per slot
    assert bench.kernel_bytes("gram_tc", cfg) == heads * (reads + writes)


def test_alu_peak_and_prep_count():
    assert bench.alu_peak_tflops(1965.0) == pytest.approx(74.4, abs=0.05)
    cfg = CONFIGS["hires"]
    F, U, d, H = 38, 3600, 128, 24
    # every input frame's 25-tap spatial sum, amortised over the F outputs, plus 5 temporal taps
    per_value = 25 * 40 / F + 5
    assert bench.kernel_alu_flops("prep_video", cfg) == pytest.approx(H * 2 * F * U * d * 2 * per_value)


def test_attention_pair_count_matches_the_oracles_visible_sets():
    from oracle.hybrid_oracle import visible_frames
    for name, kw in (("h3", {}), ("small", {}), ("small", dict(T=13, chunk=5)), ("small", dict(T=7, chunk=1))):
        cfg = CONFIGS[name].with_(**kw)
        want = sum(len(visible_frames(t, cfg.chunk, cfg.T)) for t in range(cfg.T)) * cfg.U * cfg.U
        assert bench.attention_pairs(cfg) == want
        assert bench.attention_flops(cfg) == 4 * cfg.d * want * cfg.B * cfg.H


def test_split_scan_counts_as_the_frame_scan():
    """The two-CTA scan does the frame scan's work: the same algorithmic bytes
    (one read of each P_t image pair, B_t and alpha_t, the readout states out)
    and flops, and its source is hashed for the traffic table."""
    for name in ("h3", "long", "hires"):
        cfg = CONFIGS[name]
        assert bench.kernel_bytes("scan_split_tc", cfg) == bench.kernel_bytes("scan_tc", cfg) > 0
        assert bench.kernel_flops("scan_split_tc", cfg) == bench.kernel_flops("scan_tc", cfg) > 0
    assert bench.source_digest("scan_split_tc") != bench.source_digest("scan_tc")
