"""The bench's algorithmic work model (the numerators of its roofline
fractions) against the oracle's mask and the workloads' stated sizes."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from oracle import vdn_oracle as O  # noqa: E402
from synth import CONFIGS  # noqa: E402


@pytest.mark.parametrize("T,C,R", [(1, 5, 1), (2, 5, 1), (13, 5, 1), (15, 5, 1), (15, 15, 1),
                                   (20, 5, 1), (40, 5, 1), (42, 5, 2), (75, 5, 1), (7, 3, 0)])
def test_visible_frames_count_the_oracle_mask(T, C, R):
    """Frame pairs the bench counts = true entries of the oracle's frame mask."""
    want = int(O.frame_mask(T, C, R).sum())
    assert sum(bench.visible_frames(t, T, C, R) for t in range(T)) == want


@pytest.mark.parametrize("name,frame_pairs,pairs", [
    ("tiny_f32", 193, 9.9e4),
    ("small_bf16", 668, 3.50e8),
    ("768p_bf16", 1333, 7.55e10),
    ("long_bf16", 5608, 3.18e11),
    ("batched_bf16", 288, 2.45e10),
])
def test_work_model_matches_the_workload_sizes(name, frame_pairs, pairs):
    """Frame pairs and masked (query, key) pairs of each workload (B H N^2 per
    visible frame pair), to the three digits they are quoted with."""
    wm = bench.work_model(CONFIGS[name])
    assert wm["frame_pairs"] == frame_pairs
    assert abs(wm["pairs"] / pairs - 1) < 6e-3


def test_work_model_flops_and_bytes_at_768p():
    """4 d FLOPs per visible pair (Q K^T and P V), the projection GEMM
    2 (B L)(2D) D, and the minimum bytes: q, k, v, two gates in bf16, an f32
    output, both W and the text keys and values."""
    cfg = CONFIGS["768p_bf16"]
    wm = bench.work_model(cfg)
    L, D = cfg.T * cfg.N, cfg.H * cfg.d
    assert wm["f_soft"] == 4 * cfg.d * wm["pairs"]
    assert wm["f_proj"] == 2 * cfg.B * L * 2 * D * D
    assert abs(wm["f_soft"] / 3.8645e13 - 1) < 1e-3
    assert abs(wm["f_proj"] / 4.35e12 - 1) < 1e-3
    assert 3.0e11 < wm["f_vda"] < 5.0e11
    assert abs(wm["bytes_min"] / 4.9986e9 - 1) < 1e-3
    # text keys in every video query's normaliser add B H L n_text pairs
    wt = bench.work_model(cfg, text_keys=True)
    assert wt["pairs"] - wm["pairs"] == cfg.B * cfg.H * L * cfg.n_text
