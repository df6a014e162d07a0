"""bench.py's work accounting, checked against independent counts on small
shapes (CPU): allowed query-key pairs by brute force over the token mask,
launch counts from the segment count, readout bytes from the tensor sizes."""
import numpy as np
import pytest

import bench
import oracle as O


@pytest.mark.parametrize("name,n_ctx", [("small", 0), ("ragged", 0), ("768p", 0), ("768p", 4096),
                                        ("small", 77)])
def test_softmax_pairs_match_token_count(name, n_ctx):
    wl, cfg = bench.workload_cfg(name, n_ctx)
    flops, pairs, density = bench.softmax_work(cfg)
    m = O.frame_mask(wl.T, wl.block_frames, wl.window_blocks, wl.anchors).astype(np.int64)
    TN = wl.T * wl.N
    # video x video pairs of the frame mask, then every pair touching a context token
    want = int(m.sum()) * wl.N * wl.N + (wl.L * wl.L - TN * TN)
    assert pairs == want * cfg.B * cfg.H
    assert flops == 2.0 * pairs * (cfg.d + cfg.dv)
    assert density == pytest.approx(m.mean())


def test_launch_count_covers_every_segment():
    for name in ("tiny", "small", "768p", "ragged", "vda_only"):
        _, cfg = bench.workload_cfg(name)
        _, segs = O.window_plan(cfg.T, cfg.block_frames, cfg.window_blocks, cfg.anchors)
        assert bench.softmax_launches(cfg) == -(-len(segs) // 40)
    _, cfg = bench.workload_cfg("small", 64)
    _, segs = O.window_plan(cfg.T, cfg.block_frames, cfg.window_blocks, cfg.anchors)
    assert bench.softmax_launches(cfg) == -(-(len(segs) + 1) // 40)


def test_readout_bytes():
    _, cfg = bench.workload_cfg("768p")
    BH, L = cfg.B * cfg.H, cfg.T * cfg.N
    assert bench.readout_bytes(cfg) == BH * L * 256 * 2 + 2 * BH * cfg.nb * 128 * 128 * 4
