"""The benchmark's work counts on CPU (no GPU): the kept-block FLOPs of the compact
lists equal the oracle's count of the same kept set, and the issued count (the
tensor-core kernel's 128-row x 128-key chunks, pad-only key chunks skipped) equals
a token-by-token enumeration written from the tile geometry."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import block_sparse_video_ssta_b200 as S  # noqa: E402
import oracle  # noqa: E402
import ssta_inputs as si  # noqa: E402


def _random_lists(w, seed):
    g = oracle.geometry(w)
    rng = np.random.default_rng(seed)
    kept = rng.random((w.B, w.H, g.NQ, g.NQ)) < 0.3
    kept[:, :, :, 0] = True
    idx, cnt = oracle.kept_lists(kept)
    return kept, torch.from_numpy(idx), torch.from_numpy(cnt)


def _brute_issued(w, kept):
    g = oracle.geometry(w)
    total = 0
    for b, h, i, j in zip(*np.nonzero(kept)):
        chunks = set()
        for o in range(g.N):
            if j < g.NT:
                cT, cY, cX = j // (g.nY * g.nX), (j // g.nX) % g.nY, j % g.nX
                t = cT * w.tT + o // (w.tY * w.tX)
                y = cY * w.tY + (o // w.tX) % w.tY
                x = cX * w.tX + o % w.tX
                ok = t < w.T and y < w.Y and x < w.X
            else:
                ok = (j - g.NT) * g.N + o < w.L_text
            if ok:
                chunks.add(o // 128)
        total += 4 * w.D * g.N * 128 * len(chunks)
    return float(total)


def test_work_counts_ragged_grid_with_text():
    # 5 frames in tiles of 4: the last tile row holds one valid frame, so the second
    # 128-key chunk (frames 2-3) of those tiles is pure padding; 300 text tokens make a
    # full and a partial (44-token) text tile
    w = si.with_overrides(si.get_workload("small_bf16"), H=2, T=5, Y=12, X=20, L_text=300)
    plan = S.ssta_plan(S.desc_from(w))
    kept, idx, cnt = _random_lists(w, 0)
    padded, valid = bench.kept_flops(w, plan, idx, cnt)
    assert padded == oracle.attention_flops(w, kept)
    assert valid == oracle.attention_flops(w, kept, padded=False)
    issued = bench.issued_flops(w, plan, idx)
    assert issued == _brute_issued(w, kept)
    assert issued < padded


def test_issued_equals_padded_without_pad_chunks():
    w = si.with_overrides(si.get_workload("small_bf16"), H=1, T=8, Y=16, X=16, L_text=256)
    plan = S.ssta_plan(S.desc_from(w))
    kept, idx, cnt = _random_lists(w, 1)
    padded, _ = bench.kept_flops(w, plan, idx, cnt)
    assert bench.issued_flops(w, plan, idx) == padded
