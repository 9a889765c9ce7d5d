"""Shared helpers for the GPU parity tests: run the CUDA path through the
binding, run the CPU oracle on the same generated inputs, and compare.

Inputs come from ssta_inputs only; the oracle never sees a tensor produced by
the CUDA path (it reorders, pools, scores and attends from the raster inputs
itself).  Comparison rules:
* packed tensors, unordered tensors: bit-exact;
* kept-tile lists: identical, except that a tile may differ where the
  oracle's score lies within 1e-4 of the score at the k-th rank of its row;
* O and LSE on valid rows of query tiles whose kept sets agree: max-abs and
  relative-L2 tolerances (fp32: 1e-5; bf16: 2e-2 and 5e-3, LSE 1e-3).
"""
from __future__ import annotations

import numpy as np
import torch

import block_sparse_video_ssta_b200 as S
import oracle
import ssta_inputs as si

BAND = 1e-4
TOL = {"f32": dict(o_max=1e-5, o_rel=1e-5, lse_max=1e-5),
       "bf16": dict(o_max=2e-2, o_rel=5e-3, lse_max=1e-3)}


def to_np(t):
    if t is None:
        return None
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy().astype(np.float64)


def run_gpu(w, inputs, want_scores=True):
    d = S.desc_from(w)
    p = S.ssta_plan(d)
    ts = None
    if want_scores:
        ts = torch.empty((w.B, w.H, p.num_tiles, p.num_tiles), dtype=torch.float32, device=inputs["q"].device)
    r = S.ssta_forward(d, inputs["q"], inputs["k"], inputs["v"], inputs["q_text"], inputs["k_text"],
                       inputs["v_text"], tile_scores=ts)
    torch.cuda.synchronize()
    r["status_mask"] = S.ssta_read_device_status(r["ws_mask"])
    r["status_attn"] = S.ssta_read_device_status(r["ws_attn"])
    r["tile_scores"] = ts
    return r


def oracle_mask(w, q_np, k_np, qt_np, kt_np):
    qp = oracle.tile_reorder(w, q_np, qt_np)
    kp = oracle.tile_reorder(w, k_np, kt_np)
    S64 = oracle.block_scores(w, oracle.tile_pool(w, qp), oracle.tile_pool(w, kp))
    sel = oracle.select_topk(w, S64)
    kept = oracle.kept_mask(w, sel)
    return qp, kp, S64, kept


def kth_scores(w, S64):
    """Score (float64) at rank k-1 of each row, ranks from the float32-rounded scores."""
    g = oracle.geometry(w)
    if g.k == 0:
        return np.full(S64.shape[:-1], np.inf)
    order = np.argsort(-S64.astype(np.float32), axis=-1, kind="stable")
    kth = np.take_along_axis(S64, order[..., g.k - 1: g.k], axis=-1)[..., 0]
    return kth


def gpu_kept(w, kv_idx, kv_cnt):
    g = oracle.geometry(w)
    idx = kv_idx.cpu().numpy()
    cnt = kv_cnt.cpu().numpy()
    kept = np.zeros(cnt.shape + (g.NT + g.n_text,), dtype=bool)
    for pos in np.ndindex(cnt.shape):
        ids = idx[pos][: cnt[pos]]
        assert np.all(np.diff(ids) > 0), f"list not ascending at {pos}"
        assert np.all(idx[pos][cnt[pos]:] == -1), f"padding not -1 at {pos}"
        kept[pos][ids] = True
    return kept


def compare_masks(w, kept_gpu, kept_ref, S64):
    """Returns the boolean [B,H,NQ] of rows whose kept sets agree; asserts that every
    disagreement is inside the 1e-4 band around the k-th score."""
    g = oracle.geometry(w)
    same = np.all(kept_gpu == kept_ref, axis=-1)
    if not same.all():
        kth = kth_scores(w, S64)
        for pos in zip(*np.nonzero(~same)):
            b, h, i = pos
            assert i < g.NT, f"text query tile list differs at {pos}"
            diff = np.nonzero(kept_gpu[pos][: g.NT] != kept_ref[pos][: g.NT])[0]
            assert np.all(kept_gpu[pos][g.NT:] == kept_ref[pos][g.NT:])
            gap = np.abs(S64[b, h, i, diff] - kth[b, h, i])
            assert np.all(gap <= BAND), f"mask differs outside the band at {pos}: tiles {diff}, gaps {gap}"
    return same


def compare_attention(w, O_gpu, lse_gpu, O_ref, lse_ref, rows_mask):
    """Compare on packed rows selected by rows_mask [B,H,Lq] (valid rows of agreeing tiles).
    A row that keeps no key must be O = 0, LSE = -inf on both sides."""
    tol = TOL[w.dtype]
    a = O_gpu[rows_mask]
    b = O_ref[rows_mask]
    assert np.isfinite(a).all()
    err = np.abs(a - b)
    max_abs = float(err.max()) if err.size else 0.0
    rel = float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))
    la, lb = lse_gpu[rows_mask], lse_ref[rows_mask]
    empty = np.isneginf(la) & np.isneginf(lb)                 # rows with no kept key on both sides
    lse_err = float(np.abs(np.where(empty, 0.0, la) - np.where(empty, 0.0, lb)).max()) if err.size else 0.0
    assert max_abs <= tol["o_max"], f"O max-abs {max_abs} > {tol['o_max']}"
    assert rel <= tol["o_rel"], f"O rel-L2 {rel} > {tol['o_rel']}"
    assert lse_err <= tol["lse_max"], f"LSE max-abs {lse_err} > {tol['lse_max']}"
    return max_abs, rel, lse_err


def full_check(w, seed=0, device="cuda", q_tiles=None, heads=None):
    """Run the whole chain on the GPU and check every stage against the oracle.

    ``q_tiles``: query tiles whose O/LSE are compared (default all);
    ``heads``: heads compared (default all).  Masks are always compared on the
    selected heads over all tiles.
    """
    x = si.make_inputs(w, seed, device=device)
    r = run_gpu(w, x)
    assert r["status_mask"] == 0 and r["status_attn"] == 0
    heads = list(range(w.H)) if heads is None else list(heads)
    g = oracle.geometry(w)
    stats = {}
    hsel = torch.tensor(heads, device=x["q"].device)
    sub = lambda t: None if t is None else t.index_select(1, hsel)
    q_np, k_np, v_np = (to_np(sub(x[n])) for n in ("q", "k", "v"))
    qt_np, kt_np, vt_np = (to_np(sub(x[n])) for n in ("q_text", "k_text", "v_text"))
    qp, kp, S64, kept_ref = oracle_mask(w, q_np, k_np, qt_np, kt_np)
    vp = oracle.tile_reorder(w, v_np, vt_np)
    # Step 1: packed tensors bit-exact
    np.testing.assert_array_equal(to_np(sub(r["qp"])), qp)
    np.testing.assert_array_equal(to_np(sub(r["kp"])), kp)
    np.testing.assert_array_equal(to_np(sub(r["vp"])), vp)
    # Step 2 scores (float32 vs float64)
    ts = to_np(sub(r["tile_scores"]))
    stats["score_max_abs_err"] = float(np.abs(ts - S64).max())
    # Steps 2-4 masks
    kept_gpu = gpu_kept(w, sub(r["kv_idx"]), sub(r["kv_cnt"]))
    same = compare_masks(w, kept_gpu, kept_ref, S64)
    stats["rows_mask_mismatch"] = int((~same).sum())
    # Step 4 attention on agreeing, requested tiles
    tiles = list(range(g.NQ)) if q_tiles is None else list(q_tiles)
    O_ref, lse_ref = oracle.attention(w, qp, kp, vp, kept_ref, q_tiles=tiles, scale=getattr(w, "scale", None))
    valid = oracle.valid_token_mask(w)
    rows = np.zeros((w.B, len(heads), g.Lq), dtype=bool)
    for i in tiles:
        r0, r1 = i * g.N, min((i + 1) * g.N, g.Lq)
        rows[:, :, r0:r1] = same[:, :, i, None] & valid[None, None, r0:r1]
    O_gpu = to_np(sub(r["O_packed"]))
    lse_gpu = to_np(sub(r["LSE"]))
    stats["o_max_abs"], stats["o_rel_l2"], stats["lse_max_abs"] = compare_attention(
        w, O_gpu, lse_gpu, O_ref, lse_ref, rows)
    # unorder: the GPU's raster O against the oracle's own O put back in raster order
    rows_t = np.where(rows, 0.0, np.nan)[..., None]
    O_r, O_t = oracle.tile_unorder(w, O_ref + rows_t)
    got = to_np(sub(r["O"]))
    m = np.isfinite(O_r)
    assert np.abs(got[m] - O_r[m]).max(initial=0.0) <= TOL[w.dtype]["o_max"]
    if w.L_text:
        mt = np.isfinite(O_t)
        assert np.abs(to_np(sub(r["O_text"]))[mt] - O_t[mt]).max(initial=0.0) <= TOL[w.dtype]["o_max"]
    stats["rows_compared"] = int(rows.sum())
    return stats
