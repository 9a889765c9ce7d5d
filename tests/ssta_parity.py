"""Shared helpers for the GPU parity tests: run the CUDA path through the
binding, run the CPU oracle on the same generated inputs, and compare.

Inputs come from ssta_inputs only; the oracle never sees a tensor produced by
the CUDA path (it reorders, pools, scores and attends from the raster inputs
itself).  Comparison rules:
* packed tensors: bit-exact against the oracle's packing of the raster inputs;
* block scores (the ``tile_scores`` output): within the fp32 rounding bound of
  ``score_bound`` (pooling and dot products in float32 against float64);
* kept-tile lists: identical, except that a tile may differ where the
  oracle's score lies within 1e-4 of the score at the k-th rank of its row;
* O and LSE on valid rows: max-abs and relative-L2 tolerances (fp32: 1e-5;
  bf16: 2e-2 and 5e-3, LSE 1e-3) against the oracle's attention over the
  oracle's kept set; on a row whose set differs inside the score band (both
  choices are right up to rounding) the oracle attends over the GPU's set for
  that row instead, so the output of the choice the GPU made is still checked;
* unorder: the GPU's raster O is bit-exact against the oracle's unorder of
  the GPU's packed O (a pure copy), and within the O tolerance of the
  oracle's own O.
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


def oracle_mask(w, q_np, k_np, qt_np, kt_np, with_means=False):
    qp = oracle.tile_reorder(w, q_np, qt_np)
    kp = oracle.tile_reorder(w, k_np, kt_np)
    qbar, kbar = oracle.tile_pool(w, qp), oracle.tile_pool(w, kp)
    S64 = oracle.block_scores(w, qbar, kbar)
    sel = oracle.select_topk(w, S64)
    kept = oracle.kept_mask(w, sel)
    if with_means:
        return qp, kp, S64, kept, qbar, kbar
    return qp, kp, S64, kept


U32 = 2.0 ** -24   # unit roundoff of float32


def score_bound(w, qp, kp, qbar, kbar):
    """Per-element bound [B,H,NT,NT] on |float32 score - float64 score|.

    Rounding model: a float32 sum of n terms is off by about sqrt(n)*u times
    the terms' scale (u = 2^-24; the statistical form of the n*u worst case,
    Higham, "Accuracy and Stability of Numerical Algorithms", section 2.8),
    taken here with a safety factor of 4.  So a tile mean is off by at most
    4*sqrt(N)*u times the mean absolute token value plus 2u of itself, and the
    dot product over D channels adds 4*sqrt(D)*u times the sum of absolute
    products; the similarity bound propagates both to first order, times 2.
    The importance score is built from cosines: their bound divides the dot
    bound by the norms and adds the norms' own relative error; the score's
    bound is lam/2 times that plus (1 - lam)/2 times the largest key-key cosine
    bound, times 2, plus 1e-7.

    The result is capped at BAND / 2: a score error e can flip a tile only if
    its score lies within 2e of the k-th score, so the mask band of 1e-4 only
    covers every flip when e <= BAND / 2.
    """
    g = oracle.geometry(w)
    aq = oracle.tile_pool(w, np.abs(qp))            # mean |token| per tile and channel
    ak = oracle.tile_pool(w, np.abs(kp))
    eq = 4 * np.sqrt(g.N) * U32 * aq + 2 * U32 * np.abs(qbar)    # bound on each pooled channel
    ek = 4 * np.sqrt(g.N) * U32 * ak + 2 * U32 * np.abs(kbar)

    def dot_bound(ea, a, eb, b):
        A, Bv = np.abs(a), np.abs(b)
        return (np.einsum("bhid,bhjd->bhij", ea, Bv) + np.einsum("bhid,bhjd->bhij", A, eb)
                + np.einsum("bhid,bhjd->bhij", ea, eb) + 4 * np.sqrt(g.D) * U32 * np.einsum("bhid,bhjd->bhij", A, Bv))

    e_qk = dot_bound(eq, qbar, ek, kbar)
    if getattr(w, "score_mode", "similarity") != "importance":
        return np.minimum(2.0 * e_qk + 1e-7, BAND / 2)

    def cos_bound(e_dot, a, ea, b, eb):
        na = np.linalg.norm(a, axis=-1)
        nb = np.linalg.norm(b, axis=-1)
        rel_a = np.linalg.norm(ea, axis=-1) / np.maximum(na, 1e-30) + 4 * np.sqrt(g.D) * U32
        rel_b = np.linalg.norm(eb, axis=-1) / np.maximum(nb, 1e-30) + 4 * np.sqrt(g.D) * U32
        return e_dot / np.maximum(na[..., :, None] * nb[..., None, :], 1e-30) + rel_a[..., :, None] + rel_b[..., None, :]

    lam = float(getattr(w, "lam", 0.9))
    c_qk = cos_bound(e_qk, qbar, eq, kbar, ek)
    c_kk = cos_bound(dot_bound(ek, kbar, ek, kbar), kbar, ek, kbar, ek)
    red = c_kk.max(axis=-2)                          # the mean of bounded terms is within their max
    return np.minimum(2.0 * (lam / 2.0 * c_qk + (1.0 - lam) / 2.0 * red[..., None, :]) + 1e-7, BAND / 2)


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


def full_check(w, seed=0, device="cuda", q_tiles=None, heads=None, gen_device=None):
    """Run the whole chain on the GPU and check every stage against the oracle.

    ``q_tiles``: query tiles whose O/LSE are compared (default all);
    ``heads``: heads compared (default all).  Masks and scores are always
    compared on the selected heads over all tiles.  ``gen_device``: where the
    inputs are generated (default ``device``); they are copied to ``device``.
    """
    x = si.make_inputs(w, seed, device=gen_device or device)
    if gen_device is not None and gen_device != device:
        x = {k: (None if t is None else t.to(device)) for k, t in x.items()}
    r = run_gpu(w, x)
    assert r["status_mask"] == 0 and r["status_attn"] == 0
    heads = list(range(w.H)) if heads is None else list(heads)
    g = oracle.geometry(w)
    stats = {}
    hsel = torch.tensor(heads, device=x["q"].device)
    sub = lambda t: None if t is None else t.index_select(1, hsel)
    q_np, k_np, v_np = (to_np(sub(x[n])) for n in ("q", "k", "v"))
    qt_np, kt_np, vt_np = (to_np(sub(x[n])) for n in ("q_text", "k_text", "v_text"))
    qp, kp, S64, kept_ref, qbar, kbar = oracle_mask(w, q_np, k_np, qt_np, kt_np, with_means=True)
    vp = oracle.tile_reorder(w, v_np, vt_np)
    # Step 1: packed tensors bit-exact
    np.testing.assert_array_equal(to_np(sub(r["qp"])), qp)
    np.testing.assert_array_equal(to_np(sub(r["kp"])), kp)
    np.testing.assert_array_equal(to_np(sub(r["vp"])), vp)
    # Step 2 scores (float32 on the GPU vs float64), every element within its rounding bound
    ts = to_np(sub(r["tile_scores"]))
    err = np.abs(ts - S64)
    bound = score_bound(w, qp, kp, qbar, kbar)
    worst = np.unravel_index(np.argmax(err / bound), err.shape)
    assert np.all(err <= bound), f"score error {err[worst]} > bound {bound[worst]} at {worst}"
    stats["score_max_abs_err"] = float(err.max())
    stats["score_err_over_bound"] = float((err / bound).max())
    # Steps 2-4 masks
    kept_gpu = gpu_kept(w, sub(r["kv_idx"]), sub(r["kv_cnt"]))
    same = compare_masks(w, kept_gpu, kept_ref, S64)
    stats["rows_mask_mismatch"] = int((~same).sum())
    # Step 4 attention on the requested tiles: the oracle's kept set, except on rows whose
    # set differs inside the score band, where the oracle attends over the GPU's choice
    kept_eval = kept_ref.copy()
    kept_eval[~same] = kept_gpu[~same]
    tiles = list(range(g.NQ)) if q_tiles is None else list(q_tiles)
    O_ref, lse_ref = oracle.attention(w, qp, kp, vp, kept_eval, q_tiles=tiles, scale=getattr(w, "scale", None))
    valid = oracle.valid_token_mask(w)
    rows = np.zeros((w.B, len(heads), g.Lq), dtype=bool)
    for i in tiles:
        r0, r1 = i * g.N, min((i + 1) * g.N, g.Lq)
        rows[:, :, r0:r1] = valid[None, None, r0:r1]
    O_gpu = to_np(sub(r["O_packed"]))
    lse_gpu = to_np(sub(r["LSE"]))
    stats["o_max_abs"], stats["o_rel_l2"], stats["lse_max_abs"] = compare_attention(
        w, O_gpu, lse_gpu, O_ref, lse_ref, rows)
    # unorder: a pure copy, bit-exact against the oracle's unorder of the GPU's packed O ...
    O_r_copy, O_t_copy = oracle.tile_unorder(w, O_gpu)
    got = to_np(sub(r["O"]))
    np.testing.assert_array_equal(got, O_r_copy)
    if w.L_text:
        np.testing.assert_array_equal(to_np(sub(r["O_text"])), O_t_copy)
    # ... and within the O tolerance of the oracle's own O put back in raster order
    rows_t = np.where(rows, 0.0, np.nan)[..., None]
    O_r, O_t = oracle.tile_unorder(w, O_ref + rows_t)
    m = np.isfinite(O_r)
    assert np.abs(got[m] - O_r[m]).max(initial=0.0) <= TOL[w.dtype]["o_max"]
    if w.L_text:
        mt = np.isfinite(O_t)
        assert np.abs(to_np(sub(r["O_text"]))[mt] - O_t[mt]).max(initial=0.0) <= TOL[w.dtype]["o_max"]
    stats["rows_compared"] = int(rows.sum())
    stats["rows_on_gpu_choice"] = int(sum(((~same)[:, :, i, None] & rows[:, :, i * g.N:(i + 1) * g.N]).sum()
                                          for i in tiles))
    return stats


def mask_check(w, seed, heads, device="cuda"):
    """Steps 1-3 only (packing, scores, lists) on the selected heads, every mask row."""
    x = si.make_inputs(w, seed, device=device)
    d = S.desc_from(w)
    p = S.ssta_plan(d)
    ts = torch.empty((w.B, w.H, p.num_tiles, p.num_tiles), dtype=torch.float32, device=device)
    qp = S.ssta_tile_reorder(d, x["q"], x["q_text"])
    kp = S.ssta_tile_reorder(d, x["k"], x["k_text"])
    kv_idx, kv_cnt, ws = S.ssta_build_block_mask(d, qp, kp, tile_scores=ts)
    torch.cuda.synchronize()
    assert S.ssta_read_device_status(ws) == 0
    hsel = torch.tensor(list(heads), device=device)
    sub = lambda t: None if t is None else t.index_select(1, hsel)
    q_np, k_np, qt_np, kt_np = (to_np(sub(x[n])) for n in ("q", "k", "q_text", "k_text"))
    qp_ref, kp_ref, S64, kept_ref, qbar, kbar = oracle_mask(w, q_np, k_np, qt_np, kt_np, with_means=True)
    np.testing.assert_array_equal(to_np(sub(qp)), qp_ref)
    np.testing.assert_array_equal(to_np(sub(kp)), kp_ref)
    err = np.abs(to_np(sub(ts)) - S64)
    bound = score_bound(w, qp_ref, kp_ref, qbar, kbar)
    assert np.all(err <= bound), f"score error over its bound: {(err / bound).max()}"
    kept_gpu = gpu_kept(w, sub(kv_idx), sub(kv_cnt))
    same = compare_masks(w, kept_gpu, kept_ref, S64)
    return {"rows_mask_mismatch": int((~same).sum()), "rows": int(same.size),
            "score_max_abs_err": float(err.max()), "score_err_over_bound": float((err / bound).max())}
