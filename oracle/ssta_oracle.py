"""CPU oracle for Selective and Sliding Tile Attention (SSTA), forward pass.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call
this module: only the tests, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg use it.  It shares no code with the CUDA library.

Plain, slow and direct: numpy in float64, every step written out in the order
the method states it.  Sources (page titles; sections / equations named):

* "HunyuanVideo 1.5 Technical Report" (paper-graph-ui summary), section
  "SSTA: Selective and Sliding Tile Attention":
    - the attention equation softmax(Q K^T / sqrt(d_k)) V;
    - Step 1 "3D Block Partition" (tiles of N = tile_t*tile_h*tile_w tokens,
      B = (F/tile_t)(H/tile_h)(W/tile_w) blocks, full attention inside a
      kept block);
    - Step 2 "Selective Mask Generation" (Score_s = pooled-Q . pooled-K^T,
      Topk, Indexes2mask, per-head masks);
    - Step 3 "STA (Sliding Tile Attention) Mask Generation" (window
      WS = (w_t, w_h, w_w) in tiles);
    - Step 4 "Combine Masks and Block-Sparse Attention" (the text itself
      doubts the AND of Algorithm 1 and points to a union; the union is used).
* "HunyuanVideo-1.5: An 8.3B-Parameter Video Diffusion Model Built for
  Consumer GPUs" (apoapsis blog), "Under the Hood: SSTA and Muon in Detail":
  top-k is clamped to the number of key blocks; for the importance score it
  fixes the constants of the report's Step 2 equation: lambda = 0.9 and
  beta = 1 - lambda, cosines of the pooled vectors mapped by (x + 1) / 2, a
  key tile not compared with itself in the redundancy.

Modes (descriptor fields, defaults first): ``score_mode`` "similarity" (raw
pooled dot product) or "importance" (Step 2's similarity-minus-redundancy
score in the blog's normalised form, weight ``lam``); ``combine`` "union" or
"and" (Algorithm 1's literal M_sel AND M_sta); ``window_mode`` "shift" (the
window slides inward at grid edges) or "truncate" (the window is cut at the
edges, the plain reading of "within +-w/2").

Readings where the pages leave a step open (each also listed in the design
notes): by default, similarity scores are the raw dot product of per-tile means
of q and k over the tile's valid tokens (no normalisation, no redundancy term);
in importance mode an all-zero pooled vector stays zero when normalised and a
grid of one tile has redundancy 0; the top-k decision is taken on the scores rounded to float32 with ties going to
the lower tile index; by default the window slides inward at grid edges so it
always keeps min(w, n) tiles per axis, and selection and window are united; an
optional
text segment is appended after the video tiles, attended densely by every
query and whose queries attend every valid key; pad tokens (grid rounded up to
whole tiles) are never attended; LSE is the natural-log sum of exponentials of
the scaled scores of a row.

Parity status: every function here is pinned by the CPU tests (closed forms,
brute force on tiny grids, equivalence with a library attention routine in
special cases); see tests/test_oracle_pins.py.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

__all__ = [
    "Geometry", "geometry", "valid_token_mask", "tile_reorder", "tile_unorder",
    "tile_pool", "tile_scores", "importance_scores", "block_scores", "select_topk", "window_mask", "kept_mask",
    "kept_lists", "attention", "attention_bwd", "ssta_forward", "attention_flops",
]


@dataclass(frozen=True)
class Geometry:
    B: int
    H: int
    D: int
    T: int
    Y: int
    X: int
    tT: int
    tY: int
    tX: int
    nT: int          # tiles per axis after rounding the grid up to whole tiles
    nY: int
    nX: int
    N: int           # tokens per tile
    NT: int          # video tiles
    L_text: int
    n_text: int      # text tiles (ceil(L_text / N))
    NQ: int          # query tiles = NT + n_text
    Lq: int          # packed sequence length = NT*N + L_text
    k: int           # top-k clamped to NT


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def geometry(d) -> Geometry:
    """Step 1 (3D Block Partition): tile counts after padding each axis up to a tile multiple."""
    nT, nY, nX = _ceil_div(d.T, d.tT), _ceil_div(d.Y, d.tY), _ceil_div(d.X, d.tX)
    N = d.tT * d.tY * d.tX
    NT = nT * nY * nX
    n_text = _ceil_div(d.L_text, N) if d.L_text > 0 else 0
    return Geometry(d.B, d.H, d.D, d.T, d.Y, d.X, d.tT, d.tY, d.tX, nT, nY, nX, N, NT,
                    d.L_text, n_text, NT + n_text, NT * N + d.L_text, min(max(d.topk, 0), NT))


def valid_token_mask(d) -> np.ndarray:
    """bool[Lq]: True for packed rows that hold a real (non-pad) token."""
    g = geometry(d)
    grid = np.zeros((g.nT * g.tT, g.nY * g.tY, g.nX * g.tX), dtype=bool)
    grid[: g.T, : g.Y, : g.X] = True
    video = _to_tiles(grid[..., None], g)[..., 0].reshape(g.NT * g.N)
    return np.concatenate([video, np.ones(g.L_text, dtype=bool)])


def _to_tiles(x: np.ndarray, g: Geometry) -> np.ndarray:
    """[..., T', Y', X', C] (padded grid) -> [..., NT, N, C] tile-major, raster inside a tile."""
    lead = x.shape[:-4]
    C = x.shape[-1]
    x = x.reshape(*lead, g.nT, g.tT, g.nY, g.tY, g.nX, g.tX, C)
    nl = len(lead)
    perm = list(range(nl)) + [nl + 0, nl + 2, nl + 4, nl + 1, nl + 3, nl + 5, nl + 6]
    return x.transpose(perm).reshape(*lead, g.NT, g.N, C)


def _from_tiles(x: np.ndarray, g: Geometry) -> np.ndarray:
    """Inverse of _to_tiles: [..., NT, N, C] -> [..., T', Y', X', C]."""
    lead = x.shape[:-3]
    C = x.shape[-1]
    x = x.reshape(*lead, g.nT, g.nY, g.nX, g.tT, g.tY, g.tX, C)
    nl = len(lead)
    perm = list(range(nl)) + [nl + 0, nl + 3, nl + 1, nl + 4, nl + 2, nl + 5, nl + 6]
    return x.transpose(perm).reshape(*lead, g.nT * g.tT, g.nY * g.tY, g.nX * g.tX, C)


def tile_reorder(d, x_raster: np.ndarray, x_text: np.ndarray | None) -> np.ndarray:
    """Step 1: raster [B,H,T,Y,X,D] (+ text [B,H,L_text,D]) -> packed [B,H,Lq,D].

    Tile c = (cT*nY + cY)*nX + cX holds packed rows c*N .. c*N+N-1, tokens in
    raster order inside the tile; pad tokens are zero; text rows follow the
    video tiles in their given order.  Exact copy (dtype preserved).
    """
    g = geometry(d)
    B, H = x_raster.shape[:2]
    padded = np.zeros((B, H, g.nT * g.tT, g.nY * g.tY, g.nX * g.tX, g.D), dtype=x_raster.dtype)
    padded[:, :, : g.T, : g.Y, : g.X] = x_raster
    video = _to_tiles(padded, g).reshape(B, H, g.NT * g.N, g.D)
    if g.L_text > 0:
        return np.concatenate([video, x_text], axis=2)
    return video


def tile_unorder(d, x_packed: np.ndarray):
    """Inverse of tile_reorder: packed [B,H,Lq,D] -> (raster [B,H,T,Y,X,D], text or None)."""
    g = geometry(d)
    B, H, C = x_packed.shape[0], x_packed.shape[1], x_packed.shape[-1]
    video = x_packed[:, :, : g.NT * g.N].reshape(B, H, g.NT, g.N, C)
    grid = _from_tiles(video, g)[:, :, : g.T, : g.Y, : g.X]
    text = x_packed[:, :, g.NT * g.N:] if g.L_text > 0 else None
    return np.ascontiguousarray(grid), (np.ascontiguousarray(text) if text is not None else None)


def tile_pool(d, x_packed: np.ndarray) -> np.ndarray:
    """Step 2, pooled representation: mean of each video tile over its valid tokens.

    Returns float64 [B,H,NT,D].
    """
    g = geometry(d)
    B, H = x_packed.shape[:2]
    valid = valid_token_mask(d)[: g.NT * g.N].reshape(g.NT, g.N)
    x = x_packed[:, :, : g.NT * g.N].astype(np.float64).reshape(B, H, g.NT, g.N, g.D)
    total = np.where(valid[None, None, :, :, None], x, 0.0).sum(axis=3)
    count = valid.sum(axis=1).astype(np.float64)
    return total / count[None, None, :, None]


def tile_scores(d, qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """Step 2, block similarity Score_s = Qbar Kbar^T per (batch, head): float64 [B,H,NT,NT]."""
    return np.einsum("bhid,bhjd->bhij", qbar, kbar)


def _unit(x: np.ndarray) -> np.ndarray:
    """Rows of x scaled to unit L2 length over the last axis; an all-zero row stays zero."""
    n = np.sqrt((x * x).sum(axis=-1, keepdims=True))
    return np.where(n > 0, x / np.where(n > 0, n, 1.0), 0.0)


def importance_scores(d, qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """Step 2 with the redundancy term ("Selective Mask Generation"): the block
    score Score_i = lam * Score_s - beta * Score_r, per (batch, head), with
    beta = 1 - lam and lam = 0.9 by default (the weights the blog fixes).

    * Score_s[i, j]: similarity of query tile i and key tile j, the cosine of
      their pooled vectors mapped from [-1, 1] to [0, 1] by (x + 1) / 2;
    * Score_r[j]: redundancy of key tile j, the average of the same mapped
      cosine between key tile j and each OTHER key tile (a tile is not
      compared with itself; with a single key tile there is no other tile and
      Score_r = 0).

    A pooled vector of length zero has cosine 0 with everything (its unit
    vector is taken as zero).  float64 [B,H,NT,NT]."""
    lam = float(getattr(d, "lam", 0.9))
    beta = 1.0 - lam
    B, H, NTq, NTk = qbar.shape[0], qbar.shape[1], qbar.shape[2], kbar.shape[2]
    out = np.empty((B, H, NTq, NTk))
    for b in range(B):
        for h in range(H):
            qn, kn = _unit(qbar[b, h]), _unit(kbar[b, h])
            score_s = (qn @ kn.T + 1.0) / 2.0                     # [query tile, key tile]
            score_r = np.zeros(NTk)
            for j in range(NTk):
                if NTk == 1:
                    break
                to_all = (kn @ kn[j] + 1.0) / 2.0                # key tile j against every key tile
                score_r[j] = np.delete(to_all, j).mean()          # ... the other ones only
            out[b, h] = lam * score_s - beta * score_r[None, :]
    return out


def block_scores(d, qbar: np.ndarray, kbar: np.ndarray) -> np.ndarray:
    """The block score that Topk ranks, per the descriptor's ``score_mode``."""
    if getattr(d, "score_mode", "similarity") == "importance":
        return importance_scores(d, qbar, kbar)
    return tile_scores(d, qbar, kbar)


def select_topk(d, scores: np.ndarray) -> np.ndarray:
    """Step 2, Topk + Indexes2mask: bool [B,H,NT,NT], True where key tile j is selected for query tile i.

    k = min(topk, NT).  The decision uses the scores rounded to float32; the
    order is descending score, equal scores ordered by ascending tile index
    (a stable sort of the negated scores).
    """
    g = geometry(d)
    s32 = scores.astype(np.float32)
    order = np.argsort(-s32, axis=-1, kind="stable")
    sel = np.zeros(scores.shape, dtype=bool)
    np.put_along_axis(sel, order[..., : g.k], True, axis=-1)
    return sel


def _axis_window(n: int, w: int, truncate: bool = False) -> np.ndarray:
    """bool[n, n]: per-axis window membership.  The window of tile c covers
    [c - w//2, c - w//2 + w); "shift" slides it inward at the edges so it keeps
    min(w, n) tiles, "truncate" cuts it at 0 and n."""
    m = np.zeros((n, n), dtype=bool)
    span = min(w, n)
    for c in range(n):
        if truncate:
            lo = c - w // 2
            m[c, max(lo, 0): min(lo + w, n)] = True
        else:
            start = min(max(c - w // 2, 0), n - span)
            m[c, start: start + span] = True
    return m


def window_mask(d) -> np.ndarray:
    """Step 3, M_sta: bool [NT, NT] (head-agnostic), product of the three per-axis windows."""
    g = geometry(d)
    tr = getattr(d, "window_mode", "shift") == "truncate"
    mt, my, mx = _axis_window(g.nT, d.wT, tr), _axis_window(g.nY, d.wY, tr), _axis_window(g.nX, d.wX, tr)
    m = mt[:, None, None, :, None, None] & my[None, :, None, None, :, None] & mx[None, None, :, None, None, :]
    return m.reshape(g.NT, g.NT)


def kept_mask(d, sel: np.ndarray) -> np.ndarray:
    """Step 4, combined mask: bool [B,H,NQ,NT+n_text].

    Video query tiles keep (selected | window), or (selected & window) with
    ``combine`` = "and", plus every text tile; text query tiles keep every tile.
    """
    g = geometry(d)
    B, H = sel.shape[:2]
    kept = np.zeros((B, H, g.NQ, g.NT + g.n_text), dtype=bool)
    win = window_mask(d)[None, None]
    kept[:, :, : g.NT, : g.NT] = (sel & win) if getattr(d, "combine", "union") == "and" else (sel | win)
    kept[:, :, : g.NT, g.NT:] = True
    kept[:, :, g.NT:, :] = True
    return kept


def kept_lists(kept: np.ndarray):
    """Compact form of the mask: ascending kept tile ids per query tile.

    Returns (idx int32 [B,H,NQ,W] padded with -1, cnt int32 [B,H,NQ]) with W
    the largest count.
    """
    cnt = kept.sum(axis=-1).astype(np.int32)
    W = int(cnt.max()) if cnt.size else 0
    idx = np.full(kept.shape[:-1] + (W,), -1, dtype=np.int32)
    for pos in np.ndindex(kept.shape[:-1]):
        ids = np.nonzero(kept[pos])[0]
        idx[pos][: len(ids)] = ids
    return idx, cnt


def attention(d, qp: np.ndarray, kp: np.ndarray, vp: np.ndarray, kept: np.ndarray,
              q_tiles=None, scale: float | None = None):
    """Step 4, block-sparse attention on the packed layout, in float64.

    For every query row of query tile i: scores s_j = (q . k_j) * scale over
    the valid keys j of the kept tiles of i (full attention inside each kept
    tile), LSE = log sum_j exp(s_j), O = sum_j exp(s_j - LSE) v_j.  Returns
    (O [B,H,Lq,D], LSE [B,H,Lq]); rows of tiles not in ``q_tiles`` (default:
    all) are NaN.  A query tile with no kept valid key (possible with
    ``combine`` = "and" and no text) gets O = 0 and LSE = -inf (the sum over an
    empty set).
    """
    g = geometry(d)
    scale = 1.0 / math.sqrt(g.D) if not scale else scale
    B, H = qp.shape[:2]
    valid = valid_token_mask(d)
    O = np.full((B, H, g.Lq, g.D), np.nan)
    LSE = np.full((B, H, g.Lq), np.nan)
    tiles = range(g.NQ) if q_tiles is None else q_tiles
    for b in range(B):
        for h in range(H):
            q = qp[b, h].astype(np.float64)
            k = kp[b, h].astype(np.float64)
            v = vp[b, h].astype(np.float64)
            for i in tiles:
                r0, r1 = i * g.N, min((i + 1) * g.N, g.Lq)
                rows = []
                for j in np.nonzero(kept[b, h, i])[0]:
                    c0, c1 = j * g.N, min((j + 1) * g.N, g.Lq)
                    rows.append(np.arange(c0, c1)[valid[c0:c1]])
                keys = np.concatenate(rows) if rows else np.zeros(0, dtype=np.int64)
                if keys.size == 0:
                    O[b, h, r0:r1] = 0.0
                    LSE[b, h, r0:r1] = -np.inf
                    continue
                s = (q[r0:r1] @ k[keys].T) * scale
                m = s.max(axis=1, keepdims=True)
                lse = m[:, 0] + np.log(np.exp(s - m).sum(axis=1))
                p = np.exp(s - lse[:, None])
                O[b, h, r0:r1] = p @ v[keys]
                LSE[b, h, r0:r1] = lse
    return O, LSE


def attention_bwd(d, qp: np.ndarray, kp: np.ndarray, vp: np.ndarray, dOp: np.ndarray, kept: np.ndarray,
                  scale: float | None = None, q_tiles=None, key_tiles=None):
    """Gradients of Step 4's block-sparse attention, in float64: for every valid
    query row of query tile i and the valid keys of its kept tiles, with
    P = softmax(q k^T * scale) (recomputed), O = P v, D = rowsum(dO * O):
    dS = P * (dO v^T - D), dQ = scale * dS k, dK += scale * dS^T q, dV += P^T dO.
    Pad query rows take no part (their dQ is 0); pad keys get dK = dV = 0; a query
    tile with no kept key contributes nothing.  Returns (dQ, dK, dV), each
    [B,H,Lq,D] on the packed layout.

    ``q_tiles`` / ``key_tiles`` (default: all) restrict the result to the dQ rows
    of those query tiles and the dK, dV rows of those key tiles: only the query
    tiles in ``q_tiles`` or keeping one of ``key_tiles`` are visited, and every
    other row is NaN."""
    g = geometry(d)
    scale = 1.0 / math.sqrt(g.D) if not scale else scale
    B, H = qp.shape[:2]
    valid = valid_token_mask(d)
    dQ = np.zeros((B, H, g.Lq, g.D))
    dK = np.zeros((B, H, g.Lq, g.D))
    dV = np.zeros((B, H, g.Lq, g.D))
    qsel = np.ones(g.NQ, dtype=bool) if q_tiles is None else np.isin(np.arange(g.NQ), q_tiles)
    ksel = np.ones(g.NQ, dtype=bool) if key_tiles is None else np.isin(np.arange(g.NQ), key_tiles)
    for b in range(B):
        for h in range(H):
            q = qp[b, h].astype(np.float64)
            k = kp[b, h].astype(np.float64)
            v = vp[b, h].astype(np.float64)
            do = dOp[b, h].astype(np.float64)
            for i in range(g.NQ):
                if not (qsel[i] or (kept[b, h, i] & ksel).any()):
                    continue
                r0, r1 = i * g.N, min((i + 1) * g.N, g.Lq)
                rows = np.arange(r0, r1)[valid[r0:r1]]
                cols = [np.arange(j * g.N, min((j + 1) * g.N, g.Lq)) for j in np.nonzero(kept[b, h, i])[0]]
                keys = np.concatenate([c[valid[c]] for c in cols]) if cols else np.zeros(0, dtype=np.int64)
                if keys.size == 0 or rows.size == 0:
                    continue
                s = (q[rows] @ k[keys].T) * scale
                m = s.max(axis=1, keepdims=True)
                p = np.exp(s - m)
                p /= p.sum(axis=1, keepdims=True)
                o = p @ v[keys]
                Dr = (do[rows] * o).sum(axis=1, keepdims=True)
                ds = p * (do[rows] @ v[keys].T - Dr)
                dQ[b, h, rows] = scale * ds @ k[keys]
                np.add.at(dK[b, h], keys, scale * ds.T @ q[rows])
                np.add.at(dV[b, h], keys, p.T @ do[rows])
    tile_of_row = np.arange(g.Lq) // g.N
    dQ[:, :, ~qsel[tile_of_row]] = np.nan
    dK[:, :, ~ksel[tile_of_row]] = np.nan
    dV[:, :, ~ksel[tile_of_row]] = np.nan
    return dQ, dK, dV


def attention_flops(d, kept: np.ndarray, padded: bool = True) -> float:
    """FLOPs of the kept blocks: 4*d per (query row, key) pair.

    ``padded``: every kept block counts N x N pairs (N = tile size; text
    tiles as laid out); otherwise only valid query rows x valid keys count.
    """
    g = geometry(d)
    valid = valid_token_mask(d)
    rows = np.array([min((i + 1) * g.N, g.Lq) - i * g.N for i in range(g.NQ)], dtype=np.float64)
    vrows = np.array([valid[i * g.N: min((i + 1) * g.N, g.Lq)].sum() for i in range(g.NQ)], dtype=np.float64)
    cols = rows if padded else vrows
    qrows = rows if padded else vrows
    pairs = np.einsum("bhij,i,j->", kept.astype(np.float64), qrows, cols)
    return 4.0 * g.D * float(pairs)


def ssta_forward(d, q, k, v, q_text=None, k_text=None, v_text=None, q_tiles=None):
    """The whole forward in order: reorder, pool, score, select, window, union, attend, unorder.

    Inputs are numpy arrays in raster layout.  Returns a dict with every
    intermediate (packed tensors, pooled means, scores, masks, lists, packed O
    and LSE, raster O and text O).
    """
    qp = tile_reorder(d, q, q_text)
    kp = tile_reorder(d, k, k_text)
    vp = tile_reorder(d, v, v_text)
    qbar, kbar = tile_pool(d, qp), tile_pool(d, kp)
    S = block_scores(d, qbar, kbar)
    sel = select_topk(d, S)
    kept = kept_mask(d, sel)
    idx, cnt = kept_lists(kept)
    O, LSE = attention(d, qp, kp, vp, kept, q_tiles=q_tiles, scale=getattr(d, "scale", None))
    O_raster, O_text = tile_unorder(d, O)
    return dict(qp=qp, kp=kp, vp=vp, qbar=qbar, kbar=kbar, scores=S, sel=sel, kept=kept,
                kv_idx=idx, kv_cnt=cnt, O=O, LSE=LSE, O_raster=O_raster, O_text=O_text)
