"""Pins for the CPU oracle: each check comes from outside the oracle itself.

* reorder/unorder: explicit closed-form packed index per (t, y, x), zero pad
  rows, round trip;
* pooling: closed-form means of constant and linear fields over the valid part
  of each tile;
* scores: the identity "dot of tile means = block average of the token Gram
  matrix" and orthonormal-basis inputs;
* top-k: brute force over every k-subset (max score sum, lexicographically
  smallest on ties) with planted ties;
* window: brute force over every feasible start per axis (the start closest to
  the centred one) plus the pages' "within +-w/2" interior rule;
* attention: torch's scaled_dot_product_attention in float64 on the raster
  tokens with a token-level mask built in raster space (dense, block-diagonal
  and random kept sets), and torch.logsumexp for LSE; an empty kept set gives
  O = 0 and LSE = -inf;
* importance scores: closed forms (orthonormal keys: redundancy 1/2;
  identical keys: redundancy 1), the independent identity
  sum_{a != j} k_a . k_j = (sum_a k_a) . k_j - |k_j|^2, invariance to positive
  scaling of the pooled vectors, lambda = 1 reducing to (cosine + 1) / 2, a
  single tile and all-zero vectors; top-k on them by brute force;
* truncated window: brute force over each axis and the pages' |c' - c| <= w/2
  rule; AND combination: set intersection, and its two degenerate cases;
* compact lists: a hand-built mask with out-of-order, full and empty rows
  against hand-written ascending, -1-padded lists;
* kept-block FLOP count: closed forms N^2 / v^2 for one partially valid tile
  and (rows + text rows)^2 with a partial text tile, padded and valid-only;
* backward (dQ, dK, dV): torch autograd through the float64 masked SDPA on the
  raster tokens (random kept sets with and without text, the dense case), the
  invariants sum_keys dV = sum_rows dO and sum_keys dK = 0, empty kept sets.

Sources: "HunyuanVideo 1.5 Technical Report" (paper-graph-ui summary),
section "SSTA: Selective and Sliding Tile Attention", Steps 1-4 and the
attention equation.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import ssta_inputs as si
from ssta_inputs import Workload, with_overrides


def _desc(T=5, Y=6, X=7, tT=2, tY=4, tX=3, wT=1, wY=1, wX=1, topk=2, L_text=0, H=2, D=8, B=1):
    return Workload("pin", "f32", B, H, D, T, Y, X, tT, tY, tX, wT, wY, wX, topk, L_text,
                    "tile_offset")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------------------
# Step 1: reorder / unorder
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("L_text", [0, 5])
def test_reorder_closed_form_index(L_text):
    d = _desc(L_text=L_text)
    g = oracle.geometry(d)
    x = _rand((d.B, d.H, d.T, d.Y, d.X, d.D), 1)
    xt = _rand((d.B, d.H, L_text, d.D), 2) if L_text else None
    p = oracle.tile_reorder(d, x, xt)
    assert p.shape == (d.B, d.H, g.NT * g.N + L_text, d.D)
    nY, nX = -(-d.Y // d.tY), -(-d.X // d.tX)
    N = d.tT * d.tY * d.tX
    hit = np.zeros(p.shape[2], dtype=bool)
    for t in range(d.T):
        for y in range(d.Y):
            for xx in range(d.X):
                c = ((t // d.tT) * nY + y // d.tY) * nX + xx // d.tX
                o = ((t % d.tT) * d.tY + y % d.tY) * d.tX + xx % d.tX
                r = c * N + o
                np.testing.assert_array_equal(p[:, :, r], x[:, :, t, y, xx])
                hit[r] = True
    # every other video row is a pad row and holds zeros
    assert np.all(p[:, :, : g.NT * N][:, :, ~hit[: g.NT * N]] == 0)
    assert hit[: g.NT * N].sum() == d.T * d.Y * d.X
    if L_text:
        np.testing.assert_array_equal(p[:, :, g.NT * N:], xt)
    np.testing.assert_array_equal(oracle.valid_token_mask(d)[: g.NT * N], hit[: g.NT * N])
    back, back_t = oracle.tile_unorder(d, p)
    np.testing.assert_array_equal(back, x)
    if L_text:
        np.testing.assert_array_equal(back_t, xt)


def test_geometry_of_workloads():
    # grid sizes of the video latents: tiles after rounding up, top-k clamp
    expect = {"tiny_f32": (8, 32, 8, 256), "small_bf16": (112, 256, 112, 28672),
              "p480_5s_bf16": (224, 256, 224, 57344),
              "p720_5s_bf16": (480, 256, 481, 480 * 256 + 256),
              "p720_10s_bf16": (960, 256, 961, 960 * 256 + 256)}
    for name, (NT, N, NQ, Lq) in expect.items():
        g = oracle.geometry(si.get_workload(name))
        assert (g.NT, g.N, g.NQ, g.Lq) == (NT, N, NQ, Lq), name
    assert oracle.geometry(_desc(topk=99)).k == oracle.geometry(_desc()).NT


# ---------------------------------------------------------------------------
# Step 2: pooling, scores, top-k
# ---------------------------------------------------------------------------

def test_pool_constant_and_linear():
    d = _desc(D=3)
    g = oracle.geometry(d)
    t, y, x = np.meshgrid(np.arange(d.T), np.arange(d.Y), np.arange(d.X), indexing="ij")
    field = np.stack([np.full(t.shape, 2.5), 3.0 * t - 2.0 * y + 0.5 * x, 7.0 * x], axis=-1)
    raster = np.broadcast_to(field, (d.B, d.H) + field.shape).copy()
    pooled = oracle.tile_pool(d, oracle.tile_reorder(d, raster, None))
    nY, nX = g.nY, g.nX
    for cT in range(g.nT):
        for cY in range(nY):
            for cX in range(nX):
                c = (cT * nY + cY) * nX + cX
                # mean of a linear function over a box = value at the box's valid centre
                def centre(ci, tl, n):
                    lo, hi = ci * tl, min(ci * tl + tl, n) - 1
                    return 0.5 * (lo + hi)
                mt, my, mx = centre(cT, d.tT, d.T), centre(cY, d.tY, d.Y), centre(cX, d.tX, d.X)
                np.testing.assert_allclose(pooled[0, 1, c], [2.5, 3 * mt - 2 * my + 0.5 * mx, 7 * mx],
                                           rtol=0, atol=1e-12)


def test_scores_equal_block_average_of_token_gram():
    d = _desc(D=5, T=4, Y=5, X=3)
    g = oracle.geometry(d)
    q = _rand((1, 2, d.T, d.Y, d.X, d.D), 3)
    k = _rand((1, 2, d.T, d.Y, d.X, d.D), 4)
    S = oracle.tile_scores(d, oracle.tile_pool(d, oracle.tile_reorder(d, q, None)),
                           oracle.tile_pool(d, oracle.tile_reorder(d, k, None)))
    # tile membership computed in raster space, token Gram matrix averaged per block pair
    t, y, x = np.meshgrid(np.arange(d.T), np.arange(d.Y), np.arange(d.X), indexing="ij")
    member = (((t // d.tT) * g.nY + y // d.tY) * g.nX + x // d.tX).reshape(-1)
    for h in range(2):
        G = q[0, h].reshape(-1, d.D) @ k[0, h].reshape(-1, d.D).T
        for i in range(g.NT):
            for j in range(g.NT):
                blk = G[np.ix_(member == i, member == j)]
                assert abs(blk.mean() - S[0, h, i, j]) < 1e-10


def test_scores_orthonormal_basis():
    d = _desc(D=8, T=2, Y=4, X=6, tT=2, tY=4, tX=3)   # NT = 2 tiles
    q = np.zeros((1, 1, 2, 4, 6, 8))
    k = np.zeros_like(q)
    q[..., :3, 0] = 1.0   # tile 0 -> e0
    q[..., 3:, 1] = 1.0   # tile 1 -> e1
    k[..., :3, 1] = 2.0   # tile 0 -> 2 e1
    k[..., 3:, 0] = -1.0  # tile 1 -> -e0
    S = oracle.tile_scores(d, oracle.tile_pool(d, oracle.tile_reorder(d, q, None)),
                           oracle.tile_pool(d, oracle.tile_reorder(d, k, None)))
    np.testing.assert_array_equal(S[0, 0], [[0.0, -1.0], [2.0, 0.0]])


def _brute_topk(scores_row, k):
    best, best_key = None, None
    for sub in itertools.combinations(range(len(scores_row)), k):
        total = float(sum(float(scores_row[j]) for j in sub))
        key = (-total, sub)
        if best_key is None or key < best_key:
            best, best_key = sub, key
    return set(best)


@pytest.mark.parametrize("NT_grid", [(1, 2, 3), (2, 2, 2)])
def test_topk_brute_force_with_ties(NT_grid):
    nT, nY, nX = NT_grid
    d = _desc(T=nT, Y=nY, X=nX, tT=1, tY=1, tX=1)
    NT = nT * nY * nX
    rng = np.random.default_rng(5)
    for trial in range(40):
        # quantised scores -> many exact ties; sums are exact in float64
        S = (rng.integers(-3, 4, size=(1, 1, NT, NT)) * 0.25).astype(np.float64)
        if trial % 4 == 0:
            S = rng.standard_normal((1, 1, NT, NT))
        for k in range(0, NT + 2):
            dk = with_overrides(d, topk=k)
            sel = oracle.select_topk(dk, S)
            for i in range(NT):
                want = _brute_topk(S[0, 0, i].astype(np.float32), min(k, NT))
                assert set(np.nonzero(sel[0, 0, i])[0]) == want, (trial, k, i)


def test_topk_decision_in_float32():
    # two scores that differ only below float32 resolution tie; the lower index wins
    d = _desc(T=1, Y=1, X=3, tT=1, tY=1, tX=1, topk=1)
    S = np.array([[[[1.0, 1.0 + 1e-12, 0.5]] * 3]])
    sel = oracle.select_topk(d, S)
    assert list(np.nonzero(sel[0, 0, 0])[0]) == [0]


# ---------------------------------------------------------------------------
# Step 3: window
# ---------------------------------------------------------------------------

def _brute_axis_window(n, w, c):
    span = min(w, n)
    starts = range(0, n - span + 1)
    want = c - w // 2
    s = min(starts, key=lambda s: (abs(s - want), s))
    return set(range(s, s + span))


@pytest.mark.parametrize("n", range(1, 8))
@pytest.mark.parametrize("w", range(1, 10))
def test_axis_window_brute_force(n, w):
    m = oracle.ssta_oracle._axis_window(n, w)
    for c in range(n):
        got = set(np.nonzero(m[c])[0])
        assert got == _brute_axis_window(n, w, c)
        assert c in got and len(got) == min(w, n)
        if w % 2 == 1 and c - w // 2 >= 0 and c + w // 2 <= n - 1:
            assert got == {cc for cc in range(n) if abs(cc - c) <= w // 2}
        if w % 2 == 1:   # reflection symmetry for centred (odd) windows
            assert {n - 1 - cc for cc in got} == set(np.nonzero(m[n - 1 - c])[0])


def test_window_is_product_and_counts():
    d = _desc(T=7, Y=9, X=10, tT=1, tY=2, tX=3, wT=3, wY=3, wX=5)
    g = oracle.geometry(d)
    M = oracle.window_mask(d)
    coords = [(a, b, c) for a in range(g.nT) for b in range(g.nY) for c in range(g.nX)]
    for i, (a, b, c) in enumerate(coords):
        for j, (a2, b2, c2) in enumerate(coords):
            want = (a2 in _brute_axis_window(g.nT, 3, a) and b2 in _brute_axis_window(g.nY, 3, b)
                    and c2 in _brute_axis_window(g.nX, 5, c))
            assert M[i, j] == want
        assert M[i].sum() == min(3, g.nT) * min(3, g.nY) * min(5, g.nX)


# ---------------------------------------------------------------------------
# Step 4: union and attention
# ---------------------------------------------------------------------------

def test_union_counts_and_text_rows():
    w = si.get_workload("tiny_f32")
    d = with_overrides(w, L_text=40, wT=1, wY=3, wX=1, topk=3)
    g = oracle.geometry(d)
    x = si.make_inputs(d)
    r = oracle.ssta_forward(d, *(x[k].numpy() for k in ("q", "k", "v", "q_text", "k_text", "v_text")))
    win = oracle.window_mask(d)
    kept = r["kept"]
    W = int(win[0].sum())
    assert g.n_text == 2
    assert np.all(kept[:, :, g.NT:, :])                      # text queries attend everything
    assert np.all(kept[:, :, : g.NT, g.NT:])                 # every query attends text
    assert np.all(kept[:, :, : g.NT, : g.NT] >= win)         # window kept
    assert np.all(kept[:, :, : g.NT, : g.NT] >= r["sel"])    # selection kept
    c = kept[:, :, : g.NT, : g.NT].sum(-1)
    assert np.all(c >= max(g.k, W)) and np.all(c <= min(g.NT, g.k + W))
    np.testing.assert_array_equal(r["kv_cnt"], kept.sum(-1))


def _sdpa_raster(d, q, k, v, qt, kt, vt, allowed):
    """torch SDPA (float64) on raster tokens [+ text] with a token-level boolean mask."""
    B, H = q.shape[:2]
    L = d.T * d.Y * d.X
    cat = lambda a, b: np.concatenate([a.reshape(B, H, L, d.D)] + ([b] if b is not None else []), axis=2)
    Q, K, V = (torch.from_numpy(cat(a, b)) for a, b in ((q, qt), (k, kt), (v, vt)))
    m = torch.from_numpy(allowed)
    O = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=m)
    s = (Q @ K.transpose(-1, -2)) / math.sqrt(d.D)
    lse = torch.logsumexp(s.masked_fill(~m, -math.inf), dim=-1)
    return O.numpy(), lse.numpy()


def _raster_tile_of(d):
    g = oracle.geometry(d)
    t, y, x = np.meshgrid(np.arange(d.T), np.arange(d.Y), np.arange(d.X), indexing="ij")
    return (((t // d.tT) * g.nY + y // d.tY) * g.nX + x // d.tX).reshape(-1)


def _token_mask_from_tile_mask(d, kept):
    """[B,H,Lr,Lr] token mask in raster(+text) order from a tile-level kept mask."""
    g = oracle.geometry(d)
    member = _raster_tile_of(d)
    if d.L_text:
        member = np.concatenate([member, g.NT + np.arange(d.L_text) // g.N])
    return kept[:, :, member][:, :, :, member]


def _run_oracle(d, x):
    arrs = [x[k].double().numpy() if x[k] is not None else None
            for k in ("q", "k", "v", "q_text", "k_text", "v_text")]
    return arrs, oracle.ssta_forward(d, *arrs)


def _check_against_sdpa(d, arrs, r, kept_tiles):
    O_ref, lse_ref = _sdpa_raster(d, *arrs, _token_mask_from_tile_mask(d, kept_tiles))
    B, H = arrs[0].shape[:2]
    L = d.T * d.Y * d.X
    got = np.concatenate([r["O_raster"].reshape(B, H, L, d.D)]
                         + ([r["O_text"]] if d.L_text else []), axis=2)
    np.testing.assert_allclose(got, O_ref, rtol=0, atol=1e-12)
    lse_raster, lse_text = oracle.tile_unorder(d, r["LSE"][..., None])
    lse_got = np.concatenate([lse_raster.reshape(B, H, L)] + ([lse_text[..., 0]] if d.L_text else []),
                             axis=2)
    np.testing.assert_allclose(lse_got, lse_ref, rtol=0, atol=1e-11)


@pytest.mark.parametrize("L_text", [0, 37])
def test_dense_equivalence_whole_window(L_text):
    # window covering the whole grid -> dense attention over every valid token
    w = si.get_workload("tiny_f32")
    d = with_overrides(w, T=5, Y=7, X=6, wT=9, wY=9, wX=9, topk=0, L_text=L_text, D=16)
    arrs, r = _run_oracle(d, si.make_inputs(d))
    g = oracle.geometry(d)
    assert r["kept"].all()
    _check_against_sdpa(d, arrs, r, np.ones((d.B, d.H, g.NQ, g.NQ), dtype=bool))


def test_dense_equivalence_topk_all():
    w = si.get_workload("tiny_f32")
    d = with_overrides(w, topk=1000, D=16)
    arrs, r = _run_oracle(d, si.make_inputs(d))
    g = oracle.geometry(d)
    assert r["kept"].all()
    _check_against_sdpa(d, arrs, r, np.ones((d.B, d.H, g.NQ, g.NQ), dtype=bool))


def test_block_diagonal_special_case():
    # window = own tile and top-k = 0 -> attention inside each tile only
    w = si.get_workload("tiny_f32")
    d = with_overrides(w, T=5, Y=7, X=6, topk=0, D=16)
    arrs, r = _run_oracle(d, si.make_inputs(d))
    g = oracle.geometry(d)
    eye = np.broadcast_to(np.eye(g.NQ, dtype=bool), (d.B, d.H, g.NQ, g.NQ))
    np.testing.assert_array_equal(r["kept"], eye)
    member = _raster_tile_of(d)
    allowed = np.broadcast_to(member[:, None] == member[None, :], (d.B, d.H) + (len(member),) * 2)
    O_ref, _ = _sdpa_raster(d, *arrs, np.ascontiguousarray(allowed))
    np.testing.assert_allclose(r["O_raster"].reshape(O_ref.shape), O_ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("L_text", [0, 20])
def test_general_kept_set_equals_masked_sdpa(L_text):
    w = si.get_workload("tiny_f32")
    d = with_overrides(w, T=6, Y=9, X=8, topk=3, wT=1, wY=3, wX=1, L_text=L_text, D=16, H=3)
    arrs, r = _run_oracle(d, si.make_inputs(d, seed=7))
    _check_against_sdpa(d, arrs, r, r["kept"])
    # rows sum to one: sum_j exp(s_j - LSE) over the kept valid keys
    g = oracle.geometry(d)
    valid = oracle.valid_token_mask(d)
    qp, kp = r["qp"], r["kp"]
    for i in (0, g.NQ - 1):
        rows = slice(i * g.N, min((i + 1) * g.N, g.Lq))
        keys = np.concatenate([np.arange(j * g.N, min((j + 1) * g.N, g.Lq))
                               for j in np.nonzero(r["kept"][0, 1, i])[0]])
        keys = keys[valid[keys]]
        s = qp[0, 1, rows] @ kp[0, 1, keys].T / math.sqrt(d.D)
        np.testing.assert_allclose(np.exp(s - r["LSE"][0, 1, rows, None]).sum(1), 1.0, atol=1e-12)


def test_whole_mask_brute_force_tiny():
    # pooled means, scores, top-k, window and union rebuilt from raster data by brute force
    d = si.get_workload("tiny_f32")
    x = si.make_inputs(d)
    arrs, r = _run_oracle(d, x)
    g = oracle.geometry(d)
    member = _raster_tile_of(d)
    for h in range(d.H):
        qf = arrs[0][0, h].reshape(-1, d.D)
        kf = arrs[1][0, h].reshape(-1, d.D)
        qb = np.stack([qf[member == c].mean(0) for c in range(g.NT)])
        kb = np.stack([kf[member == c].mean(0) for c in range(g.NT)])
        S = qb @ kb.T
        for i in range(g.NT):
            sel = _brute_topk(S[i].astype(np.float32), g.k)
            a, b, c = i // (g.nY * g.nX), (i // g.nX) % g.nY, i % g.nX
            win = {(a2 * g.nY + b2) * g.nX + c2
                   for a2 in _brute_axis_window(g.nT, d.wT, a)
                   for b2 in _brute_axis_window(g.nY, d.wY, b)
                   for c2 in _brute_axis_window(g.nX, d.wX, c)}
            assert set(np.nonzero(r["kept"][0, h, i])[0]) == sel | win


def test_flop_count_dense_case():
    w = si.get_workload("tiny_f32")
    g = oracle.geometry(w)
    kept = np.ones((1, w.H, g.NQ, g.NQ), dtype=bool)
    L = w.T * w.Y * w.X
    assert oracle.attention_flops(w, kept) == 4.0 * w.D * w.H * L * L


def test_flop_count_partial_tiles_closed_form():
    # one video tile of N = 4*8*8 = 256 slots holding a 3x5x2 grid (v = 30 valid tokens):
    # padded it counts N x N (query row, key) pairs, valid-only v x v
    d = _desc(T=3, Y=5, X=2, tT=4, tY=8, tX=8, topk=1, D=16, H=1)
    kept = np.ones((1, 1, 1, 1), dtype=bool)
    assert oracle.attention_flops(d, kept) == 4.0 * 16 * 256 * 256
    assert oracle.attention_flops(d, kept, padded=False) == 4.0 * 16 * 30 * 30
    # a 2x2x1 grid in 2x2x2 tiles (4 of 8 slots valid) plus 5 text tokens (one partial text
    # tile): every pair kept; padded rows (8 video, 5 text) give (8 + 5)^2 pairs, valid rows
    # (4 video, 5 text) give (4 + 5)^2
    d = _desc(T=2, Y=2, X=1, tT=2, tY=2, tX=2, topk=1, L_text=5, D=8, H=3)
    g = oracle.geometry(d)
    assert (g.NT, g.n_text, g.NQ) == (1, 1, 2)
    kept = np.ones((1, 3, 2, 2), dtype=bool)
    assert oracle.attention_flops(d, kept) == 4.0 * 8 * 3 * 13 ** 2
    assert oracle.attention_flops(d, kept, padded=False) == 4.0 * 8 * 3 * 9 ** 2
    # drop the video query tile's text key tile in head 1: that head loses 8 x 5 padded and
    # 4 x 5 valid pairs
    kept[0, 1, 0, 1] = False
    assert oracle.attention_flops(d, kept) == 4.0 * 8 * (3 * 169 - 40)
    assert oracle.attention_flops(d, kept, padded=False) == 4.0 * 8 * (3 * 81 - 20)


def test_kept_lists_of_a_hand_built_mask():
    kept = np.zeros((1, 2, 3, 6), dtype=bool)
    kept[0, 0, 0, [4, 1, 3]] = True            # set out of order: the list is ascending
    kept[0, 0, 2, :] = True                    # every tile
    kept[0, 1, 1, [5]] = True                  # row 0 of head 1 and row 1 of head 0 keep nothing
    idx, cnt = oracle.kept_lists(kept)
    assert idx.dtype == np.int32 and cnt.dtype == np.int32
    want_idx = np.full((1, 2, 3, 6), -1, dtype=np.int32)            # width = the largest count, 6
    want_idx[0, 0, 0, :3] = [1, 3, 4]
    want_idx[0, 0, 2, :] = [0, 1, 2, 3, 4, 5]
    want_idx[0, 1, 1, :1] = [5]
    np.testing.assert_array_equal(idx, want_idx)
    np.testing.assert_array_equal(cnt, [[[3, 0, 6], [0, 1, 0]]])
    # width follows the largest count; an all-empty mask gives width 0
    idx, cnt = oracle.kept_lists(kept[:, :, :2])
    assert idx.shape == (1, 2, 2, 3)
    np.testing.assert_array_equal(idx[0, 0, 0], [1, 3, 4])
    np.testing.assert_array_equal(idx[0, 1, 1], [5, -1, -1])
    idx, cnt = oracle.kept_lists(np.zeros((1, 1, 2, 4), dtype=bool))
    assert idx.shape == (1, 1, 2, 0) and cnt.tolist() == [[[0, 0]]]


# ---------------------------------------------------------------------------
# Mask modes: importance scoring, truncated window, AND combination
# ("Selective Mask Generation": Score_i = lambda Score_s - beta Score_r; the
# blog's importance-sampling routine; Algorithm 1's M_sel AND M_sta; the
# "within +-w/2" window rule)
# ---------------------------------------------------------------------------

def _imp_desc(lam=0.9, **kw):
    return with_overrides(_desc(**kw), score_mode="importance", lam=lam)


def test_importance_orthonormal_keys_closed_form():
    # keys = distinct basis vectors, query i = basis vector i: cos = delta_ij, every key-key
    # cosine off the diagonal is 0, so redundancy = (0 + 1) / 2 = 1/2 for every key
    d = _imp_desc(lam=0.7)
    NT, D = 5, 8
    kb = np.eye(D)[None, None, :NT] * np.arange(1, NT + 1)[None, None, :, None]   # scaled: norm must not matter
    qb = np.eye(D)[None, None, :NT] * 3.0
    S = oracle.importance_scores(d, qb, kb)
    want = 0.7 * (np.eye(NT) + 1.0) / 2.0 - 0.3 * 0.5
    np.testing.assert_allclose(S[0, 0], want, atol=1e-15)


def test_importance_identical_keys_have_full_redundancy():
    d = _imp_desc(lam=0.6)
    v = _rand((8,), 3)
    kb = np.tile(v, (1, 1, 4, 1)) * np.array([1.0, 2.0, 0.5, 7.0])[None, None, :, None]
    qb = _rand((1, 1, 3, 8), 4)
    S = oracle.importance_scores(d, qb, kb)
    cos = (qb[0, 0] @ v) / (np.linalg.norm(qb[0, 0], axis=1) * np.linalg.norm(v))
    want = 0.6 * (cos[:, None] + 1.0) / 2.0 - 0.4 * 1.0
    np.testing.assert_allclose(S[0, 0], np.broadcast_to(want, (3, 4)), atol=1e-14)


def test_importance_matches_sum_vector_identity():
    # independent route: sum_{a != j} k^_a . k^_j = (sum_a k^_a) . k^_j - |k^_j|^2
    d = _imp_desc(lam=0.9)
    qb, kb = _rand((2, 3, 7, 16), 5), _rand((2, 3, 9, 16), 6)
    S = oracle.importance_scores(d, qb, kb)
    qn = qb / np.linalg.norm(qb, axis=-1, keepdims=True)
    kn = kb / np.linalg.norm(kb, axis=-1, keepdims=True)
    u = kn.sum(axis=-2, keepdims=True)
    dots = (kn * u).sum(-1) - (kn * kn).sum(-1)                  # [B,H,NT]
    red = 0.5 + dots / (2.0 * (kb.shape[-2] - 1))
    want = 0.9 * (np.einsum("bhid,bhjd->bhij", qn, kn) + 1.0) / 2.0 - 0.1 * red[..., None, :]
    np.testing.assert_allclose(S, want, atol=1e-13)


def test_importance_scale_invariance_and_lambda_one():
    d = _imp_desc(lam=1.0)
    qb, kb = _rand((1, 2, 6, 8), 7), _rand((1, 2, 6, 8), 8)
    S = oracle.importance_scores(d, qb, kb)
    S2 = oracle.importance_scores(d, qb * _rand((1, 2, 6, 1), 9) ** 2 + 0 * qb, kb * 5.0)
    # positive per-row scales of q (squares of normals) and a global scale of k change nothing
    np.testing.assert_allclose(S, S2, atol=1e-14)
    cos = np.einsum("bhid,bhjd->bhij", qb / np.linalg.norm(qb, axis=-1, keepdims=True),
                    kb / np.linalg.norm(kb, axis=-1, keepdims=True))
    np.testing.assert_allclose(S, (cos + 1.0) / 2.0, atol=1e-14)   # lam = 1: similarity only


def test_importance_single_tile_and_zero_vectors():
    d = _imp_desc(lam=0.9)
    S = oracle.importance_scores(d, _rand((1, 1, 1, 4), 1), _rand((1, 1, 1, 4), 2))
    q = _rand((4,), 1); k = _rand((4,), 2)
    cos = q @ k / (np.linalg.norm(q) * np.linalg.norm(k))
    np.testing.assert_allclose(S[0, 0, 0, 0], 0.9 * (cos + 1) / 2, atol=1e-15)   # no other tile: no redundancy
    qb = np.zeros((1, 1, 2, 4)); kb = np.zeros((1, 1, 3, 4))
    S = oracle.importance_scores(d, qb, kb)                                     # zero vectors stay zero
    np.testing.assert_allclose(S, 0.9 * 0.5 - 0.1 * 0.5, atol=1e-15)


def test_importance_forward_selects_by_importance():
    w = with_overrides(si.get_workload("tiny_f32"), score_mode="importance", topk=3)
    x = si.make_inputs(w)
    r = oracle.ssta_forward(w, *(None if x[k] is None else x[k].numpy()
                                 for k in ("q", "k", "v", "q_text", "k_text", "v_text")))
    S = oracle.importance_scores(w, r["qbar"], r["kbar"])
    np.testing.assert_array_equal(r["scores"], S)
    for h in range(w.H):
        for i in range(oracle.geometry(w).NT):
            assert set(np.nonzero(r["sel"][0, h, i])[0]) == _brute_topk(S[0, h, i].astype(np.float32), 3)


def _brute_axis_window_truncated(n, w, c):
    return {cc for cc in range(n) if c - w // 2 <= cc < c - w // 2 + w}


@pytest.mark.parametrize("n", range(1, 8))
@pytest.mark.parametrize("w", range(1, 10))
def test_truncated_window_brute_force(n, w):
    m = oracle.ssta_oracle._axis_window(n, w, truncate=True)
    shift = oracle.ssta_oracle._axis_window(n, w)
    for c in range(n):
        got = set(np.nonzero(m[c])[0])
        assert got == _brute_axis_window_truncated(n, w, c)
        assert c in got
        if w % 2 == 1:   # the pages' rule: |c' - c| <= w/2, cut at the grid
            assert got == {cc for cc in range(n) if abs(cc - c) <= w // 2}
        if c - w // 2 >= 0 and c - w // 2 + w <= n:   # away from the edges both modes agree
            assert got == set(np.nonzero(shift[c])[0])


def test_truncated_window_mask_is_product():
    d = with_overrides(_desc(T=7, Y=9, X=10, tT=1, tY=2, tX=3, wT=3, wY=3, wX=5), window_mode="truncate")
    g = oracle.geometry(d)
    M = oracle.window_mask(d)
    coords = [(a, b, c) for a in range(g.nT) for b in range(g.nY) for c in range(g.nX)]
    for i, (a, b, c) in enumerate(coords):
        want = np.array([a2 in _brute_axis_window_truncated(g.nT, 3, a) and b2 in _brute_axis_window_truncated(g.nY, 3, b)
                         and c2 in _brute_axis_window_truncated(g.nX, 5, c) for (a2, b2, c2) in coords])
        np.testing.assert_array_equal(M[i], want)


def test_and_combination():
    w = with_overrides(si.get_workload("tiny_f32"), combine="and", wT=1, wY=3, wX=3, topk=3, L_text=40)
    g = oracle.geometry(w)
    x = si.make_inputs(w)
    r = oracle.ssta_forward(w, *(x[k].numpy() for k in ("q", "k", "v", "q_text", "k_text", "v_text")))
    win = oracle.window_mask(w)
    np.testing.assert_array_equal(r["kept"][:, :, : g.NT, : g.NT], r["sel"] & win[None, None])
    assert np.all(r["kept"][:, :, : g.NT, g.NT:]) and np.all(r["kept"][:, :, g.NT:, :])
    # top-k = all tiles: AND leaves the window; window = whole grid: AND leaves the selection
    wa = with_overrides(w, topk=100)
    ra = oracle.kept_mask(wa, oracle.select_topk(wa, r["scores"]))
    np.testing.assert_array_equal(ra[:, :, : g.NT, : g.NT], np.broadcast_to(win, ra[:, :, : g.NT, : g.NT].shape))
    wb = with_overrides(w, wT=9, wY=9, wX=9)
    rb = oracle.kept_mask(wb, r["sel"])
    np.testing.assert_array_equal(rb[:, :, : g.NT, : g.NT], r["sel"])


def test_empty_kept_set_gives_zero_output():
    # AND with a window that excludes every selected tile and no text: nothing to attend
    w = with_overrides(si.get_workload("tiny_f32"), combine="and", wT=1, wY=1, wX=1, topk=1)
    g = oracle.geometry(w)
    x = si.make_inputs(w)
    arrs = [x[k].numpy().astype(np.float64) for k in ("q", "k", "v")]
    qp, kp, vp = (oracle.tile_reorder(w, a, None) for a in arrs)
    kept = np.zeros((w.B, w.H, g.NQ, g.NQ), dtype=bool)
    kept[:, :, 0, 1] = True                              # tile 0 keeps tile 1 only; the others keep nothing
    O, L = oracle.attention(w, qp, kp, vp, kept)
    assert np.all(O[:, :, g.N:] == 0.0) and np.all(np.isneginf(L[:, :, g.N:]))
    assert np.all(np.isfinite(L[:, :, : g.N]))


# ---------------------------------------------------------------------------
# Backward of Step 4: dQ, dK, dV
# ---------------------------------------------------------------------------

def _sdpa_grads(d, arrs, dO_raster, dO_text, allowed):
    """torch autograd (float64) through the masked SDPA on raster tokens [+ text]."""
    q, k, v, qt, kt, vt = arrs
    B, H = q.shape[:2]
    L = d.T * d.Y * d.X
    cat = lambda a, b: np.concatenate([a.reshape(B, H, L, d.D)] + ([b] if b is not None else []), axis=2)
    Q, K, V = (torch.from_numpy(cat(a, b)).requires_grad_(True) for a, b in ((q, qt), (k, kt), (v, vt)))
    O = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=torch.from_numpy(allowed))
    (O * torch.from_numpy(cat(dO_raster, dO_text))).sum().backward()
    return Q.grad.numpy(), K.grad.numpy(), V.grad.numpy()


def _bwd_case(d, seed, kept_fn):
    g = oracle.geometry(d)
    x = si.make_inputs(d, seed)
    arrs, r = _run_oracle(d, x)
    kept = kept_fn(d, g, r)
    rng = np.random.default_rng(seed + 100)
    dO_r = rng.standard_normal((d.B, d.H, d.T, d.Y, d.X, d.D))
    dO_t = rng.standard_normal((d.B, d.H, d.L_text, d.D)) if d.L_text else None
    dOp = oracle.tile_reorder(d, dO_r, dO_t)
    dQ, dK, dV = oracle.attention_bwd(d, r["qp"], r["kp"], r["vp"], dOp, kept)
    return g, arrs, r, kept, dO_r, dO_t, dOp, (dQ, dK, dV)


def _to_raster(d, t):
    B, H = t.shape[:2]
    L = d.T * d.Y * d.X
    ras, txt = oracle.tile_unorder(d, t)
    return np.concatenate([ras.reshape(B, H, L, d.D)] + ([txt] if d.L_text else []), axis=2)


@pytest.mark.parametrize("L_text", [0, 37])
def test_backward_equals_autograd_random_kept(L_text):
    d = with_overrides(_desc(T=4, Y=8, X=6, tT=2, tY=4, tX=3, L_text=L_text, H=2, D=8), recipe="tile_offset")

    def kept_fn(d, g, r):
        rng = np.random.default_rng(7)
        kept = rng.random((d.B, d.H, g.NQ, g.NQ)) < 0.4
        kept[:, :, np.arange(g.NQ), np.arange(g.NQ)] = True        # every row keeps something
        return kept

    g, arrs, r, kept, dO_r, dO_t, dOp, grads = _bwd_case(d, 11, kept_fn)
    ref = _sdpa_grads(d, arrs, dO_r, dO_t, _token_mask_from_tile_mask(d, kept))
    for got, want in zip(grads, ref):
        np.testing.assert_allclose(_to_raster(d, got), want, rtol=0, atol=1e-11)
    valid = oracle.valid_token_mask(d)
    for t in grads:                                                    # pad rows stay zero
        assert np.all(t[:, :, ~valid] == 0.0)


def test_backward_dense_and_invariants():
    d = si.get_workload("tiny_f32")
    d = with_overrides(d, wT=9, wY=9, wX=9, topk=0, L_text=20)          # window = whole grid: dense

    def kept_fn(d, g, r):
        return r["kept"]

    g, arrs, r, kept, dO_r, dO_t, dOp, (dQ, dK, dV) = _bwd_case(d, 12, kept_fn)
    ref = _sdpa_grads(d, arrs, dO_r, dO_t, _token_mask_from_tile_mask(d, kept))
    for got, want in zip((dQ, dK, dV), ref):
        np.testing.assert_allclose(_to_raster(d, got), want, rtol=0, atol=1e-11)
    valid = oracle.valid_token_mask(d)
    # rows of P sum to 1: the dV of all keys sums to the dO of all valid query rows;
    # rows of dS sum to 0: the dK of all keys sums to 0
    np.testing.assert_allclose(dV.sum(axis=2), dOp[:, :, valid].sum(axis=2), rtol=0, atol=1e-10)
    np.testing.assert_allclose(dK.sum(axis=2), 0.0, rtol=0, atol=1e-10)


def test_backward_empty_rows_contribute_nothing():
    d = with_overrides(si.get_workload("tiny_f32"), combine="and", wT=1, wY=1, wX=1, topk=0)

    def kept_fn(d, g, r):
        return r["kept"]                                                # nothing kept anywhere

    g, arrs, r, kept, dO_r, dO_t, dOp, (dQ, dK, dV) = _bwd_case(d, 13, kept_fn)
    assert not kept.any()
    assert not dQ.any() and not dK.any() and not dV.any()


def test_backward_restricted_tiles_equal_autograd():
    """attention_bwd restricted to some dQ tiles and some dK/dV tiles (the form the
    full-size sampled GPU test uses) gives autograd's values on those rows, NaN elsewhere."""
    d = with_overrides(_desc(T=4, Y=8, X=6, tT=2, tY=4, tX=3, L_text=37, H=2, D=8), recipe="tile_offset")
    g = oracle.geometry(d)
    x = si.make_inputs(d, 13)
    arrs, r = _run_oracle(d, x)
    rng = np.random.default_rng(9)
    kept = rng.random((d.B, d.H, g.NQ, g.NQ)) < 0.4
    kept[:, :, np.arange(g.NQ), np.arange(g.NQ)] = True
    dO_r = rng.standard_normal((d.B, d.H, d.T, d.Y, d.X, d.D))
    dO_t = rng.standard_normal((d.B, d.H, d.L_text, d.D))
    dOp = oracle.tile_reorder(d, dO_r, dO_t)
    q_tiles, key_tiles = [0, g.NT - 1, g.NQ - 1], [1, g.NT - 1]
    got = oracle.attention_bwd(d, r["qp"], r["kp"], r["vp"], dOp, kept, q_tiles=q_tiles, key_tiles=key_tiles)
    ref = _sdpa_grads(d, arrs, dO_r, dO_t, _token_mask_from_tile_mask(d, kept))
    tile_of_row = np.arange(g.Lq) // g.N
    for t, want, sel in zip(got, ref, (q_tiles, key_tiles, key_tiles)):
        rows = np.isin(tile_of_row, sel)
        assert np.all(np.isfinite(t[:, :, rows])) and np.all(np.isnan(t[:, :, ~rows]))
        ras = _to_raster(d, np.where(np.isnan(t), 0.0, t))
        mask = _to_raster(d, np.broadcast_to(rows[None, None, :, None], t.shape).astype(np.float64)) > 0
        np.testing.assert_allclose(ras[mask], want[mask], rtol=0, atol=1e-11)
