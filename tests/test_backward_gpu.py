"""GPU parity of the backward (dQ, dK, dV) through the C ABI against the float64
oracle (oracle.attention_bwd), on the GPU forward's own O, LSE and kept lists
(whose agreement with the oracle's mask is checked first).

Tolerances, from the arithmetic: fp32 keeps fp32 end to end (sums over a few
thousand keys): relative L2 and max-abs (scaled by the largest reference value)
1e-4.  bf16 stores O and the three gradients in bf16 (2^-9 relative per element)
and D = rowsum(dO * O) is formed from the stored O: relative L2 1e-2, max-abs
2e-2 of the largest reference value.  Each output row is also held to its own
relative L2 error (rows above 1e-3 of the largest row norm): 1e-4 for fp32, 5e-2
for bf16 (P and dS enter the products rounded to bf16, 2^-9 relative each, and the
row is stored in bf16), so that a fault confined to a few rows cannot hide inside
the whole-tensor figures."""
import numpy as np
import pytest
import torch

import block_sparse_video_ssta_b200 as S
import oracle
import ssta_inputs as si
from ssta_inputs import with_overrides
from ssta_parity import compare_masks, gpu_kept, oracle_mask, run_gpu, to_np

pytestmark = pytest.mark.gpu

TOL = {"f32": dict(rel=1e-4, mx=1e-4, row=1e-4), "bf16": dict(rel=1e-2, mx=2e-2, row=5e-2)}


def _oracle_packed(w, x, heads=None):
    """The oracle's own packing (Step 1) and kept mask (Steps 2-3) from the raster inputs."""
    sub = (lambda t: t) if heads is None else (lambda t: None if t is None else t[:, heads])
    q_np, k_np, v_np, qt_np, kt_np, vt_np = (to_np(sub(x[n])) for n in ("q", "k", "v", "q_text", "k_text", "v_text"))
    qp, kp, S64, kept = oracle_mask(w, q_np, k_np, qt_np, kt_np)
    vp = oracle.tile_reorder(w, v_np, vt_np)
    return qp, kp, vp, S64, kept


def _dO(w, shape, seed):
    """Upstream gradient on the packed layout: seeded on the CPU, one head at a time."""
    gen = torch.Generator(device="cpu").manual_seed(seed + 1000)
    B, H, L, D = shape
    return torch.cat([torch.randn((B, 1, L, D), generator=gen, dtype=torch.float32) for _ in range(H)], dim=1)


def _check(w, seed=0):
    x = si.make_inputs(w, seed, device="cuda")
    r = run_gpu(w, x)
    d = S.desc_from(w)
    dO32 = _dO(w, tuple(r["O_packed"].shape), seed)
    dO = dO32.to(r["O_packed"].dtype)
    dq, dk, dv, ws = S.ssta_attention_bwd(d, r["qp"], r["kp"], r["vp"], r["O_packed"], r["LSE"], dO.cuda(),
                                          r["kv_idx"], r["kv_cnt"])
    assert S.ssta_read_device_status(ws) == 0
    qp, kp, vp, _, kept_ref = _oracle_packed(w, x)
    assert np.array_equal(gpu_kept(w, r["kv_idx"], r["kv_cnt"]), kept_ref)
    ref = oracle.attention_bwd(w, qp, kp, vp, dO.float().numpy().astype(np.float64), kept_ref)
    stats = {}
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        a = to_np(got)
        assert np.isfinite(a).all()
        scale = max(np.abs(want).max(), 1e-30)
        mx = float(np.abs(a - want).max()) / scale
        rel = float(np.linalg.norm(a - want) / max(np.linalg.norm(want), 1e-30))
        # worst relative L2 error of one row, over rows above 1e-3 of the largest row norm
        rn = np.linalg.norm(want.reshape(-1, want.shape[-1]), axis=1)
        en = np.linalg.norm((a - want).reshape(-1, want.shape[-1]), axis=1)
        big = rn > 1e-3 * max(rn.max(), 1e-30)
        row_rel = float((en[big] / rn[big]).max()) if big.any() else 0.0
        stats[name] = (mx, rel, row_rel)
        assert mx <= TOL[w.dtype]["mx"] and rel <= TOL[w.dtype]["rel"], (name, mx, rel)
        assert row_rel <= TOL[w.dtype]["row"], (name, row_rel)
    print(f"\n[bwd {w.name} {w.dtype}] " + " ".join(f"{k}: max {v[0]:.2e} rel {v[1]:.2e} row {v[2]:.2e}"
                                                    for k, v in stats.items()))
    return stats


CASES = [
    ("tiny_f32", {}),
    ("tiny_f32", dict(T=5, Y=7, X=6, L_text=45)),                          # ragged grid, two text tiles
    ("tiny_f32", dict(B=2, H=3, T=6, Y=9, X=8, wY=3, topk=3, L_text=7, score_mode="importance")),
    ("tiny_f32", dict(combine="and", wT=1, wY=1, wX=1, topk=0)),           # nothing kept: all zero
    ("small_bf16", dict(H=2, T=8, Y=16, X=24)),
    ("small_bf16", dict(H=2, T=7, Y=12, X=20, L_text=300)),               # ragged, text
    ("small_bf16", dict(H=2, T=4, Y=8, X=16, tT=2, tY=8, tX=8)),           # N = 128
    ("small_bf16", dict(H=2, T=8, Y=16, X=16, tT=4, tY=8, tX=16, L_text=40)),  # N = 512
    ("small_bf16", dict(H=2, T=8, Y=16, X=24, score_mode="importance", combine="and", topk=6, wT=3, wY=3, wX=3)),
    ("small_bf16", dict(B=2, H=3, T=5, Y=12, X=20, L_text=130)),          # batch 2, odd heads, ragged, partial text
]


@pytest.mark.parametrize("name,ov", CASES, ids=[str(i) for i in range(len(CASES))])
def test_backward_matches_oracle(cuda_ok, name, ov):
    _check(with_overrides(si.get_workload(name), **ov), seed=3)


def test_backward_full_size_sampled(cuda_ok):
    """The backward as bench.py times it (720p-10s, 16 heads, GPU forward's O and LSE),
    checked on head 0 against the oracle on sampled rows: dQ of a first, middle, last
    (ragged) video tile and the text tile; dK and dV of a middle and the last key tile,
    summed over every query tile keeping them."""
    w = si.get_workload("p720_10s_bf16")
    g = oracle.geometry(w)
    x = si.make_inputs(w, 0, device="cuda")
    r = run_gpu(w, x, want_scores=False)
    assert r["status_mask"] == 0 and r["status_attn"] == 0
    d = S.desc_from(w)
    dO = _dO(w, tuple(r["O_packed"].shape), 0).to(r["O_packed"].dtype)
    dq, dk, dv, ws = S.ssta_attention_bwd(d, r["qp"], r["kp"], r["vp"], r["O_packed"], r["LSE"], dO.cuda(),
                                          r["kv_idx"], r["kv_cnt"])
    assert S.ssta_read_device_status(ws) == 0
    qp, kp, vp, S64, kept_ref = _oracle_packed(w, x, heads=[0])
    kept_gpu = gpu_kept(w, r["kv_idx"][:, :1], r["kv_cnt"][:, :1])
    # rows whose kept sets differ (allowed only within the score band of the k-th rank,
    # which compare_masks checks) are left out of the sample
    same = compare_masks(w, kept_gpu, kept_ref, S64)[0, 0]
    assert int((~same).sum()) <= max(2, g.NT // 100)
    good_q = lambda i: bool(same[i])
    good_key = lambda u: bool(same[kept_ref[0, 0, :, u] | kept_gpu[0, 0, :, u]].all())
    pick = lambda start, ok, step: next(i for i in range(start, start + step * g.NT, step) if ok(i % g.NQ)) % g.NQ
    q_tiles = [pick(0, good_q, 1), pick(g.NT // 2, good_q, 1), pick(g.NT - 1, good_q, -1), g.NT]
    assert good_q(g.NT)
    key_tiles = [pick(g.NT // 2 + 7, good_key, 1), pick(g.NT - 1, good_key, -1)]
    ref = oracle.attention_bwd(w, qp, kp, vp, dO[:, :1].float().numpy().astype(np.float64), kept_ref,
                               q_tiles=q_tiles, key_tiles=key_tiles)
    stats = {}
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        rows = np.isfinite(want[0, 0, :, 0])
        a = to_np(got[:, :1])[0, 0][rows]
        b = want[0, 0][rows]
        assert np.isfinite(a).all()
        scale = max(np.abs(b).max(), 1e-30)
        mx = float(np.abs(a - b).max()) / scale
        rel = float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))
        stats[name] = (mx, rel, int(rows.sum()))
        assert mx <= TOL["bf16"]["mx"] and rel <= TOL["bf16"]["rel"], (name, mx, rel)
    print("\n[bwd 720p-10s sampled] " + " ".join(f"{k}: max {v[0]:.2e} rel {v[1]:.2e} rows {v[2]}" for k, v in stats.items()))


def test_backward_full_size_deterministic(cuda_ok):
    """Three backward calls on the same 720p-10s inputs (as bench.py times it) give the
    same bytes: every sum runs in a fixed order, and no warp may read tensor memory that
    another warp of its lane group has already overwritten (a race there changes a few
    percent of the dK and dV rows from call to call while staying inside the loose
    whole-tensor tolerances above)."""
    w = si.get_workload("p720_10s_bf16")
    x = si.make_inputs(w, 0, device="cuda")
    r = run_gpu(w, x, want_scores=False)
    del x
    d = S.desc_from(w)
    dO = torch.randn(r["O_packed"].shape, device="cuda", generator=torch.Generator(device="cuda").manual_seed(5)
                     ).to(r["O_packed"].dtype)
    first = None
    for _ in range(3):
        out = S.ssta_attention_bwd(d, r["qp"], r["kp"], r["vp"], r["O_packed"], r["LSE"], dO, r["kv_idx"], r["kv_cnt"])
        assert S.ssta_read_device_status(out[3]) == 0
        if first is None:
            first = [t.clone() for t in out[:3]]
            continue
        for name, a, b in zip(("dq", "dk", "dv"), first, out[:3]):
            assert torch.equal(a, b), (name, int((a != b).sum()))
