"""GPU parity of the backward (dQ, dK, dV) through the C ABI against the float64
oracle (oracle.attention_bwd), on the GPU forward's own O, LSE and kept lists
(whose agreement with the oracle's mask is checked first).

Tolerances, from the arithmetic: fp32 keeps fp32 end to end (sums over a few
thousand keys): relative L2 and max-abs (scaled by the largest reference value)
1e-4.  bf16 stores O and the three gradients in bf16 (2^-9 relative per element)
and D = rowsum(dO * O) is formed from the stored O: relative L2 1e-2, max-abs
2e-2 of the largest reference value."""
import numpy as np
import pytest
import torch

import block_sparse_video_ssta_b200 as S
import oracle
import ssta_inputs as si
from ssta_inputs import with_overrides
from ssta_parity import gpu_kept, oracle_mask, run_gpu, to_np

pytestmark = pytest.mark.gpu

TOL = {"f32": dict(rel=1e-4, mx=1e-4), "bf16": dict(rel=1e-2, mx=2e-2)}


def _check(w, seed=0):
    g = oracle.geometry(w)
    x = si.make_inputs(w, seed, device="cuda")
    r = run_gpu(w, x)
    d = S.desc_from(w)
    gen = torch.Generator(device="cpu").manual_seed(seed + 1000)
    dO = torch.randn(r["O_packed"].shape, generator=gen, dtype=torch.float32).to(r["O_packed"].dtype).cuda()
    dq, dk, dv, ws = S.ssta_attention_bwd(d, r["qp"], r["kp"], r["vp"], r["O_packed"], r["LSE"], dO,
                                          r["kv_idx"], r["kv_cnt"])
    assert S.ssta_read_device_status(ws) == 0
    kept = gpu_kept(w, r["kv_idx"], r["kv_cnt"])
    _, _, _, kept_ref = oracle_mask(w, *(to_np(x[n]) for n in ("q", "k", "q_text", "k_text")))
    assert np.array_equal(kept, kept_ref)
    ref = oracle.attention_bwd(w, to_np(r["qp"]), to_np(r["kp"]), to_np(r["vp"]), to_np(dO), kept)
    stats = {}
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        a = to_np(got)
        assert np.isfinite(a).all()
        scale = max(np.abs(want).max(), 1e-30)
        mx = float(np.abs(a - want).max()) / scale
        rel = float(np.linalg.norm(a - want) / max(np.linalg.norm(want), 1e-30))
        stats[name] = (mx, rel)
        assert mx <= TOL[w.dtype]["mx"] and rel <= TOL[w.dtype]["rel"], (name, mx, rel)
    print(f"\n[bwd {w.name} {w.dtype}] " + " ".join(f"{k}: max {v[0]:.2e} rel {v[1]:.2e}" for k, v in stats.items()))
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
]


@pytest.mark.parametrize("name,ov", CASES, ids=[str(i) for i in range(len(CASES))])
def test_backward_matches_oracle(cuda_ok, name, ov):
    _check(with_overrides(si.get_workload(name), **ov), seed=3)
