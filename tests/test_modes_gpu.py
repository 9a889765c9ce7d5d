"""GPU parity of the mask modes against the CPU oracle: the importance score
(Step 2's similarity-minus-redundancy score in the importance-sampling form),
Algorithm 1's AND combination of selection and window, and the window cut at
the grid edges.  Same checks as the default mode (ssta_parity.full_check)."""
import numpy as np
import pytest
import torch

import block_sparse_video_ssta_b200 as S
import oracle
import ssta_inputs as si
from ssta_inputs import with_overrides
from ssta_parity import full_check, run_gpu

pytestmark = pytest.mark.gpu


def _report(name, st):
    print(f"\n[{name}] " + " ".join(f"{k}={v:.3g}" if isinstance(v, float) else f"{k}={v}" for k, v in st.items()))


F32_MODES = [
    dict(score_mode="importance"),
    dict(score_mode="importance", lam=0.5, T=5, Y=7, X=6, L_text=45),
    dict(combine="and", wT=1, wY=3, wX=3, topk=3),
    dict(combine="and", wT=1, wY=3, wX=3, topk=3, L_text=40),
    dict(window_mode="truncate", T=6, Y=12, X=12, wT=3, wY=3, wX=3, topk=1),
    dict(score_mode="importance", combine="and", window_mode="truncate", T=6, Y=12, X=12, wT=3, wY=3, wX=3,
         topk=4, B=2, H=3, L_text=7),
    dict(score_mode="importance", lam=1.0, topk=3),
    dict(score_mode="importance", lam=0.0, topk=3),
]


@pytest.mark.parametrize("ov", F32_MODES, ids=[str(i) for i in range(len(F32_MODES))])
def test_f32_modes(cuda_ok, ov):
    w = with_overrides(si.get_workload("tiny_f32"), **ov)
    st = full_check(w, seed=4)
    _report(f"f32 {ov}", st)
    assert st["rows_mask_mismatch"] == 0


@pytest.mark.parametrize("name,ov", [("tiny_f32", {}), ("small_bf16", dict(H=2, T=8, Y=16, X=16))])
def test_and_rows_with_nothing_to_attend(cuda_ok, name, ov):
    # AND with an empty selection (top-k = 0) and no text: no row keeps anything, so
    # O = 0 and LSE = -inf everywhere (fp32 kernel and tensor-core kernel)
    w = with_overrides(si.get_workload(name), combine="and", wT=3, wY=3, wX=3, topk=0, **ov)
    st = full_check(w, seed=6)
    _report(f"and-empty {name}", st)
    x = si.make_inputs(w, 6, device="cuda")
    r = run_gpu(w, x)
    cnt = r["kv_cnt"].cpu().numpy()
    assert (cnt == 0).all()
    g = oracle.geometry(w)
    lse = r["LSE"].cpu().numpy()
    for b, h, i in zip(*np.nonzero(cnt == 0)):
        assert np.all(np.isneginf(lse[b, h, i * g.N:(i + 1) * g.N]))
        assert torch.count_nonzero(r["O_packed"][b, h, i * g.N:(i + 1) * g.N]).item() == 0


BF16_MODES = [
    dict(score_mode="importance", H=4),
    dict(score_mode="importance", H=2, T=9, Y=9, X=17, L_text=1),          # NT = 18: scalar score path
    dict(combine="and", window_mode="truncate", H=2, wT=3, wY=3, wX=5, topk=16, L_text=300),
    dict(combine="and", H=2, T=8, Y=16, X=16, wT=1, wY=1, wX=1, topk=1),   # tensor-core kernel, empty rows
]


@pytest.mark.parametrize("ov", BF16_MODES, ids=[str(i) for i in range(len(BF16_MODES))])
def test_bf16_modes(cuda_ok, ov):
    w = with_overrides(si.get_workload("small_bf16"), **ov)
    st = full_check(w, seed=7)
    _report(f"bf16 {ov}", st)
    assert st["rows_mask_mismatch"] <= 2


def test_importance_full_size_sampled(cuda_ok):
    w = with_overrides(si.get_workload("p720_10s_bf16"), score_mode="importance")
    g = oracle.geometry(w)
    tiles = list(range(0, g.NT, 32)) + list(range(g.NT, g.NQ))
    st = full_check(w, seed=0, q_tiles=tiles, heads=[0, w.H - 1])
    _report("p720_10s importance", st)
    assert st["rows_mask_mismatch"] <= max(2, g.NT // 100)


def test_importance_deterministic(cuda_ok):
    w = with_overrides(si.get_workload("small_bf16"), score_mode="importance")
    x = si.make_inputs(w, 1, device="cuda")
    a, b = run_gpu(w, x), run_gpu(w, x)
    assert torch.equal(a["tile_scores"], b["tile_scores"])
    assert torch.equal(a["kv_idx"], b["kv_idx"]) and torch.equal(a["kv_cnt"], b["kv_cnt"])
