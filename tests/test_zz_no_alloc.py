"""ssta_build_block_mask_noalloc: the block-mask builder for callers that cannot
allocate device memory at call time (its scratch is an array built into the
library).  Called through the C ABI and compared with ssta_build_block_mask,
which uses a caller-provided workspace, on two calls in a row.  Kept in a file
of its own that runs last."""
import ctypes

import pytest
import torch

import block_sparse_video_ssta_b200 as S
import ssta_inputs as si

pytestmark = pytest.mark.gpu

_f = S.lib.ssta_build_block_mask_noalloc
_f.argtypes = [ctypes.POINTER(S.Desc)] + [ctypes.c_void_p] * 6
_f.restype = ctypes.c_int


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("name,with_scores,mode", [("tiny_f32", True, "similarity"), ("small_bf16", False, "similarity"),
                                                   ("small_bf16", True, "similarity"),
                                                   ("p720_5s_bf16", False, "similarity"),
                                                   ("small_bf16", False, "importance"),
                                                   ("small_bf16", True, "importance")])
def test_noalloc_matches_workspace_entry_point(cuda_ok, name, with_scores, mode):
    w = si.with_overrides(si.get_workload(name), score_mode=mode)
    x = si.make_inputs(w, 2, device="cuda")
    d = S.desc_from(w)
    p = S.ssta_plan(d)
    qp = S.ssta_tile_reorder(d, x["q"], x["q_text"])
    kp = S.ssta_tile_reorder(d, x["k"], x["k_text"])
    ref_scores = torch.empty((w.B, w.H, p.num_tiles, p.num_tiles), dtype=torch.float32, device="cuda")
    ref_idx, ref_cnt, _ = S.ssta_build_block_mask(d, qp, kp, tile_scores=ref_scores)
    for _ in range(2):
        idx = torch.full_like(ref_idx, 12345)
        cnt = torch.full_like(ref_cnt, -5)
        scores = torch.full_like(ref_scores, float("nan")) if with_scores else None
        rc = _f(ctypes.byref(d), _ptr(qp), _ptr(kp), _ptr(idx), _ptr(cnt), _ptr(scores), _stream())
        assert rc == 0, S.ssta_status_string(rc)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        assert torch.equal(cnt, ref_cnt)
        if with_scores:
            assert torch.equal(scores, ref_scores)


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_ok):
    # 720p 10 s needs about 77 MB of scratch without a caller-provided score matrix
    d = S.desc_from(si.get_workload("p720_10s_bf16"))
    rc = _f(ctypes.byref(d), None, None, None, None, None, _stream())
    assert rc == 4 and S.ssta_status_string(rc) == "SSTA_ERR_WORKSPACE"
