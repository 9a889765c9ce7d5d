"""The mask kernels are launched as programmatic dependents of the kernel before them on
the stream: they may start early and wait (griddepcontrol.wait) for it before reading
what it wrote.  Here the kernel just before the mask build is the reorder that rewrites,
in place, the packed k (and q) the build reads, and the workspace, lists and score
matrix are reused from a call on other inputs, so a read issued ahead of the wait would
see the previous inputs, means or scores.  Every result must equal a reference built
with full synchronisation between the steps."""
import pytest
import torch

import block_sparse_video_ssta_b200 as S
import ssta_inputs as si
from ssta_inputs import with_overrides

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,ov", [("small_bf16", {}), ("small_bf16", dict(score_mode="importance")),
                                     ("tiny_f32", dict(T=6, Y=9, X=8, L_text=7))],
                         ids=["similarity", "importance", "f32"])
def test_mask_build_right_after_the_reorder_that_writes_its_inputs(cuda_ok, name, ov):
    w = with_overrides(si.get_workload(name), **ov)
    d = S.desc_from(w)
    p = S.ssta_plan(d)
    xs = [si.make_inputs(w, seed, device="cuda") for seed in (11, 12)]
    refs = []
    for x in xs:   # references: every step synchronised
        qp = S.ssta_tile_reorder(d, x["q"], x["q_text"])
        kp = S.ssta_tile_reorder(d, x["k"], x["k_text"])
        torch.cuda.synchronize()
        sc = torch.empty((w.B, w.H, p.num_tiles, p.num_tiles), dtype=torch.float32, device="cuda")
        idx, cnt, _ = S.ssta_build_block_mask(d, qp, kp, tile_scores=sc)
        torch.cuda.synchronize()
        refs.append((idx.clone(), cnt.clone(), sc.clone()))
    qp = torch.empty_like(qp)
    kp = torch.empty_like(kp)
    idx = torch.empty_like(refs[0][0])
    cnt = torch.empty_like(refs[0][1])
    sc = torch.empty_like(refs[0][2])
    ws = torch.empty(p.workspace_bytes, dtype=torch.uint8, device="cuda")
    for it in range(6):
        x = xs[it % 2]
        S.ssta_tile_reorder(d, x["q"], x["q_text"], x_packed=qp)
        S.ssta_tile_reorder(d, x["k"], x["k_text"], x_packed=kp)
        S.ssta_build_block_mask(d, qp, kp, kv_idx=idx, kv_cnt=cnt, tile_scores=sc, workspace=ws)
        torch.cuda.synchronize()
        assert S.ssta_read_device_status(ws) == 0
        r_idx, r_cnt, r_sc = refs[it % 2]
        assert torch.equal(cnt, r_cnt), it
        assert torch.equal(idx, r_idx), it
        assert torch.equal(sc, r_sc), it
