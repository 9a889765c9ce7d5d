"""The sequence-parallel forward on the GPU through NCCL (one rank: the exchange is
the identity permutation, the forward is the CUDA library) against the CPU oracle
run once on the whole tensors.  The multi-rank exchange is covered on CPU with
gloo ranks (tests/test_sequence_parallel.py).

Only rows whose kept set is unique are compared: a row where two tiles' oracle
scores sit within the 1e-4 band around the k-th score may keep either one, and
those rows are left out (the direct-call parity tests check such rows on the
GPU's own choice)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
import ssta_inputs as si
from block_sparse_video_ssta_b200.sequence_parallel import sequence_parallel_forward
from ssta_parity import BAND, TOL, kth_scores, oracle_mask, to_np

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_nccl_matches_oracle(cuda_ok):
    w = si.with_overrides(si.get_workload("small_bf16"), H=4, L_text=40)
    x = si.make_inputs(w, 1, device="cuda")
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        L = w.T * w.Y * w.X
        seq = [x[n].reshape(w.B, w.H, L, w.D) for n in ("q", "k", "v")]
        O, O_text = sequence_parallel_forward(w, *seq, x["q_text"], x["k_text"], x["v_text"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    g = oracle.geometry(w)
    q_np, k_np, v_np, qt_np, kt_np, vt_np = (to_np(x[n]) for n in ("q", "k", "v", "q_text", "k_text", "v_text"))
    qp, kp, S64, kept = oracle_mask(w, q_np, k_np, qt_np, kt_np)
    vp = oracle.tile_reorder(w, v_np, vt_np)
    O_ref, _ = oracle.attention(w, qp, kp, vp, kept)
    # rows with two or more tiles inside the band around the k-th score are ambiguous
    near = np.abs(S64 - kth_scores(w, S64)[..., None]) <= BAND
    ambiguous = np.zeros((w.B, w.H, g.NQ), dtype=bool)
    ambiguous[:, :, : g.NT] = near.sum(-1) >= 2
    assert ambiguous.mean() < 0.01
    tile_of_row = np.minimum(np.arange(g.Lq) // g.N, g.NQ - 1)
    O_ref[np.broadcast_to(ambiguous[:, :, tile_of_row], O_ref.shape[:3])] = np.nan
    O_r, O_t = oracle.tile_unorder(w, O_ref)
    got = to_np(O).reshape(O_r.shape)
    m = np.isfinite(O_r)
    tol = TOL["bf16"]
    err = np.abs(got[m] - O_r[m])
    assert err.max() <= tol["o_max"]
    assert np.linalg.norm(got[m] - O_r[m]) / np.linalg.norm(O_r[m]) <= tol["o_rel"]
    np.testing.assert_array_less(np.abs(to_np(O_text) - O_t), tol["o_max"])
