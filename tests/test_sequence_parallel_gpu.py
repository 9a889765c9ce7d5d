"""The sequence-parallel forward on the GPU through NCCL (one rank: the exchange is
the identity permutation, the forward is the CUDA library): bit-identical to a
direct call.  The multi-rank exchange is covered on CPU with gloo ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist

import block_sparse_video_ssta_b200 as S
import ssta_inputs as si
from block_sparse_video_ssta_b200.sequence_parallel import sequence_parallel_forward

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_nccl_matches_direct_call(cuda_ok):
    w = si.with_overrides(si.get_workload("small_bf16"), H=4, L_text=40)
    x = si.make_inputs(w, 1, device="cuda")
    ref = S.ssta_forward(S.desc_from(w), x["q"], x["k"], x["v"], x["q_text"], x["k_text"], x["v_text"])
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        L = w.T * w.Y * w.X
        seq = [x[n].reshape(w.B, w.H, L, w.D) for n in ("q", "k", "v")]
        O, O_text = sequence_parallel_forward(w, *seq, x["q_text"], x["k_text"], x["v_text"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert torch.equal(O, ref["O"].reshape(w.B, w.H, L, w.D))
    assert torch.equal(O_text, ref["O_text"])
