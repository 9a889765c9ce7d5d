"""Sequence-parallel exchange around the SSTA forward, on CPU with gloo ranks
(2 and 4): token-sharded q, k, v go through an all-to-all to head shards, the
forward runs per head group, and an all-to-all brings O back to token shards.
The per-head forward here is the CPU oracle (injected), so the result must equal
the oracle run once on the whole tensors, element for element; the exchange and
its layouts are what is under test."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import ssta_inputs as si
from block_sparse_video_ssta_b200.sequence_parallel import sequence_parallel_forward

NAMES = ("q", "k", "v", "q_text", "k_text", "v_text")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload(mode):
    w = si.with_overrides(si.get_workload("tiny_f32"), H=4, topk=3, wT=1, wY=3, wX=3, L_text=40)
    return si.with_overrides(w, score_mode="importance") if mode == "importance" else w


def _np(t):
    return None if t is None else t.numpy().astype(np.float64)


def _oracle_op(w_local, q, k, v, qt, kt, vt):
    r = oracle.ssta_forward(w_local, *(_np(t) for t in (q, k, v, qt, kt, vt)))
    return torch.from_numpy(r["O_raster"]), (None if r["O_text"] is None else torch.from_numpy(r["O_text"]))


def _rank(rank, world, port, mode, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = _workload(mode)
        x = si.make_inputs(w, 3, device="cpu")
        L = w.T * w.Y * w.X
        Lr = L // world
        flat = {n: x[n].double().reshape(w.B, w.H, L, w.D) for n in ("q", "k", "v")}
        mine = [flat[n][:, :, rank * Lr:(rank + 1) * Lr].contiguous() for n in ("q", "k", "v")]
        text = [x[n].double() for n in ("q_text", "k_text", "v_text")]
        O, O_text = sequence_parallel_forward(w, *mine, *text, op=_oracle_op)
        parts = [torch.empty_like(O) for _ in range(world)]
        dist.all_gather(parts, O)
        if rank == 0:
            out["O"] = torch.cat(parts, dim=2).numpy()
            out["O_text"] = O_text.numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("mode", ["similarity", "importance"])
def test_sequence_parallel_equals_single_process(world, mode):
    w = _workload(mode)
    x = si.make_inputs(w, 3, device="cpu")
    ref = oracle.ssta_forward(w, *(_np(x[n]) for n in NAMES))
    L = w.T * w.Y * w.X
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, _free_port(), mode, out), nprocs=world, join=True)
        got = dict(out)
    np.testing.assert_array_equal(got["O"], ref["O_raster"].reshape(w.B, w.H, L, w.D))
    np.testing.assert_array_equal(got["O_text"], ref["O_text"])


def test_uneven_split_is_rejected():
    w = si.with_overrides(si.get_workload("tiny_f32"), H=3)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        # one rank, H = 3 and 256 tokens split fine; a wrong token count per rank is rejected
        q = torch.zeros(1, 3, 100, w.D)
        with pytest.raises(ValueError):
            sequence_parallel_forward(w, q, q, q, op=_oracle_op)
    finally:
        dist.destroy_process_group()
