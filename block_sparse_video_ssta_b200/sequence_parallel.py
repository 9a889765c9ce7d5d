"""Sequence-parallel SSTA forward: head-sharded attention between token-sharded layers.

A video diffusion transformer run with sequence parallelism keeps the token
sequence split across ranks ("HunyuanVideo 1.5 Technical Report": 8 GPUs with
context / sequence parallelism; the apoapsis blog, "parallel_states": the
transformer redistributes attention heads across sequence-parallel groups with
all-to-all communication).  SSTA selects key tiles per head (Step 2,
"head-specific selection"), so once every rank holds the whole sequence for a
group of heads, the mask and the attention of those heads need nothing from the
other ranks.  This module performs that exchange around the forward:

1. all-to-all: token slice of every head -> every token of H/P heads;
2. the SSTA forward on the rank's heads (the CUDA library by default);
3. all-to-all back: O of the rank's heads -> O of every head for its token slice.

Text tokens (an optional, always-dense segment) are small; every rank holds all
of them, attends them for its heads, and the text output is all-gathered.

Layouts (P ranks, L = T*Y*X video tokens in raster order, L % P == 0, H % P == 0):
  inputs  q, k, v [B, H, L/P, D]  rank r holds tokens [r*L/P, (r+1)*L/P)
          q_text, k_text, v_text [B, H, L_text, D] (the same on every rank) or None
  outputs O [B, H, L/P, D] (same token slice), O_text [B, H, L_text, D] or None
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _heads_to_tokens(x, P, group):
    """[B, H, Lr, D] token slice of every head -> [B, H/P, P*Lr, D] all tokens of this rank's heads."""
    B, H, Lr, D = x.shape
    send = x.permute(1, 0, 2, 3).contiguous()                 # [H, B, Lr, D]: head groups contiguous
    recv = torch.empty_like(send)                             # [P (source rank), H/P, B, Lr, D]
    dist.all_to_all_single(recv, send, group=group)
    recv = recv.view(P, H // P, B, Lr, D)
    return recv.permute(2, 1, 0, 3, 4).reshape(B, H // P, P * Lr, D)


def _tokens_to_heads(y, P, group):
    """[B, H/P, L, D] all tokens of this rank's heads -> [B, H, L/P, D] every head of this token slice."""
    B, Hp, L, D = y.shape
    Lr = L // P
    send = y.view(B, Hp, P, Lr, D).permute(2, 1, 0, 3, 4).contiguous()   # [P (destination), H/P, B, Lr, D]
    recv = torch.empty_like(send)                                          # [P (source = head group), ...]
    dist.all_to_all_single(recv, send, group=group)
    return recv.view(P * Hp, B, Lr, D).permute(1, 0, 2, 3).contiguous()


def _cuda_forward(w, q, k, v, q_text, k_text, v_text):
    from . import desc_from, ssta_forward
    d = desc_from(w, H=q.shape[1])
    r = ssta_forward(d, q, k, v, q_text, k_text, v_text)
    return r["O"], r["O_text"]


def sequence_parallel_forward(w, q, k, v, q_text=None, k_text=None, v_text=None, group=None, op=None):
    """SSTA forward of a token-sharded sequence (see the module notes).

    ``w``: an object with the descriptor fields (grid T, Y, X, tiles, window, top-k,
    L_text, dtype, modes), H being the total head count.  ``op(w_local, q, k, v,
    q_text, k_text, v_text) -> (O_raster, O_text)`` runs the forward on raster
    inputs [B, H/P, T, Y, X, D]; by default the CUDA library.  Returns
    (O [B, H, L/P, D], O_text [B, H, L_text, D] or None).
    """
    P = dist.get_world_size(group)
    r = dist.get_rank(group)
    B, H, Lr, D = q.shape
    L = w.T * w.Y * w.X
    if H % P or L % P or Lr * P != L:
        raise ValueError(f"heads ({H}) and video tokens ({L}) must split evenly over {P} ranks; got {Lr} per rank")
    op = op or _cuda_forward
    hs = slice(r * (H // P), (r + 1) * (H // P))
    qh, kh, vh = (_heads_to_tokens(x, P, group).view(B, H // P, w.T, w.Y, w.X, D) for x in (q, k, v))
    th = [None if t is None else t[:, hs].contiguous() for t in (q_text, k_text, v_text)]
    w_local = _with_heads(w, H // P)
    O, O_text = op(w_local, qh, kh, vh, *th)
    O_seq = _tokens_to_heads(O.reshape(B, H // P, L, D).contiguous(), P, group)
    if O_text is None or w.L_text == 0:
        return O_seq, None
    parts = [torch.empty_like(O_text) for _ in range(P)]
    dist.all_gather(parts, O_text.contiguous(), group=group)
    return O_seq, torch.cat(parts, dim=1)


def _with_heads(w, H):
    """A copy of the descriptor-like object ``w`` with H heads."""
    if hasattr(w, "__dataclass_fields__"):
        import dataclasses
        return dataclasses.replace(w, H=H)
    c = type("W", (), {})()
    c.__dict__.update({k: getattr(w, k) for k in dir(w) if not k.startswith("_")})
    c.H = H
    return c
