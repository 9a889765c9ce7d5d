"""Seeded synthetic workloads for the SSTA forward path.

This module is shared by the tests, the benchmark and the smoke check.  It
holds only workload definitions (shapes, tile/window/top-k parameters as
literal numbers) and a counter-based random generator; none of the attention
method's arithmetic lives here.  Both the CUDA path and the CPU oracle consume
the tensors it returns, so the two sides see identical inputs.

Generator: splitmix64 used as a counter-based generator (Steele, Lea & Flood,
"Fast splittable pseudorandom number generators", OOPSLA 2014; the mixing
constants are those of Vigna's public-domain splitmix64).  Output ``i`` of a
stream with key ``K`` is ``mix64(K + (i + 1) * 0x9E3779B97F4A7C15)``, so any
element can be regenerated on its own and any head subset of a tensor equals
the same heads of the full tensor.  Normals come from Box-Muller on two 24-bit
uniforms taken from one 64-bit draw.

Value recipes (the workload descriptions of the video latents):
* ``tile_offset``: q, k, v i.i.d. N(0,1); one offset vector per (batch, head,
  3D tile) drawn N(0, 0.5^2) and added to both q and k of every token of that
  tile, so tile-level scores are far from flat.
* ``smooth_field``: N(0,1) plus, per (tensor, head, channel), a smooth 3D field
  that is a sum of four terms 0.5*cos(2*pi*(ft*t/T + fy*y/Y + fx*x/X) + phi),
  with integer frequencies ft, fy, fx uniform in {0,1,2} and phi uniform in
  [0, 2*pi); the field is evaluated on the valid (unpadded) grid.  Text tokens
  are N(0,1).  The result is cast to the workload dtype (bf16) last.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

__all__ = [
    "Workload", "WORKLOADS", "get_workload", "make_inputs", "counter_bits",
    "counter_normals", "mix64_int",
]

# ---------------------------------------------------------------------------
# Workloads.  Grids follow the causal video VAE's 16x spatial / 4x temporal
# compression of 480p/720p clips of 121 and 241 frames (4n+1 frames -> n+1
# latent frames).  Top-k is stored as an absolute tile count; the percentage it
# was derived from (ceil(fraction * number_of_video_tiles)) is kept in the note.
# ---------------------------------------------------------------------------


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str                 # "f32" or "bf16": storage / arithmetic type
    B: int
    H: int
    D: int
    T: int                     # valid latent grid (frames, height, width)
    Y: int
    X: int
    tT: int                    # tile extent per axis, in tokens
    tY: int
    tX: int
    wT: int                    # sliding window per axis, in tiles (odd, centred)
    wY: int
    wX: int
    topk: int                  # selected tiles per query tile (absolute)
    L_text: int                # appended always-dense text tokens (0 = none)
    recipe: str                # "tile_offset" or "smooth_field"
    seeds: tuple = (0,)
    note: str = ""
    extra: dict = field(default_factory=dict)
    # mask modes (defaults: the headline configuration)
    score_mode: str = "similarity"   # or "importance"
    lam: float = 0.9                 # importance weight of the similarity term
    combine: str = "union"           # or "and"
    window_mode: str = "shift"       # or "truncate"

    @property
    def tokens(self) -> int:
        return self.T * self.Y * self.X


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_f32", "f32", 1, 2, 128, 4, 8, 8, 2, 4, 4, 1, 1, 1, 2, 0,
                 "tile_offset", (0,), "256 tokens, 8 tiles of 32"),
        Workload("small_bf16", "bf16", 1, 16, 128, 16, 32, 56, 4, 8, 8, 3, 3, 3, 8, 0,
                 "smooth_field", (0,), "28,672 tokens, 112 tiles of 256"),
        Workload("p480_5s_bf16", "bf16", 1, 16, 128, 31, 30, 53, 4, 8, 8, 3, 3, 3, 34, 0,
                 "smooth_field", (0,),
                 "49,290 tokens padded to 32x32x56 (224 tiles); top-k = ceil(15% of 224)"),
        Workload("p720_5s_bf16", "bf16", 1, 16, 128, 31, 45, 80, 4, 8, 8, 3, 3, 5, 48, 256,
                 "smooth_field", (0,),
                 "111,600 tokens padded to 32x48x80 (480 tiles); top-k = 10% of 480; 256 text tokens"),
        Workload("p720_10s_bf16", "bf16", 1, 16, 128, 61, 45, 80, 4, 8, 8, 3, 3, 5, 77, 256,
                 "smooth_field", (0, 1, 2),
                 "219,600 tokens padded to 64x48x80 (960 tiles); top-k = ceil(8% of 960); 256 text tokens"),
    ]
}


def get_workload(name: str) -> Workload:
    return WORKLOADS[name]


# ---------------------------------------------------------------------------
# Counter-based splitmix64 on int64 tensors (two's complement wrap-around).
# ---------------------------------------------------------------------------
_MASK64 = (1 << 64) - 1
_GOLDEN = 0x9E3779B97F4A7C15
_C1 = 0xBF58476D1CE4E5B9
_C2 = 0x94D049BB133111EB


def _signed(c: int) -> int:
    c &= _MASK64
    return c - (1 << 64) if c >= (1 << 63) else c


def mix64_int(z: int) -> int:
    """splitmix64 finaliser on a Python int (exact modulo 2^64)."""
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _C1) & _MASK64
    z = ((z ^ (z >> 27)) * _C2) & _MASK64
    return z ^ (z >> 31)


def _srl(x: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of an int64 tensor."""
    return (x >> s) & ((1 << (64 - s)) - 1)


def _mix64(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _srl(z, 30)) * _signed(_C1)
    z = (z ^ _srl(z, 27)) * _signed(_C2)
    return z ^ _srl(z, 31)


def _stream_key(seed: int, stream: int) -> int:
    return mix64_int((seed & 0xFFFFFFFF) * 0x100000001B3 + stream * 0x5851F42D4C957F2D + 0x2545F4914F6CDD1D)


def counter_bits(seed: int, stream: int, idx: torch.Tensor) -> torch.Tensor:
    """64 random bits (as int64) for counters ``idx`` of stream ``(seed, stream)``."""
    key = _stream_key(seed, stream)
    z = _signed(key) + (idx + 1) * _signed(_GOLDEN)
    return _mix64(z)


def _uniform24(bits: torch.Tensor, shift: int) -> torch.Tensor:
    return (_srl(bits, shift) & 0xFFFFFF).to(torch.float32) * (1.0 / 16777216.0)


def counter_normals(seed: int, stream: int, idx: torch.Tensor) -> torch.Tensor:
    """Standard normals (float32) for counters ``idx`` via Box-Muller."""
    bits = counter_bits(seed, stream, idx)
    u1 = 1.0 - _uniform24(bits, 40)          # (0, 1]
    u2 = _uniform24(bits, 16)                # [0, 1)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


# Stream ids.
_S_NOISE = {"q": 1, "k": 2, "v": 3}
_S_TEXT = {"q": 4, "k": 5, "v": 6}
_S_FIELD = 7
_S_OFFSET = 8
_TENSOR_ID = {"q": 0, "k": 1, "v": 2}


def _raster_noise(w: Workload, seed: int, which: str, h: int, device) -> torch.Tensor:
    """N(0,1) for all (b, t, y, x, d) of head ``h``: shape [B, T, Y, X, D]."""
    per_head = w.T * w.Y * w.X * w.D
    out = torch.empty((w.B, w.T, w.Y, w.X, w.D), dtype=torch.float32, device=device)
    for b in range(w.B):
        base = (b * w.H + h) * per_head
        idx = torch.arange(base, base + per_head, dtype=torch.int64, device=device)
        out[b] = counter_normals(seed, _S_NOISE[which], idx).view(w.T, w.Y, w.X, w.D)
    return out


def _smooth_field(w: Workload, seed: int, which: str, h: int, device) -> torch.Tensor:
    """Smooth 3D field for head ``h``: shape [T, Y, X, D] (float32)."""
    D = w.D
    cidx = (( _TENSOR_ID[which] * w.H + h) * D + torch.arange(D, device=device, dtype=torch.int64)) * 4
    cidx = cidx[:, None] + torch.arange(4, device=device, dtype=torch.int64)[None, :]     # [D, 4]
    fbits = counter_bits(seed, _S_FIELD, 2 * cidx)
    pbits = counter_bits(seed, _S_FIELD, 2 * cidx + 1)
    ft = (_srl(fbits, 40) % 3).to(torch.float32)
    fy = (_srl(fbits, 20) % 3).to(torch.float32)
    fx = (fbits & 0xFFFFF) % 3
    fx = fx.to(torch.float32)
    phi = (2.0 * math.pi) * _uniform24(pbits, 40)
    t = torch.arange(w.T, device=device, dtype=torch.float32) / w.T
    y = torch.arange(w.Y, device=device, dtype=torch.float32) / w.Y
    x = torch.arange(w.X, device=device, dtype=torch.float32) / w.X
    out = torch.zeros((w.T, w.Y, w.X, D), dtype=torch.float32, device=device)
    for m in range(4):
        ph = (t[:, None, None, None] * ft[None, None, None, :, m]
              + y[None, :, None, None] * fy[None, None, None, :, m]
              + x[None, None, :, None] * fx[None, None, None, :, m])
        out += 0.5 * torch.cos((2.0 * math.pi) * ph + phi[None, None, None, :, m])
    return out


def _tile_offsets(w: Workload, seed: int, h: int, device) -> torch.Tensor:
    """Per-(batch, tile) offset vectors for head ``h``, broadcast to tokens: [B, T, Y, X, D]."""
    nT = -(-w.T // w.tT)
    nY = -(-w.Y // w.tY)
    nX = -(-w.X // w.tX)
    ntiles = nT * nY * nX
    out = torch.empty((w.B, w.T, w.Y, w.X, w.D), dtype=torch.float32, device=device)
    t = torch.arange(w.T, device=device) // w.tT
    y = torch.arange(w.Y, device=device) // w.tY
    x = torch.arange(w.X, device=device) // w.tX
    tile_of = (t[:, None, None] * nY + y[None, :, None]) * nX + x[None, None, :]    # [T, Y, X]
    for b in range(w.B):
        base = (b * w.H + h) * ntiles * w.D
        idx = torch.arange(base, base + ntiles * w.D, dtype=torch.int64, device=device)
        off = 0.5 * counter_normals(seed, _S_OFFSET, idx).view(ntiles, w.D)
        out[b] = off[tile_of]
    return out


def _torch_dtype(w: Workload):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[w.dtype]


def make_inputs(w: Workload, seed: int = 0, device="cpu", heads=None) -> dict:
    """Generate q, k, v in raster layout [B, H', T, Y, X, D] plus text [B, H', L_text, D].

    ``heads`` selects a subset of heads (default: all); element values do not
    depend on which other heads are generated.
    """
    heads = list(range(w.H)) if heads is None else list(heads)
    dt = _torch_dtype(w)
    out = {}
    for which in ("q", "k", "v"):
        t = torch.empty((w.B, len(heads), w.T, w.Y, w.X, w.D), dtype=dt, device=device)
        for hi, h in enumerate(heads):
            val = _raster_noise(w, seed, which, h, device)
            if w.recipe == "smooth_field":
                val += _smooth_field(w, seed, which, h, device)[None]
            elif w.recipe == "tile_offset":
                if which in ("q", "k"):
                    val += _tile_offsets(w, seed, h, device)
            else:
                raise ValueError(w.recipe)
            t[:, hi] = val.to(dt)
        out[which] = t
    for which in ("q", "k", "v"):
        if w.L_text > 0:
            t = torch.empty((w.B, len(heads), w.L_text, w.D), dtype=dt, device=device)
            per_head = w.L_text * w.D
            for b in range(w.B):
                for hi, h in enumerate(heads):
                    base = (b * w.H + h) * per_head
                    idx = torch.arange(base, base + per_head, dtype=torch.int64, device=device)
                    t[b, hi] = counter_normals(seed, _S_TEXT[which], idx).view(w.L_text, w.D).to(dt)
            out[which + "_text"] = t
        else:
            out[which + "_text"] = None
    return out


def with_overrides(w: Workload, **kw) -> Workload:
    """A copy of ``w`` with some fields replaced (edge-case variants in tests)."""
    d = dict(w.__dict__)
    d.update(kw)
    return Workload(**d)
