"""Seeded synthetic workloads for block-causal attention forward + JVP.

This module only describes problem shapes and draws random inputs. It holds none
of the attention or JVP arithmetic, so both the CUDA path and the fp64 oracle can
take their inputs from it without sharing any of the method's code.

Shapes follow the Causal-rCM paper (arXiv 2606.25473): Wan2.1 480p video with 81
RGB frames compressed to 21 latent frames (section 4 "Models and datasets"),
frame-wise (c1-1) and chunk-wise (c3-3) causal chunking (same section), and the
teacher-forcing packed [clean | noisy] sequence (section 3.1.1, eq. 8). The token
counts per latent frame (30x52 = 1560 and 45x80 = 3600) and the head shapes are
those of the Wan2.1-1.3B-class transformer.

Value distributions: q, k, v ~ N(0, 1) (post-RMSNorm-like) and tangents
~ N(0, std_t^2). Draw order is q, k, v, tq, tk, tv from one torch CPU generator
seeded with the workload's seed, each sampled in fp32 and then cast to the run
dtype with round-to-nearest-even.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class MaskDesc:
    """Block-causal mask descriptor.

    tokens_per_frame: spatial tokens of one latent frame (T).
    frames_per_chunk: latent frames per causal chunk (1 = frame-wise, 3 = chunk-wise).
    n_frames: latent frames of one copy of the video (F).
    tf_layout: 0 = plain block-causal over F frames (N = F*T);
               1 = teacher-forcing packing [clean F frames | noisy F frames] (N = 2*F*T).
    """

    tokens_per_frame: int
    frames_per_chunk: int
    n_frames: int
    tf_layout: int

    @property
    def seq_len(self) -> int:
        return self.n_frames * self.tokens_per_frame * (2 if self.tf_layout else 1)

    def as_tuple(self):
        return (self.tokens_per_frame, self.frames_per_chunk, self.n_frames, self.tf_layout)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    D: int
    mask: MaskDesc
    dtype: torch.dtype
    seed: int
    std_qkv: float = 1.0
    std_tangent: float = 1.0
    scale: Optional[float] = None  # None -> 1/sqrt(D)

    @property
    def N(self) -> int:
        return self.mask.seq_len

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else self.D ** -0.5


# The five workloads. C0 is the small case the oracle finishes in full; C2 is the
# teacher-forcing frame-wise layout that throughput is quoted on.
WORKLOADS = {
    "tiny_framewise_fp32": Workload(
        "tiny_framewise_fp32", 1, 2, 64, MaskDesc(16, 1, 4, 0), torch.float32, 0, 1.0, 1.0),
    "wan1.3b_framewise_infer": Workload(
        "wan1.3b_framewise_infer", 1, 12, 128, MaskDesc(1560, 1, 21, 0), torch.bfloat16, 1, 1.0, 0.5),
    "wan1.3b_tf_framewise": Workload(
        "wan1.3b_tf_framewise", 1, 12, 128, MaskDesc(1560, 1, 21, 1), torch.bfloat16, 2, 1.0, 0.5),
    "wan1.3b_tf_chunkwise": Workload(
        "wan1.3b_tf_chunkwise", 2, 12, 128, MaskDesc(1560, 3, 21, 1), torch.bfloat16, 3, 1.0, 1.0),
    "h40_framewise_infer": Workload(
        "h40_framewise_infer", 1, 40, 128, MaskDesc(3600, 1, 21, 0), torch.bfloat16, 4, 1.0, 0.5),
}

WORKLOAD_ORDER = list(WORKLOADS)
BENCH_WORKLOAD = "wan1.3b_tf_framewise"


def with_dtype(w: Workload, dtype: torch.dtype) -> Workload:
    return dataclasses.replace(w, dtype=dtype, name=f"{w.name}[{str(dtype).split('.')[-1]}]")


def small(name: str, B: int, H: int, D: int, mask: MaskDesc, dtype=torch.bfloat16, seed: int = 0,
          std_qkv: float = 1.0, std_tangent: float = 1.0) -> Workload:
    return Workload(name, B, H, D, mask, dtype, seed, std_qkv, std_tangent)


def make_inputs(w: Workload, device="cpu"):
    """Draw (q, k, v, tq, tk, tv), each [B, H, N, D] contiguous in w.dtype.

    Sampling happens on the CPU generator (so every consumer sees identical
    values), then the tensors move to `device`.
    """
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    shape = (w.B, w.H, w.N, w.D)
    out = []
    for i in range(6):
        std = w.std_qkv if i < 3 else w.std_tangent
        t = torch.randn(shape, generator=g, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        t = t.to(w.dtype)
        out.append(t.to(device) if device != "cpu" else t)
    return tuple(out)


def zero_clean_tangents(w: Workload, tq, tk, tv):
    """Teacher-forcing sCM inputs: the clean context (rows < L) has zero tangent.
    Zeroes those rows of tq, tk, tv in place and returns them."""
    if not w.mask.tf_layout:
        raise ValueError("clean tangents exist only in the teacher-forcing layout")
    L = w.mask.n_frames * w.mask.tokens_per_frame
    for t in (tq, tk, tv):
        t[:, :, :L] = 0
    return tq, tk, tv


def sample_rows(w: Workload, rows_per_head: int, seed_offset: int = 0):
    """Seeded query rows to check per (b, h): `rows_per_head` rows drawn without
    replacement from [0, N) by a generator seeded from (seed, b, h). Returns an
    int64 tensor of flat row ids bh * N + i, sorted."""
    ids = []
    n = w.N
    k = min(rows_per_head, n)
    for b in range(w.B):
        for h in range(w.H):
            g = torch.Generator(device="cpu").manual_seed(
                (w.seed * 1_000_003 + b * 1009 + h * 7 + seed_offset) & 0x7FFFFFFF)
            r = torch.randperm(n, generator=g)[:k]
            ids.append((b * w.H + h) * n + torch.sort(r).values)
    return torch.cat(ids).to(torch.int64)


def boundary_rows(w: Workload):
    """First and last row of every chunk (and the clean/noisy seam), for every
    (b, h). Flat row ids, sorted and unique."""
    m = w.mask
    G = m.frames_per_chunk * m.tokens_per_frame
    L = m.n_frames * m.tokens_per_frame
    starts = list(range(0, L, G))
    if m.tf_layout:
        starts += [L + s for s in range(0, L, G)]
    rows = set()
    for s in starts:
        rows.update([s, s + G - 1])
    rows = sorted(r for r in rows if 0 <= r < w.N)
    rows_t = torch.tensor(rows, dtype=torch.int64)
    ids = [bh * w.N + rows_t for bh in range(w.B * w.H)]
    return torch.cat(ids)
