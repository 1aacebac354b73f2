"""Seeded synthetic inputs for the Ulysses attention layer.

This module only draws random numbers and arranges them in the layouts the
library takes; it holds none of the method's arithmetic.  Both the CUDA path
and the CPU oracle are fed from it, so the two always see identical inputs.

Workloads (shapes from the pages' settings: a Qwen3-4B-shaped attention layer
-- 32 query heads, 8 KV heads, head_dim 128 -- at 8K and 64K with 4 ranks,
packed variable-length documents padded to a multiple of the rank count, and
a 256K context with 8 ranks):

  tiny_f32    B=1 n=1024   P=4 H=8  G=8 d=64  fp32, Q/K/V ~ N(0,1), fwd only
  qwen8k      B=1 n=8192   P=4 H=32 G=8 d=128 bf16 causal, Q/K/V ~ N(0,1)/sqrt(128), dO ~ N(0,1)
  qwen64k     B=1 n=65536  P=4 H=32 G=8 d=128 bf16 causal + CE loss, V=8192
  packed      16 docs, lengths U{512..8192}, padded to a multiple of P=8,
              doc-causal mask, H=32 G=8 d=128 bf16, 20% labels ignored, V=8192
  long256k    B=1 n=262144 P=8 H=32 G=8 d=128 bf16 causal

Draws: torch.Generator (CPU) seeded with 1000 + workload index; values drawn
in fp32 and rounded to bf16 (round-to-nearest-even) for the bf16 workloads.
Sequence-sharded tensors are laid out [P][B][n/P][heads][d]; with B=1 this is
the natural [n][heads][d] order (rank r holds rows [r*n/P, (r+1)*n/P)).
"""
from __future__ import annotations

import dataclasses
import math

import torch

IGNORE_INDEX = -100


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    B: int
    n: int            # sequence length (packed: filled in per draw, see make_packed_lengths)
    P: int
    H: int
    G: int
    d: int
    dtype: str        # "f32" or "bf16"
    mask: int         # 0 none, 1 causal, 2 doc-causal
    backward: bool
    vocab: int = 0    # > 0: the workload includes the loss
    qkv_std: float = 1.0
    label_mask_frac: float = 0.0
    num_docs: int = 0
    doc_len_range: tuple = (0, 0)


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_f32", 0, 1, 1024, 4, 8, 8, 64, "f32", 1, False),
        Workload("qwen8k", 1, 1, 8192, 4, 32, 8, 128, "bf16", 1, True, qkv_std=1 / math.sqrt(128)),
        Workload("qwen64k", 2, 1, 65536, 4, 32, 8, 128, "bf16", 1, True, vocab=8192,
                 qkv_std=1 / math.sqrt(128)),
        Workload("packed", 3, 1, 0, 8, 32, 8, 128, "bf16", 2, True, vocab=8192,
                 qkv_std=1 / math.sqrt(128), label_mask_frac=0.2, num_docs=16,
                 doc_len_range=(512, 8192)),
        Workload("long256k", 4, 1, 262144, 8, 32, 8, 128, "bf16", 1, True,
                 qkv_std=1 / math.sqrt(128)),
    ]
}


def generator(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def make_packed_lengths(num_docs: int, lo: int, hi: int, P: int, g: torch.Generator):
    """Document lengths uniform in [lo, hi] (inclusive); the total is padded up
    to a multiple of P and the pad forms its own final segment.
    Returns (cu_seqlens int32 [num_segments+1], n, real_tokens)."""
    lens = torch.randint(lo, hi + 1, (num_docs,), generator=g, dtype=torch.int64)
    total = int(lens.sum())
    n = ((total + P - 1) // P) * P
    cu = [0]
    for L in lens.tolist():
        cu.append(cu[-1] + L)
    if n > total:
        cu.append(n)
    return torch.tensor(cu, dtype=torch.int32), n, total


def _draw(shape, std, dtype, g):
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16) if dtype == "bf16" else x


def make_inputs(w: Workload | str, seed: int | None = None, n_override: int | None = None,
                with_grad_inputs: bool = True, with_loss: bool = True):
    """Draw one batch of the workload.  Returns a dict of CPU tensors:
    q [P][B][s][H][d], k, v [P][B][s][G][d], (do [P][B][s][H][d]),
    (logits [P][B*s][V] bf16, labels int32 [P][B*s]), cu_seqlens (doc-causal),
    and the shape fields.  n_override shrinks n (parity cases at small sizes)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    g = generator(1000 + w.index if seed is None else seed)
    cu = None
    real = None
    if w.mask == 2:
        cu, n, real = make_packed_lengths(w.num_docs, *w.doc_len_range, w.P, g)
    else:
        n = n_override or w.n
    assert n % w.P == 0
    s = n // w.P
    out = dict(workload=w, B=w.B, n=n, P=w.P, H=w.H, G=w.G, d=w.d, mask=w.mask,
               cu_seqlens=cu, real_tokens=real if real is not None else n)
    out["q"] = _draw((w.P, w.B, s, w.H, w.d), w.qkv_std, w.dtype, g)
    out["k"] = _draw((w.P, w.B, s, w.G, w.d), w.qkv_std, w.dtype, g)
    out["v"] = _draw((w.P, w.B, s, w.G, w.d), w.qkv_std, w.dtype, g)
    if w.backward and with_grad_inputs:
        out["do"] = _draw((w.P, w.B, s, w.H, w.d), 1.0, w.dtype, g)
    if w.vocab and with_loss:
        T = w.B * n
        out["logits"] = _draw((T, w.vocab), 1.0, "bf16", g)
        labels = torch.randint(0, w.vocab, (T,), generator=g, dtype=torch.int32)
        if w.label_mask_frac > 0:
            drop = torch.rand((T,), generator=g) < w.label_mask_frac
            labels[drop] = IGNORE_INDEX
        if real is not None and real < T:
            labels[real:] = IGNORE_INDEX
        out["labels"] = labels
        out["vocab"] = w.vocab
    return out


def to_natural(x_seq: torch.Tensor) -> torch.Tensor:
    """[P][B][s][heads][d] -> [B][n][heads][d] (undo the rank-major stacking)."""
    P, B, s, Hx, d = x_seq.shape
    return x_seq.permute(1, 0, 2, 3, 4).reshape(B, P * s, Hx, d)


def to_seq(x_nat: torch.Tensor, P: int) -> torch.Tensor:
    """[B][n][heads][d] -> [P][B][n/P][heads][d] (rank r takes rows [r*n/P, (r+1)*n/P))."""
    B, n, Hx, d = x_nat.shape
    return x_nat.reshape(B, P, n // P, Hx, d).permute(1, 0, 2, 3, 4).contiguous()
