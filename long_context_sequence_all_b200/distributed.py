"""Ulysses over real ranks: one process per GPU, torch.distributed for the
exchange ("Ulysses 序列平行化：突破百萬標記長上下文的訓練瓶頸", section
"Ulysses 序列平行化的原理", and "Paralelismul de Secvență Ulysses", section
"Mecanismul de funcționare Ulysses", steps 3 and 5).

Rank r of a group of P holds the positions [r*s, (r+1)*s) (s = n/P) of every
head: x_r [B][s][heads][d].  The first all-to-all gives it all n positions of
its heads [r*hl, (r+1)*hl) (hl = heads/P): [B][hl][n][d]; the second undoes it.

Each all-to-all is a group of point-to-point transfers of contiguous slabs of
s*d elements, one per (peer, batch row, local head):
  seq -> head: the local shard is first packed to [B][heads][s][d] (the
    library's seq->head permutation with a single rank), so the slab for peer
    p and head h = p*hl + hh is send[b][h]; the slab from peer p lands directly
    at out[b][hh][p*s:(p+1)*s] -- the receive writes the head layout.
  head -> seq: the slab y[b][hh][p*s:(p+1)*s] goes to peer p; the slab from
    peer p lands at recv[b][p*hl + hh]; recv [B][heads][s][d] is unpacked to
    [B][s][heads][d] (the single-rank head->seq permutation).
The slab a rank keeps is copied locally.  Per rank (P-1)/P of the tensor
crosses the interconnect each way (the pages' O(n d / P) per device).  On GPUs
the group is NCCL (grouped send/recv, no TMA or multicast involved) and the
pack, unpack and attention steps run the library's kernels; the bookkeeping
of the exchange is tested with gloo ranks on the CPU, where the tests pass
the oracle's routines as those steps.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _pack_cuda(x):
    from . import ulysses as U
    return U.ulysses_seq_to_head(x.unsqueeze(0), 1)[0]          # [B][s][H][d] -> [B][H][s][d]


def _unpack_cuda(t):
    from . import ulysses as U
    return U.ulysses_head_to_seq(t.unsqueeze(0), 1)[0]          # [B][H][s][d] -> [B][s][H][d]


def _peer(group, p):
    return p if group is None else dist.get_global_rank(group, p)


def _exchange(pairs, group, P, me):
    """pairs: (peer, send slab, receive slab) in the order both sides agree on."""
    ops = []
    for p, snd, rcv in pairs:
        if p == me:
            rcv.copy_(snd)
            continue
        ops.append(dist.P2POp(dist.isend, snd, _peer(group, p), group))
        ops.append(dist.P2POp(dist.irecv, rcv, _peer(group, p), group))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()


def seq_to_head(x, group=None, out=None, pack=None):
    """This rank's shard x [B][s][heads][d] -> its heads over the whole
    sequence [B][heads/P][n][d] (the first all-to-all)."""
    P, me = dist.get_world_size(group), dist.get_rank(group)
    B, s, heads, d = x.shape
    if heads % P:
        raise ValueError(f"{heads} heads over {P} ranks")
    hl, n = heads // P, P * s
    send = (pack or _pack_cuda)(x.contiguous())                 # [B][heads][s][d]
    out = torch.empty((B, hl, n, d), dtype=x.dtype, device=x.device) if out is None else out
    pairs = [(p, send[b, p * hl + hh], out[b, hh, p * s:(p + 1) * s])
             for p in range(P) for b in range(B) for hh in range(hl)]
    _exchange(pairs, group, P, me)
    return out


def head_to_seq(y, group=None, unpack=None):
    """This rank's heads over the whole sequence y [B][hl][n][d] -> its shard
    of every head [B][s][hl*P][d] (the second all-to-all)."""
    P, me = dist.get_world_size(group), dist.get_rank(group)
    B, hl, n, d = y.shape
    if n % P:
        raise ValueError(f"{n} positions over {P} ranks")
    s, heads = n // P, hl * P
    recv = torch.empty((B, heads, s, d), dtype=y.dtype, device=y.device)
    pairs = [(p, y[b, hh, p * s:(p + 1) * s], recv[b, p * hl + hh])
             for p in range(P) for b in range(B) for hh in range(hl)]
    _exchange(pairs, group, P, me)
    return (unpack or _unpack_cuda)(recv)


def _attn_cuda(qh, kh, vh, mask, cu_seqlens, scale):
    from . import ulysses as U
    o, lse = U.ulysses_attn_fwd(qh.unsqueeze(0), kh.unsqueeze(0), vh.unsqueeze(0), mask=mask,
                                cu_seqlens=cu_seqlens, scale=scale)
    return o[0], lse[0]


def attention(q, k, v, group=None, mask=1, cu_seqlens=None, scale=0.0, attn=None, pack=None, unpack=None):
    """The Ulysses attention layer on this rank: q [B][s][H][d], k, v
    [B][s][G][d] (its positions of every head; G % P == 0) -> O [B][s][H][d]
    and this rank's LSE [B][H/P][n].  Step 4 runs on the rank's heads with the
    library's attention (one rank's head layout)."""
    qh = seq_to_head(q, group, pack=pack)
    kh = seq_to_head(k, group, pack=pack)
    vh = seq_to_head(v, group, pack=pack)
    oh, lse = (attn or _attn_cuda)(qh, kh, vh, mask, cu_seqlens, scale)
    return head_to_seq(oh, group, unpack=unpack), lse


def aggregate_loss(shard_sum, shard_count, group=None):
    """The token-weighted loss over ranks ("Paralelismul de Secvență Ulysses",
    section "Integrarea cu Accelerate"): every rank contributes its sum of
    token losses S_r and its count of valid tokens C_r; L = sum S_r / sum C_r
    (one all-reduce of two numbers).  Returns (L, sum C) as Python numbers."""
    t = torch.tensor([float(shard_sum), float(shard_count)], dtype=torch.float64,
                     device=shard_sum.device if torch.is_tensor(shard_sum) else "cpu")
    dist.all_reduce(t, group=group)
    total_c = t[1].item()
    return (t[0].item() / total_c if total_c else float("nan")), int(total_c)
