"""The two bf16 backward paths and the fused second all-to-all.

- The fused backward (one pass, dQ summed with fp32 adds in L2) and the
  deterministic one (two passes, no atomics) both match the fp64 oracle; their
  dK and dV are bitwise equal (same products in the same order), their dQ
  agree to the bf16 rounding of two fp32 sums.
- out_seq_layout = 1 (the head->seq all-to-all done in the producing kernel's
  epilogue) gives bitwise the head-layout result permuted by
  ulysses_head_to_seq, for O and, on the deterministic path, dQ, dK, dV; the
  backward then reads O in the seq layout.
- The deterministic path is bitwise repeatable; the fused path's dK, dV are.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_bf16_close, f32_inputs
from long_context_sequence_all_b200 import ulysses as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    U.lib()
    U.ulysses_read_error()


def _case(n, P, H, G, seed, std=128 ** -0.5, d=128):
    g = torch.Generator().manual_seed(seed)
    s = n // P
    mk = lambda h, sd: (torch.randn(P, 1, s, h, d, generator=g) * sd).to(torch.bfloat16)
    return mk(H, std), mk(G, std), mk(G, std), mk(H, 1.0)


CASES = [
    (512, 2, 8, 2, U.MASK_CAUSAL, None),
    (424, 2, 8, 2, U.MASK_CAUSAL, None),        # ragged last tile
    (392, 4, 8, 4, U.MASK_NONE, None),
    (1000, 8, 16, 8, U.MASK_DOC_CAUSAL, [0, 100, 129, 400, 401, 777, 1000]),
    (8, 8, 16, 8, U.MASK_CAUSAL, None),         # one token per rank
    (424, 4, 4, 4, U.MASK_CAUSAL, None),        # MHA (G = H)
    (424, 2, 6, 2, U.MASK_CAUSAL, None),        # an odd group (3 query heads per KV head)
]


def _heads(q, k, v, do, P):
    return [U.ulysses_seq_to_head(x.cuda(), P) for x in (q, k, v, do)]


@pytest.mark.parametrize("n,P,H,G,mask,cu", CASES)
@pytest.mark.parametrize("deterministic", [False, True])
def test_both_backward_paths_match_the_oracle(n, P, H, G, mask, cu, deterministic):
    q, k, v, do = _case(n, P, H, G, seed=n + 7)
    cut = None if cu is None else torch.tensor(cu, dtype=torch.int32)
    cud = None if cut is None else cut.cuda()
    qh, kh, vh, doh = _heads(q, k, v, do, P)
    oh, lse = U.ulysses_attn_fwd(qh, kh, vh, mask=mask, cu_seqlens=cud)
    grads = U.ulysses_attn_bwd(qh, kh, vh, oh, lse, doh, mask=mask, cu_seqlens=cud, deterministic=deterministic)
    ref = oracle.ulysses_bwd(f32_inputs(q), f32_inputs(k), f32_inputs(v), f32_inputs(do), P, mask=mask,
                             cu_seqlens=None if cut is None else cut.numpy())
    for name, got, want in zip(("dQ", "dK", "dV"), grads, ref):
        assert_bf16_close(U.ulysses_head_to_seq(got, P).cpu(), want, f"{name} deterministic={deterministic}")
    assert U.ulysses_read_error() == 0


@pytest.mark.parametrize("n,P,H,G,mask,cu", CASES[:4])
def test_fused_and_deterministic_paths_agree(n, P, H, G, mask, cu):
    q, k, v, do = _case(n, P, H, G, seed=n + 11)
    cud = None if cu is None else torch.tensor(cu, dtype=torch.int32).cuda()
    qh, kh, vh, doh = _heads(q, k, v, do, P)
    oh, lse = U.ulysses_attn_fwd(qh, kh, vh, mask=mask, cu_seqlens=cud)
    f = U.ulysses_attn_bwd(qh, kh, vh, oh, lse, doh, mask=mask, cu_seqlens=cud)
    dt = U.ulysses_attn_bwd(qh, kh, vh, oh, lse, doh, mask=mask, cu_seqlens=cud, deterministic=True)
    torch.cuda.synchronize()
    assert torch.equal(f[1], dt[1]) and torch.equal(f[2], dt[2]), "dK / dV differ between the paths"
    a, b = f[0].float().cpu(), dt[0].float().cpu()
    # two fp32 sums of the same products, each rounded once to bf16
    assert float(((a - b).abs() / (2.0 ** -7 * torch.maximum(a.abs(), b.abs()) + 1e-6)).max()) <= 1.0
    assert U.ulysses_read_error() == 0


@pytest.mark.parametrize("n,P,H,G,mask,cu", CASES)
def test_seq_layout_epilogues_equal_the_separate_permutation(n, P, H, G, mask, cu):
    q, k, v, do = _case(n, P, H, G, seed=n + 13)
    cud = None if cu is None else torch.tensor(cu, dtype=torch.int32).cuda()
    qh, kh, vh, doh = _heads(q, k, v, do, P)
    oh, lse = U.ulysses_attn_fwd(qh, kh, vh, mask=mask, cu_seqlens=cud)
    os_, lse_s = U.ulysses_attn_fwd(qh, kh, vh, mask=mask, cu_seqlens=cud, out_seq_layout=True)
    torch.cuda.synchronize()
    assert os_.shape == (P, 1, n // P, H, 128)
    assert torch.equal(os_, U.ulysses_head_to_seq(oh, P)) and torch.equal(lse_s, lse)
    # deterministic backward: every output bitwise; O read in the seq layout
    ref = U.ulysses_attn_bwd(qh, kh, vh, oh, lse, doh, mask=mask, cu_seqlens=cud, deterministic=True)
    got = U.ulysses_attn_bwd(qh, kh, vh, os_, lse, doh, mask=mask, cu_seqlens=cud, deterministic=True,
                             out_seq_layout=True)
    torch.cuda.synchronize()
    for name, a, b in zip(("dQ", "dK", "dV"), got, ref):
        assert torch.equal(a, U.ulysses_head_to_seq(b, P)), name
    # fused backward: dK, dV bitwise; dQ to one bf16 rounding of its fp32 sum
    fz = U.ulysses_attn_bwd(qh, kh, vh, os_, lse, doh, mask=mask, cu_seqlens=cud, out_seq_layout=True)
    torch.cuda.synchronize()
    assert torch.equal(fz[1], U.ulysses_head_to_seq(ref[1], P)) and torch.equal(fz[2], U.ulysses_head_to_seq(ref[2], P))
    a, b = fz[0].float().cpu(), U.ulysses_head_to_seq(ref[0], P).float().cpu()
    assert float(((a - b).abs() / (2.0 ** -7 * torch.maximum(a.abs(), b.abs()) + 1e-6)).max()) <= 1.0
    assert U.ulysses_read_error() == 0


def test_repeatability():
    n, P, H, G = 1024, 4, 16, 4
    q, k, v, do = _case(n, P, H, G, seed=3)
    qh, kh, vh, doh = _heads(q, k, v, do, P)
    oh, lse = U.ulysses_attn_fwd(qh, kh, vh)
    d1 = U.ulysses_attn_bwd(qh, kh, vh, oh, lse, doh, deterministic=True)
    d2 = U.ulysses_attn_bwd(qh, kh, vh, oh, lse, doh, deterministic=True)
    f1 = U.ulysses_attn_bwd(qh, kh, vh, oh, lse, doh)
    f2 = U.ulysses_attn_bwd(qh, kh, vh, oh, lse, doh)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(d1, d2))
    assert torch.equal(f1[1], f2[1]) and torch.equal(f1[2], f2[2])
    assert U.ulysses_read_error() == 0


def test_malformed_cu_seqlens_sets_shape_error():
    """A cu_seqlens that does not end at n is flagged in the error word (the
    kernels clamp document bounds to the sequence and stay in bounds)."""
    n, P, H, G = 256, 2, 4, 2
    q, k, v, do = _case(n, P, H, G, seed=5)
    qh, kh, vh, doh = _heads(q, k, v, do, P)
    U.ulysses_read_error()
    for bad in ([0, 100, 200], [0, 150, 100, 256], [5, 100, 256]):
        cu = torch.tensor(bad, dtype=torch.int32, device="cuda")
        oh, lse = U.ulysses_attn_fwd(qh, kh, vh, mask=U.MASK_DOC_CAUSAL, cu_seqlens=cu)
        torch.cuda.synchronize()
        assert U.ulysses_read_error() == (1 << 2), bad
        U.ulysses_attn_bwd(qh, kh, vh, oh, lse, doh, mask=U.MASK_DOC_CAUSAL, cu_seqlens=cu)
        torch.cuda.synchronize()
        assert U.ulysses_read_error() == (1 << 2), bad
    good = torch.tensor([0, 100, 256], dtype=torch.int32, device="cuda")
    U.ulysses_attn_fwd(qh, kh, vh, mask=U.MASK_DOC_CAUSAL, cu_seqlens=good)
    assert U.ulysses_read_error() == 0


@pytest.mark.parametrize("n,P,H,G,mask,cu", [
    (4096, 4, 32, 8, U.MASK_CAUSAL, None),      # 32 query tiles, 8 KV heads: several waves either way
    (1000, 8, 16, 8, U.MASK_DOC_CAUSAL, [0, 100, 129, 400, 401, 777, 1000]),
    (392, 4, 8, 4, U.MASK_NONE, None),
    (424, 2, 6, 2, U.MASK_CAUSAL, None),        # an odd group: one query head per forward CTA
])
def test_block_orders_give_the_same_results(n, P, H, G, mask, cu):
    """The attention kernels start their CTAs one KV head at a time (long
    sequences) or with the heaviest tiles of every head first (short ones,
    document masks); the order is scheduling only.  With each order forced:
    O, LSE, dK, dV and the deterministic dQ are bitwise equal, the fused dQ
    (fp32 adds meeting in L2 in run-dependent order) to one bf16 rounding."""
    q, k, v, do = _case(n, P, H, G, seed=n + 17)
    cud = None if cu is None else torch.tensor(cu, dtype=torch.int32).cuda()
    qh, kh, vh, doh = _heads(q, k, v, do, P)
    res = {}
    try:
        for order in (U.BLOCK_ORDER_KV_HEAD_MAJOR, U.BLOCK_ORDER_HEAVIEST_FIRST):
            U.ulysses_set_attn_block_order(order)
            oh, lse = U.ulysses_attn_fwd(qh, kh, vh, mask=mask, cu_seqlens=cud)
            fused = U.ulysses_attn_bwd(qh, kh, vh, oh, lse, doh, mask=mask, cu_seqlens=cud)
            det = U.ulysses_attn_bwd(qh, kh, vh, oh, lse, doh, mask=mask, cu_seqlens=cud, deterministic=True)
            torch.cuda.synchronize()
            res[order] = (oh, lse, fused, det)
    finally:
        U.ulysses_set_attn_block_order(U.BLOCK_ORDER_AUTO)
    (o1, l1, f1, d1), (o2, l2, f2, d2) = res[U.BLOCK_ORDER_KV_HEAD_MAJOR], res[U.BLOCK_ORDER_HEAVIEST_FIRST]
    assert torch.equal(o1, o2) and torch.equal(l1, l2), "forward differs between the block orders"
    assert all(torch.equal(a, b) for a, b in zip(d1, d2)), "deterministic backward differs"
    assert torch.equal(f1[1], f2[1]) and torch.equal(f1[2], f2[2]), "fused dK / dV differ"
    a, b = f1[0].float().cpu(), f2[0].float().cpu()
    assert float(((a - b).abs() / (2.0 ** -7 * torch.maximum(a.abs(), b.abs()) + 1e-6)).max()) <= 1.0
    assert U.ulysses_read_error() == 0
