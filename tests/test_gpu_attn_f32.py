"""GPU parity of the exact-fp32 Ulysses layer against the fp64 oracle
(1e-5 max-abs): the tiny fp32 workload (n=1024, P=4, 8/8 heads, d=64, causal
and non-causal) through seq->head, attention, head->seq; plus ragged and
doc-causal edge cases and the fp32 backward."""
import numpy as np
import pytest
import torch

import oracle
from helpers import F32_MAX_ABS, max_abs
from long_context_sequence_all_b200 import ulysses as U
from long_context_sequence_all_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    U.lib()


def _layer_fwd(q, k, v, P, mask, cu=None):
    qh, kh, vh = (U.ulysses_seq_to_head(x.cuda(), P) for x in (q, k, v))
    oh, lse = U.ulysses_attn_fwd(qh, kh, vh, mask=mask, cu_seqlens=None if cu is None else cu.cuda())
    o = U.ulysses_head_to_seq(oh, P)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu(), (qh, kh, vh, oh, lse)


@pytest.mark.parametrize("mask", [U.MASK_NONE, U.MASK_CAUSAL])
def test_tiny_f32_workload(mask):
    inp = make_inputs("tiny_f32")
    P = inp["P"]
    o, lse, _ = _layer_fwd(inp["q"], inp["k"], inp["v"], P, mask)
    o_ref, lse_ref = oracle.ulysses_fwd(inp["q"].numpy(), inp["k"].numpy(), inp["v"].numpy(), P, mask=mask)
    assert max_abs(o, o_ref) <= F32_MAX_ABS
    assert max_abs(lse, lse_ref) <= F32_MAX_ABS
    # the round trip of the inputs is the identity
    q2 = U.ulysses_head_to_seq(U.ulysses_seq_to_head(inp["q"].cuda(), P), P).cpu()
    assert torch.equal(q2, inp["q"])


@pytest.mark.parametrize("n,P,H,G,d,mask", [
    (200, 4, 8, 4, 64, U.MASK_CAUSAL),        # ragged (not a multiple of the 64-row tile)
    (36, 4, 4, 4, 128, U.MASK_NONE),
    (8, 8, 8, 8, 64, U.MASK_CAUSAL),          # one token per rank
    (300, 2, 4, 2, 64, U.MASK_DOC_CAUSAL),
])
def test_f32_edge_cases_fwd_bwd(n, P, H, G, d, mask):
    g = torch.Generator().manual_seed(n + H)
    s = n // P
    q = torch.randn(P, 1, s, H, d, generator=g)
    k = torch.randn(P, 1, s, G, d, generator=g)
    v = torch.randn(P, 1, s, G, d, generator=g)
    do = torch.randn(P, 1, s, H, d, generator=g)
    cu = torch.tensor([0, 37, 150, 151, n], dtype=torch.int32) if mask == U.MASK_DOC_CAUSAL else None
    o, lse, (qh, kh, vh, oh, lseh) = _layer_fwd(q, k, v, P, mask, cu)
    cun = None if cu is None else cu.numpy()
    o_ref, lse_ref = oracle.ulysses_fwd(q.numpy(), k.numpy(), v.numpy(), P, mask=mask, cu_seqlens=cun)
    assert max_abs(o, o_ref) <= F32_MAX_ABS
    assert max_abs(lse, lse_ref) <= F32_MAX_ABS
    doh = U.ulysses_seq_to_head(do.cuda(), P)
    dqh, dkh, dvh = U.ulysses_attn_bwd(qh, kh, vh, oh, lseh, doh, mask=mask,
                                       cu_seqlens=None if cu is None else cu.cuda())
    dq, dk, dv = (U.ulysses_head_to_seq(x, P).cpu() for x in (dqh, dkh, dvh))
    dq_ref, dk_ref, dv_ref = oracle.ulysses_bwd(q.numpy(), k.numpy(), v.numpy(), do.numpy(), P,
                                                mask=mask, cu_seqlens=cun)
    scale = max(1.0, float(np.abs(dk_ref).max()))
    assert max_abs(dq, dq_ref) <= 2 * F32_MAX_ABS * scale
    assert max_abs(dk, dk_ref) <= 2 * F32_MAX_ABS * scale
    assert max_abs(dv, dv_ref) <= 2 * F32_MAX_ABS * scale


def test_tiny_f32_backward():
    inp = make_inputs("tiny_f32")
    P = inp["P"]
    g = torch.Generator().manual_seed(77)
    do = torch.randn(inp["q"].shape, generator=g)
    _, _, (qh, kh, vh, oh, lseh) = _layer_fwd(inp["q"], inp["k"], inp["v"], P, U.MASK_CAUSAL)
    dqh, dkh, dvh = U.ulysses_attn_bwd(qh, kh, vh, oh, lseh, U.ulysses_seq_to_head(do.cuda(), P))
    dq, dk, dv = (U.ulysses_head_to_seq(x, P).cpu() for x in (dqh, dkh, dvh))
    ref = oracle.ulysses_bwd(inp["q"].numpy(), inp["k"].numpy(), inp["v"].numpy(), do.numpy(), P)
    for got, want in zip((dq, dk, dv), ref):
        assert max_abs(got, want) <= 5 * F32_MAX_ABS
