"""GPU parity of the KV-head copies used when there are fewer KV heads than
ranks (G < P): the copying all-to-all bit-exact against the oracle's index
loops, the summing reverse against the oracle's fp64 sums, and the whole
layer (copies -> attention with one KV head per rank -> sums) against the
oracle's Ulysses procedure, which is pinned to plain GQA attention."""
import numpy as np
import pytest
import torch

import oracle
from helpers import (BF16_MAX_ABS, BF16_REL_L2, F32_MAX_ABS, assert_bf16_close, bf16_bound, f32_inputs,
                     max_abs, rel_l2, sample_rows)
from long_context_sequence_all_b200 import ulysses as U
from long_context_sequence_all_b200.workloads import make_inputs, to_natural

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    U.lib()
    U.ulysses_read_error()


def _bytes(t: torch.Tensor) -> np.ndarray:
    t = t.contiguous()
    return t.view(torch.uint8).numpy().reshape(*t.shape[:-1], t.shape[-1] * t.element_size())


@pytest.mark.parametrize("P,B,s,G,d,dtype", [
    (8, 1, 256, 2, 128, torch.bfloat16),     # Qwen-like: 4 copies per KV head
    (4, 2, 37, 1, 128, torch.bfloat16),      # one KV head, ragged, B > 1
    (16, 1, 40, 8, 128, torch.bfloat16),     # 2 copies, many ranks
    (8, 3, 5, 4, 64, torch.float32),
    (4, 1, 64, 2, 16, torch.int32),          # iota payload
    (4, 1, 9, 4, 8, torch.float64),          # G == P: plain seq->head
])
def test_replicate_bit_exact(P, B, s, G, d, dtype):
    n = P * s
    if dtype == torch.int32:
        x = torch.arange(P * B * s * G * d, dtype=torch.int32).reshape(P, B, s, G, d)
    else:
        x = torch.randn(P, B, s, G, d).to(dtype)
    y = U.ulysses_kv_seq_to_head_replicated(x.cuda(), P)
    torch.cuda.synchronize()
    assert y.shape == (P, B, 1, n, d)
    assert np.array_equal(_bytes(y.cpu()), oracle.kv_replicate_to_head(_bytes(x), B, n, P, G))
    assert U.ulysses_read_error() == 0


def _exact_payload(shape, g):
    """Multiples of 1/16 in [-4, 4): every fp32 partial sum of a few of them is
    exact, so the only rounding is the final one to the element type."""
    return torch.randint(-64, 64, shape, generator=g).double() / 16


@pytest.mark.parametrize("P,B,n,G,dtype", [(8, 1, 1024, 2, torch.bfloat16), (16, 2, 320, 1, torch.bfloat16),
                                           (4, 1, 296, 2, torch.float32), (8, 1, 64, 8, torch.bfloat16)])
def test_reduce_single_rounding_exact(P, B, n, G, dtype):
    """With exactly representable partial sums the result is the exact sum
    rounded once (RNE) to the element type, bit for bit."""
    g = torch.Generator().manual_seed(P * 1000 + n)
    x = _exact_payload((P, B, 1, n, 128), g).to(dtype)
    y = U.ulysses_kv_head_to_seq_reduce(x.cuda(), P, G)
    torch.cuda.synchronize()
    ref = oracle.kv_reduce_to_seq(x.double().numpy(), B, n, P, G)
    assert torch.equal(y.cpu(), torch.from_numpy(ref).to(dtype))


@pytest.mark.parametrize("P,G,dtype", [(8, 2, torch.bfloat16), (16, 1, torch.bfloat16), (8, 1, torch.float32)])
def test_reduce_random_within_fp32_sum_bound(P, G, dtype):
    """N(0,1) data: |got - exact| <= the fp32 summation bound
    e = (P/G - 1) * 2^-24 * sum |x_j| plus half an ulp of the element type at
    |exact| + e (the one rounding of the fp32 sum)."""
    B, n, d = 1, 2048 + 8 * P, 128
    x = torch.randn(P, B, 1, n, d, generator=torch.Generator().manual_seed(5)).to(dtype)
    y = U.ulysses_kv_head_to_seq_reduce(x.cuda(), P, G)
    torch.cuda.synchronize()
    ref = oracle.kv_reduce_to_seq(x.double().numpy(), B, n, P, G)
    abs_sum = oracle.kv_reduce_to_seq(x.double().abs().numpy(), B, n, P, G)
    acc = (P // G - 1) * 2.0 ** -24 * abs_sum
    half_ulp = (2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -24) * (np.abs(ref) + acc)
    bound = half_ulp + acc + 1e-30
    err = np.abs(y.cpu().double().numpy() - ref)
    assert (err <= bound).all(), float((err / bound).max())


def _layer(q, k, v, do, P, G, mask, cu=None):
    """The Ulysses layer with copied KV heads, every step through the C ABI."""
    cud = None if cu is None else cu.cuda()
    qh = U.ulysses_seq_to_head(q.cuda(), P)
    kh = U.ulysses_kv_seq_to_head_replicated(k.cuda(), P)
    vh = U.ulysses_kv_seq_to_head_replicated(v.cuda(), P)
    oh, lse = U.ulysses_attn_fwd(qh, kh, vh, mask=mask, cu_seqlens=cud)
    o = U.ulysses_head_to_seq(oh, P)
    doh = U.ulysses_seq_to_head(do.cuda(), P)
    dqh, dkh, dvh = U.ulysses_attn_bwd(qh, kh, vh, oh, lse, doh, mask=mask, cu_seqlens=cud)
    dq = U.ulysses_head_to_seq(dqh, P)
    dk = U.ulysses_kv_head_to_seq_reduce(dkh, P, G)
    dv = U.ulysses_kv_head_to_seq_reduce(dvh, P, G)
    torch.cuda.synchronize()
    return o, lse, dq, dk, dv, dkh, dvh


def _copy_rounding(parts, B, n, P, G):
    """A copied KV head's gradient is a sum of P/G per-rank partials, each
    already rounded to bf16 by the attention backward (half an ulp, at most
    2^-8 |partial|), before the sum's own rounding.  The single-rounding bound
    of the stated tolerance covers the last one; this returns the partials'
    share, sum_j 2^-8 |partial_j|, in seq layout."""
    a = parts.detach().cpu().double().abs().numpy() * 2.0 ** -8
    return oracle.kv_reduce_to_seq(a, B, n, P, G)


def _assert_summed_close(got, ref, extra, what):
    """|got - ref| <= bf16_bound(ref) + the partials' rounding, element-wise;
    relative L2 <= 1e-2 unchanged."""
    g, r = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    err = np.abs(g - r)
    bound = bf16_bound(r) + extra
    worst = float((err / bound).max())
    assert worst <= 1.0 and rel_l2(g, r) <= BF16_REL_L2, f"{what}: worst err/bound {worst:.2f}"


def _case(n, P, H, G, d, dtype, seed, std=128 ** -0.5):
    g = torch.Generator().manual_seed(seed)
    s = n // P
    mk = lambda h, sd: (torch.randn(P, 1, s, h, d, generator=g) * sd).to(dtype)
    return mk(H, std), mk(G, std), mk(G, std), mk(H, 1.0)


@pytest.mark.parametrize("n,P,H,G,mask", [
    (512, 4, 8, 2, U.MASK_CAUSAL),           # 2 copies per KV head
    (424, 8, 16, 2, U.MASK_CAUSAL),          # 4 copies, ragged tail
    (1000, 8, 16, 1, U.MASK_DOC_CAUSAL),     # one KV head for all ranks (MQA)
    (392, 4, 8, 1, U.MASK_NONE),
])
def test_layer_bf16_elementwise(n, P, H, G, mask):
    q, k, v, do = _case(n, P, H, G, 128, torch.bfloat16, seed=n + P)
    cu = torch.tensor([0, 100, 129, 400, 401, 777, n], dtype=torch.int32) if mask == U.MASK_DOC_CAUSAL else None
    o, lse, dq, dk, dv, dkh, dvh = _layer(q, k, v, do, P, G, mask, cu)
    cun = None if cu is None else cu.numpy()
    args = [f32_inputs(x) for x in (q, k, v)]
    o_ref, lse_ref = oracle.ulysses_fwd(*args, P, mask=mask, cu_seqlens=cun)
    assert_bf16_close(o.cpu(), o_ref, "O")
    assert max_abs(lse.cpu(), lse_ref) <= 2e-3
    dq_ref, dk_ref, dv_ref = oracle.ulysses_bwd(*args, f32_inputs(do), P, mask=mask, cu_seqlens=cun)
    assert_bf16_close(dq.cpu(), dq_ref, "dQ")
    _assert_summed_close(dk.cpu().double().numpy(), dk_ref, _copy_rounding(dkh, 1, n, P, G), "dK")
    _assert_summed_close(dv.cpu().double().numpy(), dv_ref, _copy_rounding(dvh, 1, n, P, G), "dV")
    assert U.ulysses_read_error() == 0


@pytest.mark.parametrize("n,P,H,G,d,mask", [(256, 4, 4, 1, 64, U.MASK_CAUSAL), (200, 8, 8, 2, 128, U.MASK_NONE)])
def test_layer_f32_elementwise(n, P, H, G, d, mask):
    q, k, v, do = _case(n, P, H, G, d, torch.float32, seed=n, std=1.0)
    o, lse, dq, dk, dv, _, _ = _layer(q, k, v, do, P, G, mask)
    args = [f32_inputs(x) for x in (q, k, v)]
    o_ref, lse_ref = oracle.ulysses_fwd(*args, P, mask=mask)
    assert max_abs(o.cpu(), o_ref) <= F32_MAX_ABS
    ref = oracle.ulysses_bwd(*args, f32_inputs(do), P, mask=mask)
    for got, want in zip((dq, dk, dv), ref):
        assert max_abs(got.cpu(), want) <= F32_MAX_ABS * max(1.0, float(np.abs(want).max()))
    assert U.ulysses_read_error() == 0


def test_qwen8k_on_16_ranks_sampled():
    """The 8K Qwen3-4B layer (H = 32, G = 8) on P = 16 ranks: two query heads
    per rank, every KV head copied to two ranks.  O and dQ on sampled rows of
    the first and last query heads, dK and dV on sampled key columns of the
    first and last KV heads (each summed over its four query heads, which now
    live on two ranks)."""
    inp = make_inputs("qwen8k", with_loss=False)
    n, H, G = inp["n"], inp["H"], inp["G"]
    P = 16
    to16 = lambda x: to_natural(x).reshape(1, P, n // P, x.shape[3], x.shape[4]).transpose(0, 1).contiguous()
    q, k, v, do = (to16(inp[x]) for x in ("q", "k", "v", "do"))
    o, lse, dq, dk, dv, dkh, dvh = _layer(q, k, v, do, P, G, U.MASK_CAUSAL)
    assert U.ulysses_read_error() == 0
    ek = to_natural(torch.from_numpy(_copy_rounding(dkh, 1, n, P, G)))[0].numpy()
    ev = to_natural(torch.from_numpy(_copy_rounding(dvh, 1, n, P, G)))[0].numpy()
    group = H // G
    qn, kn, vn, don = (to_natural(x)[0] for x in (q, k, v, do))
    on, dqn, dkn, dvn = (to_natural(x.cpu())[0] for x in (o, dq, dk, dv))
    rows = sample_rows(n, P, k=24)
    for h in (0, H - 1):
        kvh = h // group
        o_ref, _, dq_ref = oracle.head_rows(f32_inputs(qn[:, h]), f32_inputs(kn[:, kvh]), f32_inputs(vn[:, kvh]),
                                            rows, dout=f32_inputs(don[:, h]))
        assert_bf16_close(on[rows, h], o_ref, f"O head {h}")
        assert_bf16_close(dqn[rows, h], dq_ref, f"dQ head {h}")
    cols = np.array([0, 1, n // 2, n - 129, n - 128, n - 64, n - 2, n - 1], dtype=np.int32)
    for kvh in (0, G - 1):
        heads = range(kvh * group, (kvh + 1) * group)
        dk_ref, dv_ref = oracle.kv_cols([f32_inputs(qn[:, h]) for h in heads],
                                        [f32_inputs(don[:, h]) for h in heads],
                                        f32_inputs(kn[:, kvh]), f32_inputs(vn[:, kvh]), cols)
        _assert_summed_close(dkn[cols, kvh].double().numpy(), dk_ref, ek[cols, kvh], f"dK kv head {kvh}")
        _assert_summed_close(dvn[cols, kvh].double().numpy(), dv_ref, ev[cols, kvh], f"dV kv head {kvh}")


def test_copies_at_the_benchmarked_size():
    """The configuration the bench times: the 64K workload's K (G = 8) over
    P = 16 ranks (two copies per KV head), iota payload (int16 pairs viewed as
    bf16, every element distinct): copies bit-exact against the oracle, and
    the summing reverse of the copies gives exactly 2 x (bf16: exact doubling)."""
    P, G, n, d = 16, 8, 65536, 128
    s = n // P
    x = (torch.arange(P * s * G * d, dtype=torch.int64) % 16381 + 1).to(torch.int16).reshape(P, 1, s, G, d)
    rep = U.ulysses_kv_seq_to_head_replicated(x.cuda().view(torch.bfloat16), P)
    torch.cuda.synchronize()
    assert np.array_equal(rep.view(torch.int16).cpu().numpy(), oracle.kv_replicate_to_head(x.numpy(), 1, n, P, G))
    del rep
    # doubling is exact in bf16 for finite values: sum of the two copies == 2 x
    xb = torch.randn(P, 1, s, G, d, generator=torch.Generator().manual_seed(16)).to(torch.bfloat16)
    back = U.ulysses_kv_head_to_seq_reduce(U.ulysses_kv_seq_to_head_replicated(xb.cuda(), P), P, G)
    torch.cuda.synchronize()
    assert torch.equal(back.cpu(), (xb.float() * 2).to(torch.bfloat16))
    assert U.ulysses_read_error() == 0
