"""Failure detection of the tcgen05 kernels, without a GPU fault.

Every mbarrier wait in the attention and projection kernels is bounded.  A
test sets a limit of a few hundred cycles (ulysses_set_wait_limit), so the
first wait for a tile copy runs out: the kernel records ULY_ERR_TIMEOUT and
where it happened, drains its copies and MMAs, frees its tensor memory and
returns -- the context stays usable.  With the built-in limit restored, the
next call gives correct results.
"""
import pytest
import torch

import oracle
from helpers import assert_bf16_close, f32_inputs
from long_context_sequence_all_b200 import ulysses as U

pytestmark = pytest.mark.gpu

TIMEOUT_BIT = 1 << 9
SHORT_LIMIT = 200   # cycles; a tile copy from memory takes thousands


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    U.lib()
    U.ulysses_set_wait_limit(0)
    U.ulysses_read_error()
    yield
    U.ulysses_set_wait_limit(0)


def _inputs(n=256, P=2, H=4, G=2, d=128, seed=17):
    g = torch.Generator().manual_seed(seed)
    s = n // P
    mk = lambda h, sd: (torch.randn(P, 1, s, h, d, generator=g) * sd).to(torch.bfloat16)
    return mk(H, d ** -0.5), mk(G, d ** -0.5), mk(G, d ** -0.5), mk(H, 1.0)


def _with_short_limit(fn):
    U.ulysses_read_error()
    U.ulysses_set_wait_limit(SHORT_LIMIT)
    try:
        fn()
        torch.cuda.synchronize()
    finally:
        U.ulysses_set_wait_limit(0)
    return U.ulysses_read_error_info()


def _check_record(info, threads):
    assert info[0] & TIMEOUT_BIT, f"no timeout recorded: {info[:9]}"
    assert info[1] == 1
    assert info[2] >= 0 and info[3] >= 0 and 0 <= info[4] < threads
    assert info[8] >= 1                     # polls of the wait that gave up
    assert U.ulysses_read_error() == 0      # the record was cleared


@pytest.mark.parametrize("which", ["fwd", "bwd", "bwd_deterministic"])
def test_attention_wait_runs_out_then_next_call_is_correct(which):
    q, k, v, do = _inputs()
    P = 2
    qh, kh, vh, doh = (U.ulysses_seq_to_head(x.cuda(), P) for x in (q, k, v, do))
    oh, lse = U.ulysses_attn_fwd(qh, kh, vh)
    torch.cuda.synchronize()
    assert U.ulysses_read_error() == 0
    if which == "fwd":
        info = _with_short_limit(lambda: U.ulysses_attn_fwd(qh, kh, vh))
        _check_record(info, 384)
        o2, _ = U.ulysses_attn_fwd(qh, kh, vh)
        o_ref, _ = oracle.ulysses_fwd(f32_inputs(q), f32_inputs(k), f32_inputs(v), P)
        assert_bf16_close(U.ulysses_head_to_seq(o2, P).cpu(), o_ref, "O after a timeout")
    else:
        det = which == "bwd_deterministic"
        info = _with_short_limit(lambda: U.ulysses_attn_bwd(qh, kh, vh, oh, lse, doh, deterministic=det))
        _check_record(info, 384 if det else 512)
        grads = U.ulysses_attn_bwd(qh, kh, vh, oh, lse, doh, deterministic=det)
        ref = oracle.ulysses_bwd(f32_inputs(q), f32_inputs(k), f32_inputs(v), f32_inputs(do), P)
        for name, got, want in zip(("dQ", "dK", "dV"), grads, ref):
            assert_bf16_close(U.ulysses_head_to_seq(got, P).cpu(), want, f"{name} after a timeout")
    torch.cuda.synchronize()
    assert U.ulysses_read_error() == 0


def test_projection_wait_runs_out_then_next_call_is_correct():
    P, H, G, hidden, n = 2, 4, 2, 256, 256
    g = torch.Generator().manual_seed(23)
    x = torch.randn(P, 1, n // P, hidden, generator=g).to(torch.bfloat16)
    w = (torch.randn((H + 2 * G) * 128, hidden, generator=g) / hidden ** 0.5).to(torch.bfloat16)
    xd, wd = x.cuda(), w.cuda()
    tab = U.ulysses_rope_table(n, 128, 1.0e6)
    torch.cuda.synchronize()
    info = _with_short_limit(lambda: U.ulysses_qkv_proj_rope(xd, wd, P, H, G, tab))
    _check_record(info, 192)
    pq, pk, pv = U.ulysses_qkv_proj_rope(xd, wd, P, H, G, tab)
    rq, rk, rv = oracle.qkv_proj_rope(f32_inputs(x), f32_inputs(w), P, H, G, 128, 1.0e6)
    for name, a, b in zip("QKV", (pq, pk, pv), (rq, rk, rv)):
        assert_bf16_close(a.cpu(), b, f"{name} projection after a timeout")
    assert U.ulysses_read_error() == 0


def test_set_wait_limit_rejects_negative():
    with pytest.raises(U.UlyssesError) as e:
        U.ulysses_set_wait_limit(-1)
    assert e.value.status == 2
