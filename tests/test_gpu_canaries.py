"""Out-of-bounds canaries for the kernels beyond the layer step: every output
is a view into a larger buffer whose guard bands hold a sentinel, and the
guard bands must be untouched after the call (the check compute-sanitizer
would make, which this pool does not offer).  Ragged shapes, so that the
last tiles / vectors of every kernel are partial."""
import pytest
import torch

from long_context_sequence_all_b200 import ulysses as U

pytestmark = pytest.mark.gpu

PAD = 4096          # elements of guard band on each side (16-byte multiples for every dtype here)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    U.lib()
    U.ulysses_read_error()


def _guarded(shape, dtype, sentinel):
    n_el = 1
    for x in shape:
        n_el *= x
    buf = torch.full((n_el + 2 * PAD,), sentinel, dtype=dtype, device="cuda")
    return buf, buf[PAD:PAD + n_el].view(*shape)


def _intact(buf, sentinel):
    torch.cuda.synchronize()
    n = buf.numel()
    return bool(torch.all(buf[:PAD] == sentinel)) and bool(torch.all(buf[n - PAD:] == sentinel))


def test_kv_copy_and_sum_guards():
    P, B, s, G, d = 8, 2, 37, 2, 128
    x = torch.randn(P, B, s, G, d, device="cuda").to(torch.bfloat16)
    buf, rep = _guarded((P, B, 1, P * s, d), torch.bfloat16, 3.0)
    U.ulysses_kv_seq_to_head_replicated(x, P, out=rep)
    assert _intact(buf, 3.0)
    buf2, back = _guarded((P, B, s, G, d), torch.bfloat16, 3.0)
    U.ulysses_kv_head_to_seq_reduce(rep, P, G, out=back)
    assert _intact(buf2, 3.0)
    assert torch.equal(back, (x.float() * (P // G)).to(torch.bfloat16))
    assert U.ulysses_read_error() == 0


def test_shift_labels_guards():
    B, n, P = 3, 1000, 8
    ids = torch.randint(0, 151936, (B, n), dtype=torch.int32, device="cuda")
    cu = torch.tensor([0, 1, 2, 513, 700, n], dtype=torch.int32, device="cuda")
    buf, lab = _guarded((P, B, n // P), torch.int32, -7)
    U.ulysses_shift_labels(ids, P, cu_seqlens=cu, valid_len=n - 5, out=lab)
    assert _intact(buf, -7)
    assert int((lab == -7).sum()) == 0
    assert U.ulysses_read_error() == 0


def test_projection_guards():
    P, B, s, hidden, H, G, d = 4, 2, 70, 256, 8, 4, 128      # 560 rows: a ragged last row tile
    n = P * s
    x = torch.randn(P, B, s, hidden, device="cuda").to(torch.bfloat16)
    w = (torch.randn((H + 2 * G) * d, hidden, device="cuda") / hidden ** 0.5).to(torch.bfloat16)
    tab = U.ulysses_rope_table(n, d, 1.0e6)
    bq, q = _guarded((P, B, H // P, n, d), torch.bfloat16, 5.0)
    bk, k = _guarded((P, B, G // P, n, d), torch.bfloat16, 5.0)
    bv, v = _guarded((P, B, G // P, n, d), torch.bfloat16, 5.0)
    U.ulysses_qkv_proj_rope(x, w, P, H, G, tab, q=q, k=k, v=v)
    assert _intact(bq, 5.0) and _intact(bk, 5.0) and _intact(bv, 5.0)
    wo = (torch.randn(hidden, H * d, device="cuda") / (H * d) ** 0.5).to(torch.bfloat16)
    by, y = _guarded((P, B, s, hidden), torch.bfloat16, 5.0)
    U.ulysses_o_proj(q, wo, P, y=y)
    assert _intact(by, 5.0)
    assert U.ulysses_read_error() == 0
