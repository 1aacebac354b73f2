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


@pytest.mark.parametrize("out_seq", [False, True])
@pytest.mark.parametrize("deterministic", [False, True])
def test_attention_outputs_and_workspace_guards(out_seq, deterministic):
    """O, LSE, dQ, dK, dV and the backward workspace (exactly the size the
    library asks for) between guard bands, at a ragged length (the last query
    and key tiles partial), in both output layouts and both backward paths."""
    P, B, n, H, G, d = 4, 1, 424, 16, 4, 128
    s = n // P
    g = torch.Generator().manual_seed(424)
    mk = lambda h, sd: (torch.randn(P, B, s, h, d, generator=g) * sd).to(torch.bfloat16).cuda()
    qh, kh, vh, doh = (U.ulysses_seq_to_head(x, P) for x in (mk(H, d ** -0.5), mk(G, d ** -0.5),
                                                              mk(G, d ** -0.5), mk(H, 1.0)))
    shape_q = (P, B, s, H, d) if out_seq else (P, B, H // P, n, d)
    shape_kv = (P, B, s, G, d) if out_seq else (P, B, G // P, n, d)
    bo, o = _guarded(shape_q, torch.bfloat16, 9.0)
    bl, lse = _guarded((P, B, H // P, n), torch.float32, 9.0)
    U.ulysses_attn_fwd(qh, kh, vh, o=o, lse=lse, out_seq_layout=out_seq)
    assert _intact(bo, 9.0) and _intact(bl, 9.0)
    desc = U._desc_from(qh, kh, U.MASK_CAUSAL, None, 0.0, out_seq, deterministic)
    need = U.ulysses_attn_bwd_workspace_size(desc)
    bw, ws = _guarded((need,), torch.uint8, 77)
    bq, dq = _guarded(shape_q, torch.bfloat16, 9.0)
    bk, dk = _guarded(shape_kv, torch.bfloat16, 9.0)
    bv, dv = _guarded(shape_kv, torch.bfloat16, 9.0)
    U.ulysses_attn_bwd(qh, kh, vh, o, lse, doh, dq=dq, dk=dk, dv=dv, workspace=ws, out_seq_layout=out_seq,
                       deterministic=deterministic)
    assert _intact(bw, 77) and _intact(bq, 9.0) and _intact(bk, 9.0) and _intact(bv, 9.0)
    assert not any(bool(torch.isnan(t.float()).any()) for t in (o, dq, dk, dv))
    assert U.ulysses_read_error() == 0


def test_loss_output_guards():
    P, T, V = 3, 3 * 37, 1000
    logits = torch.randn(T, V, device="cuda").to(torch.bfloat16)
    labels = torch.randint(0, V, (T,), dtype=torch.int32, device="cuda")
    labels[::5] = -100
    bs, S = _guarded((P,), torch.float32, 4.0)
    bc, C = _guarded((P,), torch.int64, 4)
    bL, L = _guarded((1,), torch.float32, 4.0)
    need = U.ulysses_loss_workspace_size(P, T, V)
    bw, ws = _guarded((need,), torch.uint8, 77)
    U.ulysses_loss_aggregate(logits, labels, P, shard_sum=S, shard_count=C, loss=L, workspace=ws)
    assert _intact(bs, 4.0) and _intact(bc, 4) and _intact(bL, 4.0) and _intact(bw, 77)
    bz, dz = _guarded((T, V), torch.bfloat16, 4.0)
    need = U.ulysses_loss_bwd_workspace_size(P, T, V)
    bw2, ws2 = _guarded((need,), torch.uint8, 77)
    U.ulysses_loss_aggregate_bwd(logits, labels, P, dlogits=dz, shard_sum=S, shard_count=C, loss=L,
                                 workspace=ws2)
    assert _intact(bz, 4.0) and _intact(bs, 4.0) and _intact(bc, 4) and _intact(bL, 4.0) and _intact(bw2, 77)
    assert U.ulysses_read_error() == 0


def test_projection_backward_guards():
    P, B, s, hidden, H, G, d = 4, 2, 70, 256, 8, 4, 128
    n = P * s
    x = torch.randn(P, B, s, hidden, device="cuda").to(torch.bfloat16)
    w = (torch.randn((H + 2 * G) * d, hidden, device="cuda") / hidden ** 0.5).to(torch.bfloat16)
    tab = U.ulysses_rope_table(n, d, 1.0e6)
    dq = torch.randn(P, B, H // P, n, d, device="cuda").to(torch.bfloat16)
    dk = torch.randn(P, B, G // P, n, d, device="cuda").to(torch.bfloat16)
    dv = torch.randn(P, B, G // P, n, d, device="cuda").to(torch.bfloat16)
    bx, dx = _guarded((P, B, s, hidden), torch.bfloat16, 6.0)
    bw, dw = _guarded(((H + 2 * G) * d, hidden), torch.float32, 6.0)
    wsn = B * n * (H + 2 * G) * d * 2
    bws, ws = _guarded((wsn,), torch.uint8, 77)
    U.ulysses_qkv_proj_rope_bwd(x, w, P, H, G, tab, dq, dk, dv, dx=dx, dw=dw, workspace=ws)
    assert _intact(bx, 6.0) and _intact(bw, 6.0) and _intact(bws, 77)
    o_seq = torch.randn(P, B, s, H, d, device="cuda").to(torch.bfloat16)
    wo = (torch.randn(hidden, H * d, device="cuda") / (H * d) ** 0.5).to(torch.bfloat16)
    dy = torch.randn(P, B, s, hidden, device="cuda").to(torch.bfloat16)
    bdo, do = _guarded((P, B, H // P, n, d), torch.bfloat16, 6.0)
    bdw, dwo = _guarded((hidden, H * d), torch.float32, 6.0)
    U.ulysses_o_proj_bwd(o_seq, wo, dy, P, do=do, dw_o=dwo)
    assert _intact(bdo, 6.0) and _intact(bdw, 6.0)
    assert U.ulysses_read_error() == 0
