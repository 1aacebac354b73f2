"""GPU parity of the bf16 tensor-core Ulysses layer against the fp64 oracle:
max-abs <= 2e-2 and relative L2 <= 1e-2 on O (and gradients), LSE within
2e-3.  Small shapes are compared element by element (several 128-row tiles
and a ragged tail); the full-size workloads are compared on sampled heads and
rows, which the oracle computes exactly one by one."""
import numpy as np
import pytest
import torch

import oracle
from helpers import LSE_BF16_MAX_ABS, assert_bf16_close, f32_inputs, max_abs, sample_rows
from long_context_sequence_all_b200 import ulysses as U
from long_context_sequence_all_b200.workloads import make_inputs, to_natural

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    U.lib()
    U.ulysses_read_error()


def layer_fwd(q, k, v, P, mask, cu=None):
    cud = None if cu is None else cu.cuda()
    qh, kh, vh = (U.ulysses_seq_to_head(x.cuda(), P) for x in (q, k, v))
    oh, lse = U.ulysses_attn_fwd(qh, kh, vh, mask=mask, cu_seqlens=cud)
    o = U.ulysses_head_to_seq(oh, P)
    torch.cuda.synchronize()
    return o, lse, (qh, kh, vh, oh, cud)


def _rand_case(n, P, H, G, d=128, seed=0, std=128 ** -0.5):
    g = torch.Generator().manual_seed(seed)
    s = n // P
    mk = lambda h, sd: (torch.randn(P, 1, s, h, d, generator=g) * sd).to(torch.bfloat16)
    return mk(H, std), mk(G, std), mk(G, std), mk(H, 1.0)


def _lse_nat(lse_head, B, H, n):
    # [P][B][H/P][n] -> [B][H][n]
    return lse_head.cpu().permute(1, 0, 2, 3).reshape(B, H, n)


@pytest.mark.parametrize("n,P,H,G,mask,std", [
    (512, 4, 8, 2, U.MASK_CAUSAL, 128 ** -0.5),    # 4 query tiles
    (424, 4, 8, 2, U.MASK_CAUSAL, 128 ** -0.5),    # ragged tail (3 tiles + 40 rows)
    (392, 4, 8, 4, U.MASK_NONE, 128 ** -0.5),      # non-causal, ragged keys
    (1000, 8, 16, 8, U.MASK_DOC_CAUSAL, 128 ** -0.5),
    (640, 4, 8, 2, U.MASK_CAUSAL, 3.0),            # peaked softmax: running-max rescales
    (128, 4, 8, 2, U.MASK_CAUSAL, 1.0),            # a single tile
    (8, 8, 16, 8, U.MASK_CAUSAL, 1.0),             # one token per rank
])
def test_fwd_small_elementwise(n, P, H, G, mask, std):
    q, k, v, _ = _rand_case(n, P, H, G, std=std, seed=n)
    cu = None
    if mask == U.MASK_DOC_CAUSAL:
        cu = torch.tensor([0, 100, 129, 400, 401, 777, n], dtype=torch.int32)
    o, lse, _ = layer_fwd(q, k, v, P, mask, cu)
    o_ref, lse_ref = oracle.ulysses_fwd(f32_inputs(q), f32_inputs(k), f32_inputs(v), P, mask=mask,
                                        cu_seqlens=None if cu is None else cu.numpy())
    assert_bf16_close(o.cpu(), o_ref, "O")
    assert max_abs(lse.cpu(), lse_ref) <= LSE_BF16_MAX_ABS
    assert U.ulysses_read_error() == 0


def test_fwd_rejects_odd_group():
    q, k, v, _ = _rand_case(256, 4, 4, 4)
    qh, kh, vh = (U.ulysses_seq_to_head(x.cuda(), 4) for x in (q, k, v))
    with pytest.raises(U.UlyssesError) as e:
        U.ulysses_attn_fwd(qh, kh, vh)
    assert e.value.status == 6


def _check_sampled_fwd(inp, o_seq, lse_head, heads, rows):
    P, n, H = inp["P"], inp["n"], inp["H"]
    group = H // inp["G"]
    qn, kn, vn = (to_natural(inp[x])[0] for x in ("q", "k", "v"))
    on = to_natural(o_seq.cpu())[0]
    lse_n = _lse_nat(lse_head, 1, H, n)[0]
    cu = inp["cu_seqlens"]
    for h in heads:
        kvh = h // group
        o_ref, l_ref = oracle.head_rows(f32_inputs(qn[:, h]), f32_inputs(kn[:, kvh]), f32_inputs(vn[:, kvh]),
                                        rows, mask=inp["mask"],
                                        cu_seqlens=None if cu is None else cu.numpy())
        assert_bf16_close(on[rows, h], o_ref, f"O head {h}")
        assert max_abs(lse_n[h, rows], l_ref) <= LSE_BF16_MAX_ABS


@pytest.mark.parametrize("name", ["qwen8k", "qwen64k", "packed", "long256k"])
def test_fwd_workload_sampled(name):
    inp = make_inputs(name, with_loss=False, with_grad_inputs=False)
    P, n = inp["P"], inp["n"]
    o, lse, _ = layer_fwd(inp["q"], inp["k"], inp["v"], P, inp["mask"], inp["cu_seqlens"])
    assert U.ulysses_read_error() == 0
    extra = [] if inp["cu_seqlens"] is None else inp["cu_seqlens"].tolist()
    rows = sample_rows(n, P, k=48 if n <= 65536 else 24, extra=extra)
    H = inp["H"]
    _check_sampled_fwd(inp, o, lse, [0, 5, H // 2 + 1, H - 1], rows)


def test_fwd_qwen8k_full_heads():
    """8K workload: every row of one head from the first and the last GQA
    group (ranks 0 and 3), element by element."""
    inp = make_inputs("qwen8k", with_loss=False, with_grad_inputs=False)
    o, lse, _ = layer_fwd(inp["q"], inp["k"], inp["v"], inp["P"], inp["mask"])
    rows = np.arange(inp["n"], dtype=np.int32)
    _check_sampled_fwd(inp, o, lse, [1, inp["H"] - 2], rows)
