"""The whole Ulysses layer forward on the GPU, steps 1-6 through the C ABI:
QKV projection with rotary positions straight into the head layout (first
all-to-all folded in), attention per logical rank, output projection read
straight from the head layout (second all-to-all folded in) -- against the
oracle's layer.  The oracle chain stores its own Q/K/V and O in bf16 where
the layer stores them (rounding the oracle's values, not the GPU's), so the
comparison measures the kernels' arithmetic: within the bf16 tolerance."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_bf16_close
from long_context_sequence_all_b200 import ulysses as U

pytestmark = pytest.mark.gpu

D = 128


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    U.lib()
    U.ulysses_read_error()


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy()


@pytest.mark.parametrize("P,s,hidden,H,G,mask", [(4, 128, 256, 8, 4, U.MASK_CAUSAL),
                                                 (2, 192, 512, 8, 2, U.MASK_CAUSAL),
                                                 (4, 100, 256, 8, 4, U.MASK_NONE)])
def test_layer_forward_steps_1_to_6(P, s, hidden, H, G, mask):
    n = P * s
    g = torch.Generator().manual_seed(n + hidden)
    x = torch.randn(P, 1, s, hidden, generator=g).to(torch.bfloat16)
    w = (torch.randn((H + 2 * G) * D, hidden, generator=g) / hidden ** 0.5).to(torch.bfloat16)
    wo = (torch.randn(hidden, H * D, generator=g) / (H * D) ** 0.5).to(torch.bfloat16)
    tab = U.ulysses_rope_table(n, D, 1.0e6)
    q, k, v = U.ulysses_qkv_proj_rope(x.cuda(), w.cuda(), P, H, G, tab)
    o, _ = U.ulysses_attn_fwd(q, k, v, mask=mask)
    y = U.ulysses_o_proj(o, wo.cuda(), P)
    torch.cuda.synchronize()
    assert U.ulysses_read_error() == 0
    xf, wf, wof = (t.float().numpy() for t in (x, w, wo))
    rq, rk, rv = (_bf16(a) for a in oracle.qkv_proj_rope(xf, wf, P, H, G, D))
    to_seq = lambda z, hx: oracle.head_to_seq(z, 1, n, P, hx)
    omask = oracle.MASK_CAUSAL if mask == U.MASK_CAUSAL else oracle.MASK_NONE
    ro, _ = oracle.ulysses_fwd(to_seq(rq, H), to_seq(rk, G), to_seq(rv, G), P, mask=omask)
    ry = oracle.o_proj(oracle.seq_to_head(_bf16(ro), 1, n, P, H), wof, P)
    assert_bf16_close(y.cpu(), ry, "Y")
