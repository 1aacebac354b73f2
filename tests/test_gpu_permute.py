"""GPU parity of the two all-to-alls (in-HBM layout permutations): bit-exact
against the oracle's explicit index loops, at small ragged shapes and at every
workload's full size."""
import numpy as np
import pytest
import torch

import oracle
from long_context_sequence_all_b200 import ulysses as U
from long_context_sequence_all_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    U.lib()


def _bytes(t: torch.Tensor) -> np.ndarray:
    """Raw bytes of a CPU tensor, last dimension widened by the element size."""
    t = t.contiguous()
    return t.view(torch.uint8).numpy().reshape(*t.shape[:-1], t.shape[-1] * t.element_size())


def _roundtrip_case(P, B, s, heads, d, dtype):
    n = P * s
    if dtype == torch.int32:
        x = torch.arange(P * B * s * heads * d, dtype=torch.int32).reshape(P, B, s, heads, d)
    else:
        x = torch.randn(P, B, s, heads, d).to(dtype)
    h = U.ulysses_seq_to_head(x.cuda(), P)
    back = U.ulysses_head_to_seq(h, P)
    torch.cuda.synchronize()
    expect = oracle.seq_to_head(_bytes(x), B, n, P, heads)
    assert np.array_equal(_bytes(h.cpu()), expect)
    assert np.array_equal(_bytes(back.cpu()), _bytes(x))


@pytest.mark.parametrize("P,B,s,heads,d,dtype", [
    (4, 1, 256, 8, 64, torch.float32),       # tiny fp32 workload
    (4, 2, 37, 8, 128, torch.bfloat16),      # ragged token count, B > 1
    (2, 3, 5, 4, 8, torch.bfloat16),         # 16-byte rows
    (8, 1, 1, 8, 128, torch.bfloat16),       # one token per rank
    (1, 1, 100, 4, 32, torch.float32),       # P = 1: pure [n][H] -> [H][n] transpose
    (4, 1, 64, 4, 16, torch.int32),          # iota payload
    (4, 1, 33, 8, 64, torch.float64),        # 8-byte elements, 512 B rows
])
def test_permute_small(P, B, s, heads, d, dtype):
    _roundtrip_case(P, B, s, heads, d, dtype)


@pytest.mark.parametrize("name", ["qwen8k", "qwen64k", "packed", "long256k"])
def test_permute_workload_shapes(name):
    """Full-size Q (and K) of every bf16 workload, iota payload (int16 pairs
    viewed as bf16 rows) so every element is distinct and checkable."""
    w = WORKLOADS[name]
    n = w.n if w.n else 69632
    for heads in (w.H, w.G):
        s = n // w.P
        total = w.P * s * heads * w.d
        x = (torch.arange(total, dtype=torch.int64) % 65521).to(torch.int16).reshape(w.P, 1, s, heads, w.d)
        xd = x.cuda().view(torch.bfloat16)
        h = U.ulysses_seq_to_head(xd, w.P)
        back = U.ulysses_head_to_seq(h, w.P)
        torch.cuda.synchronize()
        expect = oracle.seq_to_head(x.numpy(), 1, n, w.P, heads)
        assert np.array_equal(h.view(torch.int16).cpu().numpy(), expect)
        assert torch.equal(back.view(torch.int16).cpu(), x)
        del xd, h, back
        torch.cuda.empty_cache()


def test_permute_does_not_touch_outside_output():
    """Guard bands around the output stay untouched (out-of-bounds canary)."""
    P, B, s, heads, d = 4, 1, 100, 8, 64
    x = torch.randn(P, B, s, heads, d).cuda()
    n_el = P * B * s * heads * d
    pad = 4096
    buf = torch.full((n_el + 2 * pad,), 12345.0, device="cuda")
    out = buf[pad:pad + n_el].view(P, B, heads // P, P * s, d)
    U.ulysses_seq_to_head(x, P, out=out)
    torch.cuda.synchronize()
    assert torch.all(buf[:pad] == 12345.0) and torch.all(buf[pad + n_el:] == 12345.0)
