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


def _iota(P, B, s, heads, d, offset=0):
    total = P * B * s * heads * d
    return ((torch.arange(total, dtype=torch.int64) + offset) % 65521).to(torch.int16).reshape(P, B, s, heads, d)


@pytest.mark.parametrize("P,B,s,heads,d", [
    (4, 1, 2048, (32, 8, 8), 128),      # Q, K, V of the 8K workload
    (8, 2, 203, (32, 8, 8), 128),       # ragged positions per rank, B > 1
    (2, 1, 3, (4, 2), 64),              # fewer positions than one block
    (4, 1, 300, (16, 4, 4, 16), 32),    # four tensors, 64-byte rows
])
def test_batched_permute_bit_exact_with_guard_bands(P, B, s, heads, d):
    """Up to four tensors in one call, both directions, iota payloads checked
    against the oracle's index loops; every destination sits between guard
    bands that must stay untouched (ragged last blocks included)."""
    n = P * s
    pad = 4096
    xs = [_iota(P, B, s, h, d, offset=1000 * i) for i, h in enumerate(heads)]
    bufs, outs = [], []
    for h in heads:
        el = P * B * s * h * d
        buf = torch.full((el + 2 * pad,), -7, dtype=torch.int16, device="cuda")
        bufs.append(buf)
        outs.append(buf[pad:pad + el].view(torch.bfloat16).view(P, B, h // P, n, d))
    U.ulysses_seq_to_head_batch([x.cuda().view(torch.bfloat16) for x in xs], P, outs=outs)
    torch.cuda.synchronize()
    for x, h, o, buf in zip(xs, heads, outs, bufs):
        assert np.array_equal(o.view(torch.int16).cpu().numpy(), oracle.seq_to_head(x.numpy(), B, n, P, h))
        assert torch.all(buf[:pad] == -7) and torch.all(buf[pad + o.numel():] == -7)
    back_bufs, backs = [], []
    for x in xs:
        buf = torch.full((x.numel() + 2 * pad,), -7, dtype=torch.int16, device="cuda")
        back_bufs.append(buf)
        backs.append(buf[pad:pad + x.numel()].view(torch.bfloat16).view(x.shape))
    U.ulysses_head_to_seq_batch(outs, P, outs=backs)
    torch.cuda.synchronize()
    for x, b, buf in zip(xs, backs, back_bufs):
        assert torch.equal(b.view(torch.int16).cpu(), x)
        assert torch.all(buf[:pad] == -7) and torch.all(buf[pad + x.numel():] == -7)


def test_batched_permute_rejects_overlap_and_count():
    x = torch.zeros(2, 1, 8, 4, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(2, 1, 2, 16, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(U.UlyssesError) as e:
        U.ulysses_seq_to_head_batch([x, x], 2, outs=[y, y])
    assert e.value.status == 5
    with pytest.raises(U.UlyssesError):
        U.ulysses_seq_to_head_batch([x] * 5, 2)


@pytest.mark.parametrize("name", ["qwen8k", "qwen64k", "packed", "long256k"])
def test_workload_shapes_take_the_tma_path(name):
    """The Q/K/V shapes of the workloads go through the TMA kernel (one launch
    for the three tensors), not the vector fallback."""
    w = WORKLOADS[name]
    n = w.n if w.n else 69632
    s = n // w.P
    xs = [torch.empty(w.P, 1, s, h, w.d, dtype=torch.bfloat16, device="cuda") for h in (w.H, w.G, w.G)]
    U.ulysses_profile_enable(True)
    hs = U.ulysses_seq_to_head_batch(xs, w.P)
    U.ulysses_head_to_seq_batch(hs, w.P, outs=xs)
    torch.cuda.synchronize()
    prof = U.ulysses_profile_read()
    U.ulysses_profile_enable(False)
    assert prof.get("seq_to_head", (0, 0))[1] == 1 and prof.get("head_to_seq", (0, 0))[1] == 1, prof
    assert "seq_to_head_vec" not in prof and "head_to_seq_vec" not in prof, prof
