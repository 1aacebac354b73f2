"""GPU parity of the token-weighted loss aggregation against the fp64 oracle."""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from helpers import LOSS_REL
from long_context_sequence_all_b200 import ulysses as U
from long_context_sequence_all_b200.workloads import IGNORE_INDEX, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    U.lib()
    U.ulysses_read_error()


def _check(logits, labels, P):
    S, C, L = U.ulysses_loss_aggregate(logits.cuda(), labels.cuda(), P)
    torch.cuda.synchronize()
    So, Co, Lo, bad = oracle.loss_aggregate(logits.float().numpy(), labels.numpy(), P)
    assert bad == 0
    assert np.array_equal(C.cpu().numpy(), Co)
    if Co.sum() == 0:
        assert math.isnan(L.item())
    else:
        assert abs(L.item() - Lo) <= LOSS_REL * abs(Lo), (L.item(), Lo)
    for r in range(P):
        if Co[r]:
            assert abs(S[r].item() - So[r]) <= LOSS_REL * abs(So[r]) + 1e-6
        else:
            assert S[r].item() == 0.0
    return S, C, L


@pytest.mark.parametrize("T,V,P,dtype", [(64, 8192, 4, torch.bfloat16), (40, 200, 8, torch.float32),
                                         (96, 1024, 3, torch.bfloat16), (8, 8, 8, torch.bfloat16)])
def test_loss_small(T, V, P, dtype):
    g = torch.Generator().manual_seed(T * V)
    logits = (torch.randn(T, V, generator=g) * 2).to(dtype)
    labels = torch.randint(0, V, (T,), generator=g, dtype=torch.int32)
    labels[torch.rand(T, generator=g) < 0.25] = IGNORE_INDEX
    _check(logits, labels, P)


def test_loss_empty_shard_and_all_ignored():
    T, V, P = 64, 512, 4
    logits = torch.randn(T, V).to(torch.bfloat16)
    labels = torch.randint(0, V, (T,), dtype=torch.int32)
    labels[:16] = IGNORE_INDEX                 # shard 0 has no valid token
    _check(logits, labels, P)
    labels[:] = IGNORE_INDEX
    _check(logits, labels, P)                  # L = NaN, counts 0


def test_loss_uniform_logits_closed_form():
    T, V, P = 128, 8192, 4
    logits = torch.full((T, V), 0.75, dtype=torch.bfloat16)
    labels = torch.randint(0, V, (T,), dtype=torch.int32)
    S, C, L = U.ulysses_loss_aggregate(logits.cuda(), labels.cuda(), P)
    assert abs(L.item() - math.log(V)) <= LOSS_REL * math.log(V)


def test_loss_bad_label_sets_error_word():
    T, V, P = 32, 256, 4
    logits = torch.randn(T, V).to(torch.bfloat16)
    labels = torch.randint(0, V, (T,), dtype=torch.int32)
    labels[5] = V + 3
    U.ulysses_read_error()
    S, C, L = U.ulysses_loss_aggregate(logits.cuda(), labels.cuda(), P)
    word = U.ulysses_read_error()
    assert word & (1 << 8)
    assert int(C.sum().item()) == T - 1
    assert U.ulysses_read_error() == 0          # reading clears it


def test_loss_deterministic():
    T, V, P = 4096, 2048, 4
    logits = torch.randn(T, V).to(torch.bfloat16).cuda()
    labels = torch.randint(0, V, (T,), dtype=torch.int32).cuda()
    a = U.ulysses_loss_aggregate(logits, labels, P)
    b = U.ulysses_loss_aggregate(logits, labels, P)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("name", ["qwen64k", "packed"])
def test_loss_workload(name):
    """Full-size logits of the workloads with a loss (64K x 8192 bf16; packed
    documents with 20% ignored labels and an ignored pad tail)."""
    inp = make_inputs(name, with_grad_inputs=False)
    _check(inp["logits"], inp["labels"], inp["P"])


def _read_device_int32(addr: int) -> int:
    """The int32 at device address `addr`, read with the CUDA driver's
    synchronous device-to-host copy (the context torch made current)."""
    libcuda = ctypes.CDLL("libcuda.so.1")
    libcuda.cuMemcpyDtoH_v2.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_size_t]
    out = ctypes.c_int32(0)
    st = libcuda.cuMemcpyDtoH_v2(ctypes.byref(out), addr, 4)
    assert st == 0, f"cuMemcpyDtoH_v2 returned {st}"
    return out.value


def test_error_word_address_holds_the_async_errors():
    """ulysses_error_word gives the device word that kernels OR their
    data-dependent errors into: a bad label shows up at that address, and
    ulysses_read_error reads and clears the same word."""
    addr = U.ulysses_error_word()
    assert addr and addr == U.ulysses_error_word()
    U.ulysses_read_error()
    torch.cuda.synchronize()
    assert _read_device_int32(addr) == 0
    logits = torch.randn(8, 256, device="cuda").to(torch.bfloat16)
    labels = torch.tensor([0, 1, 999, 3, 4, 5, 6, 7], dtype=torch.int32, device="cuda")
    U.ulysses_loss_aggregate(logits, labels, 2)
    torch.cuda.synchronize()
    assert _read_device_int32(addr) & (1 << 8)
    assert U.ulysses_read_error() & (1 << 8)
    assert _read_device_int32(addr) == 0
