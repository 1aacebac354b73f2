"""ulysses_loss_aggregate_noalloc, the loss entry point for callers that
cannot allocate device memory (it takes its scratch from a fixed array inside
the library instead of a caller workspace).  Its results must match the
workspace entry point's on two calls in a row (the shared array keeps the
previous call's contents), and shapes too large for the array must be
refused before anything runs.  Called through the C ABI with raw pointers.
Kept in its own file, collected last."""
import ctypes

import pytest
import torch

from helpers import LOSS_REL
from long_context_sequence_all_b200 import ulysses as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = U.lib()
    U.ulysses_read_error()
    return lib


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(L, logits, labels, P):
    dev = logits.device
    S = torch.full((P,), -1.0, dtype=torch.float32, device=dev)
    C = torch.full((P,), -1, dtype=torch.int64, device=dev)
    loss = torch.full((1,), -1.0, dtype=torch.float32, device=dev)
    T, V = logits.shape
    st = L.ulysses_loss_aggregate_noalloc(P, T, V, 1, _ptr(logits), _ptr(labels), -100, _ptr(S), _ptr(C),
                                          _ptr(loss), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, U.STATUS.get(st, st)
    return S, C, loss


def _with_workspace(L, logits, labels, P):
    dev = logits.device
    T, V = logits.shape
    n = ctypes.c_size_t(0)
    assert L.ulysses_loss_workspace_size(P, T, V, ctypes.byref(n)) == 0
    ws = torch.empty(max(256, n.value), dtype=torch.uint8, device=dev)
    S = torch.empty(P, dtype=torch.float32, device=dev)
    C = torch.empty(P, dtype=torch.int64, device=dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    st = L.ulysses_loss_aggregate(P, T, V, 1, _ptr(logits), _ptr(labels), -100, _ptr(S), _ptr(C), _ptr(loss),
                                  _ptr(ws), ws.numel(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, U.STATUS.get(st, st)
    return S, C, loss


def test_noalloc_matches_workspace_entry_point_twice(L):
    # two different calls in a row: the second sees the first call's leftovers
    for seed, (T, V, P) in ((1, (4096, 8192, 4)), (2, (2048, 1024, 8))):
        g = torch.Generator().manual_seed(seed)
        logits = torch.randn(T, V, generator=g).to(torch.bfloat16).cuda()
        labels = torch.randint(0, V, (T,), generator=g, dtype=torch.int32)
        labels[torch.rand(T, generator=g) < 0.2] = -100
        labels = labels.cuda()
        S0, C0, L0 = _with_workspace(L, logits, labels, P)
        S1, C1, L1 = _noalloc(L, logits, labels, P)
        torch.cuda.synchronize()
        assert torch.equal(C0, C1)
        assert torch.allclose(S1, S0, rtol=LOSS_REL, atol=0.0)
        assert abs(L1.item() - L0.item()) <= LOSS_REL * abs(L0.item())
    assert U.ulysses_read_error() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch(L):
    # 8192 shards of one token each need 8192 partials (128 KiB) > 64 KiB
    P, T, V = 8192, 8192, 64
    logits = torch.zeros(T, V, dtype=torch.bfloat16, device="cuda")
    labels = torch.zeros(T, dtype=torch.int32, device="cuda")
    S = torch.empty(P, dtype=torch.float32, device="cuda")
    C = torch.empty(P, dtype=torch.int64, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    st = L.ulysses_loss_aggregate_noalloc(P, T, V, 1, _ptr(logits), _ptr(labels), -100, _ptr(S), _ptr(C),
                                          _ptr(loss), None)
    assert st == 10   # ULY_ERR_WORKSPACE, nothing launched
