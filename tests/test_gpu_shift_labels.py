"""GPU parity of the label shift done before sharding: bit-exact against the
oracle (integer work), with and without packed documents and padding, at
small ragged shapes and at the packed workload's full size; and end to end
with the loss: shifted + sharded + token-weighted equals the plain unsharded
next-token loss."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from helpers import LOSS_REL
from long_context_sequence_all_b200 import ulysses as U
from long_context_sequence_all_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    U.lib()
    U.ulysses_read_error()


@pytest.mark.parametrize("B,n,P,cu,valid", [
    (1, 64, 4, None, None),
    (3, 40, 8, None, 37),                        # padding tail, B > 1
    (2, 1000, 8, [0, 1, 2, 513, 700, 1000], 998), # one-token documents, boundary at a shard edge
    (1, 8, 8, [0, 3, 8], 8),                      # one token per rank
    (1, 24, 4, None, 0),                          # no valid token
    (1, 4096, 4, [0, 1024, 2048, 3072, 4096], None),  # documents on shard boundaries
])
def test_shift_small_bit_exact(B, n, P, cu, valid):
    g = torch.Generator().manual_seed(n + B)
    ids = torch.randint(0, 151936, (B, n), generator=g, dtype=torch.int32)
    cut = None if cu is None else torch.tensor(cu, dtype=torch.int32)
    lab = U.ulysses_shift_labels(ids.cuda(), P, cu_seqlens=None if cut is None else cut.cuda(), valid_len=valid)
    torch.cuda.synchronize()
    ref = oracle.shift_labels(ids.numpy(), P, cu_seqlens=cu, valid_len=valid)
    assert np.array_equal(lab.cpu().numpy(), ref)
    assert U.ulysses_read_error() == 0


def test_shift_packed_workload_full_size():
    """The packed workload's documents and padding at full size."""
    inp = make_inputs("packed", with_loss=False)
    n, P, cu = inp["n"], inp["P"], inp["cu_seqlens"]
    g = torch.Generator().manual_seed(77)
    ids = torch.randint(0, 151936, (1, n), generator=g, dtype=torch.int32)
    valid = inp["real_tokens"]   # positions past it are the padding segment
    lab = U.ulysses_shift_labels(ids.cuda(), P, cu_seqlens=cu.cuda(), valid_len=valid)
    torch.cuda.synchronize()
    ref = oracle.shift_labels(ids.numpy(), P, cu_seqlens=cu.numpy(), valid_len=valid)
    assert np.array_equal(lab.cpu().numpy(), ref)


def test_shifted_sharded_gpu_loss_equals_unsharded_next_token_loss():
    """Shift (GPU) -> shard -> token-weighted loss (GPU) against torch's plain
    next-token cross entropy over the whole unsharded sequence."""
    B, n, P, V = 1, 8192, 4, 8192
    g = torch.Generator().manual_seed(3)
    ids = torch.randint(0, V, (B, n), generator=g, dtype=torch.int32)
    logits = torch.randn(B, n, V, generator=g).to(torch.bfloat16)
    lab = U.ulysses_shift_labels(ids.cuda(), P)
    z = logits.reshape(B, P, n // P, V).transpose(0, 1).reshape(-1, V).contiguous().cuda()
    S, C, L = U.ulysses_loss_aggregate(z, lab.reshape(-1), P)
    torch.cuda.synchronize()
    ref = F.cross_entropy(logits[:, :-1].double().reshape(-1, V), ids[:, 1:].reshape(-1).long())
    assert int(C.sum()) == B * (n - 1)
    assert abs(float(L) - ref.item()) <= LOSS_REL * abs(ref.item())
