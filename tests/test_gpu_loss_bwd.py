"""GPU parity of the fused loss aggregation + gradient (dL/dlogits with the
global valid-token count as denominator) against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_sequence_all_b200 import ulysses as U
from long_context_sequence_all_b200.workloads import IGNORE_INDEX, make_inputs

pytestmark = pytest.mark.gpu

# dlogits tolerance: bf16 output rounds to nearest (2^-9 relative), fp32 output
# carries the fp32 logsumexp error (~1e-6 relative); plus 1e-6 of the 1/C scale
# for entries near zero.
REL = {torch.bfloat16: 2.0 ** -8, torch.float32: 1e-5}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    U.lib()
    U.ulysses_read_error()


def _check(logits, labels, P):
    S, C, L, dz = U.ulysses_loss_aggregate_bwd(logits.cuda(), labels.cuda(), P)
    torch.cuda.synchronize()
    g, Cg = oracle.loss_grad(logits.float().numpy(), labels.numpy())
    got = dz.float().cpu().numpy()
    assert int(C.sum().item()) == Cg
    if Cg == 0:
        assert not got.any() and math.isnan(L.item())
        return S, C, L, dz
    tol = REL[logits.dtype] * np.abs(g) + 1e-6 / Cg
    bad = np.abs(got - g) > tol
    assert not bad.any(), (np.argwhere(bad)[:5], got[bad][:5], g[bad][:5])
    # the loss values are the forward entry point's, bit for bit
    S2, C2, L2 = U.ulysses_loss_aggregate(logits.cuda(), labels.cuda(), P)
    assert torch.equal(S.cpu(), S2.cpu()) and torch.equal(C.cpu(), C2.cpu())
    assert torch.equal(L.cpu(), L2.cpu())
    return S, C, L, dz


@pytest.mark.parametrize("T,V,P,dtype", [(64, 8192, 4, torch.bfloat16), (40, 200, 8, torch.float32),
                                         (96, 1024, 3, torch.bfloat16), (8, 8, 8, torch.bfloat16),
                                         (48, 1000, 4, torch.float32)])
def test_loss_bwd_small(T, V, P, dtype):
    g = torch.Generator().manual_seed(T * V + 1)
    logits = (torch.randn(T, V, generator=g) * 2).to(dtype)
    labels = torch.randint(0, V, (T,), generator=g, dtype=torch.int32)
    labels[torch.rand(T, generator=g) < 0.25] = IGNORE_INDEX
    labels[: T // P] = IGNORE_INDEX            # a shard with no counted token
    _check(logits, labels, P)


def test_loss_bwd_all_ignored_and_bad_labels():
    T, V, P = 32, 256, 4
    logits = torch.randn(T, V).to(torch.bfloat16)
    labels = torch.full((T,), IGNORE_INDEX, dtype=torch.int32)
    _check(logits, labels, P)                  # every row 0, loss NaN
    labels = torch.randint(0, V, (T,), dtype=torch.int32)
    labels[3], labels[9] = V, -5               # invalid: error word, zero rows, not counted
    U.ulysses_read_error()
    S, C, L, dz = U.ulysses_loss_aggregate_bwd(logits.cuda(), labels.cuda(), P)
    torch.cuda.synchronize()
    assert U.ulysses_read_error() & (1 << 8)
    assert not dz[3].float().any() and not dz[9].float().any()
    assert int(C.sum().item()) == T - 2
    ok = labels.clone()
    ok[3] = ok[9] = IGNORE_INDEX
    g, Cg = oracle.loss_grad(logits.float().numpy(), ok.numpy())
    assert np.abs(dz.float().cpu().numpy() - g).max() <= 2.0 ** -8 * np.abs(g).max() + 1e-6 / Cg


def test_loss_bwd_workload_sampled_rows():
    """The 64K workload's logits (4 x 16384 tokens, V = 8192): dL/dz on sampled
    rows against the oracle (whose per-row gradient scales with 1/C), and the
    row-sum invariant on every row."""
    inp = make_inputs("qwen64k", with_grad_inputs=False)
    z, y, P = inp["logits"], inp["labels"], inp["P"]
    S, C, L, dz = U.ulysses_loss_aggregate_bwd(z.cuda(), y.cuda(), P)
    torch.cuda.synchronize()
    assert U.ulysses_read_error() == 0
    yn = y.numpy()
    T = yn.size
    counted = (yn != IGNORE_INDEX) & (yn >= 0)
    Ctot = int(counted.sum())
    assert int(C.sum().item()) == Ctot
    rows = np.unique(np.concatenate([np.linspace(0, T - 1, 48).astype(np.int64), [0, T // P, T - 1]]))
    idx = torch.as_tensor(rows)
    g, Csub = oracle.loss_grad(z[idx].float().numpy(), yn[rows])
    if Csub:
        g = g * (Csub / Ctot)
    got = dz[idx.cuda()].float().cpu().numpy()
    tol = 2.0 ** -8 * np.abs(g) + 1e-6 / Ctot
    assert (np.abs(got - g) <= tol).all()
    # every counted row sums to ~0 (softmax sums to one; the label entry ~ -1/C
    # carries up to 2^-9/C of bf16 rounding), every other row is exactly 0
    rs = dz.float().sum(dim=1).cpu().numpy()
    assert np.abs(rs[counted]).max() < 5e-3 / Ctot
    assert not dz[torch.as_tensor(~counted).cuda()].float().any()
