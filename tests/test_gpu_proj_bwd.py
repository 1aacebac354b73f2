"""GPU parity of the projections' backward (the adjoints of steps 2-3 and 5-6)
against the oracle's qkv_proj_rope_bwd / o_proj_bwd (fp64).

Bounds, element by element, from the arithmetic of the GPU path:
- the pre-pass rounds the rotated gradient dY to bf16: |dY_gpu - dY| <= 2^-8 |dY|
  (V heads are copied exactly);
- the GEMMs multiply bf16 operands exactly and accumulate in fp32 over K terms
  (at most one fp32 ulp per addition, since the tensor core's internal rounding
  is not specified: K 2^-23 of the sum of |terms|);
- dX and dO are rounded once to bf16: half an ulp, 2^-8 |value|.
So dX: 2^-8 |ref| + (2^-8 + K 2^-23) (|dY| |W|);  dW: (2^-8 + K 2^-23) (|dY|^T |X|);
dO: 2^-8 |ref| + K 2^-23 (|dY| |W_o|);  dW_o: K 2^-23 (|dY|^T |O|).
The |.| products are formed here from the oracle's rotation (oracle.rope).
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import f32_inputs
from long_context_sequence_all_b200 import ulysses as U

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -23   # one fp32 ulp per accumulation step
HALF_ULP = 2.0 ** -8


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    U.lib()
    U.ulysses_read_error()


def _dy_exact(dq, dk, dv, P, H, G, B, n, positions=None, base=1.0e6):
    """The exact dY [P*B*s][(H+2G)*128] (fp64): head -> seq and the rotation by -pos."""
    s = n // P
    f = lambda t, heads: oracle.head_to_seq(t.detach().cpu().double().numpy(), B, n, P, heads)
    q, k, v = f(dq, H), f(dk, G), f(dv, G)          # [P][B][s][heads][d]
    out = np.empty((P, B, s, H + 2 * G, 128))
    for r in range(P):
        t = r * s + np.arange(s)
        pos = np.broadcast_to(t, (B, s)) if positions is None else positions.numpy()[:, t]
        out[r, :, :, :H] = oracle.rope(q[r], -pos[:, :, None], base)
        out[r, :, :, H:H + G] = oracle.rope(k[r], -pos[:, :, None], base)
        out[r, :, :, H + G:] = v[r]
    return out.reshape(P * B * s, (H + 2 * G) * 128)


def _assert_within(got, ref, bound, what):
    g = got.detach().cpu().double().numpy().reshape(ref.shape)
    err = np.abs(g - ref)
    worst = float((err / bound).max())
    assert np.isfinite(g).all() and worst <= 1.0, f"{what}: worst err/bound {worst:.3f}, max err {err.max():.3e}"


@pytest.mark.parametrize("P,B,n,H,G,hidden,docs", [
    (2, 1, 256, 4, 2, 256, False),     # 2 token tiles, 4 k-steps of dW
    (2, 2, 424, 4, 2, 512, False),     # ragged token tile and ragged last k-step of dW, B > 1
    (4, 1, 512, 8, 4, 256, True),      # positions restarting per document
])
def test_qkv_projection_backward(P, B, n, H, G, hidden, docs):
    g = torch.Generator().manual_seed(n + hidden)
    s, d = n // P, 128
    x = torch.randn(P, B, s, hidden, generator=g).to(torch.bfloat16)
    w = (torch.randn((H + 2 * G) * d, hidden, generator=g) / hidden ** 0.5).to(torch.bfloat16)
    dq = torch.randn(P, B, H // P, n, d, generator=g).to(torch.bfloat16)
    dk = torch.randn(P, B, G // P, n, d, generator=g).to(torch.bfloat16)
    dv = torch.randn(P, B, G // P, n, d, generator=g).to(torch.bfloat16)
    positions = None
    if docs:
        cu = [0, 100, 101, 350, n]
        positions = torch.tensor(np.concatenate([np.arange(b - a) for a, b in zip(cu[:-1], cu[1:])]),
                                 dtype=torch.int32).repeat(B, 1)
    tab = U.ulysses_rope_table(n, d, 1.0e6)
    dx, dw = U.ulysses_qkv_proj_rope_bwd(x.cuda(), w.cuda(), P, H, G, tab, dq.cuda(), dk.cuda(), dv.cuda(),
                                         positions=None if positions is None else positions.cuda())
    torch.cuda.synchronize()
    dx_ref, dw_ref = oracle.qkv_proj_rope_bwd(f32_inputs(x), f32_inputs(w), f32_inputs(dq), f32_inputs(dk),
                                              f32_inputs(dv), P, H, G, d, 1.0e6,
                                              positions=None if positions is None else positions.numpy())
    dy = np.abs(_dy_exact(dq, dk, dv, P, H, G, B, n, positions))
    xa = np.abs(x.double().numpy().reshape(P * B * s, hidden))
    wa = np.abs(w.double().numpy())
    N, M = (H + 2 * G) * d, P * B * s
    bx = HALF_ULP * np.abs(dx_ref.reshape(M, hidden)) + (HALF_ULP + N * U32) * (dy @ wa) + 1e-6
    _assert_within(dx, dx_ref.reshape(M, hidden), bx, "dX")
    bw = (HALF_ULP + M * U32) * (dy.T @ xa) + 1e-6
    _assert_within(dw, dw_ref, bw, "dW")
    assert U.ulysses_read_error() == 0


@pytest.mark.parametrize("P,B,n,H,hidden", [
    (2, 1, 384, 8, 256),
    (4, 2, 200, 8, 512),     # ragged token tiles, ragged last k-step of dW_o
])
def test_output_projection_backward(P, B, n, H, hidden):
    g = torch.Generator().manual_seed(7 * n + H)
    s, d = n // P, 128
    o_seq = torch.randn(P, B, s, H, d, generator=g).to(torch.bfloat16)
    w_o = (torch.randn(hidden, H * d, generator=g) / (H * d) ** 0.5).to(torch.bfloat16)
    dy = torch.randn(P, B, s, hidden, generator=g).to(torch.bfloat16)
    do, dw_o = U.ulysses_o_proj_bwd(o_seq.cuda(), w_o.cuda(), dy.cuda(), P)
    torch.cuda.synchronize()
    o_head = oracle.seq_to_head(f32_inputs(o_seq), B, n, P, H)
    do_ref, dwo_ref = oracle.o_proj_bwd(o_head, f32_inputs(w_o), f32_inputs(dy), P)
    M = P * B * s
    dya = np.abs(dy.double().numpy().reshape(M, hidden))
    # |dY| |W_o| per (token, feature), taken to the head layout like dO itself
    prod = (dya @ np.abs(w_o.double().numpy())).reshape(P, B, s, H, d)
    prod_head = oracle.seq_to_head(prod, B, n, P, H)
    _assert_within(do, do_ref, HALF_ULP * np.abs(do_ref) + hidden * U32 * prod_head + 1e-6, "dO")
    oa = np.abs(o_seq.double().numpy().reshape(M, H * d))
    _assert_within(dw_o, dwo_ref, M * U32 * (dya.T @ oa) + 1e-6, "dW_o")
    assert U.ulysses_read_error() == 0


def test_qkv_projection_backward_qwen8k_shapes():
    """Qwen3-4B shapes at 8K (hidden 2560, 32 query / 8 KV heads, P = 4),
    every element of dX and dW against the oracle."""
    P, B, n, H, G, hidden, d = 4, 1, 8192, 32, 8, 2560, 128
    s = n // P
    g = torch.Generator().manual_seed(2560)
    x = torch.randn(P, B, s, hidden, generator=g).to(torch.bfloat16)
    w = (torch.randn((H + 2 * G) * d, hidden, generator=g) / hidden ** 0.5).to(torch.bfloat16)
    dq = (torch.randn(P, B, H // P, n, d, generator=g) * 0.05).to(torch.bfloat16)
    dk = (torch.randn(P, B, G // P, n, d, generator=g) * 0.05).to(torch.bfloat16)
    dv = (torch.randn(P, B, G // P, n, d, generator=g) * 0.05).to(torch.bfloat16)
    tab = U.ulysses_rope_table(n, d, 1.0e6)
    dx, dw = U.ulysses_qkv_proj_rope_bwd(x.cuda(), w.cuda(), P, H, G, tab, dq.cuda(), dk.cuda(), dv.cuda())
    dx2, dw2 = U.ulysses_qkv_proj_rope_bwd(x.cuda(), w.cuda(), P, H, G, tab, dq.cuda(), dk.cuda(), dv.cuda())
    torch.cuda.synchronize()
    # dW's 480 tiles run as two k-halves each, added into a zeroed dW: still the same bits every call
    assert torch.equal(dw, dw2) and torch.equal(dx, dx2)
    dx_ref, dw_ref = oracle.qkv_proj_rope_bwd(f32_inputs(x), f32_inputs(w), f32_inputs(dq), f32_inputs(dk),
                                              f32_inputs(dv), P, H, G, d, 1.0e6)
    dy = np.abs(_dy_exact(dq, dk, dv, P, H, G, B, n))
    M, N = P * B * s, (H + 2 * G) * d
    bx = HALF_ULP * np.abs(dx_ref.reshape(M, hidden)) + (HALF_ULP + N * U32) * (dy @ np.abs(w.double().numpy())) + 1e-6
    _assert_within(dx, dx_ref.reshape(M, hidden), bx, "dX 8K")
    bw = (HALF_ULP + M * U32) * (dy.T @ np.abs(x.double().numpy().reshape(M, hidden))) + 1e-6
    _assert_within(dw, dw_ref, bw, "dW 8K")
    assert U.ulysses_read_error() == 0


def test_output_projection_backward_qwen8k_shapes():
    """Qwen3-4B shapes at 8K (hidden 2560, 32 query heads, P = 4): 320 output
    tiles of dW_o over 128 k-steps, so each tile's contraction runs as two
    halves added into a zeroed dW_o.  Every element of dO and dW_o against the
    oracle, and two calls give the same bits."""
    P, B, n, H, hidden, d = 4, 1, 8192, 32, 2560, 128
    s = n // P
    g = torch.Generator().manual_seed(8192 + hidden)
    o_seq = torch.randn(P, B, s, H, d, generator=g).to(torch.bfloat16)
    w_o = (torch.randn(hidden, H * d, generator=g) / (H * d) ** 0.5).to(torch.bfloat16)
    dy = torch.randn(P, B, s, hidden, generator=g).to(torch.bfloat16)
    do, dw_o = U.ulysses_o_proj_bwd(o_seq.cuda(), w_o.cuda(), dy.cuda(), P)
    do2, dw_o2 = U.ulysses_o_proj_bwd(o_seq.cuda(), w_o.cuda(), dy.cuda(), P)
    torch.cuda.synchronize()
    assert torch.equal(dw_o, dw_o2) and torch.equal(do, do2)
    o_head = oracle.seq_to_head(f32_inputs(o_seq), B, n, P, H)
    do_ref, dwo_ref = oracle.o_proj_bwd(o_head, f32_inputs(w_o), f32_inputs(dy), P)
    M = P * B * s
    dya = np.abs(dy.double().numpy().reshape(M, hidden))
    prod = (dya @ np.abs(w_o.double().numpy())).reshape(P, B, s, H, d)
    prod_head = oracle.seq_to_head(prod, B, n, P, H)
    _assert_within(do, do_ref, HALF_ULP * np.abs(do_ref) + hidden * U32 * prod_head + 1e-6, "dO 8K")
    oa = np.abs(o_seq.double().numpy().reshape(M, H * d))
    _assert_within(dw_o, dwo_ref, M * U32 * (dya.T @ oa) + 1e-6, "dW_o 8K")
    assert U.ulysses_read_error() == 0
