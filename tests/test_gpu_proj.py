"""GPU parity of the projections either side of Ulysses attention (tcgen05
GEMMs with the all-to-alls folded in): the QKV projection with rotary
positions written straight to the head layout, and the output projection
read straight from it, against the fp64 oracle.  Small shapes element by
element (several tiles, ragged tails, B > 1, per-document positions); the
Qwen3-4B 64K shapes on sampled rows, which the oracle computes one by one
(projection rows are independent; the positions argument places them)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_bf16_close, f32_inputs, sample_rows
from long_context_sequence_all_b200 import ulysses as U

pytestmark = pytest.mark.gpu

D = 128
BASE = 1.0e6


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    U.lib()
    U.ulysses_read_error()


def _weights(rows, cols, g):
    return (torch.randn(rows, cols, generator=g) / cols ** 0.5).to(torch.bfloat16)


def test_rope_table_matches_oracle():
    tab = U.ulysses_rope_table(70000, D, BASE)
    torch.cuda.synchronize()
    pos = np.array([0, 1, 2, 127, 4095, 65535, 69999])
    t = tab.cpu().numpy()[pos]                                  # [p][64][2]
    ones = np.zeros((pos.size, D))
    ones[:, :D // 2] = 1.0                                      # rotate (1, 0) pairs: gives (cos, sin)
    ref = oracle.rope(ones, pos, BASE)
    assert np.abs(t[..., 0] - ref[:, :D // 2]).max() < 1e-7
    assert np.abs(t[..., 1] - ref[:, D // 2:]).max() < 1e-7


@pytest.mark.parametrize("P,B,s,hidden,H,G,docs", [
    (4, 1, 80, 128, 8, 4, False),      # 320 rows: 2 full row tiles + a ragged one
    (2, 2, 100, 192, 4, 2, False),     # B > 1: row tiles cross (rank, batch) blocks
    (4, 1, 256, 256, 8, 4, True),      # positions restarting at packed documents
    (8, 1, 64, 2560, 16, 8, False),    # the Qwen3-4B hidden size, 40 k-steps
])
def test_qkv_proj_small_elementwise(P, B, s, hidden, H, G, docs):
    g = torch.Generator().manual_seed(P * 100 + s)
    n = P * s
    x = torch.randn(P, B, s, hidden, generator=g).to(torch.bfloat16)
    w = _weights((H + 2 * G) * D, hidden, g)
    positions = None
    if docs:
        cu = [0, 100, 101, 600, n]
        pos = np.concatenate([np.arange(b - a) for a, b in zip(cu[:-1], cu[1:])])
        positions = np.tile(pos, (B, 1)).astype(np.int32)
    tab = U.ulysses_rope_table(n, D, BASE)
    q, k, v = U.ulysses_qkv_proj_rope(x.cuda(), w.cuda(), P, H, G, tab,
                                      positions=None if positions is None else torch.from_numpy(positions).cuda())
    torch.cuda.synchronize()
    rq, rk, rv = oracle.qkv_proj_rope(f32_inputs(x), f32_inputs(w), P, H, G, D, BASE, positions=positions)
    assert_bf16_close(q.cpu(), rq, "Q")
    assert_bf16_close(k.cpu(), rk, "K")
    assert_bf16_close(v.cpu(), rv, "V")
    assert U.ulysses_read_error() == 0


@pytest.mark.parametrize("P,B,n,hidden,H", [(4, 1, 320, 256, 8), (2, 2, 200, 512, 4), (4, 1, 512, 2560, 32)])
def test_o_proj_small_elementwise(P, B, n, hidden, H):
    g = torch.Generator().manual_seed(n + hidden)
    o = torch.randn(P, B, H // P, n, D, generator=g).to(torch.bfloat16)
    w = _weights(hidden, H * D, g)
    y = U.ulysses_o_proj(o.cuda(), w.cuda(), P)
    torch.cuda.synchronize()
    ref = oracle.o_proj(f32_inputs(o), f32_inputs(w), P)
    assert_bf16_close(y.cpu(), ref, "Y")
    assert U.ulysses_read_error() == 0


def test_position_outside_table_sets_error_word():
    """A position past the table is a data error: reported in the error word
    (no fault), the row rotated as position 0."""
    P, B, s, hidden, H, G = 2, 1, 64, 128, 2, 2
    g = torch.Generator().manual_seed(9)
    x = torch.randn(P, B, s, hidden, generator=g).to(torch.bfloat16)
    w = _weights((H + 2 * G) * D, hidden, g)
    tab = U.ulysses_rope_table(P * s, D, BASE)
    pos = torch.arange(P * s, dtype=torch.int32).reshape(1, -1).clone()
    pos[0, 5] = P * s + 3
    q, _, _ = U.ulysses_qkv_proj_rope(x.cuda(), w.cuda(), P, H, G, tab, positions=pos.cuda())
    torch.cuda.synchronize()
    assert U.ulysses_read_error() & (1 << 2)
    pos0 = pos.numpy().copy()
    pos0[0, 5] = 0
    rq, _, _ = oracle.qkv_proj_rope(f32_inputs(x), f32_inputs(w), P, H, G, D, BASE, positions=pos0)
    assert_bf16_close(q.cpu(), rq, "Q")


@pytest.fixture(scope="module")
def qwen64k():
    """Qwen3-4B shapes at 64K on P = 4: hidden 2560, H = 32, G = 8, d = 128."""
    P, B, n, hidden, H, G = 4, 1, 65536, 2560, 32, 8
    g = torch.Generator().manual_seed(64)
    x = torch.randn(P, B, n // P, hidden, generator=g).to(torch.bfloat16)
    w = _weights((H + 2 * G) * D, hidden, g)
    wo = _weights(hidden, H * D, g)
    return dict(P=P, B=B, n=n, hidden=hidden, H=H, G=G, x=x, w=w, wo=wo)


def test_qkv_proj_qwen64k_sampled_rows(qwen64k):
    c = qwen64k
    P, n, H, G = c["P"], c["n"], c["H"], c["G"]
    tab = U.ulysses_rope_table(n, D, BASE)
    q, k, v = U.ulysses_qkv_proj_rope(c["x"].cuda(), c["w"].cuda(), P, H, G, tab)
    torch.cuda.synchronize()
    assert U.ulysses_read_error() == 0
    rows = sample_rows(n, P, k=48)
    x_nat = c["x"].reshape(n, c["hidden"])                       # B = 1: seq layout = natural order
    rq, rk, rv = oracle.qkv_proj_rope(f32_inputs(x_nat[rows])[None, None], f32_inputs(c["w"]), 1, H, G, D,
                                      BASE, positions=rows[None])
    qn = q.cpu().permute(1, 0, 2, 3, 4).reshape(1, H, n, D)[0][:, rows]   # [H][rows][d]
    kn = k.cpu().permute(1, 0, 2, 3, 4).reshape(1, G, n, D)[0][:, rows]
    vn = v.cpu().permute(1, 0, 2, 3, 4).reshape(1, G, n, D)[0][:, rows]
    assert_bf16_close(qn, rq[0, 0], "Q rows")
    assert_bf16_close(kn, rk[0, 0], "K rows")
    assert_bf16_close(vn, rv[0, 0], "V rows")


def test_o_proj_qwen64k_sampled_rows(qwen64k):
    c = qwen64k
    P, n, H = c["P"], c["n"], c["H"]
    g = torch.Generator().manual_seed(65)
    o = torch.randn(P, 1, H // P, n, D, generator=g).to(torch.bfloat16)
    y = U.ulysses_o_proj(o.cuda(), c["wo"].cuda(), P)
    torch.cuda.synchronize()
    assert U.ulysses_read_error() == 0
    rows = sample_rows(n, P, k=48)
    o_rows = o[:, :, :, rows].permute(1, 0, 2, 3, 4).reshape(1, 1, H, rows.size, D)   # P = 1 head layout
    ref = oracle.o_proj(f32_inputs(o_rows), f32_inputs(c["wo"]), 1)[0, 0]            # [rows][hidden]
    assert_bf16_close(y.cpu().reshape(n, c["hidden"])[rows], ref, "Y rows")
