"""Pins for the CPU oracle: each check ties it to something other than itself
(closed forms, the pages' worked examples, brute force, library routines,
invariants, finite differences), chosen so that a plausible mistake in the
oracle (a dropped term, a wrong sign or index, a transposed operand) fails.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import MASK_CAUSAL, MASK_DOC_CAUSAL, MASK_NONE

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def _randn(*shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float32)


def _seq(x, P):  # natural [B][n][Hx][d] -> seq layout [P][B][n/P][Hx][d]
    B, n, Hx, d = x.shape
    return np.ascontiguousarray(x.reshape(B, P, n // P, Hx, d).transpose(1, 0, 2, 3, 4))


def _nat(x):  # seq layout -> natural
    P, B, s, Hx, d = x.shape
    return np.ascontiguousarray(x.transpose(1, 0, 2, 3, 4).reshape(B, P * s, Hx, d))


# ---------------------------------------------------------------- permutations

@pytest.mark.parametrize("B,n,P,heads,d", [(1, 16, 4, 8, 3), (2, 24, 4, 4, 2), (1, 12, 3, 6, 5),
                                           (3, 8, 2, 2, 1), (1, 8, 1, 4, 2)])
def test_seq_to_head_closed_form(B, n, P, heads, d):
    """Every destination element holds the source element the all-to-all
    definition names: dst[r2][b][hh][r*s+tt][:] = src[r][b][tt][r2*hl+hh][:].
    Payload = global element index (iota), so this also proves bijectivity."""
    s, hl = n // P, heads // P
    src = np.arange(P * B * s * heads * d, dtype=np.int32).reshape(P, B, s, heads, d)
    dst = oracle.seq_to_head(src, B, n, P, heads)
    assert dst.shape == (P, B, hl, n, d)
    # independent formulation: split heads into (rank, local head) and n into (rank, tt)
    expect = src.reshape(P, B, s, P, hl, d).transpose(3, 1, 4, 0, 2, 5).reshape(P, B, hl, n, d)
    assert np.array_equal(dst, expect)
    assert np.array_equal(np.sort(dst.ravel()), np.arange(dst.size, dtype=np.int32))
    # spot-check a few indices by the formula, element by element
    for (r2, b, hh, t, x) in [(0, 0, 0, 0, 0), (P - 1, B - 1, hl - 1, n - 1, d - 1), (P // 2, 0, 0, n // 2, 0)]:
        r, tt = divmod(t, s)
        assert dst[r2, b, hh, t, x] == src[r, b, tt, r2 * hl + hh, x]


@pytest.mark.parametrize("dtype", [np.uint16, np.float32, np.float64, np.int8])
def test_roundtrip_identity(dtype):
    B, n, P, heads, d = 2, 32, 4, 8, 16
    x = rng.integers(-100, 100, size=(P, B, n // P, heads, d)).astype(dtype)
    y = oracle.head_to_seq(oracle.seq_to_head(x, B, n, P, heads), B, n, P, heads)
    assert y.dtype == x.dtype and np.array_equal(y.view(np.uint8), x.view(np.uint8))
    z = oracle.seq_to_head(oracle.head_to_seq(oracle.seq_to_head(x, B, n, P, heads), B, n, P, heads),
                           B, n, P, heads)
    assert np.array_equal(z, oracle.seq_to_head(x, B, n, P, heads))


def test_sharding_matches_pages_examples():
    """The pages print worked sharding examples (n, P -> n/P per rank).  After
    the first all-to-all, rank r2's copy of head hh holds, at rows
    [r*shard_len, (r+1)*shard_len), exactly the tokens rank r sent."""
    ex = json.load(open(os.path.join(GOLDEN, "sharding_examples.json")))["examples"]
    for e in ex:
        n, P, L = e["n"], e["P"], e["shard_len"]
        heads = P
        B, d = 1, 1
        s = n // P
        assert s == L, e["cite"]
        # payload: sending rank id in the high bits, position in the low bits
        src = np.empty((P, B, s, heads, d), np.int64)
        for r in range(P):
            src[r] = (r << 32) + (r * s + np.arange(s)).reshape(1, s, 1, 1)
        dst = oracle.seq_to_head(src, B, n, P, heads)
        for r2 in (0, P - 1):
            col = dst[r2, 0, 0, :, 0]
            assert np.array_equal(col & 0xFFFFFFFF, np.arange(n))
            assert np.array_equal(col >> 32, np.repeat(np.arange(P), L))


def test_all_to_all_volume():
    """Each rank keeps 1/P of its elements and sends (P-1)/P of them: the
    per-rank volume the pages give for each all-to-all (O(n*d/P))."""
    B, n, P, heads, d = 1, 64, 4, 8, 2
    s, hl = n // P, heads // P
    tag = np.zeros((P, B, s, heads, d), np.int32)
    for r in range(P):
        tag[r] = r
    dst = oracle.seq_to_head(tag, B, n, P, heads)
    moved = sum(int((dst[r2] != r2).sum()) for r2 in range(P))
    assert moved == (P - 1) * B * n * heads * d // P


# ------------------------------------------------------------------ attention

def _sdpa_ref(q, k, v, mask, cu=None):
    """torch scaled_dot_product_attention in float64 (library routine), GQA by
    repeating each KV head over its consecutive group of query heads."""
    B, n, H, d = q.shape
    G = k.shape[2]
    qt = torch.from_numpy(q.astype(np.float64)).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k.astype(np.float64)).permute(0, 2, 1, 3).repeat_interleave(H // G, dim=1)
    vt = torch.from_numpy(v.astype(np.float64)).permute(0, 2, 1, 3).repeat_interleave(H // G, dim=1)
    if mask == MASK_NONE:
        o = F.scaled_dot_product_attention(qt, kt, vt)
        am = torch.ones(n, n, dtype=torch.bool)
    elif mask == MASK_CAUSAL:
        o = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
        am = torch.ones(n, n, dtype=torch.bool).tril()
    else:
        doc = torch.zeros(n, dtype=torch.int64)
        for e in range(len(cu) - 1):
            doc[cu[e]:cu[e + 1]] = e
        am = (doc[:, None] == doc[None, :]) & torch.ones(n, n, dtype=torch.bool).tril()
        o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=am)
    scores = (qt @ kt.transpose(-1, -2)) / math.sqrt(d)
    lse = torch.logsumexp(scores.masked_fill(~am, float("-inf")), dim=-1)
    return o.permute(0, 2, 1, 3).numpy(), lse.numpy()


@pytest.mark.parametrize("mask", [MASK_NONE, MASK_CAUSAL, MASK_DOC_CAUSAL])
@pytest.mark.parametrize("B,n,H,G,d", [(1, 40, 4, 2, 16), (2, 33, 6, 3, 8), (1, 64, 4, 4, 32)])
def test_attention_matches_torch_sdpa(mask, B, n, H, G, d):
    q, k, v = _randn(B, n, H, d), _randn(B, n, G, d), _randn(B, n, G, d)
    cu = np.array([0, 7, 20, n], np.int32) if mask == MASK_DOC_CAUSAL else None
    o, lse = oracle.attention_fwd(q, k, v, mask=mask, cu_seqlens=cu)
    o_ref, lse_ref = _sdpa_ref(q, k, v, mask, cu)
    assert np.abs(o - o_ref).max() < 1e-12
    assert np.abs(lse - lse_ref).max() < 1e-12


def test_attention_brute_force_tiny():
    """n <= 32: materialise the n x n score matrix, exponentiate, normalise."""
    n, d = 9, 4
    q, k, v = _randn(1, n, 1, d, scale=2), _randn(1, n, 1, d, scale=2), _randn(1, n, 1, d)
    o, lse = oracle.attention_fwd(q, k, v, mask=MASK_CAUSAL)
    Q, K, V = (x[0, :, 0, :].astype(np.float64) for x in (q, k, v))
    for i in range(n):
        w = np.array([math.exp(float(Q[i] @ K[j]) / 2.0) for j in range(i + 1)])  # 1/sqrt(4) = 1/2
        assert abs(lse[0, 0, i] - math.log(w.sum())) < 1e-12
        assert np.abs(o[0, i, 0] - (w[:, None] * V[: i + 1]).sum(0) / w.sum()).max() < 1e-12


def test_zero_keys_give_prefix_mean():
    """K = 0: every visible score is 0, so O_i = mean(V_0..V_i), LSE_i = log(i+1)."""
    n, H, d = 50, 2, 8
    q, v = _randn(1, n, H, d), _randn(1, n, 1, d)
    k = np.zeros((1, n, 1, d), np.float32)
    o, lse = oracle.attention_fwd(q, k, v, mask=MASK_CAUSAL)
    V = v[0, :, 0, :].astype(np.float64)
    prefix = np.cumsum(V, axis=0) / np.arange(1, n + 1)[:, None]
    for h in range(H):
        assert np.abs(o[0, :, h] - prefix).max() < 1e-13
        assert np.abs(lse[0, h] - np.log(np.arange(1, n + 1))).max() < 1e-13
    # non-causal: every row is the full mean, LSE = log n
    o, lse = oracle.attention_fwd(q, k, v, mask=MASK_NONE)
    assert np.abs(o[0, :, 0] - V.mean(0)).max() < 1e-13
    assert np.abs(lse - math.log(n)).max() < 1e-13


def test_constant_values_and_dominant_key():
    n, d = 24, 8
    q, k = _randn(1, n, 1, d), _randn(1, n, 1, d)
    c = _randn(d)
    v = np.broadcast_to(c, (1, n, 1, d)).copy()
    o, _ = oracle.attention_fwd(q, k, v, mask=MASK_CAUSAL)
    assert np.abs(o[0, :, 0] - c).max() < 1e-14
    # one key aligned with every query and huge: O_i -> V_j* for rows that see j*
    jstar = 5
    qq = np.zeros((1, n, 1, d), np.float32); qq[..., 0] = 1.0
    kk = np.zeros((1, n, 1, d), np.float32); kk[0, jstar, 0, 0] = 400.0
    vv = _randn(1, n, 1, d)
    o, lse = oracle.attention_fwd(qq, kk, vv, mask=MASK_CAUSAL)
    assert np.abs(o[0, jstar:, 0] - vv[0, jstar, 0]).max() < 1e-40 + 1e-12
    assert abs(lse[0, 0, jstar] - 400.0 / math.sqrt(d)) < 1e-12


def test_single_document_is_causal_and_mha_special_case():
    B, n, H, d = 1, 48, 4, 16
    q, k, v = _randn(B, n, H, d), _randn(B, n, H, d), _randn(B, n, H, d)
    o1, l1 = oracle.attention_fwd(q, k, v, mask=MASK_DOC_CAUSAL, cu_seqlens=np.array([0, n], np.int32))
    o2, l2 = oracle.attention_fwd(q, k, v, mask=MASK_CAUSAL)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    # G = H is plain MHA: head h uses KV head h; compare per head with a 1-head call
    for h in range(H):
        oh, lh = oracle.attention_fwd(q[:, :, h:h + 1], k[:, :, h:h + 1], v[:, :, h:h + 1])
        assert np.array_equal(oh[:, :, 0], o2[:, :, h]) and np.array_equal(lh[:, 0], l2[:, h])
    # documents are independent: a doc's rows equal attention over that doc alone
    cu = np.array([0, 20, n], np.int32)
    o3, l3 = oracle.attention_fwd(q, k, v, mask=MASK_DOC_CAUSAL, cu_seqlens=cu)
    o4, l4 = oracle.attention_fwd(q[:, 20:], k[:, 20:], v[:, 20:], mask=MASK_CAUSAL)
    assert np.array_equal(o3[:, 20:], o4) and np.array_equal(l3[:, :, 20:], l4)


def test_gqa_group_mapping():
    """Query head q reads KV head floor(q / (H/G)): swapping the data of KV
    head 1 changes exactly query heads 2..3 of a 4-query/2-KV layer."""
    B, n, H, G, d = 1, 16, 4, 2, 8
    q, k, v = _randn(B, n, H, d), _randn(B, n, G, d), _randn(B, n, G, d)
    o, _ = oracle.attention_fwd(q, k, v)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 1], v2[:, :, 1] = _randn(B, n, d), _randn(B, n, d)
    o2, _ = oracle.attention_fwd(q, k2, v2)
    assert np.array_equal(o[:, :, :2], o2[:, :, :2])
    assert not np.allclose(o[:, :, 2:], o2[:, :, 2:])


# -------------------------------------------------------------- decomposition

@pytest.mark.parametrize("mask", [MASK_NONE, MASK_CAUSAL, MASK_DOC_CAUSAL])
@pytest.mark.parametrize("B,n,P,H,G,d", [(1, 32, 4, 8, 4, 8), (2, 24, 2, 4, 2, 16), (1, 48, 4, 4, 4, 8)])
def test_ulysses_equals_full_attention(mask, B, n, P, H, G, d):
    """Heads are independent, so shard -> all-to-all -> per-rank attention ->
    all-to-all reproduces plain attention exactly (same routine, same data,
    same order: bitwise)."""
    q, k, v, do = _randn(B, n, H, d), _randn(B, n, G, d), _randn(B, n, G, d), _randn(B, n, H, d)
    cu = np.array([0, 5, 17, n], np.int32) if mask == MASK_DOC_CAUSAL else None
    o, lse = oracle.attention_fwd(q, k, v, mask=mask, cu_seqlens=cu)
    ou, lu = oracle.ulysses_fwd(_seq(q, P), _seq(k, P), _seq(v, P), P, mask=mask, cu_seqlens=cu)
    assert np.array_equal(_nat(ou), o)
    # LSE in head layout [P][B][H/P][n] -> [B][H][n]
    assert np.array_equal(lu.transpose(1, 0, 2, 3).reshape(B, H, n), lse)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, mask=mask, cu_seqlens=cu)
    uq, uk, uv = oracle.ulysses_bwd(_seq(q, P), _seq(k, P), _seq(v, P), _seq(do, P), P,
                                    mask=mask, cu_seqlens=cu)
    assert np.array_equal(_nat(uq), dq) and np.array_equal(_nat(uk), dk) and np.array_equal(_nat(uv), dv)


def test_ulysses_rejects_indivisible_shapes():
    """Every rank must own whole query heads (H % P == 0), and the KV heads
    either split over the ranks (G % P == 0) or are copied to them (P % G == 0)."""
    k3 = _randn(1, 24, 3, 8)
    with pytest.raises(ValueError):          # G = 3 KV heads over P = 4: neither divides
        oracle.ulysses_fwd(_seq(_randn(1, 24, 12, 8), 4), _seq(k3, 4), _seq(k3, 4), 4)
    q4 = _randn(1, 32, 4, 8)
    with pytest.raises(ValueError):          # H = 6 query heads cannot split over P = 4
        oracle.ulysses_fwd(_seq(_randn(1, 32, 6, 8), 4), _seq(q4, 4), _seq(q4, 4), 4)


# ------------------------------------------------ KV heads fewer than ranks

def test_kv_replicate_with_as_many_kv_heads_as_ranks_is_seq_to_head():
    """With G == P each rank holds exactly one KV head either way, so the
    copying all-to-all reduces to the plain one (pinned by its closed form)."""
    B, n, P, d = 2, 16, 4, 3
    x = np.arange(P * B * (n // P) * P * d, dtype=np.int32).reshape(P, B, n // P, P, d)
    assert np.array_equal(oracle.kv_replicate_to_head(x, B, n, P, P),
                          oracle.seq_to_head(x, B, n, P, P))


@pytest.mark.parametrize("B,n,P,H,G", [(1, 16, 4, 8, 2), (2, 24, 8, 16, 2), (1, 8, 8, 8, 1),
                                       (1, 12, 4, 4, 1), (2, 32, 8, 32, 4)])
def test_kv_replicate_gives_each_rank_the_kv_head_of_its_query_heads(B, n, P, H, G):
    """GQA semantics rather than the copy formula: for every rank r and each of
    its query heads q = r*H/P + hh, the rank's KV copy at every position t is
    the natural-layout K[t][floor(q / (H/G))]."""
    d = 3
    k_nat = np.arange(B * n * G * d, dtype=np.int32).reshape(B, n, G, d)
    rep = oracle.kv_replicate_to_head(_seq(k_nat, P), B, n, P, G)
    assert rep.shape == (P, B, 1, n, d)
    hl, grp = H // P, H // G
    for r in range(P):
        for hh in range(hl):
            assert np.array_equal(rep[r, :, 0], k_nat[:, :, (r * hl + hh) // grp])


@pytest.mark.parametrize("P,G", [(4, 2), (8, 1), (8, 4), (4, 4)])
def test_kv_reduce_of_copies_is_copy_count_times_x(P, G):
    """The P/G copies of a KV head carry the same values, so summing them back
    gives (P/G) x exactly (a power of two: no rounding in fp64)."""
    B, n, d = 2, 24, 5
    x = _randn(P, B, n // P, G, d).astype(np.float64)
    rep = oracle.kv_replicate_to_head(x, B, n, P, G)
    assert np.array_equal(oracle.kv_reduce_to_seq(rep, B, n, P, G), x * (P // G))
    # a gradient that lives on one copy only comes back once, at its own head
    one = np.zeros_like(rep)
    one[P - 1] = rep[P - 1]
    back = oracle.kv_reduce_to_seq(one, B, n, P, G)
    kk = (P - 1) * G // P
    assert np.array_equal(back[:, :, :, kk], x[:, :, :, kk])
    assert not np.any(np.delete(back, kk, axis=3))


@pytest.mark.parametrize("mask", [MASK_NONE, MASK_CAUSAL, MASK_DOC_CAUSAL])
@pytest.mark.parametrize("B,n,P,H,G,d", [(1, 32, 4, 8, 2, 8), (2, 16, 8, 8, 1, 4), (1, 24, 4, 8, 1, 8)])
def test_ulysses_with_kv_copies_equals_full_attention(mask, B, n, P, H, G, d):
    """G < P: the decomposition with copied KV heads still reproduces plain GQA
    attention -- the forward bitwise (same routine, same data), the backward
    (whose KV gradients are now summed over the copies in another order) to
    fp64 rounding."""
    q, k, v, do = _randn(B, n, H, d), _randn(B, n, G, d), _randn(B, n, G, d), _randn(B, n, H, d)
    cu = np.array([0, 5, 13, n], np.int32) if mask == MASK_DOC_CAUSAL else None
    o, lse = oracle.attention_fwd(q, k, v, mask=mask, cu_seqlens=cu)
    ou, lu = oracle.ulysses_fwd(_seq(q, P), _seq(k, P), _seq(v, P), P, mask=mask, cu_seqlens=cu)
    assert np.array_equal(_nat(ou), o)
    assert np.array_equal(lu.transpose(1, 0, 2, 3).reshape(B, H, n), lse)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, mask=mask, cu_seqlens=cu)
    uq, uk, uv = oracle.ulysses_bwd(_seq(q, P), _seq(k, P), _seq(v, P), _seq(do, P), P,
                                    mask=mask, cu_seqlens=cu)
    assert np.array_equal(_nat(uq), dq)
    for got, ref in ((uk, dk), (uv, dv)):
        assert np.abs(_nat(got) - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


# ------------------------------------------------------------- label shift

def test_shift_labels_single_sequence_is_the_causal_lm_shift():
    """One document, no padding: label(t) = ids[t+1] and the last position is
    ignored -- the shift torch code writes as F.pad(ids[:, 1:], (0, 1), value=-100)
    -- laid out by shard (seq layout [P][B][n/P])."""
    B, n, P = 2, 24, 4
    ids = rng.integers(0, 1000, (B, n)).astype(np.int32)
    lab = oracle.shift_labels(ids, P)
    ref = F.pad(torch.from_numpy(ids)[:, 1:], (0, 1), value=-100).numpy()
    assert np.array_equal(lab, ref.reshape(B, P, n // P).transpose(1, 0, 2))
    # a one-document cu_seqlens changes nothing
    assert np.array_equal(oracle.shift_labels(ids, P, cu_seqlens=[0, n]), lab)
    # no valid token: everything ignored
    assert np.all(oracle.shift_labels(ids, P, valid_len=0) == -100)


def test_shifted_sharded_loss_equals_unsharded_causal_lm_loss():
    """Why the shift comes before sharding: the token-weighted loss over the P
    shards with the shifted labels equals the plain next-token loss of the whole
    sequence (torch cross_entropy of logits[:, :-1] against ids[:, 1:]); with
    packed documents and padding it equals the mean of every document's own
    next-token loss, each document computed alone."""
    B, n, P, V = 2, 32, 4, 11
    ids = rng.integers(0, V, (B, n)).astype(np.int32)
    logits = _randn(B, n, V)
    z_seq = logits.reshape(B, P, n // P, V).transpose(1, 0, 2, 3).reshape(-1, V)
    lab = oracle.shift_labels(ids, P)
    S, C, L, bad = oracle.loss_aggregate(z_seq, lab.reshape(-1), P)
    ref = F.cross_entropy(torch.tensor(logits[:, :-1], dtype=torch.float64).reshape(-1, V),
                          torch.from_numpy(ids[:, 1:]).reshape(-1).long())
    assert bad == 0 and C.sum() == B * (n - 1) and abs(L - ref.item()) < 1e-12
    # packed documents [0,5) [5,19) [19,30) and two padding tokens [30,32)
    cu, valid = [0, 5, 19, 30, 32], 30
    lab = oracle.shift_labels(ids, P, cu_seqlens=cu, valid_len=valid)
    S, C, L, bad = oracle.loss_aggregate(z_seq, lab.reshape(-1), P)
    tot, cnt = 0.0, 0
    for b in range(B):
        for a, e in zip(cu[:-2], cu[1:-1]):
            z = torch.tensor(logits[b, a:e - 1], dtype=torch.float64)
            tot += F.cross_entropy(z, torch.from_numpy(ids[b, a + 1:e]).long(), reduction="sum").item()
            cnt += e - a - 1
    assert C.sum() == cnt and abs(L - tot / cnt) < 1e-12
    # the label of a shard's last position is the next shard's first token
    lab = oracle.shift_labels(ids, P)
    s = n // P
    for r in range(P - 1):
        assert np.array_equal(lab[r, :, s - 1], ids[:, (r + 1) * s])


# ------------------------------------------------------------------- backward

def _loss(q, k, v, do, mask, cu):
    o, _ = oracle.attention_fwd(q, k, v, mask=mask, cu_seqlens=cu)
    return float((o * do.astype(np.float64)).sum())


@pytest.mark.parametrize("mask", [MASK_NONE, MASK_CAUSAL, MASK_DOC_CAUSAL])
def test_backward_finite_differences(mask):
    """Central differences of sum(O * dO).  Inputs are multiples of 2^-8 and the
    step is 2^-12, so x +- h is exact in fp32 and the oracle's fp64 arithmetic
    sees exactly the perturbed input."""
    B, n, H, G, d = 1, 16, 4, 2, 8
    r = np.random.default_rng(7)
    q, k, v = (np.round(r.standard_normal(s) * 256) / 256 for s in [(B, n, H, d), (B, n, G, d), (B, n, G, d)])
    do = np.round(r.standard_normal((B, n, H, d)) * 256) / 256
    q, k, v, do = (x.astype(np.float32) for x in (q, k, v, do))
    cu = np.array([0, 6, n], np.int32) if mask == MASK_DOC_CAUSAL else None
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, mask=mask, cu_seqlens=cu)
    h = 2.0 ** -12
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        idx = [tuple(r.integers(0, s) for s in x.shape) for _ in range(12)]
        for ix in idx:
            xp, xm = x.copy(), x.copy()
            xp[ix] += h
            xm[ix] -= h
            args_p = {"q": q, "k": k, "v": v}; args_p[name] = xp
            args_m = {"q": q, "k": k, "v": v}; args_m[name] = xm
            fd = (_loss(args_p["q"], args_p["k"], args_p["v"], do, mask, cu)
                  - _loss(args_m["q"], args_m["k"], args_m["v"], do, mask, cu)) / (2 * h)
            assert abs(fd - g[ix]) <= 1e-6 * max(1.0, abs(g[ix])), (name, ix, fd, g[ix])


@pytest.mark.parametrize("mask", [MASK_NONE, MASK_CAUSAL, MASK_DOC_CAUSAL])
def test_backward_invariants(mask):
    """(1) Adding one vector to every key leaves each softmax row unchanged, so
    sum_j dK_j = 0 per KV head (equivalently sum_j dS_ij = 0 per row).
    (2) Rows of P sum to 1, so sum_j dV_j = sum over the group's query heads
    and all rows of dO_i."""
    B, n, H, G, d = 1, 40, 6, 2, 8
    q, k, v, do = _randn(B, n, H, d), _randn(B, n, G, d), _randn(B, n, G, d), _randn(B, n, H, d)
    cu = np.array([0, 9, 30, n], np.int32) if mask == MASK_DOC_CAUSAL else None
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, mask=mask, cu_seqlens=cu)
    assert np.abs(dk.sum(axis=1)).max() < 1e-11
    grp = H // G
    for g in range(G):
        lhs = dv[0, :, g].sum(0)
        rhs = do[0, :, g * grp:(g + 1) * grp].astype(np.float64).sum(axis=(0, 1))
        assert np.abs(lhs - rhs).max() < 1e-11


def test_backward_matches_torch_autograd():
    """Library cross-check: torch autograd through float64 SDPA."""
    B, n, H, G, d = 1, 24, 4, 2, 16
    q, k, v, do = _randn(B, n, H, d), _randn(B, n, G, d), _randn(B, n, G, d), _randn(B, n, H, d)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, mask=MASK_CAUSAL)
    qt = torch.tensor(q, dtype=torch.float64, requires_grad=True)
    kt = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    vt = torch.tensor(v, dtype=torch.float64, requires_grad=True)
    o = F.scaled_dot_product_attention(qt.permute(0, 2, 1, 3),
                                       kt.permute(0, 2, 1, 3).repeat_interleave(H // G, 1),
                                       vt.permute(0, 2, 1, 3).repeat_interleave(H // G, 1), is_causal=True)
    (o.permute(0, 2, 1, 3) * torch.tensor(do, dtype=torch.float64)).sum().backward()
    assert np.abs(qt.grad.numpy() - dq).max() < 1e-12
    assert np.abs(kt.grad.numpy() - dk).max() < 1e-12
    assert np.abs(vt.grad.numpy() - dv).max() < 1e-12


# ------------------------------------------------------------ sampled oracle

@pytest.mark.parametrize("mask", [MASK_CAUSAL, MASK_DOC_CAUSAL, MASK_NONE])
def test_sampled_rows_and_columns_match_full(mask):
    B, n, H, G, d = 1, 64, 4, 1, 8
    q, k, v, do = _randn(B, n, H, d), _randn(B, n, G, d), _randn(B, n, G, d), _randn(B, n, H, d)
    cu = np.array([0, 10, 40, n], np.int32) if mask == MASK_DOC_CAUSAL else None
    o, lse = oracle.attention_fwd(q, k, v, mask=mask, cu_seqlens=cu)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, mask=mask, cu_seqlens=cu)
    rows = np.array([0, 1, 9, 10, 39, 40, 63])
    ro, rl, rdq = oracle.head_rows(q[0, :, 2], k[0, :, 0], v[0, :, 0], rows, dout=do[0, :, 2],
                                   mask=mask, cu_seqlens=cu)
    assert np.abs(ro - o[0, rows, 2]).max() < 1e-13
    assert np.abs(rl - lse[0, 2, rows]).max() < 1e-13
    assert np.abs(rdq - dq[0, rows, 2]).max() < 1e-13
    cols = np.array([0, 9, 10, 33, 63])
    ck, cv = oracle.kv_cols([q[0, :, h] for h in range(H)], [do[0, :, h] for h in range(H)],
                            k[0, :, 0], v[0, :, 0], cols, mask=mask, cu_seqlens=cu)
    assert np.abs(ck - dk[0, cols, 0]).max() < 1e-12
    assert np.abs(cv - dv[0, cols, 0]).max() < 1e-12


@pytest.mark.parametrize("mask", [MASK_CAUSAL, MASK_DOC_CAUSAL, MASK_NONE])
def test_row_stats_match_full_forward(mask):
    """The per-row statistics from fp64 matrix products (used for key columns
    that every row sees at full size) equal the row-by-row oracle: LSE_i, and
    D_i = <dO_i, O_i> with O from the oracle's forward; rows outside the range
    get (-inf, 0).  Chunks of 7 rows make the row range cross chunk and
    document boundaries."""
    n, H, G, d = 70, 4, 2, 8
    q, k, v, do = _randn(1, n, H, d), _randn(1, n, G, d), _randn(1, n, G, d), _randn(1, n, H, d)
    cu = np.array([0, 9, 10, 41, n], np.int32) if mask == MASK_DOC_CAUSAL else None
    o, lse = oracle.attention_fwd(q, k, v, mask=mask, cu_seqlens=cu)
    for h in range(H):
        g = h // (H // G)
        lo, hi = 5, 66
        ls, D = oracle.row_stats(q[0, :, h], k[0, :, g], v[0, :, g], do[0, :, h], lo, hi, mask=mask,
                                 cu_seqlens=cu, chunk=7)
        D_ref = (do[0, :, h].astype(np.float64) * o[0, :, h]).sum(1)
        assert np.abs(ls[lo:hi] - lse[0, h, lo:hi]).max() < 1e-12
        assert np.abs(D[lo:hi] - D_ref[lo:hi]).max() < 1e-12
        assert np.all(ls[:lo] == -np.inf) and np.all(ls[hi:] == -np.inf)
        assert np.all(D[:lo] == 0) and np.all(D[hi:] == 0)


@pytest.mark.parametrize("mask", [MASK_CAUSAL, MASK_DOC_CAUSAL, MASK_NONE])
def test_kv_cols_from_row_stats_match_full_backward(mask):
    """dK, dV at key columns from supplied row statistics (row_stats over
    rows_seeing(cols)) equal the full backward; rows_seeing is the smallest
    range holding every row that sees a listed key (brute force)."""
    n, H, G, d = 64, 4, 1, 8
    q, k, v, do = _randn(1, n, H, d), _randn(1, n, G, d), _randn(1, n, G, d), _randn(1, n, H, d)
    cu = np.array([0, 10, 40, n], np.int32) if mask == MASK_DOC_CAUSAL else None
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, mask=mask, cu_seqlens=cu)
    for cols in (np.array([0, 1, 33]), np.array([12, 20]), np.array([45, 63])):
        lo, hi = oracle.rows_seeing(cols, n, mask=mask, cu_seqlens=cu)
        doc = None if cu is None else np.searchsorted(cu, np.arange(n), side="right") - 1
        sees = [i for i in range(n) for j in cols
                if mask == MASK_NONE or (j <= i and (doc is None or doc[i] == doc[j]))]
        assert lo == min(sees) and hi == max(sees) + 1
        stats = [oracle.row_stats(q[0, :, h], k[0, :, 0], v[0, :, 0], do[0, :, h], lo, hi, mask=mask,
                                  cu_seqlens=cu, chunk=16) for h in range(H)]
        ck, cv = oracle.kv_cols([q[0, :, h] for h in range(H)], [do[0, :, h] for h in range(H)],
                                k[0, :, 0], v[0, :, 0], cols, mask=mask, cu_seqlens=cu, stats=stats)
        assert np.abs(ck - dk[0, cols, 0]).max() < 1e-12
        assert np.abs(cv - dv[0, cols, 0]).max() < 1e-12


@pytest.mark.parametrize("mask", [MASK_CAUSAL, MASK_DOC_CAUSAL, MASK_NONE])
def test_row_step_sums_to_full_backward(mask):
    """The per-row step (used to time the oracle on a row sample) summed over
    every row gives exactly the full forward and backward of the head."""
    n, d = 48, 8
    q, k, v, do = _randn(1, n, 1, d), _randn(1, n, 1, d), _randn(1, n, 1, d), _randn(1, n, 1, d)
    cu = np.array([0, 11, 30, n], np.int32) if mask == MASK_DOC_CAUSAL else None
    o, lse = oracle.attention_fwd(q, k, v, mask=mask, cu_seqlens=cu)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, mask=mask, cu_seqlens=cu)
    rows = np.arange(n)
    so, sl, sdq, sdk, sdv = oracle.head_rows_step(q[0, :, 0], k[0, :, 0], v[0, :, 0], do[0, :, 0], rows,
                                                  mask=mask, cu_seqlens=cu)
    assert np.abs(so - o[0, :, 0]).max() < 1e-12 and np.abs(sl - lse[0, 0]).max() < 1e-12
    assert np.abs(sdq - dq[0, :, 0]).max() < 1e-12
    assert np.abs(sdk - dk[0, :, 0]).max() < 1e-12 and np.abs(sdv - dv[0, :, 0]).max() < 1e-12


# ----------------------------------------------------------------------- loss

def test_loss_uniform_logits_closed_form():
    """All logits equal: softmax is uniform, every token's CE is log V
    (= 9.0109131... for V = 8192), and so is the weighted mean."""
    T, V, P = 64, 8192, 4
    z = np.full((T, V), 0.375, np.float32)
    y = rng.integers(0, V, T).astype(np.int32)
    y[::5] = -100
    S, C, L, bad = oracle.loss_aggregate(z, y, P)
    assert bad == 0
    assert abs(L - math.log(8192)) < 1e-12 and abs(math.log(8192) - 9.010913347279288) < 1e-12
    per = T // P
    for r in range(P):
        c = int((y[r * per:(r + 1) * per] != -100).sum())
        assert C[r] == c and abs(S[r] - c * math.log(V)) < 1e-9


def _ce_ref(z, y):
    return F.cross_entropy(torch.tensor(z, dtype=torch.float64), torch.tensor(y, dtype=torch.int64),
                           ignore_index=-100, reduction="mean").item()


@pytest.mark.parametrize("P", [1, 2, 4, 8])
def test_loss_weighted_equals_unsharded_mean(P):
    """sum_r S_r / sum_r C_r equals the unsharded mean (torch cross_entropy,
    float64) for any shard split, including shards with no valid token."""
    T, V = 64, 300
    z = _randn(T, V, scale=3.0)
    y = rng.integers(0, V, T).astype(np.int32)
    y[rng.random(T) < 0.3] = -100
    if P > 1:
        y[: T // P] = -100   # shard 0 has no valid token
    S, C, L, bad = oracle.loss_aggregate(z, y, P)
    assert bad == 0
    assert abs(L - _ce_ref(z, y)) < 1e-12
    if P > 1:
        assert C[0] == 0 and S[0] == 0.0
    # per-shard sums against torch's per-token losses
    per_tok = F.cross_entropy(torch.tensor(z, dtype=torch.float64), torch.tensor(y, dtype=torch.int64),
                              ignore_index=-100, reduction="none").numpy()
    for r in range(P):
        sl = slice(r * T // P, (r + 1) * T // P)
        assert abs(S[r] - per_tok[sl].sum()) < 1e-10
        assert C[r] == int((y[sl] != -100).sum())
    # the mean of per-shard means is NOT the answer when counts differ
    if P == 4:
        means = [S[r] / C[r] for r in range(P) if C[r] > 0]
        assert abs(np.mean(means) - L) > 1e-6


def test_loss_edge_cases():
    T, V, P = 16, 50, 4
    z = _randn(T, V)
    y = np.full(T, -100, np.int32)
    S, C, L, bad = oracle.loss_aggregate(z, y, P)
    assert math.isnan(L) and C.sum() == 0 and bad == 0
    y = rng.integers(0, V, T).astype(np.int32)
    y[3], y[7] = V, -5           # out of range, not the ignore index
    S, C, L, bad = oracle.loss_aggregate(z, y, P)
    assert bad == 2 and C.sum() == T - 2
    ok = y.copy(); ok[3] = ok[7] = -100
    assert abs(L - _ce_ref(z, ok)) < 1e-12
    # large logits: the max shift keeps it finite
    z2 = _randn(T, V) * 1e4
    y2 = rng.integers(0, V, T).astype(np.int32)
    S, C, L, bad = oracle.loss_aggregate(z2, y2, P)
    assert math.isfinite(L) and abs(L - _ce_ref(z2, y2)) < 1e-9 * max(1, abs(L))


def test_loss_grad_equals_torch_autograd():
    """dL/dz of the aggregated loss equals torch's float64 autograd gradient of
    the unsharded mean cross-entropy (ignore_index -100): one global count."""
    T, V = 48, 77
    z = _randn(T, V, scale=2.0)
    y = rng.integers(0, V, T).astype(np.int32)
    y[rng.random(T) < 0.25] = -100
    g, C = oracle.loss_grad(z, y)
    zt = torch.tensor(z, dtype=torch.float64, requires_grad=True)
    F.cross_entropy(zt, torch.tensor(y, dtype=torch.int64), ignore_index=-100, reduction="mean").backward()
    assert C == int((y != -100).sum())
    assert np.abs(g - zt.grad.numpy()).max() < 1e-15


def test_loss_grad_finite_differences():
    """Central differences of the oracle's own aggregated loss (P shards, one
    shard without valid tokens) match dL/dz at label and non-label entries."""
    T, V, P = 24, 40, 4
    z = _randn(T, V)
    y = rng.integers(0, V, T).astype(np.int32)
    y[: T // P] = -100
    y[rng.random(T) < 0.2] = -100
    g, C = oracle.loss_grad(z, y)
    h = np.float32(1.0 / 256)   # a power of two: z +- h is exact in float32
    picks = [(t, int(y[t])) for t in range(T) if y[t] >= 0][:6]
    picks += [(int(rng.integers(0, T)), int(rng.integers(0, V))) for _ in range(20)]
    for t, v in picks:
        zp, zm = z.copy(), z.copy()
        zp[t, v] += h
        zm[t, v] -= h
        Lp = oracle.loss_aggregate(zp, y, P)[2]
        Lm = oracle.loss_aggregate(zm, y, P)[2]
        fd = (Lp - Lm) / (float(zp[t, v]) - float(zm[t, v]))
        assert abs(fd - g[t, v]) < 1e-6, (t, v, fd, g[t, v])


def test_loss_grad_closed_forms_and_invariants():
    T, V = 32, 64
    z = _randn(T, V, scale=3.0)
    y = rng.integers(0, V, T).astype(np.int32)
    y[::4] = -100
    y[5], y[6] = V, -7               # invalid labels: not counted, zero rows
    g, C = oracle.loss_grad(z, y)
    counted = (y >= 0) & (y < V)
    assert C == int(counted.sum())
    # softmax sums to one: every counted row of dL/dz sums to zero
    assert np.abs(g[counted].sum(axis=1)).max() < 1e-15
    assert not g[~counted].any()
    # the label entry is the only negative one: (p_y - 1) / C < 0 < p_v / C
    for t in np.flatnonzero(counted):
        assert g[t, y[t]] < 0 and (np.delete(g[t], y[t]) > 0).all()
    # uniform logits: (1/V - [v == y]) / C exactly
    zu = np.full((T, V), -1.25, np.float32)
    gu, Cu = oracle.loss_grad(zu, y)
    ref = np.zeros((T, V))
    for t in np.flatnonzero(counted):
        ref[t] = 1.0 / V / Cu
        ref[t, y[t]] -= 1.0 / Cu
    assert np.abs(gu - ref).max() < 1e-16
    # nothing counted: all zero (no NaN)
    g0, C0 = oracle.loss_grad(z, np.full(T, -100, np.int32))
    assert C0 == 0 and not g0.any()


def test_pages_loss_parity_bound_is_met_by_sharding():
    """The pages report SP and DP losses within 1e-5 of each other; with exact
    token weighting the oracle's sharded loss equals the unsharded mean to
    rounding, far inside that bound."""
    bound = json.load(open(os.path.join(GOLDEN, "sharding_examples.json")))["loss_parity"]["max_abs_diff"]
    T, V = 256, 1000
    z = _randn(T, V)
    y = rng.integers(0, V, T).astype(np.int32)
    y[rng.random(T) < 0.2] = -100
    ref = _ce_ref(z, y)
    for P in (1, 2, 4, 8, 16):
        assert abs(oracle.loss_aggregate(z, y, P)[2] - ref) < bound * 1e-6


# ------------------------------------------- projections and rotary positions

def test_rope_is_a_complex_rotation():
    """Pairing element e with e + d/2 as the complex number x_e + i x_{e+d/2},
    the encoding multiplies it by exp(i * pos * base^(-2e/d)) (numpy's complex
    exponential, an independent formulation); position 0 is the identity and
    the first pair turns by exactly pos radians."""
    d, base = 16, 1.0e6
    x = rng.standard_normal((5, d))
    pos = np.array([0, 1, 7, 4096, 262143], np.float64)
    z = (x[:, :d // 2] + 1j * x[:, d // 2:]) * np.exp(1j * pos[:, None] * base ** (-2.0 * np.arange(d // 2) / d))
    y = oracle.rope(x, pos, base)
    assert np.abs(y[:, :d // 2] - z.real).max() < 1e-12 and np.abs(y[:, d // 2:] - z.imag).max() < 1e-12
    assert np.array_equal(y[0], x[0])
    ang = np.arctan2(y[1, d // 2], y[1, 0]) - np.arctan2(x[1, d // 2], x[1, 0])
    assert abs((ang + np.pi) % (2 * np.pi) - np.pi - 1.0) < 1e-12
    # every pair keeps its length
    assert np.allclose(np.hypot(y[:, :d // 2], y[:, d // 2:]), np.hypot(x[:, :d // 2], x[:, d // 2:]), atol=1e-12)


def test_rope_scores_depend_only_on_relative_position():
    """<rope(q, i), rope(k, j)> is a function of i - j: shifting both positions
    by the same offset (a shard's offset, say) leaves every score unchanged."""
    d = 32
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    for i, j, c in [(5, 2, 1000), (300, 301, 65536), (0, 0, 131072)]:
        a = oracle.rope(q, i) @ oracle.rope(k, j)
        b = oracle.rope(q, i + c) @ oracle.rope(k, j + c)
        assert abs(a - b) < 1e-9 * max(1.0, abs(a))
    assert abs(oracle.rope(q, 9) @ oracle.rope(k, 9) - q @ k) < 1e-12


@pytest.mark.parametrize("P,B,H,G", [(4, 1, 8, 4), (2, 2, 4, 2), (4, 1, 8, 2)])
def test_qkv_projection_sharded_equals_unsharded(P, B, H, G):
    """Sharding must not change what attention sees: every rank rotates its
    tokens by their positions in the whole sequence, so the P-rank projection
    (in head layout) holds the single-rank result (to fp64 rounding: the
    library product may block rows differently).  A rank that used its local
    positions would fail this."""
    d, hidden, n = 8, 24, 32
    x_nat = rng.standard_normal((B, n, hidden))
    w = rng.standard_normal(((H + 2 * G) * d, hidden)) / np.sqrt(hidden)
    q1, k1, v1 = oracle.qkv_proj_rope(x_nat[None], w, 1, H, G, d)       # P = 1: [1][B][H][n][d]
    qP, kP, vP = oracle.qkv_proj_rope(x_nat.reshape(B, P, n // P, hidden).transpose(1, 0, 2, 3), w, P, H, G, d)
    nat = lambda z: z.transpose(1, 0, 2, 3, 4).reshape(B, -1, n, d)     # [B][heads][n][d]
    same = lambda a, b: np.abs(a - b).max() < 1e-12
    assert same(nat(qP), q1[0])
    if G % P == 0:
        assert same(nat(kP), k1[0]) and same(nat(vP), v1[0])
    else:   # one copied KV head per rank: rank r holds KV head r*G/P
        for r in range(P):
            assert same(kP[r, :, 0], k1[0][:, r * G // P]) and same(vP[r, :, 0], v1[0][:, r * G // P])
    # local positions (the failure the ms-swift page describes) would differ
    pos_local = np.tile(np.arange(n) % (n // P), (B, 1))
    qL, _, _ = oracle.qkv_proj_rope(x_nat.reshape(B, P, n // P, hidden).transpose(1, 0, 2, 3), w, P, H, G, d,
                                    positions=pos_local)
    assert not np.allclose(nat(qL)[:, :, n // P:], q1[0][:, :, n // P:])


def test_qkv_projection_one_hot_reads_weight_columns():
    """A token whose hidden state is the unit vector e_c projects to column c
    of the weight matrix, split into H query heads, then G key heads, then G
    value heads of d rows each (position 0: no rotation)."""
    P, H, G, d, hidden, n = 2, 4, 2, 8, 16, 4
    w = rng.standard_normal(((H + 2 * G) * d, hidden))
    x = np.zeros((P, 1, n // P, hidden))
    c = 5
    x[0, 0, 0, c] = 1.0                 # token 0 of rank 0 (global position 0)
    q, k, v = oracle.qkv_proj_rope(x, w, P, H, G, d)
    col = w[:, c].reshape(H + 2 * G, d)
    for h in range(H):
        assert np.array_equal(q[h // (H // P), 0, h % (H // P), 0], col[h])
    for g in range(G):
        assert np.array_equal(k[g // (G // P), 0, g % (G // P), 0], col[H + g])
        assert np.array_equal(v[g // (G // P), 0, g % (G // P), 0], col[H + G + g])
    assert not np.any(q[:, :, :, 1:]) and not np.any(v[:, :, :, 1:])


def test_output_projection_matches_torch_linear():
    """Step 6 against torch.nn.functional.linear on the natural layout (the
    head layout turned back by an independent numpy transpose)."""
    P, B, H, d, n, hidden = 4, 2, 8, 8, 16, 12
    o_head = rng.standard_normal((P, B, H // P, n, d))
    w = rng.standard_normal((hidden, H * d))
    y = oracle.o_proj(o_head, w, P)                                     # [P][B][s][hidden]
    o_nat = o_head.transpose(1, 3, 0, 2, 4).reshape(B, n, H * d)        # heads r*H/P + hh in order
    ref = F.linear(torch.from_numpy(o_nat), torch.from_numpy(w)).numpy()
    assert np.abs(y.transpose(1, 0, 2, 3).reshape(B, n, hidden) - ref).max() < 1e-12


@pytest.mark.parametrize("P,H,G", [(4, 8, 4), (4, 8, 2), (2, 4, 2)])
def test_whole_layer_sharded_equals_plain_layer(P, H, G):
    """Steps 1-6 composed (shard, project and rotate at global positions,
    first all-to-all -- copying KV heads when G < P --, per-rank attention,
    second all-to-all, output projection) equal the plain single-device layer
    written with torch float64 library calls: linear, the rotation as a complex
    multiplication, scaled_dot_product_attention with GQA, linear."""
    B, n, hidden, d = 1, 32, 24, 8
    x = rng.standard_normal((B, n, hidden))
    w = rng.standard_normal(((H + 2 * G) * d, hidden)) / np.sqrt(hidden)
    wo = rng.standard_normal((hidden, H * d)) / np.sqrt(H * d)
    x_seq = x.reshape(B, P, n // P, hidden).transpose(1, 0, 2, 3)
    qh, kh, vh = oracle.qkv_proj_rope(x_seq, w, P, H, G, d)
    if G % P == 0:
        k_seq, v_seq = oracle.head_to_seq(kh, B, n, P, G), oracle.head_to_seq(vh, B, n, P, G)
    else:   # recover the G heads from their copies (rank r holds head r*G/P)
        k_seq = np.stack([kh[g * (P // G), :, 0] for g in range(G)], 2)       # [B][n][G][d]
        v_seq = np.stack([vh[g * (P // G), :, 0] for g in range(G)], 2)
        k_seq, v_seq = (z.reshape(B, P, n // P, G, d).transpose(1, 0, 2, 3, 4) for z in (k_seq, v_seq))
    q_seq = oracle.head_to_seq(qh, B, n, P, H)
    o_seq, _ = oracle.ulysses_fwd(q_seq.astype(np.float32), k_seq.astype(np.float32),
                                  v_seq.astype(np.float32), P)
    y = oracle.o_proj(oracle.seq_to_head(o_seq, B, n, P, H), wo, P)          # [P][B][s][hidden]
    # plain layer in torch float64 (inputs rounded to fp32 where the oracle's attention reads fp32)
    xt, wt, wot = (torch.from_numpy(a) for a in (x, w, wo))
    proj = F.linear(xt, wt).reshape(B, n, H + 2 * G, d)
    half = d // 2
    ang = torch.arange(n, dtype=torch.float64)[:, None] * 1.0e6 ** (-2.0 * torch.arange(half, dtype=torch.float64) / d)
    rot = torch.polar(torch.ones_like(ang), ang)                                # e^{i angle}

    def rope_t(z):
        c = torch.complex(z[..., :half], z[..., half:]) * rot[None, :, None, :]
        return torch.cat([c.real, c.imag], -1)
    q, k, v = rope_t(proj[:, :, :H]), rope_t(proj[:, :, H:H + G]), proj[:, :, H + G:]
    f32 = lambda z: z.float().double()
    o = F.scaled_dot_product_attention(f32(q).transpose(1, 2), f32(k).transpose(1, 2), f32(v).transpose(1, 2),
                                       is_causal=True, enable_gqa=True).transpose(1, 2).reshape(B, n, H * d)
    ref = F.linear(o, wot).numpy()
    got = y.transpose(1, 0, 2, 3).reshape(B, n, hidden)
    assert np.abs(got - ref).max() < 1e-9


def _torch_layer_proj(x_nat, w, H, G, d, P, pos, base=1.0e6):
    """Forward of the QKV projection in torch float64, laid out in the head
    layout with torch reshapes (independent of the oracle's index loops)."""
    B, n, hidden = x_nat.shape
    y = F.linear(x_nat, w).reshape(B, n, H + 2 * G, d)
    half = d // 2
    ang = pos[..., None] * base ** (-2.0 * torch.arange(half, dtype=torch.float64) / d)   # [B][n][half]
    rot = torch.polar(torch.ones_like(ang), ang)[:, :, None, :]

    def rope_t(z):
        c = torch.complex(z[..., :half], z[..., half:]) * rot
        return torch.cat([c.real, c.imag], -1)
    q, k, v = rope_t(y[:, :, :H]), rope_t(y[:, :, H:H + G]), y[:, :, H + G:]
    head = lambda z, hx: z.reshape(B, n, P, hx // P, d).permute(2, 0, 3, 1, 4)   # [P][B][hx/P][n][d]
    return head(q, H), head(k, G), head(v, G)


def test_rotation_inverse_is_negative_angle():
    x = rng.standard_normal((6, 16))
    pos = np.array([0, 3, 100, 65535, 262143, 7])
    assert np.abs(oracle.rope(oracle.rope(x, pos), -pos) - x).max() < 1e-10


@pytest.mark.parametrize("P,B,H,G,docs", [(4, 1, 8, 4, False), (2, 2, 4, 2, True)])
def test_qkv_projection_backward_matches_torch_autograd(P, B, H, G, docs):
    d, hidden, n = 8, 20, 24
    x = rng.standard_normal((B, n, hidden))
    w = rng.standard_normal(((H + 2 * G) * d, hidden)) / np.sqrt(hidden)
    pos = np.tile(np.concatenate([np.arange(10), np.arange(n - 10)]) if docs else np.arange(n), (B, 1))
    xt = torch.tensor(x, requires_grad=True)
    wt = torch.tensor(w, requires_grad=True)
    q, k, v = _torch_layer_proj(xt, wt, H, G, d, P, torch.tensor(pos, dtype=torch.float64))
    gq, gk, gv = (rng.standard_normal(tuple(z.shape)) for z in (q, k, v))
    ((q * torch.tensor(gq)).sum() + (k * torch.tensor(gk)).sum() + (v * torch.tensor(gv)).sum()).backward()
    x_seq = x.reshape(B, P, n // P, hidden).transpose(1, 0, 2, 3)
    # the oracle's own forward agrees with the torch one (same layout)
    oq, ok_, ov = oracle.qkv_proj_rope(x_seq, w, P, H, G, d, positions=pos)
    assert np.abs(oq - q.detach().numpy()).max() < 1e-12 and np.abs(ov - v.detach().numpy()).max() < 1e-12
    dx, dw = oracle.qkv_proj_rope_bwd(x_seq, w, gq, gk, gv, P, H, G, d, positions=pos)
    assert np.abs(dx.transpose(1, 0, 2, 3).reshape(B, n, hidden) - xt.grad.numpy()).max() < 1e-11
    assert np.abs(dw - wt.grad.numpy()).max() < 1e-11


def test_qkv_projection_backward_with_kv_copies_finite_differences():
    """G < P: the copies' gradients are summed before the projection's
    backward; central differences of sum(Q*gq + K*gk + V*gv) in x and w."""
    P, B, H, G, d, hidden, n = 4, 1, 8, 2, 8, 12, 16
    x = np.round(rng.standard_normal((P, B, n // P, hidden)) * 64) / 64
    w = np.round(rng.standard_normal(((H + 2 * G) * d, hidden)) * 64) / 64
    q, k, v = oracle.qkv_proj_rope(x, w, P, H, G, d)
    gq, gk, gv = (rng.standard_normal(z.shape) for z in (q, k, v))
    dx, dw = oracle.qkv_proj_rope_bwd(x, w, gq, gk, gv, P, H, G, d)

    def f(xx, ww):
        a, b, c = oracle.qkv_proj_rope(xx, ww, P, H, G, d)
        return float((a * gq).sum() + (b * gk).sum() + (c * gv).sum())
    h = 2.0 ** -10
    for arr, grad, which in ((x, dx, 0), (w, dw, 1)):
        for _ in range(6):
            ix = tuple(rng.integers(0, m) for m in arr.shape)
            ap, am = arr.copy(), arr.copy()
            ap[ix] += h
            am[ix] -= h
            fp = f(ap, w) if which == 0 else f(x, ap)
            fm = f(am, w) if which == 0 else f(x, am)
            assert abs((fp - fm) / (2 * h) - grad[ix]) < 1e-8 * max(1.0, abs(grad[ix]))


def test_output_projection_backward_matches_torch_autograd():
    P, B, H, d, n, hidden = 4, 2, 8, 8, 16, 12
    o_head = rng.standard_normal((P, B, H // P, n, d))
    w = rng.standard_normal((hidden, H * d))
    gy = rng.standard_normal((P, B, n // P, hidden))
    ot = torch.tensor(o_head, requires_grad=True)
    wt = torch.tensor(w, requires_grad=True)
    o_nat = ot.permute(1, 3, 0, 2, 4).reshape(B, n, H * d)
    y = F.linear(o_nat, wt)                                               # [B][n][hidden]
    (y * torch.tensor(gy.transpose(1, 0, 2, 3).reshape(B, n, hidden))).sum().backward()
    do_head, dw = oracle.o_proj_bwd(o_head, w, gy, P)
    assert np.abs(do_head - ot.grad.numpy()).max() < 1e-12
    assert np.abs(dw - wt.grad.numpy()).max() < 1e-11
