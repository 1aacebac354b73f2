"""Plain CPU oracle for the Ulysses attention layer -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline / reference arm may import this package.  The product path (the CUDA
library and its binding) never imports, links or executes anything here.

The arithmetic lives in ``ulysses_oracle.c`` (plain loops, fp64, OpenMP over
independent rows); this module builds it with gcc and marshals numpy arrays.
The projections either side of the attention (a library fp64 matrix product
as their one step) and the rotary position encoding are written here in
numpy, fp64.  It shares no code with the CUDA path.  Every function is pinned by
tests under ``tests/`` against closed forms, brute force, invariants, library
routines and finite differences.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ulysses_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

MASK_NONE, MASK_CAUSAL, MASK_DOC_CAUSAL = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (gcc, OpenMP, -O3)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O3", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
               "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i, l, dbl = ctypes.c_int, ctypes.c_long, ctypes.c_double
            lib.oracle_seq_to_head.argtypes = [i, i, i, i, l, P, P]
            lib.oracle_head_to_seq.argtypes = [i, i, i, i, l, P, P]
            lib.oracle_kv_replicate_to_head.argtypes = [i, i, i, i, l, P, P]
            lib.oracle_kv_reduce_to_seq.argtypes = [i, i, i, i, i, P, P]
            lib.oracle_shift_labels.argtypes = [i, i, i, P, P, i, i, i, P]
            attn = [i, i, i, i, i, i, P, i, dbl]
            lib.oracle_attention_fwd.argtypes = attn + [P, P, P, P, P]
            lib.oracle_attention_bwd.argtypes = attn + [P, P, P, P, P, P, P]
            uly = [i, i, i, i, i, i, i, P, i, dbl]
            lib.oracle_ulysses_fwd.argtypes = uly + [P, P, P, P, P]
            lib.oracle_ulysses_bwd.argtypes = uly + [P, P, P, P, P, P, P]
            lib.oracle_head_rows.argtypes = [i, i, i, P, i, dbl, P, P, P, P, P, i, P, P, P]
            lib.oracle_kv_cols.argtypes = [i, i, i, P, i, dbl, i, P, P, P, P, P, i, P, P]
            lib.oracle_kv_cols_stats.argtypes = [i, i, i, P, i, dbl, i, P, P, P, P, P, P, P, i, P, P]
            lib.oracle_head_rows_step.argtypes = [i, i, i, P, i, dbl, P, P, P, P, P, i, P, P, P, P, P]
            lib.oracle_loss.argtypes = [i, l, i, P, P, i, P, P, P]
            lib.oracle_loss.restype = l
            lib.oracle_loss_grad.argtypes = [l, i, P, P, i, P]
            lib.oracle_loss_grad.restype = ctypes.c_longlong
            _lib = lib
    return _lib


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else ctypes.c_void_p(0)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _check_ulysses(n, P, H, G):
    """Divisibility the method needs: n % P (every rank holds n/P positions),
    H % P (every rank owns whole query heads), H % G (GQA groups), and either
    G % P (every rank owns whole KV heads) or P % G (fewer KV heads than
    ranks: every rank receives a copy of the one KV head it uses)."""
    if P <= 0 or n % P or H % P or H % G or (G % P and P % G):
        raise ValueError(f"need n%P == H%P == H%G == 0 and G%P == 0 or P%G == 0, "
                         f"got n={n} P={P} H={H} G={G}")


def _cu(cu_seqlens):
    if cu_seqlens is None:
        return None, 0
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    return cu, int(cu.size - 1)


# --------------------------------------------------------------------------
# Steps 1, 3, 5: sharding and the two all-to-alls (byte-exact, any dtype)
# --------------------------------------------------------------------------

def seq_to_head(x: np.ndarray, B: int, n: int, P: int, heads: int) -> np.ndarray:
    """[P][B][n/P][heads][d] -> [P][B][heads/P][n][d] (any dtype, byte copy)."""
    x = np.ascontiguousarray(x)
    d = x.size // (B * n * heads)
    out = np.empty(P * B * (heads // P) * n * d, dtype=x.dtype)
    _load().oracle_seq_to_head(B, n, P, heads, d * x.itemsize, _ptr(x), _ptr(out))
    return out.reshape(P, B, heads // P, n, d)


def head_to_seq(x: np.ndarray, B: int, n: int, P: int, heads: int) -> np.ndarray:
    """[P][B][heads/P][n][d] -> [P][B][n/P][heads][d] (any dtype, byte copy)."""
    x = np.ascontiguousarray(x)
    d = x.size // (B * n * heads)
    out = np.empty(P * B * (n // P) * heads * d, dtype=x.dtype)
    _load().oracle_head_to_seq(B, n, P, heads, d * x.itemsize, _ptr(x), _ptr(out))
    return out.reshape(P, B, n // P, heads, d)


def kv_replicate_to_head(x: np.ndarray, B: int, n: int, P: int, G: int) -> np.ndarray:
    """KV heads fewer than ranks (P % G == 0): seq layout [P][B][n/P][G][d] ->
    [P][B][1][n][d], rank r receiving KV head floor(r*G/P) (any dtype, byte copy)."""
    x = np.ascontiguousarray(x)
    d = x.size // (B * n * G)
    out = np.empty(P * B * n * d, dtype=x.dtype)
    _load().oracle_kv_replicate_to_head(B, n, P, G, d * x.itemsize, _ptr(x), _ptr(out))
    return out.reshape(P, B, 1, n, d)


def kv_reduce_to_seq(x: np.ndarray, B: int, n: int, P: int, G: int) -> np.ndarray:
    """Gradients of the replicated KV heads, [P][B][1][n][d] -> seq layout
    [P][B][n/P][G][d] (fp64): each KV head's gradient is the sum over its copies."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    d = x.size // (P * B * n)
    out = np.empty((P, B, n // P, G, d), np.float64)
    _load().oracle_kv_reduce_to_seq(B, n, P, G, d, _ptr(x), _ptr(out))
    return out


def shift_labels(ids: np.ndarray, P: int, cu_seqlens=None, valid_len=None, ignore_index=-100):
    """Next-token labels of ids [B][n], shifted before sharding: label(t) =
    ids[t+1] unless t+1 >= valid_len or t+1 starts a packed document, then
    ignore_index.  Returns the seq layout [P][B][n/P] (int32)."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    B, n = ids.shape
    cu, nd = _cu(cu_seqlens)
    vl = n if valid_len is None else int(valid_len)
    out = np.empty((P, B, n // P), np.int32)
    _load().oracle_shift_labels(B, n, P, _ptr(ids), _ptr(cu), nd, vl, ignore_index, _ptr(out))
    return out


# --------------------------------------------------------------------------
# Step 4: plain full-sequence GQA attention on the natural layout [B][n][H][d]
# --------------------------------------------------------------------------

def attention_fwd(q, k, v, mask=MASK_CAUSAL, cu_seqlens=None, scale=0.0):
    """O [B][n][H][d] (fp64) and LSE [B][H][n] of plain multi-head GQA attention."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, n, H, d = q.shape
    G = k.shape[2]
    cu, nd = _cu(cu_seqlens)
    o = np.empty((B, n, H, d), np.float64)
    lse = np.empty((B, H, n), np.float64)
    _load().oracle_attention_fwd(B, n, H, G, d, mask, _ptr(cu), nd, scale,
                                 _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse))
    return o, lse


def attention_bwd(q, k, v, dout, mask=MASK_CAUSAL, cu_seqlens=None, scale=0.0):
    """dQ, dK, dV (fp64, natural layout) of sum(O * dO)."""
    q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
    B, n, H, d = q.shape
    G = k.shape[2]
    cu, nd = _cu(cu_seqlens)
    dq = np.empty((B, n, H, d), np.float64)
    dk = np.empty((B, n, G, d), np.float64)
    dv = np.empty((B, n, G, d), np.float64)
    _load().oracle_attention_bwd(B, n, H, G, d, mask, _ptr(cu), nd, scale,
                                 _ptr(q), _ptr(k), _ptr(v), _ptr(dout),
                                 _ptr(dq), _ptr(dk), _ptr(dv))
    return dq, dk, dv


# --------------------------------------------------------------------------
# The explicit Ulysses procedure (seq layout in and out)
# --------------------------------------------------------------------------

def ulysses_fwd(q_seq, k_seq, v_seq, P, mask=MASK_CAUSAL, cu_seqlens=None, scale=0.0):
    """q_seq [P][B][s][H][d], k/v_seq [P][B][s][G][d] -> O_seq [P][B][s][H][d]
    (fp64) and LSE in head layout [P][B][H/P][n]."""
    q, k, v = _f32(q_seq), _f32(k_seq), _f32(v_seq)
    _, B, s, H, d = q.shape
    G = k.shape[3]
    n = P * s
    _check_ulysses(n, P, H, G)
    cu, nd = _cu(cu_seqlens)
    o = np.empty((P, B, s, H, d), np.float64)
    lse = np.empty((P, B, H // P, n), np.float64)
    _load().oracle_ulysses_fwd(B, n, P, H, G, d, mask, _ptr(cu), nd, scale,
                               _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse))
    return o, lse


def ulysses_bwd(q_seq, k_seq, v_seq, do_seq, P, mask=MASK_CAUSAL, cu_seqlens=None, scale=0.0):
    """dQ_seq, dK_seq, dV_seq (fp64, seq layout) of sum(O * dO)."""
    q, k, v, do = _f32(q_seq), _f32(k_seq), _f32(v_seq), _f32(do_seq)
    _, B, s, H, d = q.shape
    G = k.shape[3]
    n = P * s
    _check_ulysses(n, P, H, G)
    cu, nd = _cu(cu_seqlens)
    dq = np.empty((P, B, s, H, d), np.float64)
    dk = np.empty((P, B, s, G, d), np.float64)
    dv = np.empty((P, B, s, G, d), np.float64)
    _load().oracle_ulysses_bwd(B, n, P, H, G, d, mask, _ptr(cu), nd, scale,
                               _ptr(q), _ptr(k), _ptr(v), _ptr(do),
                               _ptr(dq), _ptr(dk), _ptr(dv))
    return dq, dk, dv


# --------------------------------------------------------------------------
# Exact values at sampled rows / key columns (large workloads)
# --------------------------------------------------------------------------

def head_rows(q, k, v, rows, dout=None, mask=MASK_CAUSAL, cu_seqlens=None, scale=0.0):
    """One query head q [n][d] with its KV head k, v [n][d]: exact O, LSE (and
    dQ if dout is given) at the listed query rows."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    n, d = q.shape
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    cu, nd = _cu(cu_seqlens)
    o = np.empty((rows.size, d), np.float64)
    lse = np.empty(rows.size, np.float64)
    dq = np.empty((rows.size, d), np.float64) if dout is not None else None
    dout = _f32(dout) if dout is not None else None
    _load().oracle_head_rows(n, d, mask, _ptr(cu), nd, scale, _ptr(q), _ptr(k), _ptr(v),
                             _ptr(dout), _ptr(rows), rows.size, _ptr(o), _ptr(lse), _ptr(dq))
    return (o, lse, dq) if dout is not None else (o, lse)


def kv_cols(qs, douts, k, v, cols, mask=MASK_CAUSAL, cu_seqlens=None, scale=0.0, stats=None):
    """One KV head k, v [n][d] and its query heads qs[e], douts[e] [n][d]:
    exact dK, dV at the listed key columns, summed over the query heads.

    stats: None (the C routine computes LSE_i and D_i of every row that sees a
    listed key, one row at a time), or a list of (lse [n], D [n]) per query
    head covering at least those rows (e.g. from row_stats)."""
    qs = [_f32(x) for x in qs]
    douts = [_f32(x) for x in douts]
    k, v = _f32(k), _f32(v)
    n, d = k.shape
    cols = np.ascontiguousarray(cols, dtype=np.int32)
    cu, nd = _cu(cu_seqlens)
    qp = (ctypes.c_void_p * len(qs))(*[x.ctypes.data for x in qs])
    dp = (ctypes.c_void_p * len(douts))(*[x.ctypes.data for x in douts])
    dk = np.empty((cols.size, d), np.float64)
    dv = np.empty((cols.size, d), np.float64)
    if stats is None:
        _load().oracle_kv_cols(n, d, mask, _ptr(cu), nd, scale, len(qs),
                               ctypes.cast(qp, ctypes.c_void_p), ctypes.cast(dp, ctypes.c_void_p),
                               _ptr(k), _ptr(v), _ptr(cols), cols.size, _ptr(dk), _ptr(dv))
        return dk, dv
    if len(stats) != len(qs):
        raise ValueError("one (lse, D) pair per query head")
    ls = [np.ascontiguousarray(a, dtype=np.float64) for a, _ in stats]
    Ds = [np.ascontiguousarray(b, dtype=np.float64) for _, b in stats]
    if any(a.shape != (n,) for a in ls + Ds):
        raise ValueError("lse and D must have n entries")
    lp = (ctypes.c_void_p * len(ls))(*[x.ctypes.data for x in ls])
    Dp = (ctypes.c_void_p * len(Ds))(*[x.ctypes.data for x in Ds])
    _load().oracle_kv_cols_stats(n, d, mask, _ptr(cu), nd, scale, len(qs),
                                 ctypes.cast(qp, ctypes.c_void_p), ctypes.cast(dp, ctypes.c_void_p),
                                 _ptr(k), _ptr(v), ctypes.cast(lp, ctypes.c_void_p),
                                 ctypes.cast(Dp, ctypes.c_void_p), _ptr(cols), cols.size, _ptr(dk), _ptr(dv))
    return dk, dv


def rows_seeing(cols, n, mask=MASK_CAUSAL, cu_seqlens=None):
    """[lo, hi): the smallest row range holding every query row that sees one
    of the listed key columns (causal: j <= i; doc-causal: also the same
    document; no mask: every row)."""
    cols = np.asarray(cols)
    if mask == MASK_NONE:
        return 0, n
    lo = int(cols.min())
    if mask == MASK_CAUSAL:
        return lo, n
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    last = int(cols.max())
    e = int(np.searchsorted(cu, last, side="right")) - 1
    return lo, int(min(n, cu[e + 1]))


def row_stats(q, k, v, dout, lo, hi, mask=MASK_CAUSAL, cu_seqlens=None, scale=0.0, chunk=512):
    """LSE_i and D_i = <dO_i, O_i> of the query rows [lo, hi) of one head
    (q, dout [n][d]) with its KV head (k, v [n][d]), straight from the
    definition in float64 with library matrix products (torch CPU), a chunk
    of rows at a time (rows are independent):
        s_ij = scale q_i.k_j over the visible keys j, m_i = max_j s_ij,
        LSE_i = m_i + log sum_j exp(s_ij - m_i),
        O_i = sum_j exp(s_ij - LSE_i) v_j,  D_i = <dO_i, O_i>.
    Rows outside [lo, hi) get LSE = -inf, D = 0; a row that sees no key too."""
    import torch
    q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
    n, d = q.shape
    sc = scale if scale > 0 else 1.0 / np.sqrt(d)
    Q, K, V, dO = (torch.from_numpy(x).double() for x in (q, k, v, dout))
    doc = None
    if mask == MASK_DOC_CAUSAL:
        cu = torch.from_numpy(np.asarray(cu_seqlens, dtype=np.int64))
        doc = torch.searchsorted(cu, torch.arange(n, dtype=torch.int64), right=True) - 1
    lse = np.full(n, -np.inf)
    D = np.zeros(n)
    for r0 in range(lo, hi, chunk):
        r1 = min(hi, r0 + chunk)
        k0, k1 = 0, n
        if mask != MASK_NONE:
            k1 = r1
            if mask == MASK_DOC_CAUSAL:
                k0 = int(cu[doc[r0]])
        S = Q[r0:r1] @ K[k0:k1].T
        S.mul_(sc)
        if mask != MASK_NONE:
            # keys before the chunk's first row are visible to all its rows
            # (causal); the mask is needed from there on, and for documents
            # from the chunk's first document start
            c0 = r0 if mask == MASK_CAUSAL else k0
            i = torch.arange(r0, r1).unsqueeze(1)
            j = torch.arange(c0, k1).unsqueeze(0)
            allowed = j <= i
            if mask == MASK_DOC_CAUSAL:
                allowed &= doc[c0:k1].unsqueeze(0) == doc[r0:r1].unsqueeze(1)
            S[:, c0 - k0:].masked_fill_(~allowed, float("-inf"))
        m = S.max(dim=1).values
        seen = torch.isfinite(m)
        ms = torch.where(seen, m, torch.zeros_like(m))
        S.sub_(ms.unsqueeze(1)).exp_()          # S now holds exp(s_ij - m_i)
        ls = S.sum(dim=1)
        O = (S @ V[k0:k1]) / torch.where(seen, ls, torch.ones_like(ls)).unsqueeze(1)
        lse[r0:r1] = torch.where(seen, ms + torch.log(ls), torch.full_like(m, float("-inf"))).numpy()
        D[r0:r1] = torch.where(seen, (dO[r0:r1] * O).sum(dim=1), torch.zeros_like(m)).numpy()
    return lse, D


def head_rows_step(q, k, v, dout, rows, mask=MASK_CAUSAL, cu_seqlens=None, scale=0.0, dk=None, dv=None):
    """All the work of the listed query rows of one head (q, k, v, dout [n][d]):
    returns O, LSE, dQ at those rows and adds their dK, dV terms into dk, dv
    ([n][d] fp64, zero-initialised if not given)."""
    q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
    n, d = q.shape
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    cu, nd = _cu(cu_seqlens)
    o = np.empty((rows.size, d), np.float64)
    lse = np.empty(rows.size, np.float64)
    dq = np.empty((rows.size, d), np.float64)
    dk = np.zeros((n, d), np.float64) if dk is None else dk
    dv = np.zeros((n, d), np.float64) if dv is None else dv
    _load().oracle_head_rows_step(n, d, mask, _ptr(cu), nd, scale, _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(dout), _ptr(rows), rows.size, _ptr(o), _ptr(lse), _ptr(dq),
                                  _ptr(dk), _ptr(dv))
    return o, lse, dq, dk, dv


# --------------------------------------------------------------------------
# Token-weighted loss aggregation
# --------------------------------------------------------------------------

def loss_aggregate(logits, labels, P, ignore_index=-100):
    """logits [T][V] (shard r = rows [r*T/P, (r+1)*T/P)), labels [T] ->
    (S [P] fp64, C [P] int64, L fp64, number of bad labels)."""
    z = _f32(logits)
    T, V = z.shape
    y = np.ascontiguousarray(labels, dtype=np.int32)
    S = np.empty(P, np.float64)
    C = np.empty(P, np.int64)
    L = np.empty(1, np.float64)
    bad = _load().oracle_loss(P, T, V, _ptr(z), _ptr(y), ignore_index, _ptr(S), _ptr(C), _ptr(L))
    return S, C, float(L[0]), int(bad)


def loss_grad(logits, labels, ignore_index=-100):
    """dL/dlogits of the aggregated loss L = sum S_r / sum C_r: logits [T][V],
    labels [T] -> (dlogits [T][V] fp64, global count C)."""
    z = _f32(logits)
    T, V = z.shape
    y = np.ascontiguousarray(labels, dtype=np.int32)
    g = np.empty((T, V), np.float64)
    C = _load().oracle_loss_grad(T, V, _ptr(z), _ptr(y), ignore_index, _ptr(g))
    return g, int(C)


# --------------------------------------------------------------------------
# Steps 2 and 6: QKV projection with rotary positions, output projection
# --------------------------------------------------------------------------

def rope(x, pos, base=1.0e6):
    """Rotary position encoding of the last axis (d even), fp64, in the
    rotate-half pairing: element e and e + d/2 form a pair rotated by the angle
    pos * base^(-2e/d):
        y[e]       = x[e] cos - x[e + d/2] sin
        y[e + d/2] = x[e + d/2] cos + x[e] sin
    x [..., d], pos broadcastable to x[..., 0]."""
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    half = d // 2
    theta = base ** (-2.0 * np.arange(half, dtype=np.float64) / d)
    ang = np.asarray(pos, np.float64)[..., None] * theta
    c, sn = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * sn, x2 * c + x1 * sn], axis=-1)


def qkv_proj_rope(x_seq, w_qkv, P, H, G, d, base=1.0e6, positions=None):
    """Ulysses steps 2-3 ("Paralelismul de Secvență Ulysses", section
    "Mecanismul de funcționare Ulysses"): every rank projects its own tokens,
    rotates Q and K by each token's position in the WHOLE sequence (rank r's
    local token tt sits at t = r*n/P + tt: the shard's offset; ms-swift page,
    section 6.2, names a RoPE that ignores this offset as a failure), and the
    first all-to-all gives every rank all positions of its heads.
      x_seq [P][B][s][hidden], w_qkv [(H+2G)*d][hidden] (rows: H query heads,
      then G key heads, then G value heads, d rows each),
      positions: None (t itself) or [B][n] (e.g. restarting per document).
    Returns q [P][B][H/P][n][d], k and v [P][B][G/P][n][d] (fp64); with fewer
    KV heads than ranks (P % G == 0) k and v are [P][B][1][n][d], every rank
    holding a copy of the KV head its query heads use."""
    x = np.asarray(x_seq, np.float64)
    w = np.asarray(w_qkv, np.float64)
    P_, B, s, hidden = x.shape
    n = P * s
    _check_ulysses(n, P, H, G)
    if w.shape != ((H + 2 * G) * d, hidden):
        raise ValueError(f"w_qkv shape {w.shape}, expected {((H + 2 * G) * d, hidden)}")
    q_seq = np.empty((P, B, s, H, d))
    k_seq = np.empty((P, B, s, G, d))
    v_seq = np.empty((P, B, s, G, d))
    for r in range(P):
        y = (x[r].reshape(B * s, hidden) @ w.T).reshape(B, s, H + 2 * G, d)
        t = r * s + np.arange(s)
        pos = np.broadcast_to(t, (B, s)) if positions is None else np.asarray(positions)[:, t]
        q_seq[r] = rope(y[:, :, :H], pos[:, :, None], base)
        k_seq[r] = rope(y[:, :, H:H + G], pos[:, :, None], base)
        v_seq[r] = y[:, :, H + G:]
    kv = (lambda z: seq_to_head(z, B, n, P, G)) if G % P == 0 else \
        (lambda z: kv_replicate_to_head(z, B, n, P, G))
    return seq_to_head(q_seq, B, n, P, H), kv(k_seq), kv(v_seq)


def o_proj(o_head, w_o, P):
    """Ulysses steps 5-6: the second all-to-all returns every rank its own
    positions for all heads, then each rank applies the output projection to
    its tokens.  o_head [P][B][H/P][n][d], w_o [hidden][H*d] -> y seq layout
    [P][B][n/P][hidden] (fp64)."""
    o = np.asarray(o_head, np.float64)
    P_, B, hl, n, d = o.shape
    H = hl * P
    o_seq = head_to_seq(o, B, n, P, H)                 # [P][B][s][H][d]
    w = np.asarray(w_o, np.float64)
    y = o_seq.reshape(P * B * (n // P), H * d) @ w.T
    return y.reshape(P, B, n // P, w.shape[0])


def qkv_proj_rope_bwd(x_seq, w_qkv, dq_head, dk_head, dv_head, P, H, G, d, base=1.0e6, positions=None):
    """Backward of qkv_proj_rope (the adjoint of steps 2-3): the gradients of
    the rotated Q, K and of V go back through the all-to-all (head -> seq; the
    copies of a KV head are summed when G < P), through the rotation (its
    transpose: the same rotation by -pos), and through the projection:
        dY(t) = [R(-pos) dQ(t) | R(-pos) dK(t) | dV(t)],
        dX_r = dY_r W,   dW = sum over ranks of dY_r^T X_r.
    Returns dx_seq [P][B][s][hidden] and dw [(H+2G)*d][hidden] (fp64)."""
    x = np.asarray(x_seq, np.float64)
    w = np.asarray(w_qkv, np.float64)
    P_, B, s, hidden = x.shape
    n = P * s
    _check_ulysses(n, P, H, G)
    dq = head_to_seq(np.asarray(dq_head, np.float64), B, n, P, H)              # [P][B][s][H][d]
    if G % P == 0:
        dk = head_to_seq(np.asarray(dk_head, np.float64), B, n, P, G)
        dv = head_to_seq(np.asarray(dv_head, np.float64), B, n, P, G)
    else:
        dk = kv_reduce_to_seq(dk_head, B, n, P, G)
        dv = kv_reduce_to_seq(dv_head, B, n, P, G)
    dx = np.empty_like(x)
    dw = np.zeros_like(w)
    for r in range(P):
        t = r * s + np.arange(s)
        pos = np.broadcast_to(t, (B, s)) if positions is None else np.asarray(positions)[:, t]
        dy = np.concatenate([rope(dq[r], -pos[:, :, None], base), rope(dk[r], -pos[:, :, None], base), dv[r]],
                            axis=2).reshape(B * s, (H + 2 * G) * d)
        dx[r] = (dy @ w).reshape(B, s, hidden)
        dw += dy.T @ x[r].reshape(B * s, hidden)
    return dx, dw


def o_proj_bwd(o_head, w_o, dy_seq, P):
    """Backward of o_proj (the adjoint of steps 5-6): dO_seq = dY W_o, back to
    the head layout by the first all-to-all; dW_o = sum over ranks of
    dY_r^T O_r.  Returns do_head [P][B][H/P][n][d] and dw_o [hidden][H*d] (fp64)."""
    o = np.asarray(o_head, np.float64)
    P_, B, hl, n, d = o.shape
    H = hl * P
    w = np.asarray(w_o, np.float64)
    dy = np.asarray(dy_seq, np.float64).reshape(P * B * (n // P), w.shape[0])
    o_seq = head_to_seq(o, B, n, P, H).reshape(P * B * (n // P), H * d)
    do_seq = (dy @ w).reshape(P, B, n // P, H, d)
    return seq_to_head(do_seq, B, n, P, H), dy.T @ o_seq
