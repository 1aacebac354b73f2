"""ctypes binding of ``libulysses.so`` -- argument marshalling only.

Every entry point of the C ABI (``include/ulysses.h``) is exposed under the
same name.  The functions take CUDA torch tensors (torch is used for device
memory and streams only), pass raw device pointers and the current CUDA
stream to the library, and raise :class:`UlyssesError` on a non-OK status.
All arithmetic happens in the library's kernels; there is no fallback: if the
library is missing or cannot be loaded, every call fails loudly.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libulysses.so")

ULY_F32, ULY_BF16 = 0, 1
MASK_NONE, MASK_CAUSAL, MASK_DOC_CAUSAL = 0, 1, 2
STATUS = {0: "ULY_OK", 1: "ULY_ERR_NULL", 2: "ULY_ERR_SHAPE", 3: "ULY_ERR_DTYPE",
          4: "ULY_ERR_ALIGN", 5: "ULY_ERR_ALIAS", 6: "ULY_ERR_UNSUPPORTED", 7: "ULY_ERR_CUDA",
          8: "ULY_ERR_LABEL", 9: "ULY_ERR_TIMEOUT", 10: "ULY_ERR_WORKSPACE"}
EXPORTS = ["ulysses_seq_to_head", "ulysses_head_to_seq", "ulysses_seq_to_head_batch", "ulysses_head_to_seq_batch",
           "ulysses_kv_seq_to_head_replicated",
           "ulysses_kv_head_to_seq_reduce", "ulysses_shift_labels", "ulysses_rope_table",
           "ulysses_qkv_proj_rope", "ulysses_o_proj", "ulysses_qkv_proj_rope_bwd_workspace_size",
           "ulysses_qkv_proj_rope_bwd", "ulysses_o_proj_bwd", "ulysses_attn_fwd",
           "ulysses_attn_bwd_workspace_size", "ulysses_attn_bwd", "ulysses_loss_workspace_size",
           "ulysses_loss_aggregate", "ulysses_loss_aggregate_noalloc", "ulysses_loss_bwd_workspace_size",
           "ulysses_loss_aggregate_bwd", "ulysses_read_error", "ulysses_read_error_info", "ulysses_error_word",
           "ulysses_set_wait_limit", "ulysses_set_attn_block_order",
           "ulysses_status_string", "ulysses_profile_enable", "ulysses_profile_read",
           "ulysses_kernel_count", "ulysses_kernel_name",
           "ulysses_launch_count"]


class UlyssesError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class AttnDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("seq_len", ctypes.c_int32), ("world", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("dtype", ctypes.c_int32), ("mask", ctypes.c_int32),
                ("cu_seqlens", ctypes.c_void_p), ("num_docs", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("out_seq_layout", ctypes.c_int32),
                ("deterministic", ctypes.c_int32)]


class PermuteItem(ctypes.Structure):
    _fields_ = [("src", ctypes.c_void_p), ("dst", ctypes.c_void_p), ("heads", ctypes.c_int32)]


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """Load the library (once).  Raises if it is missing: there is no fallback."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                                   "`python -m long_context_sequence_all_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
            for name in ("ulysses_seq_to_head", "ulysses_head_to_seq"):
                getattr(L, name).argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp]
                getattr(L, name).restype = ctypes.c_int
            for name in ("ulysses_seq_to_head_batch", "ulysses_head_to_seq_batch"):
                getattr(L, name).argtypes = [i32, i32, i32, i32, i32, i32, ctypes.POINTER(PermuteItem), vp]
                getattr(L, name).restype = ctypes.c_int
            L.ulysses_kv_seq_to_head_replicated.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp]
            L.ulysses_kv_head_to_seq_reduce.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp]
            L.ulysses_shift_labels.argtypes = [i32, i32, i32, vp, vp, i32, i32, i32, vp, vp]
            L.ulysses_rope_table.argtypes = [i32, i32, ctypes.c_double, vp, vp]
            L.ulysses_qkv_proj_rope.argtypes = [i32, i32, i32, i32, i32, i32, i32, vp, vp, vp, i32, vp,
                                                vp, vp, vp, vp]
            L.ulysses_o_proj.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp, vp]
            L.ulysses_qkv_proj_rope_bwd_workspace_size.argtypes = [i32, i32, i32, i32, i32, ctypes.POINTER(sz)]
            L.ulysses_qkv_proj_rope_bwd.argtypes = [i32, i32, i32, i32, i32, i32, i32, vp, vp, vp, i32, vp, vp, vp,
                                                    vp, vp, vp, vp, sz, vp]
            L.ulysses_o_proj_bwd.argtypes = [i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]
            for name in ("ulysses_qkv_proj_rope_bwd_workspace_size", "ulysses_qkv_proj_rope_bwd",
                         "ulysses_o_proj_bwd"):
                getattr(L, name).restype = ctypes.c_int
            for name in ("ulysses_kv_seq_to_head_replicated", "ulysses_kv_head_to_seq_reduce",
                         "ulysses_shift_labels", "ulysses_rope_table", "ulysses_qkv_proj_rope",
                         "ulysses_o_proj"):
                getattr(L, name).restype = ctypes.c_int
            D = ctypes.POINTER(AttnDesc)
            L.ulysses_attn_fwd.argtypes = [D, vp, vp, vp, vp, vp, vp]
            L.ulysses_attn_bwd_workspace_size.argtypes = [D, ctypes.POINTER(sz)]
            L.ulysses_attn_bwd.argtypes = [D, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            L.ulysses_loss_workspace_size.argtypes = [i32, i64, i32, ctypes.POINTER(sz)]
            L.ulysses_loss_aggregate.argtypes = [i32, i64, i32, i32, vp, vp, i32, vp, vp, vp, vp, sz, vp]
            L.ulysses_loss_aggregate_noalloc.argtypes = [i32, i64, i32, i32, vp, vp, i32, vp, vp, vp, vp]
            L.ulysses_loss_aggregate_noalloc.restype = ctypes.c_int
            L.ulysses_loss_bwd_workspace_size.argtypes = [i32, i64, i32, ctypes.POINTER(sz)]
            L.ulysses_loss_aggregate_bwd.argtypes = [i32, i64, i32, i32, vp, vp, i32, vp, vp, vp, vp, vp, sz, vp]
            L.ulysses_read_error.argtypes = [ctypes.POINTER(i32)]
            L.ulysses_error_word.argtypes = [ctypes.POINTER(vp)]
            L.ulysses_error_word.restype = ctypes.c_int
            L.ulysses_read_error_info.argtypes = [ctypes.POINTER(i32), i32]
            L.ulysses_set_wait_limit.argtypes = [i64]
            L.ulysses_set_wait_limit.restype = ctypes.c_int
            L.ulysses_set_attn_block_order.argtypes = [ctypes.c_int32]
            L.ulysses_set_attn_block_order.restype = ctypes.c_int
            L.ulysses_status_string.argtypes = [ctypes.c_int]
            L.ulysses_status_string.restype = ctypes.c_char_p
            L.ulysses_launch_count.restype = ctypes.c_uint64
            L.ulysses_profile_enable.argtypes = [i32]
            L.ulysses_profile_enable.restype = ctypes.c_int
            L.ulysses_profile_read.argtypes = [i32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i64)]
            L.ulysses_profile_read.restype = ctypes.c_int
            L.ulysses_kernel_count.restype = i32
            L.ulysses_kernel_name.argtypes = [i32]
            L.ulysses_kernel_name.restype = ctypes.c_char_p
            for name in ("ulysses_attn_fwd", "ulysses_attn_bwd_workspace_size", "ulysses_attn_bwd",
                         "ulysses_loss_workspace_size", "ulysses_loss_aggregate", "ulysses_read_error",
                         "ulysses_read_error_info", "ulysses_loss_bwd_workspace_size",
                         "ulysses_loss_aggregate_bwd"):
                getattr(L, name).restype = ctypes.c_int
            _lib = L
    return _lib


def _check(st: int, where: str):
    if st != 0:
        raise UlyssesError(st, where)


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return ULY_BF16
    if t.dtype == torch.float32:
        return ULY_F32
    raise UlyssesError(3, f"dtype {t.dtype}")


def make_desc(B, n, P, H, G, d, dtype_code, mask, cu_seqlens=None, scale=0.0, out_seq_layout=False,
              deterministic=False) -> AttnDesc:
    nd = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    return AttnDesc(B, n, P, H, G, d, dtype_code, mask,
                    ctypes.c_void_p(cu_seqlens.data_ptr()) if cu_seqlens is not None else None,
                    nd, float(scale), int(bool(out_seq_layout)), int(bool(deterministic)))


# --------------------------------------------------------------- all-to-alls

def ulysses_seq_to_head(x: torch.Tensor, P: int, out: torch.Tensor | None = None, stream=None):
    """[P][B][n/P][heads][d] -> [P][B][heads/P][n][d] (bit-exact copy)."""
    P_, B, s, heads, d = x.shape
    if P_ != P or heads % P:
        raise UlyssesError(2, f"ulysses_seq_to_head: shape {tuple(x.shape)} with P={P}")
    n = P * s
    if out is None:
        out = torch.empty((P, B, heads // P, n, d), dtype=x.dtype, device=x.device)
    _check(lib().ulysses_seq_to_head(B, n, P, heads, d, x.element_size(), _p(x), _p(out),
                                     _stream(stream)), "ulysses_seq_to_head")
    return out


def ulysses_head_to_seq(x: torch.Tensor, P: int, out: torch.Tensor | None = None, stream=None):
    """[P][B][heads/P][n][d] -> [P][B][n/P][heads][d] (bit-exact copy)."""
    P_, B, hl, n, d = x.shape
    if P_ != P or hl == 0 or n % P:
        raise UlyssesError(2, f"ulysses_head_to_seq: shape {tuple(x.shape)} with P={P}")
    heads = hl * P
    if out is None:
        out = torch.empty((P, B, n // P, heads, d), dtype=x.dtype, device=x.device)
    _check(lib().ulysses_head_to_seq(B, n, P, heads, d, x.element_size(), _p(x), _p(out),
                                     _stream(stream)), "ulysses_head_to_seq")
    return out


def _batch(to_head: bool, xs, P: int, outs=None, stream=None):
    if not 1 <= len(xs) <= 4:
        raise UlyssesError(2, "batched all-to-all: 1 to 4 tensors")
    x0 = xs[0]
    if to_head:
        _, B, s, _, d = x0.shape
        n = P * s
        heads = [x.shape[3] for x in xs]
        shape = lambda x: (P, B, x.shape[3] // P, n, d)
    else:
        _, B, _, n, d = x0.shape
        heads = [x.shape[2] * P for x in xs]
        shape = lambda x: (P, B, n // P, x.shape[2] * P, d)
    for x in xs:
        if x.dtype != x0.dtype or x.shape[0] != P or x.shape[1] != B or x.shape[-1] != d:
            raise UlyssesError(2, f"batched all-to-all: shapes {[tuple(y.shape) for y in xs]} with P={P}")
    if outs is None:
        outs = [torch.empty(shape(x), dtype=x.dtype, device=x.device) for x in xs]
    arr = (PermuteItem * len(xs))(*[PermuteItem(x.data_ptr(), o.data_ptr(), h) for x, o, h in zip(xs, outs, heads)])
    fn = lib().ulysses_seq_to_head_batch if to_head else lib().ulysses_head_to_seq_batch
    _check(fn(B, n, P, d, x0.element_size(), len(xs), arr, _stream(stream)),
           "ulysses_seq_to_head_batch" if to_head else "ulysses_head_to_seq_batch")
    return outs


def ulysses_seq_to_head_batch(xs, P: int, outs=None, stream=None):
    """The first all-to-all of up to four tensors in one call (e.g. Q, K, V):
    each [P][B][n/P][heads_i][d] -> [P][B][heads_i/P][n][d]."""
    return _batch(True, xs, P, outs, stream)


def ulysses_head_to_seq_batch(xs, P: int, outs=None, stream=None):
    """The second all-to-all of up to four tensors in one call:
    each [P][B][heads_i/P][n][d] -> [P][B][n/P][heads_i][d]."""
    return _batch(False, xs, P, outs, stream)


def ulysses_kv_seq_to_head_replicated(x: torch.Tensor, P: int, out: torch.Tensor | None = None,
                                      stream=None):
    """G < P KV heads: [P][B][n/P][G][d] -> [P][B][1][n][d], rank r receiving
    KV head floor(r*G/P) (bit-exact copy)."""
    P_, B, s, G, d = x.shape
    if P_ != P or G <= 0 or P % G:
        raise UlyssesError(2, f"ulysses_kv_seq_to_head_replicated: shape {tuple(x.shape)} with P={P}")
    n = P * s
    if out is None:
        out = torch.empty((P, B, 1, n, d), dtype=x.dtype, device=x.device)
    _check(lib().ulysses_kv_seq_to_head_replicated(B, n, P, G, d, x.element_size(), _p(x), _p(out),
                                                   _stream(stream)),
           "ulysses_kv_seq_to_head_replicated")
    return out


def ulysses_kv_head_to_seq_reduce(x: torch.Tensor, P: int, G: int, out: torch.Tensor | None = None,
                                  stream=None):
    """Gradients of the KV copies, [P][B][1][n][d] -> seq layout [P][B][n/P][G][d],
    each KV head's gradient summed over its P/G copies (fp32 sum, one rounding)."""
    P_, B, one, n, d = x.shape
    if P_ != P or one != 1 or G <= 0 or P % G or n % P:
        raise UlyssesError(2, f"ulysses_kv_head_to_seq_reduce: shape {tuple(x.shape)} with P={P}, G={G}")
    if out is None:
        out = torch.empty((P, B, n // P, G, d), dtype=x.dtype, device=x.device)
    _check(lib().ulysses_kv_head_to_seq_reduce(B, n, P, G, d, _dtype_code(x), _p(x), _p(out),
                                               _stream(stream)),
           "ulysses_kv_head_to_seq_reduce")
    return out


def ulysses_shift_labels(input_ids: torch.Tensor, P: int, cu_seqlens: torch.Tensor | None = None,
                         valid_len: int | None = None, ignore_index: int = -100,
                         out: torch.Tensor | None = None, stream=None):
    """Next-token labels of input_ids [B][n] (int32), shifted before sharding:
    returns the seq layout [P][B][n/P] (int32)."""
    B, n = input_ids.shape
    if input_ids.dtype != torch.int32 or n % P or (cu_seqlens is not None and cu_seqlens.dtype != torch.int32):
        raise UlyssesError(2, f"ulysses_shift_labels: ids {tuple(input_ids.shape)} {input_ids.dtype} with P={P}")
    nd = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty((P, B, n // P), dtype=torch.int32, device=input_ids.device)
    vl = n if valid_len is None else int(valid_len)
    _check(lib().ulysses_shift_labels(B, n, P, _p(input_ids), _p(cu_seqlens), nd, vl, ignore_index,
                                      _p(out), _stream(stream)), "ulysses_shift_labels")
    return out


# --------------------------------------------------------------- projections

def ulysses_rope_table(max_pos: int, head_dim: int = 128, base: float = 1.0e6, out=None, device=None,
                       stream=None):
    """(cos, sin) of p * base^(-2e/d) for p < max_pos, e < d/2: float32 [max_pos][d/2][2]."""
    if out is None:
        out = torch.empty((max_pos, head_dim // 2, 2), dtype=torch.float32, device=device or "cuda")
    _check(lib().ulysses_rope_table(max_pos, head_dim, float(base), _p(out), _stream(stream)),
           "ulysses_rope_table")
    return out


def ulysses_qkv_proj_rope(x: torch.Tensor, w_qkv: torch.Tensor, P: int, H: int, G: int,
                          rope_table: torch.Tensor, positions: torch.Tensor | None = None,
                          q=None, k=None, v=None, stream=None):
    """x seq layout [P][B][n/P][hidden] (bf16), w_qkv [(H+2G)*128][hidden] ->
    q [P][B][H/P][n][128], k, v [P][B][G/P][n][128] (rotated Q, K; head layout)."""
    P_, B, s, hidden = x.shape
    n, d = P * s, 128
    if P_ != P or tuple(w_qkv.shape) != ((H + 2 * G) * d, hidden):
        raise UlyssesError(2, f"ulysses_qkv_proj_rope: x {tuple(x.shape)}, w {tuple(w_qkv.shape)} with P={P}")
    if rope_table.dtype != torch.float32 or rope_table.dim() != 3 or tuple(rope_table.shape[1:]) != (d // 2, 2):
        raise UlyssesError(2, f"ulysses_qkv_proj_rope: rope table {tuple(rope_table.shape)} {rope_table.dtype}")
    if positions is not None and (positions.dtype != torch.int32 or tuple(positions.shape) != (B, n)):
        raise UlyssesError(2, f"ulysses_qkv_proj_rope: positions {tuple(positions.shape)} {positions.dtype}")
    dev = x.device
    q = torch.empty((P, B, H // P, n, d), dtype=x.dtype, device=dev) if q is None else q
    k = torch.empty((P, B, max(G // P, 1), n, d), dtype=x.dtype, device=dev) if k is None else k
    v = torch.empty_like(k) if v is None else v
    _check(lib().ulysses_qkv_proj_rope(B, n, P, hidden, H, G, d, _p(x), _p(w_qkv), _p(rope_table),
                                       rope_table.shape[0], _p(positions), _p(q), _p(k), _p(v),
                                       _stream(stream)), "ulysses_qkv_proj_rope")
    return q, k, v


def ulysses_o_proj(o: torch.Tensor, w_o: torch.Tensor, P: int, y=None, stream=None):
    """o head layout [P][B][H/P][n][128] (bf16), w_o [hidden][H*128] -> y seq
    layout [P][B][n/P][hidden]."""
    P_, B, hl, n, d = o.shape
    hidden = w_o.shape[0]
    if P_ != P or tuple(w_o.shape) != (hidden, hl * P * d):
        raise UlyssesError(2, f"ulysses_o_proj: o {tuple(o.shape)}, w_o {tuple(w_o.shape)} with P={P}")
    y = torch.empty((P, B, n // P, hidden), dtype=o.dtype, device=o.device) if y is None else y
    _check(lib().ulysses_o_proj(B, n, P, hidden, hl * P, d, _p(o), _p(w_o), _p(y), _stream(stream)),
           "ulysses_o_proj")
    return y


def ulysses_qkv_proj_rope_bwd(x, w_qkv, P, H, G, rope_table, dq, dk, dv, positions=None, dx=None, dw=None,
                              workspace=None, stream=None):
    """Backward of ulysses_qkv_proj_rope: x seq layout [P][B][n/P][hidden] and
    w_qkv as for the forward; dq [P][B][H/P][n][128], dk, dv [P][B][G/P][n][128]
    (bf16 head layout) -> (dx bf16 like x, dw float32 like w_qkv)."""
    P_, B, s, hidden = x.shape
    n, d = P * s, 128
    if P_ != P or tuple(w_qkv.shape) != ((H + 2 * G) * d, hidden):
        raise UlyssesError(2, f"ulysses_qkv_proj_rope_bwd: x {tuple(x.shape)}, w {tuple(w_qkv.shape)} with P={P}")
    if positions is not None and (positions.dtype != torch.int32 or tuple(positions.shape) != (B, n)):
        raise UlyssesError(2, f"ulysses_qkv_proj_rope_bwd: positions {tuple(positions.shape)} {positions.dtype}")
    dx = torch.empty_like(x) if dx is None else dx
    dw = torch.empty(w_qkv.shape, dtype=torch.float32, device=x.device) if dw is None else dw
    need = ctypes.c_size_t(0)
    _check(lib().ulysses_qkv_proj_rope_bwd_workspace_size(B, n, H, G, d, ctypes.byref(need)),
           "ulysses_qkv_proj_rope_bwd_workspace_size")
    if workspace is None:
        workspace = torch.empty(max(need.value, 256), dtype=torch.uint8, device=x.device)
    _check(lib().ulysses_qkv_proj_rope_bwd(B, n, P, hidden, H, G, d, _p(x), _p(w_qkv), _p(rope_table),
                                           rope_table.shape[0], _p(positions), _p(dq), _p(dk), _p(dv), _p(dx),
                                           _p(dw), _p(workspace), workspace.numel(), _stream(stream)),
           "ulysses_qkv_proj_rope_bwd")
    return dx, dw


def ulysses_o_proj_bwd(o_seq, w_o, dy, P, do=None, dw_o=None, stream=None):
    """Backward of ulysses_o_proj: o_seq [P][B][n/P][H][128] (the attention output
    in the seq layout), w_o [hidden][H*128], dy seq layout [P][B][n/P][hidden]
    -> (dO bf16 head layout [P][B][H/P][n][128], dW_o float32 like w_o)."""
    P_, B, s, H, d = o_seq.shape
    hidden = w_o.shape[0]
    n = P * s
    if P_ != P or tuple(w_o.shape) != (hidden, H * d) or tuple(dy.shape) != (P, B, s, hidden):
        raise UlyssesError(2, f"ulysses_o_proj_bwd: o {tuple(o_seq.shape)}, w_o {tuple(w_o.shape)}, "
                              f"dy {tuple(dy.shape)} with P={P}")
    do = torch.empty((P, B, H // P, n, d), dtype=o_seq.dtype, device=o_seq.device) if do is None else do
    dw_o = torch.empty(w_o.shape, dtype=torch.float32, device=o_seq.device) if dw_o is None else dw_o
    _check(lib().ulysses_o_proj_bwd(B, n, P, hidden, H, d, _p(o_seq), _p(w_o), _p(dy), _p(do), _p(dw_o),
                                    _stream(stream)), "ulysses_o_proj_bwd")
    return do, dw_o


# ----------------------------------------------------------------- attention

def _desc_from(q, k, mask, cu_seqlens, scale, out_seq_layout=False, deterministic=False):
    P, B, hl, n, d = q.shape
    gl = k.shape[2]
    return make_desc(B, n, P, hl * P, gl * P, d, _dtype_code(q), mask, cu_seqlens, scale,
                     out_seq_layout, deterministic)


def _seq_shape(x):
    """Seq-layout shape [P][B][n/P][heads][d] of a head-layout tensor [P][B][heads/P][n][d]."""
    P, B, hx, n, d = x.shape
    return (P, B, n // P, hx * P, d)


def ulysses_attn_fwd(q, k, v, mask=MASK_CAUSAL, cu_seqlens=None, scale=0.0, o=None, lse=None,
                     out_seq_layout=False, stream=None):
    """Head layout in: q [P][B][H/P][n][d], k, v [P][B][G/P][n][d] -> o like q
    (or, with out_seq_layout, o in the seq layout [P][B][n/P][H][d]: the second
    all-to-all done by the attention kernel), lse float32 [P][B][H/P][n]."""
    desc = _desc_from(q, k, mask, cu_seqlens, scale, out_seq_layout)
    if o is None:
        o = torch.empty(_seq_shape(q), dtype=q.dtype, device=q.device) if out_seq_layout else torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[:4], dtype=torch.float32, device=q.device)
    _check(lib().ulysses_attn_fwd(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(o), _p(lse),
                                  _stream(stream)), "ulysses_attn_fwd")
    return o, lse


def ulysses_attn_bwd_workspace_size(desc: AttnDesc) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().ulysses_attn_bwd_workspace_size(ctypes.byref(desc), ctypes.byref(n)),
           "ulysses_attn_bwd_workspace_size")
    return n.value


def ulysses_attn_bwd(q, k, v, o, lse, dout, mask=MASK_CAUSAL, cu_seqlens=None, scale=0.0,
                     dq=None, dk=None, dv=None, workspace=None, out_seq_layout=False,
                     deterministic=False, stream=None):
    """Gradients of sum(O * dO), inputs in the head layout: dq like q, dk/dv
    like k, or all three in the seq layout with out_seq_layout.
    deterministic: the atomic-free two-pass backward (bitwise repeatable)."""
    desc = _desc_from(q, k, mask, cu_seqlens, scale, out_seq_layout, deterministic)
    mk = (lambda x: torch.empty(_seq_shape(x), dtype=x.dtype, device=x.device)) if out_seq_layout \
        else torch.empty_like
    dq = mk(q) if dq is None else dq
    dk = mk(k) if dk is None else dk
    dv = mk(v) if dv is None else dv
    need = ulysses_attn_bwd_workspace_size(desc)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check(lib().ulysses_attn_bwd(ctypes.byref(desc), _p(q), _p(k), _p(v), _p(o), _p(lse), _p(dout),
                                  _p(dq), _p(dk), _p(dv), _p(workspace), workspace.numel(),
                                  _stream(stream)), "ulysses_attn_bwd")
    return dq, dk, dv


# ---------------------------------------------------------------------- loss

def ulysses_loss_workspace_size(P: int, tokens: int, vocab: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().ulysses_loss_workspace_size(P, tokens, vocab, ctypes.byref(n)),
           "ulysses_loss_workspace_size")
    return n.value


def ulysses_loss_aggregate(logits, labels, P, ignore_index=-100, shard_sum=None, shard_count=None,
                           loss=None, workspace=None, stream=None):
    """logits [T][V] (bf16/fp32; shard r = rows [r*T/P, (r+1)*T/P)), labels int32 [T] ->
    (shard_sum float32 [P], shard_count int64 [P], loss float32 [1]) on the device."""
    T, V = logits.shape
    dev = logits.device
    shard_sum = torch.empty(P, dtype=torch.float32, device=dev) if shard_sum is None else shard_sum
    shard_count = torch.empty(P, dtype=torch.int64, device=dev) if shard_count is None else shard_count
    loss = torch.empty(1, dtype=torch.float32, device=dev) if loss is None else loss
    need = ulysses_loss_workspace_size(P, T, V)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(lib().ulysses_loss_aggregate(P, T, V, _dtype_code(logits), _p(logits), _p(labels),
                                        ignore_index, _p(shard_sum), _p(shard_count), _p(loss),
                                        _p(workspace), workspace.numel(), _stream(stream)),
           "ulysses_loss_aggregate")
    return shard_sum, shard_count, loss


def ulysses_loss_bwd_workspace_size(P: int, tokens: int, vocab: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().ulysses_loss_bwd_workspace_size(P, tokens, vocab, ctypes.byref(n)),
           "ulysses_loss_bwd_workspace_size")
    return n.value


def ulysses_loss_aggregate_bwd(logits, labels, P, ignore_index=-100, dlogits=None, shard_sum=None,
                               shard_count=None, loss=None, workspace=None, stream=None):
    """The aggregated loss and dL/dlogits in one pass: returns (shard_sum, shard_count,
    loss, dlogits); dlogits has the shape and dtype of logits."""
    T, V = logits.shape
    dev = logits.device
    dlogits = torch.empty_like(logits) if dlogits is None else dlogits
    if dlogits.shape != logits.shape or dlogits.dtype != logits.dtype:
        raise ValueError("dlogits must match logits in shape and dtype")
    shard_sum = torch.empty(P, dtype=torch.float32, device=dev) if shard_sum is None else shard_sum
    shard_count = torch.empty(P, dtype=torch.int64, device=dev) if shard_count is None else shard_count
    loss = torch.empty(1, dtype=torch.float32, device=dev) if loss is None else loss
    need = ulysses_loss_bwd_workspace_size(P, T, V)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(lib().ulysses_loss_aggregate_bwd(P, T, V, _dtype_code(logits), _p(logits), _p(labels),
                                            ignore_index, _p(dlogits), _p(shard_sum), _p(shard_count),
                                            _p(loss), _p(workspace), workspace.numel(), _stream(stream)),
           "ulysses_loss_aggregate_bwd")
    return shard_sum, shard_count, loss, dlogits


def ulysses_loss_aggregate_noalloc(logits, labels, P, ignore_index=-100, shard_sum=None,
                                   shard_count=None, loss=None, stream=None):
    """Same as ulysses_loss_aggregate, but the library takes its scratch from a
    fixed array of its own: for callers that cannot allocate device memory
    (see the header for the size limit and the rules of the shared array)."""
    T, V = logits.shape
    dev = logits.device
    shard_sum = torch.empty(P, dtype=torch.float32, device=dev) if shard_sum is None else shard_sum
    shard_count = torch.empty(P, dtype=torch.int64, device=dev) if shard_count is None else shard_count
    loss = torch.empty(1, dtype=torch.float32, device=dev) if loss is None else loss
    _check(lib().ulysses_loss_aggregate_noalloc(P, T, V, _dtype_code(logits), _p(logits), _p(labels),
                                                ignore_index, _p(shard_sum), _p(shard_count), _p(loss),
                                                _stream(stream)), "ulysses_loss_aggregate_noalloc")
    return shard_sum, shard_count, loss


# -------------------------------------------------------------------- misc

def ulysses_read_error() -> int:
    """Read and clear the device error word (synchronises the device)."""
    w = ctypes.c_int32(0)
    _check(lib().ulysses_read_error(ctypes.byref(w)), "ulysses_read_error")
    return w.value


def ulysses_error_word() -> int:
    """Device address of the current device's asynchronous error word (int32)."""
    p = ctypes.c_void_p(0)
    _check(lib().ulysses_error_word(ctypes.byref(p)), "ulysses_error_word")
    return int(p.value or 0)


def ulysses_read_error_info() -> list:
    """Read and clear the whole error record (16 words, see the header)."""
    buf = (ctypes.c_int32 * 16)()
    _check(lib().ulysses_read_error_info(buf, 16), "ulysses_read_error_info")
    return list(buf)


def ulysses_set_wait_limit(cycles: int = 0):
    """Cycles a pipeline wait of the tcgen05 kernels may last before it reports
    ULY_ERR_TIMEOUT (0: the built-in limit).  For tests of the timeout path."""
    _check(lib().ulysses_set_wait_limit(int(cycles)), "ulysses_set_wait_limit")


BLOCK_ORDER_AUTO, BLOCK_ORDER_KV_HEAD_MAJOR, BLOCK_ORDER_HEAVIEST_FIRST = 0, 1, 2


def ulysses_set_attn_block_order(order: int = BLOCK_ORDER_AUTO):
    """Block order of the attention kernels (BLOCK_ORDER_*; the default picks
    per launch).  The results do not depend on it; for tests that compare."""
    _check(lib().ulysses_set_attn_block_order(int(order)), "ulysses_set_attn_block_order")


def ulysses_status_string(status: int) -> str:
    return lib().ulysses_status_string(status).decode()


def ulysses_launch_count() -> int:
    return int(lib().ulysses_launch_count())


def ulysses_profile_enable(on: bool = True):
    _check(lib().ulysses_profile_enable(1 if on else 0), "ulysses_profile_enable")


def ulysses_profile_read() -> dict:
    """{kernel name: (total device ms, launches)} for every kernel timed since
    the last ulysses_profile_enable(True)."""
    L = lib()
    out = {}
    for k in range(L.ulysses_kernel_count()):
        ms, n = ctypes.c_double(0), ctypes.c_int64(0)
        _check(L.ulysses_profile_read(k, ctypes.byref(ms), ctypes.byref(n)), "ulysses_profile_read")
        if n.value:
            out[L.ulysses_kernel_name(k).decode()] = (ms.value, n.value)
    return out
