"""CPU-only checks of the C ABI: the library loads, exports every function the
header declares, and rejects bad arguments before launching anything (these
calls validate on the host and never reach a kernel)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ulysses.h")


@pytest.fixture(scope="module")
def L():
    from long_context_sequence_all_b200 import build, ulysses
    build.build()
    return ulysses.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ulysses_\w+)\s*\(", text)))


def test_header_declares_the_five_path_entry_points():
    names = declared_functions()
    for n in ["ulysses_seq_to_head", "ulysses_attn_fwd", "ulysses_attn_bwd", "ulysses_head_to_seq",
              "ulysses_loss_aggregate"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    from long_context_sequence_all_b200 import ulysses
    assert set(ulysses.EXPORTS) <= set(declared_functions())


def test_status_strings(L):
    from long_context_sequence_all_b200 import ulysses
    for code, name in ulysses.STATUS.items():
        assert ulysses.ulysses_status_string(code)
    assert ulysses.ulysses_status_string(0) == "ok"


def test_permute_validation(L):
    vp = ctypes.c_void_p
    a, b = vp(1 << 20), vp(1 << 30)   # never dereferenced: validation fails first
    assert L.ulysses_seq_to_head(1, 1024, 4, 8, 64, 4, None, b, None) == 1        # NULL
    assert L.ulysses_seq_to_head(1, 1022, 4, 8, 64, 4, a, b, None) == 2           # n % P
    assert L.ulysses_seq_to_head(1, 1024, 4, 6, 64, 4, a, b, None) == 2           # heads % P
    assert L.ulysses_seq_to_head(1, 1024, 4, 8, 64, 3, a, b, None) == 3           # elem bytes
    assert L.ulysses_seq_to_head(1, 1024, 4, 8, 6, 2, a, b, None) == 4            # row not 16 B
    assert L.ulysses_seq_to_head(1, 1024, 4, 8, 64, 4, vp((1 << 20) + 4), b, None) == 4  # misaligned
    assert L.ulysses_head_to_seq(1, 1024, 4, 8, 64, 4, a, vp((1 << 20) + 4096), None) == 5  # overlap
    assert L.ulysses_seq_to_head(0, 1024, 4, 8, 64, 4, a, b, None) == 2


def test_kv_copy_validation(L):
    vp = ctypes.c_void_p
    a, b = vp(1 << 20), vp(1 << 30)
    rep, red = L.ulysses_kv_seq_to_head_replicated, L.ulysses_kv_head_to_seq_reduce
    assert rep(1, 1024, 8, 2, 128, 2, None, b, None) == 1                 # NULL
    assert rep(1, 1024, 8, 3, 128, 2, a, b, None) == 2                    # P % G
    assert rep(1, 1020, 8, 2, 128, 2, a, b, None) == 2                    # n % P
    assert rep(1, 1024, 8, 2, 128, 3, a, b, None) == 3                    # elem bytes
    assert rep(1, 1024, 8, 2, 4, 2, a, b, None) == 4                      # row not 16 B
    # the copies (dst, P rows per position) overlap a source placed inside them
    assert rep(1, 1024, 8, 2, 128, 2, vp((1 << 20) + 1024 * 2 * 256), a, None) == 5
    assert red(1, 1024, 8, 2, 128, 7, a, b, None) == 3                    # dtype
    assert red(1, 1024, 8, 3, 128, 1, a, b, None) == 2
    assert red(1, 1024, 8, 2, 128, 1, a, vp((1 << 20) + 1024 * 8 * 256 - 16), None) == 5
    assert red(1, 1024, 8, 2, 128, 1, vp((1 << 20) + 8), b, None) == 4    # misaligned


def test_shift_labels_validation(L):
    vp = ctypes.c_void_p
    ids, lab, cu = vp(1 << 20), vp(1 << 30), vp(1 << 24)
    f = L.ulysses_shift_labels
    assert f(1, 1024, 4, None, None, 0, 1024, -100, lab, None) == 1
    assert f(1, 1023, 4, ids, None, 0, 1023, -100, lab, None) == 2        # n % P
    assert f(1, 1024, 4, ids, None, 0, 1025, -100, lab, None) == 2        # valid_len > n
    assert f(1, 1024, 4, ids, None, 0, -1, -100, lab, None) == 2
    assert f(1, 1024, 4, ids, None, 3, 1024, -100, lab, None) == 1        # docs without cu
    assert f(2, 1024, 4, ids, None, 0, 1024, -100, vp((1 << 20) + 4096), None) == 5
    assert f(1, 1024, 4, ids, vp((1 << 30) + 64), 2, 1024, -100, lab, None) == 5  # cu inside labels


def test_projection_validation(L):
    vp = ctypes.c_void_p
    x, w, tab, q, k, v = (vp(1 << (30 + i)) for i in range(6))
    f = L.ulysses_qkv_proj_rope
    args = lambda **kw: [kw.get("B", 1), kw.get("n", 8192), kw.get("P", 4), kw.get("hidden", 2560),
                         kw.get("H", 32), kw.get("G", 8), kw.get("d", 128), x, w, tab,
                         kw.get("max_pos", 8192), None, q, k, v, None]
    assert f(*args(n=8190)) == 2                       # n % P
    assert f(*args(G=2)) == 6                          # fewer KV heads than ranks: not fused
    assert f(*args(d=64)) == 6
    assert f(*args(hidden=2500)) == 6                  # hidden % 64
    assert f(*args(max_pos=100)) == 2                  # table shorter than the sequence
    a = args()
    a[12] = vp((1 << 30) + 64)                         # q inside x
    assert f(*a) == 5
    a = args()
    a[7] = None
    assert f(*a) == 1
    g = L.ulysses_o_proj
    assert g(1, 8192, 4, 2500, 32, 128, x, w, q, None) == 6           # hidden % 256
    assert g(1, 8190, 4, 2560, 32, 128, x, w, q, None) == 2
    assert g(1, 8192, 4, 2560, 32, 128, x, w, vp((1 << 30) + 16), None) == 5
    assert L.ulysses_rope_table(0, 128, 1e6, tab, None) == 2
    assert L.ulysses_rope_table(8192, 127, 1e6, tab, None) == 2
    assert L.ulysses_rope_table(8192, 128, 0.5, tab, None) == 2
    assert L.ulysses_rope_table(8192, 128, 1e6, vp((1 << 30) + 4), None) == 4


def test_attn_desc_validation(L):
    from long_context_sequence_all_b200 import ulysses as U
    n = ctypes.c_size_t(0)
    ok = U.make_desc(1, 8192, 4, 32, 8, 128, U.ULY_BF16, U.MASK_CAUSAL)
    assert L.ulysses_attn_bwd_workspace_size(ctypes.byref(ok), ctypes.byref(n)) == 0
    assert n.value >= 8192 * 32 * 4
    bad = [U.make_desc(1, 8190, 4, 32, 8, 128, U.ULY_BF16, 1),   # n % P
           U.make_desc(1, 8192, 4, 30, 8, 128, U.ULY_BF16, 1),   # H % P
           U.make_desc(1, 8192, 4, 32, 6, 128, U.ULY_BF16, 1),   # G % P, H % G
           U.make_desc(1, 8192, 4, 32, 8, 128, 7, 1)]            # dtype
    codes = [L.ulysses_attn_bwd_workspace_size(ctypes.byref(d), ctypes.byref(n)) for d in bad]
    assert codes == [2, 2, 2, 3]
    assert L.ulysses_attn_bwd_workspace_size(
        ctypes.byref(U.make_desc(1, 8192, 4, 32, 8, 64, U.ULY_BF16, 1)), ctypes.byref(n)) == 6
    assert L.ulysses_attn_bwd_workspace_size(
        ctypes.byref(U.make_desc(1, 8192, 4, 32, 8, 128, U.ULY_BF16, 2)), ctypes.byref(n)) == 1  # no cu
    d = U.make_desc(1, 8192, 4, 32, 8, 128, U.ULY_BF16, 1)
    vp = ctypes.c_void_p
    assert L.ulysses_attn_fwd(ctypes.byref(d), None, vp(1 << 20), vp(1 << 21), vp(1 << 22),
                              vp(1 << 23), None) == 1
    # bwd without workspace
    assert L.ulysses_attn_bwd(ctypes.byref(d), *[vp(1 << (20 + i)) for i in range(9)], None, 0, None) == 10


def test_attn_desc_flags_and_workspace_sizes(L):
    """out_seq_layout and deterministic take 0 or 1.  The bf16 workspace holds
    D and LSE log2(e) per query row (n rounded up to 128 per head); the fused
    backward adds its fp32 dQ accumulator (512 bytes per padded query row)
    after a 256-byte boundary."""
    from long_context_sequence_all_b200 import ulysses as U
    n = ctypes.c_size_t(0)
    B, N, P, H, G = 1, 8000, 4, 32, 8
    rows_pad = B * H * ((N + 127) // 128 * 128)
    stats = 2 * 4 * ((rows_pad + 63) // 64 * 64)
    det = U.make_desc(B, N, P, H, G, 128, U.ULY_BF16, 1, deterministic=True)
    assert L.ulysses_attn_bwd_workspace_size(ctypes.byref(det), ctypes.byref(n)) == 0
    assert n.value == stats
    fused = U.make_desc(B, N, P, H, G, 128, U.ULY_BF16, 1, out_seq_layout=True)
    assert L.ulysses_attn_bwd_workspace_size(ctypes.byref(fused), ctypes.byref(n)) == 0
    assert n.value == (stats + 255) // 256 * 256 + rows_pad * 128 * 4
    for field in ("out_seq_layout", "deterministic"):
        bad = U.make_desc(B, N, P, H, G, 128, U.ULY_BF16, 1)
        setattr(bad, field, 2)
        assert L.ulysses_attn_bwd_workspace_size(ctypes.byref(bad), ctypes.byref(n)) == 2


def test_loss_validation(L):
    vp = ctypes.c_void_p
    n = ctypes.c_size_t(0)
    assert L.ulysses_loss_workspace_size(4, 65536, 8192, ctypes.byref(n)) == 0 and n.value > 0
    assert L.ulysses_loss_workspace_size(4, 65535, 8192, ctypes.byref(n)) == 2
    args = [vp(1 << 30), vp(1 << 20), -100, vp(1 << 21), vp(1 << 22), vp(1 << 23), vp(1 << 24), 1 << 20, None]
    assert L.ulysses_loss_aggregate(4, 1023, 8192, 1, *args) == 2
    assert L.ulysses_loss_aggregate(4, 1024, 8191, 1, *args) == 4           # row not 16 B
    assert L.ulysses_loss_aggregate(4, 1024, 8192, 9, *args) == 3
    small = args[:-3] + [vp(1 << 24), 8, None]
    assert L.ulysses_loss_aggregate(4, 1024, 8192, 1, *small) == 10


def test_library_has_no_cpu_fallback_symbols():
    """The product binding never imports the oracle."""
    src = open(os.path.join(ROOT, "long_context_sequence_all_b200", "ulysses.py")).read()
    assert "oracle" not in src.replace("no fallback", "")


def test_smoke_shape_passes_host_validation(L):
    """The shape smoke() runs on the GPU is one the library accepts (H, G
    divisible by P, H by G), so the round-end smoke cannot fail on validation."""
    import __graft_entry__ as ge
    from long_context_sequence_all_b200 import ulysses as U
    P, n, H, G, d = ge.SMOKE_SHAPE
    n_ws = ctypes.c_size_t(0)
    desc = U.make_desc(1, n, P, H, G, d, U.ULY_BF16, U.MASK_CAUSAL)
    assert L.ulysses_attn_bwd_workspace_size(ctypes.byref(desc), ctypes.byref(n_ws)) == 0
    assert L.ulysses_loss_bwd_workspace_size(P, 256, 8192, ctypes.byref(n_ws)) == 0


def test_every_profiled_kernel_has_a_distinct_name(L):
    """The per-kernel timing table names every kernel id (an id without a
    name would make the profile unreadable)."""
    names = [L.ulysses_kernel_name(k) for k in range(L.ulysses_kernel_count())]
    assert all(n for n in names), names
    names = [n.decode() for n in names]
    assert len(set(names)) == len(names) and "unknown" not in names
    for k in ("attn_fwd_sm100", "attn_dkdv_sm100", "attn_dq_sm100", "seq_to_head", "head_to_seq",
              "loss_partial", "qkv_proj_sm100", "o_proj_sm100", "kv_seq_to_head_rep", "shift_labels"):
        assert k in names
    assert L.ulysses_kernel_name(L.ulysses_kernel_count()) == b"unknown"


def test_loss_gradient_validation(L):
    vp = ctypes.c_void_p
    T, V, P = 1024, 8192, 4
    n = ctypes.c_size_t(0)
    assert L.ulysses_loss_bwd_workspace_size(P, T, V, ctypes.byref(n)) == 0 and n.value > 0
    need = n.value
    z, y, dz = vp(1 << 32), vp(1 << 30), vp(1 << 34)           # logits 16 MiB, labels, dlogits
    S, C, Lo, ws = vp(1 << 24), vp((1 << 24) + 4096), vp((1 << 24) + 8192), vp(1 << 26)
    f = L.ulysses_loss_aggregate_bwd
    ok = [P, T, V, 1, z, y, -100, dz, S, C, Lo, ws, need, None]
    bad = list(ok); bad[7] = None
    assert f(*bad) == 1                                          # no dlogits
    bad = list(ok); bad[12] = need - 16
    assert f(*bad) == 10                                         # workspace too small
    bad = list(ok); bad[7] = vp((1 << 32) + 1024)
    assert f(*bad) == 5                                          # dlogits inside the logits
    bad = list(ok); bad[11] = vp((1 << 34) + 4096)
    assert f(*bad) == 5                                          # workspace inside dlogits
    bad = list(ok); bad[7] = vp((1 << 34) + 8)
    assert f(*bad) == 4                                          # misaligned dlogits
    bad = list(ok); bad[1] = T - 1
    assert f(*bad) == 2                                          # tokens % P


def test_error_word_null_argument(L):
    assert L.ulysses_error_word(None) == 1


def test_attn_block_order_setter_validates(L):
    """ulysses_set_attn_block_order takes the three ULY_BLOCK_ORDER_* values
    and rejects anything else with ULY_ERR_SHAPE (no device work)."""
    try:
        for order in (1, 2, 0):
            assert L.ulysses_set_attn_block_order(order) == 0
        for bad in (-1, 3, 100):
            assert L.ulysses_set_attn_block_order(bad) == 2
    finally:
        L.ulysses_set_attn_block_order(0)
