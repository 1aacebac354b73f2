"""Shared comparison helpers and tolerances for the GPU parity tests."""
import numpy as np
import torch

# Tolerances (stated for the workloads): permutations bit-exact; fp32
# attention within 1e-5 max-abs; bf16 attention and gradients within 2e-2
# max-abs and 1e-2 relative L2; the loss within 1e-5 relative (the pages' SP
# vs DP loss difference bound).
F32_MAX_ABS = 1e-5
BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 1e-2
LOSS_REL = 1e-5
LSE_BF16_MAX_ABS = 2e-3   # LSE is fp32 from fp32 scores; only input rounding matters


def to64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def f32_inputs(x: torch.Tensor) -> np.ndarray:
    """Exact fp32 copy of a (bf16 or fp32) tensor for the oracle."""
    return x.detach().to("cpu", torch.float32).numpy()


def rel_l2(a, b):
    a, b = to64(a), to64(b)
    den = np.linalg.norm(b.ravel())
    return float(np.linalg.norm((a - b).ravel()) / (den if den > 0 else 1.0))


def max_abs(a, b):
    a, b = to64(a), to64(b)
    return float(np.abs(a - b).max()) if a.size else 0.0


BF16_ULP_REL = 2.0 ** -7   # one bf16 ulp is at most 2^-7 |x| (8 significant bits)


def assert_bf16_close(got, ref, what="", max_abs_tol=BF16_MAX_ABS, rel_tol=BF16_REL_L2):
    """Element-wise |got - ref| <= max(2e-2, one bf16 ulp of |ref|) and
    relative L2 <= 1e-2.  The ulp term only matters for |ref| > 2.56, where a
    bf16 output cannot resolve 2e-2 (the exact value rounded to bf16 may
    already be 2^-8 |ref| away); below that the bound is the plain 2e-2."""
    g, r = to64(got), to64(ref)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    err = np.abs(g - r)
    bound = np.maximum(max_abs_tol, BF16_ULP_REL * np.abs(r))
    worst = float((err / bound).max()) if err.size else 0.0
    ma, rl = (float(err.max()) if err.size else 0.0), rel_l2(g, r)
    assert worst <= 1.0 and rl <= rel_tol, \
        f"{what}: max_abs={ma:.3e} (worst err/bound {worst:.2f}) rel_l2={rl:.3e}"
    return ma, rl


def sample_rows(n: int, P: int, k: int = 64, extra=(), seed: int = 0):
    """Rows to check at large n: first/last rows of every shard, the ragged tail,
    given extra positions (document boundaries), and k spread at random."""
    s = n // P
    rows = set()
    for r in range(P):
        rows.update([r * s, r * s + 1, (r + 1) * s - 1])
    rows.update([0, n - 1, max(0, n - 128), max(0, n - 129)])
    for e in extra:
        for dlt in (-1, 0, 1):
            if 0 <= e + dlt < n:
                rows.add(e + dlt)
    rng = np.random.default_rng(seed)
    rows.update(rng.integers(0, n, k).tolist())
    return np.array(sorted(rows), dtype=np.int32)
