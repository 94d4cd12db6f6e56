"""Comparison rules shared by the GPU parity tests.

Selection (index sets): the GPU set G and the oracle set O must have the same size,
and every position in G xor O must lie in the oracle's tie band around its k-th
value: |s'_j - s'_(k)| <= 1e-3 * |s'_(k)| + 1e-6. Outside the band the sets agree
exactly. Outputs: max-abs error <= 1e-4 for fp32 and <= 2e-2 for bf16.
"""
import numpy as np

ATOL_F32 = 1e-4
ATOL_BF16 = 2e-2
BAND_REL = 1e-3
BAND_ABS = 1e-6


def atol_for(dtype_name: str) -> float:
    return ATOL_F32 if dtype_name in ("f32", "float32") else ATOL_BF16


def check_selection(gpu_idx, gpu_count, ref_idx, ref_count, ref_sprime, mid0, topk):
    """Compare one sequence's selection. Returns the number of band swaps."""
    gpu_idx = np.asarray(gpu_idx, dtype=np.int64)
    cnt = int(gpu_count)
    assert cnt == int(ref_count), (cnt, ref_count)
    sel = gpu_idx[:cnt]
    assert np.all(gpu_idx[cnt:topk] == -1), "padding after count must be -1"
    assert np.all(np.diff(sel) > 0), "indices must be strictly ascending"
    if cnt == 0:
        return 0
    n_mid = len(ref_sprime)
    assert sel.min() >= mid0 and sel.max() < mid0 + n_mid, "index outside the middle"
    ref = set(np.asarray(ref_idx[:cnt], dtype=np.int64).tolist())
    got = set(sel.tolist())
    diff = got ^ ref
    if not diff:
        return 0
    sp = np.asarray(ref_sprime, dtype=np.float64)
    kth = np.sort(sp)[::-1][cnt - 1]
    tol = BAND_REL * abs(kth) + BAND_ABS
    for j in diff:
        assert abs(sp[j - mid0] - kth) <= tol, f"position {j} differs outside the tie band " \
                                               f"(s'={sp[j - mid0]}, k-th={kth}, tol={tol})"
    return len(diff) // 2


def max_abs(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    assert np.isfinite(a).all(), "non-finite values in the GPU output"
    return float(np.abs(a - b).max()) if a.size else 0.0
