"""Activation rows aimed at the quantizer's rounding boundaries (test inputs
only: the expected codes always come from the oracle).

Each row holds its absmax A in its first entry, so its scale is s = A / 127
in fp32 (per-token symmetric INT8, LiquidGEMM review page, referee summary:
W4A8 with per-token INT8 activations).  The other entries sit a few ulps to
either side of (k + 1/2) * s for every k in -127 .. 126, where x / s is
within a hair of a half-integer and the rounding of the quotient decides the
code.  Row magnitudes span tiny to huge scales, and one row has a subnormal
scale (its reciprocal overflows)."""
import numpy as np

# absmax of each row: ordinary, small, large, tiny (normal scale), huge,
# subnormal scale
ROW_ABSMAX = (1.0, 3.0e-3, 7.5e4, 1.0e-30, 2.0e33, 1.0e-39)
ULP_OFFSETS = (-64, -16, -6, -5, -4, -3, -2, -1, 0, 1, 2, 3, 4, 5, 6, 16, 64)


def _step(x: np.float32, n: int) -> np.float32:
    """x moved by n ulps (towards +inf for n > 0)."""
    d = np.float32(np.inf) if n > 0 else np.float32(-np.inf)
    for _ in range(abs(n)):
        x = np.nextafter(x, d, dtype=np.float32)
    return x


def boundary_rows(K: int, absmax=ROW_ABSMAX, seed: int = 7) -> np.ndarray:
    """[len(absmax), K] float32; K >= 1.  Entries past the boundary points are
    uniform in (-A, A); every |x| <= A."""
    rng = np.random.default_rng(seed)
    rows = []
    for A in absmax:
        A = np.float32(A)
        s = np.float32(A / np.float32(127.0))
        vals = [A]
        for k in range(-127, 127):
            h = np.float32(np.float32(k + 0.5) * s)
            for n in ULP_OFFSETS:
                v = _step(h, n)
                if abs(v) <= A:
                    vals.append(v)
        vals = np.array(vals, dtype=np.float32)
        if vals.size >= K:
            row = vals[:K].copy()
        else:
            fill = (rng.uniform(-1.0, 1.0, K - vals.size) * float(A)).astype(np.float32)
            row = np.concatenate([vals, np.clip(fill, -A, A)])
        rows.append(row)
    return np.stack(rows).astype(np.float32)
