"""Offline calibration of the 16-entry level table of the LUT4 cache format.

UltraQuant (page "UltraQuant: 4-bit KV caching for long agents", method
section) refits the 16-entry table on captured activations instead of using
the theoretical Lloyd-Max centroids. Here the activations are synthetic (no
model is in scope): rows are rotated with the cache's rotation, normalised
to u = (y - m)/s in [0, 15] with the cache's row statistics (minimum and
(maximum - minimum)/15, in float64 -- calibration only sees the distribution,
not the bit-exact parameters), and a one-dimensional Lloyd-Max iteration
(nearest-level cells, then cell means) runs on the pooled u values. The
levels are finally rounded to the 1/16 grid the decode's integer tensor-core
path needs (16 t is an integer in [0, 240]), strictly increasing.

This is host code for an offline step; the cache path itself (append,
dequantize, decode) runs in the library's kernels with the table as input.
"""

import numpy as np


def _hadamard(b):
    h = np.array([[1.0]])
    while h.shape[0] < b:
        h = np.block([[h, h], [h, -h]])
    return h / np.sqrt(b)


def rotate_rows(x, rot_block):
    """Block Hadamard rotation (natural order, orthonormal) of rows [..., d]
    in float64; rot_block 0 leaves the rows as they are."""
    x = np.asarray(x, np.float64)
    if not rot_block:
        return x.copy()
    d = x.shape[-1]
    h = _hadamard(rot_block)
    y = x.reshape(-1, d // rot_block, rot_block) @ h.T
    return y.reshape(x.shape)


def normalised_codes_domain(y):
    """u = (y - min) / ((max - min) / 15) per row, in [0, 15]."""
    mn = y.min(axis=-1, keepdims=True)
    mx = y.max(axis=-1, keepdims=True)
    s = (mx - mn) / 15.0
    s = np.where(s > 0, s, 1.0)
    return (y - mn) / s


def lloyd_max(u, iters=60, init=None):
    """One-dimensional Lloyd-Max (k-means) with 16 levels on samples u."""
    u = np.sort(np.asarray(u, np.float64).ravel())
    t = np.arange(16, dtype=np.float64) if init is None else np.array(init, np.float64)
    for _ in range(iters):
        mids = 0.5 * (t[1:] + t[:-1])
        cell = np.searchsorted(mids, u, side="left")  # ties to the lower level
        sums = np.bincount(cell, weights=u, minlength=16)
        cnts = np.bincount(cell, minlength=16)
        new = np.where(cnts > 0, sums / np.maximum(cnts, 1), t)
        if np.allclose(new, t, rtol=0, atol=1e-12):
            t = new
            break
        t = new
    return t


def round_to_grid(t):
    """Levels on the 1/16 grid in [0, 15], strictly increasing (a level that
    rounds onto its predecessor moves up one grid step, and down from the
    top when the grid runs out), float32."""
    g = np.sort(np.clip(np.round(np.asarray(t, np.float64) * 16.0), 0, 240)).astype(np.int64)
    for k in range(1, 16):
        g[k] = max(g[k], g[k - 1] + 1)
    if g[15] > 240:
        g[15] = 240
        for k in range(14, -1, -1):
            g[k] = min(g[k], g[k + 1] - 1)
    return (g / 16.0).astype(np.float32)


def calibrate_levels(rows, rot_block, iters=60):
    """Level table for rows [N][d] of synthetic activations (float) rotated
    with a block Hadamard of size rot_block (0: none)."""
    u = normalised_codes_domain(rotate_rows(rows, rot_block))
    return round_to_grid(lloyd_max(u, iters))
