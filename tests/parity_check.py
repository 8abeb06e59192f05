"""Parity checks shared by the GPU tests: compare a CUDA output with the
oracle's row by row, not only pooled over the whole tensor.

A "row" is one output vector o_{t,h} of length d_h for one (sequence, loop,
head).  Pooling the error over every row of a call hides a single wrong row:
on a 64-row call one row that is 15 % off moves the pooled relative L2 by
about 0.019.  So each check asserts three things at the stated tolerance:

* the pooled relative L2 over all rows;
* the relative L2 of every row on its own;
* every element: |got - ref| <= tol * max|ref_row| (the row's largest
  magnitude), so a few bad elements of an otherwise good row fail too.
"""

import numpy as np


def _as64(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def row_errors(got, ref):
    """(pooled relative L2, per-row relative L2 array, per-element ratio array)
    for arrays whose last axis is the row."""
    got, ref = _as64(got), _as64(ref)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    g2 = got.reshape(-1, got.shape[-1])
    r2 = ref.reshape(-1, ref.shape[-1])
    d = g2 - r2
    pooled = float(np.linalg.norm(d) / max(np.linalg.norm(r2), 1e-300))
    rn = np.linalg.norm(r2, axis=1)
    rows = np.linalg.norm(d, axis=1) / np.maximum(rn, 1e-300)
    inf = np.max(np.abs(r2), axis=1, keepdims=True)
    elem = np.abs(d) / np.maximum(inf, 1e-300)
    return pooled, rows, elem


def assert_rows_close(got, ref, tol, what="", elem_tol=None):
    """Assert the pooled and per-row relative L2 at tolerance tol, and the
    per-element bound at elem_tol (default tol); returns (pooled, worst row)
    for printing."""
    got64 = _as64(got)
    fin = np.isfinite(got64)
    assert np.all(fin), (f"{what}: {int((~fin).sum())} of {fin.size} outputs non-finite "
                         f"(in {int((~fin).reshape(-1, fin.shape[-1]).any(axis=1).sum())} rows)")
    pooled, rows, elem = row_errors(got64, ref)
    worst = int(np.argmax(rows))
    assert pooled <= tol, f"{what}: pooled rel L2 {pooled:.3e} > {tol}"
    assert rows[worst] <= tol, (f"{what}: row {np.unravel_index(worst, got64.shape[:-1])} "
                                f"rel L2 {rows[worst]:.3e} > {tol}")
    e = float(elem.max())
    et = tol if elem_tol is None else elem_tol
    assert e <= et, f"{what}: element error {e:.3e} of the row's max magnitude > {et}"
    return pooled, float(rows[worst])
