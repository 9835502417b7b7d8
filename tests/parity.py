"""Shared helpers of the GPU parity tests: run the C-ABI path on seeded inputs and
compare with the fp64 oracle on the same inputs.

Tolerances: bf16 outputs with fp32 accumulation must stay within max-abs 2e-2 and
mean-abs 2e-3 of the oracle; as the outputs shrink like 1/sqrt(len) at long
context, the relative L2 error (<= 1e-2) and the lse error (<= 1e-2 absolute) are
checked too.  fp32 caches get the tighter 1e-4 / 1e-5 / 1e-4 bounds.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL = {
    torch.bfloat16: dict(max_abs=2e-2, mean_abs=2e-3, rel_l2=1e-2, lse=1e-2),
    torch.float32: dict(max_abs=1e-4, mean_abs=1e-5, rel_l2=1e-4, lse=1e-4),
}


def bits(t: torch.Tensor) -> np.ndarray:
    """A torch tensor as what the oracle reads: bf16 -> uint16 bit patterns, fp32 -> float32."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def errors(got, want, got_lse=None, want_lse=None):
    g = np.asarray(got, dtype=np.float64)
    w = np.asarray(want, dtype=np.float64)
    d = np.abs(g - w)
    e = dict(max_abs=float(d.max()), mean_abs=float(d.mean()),
             rel_l2=float(np.linalg.norm(g - w) / max(np.linalg.norm(w), 1e-30)))
    if got_lse is not None:
        e["lse"] = float(np.abs(np.asarray(got_lse, np.float64) - np.asarray(want_lse, np.float64)).max())
    return e


def assert_close(got, want, dtype, got_lse=None, want_lse=None, what=""):
    e = errors(got, want, got_lse, want_lse)
    tol = TOL[dtype]
    bad = {k: (v, tol[k]) for k, v in e.items() if v > tol[k]}
    assert not bad, f"{what}: exceeds tolerance {bad} (all errors {e})"
    return e


def oracle_rows(q, k, v, mask_row, S, W, pos0, rows=None, scale=None):
    """Oracle output for query tensor q [B][n][Hq][d] at positions pos0.. over the dense
    history k, v [B][L][Hkv][d] (torch tensors, any device)."""
    return oracle.attend(bits(q), bits(k), bits(v), np.asarray(mask_row, dtype=bool), S, W, pos0=pos0,
                         scale=scale, rows=rows)
