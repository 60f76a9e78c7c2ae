"""The scalar-A-per-head scan written out in matrix form, float64 numpy.

TEST INFRASTRUCTURE ONLY: the test suite is the only caller. The CUDA
library never imports this module and this module never imports the CUDA
library.

"Mamba & State Space Models — Guide Complet", §5 "Mamba-2" / "SSD — State
Space Dual": when A is one scalar per head, the whole sequence's output is
one masked matrix product, y = (L ◦ S)·u, with L a causal (lower-triangular)
mask and S a structured semiseparable matrix. Written out for head h
(channels d = h·P + p, B and C shared by the heads) with

    Δ_t      = softplus(dt[b,t,h] + dt_bias[h])   (or no softplus)
    Acum_t   = Σ_{k ≤ t} Δ_k·A[h]
    L[i, j]  = exp(Acum_i − Acum_j) for j ≤ i, else 0
    S[i, j]  = C_i · B_j
    y_h      = ((L ◦ S)·diag(Δ))·x_h + diag(exp(Acum))·C·h0_h + D[h]·x_h,

times silu(z). The final state is exp(Acum_last)·h0_h + Σ_j
exp(Acum_last − Acum_j)·Δ_j·B_j ⊗ x_j. Every product is formed as the plain
dense T×T matrix (no chunking), so this is the definition, not an algorithm;
it is pinned against the recurrence oracle in the tests.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np


def _softplus(v: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, v)


def _silu(v: np.ndarray) -> np.ndarray:
    return v / (1.0 + np.exp(-v))


def ssd_matrix_form(x, dt, A, B, C, D=None, z=None, dt_bias=None, softplus: bool = True,
                    h0=None) -> Tuple[np.ndarray, np.ndarray]:
    """y [batch, T, H·P] and the final state [batch, H·P, N] in float64.

    x, z [batch, T, H·P]; dt [batch, T, H]; A, D, dt_bias [H]; B, C
    [batch, T, N]; h0 [batch, H·P, N] or None (zero)."""
    x = np.asarray(x, dtype=np.float64)
    dt = np.asarray(dt, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    C = np.asarray(C, dtype=np.float64)
    batch, T, dim = x.shape
    H = dt.shape[2]
    P = dim // H
    N = B.shape[2]
    Dv = np.zeros(H) if D is None else np.asarray(D, dtype=np.float64)
    bias = np.zeros(H) if dt_bias is None else np.asarray(dt_bias, dtype=np.float64)
    y = np.zeros((batch, T, dim))
    final = np.zeros((batch, dim, N))
    causal = np.tril(np.ones((T, T), dtype=bool))
    for b in range(batch):
        S = C[b] @ B[b].T  # S[i, j] = C_i · B_j
        for h in range(H):
            v = dt[b, :, h] + bias[h]
            delta = _softplus(v) if softplus else v
            acum = np.cumsum(delta * A[h])
            diff = acum[:, None] - acum[None, :]
            L = np.where(causal, np.exp(np.where(causal, diff, 0.0)), 0.0)
            M = (L * S) * delta[None, :]
            xh = x[b, :, h * P:(h + 1) * P]  # [T, P]
            yh = M @ xh + Dv[h] * xh
            hT = (np.exp(acum[-1] - acum) * delta)[:, None] * B[b]  # [T, N]
            state = hT.T @ xh  # [N, P]
            if h0 is not None:
                h0h = np.asarray(h0, dtype=np.float64)[b, h * P:(h + 1) * P, :].T  # [N, P]
                yh = yh + np.exp(acum)[:, None] * (C[b] @ h0h)
                state = state + np.exp(acum[-1]) * h0h
            if z is not None:
                yh = yh * _silu(np.asarray(z, dtype=np.float64)[b, :, h * P:(h + 1) * P])
            y[b, :, h * P:(h + 1) * P] = yh
            final[b, h * P:(h + 1) * P, :] = state.T
    return y, final


def decay_mask(dt, A_h: float, softplus: bool = True, dt_bias: float = 0.0) -> np.ndarray:
    """The mask L of one head and batch row: L[i, j] = exp(Acum_i − Acum_j)
    on j ≤ i, else 0 (dt: [T])."""
    v = np.asarray(dt, dtype=np.float64) + dt_bias
    delta = _softplus(v) if softplus else v
    acum = np.cumsum(delta * A_h)
    T = acum.shape[0]
    causal = np.tril(np.ones((T, T), dtype=bool))
    return np.where(causal, np.exp(np.where(causal, acum[:, None] - acum[None, :], 0.0)), 0.0)
