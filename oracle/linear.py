"""fp64 CPU oracle of the projection GEMMs around attention (a linear layer without
bias), forward and backward.

TEST INFRASTRUCTURE ONLY.  The tests and the CPU-baseline leg of the benchmark are
the only callers; the CUDA library never imports or calls anything here, and this
module imports nothing from the library.

The three products are the ones the Forge paper ("Building an LLM Training Framework
from Scratch in C++ and Metal on Apple Silicon") measures for training (section
"Results", the GEMM table, and section "Finding 4.2" for the transposed variants):
with tokens t, input features i and output features o,

  forward   Y  = X W^T      Y[t][o]  = sum_i X[t][i] W[o][i]
  backward  dX = dY W       dX[t][i] = sum_o dY[t][o] W[o][i]
            dW = dY^T X     dW[o][i] = sum_t dY[t][o] X[t][i]

Each is one library matrix product in fp64 on the exact values of the inputs; no
blocking or reordering beyond that.
"""
from __future__ import annotations

import numpy as np


def linear_fwd(x, w):
    """Y = X W^T.  x: [tokens, in], w: [out, in] -> [tokens, out]."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T


def linear_bwd_dx(dy, w):
    """dX = dY W.  dy: [tokens, out], w: [out, in] -> [tokens, in]."""
    return np.asarray(dy, dtype=np.float64) @ np.asarray(w, dtype=np.float64)


def linear_bwd_dw(dy, x):
    """dW = dY^T X.  dy: [tokens, out], x: [tokens, in] -> [out, in]."""
    return np.asarray(dy, dtype=np.float64).T @ np.asarray(x, dtype=np.float64)
