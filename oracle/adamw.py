"""fp64 CPU oracle of one AdamW step over a list of tensors.

TEST INFRASTRUCTURE ONLY.  The tests and the CPU-baseline leg of the benchmark are
the only callers; the CUDA library never imports or calls anything here, and this
module imports nothing from the library.

The step follows the training recipe of the Forge paper ("Building an LLM Training
Framework from Scratch in C++ and Metal on Apple Silicon"), sections "Training
details" and "Related work": AdamW with decoupled weight decay applied only to
parameters of rank two or more, epsilon outside the square root, and gradient
clipping at a global norm, the clip factor applied where the optimizer reads the
gradient.  In the order written there:

  1. global norm   N = sqrt(sum over all tensors and elements of g^2)
  2. clip factor   c = max_norm / N if max_norm > 0 and N > max_norm, else 1
  3. per element   g' = c g
                   m  = beta1 m + (1 - beta1) g'
                   v  = beta2 v + (1 - beta2) g'^2
                   m^ = m / (1 - beta1^t),  v^ = v / (1 - beta2^t)
                   p  = p - lr (m^ / (sqrt(v^) + eps) + wd p)
     with wd = weight_decay for the decayed tensors and 0 for the others, and p on
     the right the value before the step.

Readings where the pages are silent: the clip factor is max_norm / N exactly (no
epsilon added to N), the form of the llm.c code the pages say they follow; the
moments, bias corrections and hyperparameters are the standard AdamW ones, passed
in as arguments.
"""
from __future__ import annotations

import math

import numpy as np


def global_norm(grads) -> float:
    """Step 1: the l2 norm over every element of every gradient (fp64)."""
    return math.sqrt(sum(float(np.sum(np.asarray(g, dtype=np.float64) ** 2)) for g in grads))


def clip_factor(norm: float, max_norm: float) -> float:
    """Step 2: the factor folded into the gradient read."""
    return max_norm / norm if (max_norm > 0 and norm > max_norm) else 1.0


def adamw_step(params, grads, exp_avgs, exp_avg_sqs, decay, lr, beta1, beta2, eps,
               weight_decay, step, max_norm):
    """One step.  Arrays of any shape (fp64 copies are made); decay: one bool per tensor.
    Returns (new params, new exp_avgs, new exp_avg_sqs, global norm)."""
    norm = global_norm(grads)
    c = clip_factor(norm, max_norm)
    bc1 = 1.0 - beta1 ** step
    bc2 = 1.0 - beta2 ** step
    new_p, new_m, new_v = [], [], []
    for p, g, m, v, dec in zip(params, grads, exp_avgs, exp_avg_sqs, decay):
        p = np.array(p, dtype=np.float64)
        g = c * np.asarray(g, dtype=np.float64)
        m = beta1 * np.asarray(m, dtype=np.float64) + (1.0 - beta1) * g
        v = beta2 * np.asarray(v, dtype=np.float64) + (1.0 - beta2) * g * g
        m_hat = m / bc1
        v_hat = v / bc2
        wd = weight_decay if dec else 0.0
        p = p - lr * (m_hat / (np.sqrt(v_hat) + eps) + wd * p)
        new_p.append(p)
        new_m.append(m)
        new_v.append(v)
    return new_p, new_m, new_v, norm
