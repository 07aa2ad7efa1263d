"""AdamW update of the adapters, in fp64 (test infrastructure, like the rest of ``oracle``).

The adapters are the trained parameters and the optimizer state lives beside them ([LACH] "Step 5":
lr 2e-4; [CODE] "Why GPU Memory Has Always Been the Bottleneck": Adam keeps two extra tensors per
parameter). The rule is Adam with decoupled weight decay (Loshchilov & Hutter, "Decoupled Weight
Decay Regularization"), with bias corrections 1 - beta^t:

    m <- b1 m + (1 - b1) g ;  v <- b2 v + (1 - b2) g^2
    p <- p (1 - lr wd) - lr / (1 - b1^t) * m / (sqrt(v) / sqrt(1 - b2^t) + eps)

Pinned against torch.optim.AdamW (a library routine) in the CPU tests.
"""
from __future__ import annotations

import numpy as np


def adamw_step(p, g, m, v, t, lr=2e-4, b1=0.9, b2=0.999, eps=1e-8, wd=0.0):
    """One update at step t (t >= 1). Returns new (p, m, v); inputs are not modified."""
    p, g, m, v = (np.asarray(a, dtype=np.float64) for a in (p, g, m, v))
    m = b1 * m + (1.0 - b1) * g
    v = b2 * v + (1.0 - b2) * g * g
    p = p * (1.0 - lr * wd) - (lr / (1.0 - b1 ** t)) * m / (np.sqrt(v) / np.sqrt(1.0 - b2 ** t) + eps)
    return p, m, v
