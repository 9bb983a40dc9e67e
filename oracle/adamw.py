"""One AdamW step on the LoRA parameters, in float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): the CUDA path never imports this.

"QLoRA Paper Breakdown: 4-Bit NormalFloat (NF4), Double Quantization, and Paged Optimizers"
(fullstackaihub teardown), section 5: the AdamW states m_t, v_t of the LoRA parameters live
in unified memory, evicted to host RAM under memory pressure and paged back for the optimizer
step; "QLoRA, explained." step 6: only the adapters are optimized.

Reading: the pages name the optimizer (paged AdamW) but give no update formula; the plainest
reading is AdamW with decoupled weight decay:

    m = b1 m + (1 - b1) g
    v = b2 v + (1 - b2) g^2
    p = p - lr ( (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps) + wd p )

with fp32 parameters and states (the gradients are the adapters' bf16 gradients).  Pins
(``tests/test_oracle_adamw.py``): the first step from zero states moves every parameter by
lr * g / (|g| + eps) (bias correction makes m-hat = g and v-hat = g^2); a zero gradient with
zero states leaves only the decay p (1 - lr wd); a hand-computed two-step example in exact
rationals (with a square root that is exact).
"""

from __future__ import annotations

import numpy as np


def adamw_step(p, g, m, v, lr: float, beta1: float, beta2: float, eps: float, weight_decay: float, step: int):
    """Returns (p, m, v) after step number `step` (1-based), all float64."""
    p = np.asarray(p, np.float64)
    g = np.asarray(g, np.float64)
    m = beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * g
    v = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * g * g
    mhat = m / (1.0 - beta1 ** step)
    vhat = v / (1.0 - beta2 ** step)
    p = p - lr * (mhat / (np.sqrt(vhat) + eps) + weight_decay * p)
    return p, m, v
