"""Float64 AdamW update (test infrastructure, like the rest of ``oracle``).

The optimizer paragraph of the nanochat announcement (vpshk.cn) names Muon +
AdamW, with a plan to drop Muon for Adam with a learning rate per module.  The
pages define neither; AdamW is the textbook one: Adam's bias-corrected moment
estimates (Kingma & Ba, "Adam: A Method for Stochastic Optimization", 2015)
with the weight decay applied to the parameters, decoupled from the gradient
(Loshchilov & Hutter, "Decoupled Weight Decay Regularization", 2019).  Muon is
not defined on the pages and is not implemented.
"""
from __future__ import annotations

import numpy as np


def adamw_step(theta, grad, m, v, step, lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0):
    """One AdamW update at step t = `step` (1 for the first), in place on
    float64 arrays theta, m, v:

        m <- b1 m + (1 - b1) g
        v <- b2 v + (1 - b2) g^2
        m_hat = m / (1 - b1^t),  v_hat = v / (1 - b2^t)
        theta <- theta - lr (weight_decay theta + m_hat / (sqrt(v_hat) + eps))
    """
    g = np.asarray(grad, dtype=np.float64)
    m *= beta1
    m += (1.0 - beta1) * g
    v *= beta2
    v += (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** step)
    v_hat = v / (1.0 - beta2 ** step)
    theta -= lr * (weight_decay * theta + m_hat / (np.sqrt(v_hat) + eps))
    return theta, m, v
