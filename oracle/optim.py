"""AdamW step for the LoRA parameters (oracle).

Test infrastructure only; see the package docstring.

The pages train only the adapters A and B, with an Adam-type optimiser whose
states may be paged ("QLoRA技术从入门到精通" section 3(3); "LoRA 与 QLoRA：把大
模型微调拆成可负担的工程" section 6.3).  The update rule is AdamW, Adam with
decoupled weight decay (Loshchilov and Hutter, "Decoupled Weight Decay
Regularization"), for step t >= 1 and gradient g (times grad_scale):

    m  <- beta1 m + (1 - beta1) g
    v  <- beta2 v + (1 - beta2) g^2
    m^ = m / (1 - beta1^t),   v^ = v / (1 - beta2^t)
    p  <- p - lr (m^ / (sqrt(v^) + eps) + weight_decay p)

Here every operation is carried out in fp64 on the fp32 inputs.
"""

import numpy as np

F64 = np.float64


def adamw_step(p, g, m, v, t, lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0,
               grad_scale=1.0):
    """Returns the new (p, m, v) in fp64."""
    p, g, m, v = (np.asarray(a, dtype=F64) for a in (p, g, m, v))
    g = g * grad_scale
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** t)
    v_hat = v / (1.0 - beta2 ** t)
    p = p - lr * (m_hat / (np.sqrt(v_hat) + eps) + weight_decay * p)
    return p, m, v
