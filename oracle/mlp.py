"""fp64 loss of the MLP classifier used by the small synthetic workload.

TEST INFRASTRUCTURE (see oracle/__init__.py).  The model is the one the workload
names: input -> Linear -> ReLU -> Linear -> logits, mean cross-entropy with natural log.
The flat parameter order is W1[hidden][in], b1[hidden], W2[out][hidden], b2[out].
The loss is evaluated in inference mode only, as the zero-order method requires
("Probe-Space Preconditioning for Fast and Stable Zero-Order Training", abstract).
"""
import numpy as np


def unflatten(P, n_in, n_hidden, n_out):
    P = np.asarray(P, np.float64)
    o = 0
    W1 = P[o:o + n_hidden * n_in].reshape(n_hidden, n_in); o += n_hidden * n_in
    b1 = P[o:o + n_hidden]; o += n_hidden
    W2 = P[o:o + n_out * n_hidden].reshape(n_out, n_hidden); o += n_out * n_hidden
    b2 = P[o:o + n_out]; o += n_out
    assert o == P.size, "parameter count does not match the shape"
    return W1, b1, W2, b2


def per_sample_loss(P, X, y, n_in=64, n_hidden=256, n_out=10):
    """Cross-entropy of each sample, fp64, max-shifted log-sum-exp."""
    W1, b1, W2, b2 = unflatten(P, n_in, n_hidden, n_out)
    X = np.asarray(X, np.float64)
    h = np.maximum(X @ W1.T + b1, 0.0)
    logits = h @ W2.T + b2
    m = logits.max(axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.exp(logits - m).sum(axis=1))
    return lse - logits[np.arange(len(y)), np.asarray(y)]


def loss(P, X, y, n_in=64, n_hidden=256, n_out=10):
    """Mean cross-entropy over the batch."""
    return float(per_sample_loss(P, X, y, n_in, n_hidden, n_out).mean())
