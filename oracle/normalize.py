"""Oracle of the q / k L2 normalisation the kernels can fuse, fp64 numpy.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU legs of ``bench.py`` may import this module; the product path never does.

The recurrence reads unit-norm queries and keys (the workloads draw q and k
and normalise them per (token, head) over the key width, without an
epsilon).  With the fused prologue the kernels receive the raw q, k and
normalise them themselves:

    q^ = q / ||q||,   k^ = k / ||k||                (per token, over DK)

and the reverse pass maps the gradients of q^, k^ back to the raw inputs:

    dq = (dq^ - q^ (q^ . dq^)) / ||q||   (the same for k).
"""
import numpy as np


def l2_normalise(x):
    """Rows of x [T, DK] divided by their Euclidean norms."""
    x = np.asarray(x, np.float64)
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def l2_normalise_grad(x, dy):
    """Gradient with respect to x of sum(dy * l2_normalise(x))."""
    x = np.asarray(x, np.float64)
    n = np.linalg.norm(x, axis=1, keepdims=True)
    y = x / n
    return (dy - y * np.sum(y * dy, axis=1, keepdims=True)) / n
