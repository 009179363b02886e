"""Oracle of the in-kernel decay activation, fp64 numpy.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU legs of ``bench.py`` may import this module; the product path never does.

The pages fuse the key-axis decay gate's activation into the chunk kernel so
that no full-sequence decay tensor is written (CARVE technical summary,
gist.science, section 2.3 "Key-Axis Decay und Fusion"; the same section of
the Dutch summary), but they do not print the activation.  The reading
taken here is the one the workloads' own log-decay is drawn with: from a raw
decay logit a and a positive scale s,

    g = -s * softplus(a) = -s * log(1 + exp(a))        (g < 0 for every a)

and, for the reverse pass, dL/da = dL/dg * dg/da with dg/da = -s * sigmoid(a).
The recurrence itself is unchanged: it receives g.
"""
import numpy as np


def softplus(a):
    a = np.asarray(a, np.float64)
    # log(1 + exp(a)) without overflow: max(a, 0) + log1p(exp(-|a|))
    return np.maximum(a, 0.0) + np.log1p(np.exp(-np.abs(a)))


def decay_from_logits(a, scale):
    """g = -scale * softplus(a)."""
    return -float(scale) * softplus(a)


def decay_grad(a, scale):
    """dg/da = -scale * sigmoid(a)."""
    a = np.asarray(a, np.float64)
    return -float(scale) / (1.0 + np.exp(-a))
