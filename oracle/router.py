"""Router of the MoE layer (float64, numpy).  Test infrastructure only.

The pages show the routing weights only where the per-expert loop consumes
them ("Efficient MoE Training for Biological Foundation Models", Challenge 1:
each expert's output is scaled by routing_weights[token, slot] before the
index_add back to token order); they do not print the router.  Reading taken,
the plainest one consistent with the Mixtral model the pages benchmark:

* probabilities = softmax of the token's E router logits;
* the k experts with the largest probabilities are kept, in descending
  order, ties going to the lower expert id;
* the kept probabilities are renormalised to sum to one.

Because the renormalisation divides out the softmax denominator, the kept
probabilities equal a softmax over the k kept logits, and the selection only
compares logits (softmax is strictly increasing).  A NaN logit ranks below
every number (as -inf).  A row whose kept logits include +inf, or are all
-inf, has no defined probabilities (NaN).  This module follows the definition
step by step (softmax first); the tests pin it against the reduced forms.
"""
from __future__ import annotations

import numpy as np


def route_topk(logits: np.ndarray, k: int):
    """logits [T, E] -> (topk_idx int32 [T, k], topk_prob float64 [T, k])."""
    lg = np.asarray(logits, dtype=np.float64)
    T, E = lg.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    key = np.where(np.isnan(lg), -np.inf, lg)
    # softmax over all experts, shifted by the row maximum
    with np.errstate(invalid="ignore"):
        m = key.max(axis=1, keepdims=True)
        p = np.exp(key - m)
        p = p / p.sum(axis=1, keepdims=True)
    # k largest, descending, ties to the lower id: a stable sort of -key
    # (ranking the logits ranks the probabilities, and keeps ties exact)
    order = np.argsort(-key, axis=1, kind="stable")[:, :k]
    top = np.take_along_axis(p, order, axis=1)
    with np.errstate(invalid="ignore"):
        top = top / top.sum(axis=1, keepdims=True)
    return order.astype(np.int32), top
