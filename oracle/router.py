"""Router with top-k selection: the step that produces the routing the
routed-expert path takes as input.

TEST INFRASTRUCTURE ONLY, like the rest of this package: a plain float64
restatement for the tests; the CUDA library never calls it.

Source ("MiMo-V2.6-Flash-RL GGUF for a single DGX Spark", "Architecture
notes"): 256 routed experts, 8 active per token, no shared expert, sigmoid
routing.  The pages say no more about the router; the readings taken here:
  - router weights Wr are [E][H] (one row of H weights per expert) and the
    logit of expert e for token t is z[t][e] = sum_h x[t][h] Wr[e][h];
  - the score is the logistic sigmoid s = 1 / (1 + exp(-z));
  - the k experts with the largest score are selected, in descending order;
    since the sigmoid is strictly increasing the order is taken on z, which
    keeps experts apart where their scores round to the same float64 value,
    and equal z go to the lower expert id first;
  - the routing weights are the selected scores divided by their sum.
The synthetic workloads of the expert path draw their routing weights as a
softmax over the k selected logits instead; ``score="softmax"`` gives that
reading (weights exp(z_i) / sum over the selected j of exp(z_j)), with the
same selection.
"""
from __future__ import annotations

import numpy as np

SCORES = ("sigmoid", "softmax")


def router_logits(x, Wr):
    """z [T][E] float64: every logit as an explicit float64 dot product."""
    x = np.asarray(x, dtype=np.float64)
    Wr = np.asarray(Wr, dtype=np.float64)
    T, H = x.shape
    E, H2 = Wr.shape
    assert H == H2
    z = np.empty((T, E), np.float64)
    for t in range(T):
        for e in range(E):
            z[t, e] = np.dot(x[t], Wr[e])
    return z


def topk_from_logits(z, k: int, score: str = "sigmoid"):
    """The selection and weighting steps alone, on given logits z [T][E]
    (any float type, compared as given): (ids int32 [T][k], w float64 [T][k]).
    Descending z, equal z by ascending expert id; weights as in the module
    docstring, computed in float64."""
    assert score in SCORES
    z = np.asarray(z)
    T, E = z.shape
    assert 1 <= k <= E
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-z[t, e], e))[:k]
        zs = np.array([float(z[t, e]) for e in order], np.float64)
        if score == "sigmoid":
            sel = 1.0 / (1.0 + np.exp(-zs))
        else:
            sel = np.exp(zs - zs[0])          # zs[0] is the largest selected logit
        ids[t] = order
        w[t] = sel / sel.sum()
    return ids, w


def router_topk(x, Wr, k: int, score: str = "sigmoid"):
    """(topk_ids int32 [T][k], topk_w float32 [T][k], scores float64 [T][E]);
    scores are the sigmoid of the logits for either weighting."""
    z = router_logits(x, Wr)
    s = 1.0 / (1.0 + np.exp(-z))
    ids, w = topk_from_logits(z, k, score)
    return ids, w.astype(np.float32), s
