"""Second-direction restatements used only to pin the plain definition.

TEST INFRASTRUCTURE ONLY (see the package docstring).

* ``online_softmax_attend``: the running-max / running-sum method of
  "大模型面试笔记" section 2 ("在线安全softmax": per block, take the block
  maximum, update the global maximum m, multiply the accumulated denominator l
  by a compensation factor and add the new block's exponentials) and of the P1
  lesson, "步骤2" / "Numerical trick" (the accumulated output is rescaled with
  the same factor and divided by l once at the end).  Written here as plain
  Python loops over tiles of keys, for small inputs only.
* ``split_partials`` / ``combine_partials``: the split-KV scheme of
  "[BEE-30062]" section "背景" (Flash-Decoding splits keys and values into
  chunks processed in parallel and reduces the partial softmax results in a
  numerically stable way).  The pages do not print the reduction; the reading
  used is the max-shift algebra of the online softmax applied to whole chunks:
  with per-chunk normalised outputs O_c and log-sum-exps lse_c,
  lse = M + ln(sum_c exp(lse_c - M)) with M = max_c lse_c and
  O = sum_c exp(lse_c - lse) O_c; a chunk with no visible key has
  lse_c = -inf and weight 0.
"""

from __future__ import annotations

import math

import numpy as np

from .attention import visible_mask


def online_softmax_attend(q, keys, values, scale: float, tile: int,
                          visible=None) -> tuple[list[float], float]:
    """One query vector against ``keys``/``values`` (lists of vectors), visiting
    keys ``tile`` at a time with a running maximum and running denominator.

    Returns ``(o, lse)``.  ``visible`` optionally lists which keys count.
    """
    n = len(keys)
    dv = len(values[0])
    run_max = -math.inf
    run_den = 0.0
    acc = [0.0] * dv
    for lo in range(0, n, tile):
        idx = [j for j in range(lo, min(lo + tile, n)) if visible is None or visible[j]]
        if not idx:
            continue
        scores = {j: scale * sum(a * b for a, b in zip(q, keys[j])) for j in idx}
        block_max = max(scores.values())
        new_max = max(run_max, block_max)
        # compensation factor for what was accumulated under the old maximum
        corr = 0.0 if run_max == -math.inf else math.exp(run_max - new_max)
        run_den *= corr
        for c in range(dv):
            acc[c] *= corr
        for j in idx:
            p = math.exp(scores[j] - new_max)
            run_den += p
            for c in range(dv):
                acc[c] += p * values[j][c]
        run_max = new_max
    if run_den == 0.0:
        raise ValueError("no visible key")
    return [a / run_den for a in acc], run_max + math.log(run_den)


def split_partials(q, k, v, scale: float, causal: bool, chunk: int):
    """Per-chunk normalised outputs and log-sum-exps for one head.

    ``q [Nq, d]``, ``k, v [Lk, d]``; the keys are cut into consecutive chunks
    of ``chunk`` positions and each chunk is attended to independently with the
    global visibility mask restricted to it.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    Nq, Lk = q.shape[0], k.shape[0]
    vis = visible_mask(Nq, Lk, causal)
    outs, lses = [], []
    for c0 in range(0, Lk, chunk):
        c1 = min(c0 + chunk, Lk)
        o_c = np.zeros((Nq, v.shape[1]))
        lse_c = np.full(Nq, -np.inf)
        for t in range(Nq):
            cols = np.nonzero(vis[t, c0:c1])[0] + c0
            if cols.size == 0:
                continue
            s = scale * (k[cols] @ q[t])
            m = s.max()
            w = np.exp(s - m)
            o_c[t] = (w @ v[cols]) / w.sum()
            lse_c[t] = m + np.log(w.sum())
        outs.append(o_c)
        lses.append(lse_c)
    return np.stack(outs), np.stack(lses)          # [C, Nq, d], [C, Nq]


def combine_partials(outs: np.ndarray, lses: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Merge chunk partials ``outs [C, Nq, d]``, ``lses [C, Nq]`` into the full result."""
    M = lses.max(axis=0)                                        # [Nq]
    if not np.isfinite(M).all():
        raise ValueError("a query row has no visible key")
    z = np.exp(lses - M[None, :]).sum(axis=0)                   # exp(-inf) = 0
    lse = M + np.log(z)
    w = np.exp(lses - lse[None, :])                             # [C, Nq]
    return (w[:, :, None] * outs).sum(axis=0), lse
