"""Load-balance controls of DeepSeek-V3-style routing — TEST INFRASTRUCTURE ONLY.

Nothing in the library imports this module (see oracle/__init__.py).  Two
rows of the layer's "next" list, written from the pages:

1. Selection-bias update ([STA324] §8.6: selection uses s_e + b_e, an
   overloaded expert's bias goes down and an underloaded one's goes up,
   under a load-control rule; the gate weights stay on the raw affinities;
   [TRAIN] "代表性路线": DeepSeek-V3 controls load mainly with dynamic
   expert biases).  Reading: the pages give only the direction of the
   rule, so the plainest rule with that direction is used,
       b_e <- b_e - gamma * sign(n_e - mean_e n_e),
   with n_e the batch's pre-drop valid slot counts (the same load the aux
   loss's f uses) and the step gamma a parameter (unpinned).

2. Sequence-wise auxiliary loss ([STA324] §8.6 and [TRAIN]: DeepSeek-V3
   keeps a small complementary sequence-wise auxiliary term; neither page
   writes it out).  Reading: the §8.5 Switch loss evaluated on each
   sequence of seq_len consecutive tokens and averaged over sequences,
       L = alpha * E * mean_s sum_e f_{s,e} P_{s,e},
       f_{s,e} = n_{s,e} / sum_e n_{s,e}   (valid slots of sequence s),
       P_{s,e} = mean_{t in s} q_{t,e},
   with q = p for softmax scores and, for sigmoid affinities, q = sigma /
   sum_e sigma (the pages define P as the mean soft probability; dividing
   the affinities by their sum is the plainest way to make them one).
   f is held constant for the gradient ([STA324] §8.5), so
       dL/dq_{t,e} = alpha * E * f_{s(t),e} / (seq_len * n_seq),
   and for sigmoid scores, with S_t = sum_e sigma_{t,e},
       dL/dsigma_{t,j} = (dq_j - sum_i dq_i q_i) / S_t,
       dL/ds_{t,j} = dL/dsigma_{t,j} * sigma_j (1 - sigma_j).
   With one sequence covering the batch it equals the batch loss.
"""
from __future__ import annotations

import numpy as np

SOFTMAX, SIGMOID = 0, 1


def bias_update(counts, bias, gamma):
    """b_e - gamma * sign(n_e - mean(n)) (float64)."""
    n = np.asarray(counts, dtype=np.float64)
    b = np.asarray(bias, dtype=np.float64)
    return b - gamma * np.sign(n - n.mean())


def normalized_scores(p, score_fn):
    """q: softmax probabilities as they are, sigmoid affinities / their sum."""
    p = np.asarray(p, dtype=np.float64)
    if score_fn == SOFTMAX:
        return p
    return p / p.sum(axis=1, keepdims=True)


def seq_counts(expert, T, K, E, seq_len):
    """n_{s,e}: valid (non-sentinel) slots of each sequence per expert.

    expert: [T*K] expert of each slot, -1 for sentinel slots (pre-drop)."""
    ex = np.asarray(expert).reshape(T, K)
    n_seq = T // seq_len
    n = np.zeros((n_seq, E))
    for s in range(n_seq):
        blk = ex[s * seq_len:(s + 1) * seq_len].reshape(-1)
        blk = blk[blk >= 0]
        n[s] = np.bincount(blk, minlength=E)[:E]
    return n


def seq_aux_loss(p, expert, K, alpha, seq_len, score_fn=SOFTMAX):
    """(L, f [n_seq,E], P [n_seq,E]) of the sequence-wise aux loss."""
    p = np.asarray(p, dtype=np.float64)
    T, E = p.shape
    if seq_len <= 0 or T % seq_len:
        raise ValueError("seq_len must divide T")
    n_seq = T // seq_len
    n = seq_counts(expert, T, K, E, seq_len)
    tot = n.sum(axis=1, keepdims=True)
    f = np.divide(n, tot, out=np.zeros_like(n), where=tot > 0)
    q = normalized_scores(p, score_fn)
    P = q.reshape(n_seq, seq_len, E).mean(axis=1)
    return float(alpha * E * np.mean((f * P).sum(axis=1))), f, P


def seq_aux_grad_scores(p, f, alpha, seq_len, score_fn=SOFTMAX):
    """dL/dp (softmax: w.r.t. the probabilities, to go through the softmax
    backward) or dL/ds (sigmoid: w.r.t. the logits), [T, E]."""
    p = np.asarray(p, dtype=np.float64)
    T, E = p.shape
    n_seq = T // seq_len
    dq = alpha * E * np.repeat(f, seq_len, axis=0) / (seq_len * n_seq)
    if score_fn == SOFTMAX:
        return dq
    S = p.sum(axis=1, keepdims=True)
    q = p / S
    dsig = (dq - (dq * q).sum(axis=1, keepdims=True)) / S
    return dsig * p * (1.0 - p)
