"""TEST INFRASTRUCTURE ONLY: independent fp64 checkers for the C oracle, for tiny inputs.

These restate the RSM mixer in closed forms that do not run the token-by-token recurrence:

* ``quadratic_form``: the unrolled sum, with every product of decays written out,
      o_t = sum_{s<=t} sum_i q_{t,i} k_{s,i} (1 - a_{s,i}) prod_{u=s+1..t} a_{u,i} v_s
            + sum_i q_{t,i} (prod_{u<=t} a_{u,i}) H0[i,:]
  where a_{u,i} = exp(sigmoid(l_{u,i}) f_u) on the selected slots and exactly 1 elsewhere
  (Raven README, "How Raven Works": gated write H = H*decay + (1-decay) k (x) v, read o = q.H;
  the H0 term is the same unrolling applied to a non-zero initial state).
* ``dense_masked_form``: the TopK = M limit, where every slot is written every step and the layer
  is a gated linear-attention recurrence with per-slot gate (paperlayer.ai summary, sections
  3.4 "State-Space Models as RSMs" and A.5 "Efficient Training using Gated Linear Attention");
  computed as a masked matrix product with cumulative log-gates.
* ``router_scores`` / ``selection_counts``: the router variants' scores (sigmoid or softmax over the
  row, optionally normalised over the TopK set) and the per-slot selection counts, from library
  routines (scipy's expit and softmax, numpy sums and bincount).
* ``window_form``: the one-hot cyclic router with full overwrite, which turns the slot store into
  a window of the last M tokens ("Raven Part 1 -- Memory as a Set of Slots", "Key claims": a
  one-hot cyclic router recovers sliding-window attention; paperlayer.ai summary section 2.2).

Routing here uses numpy's stable argsort (a library sort), not the oracle's insertion sort.
"""
from __future__ import annotations

import numpy as np


def topk_stable(logits: np.ndarray, K: int) -> np.ndarray:
    """TopK slots per row by (logit desc, index asc), via a stable library sort of -logit."""
    x = np.asarray(logits, dtype=np.float32).astype(np.float64)
    order = np.argsort(-x, axis=-1, kind="stable")
    return order[..., :K].astype(np.int32)


def router_scores(logits, K: int, router: str = "sigmoid"):
    """Scores of every slot under a router variant, zero off the TopK set, with library routines:
    scipy's expit (sigmoid) or softmax over the row's M slots, then, for the normalised variants,
    division by the sum over the selected slots. Returns (selected mask, scores) [T,M]."""
    from scipy.special import expit, softmax
    lg = np.asarray(logits, dtype=np.float32).astype(np.float64)
    sel = np.zeros(lg.shape, dtype=bool)
    np.put_along_axis(sel, topk_stable(lg, K), True, axis=-1)
    s = softmax(lg, axis=-1) if router.startswith("softmax") else expit(lg)
    s = np.where(sel, s, 0.0)
    if router.endswith("_norm"):
        s = s / s.sum(axis=-1, keepdims=True)
    return sel, s


def gates(logits, f, K: int, router: str = "sigmoid"):
    """Per-(token, slot) decay a (1 off the selected set) and write weight (1-a) (0 off it).

    logits: [T,M] fp32; f: [T] or [T,M]. Returns (a, one_minus_a) as float64 [T,M].
    """
    lg = np.asarray(logits, dtype=np.float32).astype(np.float64)
    T, M = lg.shape
    fx = np.asarray(f, dtype=np.float32).astype(np.float64)
    if fx.ndim == 1:
        fx = np.repeat(fx[:, None], M, axis=1)
    sel, s = router_scores(lg, K, router)
    a = np.where(sel, np.exp(s * fx), 1.0)
    one_minus_a = np.where(sel, 1.0 - np.exp(s * fx), 0.0)
    return a, one_minus_a


def quadratic_form(q, k, v, logits, f, K: int, H0=None, router: str = "sigmoid"):
    """Unrolled closed form for one (b,h) stream. q,k,logits [T,M]; v [T,Dv]; f [T] or [T,M].

    Returns (o [T,Dv], HT [M,Dv]) in float64. O(T^2 M Dv): tiny inputs only.
    """
    q = np.asarray(q, np.float32).astype(np.float64)
    k = np.asarray(k, np.float32).astype(np.float64)
    v = np.asarray(v, np.float32).astype(np.float64)
    T, M = q.shape
    Dv = v.shape[1]
    a, oma = gates(logits, f, K, router)
    h0 = np.zeros((M, Dv)) if H0 is None else np.asarray(H0, np.float64)
    o = np.zeros((T, Dv))
    for t in range(T):
        for s in range(t + 1):
            for i in range(M):
                prod = 1.0
                for u in range(s + 1, t + 1):
                    prod *= a[u, i]
                o[t] += q[t, i] * k[s, i] * oma[s, i] * prod * v[s]
        for i in range(M):
            prod = 1.0
            for u in range(0, t + 1):
                prod *= a[u, i]
            o[t] += q[t, i] * prod * h0[i]
    HT = np.zeros((M, Dv))
    for i in range(M):
        prod_all = 1.0
        for u in range(T):
            prod_all *= a[u, i]
        HT[i] = prod_all * h0[i]
        for s in range(T):
            prod = 1.0
            for u in range(s + 1, T):
                prod *= a[u, i]
            HT[i] += k[s, i] * oma[s, i] * prod * v[s]
    return o, HT


def dense_masked_form(q, k, v, logits, f, H0=None):
    """TopK = M limit as O = ((Q*e^G) (W*e^-G)^T * causal) V + (Q*e^G) H0, G = cumsum(log a).

    Valid only while e^-G stays finite (short sequences, mild decays).
    """
    q = np.asarray(q, np.float32).astype(np.float64)
    k = np.asarray(k, np.float32).astype(np.float64)
    v = np.asarray(v, np.float32).astype(np.float64)
    T, M = q.shape
    lg = np.asarray(logits, np.float32).astype(np.float64)
    fx = np.asarray(f, np.float32).astype(np.float64)
    if fx.ndim == 1:
        fx = np.repeat(fx[:, None], M, axis=1)
    s = 1.0 / (1.0 + np.exp(-lg))
    loga = s * fx                      # every slot selected: log-gate is s*f everywhere
    G = np.cumsum(loga, axis=0)        # inclusive cumulative log-gate
    W = k * (1.0 - np.exp(loga))
    A = (q * np.exp(G)) @ (W * np.exp(-G)).T
    A = np.tril(A)                     # s <= t, read after write
    o = A @ v
    if H0 is not None:
        o += (q * np.exp(G)) @ np.asarray(H0, np.float64)
    HT = (np.exp(G[-1])[:, None] * (np.zeros((M, v.shape[1])) if H0 is None else np.asarray(H0, np.float64))
          + (W * np.exp(G[-1][None, :] - G)).T @ v)
    return o, HT


def selection_counts(logits, K: int):
    """Tokens that select each slot: a bincount of the stable library sort's TopK. logits [T,M]."""
    lg = np.asarray(logits, dtype=np.float32)
    return np.bincount(topk_stable(lg, K).ravel(), minlength=lg.shape[-1]).astype(np.int32)


def window_form(q, v, M: int):
    """One-hot cyclic router with full overwrite: o_t = sum_{s=t-M+1..t, s>=0} q_{t, s mod M} v_s."""
    q = np.asarray(q, np.float32).astype(np.float64)
    v = np.asarray(v, np.float32).astype(np.float64)
    T = q.shape[0]
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        for s in range(max(0, t - M + 1), t + 1):
            o[t] += q[t, s % M] * v[s]
    HT = np.zeros((M, v.shape[1]))
    for s in range(T):
        HT[s % M] = v[s]
    return o, HT
