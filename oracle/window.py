"""Sliding-window tree attention of the draft model: the oracle.

TEST INFRASTRUCTURE ONLY (like the rest of this package): only the test
suite and the CPU-baseline leg of ``bench.py`` may import it.

LongSpec's draft model is one transformer block whose self-attention is a
sliding window of 512 positions (LongSpec paper summary, "Summary": draft
model with sliding-window self-attention, window 512, and cross-attention
into the target's KV cache), so its own cache stays constant in size: a ring
of W slots that holds the last W positions.  Readings where the pages are
silent (stated in the design notes):

- a query at position p sees the W positions p - W + 1 .. p, itself
  included (the usual sliding window);
- while drafting a tree, a node at depth d (1 for the nodes whose parent is
  -1) sits at position L + d - 1 after an L-token context, and its window
  holds its ancestors-or-self (d tree keys) and the last W - d context
  positions, L + d - W .. L - 1 (clipped at 0);
- the ring stores context position p at slot p mod W, so it holds exactly
  positions max(0, L - W) .. L - 1;
- W > T, so a node's whole root path is inside its window.

Plain numpy in fp64, one (b, h, t) row at a time, keys listed one by one.
"""
from __future__ import annotations

import numpy as np


# Planted mistakes, used only by the pin-sensitivity test (None in all other
# use): "window+1" (one context key too many), "no-ring" (position p read at
# slot p, not p mod W), "no-self" (a node does not see itself), "depth-0"
# (depths counted from 0).
MUTATION = None


def _f64(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def depths(parent_b) -> list:
    """1-based depth of every node of one tree (parent[i] in [-1, i))."""
    d = []
    for i, p in enumerate(int(x) for x in parent_b):
        if not (p == -1 or 0 <= p < i):
            raise ValueError(f"parent[{i}] = {p}")
        d.append(1 if p == -1 else d[p] + 1)
    if MUTATION == "depth-0":
        d = [x - 1 for x in d]
    return d


def ancestors_or_self(parent_b, t: int) -> list:
    out = []
    j = t
    while j != -1:
        out.append(j)
        j = int(parent_b[j])
    if MUTATION == "no-self":
        out.remove(t)
    return sorted(out)


def window_attention(q, k_ring, v_ring, prefix_len, k_tree, v_tree, parent, W: int,
                     scale: float = 0.0, rows=None):
    """q [B][Hq][T][D], k/v_ring [B][Hkv][W][D], k/v_tree [B][Hkv][T][D]
    (bf16 bits as uint16), prefix_len [B] (total context length L_b, may
    exceed W), parent [B][T].  Returns (out, lse) in fp64, shapes
    [B][Hq][T][D] and [B][Hq][T], or [n][D] and [n] for rows = (b, h, t)
    triples.  A row with no visible key would have lse -inf; with W > T
    every row sees at least itself."""
    qf, krf, vrf = _f64(q), _f64(k_ring), _f64(v_ring)
    ktf, vtf = _f64(k_tree), _f64(v_tree)
    B, Hq, T, D = qf.shape
    Hkv = krf.shape[1]
    if krf.shape[2] != W or W <= T:
        raise ValueError("the ring must have W > T slots")
    G = Hq // Hkv
    s = scale if scale > 0 else 1.0 / np.sqrt(D)
    sel = [(b, h, t) for b in range(B) for h in range(Hq) for t in range(T)] if rows is None \
        else [tuple(int(x) for x in r) for r in rows]
    out = np.zeros((len(sel), D))
    lse = np.zeros(len(sel))
    dep = [depths(parent[b]) for b in range(B)]
    for n, (b, h, t) in enumerate(sel):
        kvh = h // G
        L = int(prefix_len[b])
        d = dep[b][t]
        keys, vals = [], []
        first = L + d - W - (1 if MUTATION == "window+1" else 0)
        for p in range(max(0, first), L):                  # context positions in the window
            slot = min(p, W - 1) if MUTATION == "no-ring" else p % W
            keys.append(krf[b, kvh, slot])
            vals.append(vrf[b, kvh, slot])
        for j in ancestors_or_self(parent[b], t):          # the root path, itself included
            keys.append(ktf[b, kvh, j])
            vals.append(vtf[b, kvh, j])
        x = np.array([s * float(np.dot(qf[b, h, t], k)) for k in keys])
        m = x.max()
        e = np.exp(x - m)
        out[n] = (e[:, None] * np.array(vals)).sum(0) / e.sum()
        lse[n] = m + np.log(e.sum())
    if rows is None:
        return out.reshape(B, Hq, T, D), lse.reshape(B, Hq, T)
    return out, lse
