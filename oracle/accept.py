"""Greedy acceptance of a speculated token tree: the oracle.

TEST INFRASTRUCTURE ONLY (like the rest of this package): only the test
suite and the CPU-baseline leg of ``bench.py`` may import it.

LongSpec verifies its 4/16/16/16/16 draft tree against the target model and
is run and evaluated at temperature 0 (LongSpec README, "Inference": every
command passes ``--temperature 0``; the reported "acceptance length", LongSpec
README "Results").  At temperature 0 the target's token after a position is
the argmax of its logits there, so node i of the tree is accepted exactly
when every node on its root path carries the target's argmax token at that
node's parent position.  The emitted tokens are the deepest accepted chain
plus one token the target adds after it (its argmax at the chain's last
position).  Readings where the pages are silent (stated in the design notes):
the smallest node id wins among equally deep accepted nodes; argmax ties go
to the smallest token id; a NaN logit counts as -inf (so a row of NaNs and
-infs picks its first entry); a root-level node (parent -1) is judged at the
prefix-end position.

Plain numpy, one sequence at a time, in the order of the definition.
"""
from __future__ import annotations

import numpy as np


class BadParent(ValueError):
    pass


# Planted mistakes, used only by the pin-sensitivity test (None in all other
# use): "ties-last" (argmax ties to the largest token), "own-row" (a node is
# judged at the row after itself instead of its parent's), "shallowest"
# (the shallowest accepted node wins), "bonus-root" (the bonus always comes
# from the prefix-end row), "nan-wins" (NaN is not read as -inf).
MUTATION = None


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def argmax_rows(logits_bits: np.ndarray) -> np.ndarray:
    """First index of the largest value of every row (bf16 bits, [..., V]),
    NaN read as -inf."""
    x = bf16_to_f64(logits_bits)
    if MUTATION != "nan-wins":
        x = np.where(np.isnan(x), -np.inf, x)
    if MUTATION == "ties-last":
        return (x.shape[-1] - 1 - np.argmax(x[..., ::-1], axis=-1)).astype(np.int64)
    return np.argmax(x, axis=-1).astype(np.int64)


def accept_greedy(logits_bits: np.ndarray, draft_tokens: np.ndarray, parent: np.ndarray):
    """logits_bits: uint16 [B][T+1][V] (row 0: the prefix end, row 1+i: the
    position after node i); draft_tokens, parent: int [B][T].

    Returns (accept_len [B], path [B][T] with -1 past accept_len, bonus [B]).
    Raises BadParent unless every parent[b][i] is -1 or in [0, i).
    """
    B, T = draft_tokens.shape
    amax = argmax_rows(logits_bits)                  # [B][T+1]
    accept_len = np.zeros(B, dtype=np.int64)
    path = np.full((B, T), -1, dtype=np.int64)
    bonus = np.zeros(B, dtype=np.int64)
    for b in range(B):
        par = [int(x) for x in parent[b]]
        for i, p in enumerate(par):
            if not (p == -1 or 0 <= p < i):
                raise BadParent(f"parent[{b}][{i}] = {p}")
        accepted = [False] * T
        depth = [0] * T
        for i in range(T):                           # parents come first
            p = par[i]
            row = 0 if p == -1 else p + 1
            if MUTATION == "own-row":
                row = i + 1
            ok_parent = True if p == -1 else accepted[p]
            accepted[i] = ok_parent and int(draft_tokens[b][i]) == int(amax[b][row])
            depth[i] = 1 if p == -1 else depth[p] + 1
        best = -1
        for i in range(T):                           # deepest; the smallest id on ties
            if not accepted[i]:
                continue
            if best < 0:
                best = i
            elif MUTATION == "shallowest":
                if depth[i] < depth[best]:
                    best = i
            elif depth[i] > depth[best]:
                best = i
        if best < 0:
            bonus[b] = amax[b][0]
            continue
        chain = []
        j = best
        while j != -1:
            chain.append(j)
            j = par[j]
        chain.reverse()
        accept_len[b] = len(chain)
        path[b, :len(chain)] = chain
        bonus[b] = amax[b][0 if MUTATION == "bonus-root" else best + 1]
    return accept_len, path, bonus
