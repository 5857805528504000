"""Commit of the accepted path into the KV cache: the oracle.

TEST INFRASTRUCTURE ONLY (like the rest of this package): only the test
suite and the CPU-baseline leg of ``bench.py`` may import it.

After verification and greedy acceptance, the accepted tokens join the
target model's context (LongSpec README, "Introduction": the target model
verifies the speculated tree and keeps what it accepts).  Their K/V rows,
computed by the verification pass as tree keys, are appended to the cache
right after the prefix, in path order, and the prefix grows by the accepted
length; rejected branches leave no trace.  Readings where the pages are
silent (stated in the design notes): a sequence whose accepted length or
path is out of range, or whose cache would overflow L_cap, is left as it
was and reported; cache rows past the new prefix end keep their contents.

Plain numpy, one row at a time, in the order of the definition.
"""
from __future__ import annotations

import numpy as np


# Planted mistakes, used only by the pin-sensitivity test (None in all other
# use): "skip-one" (rows written one position late), "reversed" (the path
# written leaf first), "no-advance" (prefix_len not advanced), "v-from-k"
# (the V cache gets the tree K rows).
MUTATION = None


class CommitError(ValueError):
    def __init__(self, b: int, kind: str):
        super().__init__(f"sequence {b}: {kind}")
        self.b = b
        self.kind = kind         # "path", "range" or "block"


def _check(b, L, n, path_b, T, L_cap):
    if not 0 <= n <= T:
        return "path"
    if not 0 <= L <= L_cap or L + n > L_cap:
        return "range"
    if any(not 0 <= int(path_b[d]) < T for d in range(n)):
        return "path"
    return None


def commit(k_cache, v_cache, prefix_len, k_tree, v_tree, accept_len, path):
    """Contiguous cache [B][Hkv][L_cap][D].  Returns (k, v, new_len, errors):
    new copies, and the list of CommitError for sequences left unchanged."""
    k, v = k_cache.copy(), v_cache.copy()
    new_len = np.array(prefix_len, dtype=np.int64).copy()
    B, Hkv, L_cap, _ = k.shape
    T = k_tree.shape[2]
    errors = []
    for b in range(B):
        L, n = int(prefix_len[b]), int(accept_len[b])
        bad = _check(b, L, n, path[b], T, L_cap)
        if bad:
            errors.append(CommitError(b, bad))
            continue
        for h in range(Hkv):
            for d in range(n):
                node = int(path[b][n - 1 - d if MUTATION == "reversed" else d])
                pos = L + d + (1 if MUTATION == "skip-one" and L + d + 1 < L_cap else 0)
                k[b, h, pos] = k_tree[b, h, node]
                v[b, h, pos] = (k_tree if MUTATION == "v-from-k" else v_tree)[b, h, node]
        new_len[b] = L if MUTATION == "no-advance" else L + n
    return k, v, new_len, errors


def commit_paged(k_cache, v_cache, block_table, prefix_len, k_tree, v_tree, accept_len, path, L_cap):
    """Paged cache [num_blocks][Hkv][block_size][D]: position p of sequence b
    is row p % block_size of block block_table[b][p // block_size]."""
    k, v = k_cache.copy(), v_cache.copy()
    new_len = np.array(prefix_len, dtype=np.int64).copy()
    num_blocks, Hkv, bs, _ = k.shape
    B, T = path.shape
    errors = []
    for b in range(B):
        L, n = int(prefix_len[b]), int(accept_len[b])
        bad = _check(b, L, n, path[b], T, L_cap)
        if not bad and any(not 0 <= int(block_table[b][(L + d) // bs]) < num_blocks for d in range(n)):
            bad = "block"
        if bad:
            errors.append(CommitError(b, bad))
            continue
        for h in range(Hkv):
            for d in range(n):
                pos = L + d + (1 if MUTATION == "skip-one" and L + d + 1 < L_cap else 0)
                blk = int(block_table[b][pos // bs])
                node = int(path[b][n - 1 - d if MUTATION == "reversed" else d])
                k[blk, h, pos % bs] = k_tree[b, h, node]
                v[blk, h, pos % bs] = (k_tree if MUTATION == "v-from-k" else v_tree)[b, h, node]
        new_len[b] = L if MUTATION == "no-advance" else L + n
    return k, v, new_len, errors
