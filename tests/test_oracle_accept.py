"""The greedy-acceptance oracle, pinned to things other than itself (CPU).

- A chain tree is ordinary greedy speculative decoding: the accepted length
  is the number of leading draft tokens that equal the target's next token,
  counted by a plain loop.
- Brute force: every root path is checked against the definition with a
  hand-written first-maximum scan; the deepest accepted path (smallest id on
  ties) must be the oracle's.
- Argmax ties go to the smallest token id; no match gives length 0 and the
  bonus token of the prefix end; a bad parent array is rejected.
"""
import itertools

import numpy as np
import pytest

from oracle import accept as A
from tree_masked_verification_b200.inputs import accept_inputs, bf16_bits


def _first_max(row):
    best, idx = None, -1
    for i, v in enumerate(row):
        if best is None or v > best:
            best, idx = v, i
    return idx


def _inputs(B, T, V, seed, tree, p):
    d = accept_inputs(B, T, V, seed, tree=tree, p_match=p)
    return bf16_bits(d["logits"]), d["draft_tokens"].numpy(), d["parent"].numpy()


@pytest.mark.parametrize("seed", range(6))
def test_chain_tree_is_sequential_greedy_decoding(seed):
    T, V = 7, 40
    bits, tok, par = _inputs(1, T, V, seed, "chain", 0.7)
    vals = A.bf16_to_f64(bits)[0]
    n = 0
    for i in range(T):                 # token i must be the target's choice after position i
        if tok[0, i] != _first_max(list(vals[i])):
            break
        n += 1
    length, path, bonus = A.accept_greedy(bits, tok, par)
    assert length[0] == n
    assert list(path[0, :n]) == list(range(n)) and (path[0, n:] == -1).all()
    assert bonus[0] == _first_max(list(vals[n]))


@pytest.mark.parametrize("seed", range(8))
def test_brute_force_over_root_paths(seed):
    B, T, V = 2, 8, 6
    bits, tok, par = _inputs(B, T, V, 100 + seed, "random", 0.75)
    vals = A.bf16_to_f64(bits)
    length, path, bonus = A.accept_greedy(bits, tok, par)
    for b in range(B):
        best = []
        for i in range(T):
            chain = [i]
            while par[b, chain[-1]] != -1:
                chain.append(int(par[b, chain[-1]]))
            chain.reverse()
            ok = all(tok[b, j] == _first_max(list(vals[b, 0 if k == 0 else chain[k - 1] + 1]))
                     for k, j in enumerate(chain))
            if ok and (len(chain) > len(best) or (len(chain) == len(best) and chain[-1] < best[-1])):
                best = chain
        assert length[b] == len(best)
        assert list(path[b, :len(best)]) == best
        last_row = 0 if not best else best[-1] + 1
        assert bonus[b] == _first_max(list(vals[b, last_row]))


def test_argmax_ties_go_to_the_smallest_token():
    vals = np.zeros((1, 2, 5), dtype=np.float32)
    vals[0, 0, [1, 3]] = 2.0           # a tie at the prefix end
    vals[0, 1, [0, 4]] = 1.0           # and after node 0
    bits = (vals.view(np.uint32) >> 16).astype(np.uint16)
    length, path, bonus = A.accept_greedy(bits, np.array([[1]]), np.array([[-1]]))
    assert length[0] == 1 and path[0, 0] == 0 and bonus[0] == 0
    length, _, bonus = A.accept_greedy(bits, np.array([[3]]), np.array([[-1]]))
    assert length[0] == 0 and bonus[0] == 1


def test_no_match_and_all_match():
    d = accept_inputs(1, 68, 500, 7, p_match=1.0)
    bits = bf16_bits(d["logits"])
    par = d["parent"].numpy()
    length, path, _ = A.accept_greedy(bits, d["draft_tokens"].numpy(), par)
    assert length[0] == 5              # every node matches: the tree's depth
    wrong = (d["draft_tokens"].numpy() + 1) % 500
    length, path, bonus = A.accept_greedy(bits, wrong, par)
    assert length[0] == 0 and (path == -1).all() and bonus[0] == d["planted"][0, 0]


def test_bad_parent_is_rejected():
    for par in ([[-1, 1]], [[-1, 2, 0]], [[0]]):
        p = np.array(par)
        with pytest.raises(A.BadParent):
            A.accept_greedy(np.zeros((1, p.shape[1] + 1, 3), np.uint16), np.zeros_like(p), p)


def test_every_shape_of_a_small_tree():
    """All parent arrays of 4 nodes, every draft choice in {match, no match}
    per node: the oracle against the brute-force reading."""
    V = 3
    rng = np.random.default_rng(5)
    for par in itertools.product(*[range(-1, i) for i in range(4)]):
        par = np.array([par])
        vals = rng.standard_normal((1, 5, V)).astype(np.float32)
        bits = (vals.view(np.uint32) >> 16).astype(np.uint16)
        f = A.bf16_to_f64(bits)[0]
        for mask in range(16):
            tok = np.array([[(_first_max(list(f[0 if par[0, i] == -1 else par[0, i] + 1])) +
                              (0 if mask >> i & 1 else 1)) % V for i in range(4)]])
            length, _, _ = A.accept_greedy(bits, tok, par)
            best = 0
            for i in range(4):
                chain, j = [], i
                while j != -1:
                    chain.append(j)
                    j = par[0, j]
                if all(mask >> j & 1 for j in chain):
                    best = max(best, len(chain))
            assert length[0] == best


def test_nan_counts_as_minus_inf():
    """NaN logits: the first maximum of the row with every NaN read as -inf;
    a row of NaNs and -infs picks its first entry (token 0)."""
    nan, inf = np.float32(np.nan), np.float32(np.inf)
    vals = np.array([[[nan, 1.0, 3.0, nan], [nan, -inf, nan, -inf], [nan, nan, nan, nan]]],
                    dtype=np.float32)
    bits = (vals.view(np.uint32) >> 16).astype(np.uint16)
    assert list(A.argmax_rows(bits)[0]) == [2, 0, 0]
    length, path, bonus = A.accept_greedy(bits, np.array([[2, 0]]), np.array([[-1, 0]]))
    assert length[0] == 2 and list(path[0]) == [0, 1] and bonus[0] == 0
