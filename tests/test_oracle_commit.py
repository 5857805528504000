"""The KV-commit oracle, pinned to things other than itself (CPU).

- The committed context is what the accepted node attended to: for the node
  at depth d of the accepted path, verification attention (prefix + its
  ancestors-or-self under the tree mask) equals plain prefix-only attention
  over the committed cache cut at L_b + d (an independent route through the
  attention oracle, 1e-12).
- A chain fully accepted appends the tree rows in order: numpy
  concatenation of prefix and tree rows.
- The paged commit, gathered back through the block table, equals the
  contiguous commit; rows outside [L_b, L_b + n_b) are untouched.
- Out-of-range lengths, paths and block ids leave the sequence unchanged.
"""
import numpy as np
import pytest

import oracle
from oracle import commit as C
from tree_masked_verification_b200.inputs import Workload, bf16_bits, commit_inputs, paged_cache

W = Workload("commit", B=3, Hq=4, Hkv=2, D=64, T=12, L_cap=48, seed=31, tree="random",
             prefix_range=(0, 36))


def _np(inp):
    return {k: (bf16_bits(v) if v.dtype.is_floating_point else v.numpy()) for k, v in inp.items()}


def _commit(x):
    return C.commit(x["k_prefix"], x["v_prefix"], x["prefix_len"], x["k_tree"], x["v_tree"],
                    x["accept_len"], x["path"])


@pytest.mark.parametrize("seed", range(4))
def test_committed_context_is_what_the_accepted_node_attended_to(seed):
    x = _np(commit_inputs(W.replace(seed=40 + seed), seed))
    k, v, new_len, errors = _commit(x)
    assert not errors
    np.testing.assert_array_equal(new_len, x["prefix_len"] + x["accept_len"])
    verify = oracle.Problem(x["q"], x["k_prefix"], x["v_prefix"], x["prefix_len"], x["k_tree"],
                            x["v_tree"], x["parent"])
    for b in range(W.B):
        for d in range(1, int(x["accept_len"][b]) + 1):
            node = int(x["path"][b, d - 1])
            rows = np.array([[b, h, node] for h in range(W.Hq)], dtype=np.int32)
            o_ref, l_ref = verify.attention(rows)
            lens = x["prefix_len"].copy()
            lens[b] += d
            after = oracle.Problem(x["q"], k, v, lens, x["k_tree"], x["v_tree"], x["parent"])
            o, l = after.prefix_partial(0, W.L_cap, rows)
            np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
            np.testing.assert_allclose(l, l_ref, rtol=0, atol=1e-12)


def test_chain_fully_accepted_appends_in_order():
    w = W.replace(tree="chain", T=5, seed=50)
    x = _np(w.generate())
    x["accept_len"] = np.full(w.B, 5, dtype=np.int32)
    x["path"] = np.tile(np.arange(5, dtype=np.int32), (w.B, 1))
    k, v, new_len, _ = _commit(x)
    for b in range(w.B):
        L = int(x["prefix_len"][b])
        want_k = np.concatenate([x["k_prefix"][b, :, :L], x["k_tree"][b]], axis=1)
        want_v = np.concatenate([x["v_prefix"][b, :, :L], x["v_tree"][b]], axis=1)
        np.testing.assert_array_equal(k[b, :, :L + 5], want_k)
        np.testing.assert_array_equal(v[b, :, :L + 5], want_v)
        np.testing.assert_array_equal(k[b, :, L + 5:], x["k_prefix"][b, :, L + 5:])
        assert new_len[b] == L + 5


@pytest.mark.parametrize("bs", [16, 32])
def test_paged_commit_equals_contiguous(bs):
    inp = commit_inputs(W.replace(seed=60), 7)
    x = _np(inp)
    kc, vc, table = paged_cache(inp["k_prefix"], inp["v_prefix"], inp["prefix_len"].tolist(), bs, 9,
                                reserve=W.T)
    kc, vc, table = bf16_bits(kc), bf16_bits(vc), table.numpy()
    k, v, new_len, errors = _commit(x)
    kp, vp, new_len_p, errors_p = C.commit_paged(kc, vc, table, x["prefix_len"], x["k_tree"],
                                                 x["v_tree"], x["accept_len"], x["path"], W.L_cap)
    assert not errors and not errors_p
    np.testing.assert_array_equal(new_len, new_len_p)
    for b in range(W.B):
        for pos in range(int(new_len[b])):      # gather back through the table
            blk = table[b, pos // bs]
            np.testing.assert_array_equal(kp[blk, :, pos % bs], k[b, :, pos])
            np.testing.assert_array_equal(vp[blk, :, pos % bs], v[b, :, pos])
    untouched = np.ones(kc.shape[:3], dtype=bool)
    for b in range(W.B):
        for pos in range(int(x["prefix_len"][b]), int(new_len[b])):
            untouched[table[b, pos // bs], :, pos % bs] = False
    np.testing.assert_array_equal(kp[untouched], kc[untouched])


def test_bad_inputs_leave_the_sequence_unchanged():
    x = _np(commit_inputs(W.replace(seed=70), 3))
    x["prefix_len"] = np.array([10, 47, 5], dtype=np.int32)
    x["accept_len"] = np.array([13, 2, 2], dtype=np.int32)      # n > T; L + n > L_cap
    x["path"][2, :2] = [0, 12]                                  # node id 12 = T
    k, v, new_len, errors = _commit(x)
    assert [(e.b, e.kind) for e in errors] == [(0, "path"), (1, "range"), (2, "path")]
    np.testing.assert_array_equal(k, x["k_prefix"])
    np.testing.assert_array_equal(new_len, x["prefix_len"])
