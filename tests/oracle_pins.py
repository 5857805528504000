"""Pins of the fp64 oracle against things other than itself.

Each ``pin_*`` function raises AssertionError (or OracleError) when the oracle
disagrees with what the mathematics or the pages fix.  They are run as tests
in ``test_oracle_pins.py`` and, with a planted mistake in the oracle, in
``test_oracle_pin_sensitivity.py`` to show that every planted mistake is
caught by at least one pin.

Independent constructions used here (none retypes the oracle's code):
  * tree ancestry by transitive closure of the parent adjacency matrix,
    computed by repeated Boolean matrix squaring (numpy);
  * softmax attention evaluated directly as sum e^x v / sum e^x with no max
    subtraction, at 60 significant digits (mpmath);
  * causal decoding attention with the mask taken from index comparison
    (numpy fp64), for chain-shaped trees and T = 1;
  * closed forms: q = 0, constant V, a single visible key, a hand-worked
    two-node example.
"""
from __future__ import annotations

import itertools
import math

import mpmath
import numpy as np
import torch

import oracle
from tree_masked_verification_b200.inputs import (Workload, bf16_bits,
                                                  tree_chain)


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def closure_ancestry(parent) -> np.ndarray:
    """R[i][j] = 1 iff j is i or an ancestor of i: reflexive-transitive
    closure of the child->parent edge relation by Boolean squaring."""
    parent = np.asarray(parent)
    T = parent.shape[0]
    R = np.eye(T, dtype=bool)
    for i, p in enumerate(parent):
        if p >= 0:
            R[i, p] = True
    while True:
        R2 = R | ((R.astype(np.int64) @ R.astype(np.int64)) > 0)
        if (R2 == R).all():
            return R
        R = R2


def bits_to_bool(bits: np.ndarray, T: int) -> np.ndarray:
    out = np.zeros((T, T), dtype=bool)
    for i in range(T):
        for j in range(T):
            out[i, j] = (int(bits[i, j // 32]) >> (j % 32)) & 1
    return out


def all_parent_arrays(T: int):
    return itertools.product(*[range(-1, i) for i in range(T)])


def problem_from(inp: dict, scale: float = 0.0) -> oracle.Problem:
    return oracle.Problem(
        bf16_bits(inp["q"]), bf16_bits(inp["k_prefix"]),
        bf16_bits(inp["v_prefix"]), inp["prefix_len"].numpy(),
        bf16_bits(inp["k_tree"]), bf16_bits(inp["v_tree"]),
        inp["parent"].numpy(), scale=scale)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


def tiny_workloads():
    """Small seeded problems with ragged prefixes, GQA and random trees."""
    return [
        Workload("pin-a", B=2, Hq=4, Hkv=2, D=4, T=5, L_cap=8, seed=11,
                 tree="random", prefix_range=(0, 8)),
        Workload("pin-b", B=1, Hq=3, Hkv=1, D=3, T=4, L_cap=6, seed=12,
                 tree="random", prefix_range=(0, 6)),
        Workload("pin-c", B=1, Hq=2, Hkv=2, D=8, T=6, L_cap=5, seed=13,
                 tree="random", k_peaked=True),
    ]


# ---------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------

def pin_mask_closure(max_T: int = 6):
    """Every parent array with T <= max_T: the oracle's ancestor-or-self bits
    equal the Boolean-closure ancestry."""
    for T in range(1, max_T + 1):
        for par in all_parent_arrays(T):
            bits = oracle.tree_mask(par)
            got = bits_to_bool(bits, T)
            assert (got == closure_ancestry(par)).all(), (T, par)


def pin_mask_levels_depth():
    """4/16/16/16/16 tree (LongSpec README, Evaluation): a node of level l
    sees exactly l tree nodes, one per level."""
    w = Workload("levels", B=1, Hq=1, Hkv=1, D=4, T=68, L_cap=0, seed=7)
    par = w.parents()[0]
    bits = bits_to_bool(oracle.tree_mask(par), 68)
    level = np.repeat(np.arange(1, 6), [4, 16, 16, 16, 16])
    for i in range(68):
        seen = np.nonzero(bits[i])[0]
        assert len(seen) == level[i], (i, seen)
        assert sorted(level[seen].tolist()) == list(range(1, level[i] + 1))


def _mp_row(q, keys, vals, scale):
    """Direct softmax attention at 60 digits: sum e^x v / sum e^x."""
    with mpmath.workdps(60):
        xs = [scale * mpmath.fsum(mpmath.mpf(float(a)) * mpmath.mpf(float(b))
                                  for a, b in zip(q, k)) for k in keys]
        ws = [mpmath.e ** x for x in xs]
        Z = mpmath.fsum(ws)
        D = len(q)
        out = [mpmath.fsum(w * mpmath.mpf(float(v[d])) for w, v in zip(ws, vals)) / Z
               for d in range(D)]
        return [float(o) for o in out], float(mpmath.log(Z))


def pin_brute_force():
    """Oracle == direct high-precision evaluation on tiny problems."""
    for w in tiny_workloads():
        inp = w.generate()
        p = problem_from(inp)
        out, lse = p.attention()
        q, kp, vp = f64(inp["q"]), f64(inp["k_prefix"]), f64(inp["v_prefix"])
        kt, vt = f64(inp["k_tree"]), f64(inp["v_tree"])
        lens, par = inp["prefix_len"].numpy(), inp["parent"].numpy()
        G = w.Hq // w.Hkv
        with mpmath.workdps(60):
            scale = 1 / mpmath.sqrt(w.D)
        for b in range(w.B):
            R = closure_ancestry(par[b])
            for h in range(w.Hq):
                kvh = h // G
                for t in range(w.T):
                    keys = list(kp[b, kvh, :lens[b]]) + [kt[b, kvh, i] for i in range(w.T) if R[t, i]]
                    vals = list(vp[b, kvh, :lens[b]]) + [vt[b, kvh, i] for i in range(w.T) if R[t, i]]
                    o_ref, l_ref = _mp_row(q[b, h, t], keys, vals, scale)
                    np.testing.assert_allclose(out[b, h, t], o_ref, rtol=0, atol=1e-12)
                    assert abs(lse[b, h, t] - l_ref) <= 1e-12, (b, h, t)


def pin_two_pass_merge():
    """lse-merge of prefix-only and tree-only partials == one pass; any cut
    of the prefix into chunks (split-KV) gives the same result."""
    rng = np.random.default_rng(5)
    for w in tiny_workloads():
        p = problem_from(w.generate())
        out, lse = p.attention()
        n, D = p.n_rows, p.D
        for trial in range(4):
            cuts = sorted(rng.integers(0, w.L_cap + 1, size=trial + 1).tolist())
            bounds = [0] + cuts + [w.L_cap]
            parts_o, parts_l = [], []
            for a, b in zip(bounds[:-1], bounds[1:]):
                o, l = p.prefix_partial(a, b)
                parts_o.append(o.reshape(n, D))
                parts_l.append(l.reshape(n))
            o, l = p.tree_partial()
            parts_o.append(o.reshape(n, D))
            parts_l.append(l.reshape(n))
            mo, ml = oracle.lse_merge(np.stack(parts_o), np.stack(parts_l))
            np.testing.assert_allclose(mo, out.reshape(n, D), rtol=0, atol=1e-12)
            np.testing.assert_allclose(ml, lse.reshape(n), rtol=0, atol=1e-12)


def _causal_decode(q, k_all, v_all, L, scale):
    """Textbook causal decoding: token t (at position L + t) attends to
    positions 0..L+t; mask from index comparison."""
    T = q.shape[0]
    s = scale * (q @ k_all.T)
    pos = np.arange(k_all.shape[0])[None, :]
    allowed = pos <= (L + np.arange(T))[:, None]
    s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    return (e @ v_all) / z, (m + np.log(z))[:, 0]


def pin_chain_is_causal_decode():
    """A chain-shaped tree (parent = [-1, 0, 1, ...]) reduces to ordinary
    causal decoding over [prefix; T tokens]; T = 1 is single-token decode."""
    for T in (1, 5):
        for L in (0, 7):
            w = Workload("chain", B=1, Hq=4, Hkv=2, D=8, T=T, L_cap=7, seed=20 + T,
                         tree="chain", prefix_range=(L, L))
            inp = w.generate()
            assert (inp["parent"].numpy()[0] == tree_chain(T)).all()
            p = problem_from(inp)
            out, lse = p.attention()
            scale = 1 / math.sqrt(w.D)
            for h in range(w.Hq):
                kvh = h // (w.Hq // w.Hkv)
                k_all = np.concatenate([f64(inp["k_prefix"])[0, kvh, :L], f64(inp["k_tree"])[0, kvh]])
                v_all = np.concatenate([f64(inp["v_prefix"])[0, kvh, :L], f64(inp["v_tree"])[0, kvh]])
                o_ref, l_ref = _causal_decode(f64(inp["q"])[0, h], k_all, v_all, L, scale)
                np.testing.assert_allclose(out[0, h], o_ref, rtol=0, atol=1e-12)
                np.testing.assert_allclose(lse[0, h], l_ref, rtol=0, atol=1e-12)


def pin_closed_form_q_zero():
    """q = 0: every visible score is 0, so lse = ln(L_b + depth(t)) exactly
    and out = mean of the visible V rows (depth counted on the 4/16/16/16/16
    level tree: level l sees l tree nodes)."""
    for L in (0, 1, 9):
        w = Workload("qzero", B=1, Hq=2, Hkv=1, D=4, T=68, L_cap=9, seed=30,
                     prefix_range=(L, L))
        inp = w.generate()
        inp["q"] = torch.zeros_like(inp["q"])
        p = problem_from(inp)
        out, lse = p.attention()
        level = np.repeat(np.arange(1, 6), [4, 16, 16, 16, 16])
        par = inp["parent"].numpy()[0]
        vp, vt = f64(inp["v_prefix"])[0, 0, :L], f64(inp["v_tree"])[0, 0]
        for t in range(68):
            np.testing.assert_allclose(lse[0, :, t], math.log(L + level[t]), rtol=0, atol=1e-13)
            chain = [t]
            while par[chain[-1]] != -1:
                chain.append(par[chain[-1]])
            mean = (vp.sum(axis=0) + vt[chain].sum(axis=0)) / (L + len(chain))
            for h in range(2):
                np.testing.assert_allclose(out[0, h, t], mean, rtol=0, atol=1e-13)


def pin_closed_form_constant_v():
    """V rows all equal to one row c_kvh per KV head -> out = c_kvh for every
    query head of the group, whatever q and K are (GQA grouping h -> h / G)."""
    w = Workload("constv", B=1, Hq=4, Hkv=2, D=4, T=5, L_cap=6, seed=31, tree="random")
    inp = w.generate()
    c = torch.tensor([[1.0, -2.0, 0.5, 3.0], [-4.0, 0.25, 2.0, -1.0]], dtype=torch.bfloat16)
    for kvh in range(2):
        inp["v_prefix"][0, kvh] = c[kvh]
        inp["v_tree"][0, kvh] = c[kvh]
    out, _ = problem_from(inp).attention()
    for h in range(4):
        np.testing.assert_allclose(out[0, h], np.broadcast_to(f64(c)[h // 2], (5, 4)),
                                   rtol=0, atol=1e-14)


def pin_closed_form_single_key():
    """L = 0 and a root node: the only visible key is the node itself, so
    out = v_root and lse = scale * q . k_root (exact rational arithmetic)."""
    from fractions import Fraction
    w = Workload("single", B=1, Hq=2, Hkv=1, D=8, T=3, L_cap=4, seed=32,
                 tree="random", prefix_range=(0, 0))
    inp = w.generate()
    out, lse = problem_from(inp, scale=0.5).attention()
    for h in range(2):
        qv = [Fraction(float(x)) for x in f64(inp["q"])[0, h, 0]]
        kv = [Fraction(float(x)) for x in f64(inp["k_tree"])[0, 0, 0]]
        exact = Fraction(1, 2) * sum(a * b for a, b in zip(qv, kv))
        assert abs(lse[0, h, 0] - float(exact)) <= 1e-15
        np.testing.assert_array_equal(out[0, h, 0], f64(inp["v_tree"])[0, 0, 0])


def pin_worked_example():
    """Hand-worked example, scale 1, D = 2, prefix keys (1,0), (0,1), tree
    parent = [-1, 0]:  node 0 sees both prefix keys and itself, node 1 sees
    both prefix keys, node 0 and itself."""
    bf = lambda rows: torch.tensor(rows, dtype=torch.bfloat16)
    inp = dict(
        q=bf([[[[1, 0], [0, 1]]]]),
        k_prefix=bf([[[[1, 0], [0, 1]]]]), v_prefix=bf([[[[1, 0], [0, 1]]]]),
        k_tree=bf([[[[2, 0], [0, 2]]]]), v_tree=bf([[[[2, 2], [-1, 1]]]]),
        prefix_len=torch.tensor([2], dtype=torch.int32),
        parent=torch.tensor([[-1, 0]], dtype=torch.int32))
    out, lse = problem_from(inp, scale=1.0).attention()
    e = math.e
    # node 0: scores 1, 0, 2 against (1,0), (0,1), (2,2)
    z0 = e + 1 + e * e
    o0 = np.array([e * 1 + 0 + e * e * 2, 0 + 1 + e * e * 2]) / z0
    # node 1: scores 0, 1, 0, 2 against (1,0), (0,1), (2,2), (-1,1)
    z1 = 1 + e + 1 + e * e
    o1 = np.array([1 + 0 + 2 - e * e, 0 + e + 2 + e * e]) / z1
    np.testing.assert_allclose(out[0, 0, 0], o0, rtol=0, atol=1e-14)
    np.testing.assert_allclose(out[0, 0, 1], o1, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], [math.log(z0), math.log(z1)], rtol=0, atol=1e-14)


def pin_relabel_equivariance():
    """Renumbering the tree nodes in another topological order permutes the
    output rows the same way."""
    w = Workload("perm", B=1, Hq=2, Hkv=1, D=4, T=68, L_cap=5, seed=33)
    inp = w.generate()
    par = inp["parent"].numpy()[0]
    out, lse = problem_from(inp).attention()
    # reverse the order of the nodes within every level: still topological
    level = np.repeat(np.arange(5), [4, 16, 16, 16, 16])
    perm = np.concatenate([np.nonzero(level == l)[0][::-1] for l in range(5)])  # new -> old
    inv = np.empty_like(perm)
    inv[perm] = np.arange(68)                                                  # old -> new
    new_par = np.array([-1 if par[o] == -1 else inv[par[o]] for o in perm], dtype=np.int32)
    inp2 = dict(inp)
    inp2["q"] = inp["q"][:, :, perm]
    inp2["k_tree"] = inp["k_tree"][:, :, perm]
    inp2["v_tree"] = inp["v_tree"][:, :, perm]
    inp2["parent"] = torch.from_numpy(new_par[None])
    out2, lse2 = problem_from(inp2).attention()
    np.testing.assert_allclose(out2, out[:, :, perm], rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse2, lse[:, :, perm], rtol=0, atol=1e-13)


ALL_PINS = [pin_mask_closure, pin_mask_levels_depth, pin_brute_force,
            pin_two_pass_merge, pin_chain_is_causal_decode,
            pin_closed_form_q_zero, pin_closed_form_constant_v,
            pin_closed_form_single_key, pin_worked_example,
            pin_relabel_equivariance]
