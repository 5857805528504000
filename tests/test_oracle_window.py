"""The sliding-window tree-attention oracle, pinned to things other than
itself (CPU).

- Window wider than everything: equals the verification oracle (plain C,
  prefix + ancestor-or-self mask) on the same keys.
- Brute force on a linearised sequence: each node's root path is laid out
  after the full context at positions L .. L+d-1, the textbook sliding-window
  mask (query position - W < key position <= query position) is taken by
  index comparison, and softmax is evaluated in 40-digit arithmetic without
  max subtraction: no ring, no depth bookkeeping.
- A chain tree reduces to ordinary sliding-window causal decoding.
"""
import mpmath
import numpy as np
import pytest
import torch

import oracle
from oracle import window as Wn
from tree_masked_verification_b200.inputs import Workload, bf16_bits, window_ring


def _case(B, Hq, Hkv, D, T, lens, W, tree, seed):
    w = Workload("win", B=B, Hq=Hq, Hkv=Hkv, D=D, T=T, L_cap=max(lens) + 1, seed=seed, tree=tree)
    inp = w.generate()
    inp["prefix_len"] = torch.tensor(lens, dtype=torch.int32)
    k_ring, v_ring = window_ring(inp["k_prefix"], inp["v_prefix"], lens, W)
    return inp, k_ring, v_ring


def _brute(inp, b, h, t, W, G):
    f = lambda x: (np.asarray(bf16_bits(x)).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    q = f(inp["q"][b, h, t])
    kc, vc = f(inp["k_prefix"][b, h // G]), f(inp["v_prefix"][b, h // G])
    kt, vt = f(inp["k_tree"][b, h // G]), f(inp["v_tree"][b, h // G])
    L = int(inp["prefix_len"][b])
    par = inp["parent"][b].tolist()
    path = []
    j = t
    while j != -1:
        path.append(j)
        j = par[j]
    path.reverse()
    seq_k = [kc[p] for p in range(L)] + [kt[j] for j in path]     # linear positions 0 .. L+d-1
    seq_v = [vc[p] for p in range(L)] + [vt[j] for j in path]
    qp = L + len(path) - 1
    vis = [kp for kp in range(len(seq_k)) if qp - W < kp <= qp]
    mpmath.mp.dps = 40
    s = 1 / mpmath.sqrt(q.shape[0])
    e = [mpmath.exp(s * mpmath.fsum(mpmath.mpf(a) * mpmath.mpf(c) for a, c in zip(q, seq_k[kp])))
         for kp in vis]
    Z = mpmath.fsum(e)
    out = [float(mpmath.fsum(ei * mpmath.mpf(seq_v[kp][d]) for ei, kp in zip(e, vis)) / Z)
           for d in range(q.shape[0])]
    return np.array(out), float(mpmath.log(Z))


def test_wide_window_equals_the_verification_oracle():
    inp, k_ring, v_ring = _case(2, 4, 2, 16, 9, [20, 33], 64, "random", 5)
    o, l = Wn.window_attention(bf16_bits(inp["q"]), bf16_bits(k_ring), bf16_bits(v_ring),
                               inp["prefix_len"].numpy(), bf16_bits(inp["k_tree"]),
                               bf16_bits(inp["v_tree"]), inp["parent"].numpy(), 64)
    ring_as_prefix = oracle.Problem(bf16_bits(inp["q"]), bf16_bits(torch.nan_to_num(k_ring)),
                                    bf16_bits(torch.nan_to_num(v_ring)), inp["prefix_len"].numpy(),
                                    bf16_bits(inp["k_tree"]), bf16_bits(inp["v_tree"]),
                                    inp["parent"].numpy())
    o_ref, l_ref = ring_as_prefix.attention()
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, l_ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("lens,W,tree", [
    ([3, 11], 8, "random"),      # L < W, window cuts into the context for deep nodes
    ([8, 8], 8, "random"),       # L = W
    ([29, 17], 8, "random"),     # L > W, ring wrapped, W not dividing L
    ([40, 5], 16, "chain"),      # chain: ordinary sliding-window causal decoding
])
def test_brute_force_on_the_linearised_sequence(lens, W, tree):
    inp, k_ring, v_ring = _case(2, 4, 2, 8, 6, lens, W, tree, 7)
    o, l = Wn.window_attention(bf16_bits(inp["q"]), bf16_bits(k_ring), bf16_bits(v_ring),
                               inp["prefix_len"].numpy(), bf16_bits(inp["k_tree"]),
                               bf16_bits(inp["v_tree"]), inp["parent"].numpy(), W)
    for b in range(2):
        for h in range(4):
            for t in range(6):
                ro, rl = _brute(inp, b, h, t, W, 2)
                np.testing.assert_allclose(o[b, h, t], ro, rtol=0, atol=1e-12)
                assert abs(l[b, h, t] - rl) <= 1e-12


def test_window_must_exceed_the_tree():
    inp, k_ring, v_ring = _case(1, 2, 1, 8, 8, [4], 8, "chain", 3)
    with pytest.raises(ValueError):
        Wn.window_attention(bf16_bits(inp["q"]), bf16_bits(k_ring), bf16_bits(v_ring),
                            inp["prefix_len"].numpy(), bf16_bits(inp["k_tree"]),
                            bf16_bits(inp["v_tree"]), inp["parent"].numpy(), 8)
