"""Sliding-window tree attention (the draft model's self-attention) against
the oracle (needs a B200).

The ring holds the last W context positions at slot p mod W; slots no
position reaches are NaN in these inputs, so a kernel that read them as
keys would fail.  Cases: context shorter than, equal to and longer than the
window, ring wrapped at a tile boundary and inside a tile, GQA, D 64/128,
the LongSpec tree, a chain, an empty context, and the full-size draft
workload (32 heads over 8 KV heads, 68 nodes, W 512, 32k context) in the
benchmark's launch configuration on sampled KV heads.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import window as Wn
from tests import hta_testlib as H
from tree_masked_verification_b200 import hta
from tree_masked_verification_b200.inputs import WORKLOADS, Workload, bf16_bits, window_ring


def _bits(t):
    return bf16_bits(t)


def _ring_case(B, Hq, Hkv, D, T, lens, W, tree, seed):
    """Inputs with a full context of max(lens) positions, laid into a ring."""
    w = Workload("wn", B=B, Hq=Hq, Hkv=Hkv, D=D, T=T, L_cap=max(max(lens), 1), seed=seed, tree=tree)
    inp = w.generate()
    inp["prefix_len"] = torch.tensor(lens, dtype=torch.int32)
    inp["k_ring"], inp["v_ring"] = window_ring(inp["k_prefix"], inp["v_prefix"], lens, W)
    return inp


def _oracle(inp, W, rows=None):
    return Wn.window_attention(_bits(inp["q"]), _bits(inp["k_ring"]), _bits(inp["v_ring"]),
                               inp["prefix_len"].numpy(), _bits(inp["k_tree"]), _bits(inp["v_tree"]),
                               inp["parent"].numpy(), W, rows=rows)


def _gpu(inp):
    d = {k: inp[k].cuda().contiguous() for k in ("q", "k_ring", "v_ring", "prefix_len", "k_tree",
                                                  "v_tree", "parent")}
    ws = hta.new_window_workspace(hta.dims_of(d["q"], d["k_ring"]))
    out, lse = hta.window_verify(d["q"], d["k_ring"], d["v_ring"], d["prefix_len"], d["k_tree"],
                                 d["v_tree"], d["parent"], workspace=ws)
    return out, lse, hta.get_status(ws)


CASES = {
    # (B, Hq, Hkv, D, T, lens, W, tree)
    "short-context": (2, 8, 2, 128, 20, [50, 100], 128, "random"),
    "exact-window": (1, 4, 2, 128, 9, [256], 256, "random"),
    "wrapped-in-tile": (2, 4, 2, 64, 12, [1000, 777], 256, "random"),
    "wrapped-at-tile": (1, 4, 1, 128, 12, [1024], 256, "random"),
    "longspec-tree": (1, 8, 2, 128, 68, [3001], 512, "levels"),
    "chain": (2, 2, 1, 64, 5, [600, 129], 128, "chain"),
    "empty-context": (2, 4, 2, 128, 7, [0, 40], 128, "random"),
    # deep nodes whose window starts past the first key tile: their rows see
    # no key in that tile (a fully masked tile before the first real one)
    "deep-chain-wrapped": (1, 2, 1, 128, 40, [1000], 256, "chain"),
    # a 1024-slot ring (9 key tiles per call), four ragged contexts
    "wide-ring-ragged": (4, 8, 2, 128, 20, [5000, 1024, 700, 2049], 1024, "random"),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(CASES))
def test_window_matches_oracle(name):
    B, Hq, Hkv, D, T, lens, W, tree = CASES[name]
    inp = _ring_case(B, Hq, Hkv, D, T, lens, W, tree, seed=90 + len(name))
    out, lse, status = _gpu(inp)
    assert status == hta.OK
    o_ref, l_ref = _oracle(inp, W)
    H.assert_parity(out, lse, o_ref, l_ref, name)


@pytest.mark.gpu
def test_window_full_size_sampled_heads():
    """draft-window-512 (the benchmark's workload and launch configuration):
    every row of two KV heads against the oracle."""
    w = WORKLOADS["draft-window-512"]
    inp = w.generate()
    inp["k_ring"], inp["v_ring"] = inp["k_prefix"], inp["v_prefix"]
    out, lse, status = _gpu(inp)
    assert status == hta.OK
    for kvh in (0, w.Hkv - 1):
        rows = np.array([[0, kvh * w.G + g, t] for g in range(w.G) for t in range(w.T)], dtype=np.int32)
        o_ref, l_ref = _oracle(inp, w.L_cap, rows)
        H.assert_parity(out[0, rows[:, 1], rows[:, 2]], lse[0, rows[:, 1], rows[:, 2]], o_ref, l_ref,
                        f"kvh{kvh}")


@pytest.mark.gpu
def test_bad_parent_gives_nan_rows_and_status():
    inp = _ring_case(1, 4, 2, 128, 8, [300], 128, "random", seed=5)
    inp["parent"][0, 3] = 5
    out, lse, status = _gpu(inp)
    assert status == hta.ERR_BAD_PARENT
    assert torch.isnan(lse).all()


def test_window_rejects_bad_ring_sizes_on_host():
    lib = hta.load()
    for W, T in ((100, 8), (128, 128), (384 + 64, 8)):
        d = hta.Dims(1, 4, 2, 128, T, W, 0.0)
        ptrs = [4096 * (i + 1) for i in range(9)]
        assert lib.longspec_hta_window_verify(ctypes.byref(d), *ptrs, 4096 * 20, 1 << 30, None) == hta.ERR_INVALID_DIMS
