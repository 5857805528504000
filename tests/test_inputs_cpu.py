"""Seeded input generators and the benchmark's byte counts (CPU).

The generators hold no arithmetic of the method; these tests check that they
are deterministic and lay data out as their docstrings say (ring slots,
block tables with room for appended tokens, planted argmax tokens), and that
the byte counts the roofline uses follow the workload kind.
"""
import math

import numpy as np
import torch

import bench
from tree_masked_verification_b200.inputs import (WORKLOADS, Workload, accept_inputs, commit_inputs,
                                                  paged_cache, window_ring)


def test_generators_are_deterministic():
    a, b = accept_inputs(2, 68, 500, 7), accept_inputs(2, 68, 500, 7)
    assert all(torch.equal(a[k], b[k]) for k in a)
    w = Workload("d", B=2, Hq=4, Hkv=2, D=64, T=12, L_cap=100, seed=3, tree="random",
                 prefix_range=(0, 80))
    c1, c2 = commit_inputs(w, 5), commit_inputs(w, 5)
    assert all(torch.equal(c1[k], c2[k]) for k in c1)


def test_planted_token_is_each_rows_unique_maximum():
    d = accept_inputs(3, 20, 1000, 11, tree="random", p_match=1.0)
    x = d["logits"].float()
    top = x.argmax(-1)
    assert torch.equal(top.to(torch.int32), d["planted"])
    assert ((x == x.max(-1, keepdim=True).values).sum(-1) == 1).all()
    par = d["parent"].long()
    rows = torch.where(par < 0, torch.zeros_like(par), par + 1)
    assert torch.equal(d["draft_tokens"], torch.gather(d["planted"], 1, rows))   # p_match = 1


def test_commit_paths_are_root_paths():
    w = Workload("p", B=8, Hq=2, Hkv=1, D=64, T=30, L_cap=50, seed=9, tree="random",
                 prefix_range=(0, 20))
    inp = commit_inputs(w, 4)
    par = inp["parent"].numpy()
    for b in range(w.B):
        n = int(inp["accept_len"][b])
        path = inp["path"][b].tolist()
        assert all(x == -1 for x in path[n:])
        for d in range(n):
            assert par[b, path[d]] == (path[d - 1] if d else -1)


def test_window_ring_slots():
    k = torch.arange(2 * 1 * 40 * 8, dtype=torch.float32).reshape(2, 1, 40, 8).to(torch.bfloat16)
    kr, vr = window_ring(k, k, [37, 5], 16)
    for p in range(37 - 16, 37):
        assert torch.equal(kr[0, 0, p % 16], k[0, 0, p])
    assert torch.isnan(kr[1, 0, 5:].float()).all() and torch.equal(kr[1, 0, :5], k[1, 0, :5])


def test_paged_cache_reserves_room_for_appended_tokens():
    k = torch.randn(2, 2, 100, 64).to(torch.bfloat16)
    kc, vc, table = paged_cache(k, k, [30, 90], 16, seed=1, reserve=20)
    assert (table[0, : math.ceil(50 / 16)] >= 0).all() and (table[0, math.ceil(50 / 16):] == -1).all()
    assert (table[1] >= 0).sum() == math.ceil(100 / 16)          # capped at L_cap
    ids = table[table >= 0]
    assert len(set(ids.tolist())) == len(ids)                      # no block shared
    for b, L in ((0, 30), (1, 90)):
        for pos in range(L):
            assert torch.equal(kc[table[b, pos // 16], :, pos % 16], k[b, :, pos])


def test_window_workload_counts_only_the_window():
    w = WORKLOADS["draft-window-512"]
    assert (w.visible_lens() == 511).all() and (w.prefix_lens() == 32768).all()
    kv = 2 * w.Hkv * w.D * 2 * 511
    assert bench.prefix_algorithmic_bytes(w) == kv + w.B * w.Hq * w.T * w.D * 2
    assert w.algorithmic_bytes() > kv
    full = WORKLOADS["llama3-8b-32k"]
    assert bench.prefix_algorithmic_bytes(full) == 2 * 8 * 128 * 2 * 32768 + 32 * 68 * 128 * 2
    f = bench.floors(full, 6551.4)
    assert math.isclose(f["hbm_us"], bench.prefix_algorithmic_bytes(full) / 6551.4e9 * 1e6)
    assert f["tensor_us"] >= f["tensor_useful_us"] > 0


def test_verify_and_prefix_bytes_differ_by_the_tree():
    v = WORKLOADS["llama3-8b-32k"]
    p = v.replace(kind="prefix")
    tree = 2 * v.B * v.Hkv * v.T * v.D * 2 + v.B * v.T * 4
    assert v.algorithmic_bytes() - p.algorithmic_bytes() == tree
    assert np.array_equal(v.visible_lens(), v.prefix_lens())
