"""KV commit of the accepted path against the oracle (needs a B200).

Pure data movement, so the bar is bit-exact: the whole cache (every row,
touched or not) and the advanced prefix lengths must equal the oracle's.
Covers the contiguous and paged caches, acceptance feeding the commit on
the device with no host round trip, and the device-detected errors.
"""
import numpy as np
import pytest
import torch

from oracle import accept as A
from oracle import commit as C
from tree_masked_verification_b200 import hta
from tree_masked_verification_b200.inputs import (Workload, accept_inputs, bf16_bits, commit_inputs,
                                                  paged_cache)

pytestmark = pytest.mark.gpu

SMALL = Workload("cm1", B=3, Hq=4, Hkv=2, D=64, T=12, L_cap=300, seed=81, tree="random",
                 prefix_range=(0, 280))
LONGSPEC = Workload("cm2", B=4, Hq=32, Hkv=8, D=128, T=68, L_cap=4096, seed=82, tree="levels",
                    prefix_range=(1000, 4000))


def _dev(inp):
    return {k: v.cuda().contiguous() for k, v in inp.items()}


def _bits(t):
    return bf16_bits(t.cpu())


@pytest.mark.parametrize("w", [SMALL, LONGSPEC], ids=["small-d64", "longspec-d128"])
@pytest.mark.parametrize("seed", [0, 1])
def test_commit_contiguous_matches_oracle(w, seed):
    inp = commit_inputs(w.replace(seed=w.seed + seed), seed)
    d = _dev(inp)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    hta.commit(d["k_prefix"], d["v_prefix"], d["prefix_len"], d["k_tree"], d["v_tree"],
               d["accept_len"], d["path"], workspace=ws)
    assert hta.get_status(ws) == hta.OK
    k, v, new_len, errors = C.commit(bf16_bits(inp["k_prefix"]), bf16_bits(inp["v_prefix"]),
                                     inp["prefix_len"].numpy(), bf16_bits(inp["k_tree"]),
                                     bf16_bits(inp["v_tree"]), inp["accept_len"].numpy(),
                                     inp["path"].numpy())
    assert not errors
    np.testing.assert_array_equal(_bits(d["k_prefix"]), k)
    np.testing.assert_array_equal(_bits(d["v_prefix"]), v)
    np.testing.assert_array_equal(d["prefix_len"].cpu().numpy(), new_len)


@pytest.mark.parametrize("bs", [16, 64, 128])
@pytest.mark.parametrize("w", [SMALL, LONGSPEC], ids=["small-d64", "longspec-d128"])
def test_commit_paged_matches_oracle(w, bs):
    inp = commit_inputs(w, 5)
    kc, vc, table = paged_cache(inp["k_prefix"], inp["v_prefix"], inp["prefix_len"].tolist(), bs,
                                seed=bs, reserve=w.T)
    d = _dev({"kc": kc, "vc": vc, "table": table, "prefix_len": inp["prefix_len"],
              "k_tree": inp["k_tree"], "v_tree": inp["v_tree"], "accept_len": inp["accept_len"],
              "path": inp["path"]})
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    hta.commit_paged(d["kc"], d["vc"], d["table"], d["prefix_len"], d["k_tree"], d["v_tree"],
                     d["accept_len"], d["path"], L_cap=w.L_cap, workspace=ws)
    assert hta.get_status(ws) == hta.OK
    k, v, new_len, errors = C.commit_paged(bf16_bits(kc), bf16_bits(vc), table.numpy(),
                                           inp["prefix_len"].numpy(), bf16_bits(inp["k_tree"]),
                                           bf16_bits(inp["v_tree"]), inp["accept_len"].numpy(),
                                           inp["path"].numpy(), w.L_cap)
    assert not errors
    np.testing.assert_array_equal(_bits(d["kc"]), k)
    np.testing.assert_array_equal(_bits(d["vc"]), v)
    np.testing.assert_array_equal(d["prefix_len"].cpu().numpy(), new_len)


def test_accept_then_commit_on_the_device():
    """Acceptance writes accept_len and path; the commit reads them on the
    same stream with no host synchronisation in between."""
    w = LONGSPEC
    acc = accept_inputs(w.B, w.T, 32000, seed=3, p_match=0.85)
    inp = w.generate()
    d = _dev({**inp, "logits": acc["logits"], "draft_tokens": acc["draft_tokens"],
              "parent": acc["parent"]})
    ws = hta.new_accept_workspace(w.B, w.T, 32000)
    n, path, _ = hta.accept_greedy(d["logits"], d["draft_tokens"], d["parent"], workspace=ws)
    hta.commit(d["k_prefix"], d["v_prefix"], d["prefix_len"], d["k_tree"], d["v_tree"], n, path,
               workspace=ws)
    assert hta.get_status(ws) == hta.OK
    rn, rpath, _ = A.accept_greedy(bf16_bits(acc["logits"]), acc["draft_tokens"].numpy(),
                                   acc["parent"].numpy())
    k, v, new_len, errors = C.commit(bf16_bits(inp["k_prefix"]), bf16_bits(inp["v_prefix"]),
                                     inp["prefix_len"].numpy(), bf16_bits(inp["k_tree"]),
                                     bf16_bits(inp["v_tree"]), rn, rpath)
    assert not errors and rn.max() > 0
    np.testing.assert_array_equal(_bits(d["k_prefix"]), k)
    np.testing.assert_array_equal(_bits(d["v_prefix"]), v)
    np.testing.assert_array_equal(d["prefix_len"].cpu().numpy(), new_len)


@pytest.mark.parametrize("case", ["len-over-T", "overflow", "bad-node", "bad-block"])
def test_bad_inputs_are_reported_and_leave_the_sequence(case):
    w = SMALL
    inp = commit_inputs(w, 11)
    inp["prefix_len"] = torch.tensor([10, 200, 50], dtype=torch.int32)
    inp["accept_len"] = torch.tensor([2, 3, 1], dtype=torch.int32)
    inp["path"][:, :3] = torch.tensor([[0, 1, 2]] * 3, dtype=torch.int32)
    want = hta.OK
    if case == "len-over-T":
        inp["accept_len"][1] = w.T + 1
        want = hta.ERR_BAD_PATH
    elif case == "overflow":
        inp["prefix_len"][1] = w.L_cap - 2
        want = hta.ERR_PREFIX_LEN_RANGE
    elif case == "bad-node":
        inp["path"][1, 2] = w.T
        want = hta.ERR_BAD_PATH
    kc, vc, table = paged_cache(inp["k_prefix"], inp["v_prefix"], inp["prefix_len"].tolist(), 16,
                                seed=4, reserve=w.T)
    if case == "bad-block":
        table[1, (200 + 2) // 16] = kc.shape[0] + 3
        want = hta.ERR_BAD_BLOCK
    d = _dev({"kc": kc, "vc": vc, "table": table, "prefix_len": inp["prefix_len"],
              "k_tree": inp["k_tree"], "v_tree": inp["v_tree"], "accept_len": inp["accept_len"],
              "path": inp["path"]})
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    hta.commit_paged(d["kc"], d["vc"], d["table"], d["prefix_len"], d["k_tree"], d["v_tree"],
                     d["accept_len"], d["path"], L_cap=w.L_cap, workspace=ws)
    assert hta.get_status(ws) == want
    k, v, new_len, errors = C.commit_paged(bf16_bits(kc), bf16_bits(vc), table.numpy(),
                                           inp["prefix_len"].numpy(), bf16_bits(inp["k_tree"]),
                                           bf16_bits(inp["v_tree"]), inp["accept_len"].numpy(),
                                           inp["path"].numpy(), w.L_cap)
    assert [e.b for e in errors] == [1]
    np.testing.assert_array_equal(_bits(d["kc"]), k)
    np.testing.assert_array_equal(_bits(d["vc"]), v)
    np.testing.assert_array_equal(d["prefix_len"].cpu().numpy(), new_len)


@pytest.mark.parametrize("paged", [False, True], ids=["contiguous", "paged16"])
def test_long_accepted_chain(paged):
    """A 200-node chain accepted whole: 200 rows per KV head appended, across
    many 16-key blocks."""
    w = Workload("cm3", B=2, Hq=4, Hkv=2, D=128, T=200, L_cap=1200, seed=83, tree="chain",
                 prefix_range=(100, 900))
    inp = w.generate()
    inp["accept_len"] = torch.tensor([200, 137], dtype=torch.int32)
    inp["path"] = torch.tile(torch.arange(200, dtype=torch.int32), (2, 1))
    inp["path"][1, 137:] = -1
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    if paged:
        kc, vc, table = paged_cache(inp["k_prefix"], inp["v_prefix"], inp["prefix_len"].tolist(), 16,
                                    seed=6, reserve=w.T)
        d = _dev({"kc": kc, "vc": vc, "table": table, "prefix_len": inp["prefix_len"],
                  "k_tree": inp["k_tree"], "v_tree": inp["v_tree"], "accept_len": inp["accept_len"],
                  "path": inp["path"]})
        hta.commit_paged(d["kc"], d["vc"], d["table"], d["prefix_len"], d["k_tree"], d["v_tree"],
                         d["accept_len"], d["path"], L_cap=w.L_cap, workspace=ws)
        k, v, new_len, errors = C.commit_paged(bf16_bits(kc), bf16_bits(vc), table.numpy(),
                                               inp["prefix_len"].numpy(), bf16_bits(inp["k_tree"]),
                                               bf16_bits(inp["v_tree"]), inp["accept_len"].numpy(),
                                               inp["path"].numpy(), w.L_cap)
        got_k, got_v = d["kc"], d["vc"]
    else:
        d = _dev(inp)
        hta.commit(d["k_prefix"], d["v_prefix"], d["prefix_len"], d["k_tree"], d["v_tree"],
                   d["accept_len"], d["path"], workspace=ws)
        k, v, new_len, errors = C.commit(bf16_bits(inp["k_prefix"]), bf16_bits(inp["v_prefix"]),
                                         inp["prefix_len"].numpy(), bf16_bits(inp["k_tree"]),
                                         bf16_bits(inp["v_tree"]), inp["accept_len"].numpy(),
                                         inp["path"].numpy())
        got_k, got_v = d["k_prefix"], d["v_prefix"]
    assert hta.get_status(ws) == hta.OK and not errors
    np.testing.assert_array_equal(_bits(got_k), k)
    np.testing.assert_array_equal(_bits(got_v), v)
    np.testing.assert_array_equal(d["prefix_len"].cpu().numpy(), new_len)
