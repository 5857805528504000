"""Greedy tree acceptance against the oracle (needs a B200).

Integer outputs, so the bar is bit-exact: accept_len, the accepted path and
the bonus token of the CUDA path must equal the oracle's on the same seeded
logits.  Cases cover the LongSpec tree (4/16/16/16/16, 68 nodes) at a
Llama-3 vocabulary, chains, random trees up to 256 nodes, vocabularies whose
rows are not 16-byte aligned, argmax ties across slices, NaN and -inf
logits, empty and full acceptance, and a bad parent array.
"""
import numpy as np
import pytest
import torch

from oracle import accept as A
from tree_masked_verification_b200 import hta
from tree_masked_verification_b200.inputs import accept_inputs, bf16_bits

pytestmark = pytest.mark.gpu


def _run(logits, tok, par):
    dev = [t.cuda().contiguous() for t in (logits, tok, par)]
    ws = hta.new_accept_workspace(*tok.shape, logits.shape[-1])
    n, path, bonus = hta.accept_greedy(*dev, workspace=ws)
    status = hta.get_status(ws)
    return n.cpu().numpy(), path.cpu().numpy(), bonus.cpu().numpy(), status


def _check(logits, tok, par, what=""):
    n, path, bonus, status = _run(logits, tok, par)
    assert status == hta.OK, what
    rn, rpath, rbonus = A.accept_greedy(bf16_bits(logits), tok.numpy(), par.numpy())
    np.testing.assert_array_equal(n, rn, err_msg=f"{what}: accept_len")
    np.testing.assert_array_equal(path, rpath, err_msg=f"{what}: path")
    np.testing.assert_array_equal(bonus, rbonus, err_msg=f"{what}: bonus")
    return n


CASES = {
    # the LongSpec tree at the Llama-3 vocabulary (the benchmark's shape)
    "longspec-llama3": dict(B=4, T=68, V=128256, tree="levels", p=0.8),
    "longspec-vicuna": dict(B=8, T=68, V=32000, tree="levels", p=0.9),
    # V % 8 != 0: rows are not 16-byte aligned, the scalar path reads them
    "unaligned-rows": dict(B=3, T=20, V=1001, tree="random", p=0.7),
    "max-nodes": dict(B=2, T=256, V=5000, tree="random", p=0.95),
    "chain": dict(B=5, T=5, V=64, tree="chain", p=0.85),
    "single-node": dict(B=1, T=1, V=7, tree="chain", p=1.0),
    "tail-only": dict(B=2, T=9, V=5, tree="random", p=0.8),
}


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("seed", [0, 1])
def test_accept_matches_oracle(name, seed):
    c = CASES[name]
    d = accept_inputs(c["B"], c["T"], c["V"], 1000 * seed + len(name), tree=c["tree"],
                      p_match=c["p"])
    _check(d["logits"], d["draft_tokens"], d["parent"], f"{name}/{seed}")


def test_full_and_empty_acceptance():
    d = accept_inputs(2, 68, 128256, 5, p_match=1.0)
    n = _check(d["logits"], d["draft_tokens"], d["parent"], "all match")
    assert (n == 5).all()
    wrong = (d["draft_tokens"] + 1) % 128256
    n = _check(d["logits"], wrong.to(torch.int32), d["parent"], "no match")
    assert (n == 0).all()


def test_argmax_ties_across_slices_go_to_the_smallest_token():
    """Equal maxima placed in different slices of one row (the kernel splits
    a 128256-token row into slices): the smallest token id must win."""
    B, T, V = 1, 3, 128256
    d = accept_inputs(B, T, V, 9, tree="chain", p_match=1.0)
    logits = d["logits"].clone()
    for r, ids in enumerate(([5, 70000, 128255], [128255, 64000], [1, 0], [99999, 100000])):
        logits[0, r, ids] = 20.0
    tok = torch.tensor([[5, 64000, 0]], dtype=torch.int32)
    n = _check(logits, tok, d["parent"], "ties")
    assert n[0] == 3


def test_constant_rows_pick_token_zero():
    logits = torch.zeros(2, 5, 3000, dtype=torch.bfloat16)
    par = torch.tensor([[-1, 0, 1, -1], [-1, -1, 1, 2]], dtype=torch.int32)
    tok = torch.tensor([[0, 0, 1, 0], [1, 0, 0, 0]], dtype=torch.int32)
    n = _check(logits, tok, par, "constant")
    assert list(n) == [2, 3]


def test_nan_and_minus_inf_logits():
    """NaN counts as -inf on both sides; rows of only NaN and -inf pick
    token 0, rows with a finite entry pick their first maximum."""
    B, T, V = 2, 6, 2048
    d = accept_inputs(B, T, V, 11, tree="random", p_match=0.9)
    logits = d["logits"].clone()
    logits[0, 0, ::3] = float("nan")
    logits[0, 1] = float("-inf")
    logits[0, 1, 1::2] = float("nan")
    logits[1, 2] = float("nan")
    logits[1, 3, :1000] = float("-inf")
    _check(logits, d["draft_tokens"], d["parent"], "nan/-inf")


def test_bad_parent_is_reported():
    d = accept_inputs(3, 10, 500, 13, tree="random", p_match=0.9)
    par = d["parent"].clone()
    par[2, 4] = 7                           # a parent after its child
    n, path, _, status = _run(d["logits"], d["draft_tokens"], par)
    assert status == hta.ERR_BAD_PARENT
    assert n[2] == 0 and (path[2] == -1).all()
    rn, rpath, _ = A.accept_greedy(bf16_bits(d["logits"][:2]), d["draft_tokens"][:2].numpy(),
                                   par[:2].numpy())
    np.testing.assert_array_equal(n[:2], rn)
    np.testing.assert_array_equal(path[:2], rpath)


def test_rejects_misaligned_logits():
    d = accept_inputs(1, 4, 64, 1, tree="chain")
    flat = torch.zeros(1 * 5 * 64 + 1, dtype=torch.bfloat16, device="cuda")
    logits = flat[1:].view(1, 5, 64)        # 2-byte offset
    with pytest.raises(hta.HtaError) as e:
        hta.accept_greedy(logits, d["draft_tokens"].cuda(), d["parent"].cuda())
    assert e.value.code == hta.ERR_MISALIGNED


def test_many_sequences():
    """64 sequences of the LongSpec tree (4 416 logits rows): one accept CTA
    per sequence, slices spread over every row."""
    d = accept_inputs(64, 68, 4096, 21, p_match=0.85)
    _check(d["logits"], d["draft_tokens"], d["parent"], "B=64")
