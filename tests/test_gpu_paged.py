"""Paged prefix KV cache (block table) for verify and prefix-only attention
(needs a B200).

The paged calls read the same keys through a block table, so their results
must equal those of the contiguous calls bit for bit (same kernels, same
split); they are also checked against the oracle on the gathered keys.
"""
import pytest
import torch

from tests import hta_testlib as H
from tree_masked_verification_b200 import hta
from tree_masked_verification_b200.inputs import WORKLOADS, Workload, paged_cache

pytestmark = pytest.mark.gpu

RAGGED = Workload("pg1", B=2, Hq=8, Hkv=2, D=128, T=20, L_cap=1000, seed=71, tree="random",
                  prefix_range=(1, 1000))
D64 = Workload("pg2", B=1, Hq=2, Hkv=1, D=64, T=8, L_cap=300, seed=72, tree="random")


def _paged_inputs(w, block_size, seed):
    cpu = w.generate()
    kc, vc, table = paged_cache(cpu["k_prefix"], cpu["v_prefix"], cpu["prefix_len"].tolist(),
                                block_size, seed)
    dev = H.to_device(cpu)
    return cpu, dev, kc.cuda(), vc.cuda(), table.cuda()


@pytest.mark.parametrize("block_size", [16, 32, 64, 128])
@pytest.mark.parametrize("w", [RAGGED, D64], ids=["ragged-d128", "d64"])
def test_verify_paged_equals_contiguous_and_matches_oracle(w, block_size):
    cpu, dev, kc, vc, table = _paged_inputs(w, block_size, seed=100 + block_size)
    ws = hta.new_workspace(hta.dims_of(dev["q"], dev["k_prefix"], w.scale))
    ref_o, ref_l = hta.verify(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                              dev["k_tree"], dev["v_tree"], dev["parent"], scale=w.scale)
    out, lse = hta.verify_paged(dev["q"], kc, vc, table, dev["prefix_len"], dev["k_tree"],
                                dev["v_tree"], dev["parent"], L_cap=w.L_cap, workspace=ws,
                                scale=w.scale)
    assert hta.get_status(ws) == hta.OK
    assert torch.equal(out, ref_o), "paged and contiguous outputs differ"
    assert torch.equal(lse, ref_l), "paged and contiguous lse differ"
    o_or, l_or = H.oracle_problem(cpu, w.scale).attention()
    H.assert_parity(out, lse, o_or, l_or, f"paged bs={block_size}")


@pytest.mark.parametrize("block_size", [16, 128])
def test_prefix_attention_paged_equals_contiguous(block_size):
    w = RAGGED.replace(kind="prefix", tree="chain")
    cpu, dev, kc, vc, table = _paged_inputs(w, block_size, seed=200 + block_size)
    ref_o, ref_l = hta.prefix_attention(dev["q"], dev["k_prefix"], dev["v_prefix"],
                                        dev["prefix_len"], scale=w.scale)
    out, lse = hta.prefix_attention_paged(dev["q"], kc, vc, table, dev["prefix_len"],
                                          L_cap=w.L_cap, scale=w.scale)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
    o_or, l_or = H.oracle_problem(cpu, w.scale).prefix_partial(0, w.L_cap)
    H.assert_parity(out, lse, o_or, l_or, f"prefix-only paged bs={block_size}")


def test_bad_block_id_is_reported():
    w = RAGGED
    cpu, dev, kc, vc, table = _paged_inputs(w, 32, seed=300)
    table[1, 0] = kc.shape[0] + 5          # past the last cache block
    ws = hta.new_workspace(hta.dims_of(dev["q"], dev["k_prefix"], w.scale))
    hta.verify_paged(dev["q"], kc, vc, table, dev["prefix_len"], dev["k_tree"], dev["v_tree"],
                     dev["parent"], L_cap=w.L_cap, workspace=ws, scale=w.scale)
    assert hta.get_status(ws) == hta.ERR_BAD_BLOCK
    assert hta.get_status(ws) == hta.OK    # read and cleared


def test_verify_paged_full_size_equals_contiguous():
    """llama3-8b-32k with 16-key blocks in the benchmark's launch
    configuration: bit-identical to the contiguous call."""
    w = WORKLOADS["llama3-8b-32k"]
    cpu = w.generate()
    kc, vc, table = paged_cache(cpu["k_prefix"], cpu["v_prefix"], cpu["prefix_len"].tolist(), 16, 400)
    dev = H.to_device(cpu)
    ws = hta.new_workspace(hta.dims_of(dev["q"], dev["k_prefix"], w.scale))
    ref_o, ref_l = hta.verify(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                              dev["k_tree"], dev["v_tree"], dev["parent"], workspace=ws)
    assert hta.get_status(ws) == hta.OK
    kc, vc, table = kc.cuda(), vc.cuda(), table.cuda()
    out, lse = hta.verify_paged(dev["q"], kc, vc, table, dev["prefix_len"], dev["k_tree"],
                                dev["v_tree"], dev["parent"], L_cap=w.L_cap, workspace=ws)
    assert hta.get_status(ws) == hta.OK
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
    del dev, kc, vc
    torch.cuda.empty_cache()
