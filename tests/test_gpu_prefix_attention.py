"""Prefix-only attention (the draft model's cross-attention into the
target's KV cache) against the oracle (needs a B200).

The reference is the oracle's prefix pass over keys [0, L_b): plain
unmasked softmax attention of each query row to its sequence's prefix.
"""
import numpy as np
import pytest
import torch

from tests import hta_testlib as H
from tree_masked_verification_b200 import hta
from tree_masked_verification_b200.inputs import WORKLOADS, Workload

pytestmark = pytest.mark.gpu

SMALL = {
    # single query token, D = 64
    "t1-d64": Workload("px1", B=1, Hq=2, Hkv=1, D=64, T=1, L_cap=300, seed=61, tree="chain",
                       kind="prefix"),
    # GQA, ragged prefix lengths over several 128-key tiles
    "gqa-ragged": Workload("px2", B=2, Hq=4, Hkv=2, D=128, T=3, L_cap=700, seed=62, tree="chain",
                           prefix_range=(1, 700), kind="prefix"),
    # more rows than one 128-row tile
    "rows-200": Workload("px3", B=1, Hq=8, Hkv=2, D=128, T=50, L_cap=1000, seed=63, tree="chain",
                         kind="prefix"),
}


def _oracle(w, cpu):
    return H.oracle_problem(cpu, w.scale).prefix_partial(0, w.L_cap)


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("kernel", [hta.PREFIX_TCGEN05, hta.PREFIX_SIMT], ids=["tc", "simt"])
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_prefix_attention_small_matches_oracle(name, kernel, splits):
    w = SMALL[name]
    cpu = w.generate()
    ref_out, ref_lse = _oracle(w, cpu)
    dev = H.to_device(cpu)
    ws = hta.new_workspace(hta.dims_of(dev["q"], dev["k_prefix"], w.scale), splits)
    out, lse = hta.prefix_attention(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                                    workspace=ws, scale=w.scale, num_splits=splits,
                                    prefix_kernel=kernel)
    assert hta.get_status(ws) == hta.OK
    H.assert_parity(out, lse, ref_out, ref_lse, f"{name}/{kernel}/{splits}")


def test_prefix_attention_empty_prefix_gives_zero_and_minus_inf():
    """A sequence with L_b = 0 sees no key: out 0, lse -inf; the other
    sequence of the batch is unaffected."""
    w = SMALL["gqa-ragged"]
    cpu = w.generate()
    cpu["prefix_len"][0] = 0
    ref_out, ref_lse = _oracle(w, cpu)
    dev = H.to_device(cpu)
    out, lse = hta.prefix_attention(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                                    scale=w.scale)
    torch.cuda.synchronize()
    assert (out[0].float() == 0).all()
    assert torch.isneginf(lse[0]).all()
    H.assert_parity(out[1], lse[1], ref_out[1], ref_lse[1], "second sequence")


def test_prefix_attention_q_zero_is_the_mean_of_v():
    """q = 0: every score is 0, so out is the plain mean of the L_b value
    rows and lse = ln(L_b), a closed form independent of the oracle."""
    w = SMALL["gqa-ragged"]
    cpu = w.generate()
    cpu["q"].zero_()
    dev = H.to_device(cpu)
    out, lse = hta.prefix_attention(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                                    scale=w.scale)
    torch.cuda.synchronize()
    lens = cpu["prefix_len"].numpy()
    for b in range(w.B):
        L = int(lens[b])
        assert np.abs(lse[b].cpu().numpy() - np.log(L)).max() <= H.LSE_ABS
        for h in range(w.Hq):
            mean = cpu["v_prefix"][b, h // w.G, :L].double().mean(0)
            assert (out[b, h].double().cpu() - mean[None]).abs().max() <= H.OUT_MAX_ABS


def test_prefix_attention_full_size_sampled_rows():
    """The draft cross-attention workload (32 heads over 8 KV heads, 4 query
    tokens, 32k prefix) in the benchmark's launch configuration."""
    w = WORKLOADS["draft-xattn-32k"]
    dev = H.make_inputs(w)
    ws = hta.new_workspace(hta.dims_of(dev["q"], dev["k_prefix"], w.scale))
    out, lse = hta.prefix_attention(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                                    workspace=ws)
    assert hta.get_status(ws) == hta.OK
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    for b, kvh in ((0, 0), (0, w.Hkv - 1)):
        inp = w.generate_head(b, kvh)
        rows = np.array([[0, g, t] for g in range(w.G) for t in range(w.T)], dtype=np.int32)
        ro, rl = H.oracle_problem(inp, w.scale).prefix_partial(0, w.L_cap, rows)
        idx_h = torch.tensor([kvh * w.G + g for g in range(w.G) for _ in range(w.T)])
        idx_t = torch.tensor([t for _ in range(w.G) for t in range(w.T)])
        H.assert_parity(out[b, idx_h, idx_t], lse[b, idx_h, idx_t], ro, rl, f"b{b}/kvh{kvh}")
    del dev
    torch.cuda.empty_cache()
