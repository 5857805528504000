"""CUDA path against the fp64 oracle, through the C ABI (needs a B200).

Small cases (oracle in seconds, several tiles and a ragged tail) are compared
element by element; the full-size workloads are compared on sampled rows and
on properties that hold at any size.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests import hta_testlib as H
from tree_masked_verification_b200 import build, hta
from tree_masked_verification_b200.inputs import WORKLOADS, Workload, tree_chain

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    hta.load()
    torch.cuda.init()


SMALL = {
    # packed rows 272 = 3 row tiles, ragged 1000-key prefix (7 tiles + 104)
    "llama-like-L1000": Workload("s1", B=1, Hq=8, Hkv=2, D=128, T=68, L_cap=1000, seed=101),
    # MHA, batch, ragged per-sequence lengths incl. tiny ones
    "vicuna-like-ragged": Workload("s2", B=3, Hq=4, Hkv=4, D=128, T=68, L_cap=900, seed=102,
                                   prefix_range=(1, 900)),
    # G = 5, peaked keys, 340 packed rows
    "qwq-like-peaked": Workload("s3", B=1, Hq=10, Hkv=2, D=128, T=68, L_cap=1500, seed=103,
                                k_peaked=True),
    "tiny": WORKLOADS["tiny"],
    "d64-random-tree": Workload("s4", B=2, Hq=4, Hkv=2, D=64, T=40, L_cap=700, seed=104,
                                tree="random", prefix_range=(300, 700)),
    "chain5": Workload("s5", B=1, Hq=8, Hkv=2, D=128, T=5, L_cap=2048, seed=105, tree="chain"),
    "single-token": Workload("s6", B=2, Hq=4, Hkv=1, D=128, T=1, L_cap=513, seed=106,
                             tree="chain"),
    "max-tree-256": Workload("s7", B=1, Hq=2, Hkv=1, D=128, T=256, L_cap=384, seed=107,
                             tree="random"),
    "deep-chain-256": Workload("s8", B=1, Hq=1, Hkv=1, D=64, T=256, L_cap=130, seed=108,
                               tree="chain"),
    "empty-prefix": Workload("s9", B=2, Hq=4, Hkv=2, D=128, T=68, L_cap=256, seed=109,
                             prefix_range=(0, 0)),
}


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("kernel", [hta.PREFIX_TCGEN05, hta.PREFIX_SIMT], ids=["tc", "simt"])
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_verify_small_matches_oracle(name, kernel, splits):
    w = SMALL[name]
    cpu = w.generate()
    ref_out, ref_lse = H.oracle_problem(cpu, w.scale).attention()
    dev = H.to_device(cpu)
    ws = hta.new_workspace(hta.dims_of(dev["q"], dev["k_prefix"], w.scale), splits)
    out, lse = hta.verify(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                          dev["k_tree"], dev["v_tree"], dev["parent"], workspace=ws,
                          scale=w.scale, num_splits=splits, prefix_kernel=kernel)
    assert hta.get_status(ws) == hta.OK
    H.assert_parity(out, lse, ref_out, ref_lse, f"{name}/{kernel}/{splits}")


@pytest.mark.parametrize("name", ["llama-like-L1000", "qwq-like-peaked", "d64-random-tree",
                                  "vicuna-like-ragged"])
@pytest.mark.parametrize("splits", [1, 4])
def test_prefix_partials_match_oracle_chunks(name, splits):
    """Each split-KV chunk's (O_c, lse_c) against the oracle's prefix-only
    pass over the same key range."""
    w = SMALL[name]
    cpu = w.generate()
    p = H.oracle_problem(cpu, w.scale)
    dev = H.to_device(cpu)
    for kernel in (hta.PREFIX_TCGEN05, hta.PREFIX_SIMT):
        o, l, C = hta.prefix_partial(dev["q"], dev["k_prefix"], dev["v_prefix"],
                                     dev["prefix_len"], scale=w.scale, num_splits=splits,
                                     prefix_kernel=kernel)
        torch.cuda.synchronize()
        S = o.shape[3]
        lens = cpu["prefix_len"].numpy()
        for c in range(S):
            ro, rl = p.prefix_partial(c * C, (c + 1) * C)
            lc = l[:, :, :, c].cpu().numpy().astype(np.float64)
            empty = np.isneginf(rl)
            assert (np.isneginf(lc) == empty).all(), (name, kernel, c)
            if (~empty).any():
                for b in range(w.B):
                    if c * C >= lens[b]:
                        continue
                    H.assert_parity(o[b, :, :, c], l[b, :, :, c], ro[b], rl[b],
                                    f"{name}/k{kernel}/chunk{c}/b{b}")


@pytest.mark.parametrize("name", ["llama-like-L1000", "max-tree-256", "deep-chain-256", "tiny",
                                  "d64-random-tree"])
def test_tree_partial_matches_oracle(name):
    w = SMALL[name]
    cpu = w.generate()
    ro, rl = H.oracle_problem(cpu, w.scale).tree_partial()
    dev = H.to_device(cpu)
    o, l = hta.tree_partial(dev["q"], dev["k_tree"], dev["v_tree"], dev["parent"], scale=w.scale)
    H.assert_parity(o, l, ro, rl, f"tree/{name}")


@pytest.mark.parametrize("name", ["llama-like-L1000", "max-tree-256", "deep-chain-256", "tiny",
                                  "d64-random-tree"])
def test_verify_with_empty_prefix_is_the_tree_partial(name):
    """With L_b = 0 for every sequence a verification call sees its tree keys
    only, so its out / lse are the oracle's tree-only pass (lse at 1e-3):
    the tree pass of the full call, trees of up to 256 nodes and 256-deep
    chains included, with every prefix chunk empty."""
    w = SMALL[name]
    cpu = w.generate()
    cpu["prefix_len"].zero_()
    ro, rl = H.oracle_problem(cpu, w.scale).tree_partial()
    dev = H.to_device(cpu)
    ws = hta.new_workspace(hta.dims_of(dev["q"], dev["k_prefix"], w.scale))
    out, lse = hta.verify(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                          dev["k_tree"], dev["v_tree"], dev["parent"], workspace=ws, scale=w.scale)
    assert hta.get_status(ws) == hta.OK
    H.assert_parity(out, lse, ro, rl, f"empty prefix = tree partial/{name}")


def _trees():
    out = []
    for name in ("llama3-8b-32k", "vicuna-7b-b8", "tiny", "ultra-256k-chain5"):
        out.append(WORKLOADS[name].parents())
    rng = np.random.default_rng(7)
    for T in (1, 2, 31, 32, 33, 64, 65, 200, 256):
        par = np.array([-1] + [int(rng.integers(-1, i)) for i in range(1, T)], dtype=np.int32)
        out.append(par[None])
        out.append(tree_chain(T)[None])
    out.append(np.stack([tree_chain(100), np.array([-1] * 100, dtype=np.int32)]))
    return out


def test_tree_mask_bits_exact():
    for par in _trees():
        B, T = par.shape
        got = hta.tree_mask(torch.from_numpy(par).cuda()).cpu().numpy().view(np.uint32)
        for b in range(B):
            ref = oracle.tree_mask(par[b])
            assert (got[b] == ref).all(), (B, T, b)


@pytest.mark.parametrize("name", ["llama3-8b-32k", "vicuna-7b-b8", "qwq-32b-32k-peaked",
                                  "ultra-256k", "ultra-256k-chain5", "tiny"])
def test_full_size_sampled_rows(name):
    """Full-size workload in the benchmark's launch configuration; sampled
    rows against the oracle, every output finite."""
    w = WORKLOADS[name]
    dev = H.make_inputs(w)
    ws = hta.new_workspace(hta.dims_of(dev["q"], dev["k_prefix"], w.scale))
    out, lse = hta.verify(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                          dev["k_tree"], dev["v_tree"], dev["parent"], workspace=ws)
    assert hta.get_status(ws) == hta.OK
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    for b, kvh, gts in H.sample_rows(w):
        ro, rl = H.oracle_rows_for_head(w, b, kvh, gts)
        idx_h = torch.tensor([kvh * w.G + g for g, _ in gts])
        idx_t = torch.tensor([t for _, t in gts])
        H.assert_parity(out[b, idx_h, idx_t], lse[b, idx_h, idx_t], ro, rl, f"{name}/b{b}/kvh{kvh}")
    del dev
    torch.cuda.empty_cache()


def test_full_size_q_zero_closed_form():
    """q = 0 at the Llama size: lse = ln(L + depth(t)) for every row, and out
    is the mean of the visible V rows (checked on sampled rows)."""
    w = WORKLOADS["llama3-8b-32k"]
    cpu = w.generate()
    cpu["q"].zero_()
    dev = H.to_device(cpu)
    out, lse = hta.verify(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                          dev["k_tree"], dev["v_tree"], dev["parent"])
    par = cpu["parent"].numpy()[0]
    depth = np.zeros(w.T, dtype=np.int64)
    for i, p in enumerate(par):
        depth[i] = 1 if p == -1 else depth[p] + 1
    expect = np.log(w.L_cap + depth)
    got = lse[0].cpu().numpy()
    assert np.abs(got - expect[None, :]).max() <= H.LSE_ABS
    vp = cpu["v_prefix"][0].double()
    vt = cpu["v_tree"][0].double()
    for h in (0, 31):
        kvh = h // w.G
        for t in (0, 5, 67):
            chain = [t]
            while par[chain[-1]] != -1:
                chain.append(par[chain[-1]])
            mean = (vp[kvh].sum(0) + vt[kvh, chain].sum(0)) / (w.L_cap + len(chain))
            assert (out[0, h, t].double().cpu() - mean).abs().max() <= H.OUT_MAX_ABS


def test_tree_dominant_cases():
    """Cases where the tree carries most of the softmax mass, so a wrong tree
    pass cannot hide under the tolerance: no prefix at all, and a short prefix
    with tree keys scaled up."""
    w = Workload("dom", B=2, Hq=8, Hkv=2, D=128, T=68, L_cap=300, seed=111, prefix_range=(0, 300))
    cpu = w.generate()
    cpu["k_tree"] = (cpu["k_tree"].float() * 3.0).to(torch.bfloat16)
    cpu["prefix_len"][0] = 0
    ref_out, ref_lse = H.oracle_problem(cpu).attention()
    ref_tree_o, ref_tree_l = H.oracle_problem(cpu).tree_partial()
    dev = H.to_device(cpu)
    out, lse = hta.verify(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                          dev["k_tree"], dev["v_tree"], dev["parent"])
    H.assert_parity(out, lse, ref_out, ref_lse, "tree-dominant")
    # with L_b = 0 the result is the tree partial itself
    H.assert_parity(out[0], lse[0], ref_tree_o[0], ref_tree_l[0], "L=0 == tree only")


def test_garbage_past_prefix_len_is_ignored():
    """K/V slots past L_b hold NaN/inf: the result must not change."""
    w = Workload("nan", B=3, Hq=8, Hkv=2, D=128, T=68, L_cap=1024, seed=112,
                 prefix_range=(1, 1000))
    cpu = w.generate()
    lens = cpu["prefix_len"].numpy()
    for b in range(w.B):
        cpu["k_prefix"][b, :, lens[b]:] = float("nan")
        cpu["v_prefix"][b, :, lens[b]:] = float("inf")
    ref_out, ref_lse = H.oracle_problem(cpu).attention()
    dev = H.to_device(cpu)
    for kernel in (hta.PREFIX_TCGEN05, hta.PREFIX_SIMT):
        out, lse = hta.verify(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                              dev["k_tree"], dev["v_tree"], dev["parent"], prefix_kernel=kernel)
        H.assert_parity(out, lse, ref_out, ref_lse, f"nan-tail/{kernel}")


def test_bad_parent_is_reported_and_rows_are_nan():
    w = Workload("badpar", B=2, Hq=4, Hkv=2, D=128, T=68, L_cap=256, seed=113)
    cpu = w.generate()
    ref_out, ref_lse = H.oracle_problem(cpu).attention()
    cpu["parent"][1, 10] = 50          # parent after the child: invalid
    dev = H.to_device(cpu)
    ws = hta.new_workspace(hta.dims_of(dev["q"], dev["k_prefix"]))
    out, lse = hta.verify(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                          dev["k_tree"], dev["v_tree"], dev["parent"], workspace=ws)
    assert hta.get_status(ws) == hta.ERR_BAD_PARENT
    assert hta.get_status(ws) == hta.OK          # cleared by the read
    assert torch.isnan(out[1].float()).all() and torch.isnan(lse[1]).all()
    H.assert_parity(out[0], lse[0], ref_out[0], ref_lse[0], "batch 0 unaffected")


def test_prefix_len_out_of_range_is_reported():
    w = Workload("badlen", B=2, Hq=4, Hkv=2, D=128, T=68, L_cap=256, seed=114)
    cpu = w.generate()
    dev = H.to_device(cpu)
    dev["prefix_len"][1] = 300
    ws = hta.new_workspace(hta.dims_of(dev["q"], dev["k_prefix"]))
    out, lse = hta.verify(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                          dev["k_tree"], dev["v_tree"], dev["parent"], workspace=ws)
    assert hta.get_status(ws) == hta.ERR_PREFIX_LEN_RANGE
    assert torch.isnan(out[1].float()).all()
    assert torch.isfinite(out[0].float()).all()


def test_deterministic_bits():
    w = SMALL["llama-like-L1000"]
    dev = H.make_inputs(w)
    a = hta.verify(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                   dev["k_tree"], dev["v_tree"], dev["parent"])
    b = hta.verify(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                   dev["k_tree"], dev["v_tree"], dev["parent"])
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("name", ["llama3-8b-32k", "qwq-32b-32k-peaked"])
def test_deterministic_bits_full_size(name):
    """Repeated calls at full size (43 key tiles per CTA, a 16-row remainder
    tile) give the same bits: a pipeline race between the warps of a CTA
    would show here first."""
    w = WORKLOADS[name]
    dev = H.make_inputs(w)
    ws = hta.new_workspace(hta.dims_of(dev["q"], dev["k_prefix"], w.scale))
    ref = None
    for _ in range(3):
        o, l = hta.verify(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                          dev["k_tree"], dev["v_tree"], dev["parent"], workspace=ws)
        assert hta.get_status(ws) == hta.OK
        if ref is None:
            ref = (o.clone(), l.clone())
        else:
            assert torch.equal(o, ref[0]) and torch.equal(l, ref[1])
    del dev
    torch.cuda.empty_cache()


def test_host_buffer_entry_point_matches_device_call():
    w = SMALL["vicuna-like-ragged"]
    cpu = {k: v.pin_memory() for k, v in w.generate().items()}
    dev = H.to_device(cpu)
    ref = hta.verify(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                     dev["k_tree"], dev["v_tree"], dev["parent"])
    dims = hta.dims_of(cpu["q"], cpu["k_prefix"])
    arena = torch.empty(hta.host_arena_bytes(dims), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(cpu["q"]).pin_memory()
    lse = torch.empty(cpu["q"].shape[:3], dtype=torch.float32).pin_memory()
    hta.verify_host(cpu["q"], cpu["k_prefix"], cpu["v_prefix"], cpu["prefix_len"],
                    cpu["k_tree"], cpu["v_tree"], cpu["parent"], out, lse, arena)
    torch.cuda.synchronize()
    assert torch.equal(out, ref[0].cpu()) and torch.equal(lse, ref[1].cpu())


def test_tc_matches_simt_at_llama_size():
    """The two prefix kernels agree at the full Llama size (GPU cross-check)."""
    w = WORKLOADS["llama3-8b-32k"]
    dev = H.make_inputs(w)
    a = hta.verify(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                   dev["k_tree"], dev["v_tree"], dev["parent"], prefix_kernel=hta.PREFIX_TCGEN05)
    b = hta.verify(dev["q"], dev["k_prefix"], dev["v_prefix"], dev["prefix_len"],
                   dev["k_tree"], dev["v_tree"], dev["parent"], prefix_kernel=hta.PREFIX_SIMT)
    assert (a[0].float() - b[0].float()).abs().max() <= 1e-2
    assert (a[1] - b[1]).abs().max() <= 1e-3
