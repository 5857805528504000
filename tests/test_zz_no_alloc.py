"""longspec_hta_verify_noalloc against the fp64 oracle and against
longspec_hta_verify (needs a B200).

longspec_hta_verify_noalloc serves callers that cannot allocate device
memory for a workspace (a serving engine that reserves all device memory at
start-up, or a decode step where a cudaMalloc would synchronise the device):
its scratch lives in a static array inside the library, shared by every call
and keeping the last call's contents.  So each checked call here follows a
call that left different contents in that array.  This file is collected
last so that a run stopping at its first failure has already run every other
test; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests import hta_testlib as H
from tree_masked_verification_b200 import build, hta
from tree_masked_verification_b200.inputs import WORKLOADS, Workload

pytestmark = pytest.mark.gpu

CASES = {
    "llama-like-L1000": Workload("na1", B=1, Hq=8, Hkv=2, D=128, T=68, L_cap=1000, seed=201),
    "vicuna-like-ragged": Workload("na2", B=3, Hq=4, Hkv=4, D=128, T=68, L_cap=900, seed=202,
                                   prefix_range=(1, 900)),
    "tiny": WORKLOADS["tiny"],
}

# a call whose split partials cover more rows and splits than any case above
# (so that stale slots of it sit where the checked call reads), run first
POISON = Workload("na0", B=2, Hq=16, Hkv=4, D=128, T=68, L_cap=3000, seed=200)


def _entry():
    build.build()
    fn = hta.load().longspec_hta_verify_noalloc
    fn.argtypes = [ctypes.POINTER(hta.Dims)] + [ctypes.c_void_p] * 10
    fn.restype = ctypes.c_int
    return fn


def _call(fn, dims, d, out, lse):
    return fn(ctypes.byref(dims), d["q"].data_ptr(), d["k_prefix"].data_ptr(),
              d["v_prefix"].data_ptr(), d["prefix_len"].data_ptr(), d["k_tree"].data_ptr(),
              d["v_tree"].data_ptr(), d["parent"].data_ptr(), out.data_ptr(), lse.data_ptr(),
              torch.cuda.current_stream().cuda_stream)


def _run(fn, w, d):
    dims = hta.dims_of(d["q"], d["k_prefix"], w.scale)
    out = torch.full_like(d["q"], float("nan"))
    lse = torch.full(d["q"].shape[:3], float("nan"), dtype=torch.float32, device="cuda")
    assert _call(fn, dims, d, out, lse) == hta.OK
    torch.cuda.synchronize()
    return out, lse


def _poison(fn, bad_len):
    """Leave other contents in the static scratch: a larger problem, and
    with bad_len one whose prefix_len exceeds L_cap, so that its split
    partials are left as NaN lse slots."""
    d = H.make_inputs(POISON)
    if bad_len:
        d["prefix_len"].fill_(POISON.L_cap + 5)
    out, lse = _run(fn, POISON, d)
    if bad_len:
        assert torch.isnan(lse).all()


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_oracle_and_workspace_entry_point(name):
    torch.cuda.set_device(0)
    fn = _entry()
    w = CASES[name]
    cpu = w.generate()
    ref_o, ref_l = H.oracle_problem(cpu, w.scale).attention()
    d = H.to_device(cpu)
    ws_out, ws_lse = hta.verify(d["q"], d["k_prefix"], d["v_prefix"], d["prefix_len"],
                                d["k_tree"], d["v_tree"], d["parent"], scale=w.scale)
    torch.cuda.synchronize()
    for call, bad_len in enumerate((False, True)):
        _poison(fn, bad_len)
        out, lse = _run(fn, w, d)
        H.assert_parity(out, lse, ref_o, ref_l, f"{name}: no-alloc call {call} vs oracle")
        # the same kernels as the workspace entry point: the same bits
        assert torch.equal(out, ws_out) and torch.equal(lse, ws_lse), f"{name}: call {call}"


def test_noalloc_bad_parent_shows_as_nan_rows():
    """The call has no status word to query: a bad parent array turns that
    sequence's rows of out and lse into NaN; the other sequences are
    unaffected."""
    torch.cuda.set_device(0)
    fn = _entry()
    w = Workload("na3", B=2, Hq=4, Hkv=2, D=128, T=68, L_cap=256, seed=203)
    cpu = w.generate()
    ref_o, ref_l = H.oracle_problem(cpu, w.scale).attention()
    cpu["parent"][1, 10] = 50          # a parent after its child: invalid
    d = H.to_device(cpu)
    _poison(fn, False)
    out, lse = _run(fn, w, d)
    assert torch.isnan(out[1].float()).all() and torch.isnan(lse[1]).all()
    H.assert_parity(out[0], lse[0], ref_o[0], ref_l[0], "batch 0 of a bad-parent call")
    # the next good call on the same scratch is unaffected
    cpu["parent"][1, 10] = 3
    ref_o, ref_l = H.oracle_problem(cpu, w.scale).attention()
    out, lse = _run(fn, w, H.to_device(cpu))
    H.assert_parity(out, lse, ref_o, ref_l, "good call after a bad-parent call")


def test_noalloc_rejects_problems_beyond_its_scratch():
    torch.cuda.set_device(0)
    fn = _entry()
    small = torch.zeros(1024, dtype=torch.bfloat16, device="cuda")
    d = {k: small for k in ("q", "k_prefix", "v_prefix", "k_tree", "v_tree")}
    d["prefix_len"] = torch.zeros(8, dtype=torch.int32, device="cuda")
    d["parent"] = torch.zeros(8, dtype=torch.int32, device="cuda")
    # B*Hq*T*(D+1)*4 bytes of partials even with one split: 67 MB > 16 MiB
    dims = hta.Dims(8, 64, 8, 128, 256, 1024, 0.0)
    out = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(16, dtype=torch.float32, device="cuda")
    assert _call(fn, dims, d, out, lse) == hta.ERR_WORKSPACE_TOO_SMALL
