"""longspec_hta_verify_noalloc against longspec_hta_verify (needs a B200).

longspec_hta_verify_noalloc serves callers that cannot allocate device
memory for a workspace (a serving engine that reserves all device memory at
start-up, or a decode step where a cudaMalloc would synchronise the device):
its scratch lives in a static array inside the library.  This file is
collected last so that a run stopping at its first failure has already run
every other test; it also passes alone in a fresh process.
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


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_workspace_entry_point_twice(name):
    torch.cuda.set_device(0)
    fn = _entry()
    w = CASES[name]
    d = H.make_inputs(w)
    ref_out, ref_lse = hta.verify(d["q"], d["k_prefix"], d["v_prefix"], d["prefix_len"],
                                  d["k_tree"], d["v_tree"], d["parent"], scale=w.scale)
    torch.cuda.synchronize()
    ref_o = ref_out.double().cpu().numpy()
    ref_l = ref_lse.double().cpu().numpy()
    dims = hta.dims_of(d["q"], d["k_prefix"], w.scale)
    for call in range(2):   # the static scratch keeps the first call's contents
        out = torch.full_like(d["q"], float("nan"))
        lse = torch.full(d["q"].shape[:3], float("nan"), dtype=torch.float32, device="cuda")
        assert _call(fn, dims, d, out, lse) == hta.OK
        torch.cuda.synchronize()
        H.assert_parity(out, lse, ref_o, ref_l, f"{name}: no-alloc call {call}")


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
