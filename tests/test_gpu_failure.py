"""Failure detection on the GPU, without a fault (needs a B200).

Every in-kernel wait of the verification pipeline is bounded; a wait that
runs out sets PIPELINE_TIMEOUT in the workspace status word.  The self-test
entry point leaves one such wait to run out (a barrier that nothing
completes), so the whole path -- bound, status bit, host read-out -- runs
for real, and the context must stay usable afterwards.
"""
import time

import pytest
import torch

from tests import hta_testlib as H
from tree_masked_verification_b200 import build, hta
from tree_masked_verification_b200.inputs import WORKLOADS

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_sets_the_status_then_the_context_works():
    torch.cuda.set_device(0)
    build.build()
    w = WORKLOADS["tiny"]
    cpu = w.generate()
    d = H.to_device(cpu)
    dims = hta.dims_of(d["q"], d["k_prefix"], w.scale)
    ws = hta.new_workspace(dims, 0, d["q"].device)
    assert hta.get_status(ws) == hta.OK

    t0 = time.monotonic()
    assert hta.selftest_wait_timeout(ws) == hta.OK
    assert hta.get_status(ws) == hta.ERR_PIPELINE_TIMEOUT
    waited = time.monotonic() - t0
    # the bound is 4e9 SM cycles: about 2 s at B200 clocks, never unbounded
    assert 0.5 < waited < 30.0, waited
    # get_status cleared the word, and the device still runs the pipeline
    assert hta.get_status(ws) == hta.OK
    out, lse = hta.verify(d["q"], d["k_prefix"], d["v_prefix"], d["prefix_len"], d["k_tree"],
                          d["v_tree"], d["parent"], workspace=ws, scale=w.scale)
    torch.cuda.synchronize()
    assert hta.get_status(ws) == hta.OK
    ref_o, ref_l = H.oracle_problem(cpu, w.scale).attention()
    H.assert_parity(out, lse, ref_o, ref_l, "after the self-test")


def test_selftest_rejects_bad_workspace_pointers():
    torch.cuda.set_device(0)
    build.build()
    assert hta.load().longspec_hta_selftest_wait_timeout(None, None) == hta.ERR_NULL_POINTER
    buf = torch.zeros(64, dtype=torch.uint8, device="cuda")
    assert hta.load().longspec_hta_selftest_wait_timeout(buf.data_ptr() + 4, None) == hta.ERR_MISALIGNED
