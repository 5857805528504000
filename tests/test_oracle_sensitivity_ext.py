"""Plant a mistake in the acceptance, commit and sliding-window oracles (on
the CPU) and check that some pin fails.

Each oracle has a test-only switch, MUTATION, that plants one plausible slip
(a wrong index, a wrong tie-break, a dropped key, a missing update); the
pins of tests/test_oracle_accept.py, test_oracle_commit.py and
test_oracle_window.py, which rest on constructions of their own, must catch
every one of them.
"""
import pytest

from oracle import accept as A
from oracle import commit as C
from oracle import window as Wn
from tests import test_oracle_accept as pa
from tests import test_oracle_commit as pc
from tests import test_oracle_window as pw

ACCEPT_PINS = ([lambda s=s: pa.test_chain_tree_is_sequential_greedy_decoding(s) for s in range(6)]
               + [lambda s=s: pa.test_brute_force_over_root_paths(s) for s in range(8)]
               + [pa.test_argmax_ties_go_to_the_smallest_token, pa.test_no_match_and_all_match,
                  pa.test_every_shape_of_a_small_tree, pa.test_nan_counts_as_minus_inf])

COMMIT_PINS = ([lambda s=s: pc.test_committed_context_is_what_the_accepted_node_attended_to(s)
                for s in range(4)]
               + [pc.test_chain_fully_accepted_appends_in_order]
               + [lambda bs=bs: pc.test_paged_commit_equals_contiguous(bs) for bs in (16, 32)]
               + [pc.test_bad_inputs_leave_the_sequence_unchanged])

WINDOW_CASES = [([3, 11], 8, "random"), ([8, 8], 8, "random"), ([29, 17], 8, "random"),
                ([40, 5], 16, "chain")]
WINDOW_PINS = ([pw.test_wide_window_equals_the_verification_oracle]
               + [lambda c=c: pw.test_brute_force_on_the_linearised_sequence(*c) for c in WINDOW_CASES])


def _caught(module, mutation, pins):
    caught = 0
    module.MUTATION = mutation
    try:
        for pin in pins:
            try:
                pin()
            except (AssertionError, ValueError):   # a failed check, or an impossible result
                caught += 1
    finally:
        module.MUTATION = None
    return caught


@pytest.mark.parametrize("mutation", ["ties-last", "own-row", "shallowest", "bonus-root", "nan-wins"])
def test_planted_acceptance_mistake_is_caught(mutation):
    assert _caught(A, mutation, ACCEPT_PINS) > 0, f"no pin caught {mutation!r}"


@pytest.mark.parametrize("mutation", ["skip-one", "reversed", "no-advance", "v-from-k"])
def test_planted_commit_mistake_is_caught(mutation):
    assert _caught(C, mutation, COMMIT_PINS) > 0, f"no pin caught {mutation!r}"


@pytest.mark.parametrize("mutation", ["window+1", "no-ring", "no-self", "depth-0"])
def test_planted_window_mistake_is_caught(mutation):
    assert _caught(Wn, mutation, WINDOW_PINS) > 0, f"no pin caught {mutation!r}"


def test_unmutated_oracles_pass_every_pin():
    for module, pins in ((A, ACCEPT_PINS), (C, COMMIT_PINS), (Wn, WINDOW_PINS)):
        assert _caught(module, None, pins) == 0
