"""Per-step budget schedules and the sparse-stage gate (host only, CPU).

The pages' stage paragraph: budgets follow a precomputed per-step schedule
with at most two distinct values; the stage gates on self attention, a
minimum sequence length (8192 tokens by default) and the absence of a token
mask or causal flag.  Budgets are checked against the oracle's k per step.
"""
import numpy as np
import pytest

import oracle


@pytest.fixture(scope="module")
def sa():
    import prompt_aware_head_b200 as sa
    return sa


def test_two_value_schedule_matches_the_oracle_budget_per_step(sa):
    # 50 steps: the first 10 dense, the rest at the joint workload's budget (C = 256)
    sched = np.array([1.0] * 10 + [0.3] * 40, np.float32)
    k, dense = sa.sa_budget_schedule(sched, 256)
    assert list(k) == [oracle.budget(float(r), 256) for r in sched]
    assert list(k[:10]) == [256] * 10 and list(k[10:]) == [76] * 40
    assert dense.tolist() == [True] * 10 + [False] * 40


def test_constant_and_interleaved_schedules(sa):
    k, dense = sa.sa_budget_schedule([0.2] * 7, 512)
    assert k.tolist() == [102] * 7 and not dense.any()
    sched = [0.5, 0.3, 0.5, 0.3]  # two values in any order
    k, _ = sa.sa_budget_schedule(sched, 64)
    assert k.tolist() == [oracle.budget(r, 64) for r in sched] == [32, 19, 32, 19]
    # a budget the 1e-4 guard rounds up to every candidate is dense; just below it is not
    k, dense = sa.sa_budget_schedule([0.999995, 0.99999], 10)
    assert k.tolist() == [oracle.budget(0.999995, 10), oracle.budget(0.99999, 10)] == [10, 9]
    assert dense.tolist() == [True, False]


@pytest.mark.parametrize("sched,n_cand", [
    ([1.0, 0.5, 0.3], 64),          # a third distinct value
    ([0.3, 0.0], 64),               # density 0
    ([0.3, 1.5], 64),               # above 1
    ([0.3, float("nan")], 64),
    ([], 64),                       # no steps
    ([0.3], 0),                     # no candidates
])
def test_bad_schedules_are_refused(sa, sched, n_cand):
    with pytest.raises(sa.SAError) as e:
        sa.sa_budget_schedule(sched, n_cand)
    assert e.value.status == sa.SA_ERR_INVALID_ARG


def test_stage_gate(sa):
    assert sa.DEFAULT_MIN_SEQ_LEN == 8192
    assert sa.sa_sparse_stage_gate(8192) and not sa.sa_sparse_stage_gate(8191)
    assert sa.sa_sparse_stage_gate(16896) and sa.sa_sparse_stage_gate(33280)
    assert not sa.sa_sparse_stage_gate(4096)                      # the sdxl shape stays dense by default
    assert sa.sa_sparse_stage_gate(4096, min_seq_len=4096)
    assert sa.sa_sparse_stage_gate(64, min_seq_len=0)             # 0: no floor, every length qualifies
    assert not sa.sa_sparse_stage_gate(8191, min_seq_len=-1)      # negative: reserved, the default floor for now
    assert not sa.sa_sparse_stage_gate(16896, self_attention=False)
    assert not sa.sa_sparse_stage_gate(16896, token_mask=True)          # a general token mask declines
    assert not sa.sa_sparse_stage_gate(16896, token_mask="general")
    assert sa.sa_sparse_stage_gate(16896, token_mask="keys")              # a key padding mask is served
    assert sa.sa_sparse_stage_decline(16896, token_mask=sa.SA_TOKEN_MASK_KEY_PADDING) == 0
    assert sa.sa_sparse_stage_decline(16896, token_mask=7) == sa.SA_DECLINE_TOKEN_MASK  # unknown kinds: general
    assert not sa.sa_sparse_stage_gate(16896, causal=True)


def test_decline_reasons(sa):
    assert sa.sa_sparse_stage_decline(16896) == 0
    assert sa.sa_sparse_stage_decline(4096) == sa.SA_DECLINE_SHORT
    assert sa.sa_sparse_stage_decline(16896, self_attention=False, causal=True) == \
        sa.SA_DECLINE_NOT_SELF_ATTENTION | sa.SA_DECLINE_CAUSAL
    assert sa.sa_sparse_stage_decline(100, token_mask=True) == sa.SA_DECLINE_TOKEN_MASK | sa.SA_DECLINE_SHORT
    for N in (100, 8192, 40000):
        for floor in (0, 8192, -1):
            for flags in ((True, False, False), (False, True, True), (True, True, False)):
                assert sa.sa_sparse_stage_gate(N, floor, *flags) == (sa.sa_sparse_stage_decline(N, floor, *flags) == 0)


def test_declines_are_logged_once_per_reason_and_length(sa, caplog):
    import logging
    caplog.set_level(logging.INFO, logger="prompt_aware_head_b200")
    for _ in range(3):
        assert not sa.sa_sparse_stage_gate(1234)              # short: logged once
        assert not sa.sa_sparse_stage_gate(1234, causal=True)  # another reason set: once more
        assert not sa.sa_sparse_stage_gate(1298)              # another length: once more
        assert sa.sa_sparse_stage_gate(20000)                 # taken: nothing
    msgs = [r.getMessage() for r in caplog.records if r.name == "prompt_aware_head_b200"]
    assert msgs == ["sparse attention declined at N=1234: below the minimum length",
                    "sparse attention declined at N=1234: causal, below the minimum length",
                    "sparse attention declined at N=1298: below the minimum length"]
