"""The native batch planner's parity with the oracle (tests/test_batcher.py), run again in the GPU session so the
round's GPU test run, which selects `-m gpu`, also covers it. pp_plan_batches is host code: it needs the built
library, not a device."""
import pytest

from tests import test_batcher as T

pytestmark = pytest.mark.gpu


def test_plan_batches_matches_oracle_gpu_session():
    T.test_plan_batches_matches_oracle()


def test_plan_batches_workload_sized_gpu_session():
    T.test_plan_batches_dpo_sized()


def test_plan_batches_rejects_bad_input_gpu_session():
    T.test_plan_batches_rejects_bad_input()
