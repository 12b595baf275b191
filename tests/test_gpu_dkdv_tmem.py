"""GPU parity of the dK/dV kernel variant that keeps K~ and V in TMEM as MMA operands
(RA_BWD_DKDV_TMEM=1 selects it per call): every gradient against the float64 oracle, and
against the default dK/dV kernel on the same inputs (same per-element arithmetic and the
same order of 16-query MMA steps, so they agree to fp32 accumulation order at most).

The variant is off by default and has not been run on a GPU yet, so these tests run only
when RA_TEST_DKDV_TMEM=1 is set in the environment."""
import os

import numpy as np
import pytest

from helpers import compare, gpu_run, make, oracle_run, small_workload

pytestmark = [
    pytest.mark.gpu,
    pytest.mark.skipif(os.environ.get("RA_TEST_DKDV_TMEM") != "1",
                       reason="TMEM-operand dK/dV: set RA_TEST_DKDV_TMEM=1 to run"),
]


def rel(a, b):
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-30))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n", [1, 31, 32, 33, 128, 129, 383])
def test_dkdv_tmem_matches_oracle_and_default(monkeypatch, n, d, causal):
    wl = small_workload(1, 2, n, d, "bf16", causal, seed=7 * n + d)
    inp = make(wl)
    base = gpu_run(inp)
    monkeypatch.setenv("RA_BWD_DKDV_TMEM", "1")
    got = gpu_run(inp)
    compare(got, oracle_run(inp), "bf16", small=True)
    for key in ("dq", "dk", "dv", "dalpha"):
        assert rel(got[key], base[key]) <= 1e-5, key


def test_dkdv_tmem_many_tiles(monkeypatch):
    wl = small_workload(2, 3, 1100, 128, "bf16", True, seed=23)
    inp = make(wl)
    monkeypatch.setenv("RA_BWD_DKDV_TMEM", "1")
    compare(gpu_run(inp), oracle_run(inp), "bf16", small=True)
