"""The per-shape autotuner's host side, without a GPU: the ranking statistic
(the mean between the 5/16 and 11/16 quantiles of the per-call times, after
the EXL2 runtime autotune described in the nightvoyager.top exllamav2
report, "创新之处"), the cache of choices per (M, K, N) and what dispatch and
workspace sizing make of a recorded choice."""
import numpy as np
import pytest

import mixed_bitwidth_weight_b200 as q

pytestmark = pytest.mark.filterwarnings("ignore")


@pytest.fixture(autouse=True)
def clean_cache():
    q.qgemm_tune_clear()
    yield
    q.qgemm_tune_clear()


def brute_iqm(v):
    v = sorted(v)
    n = len(v)
    a = min(n - 1, (5 * n) // 16)
    b = max(a + 1, -(-11 * n // 16))
    return sum(v[a:b]) / (b - a)


def test_iqm_matches_its_definition():
    assert q.qgemm_iqm(list(range(16))) == sum(range(5, 11)) / 6
    rng = np.random.default_rng(0)
    for n in (1, 2, 3, 7, 16, 17, 200, 201):
        v = rng.exponential(1.0, n).astype(np.float32)
        assert q.qgemm_iqm(v) == pytest.approx(brute_iqm(v.tolist()), rel=1e-6)


def test_iqm_ignores_outliers_and_order():
    v = [5.0] * 100 + [1e6] * 10 + [0.0] * 10
    rng = np.random.default_rng(1)
    rng.shuffle(v)
    assert q.qgemm_iqm(v) == 5.0
    with pytest.raises(ValueError):
        q.qgemm_iqm([])


def test_recorded_choice_drives_dispatch_and_plan():
    M, K, N = 1, 8192, 28672
    assert q.qgemm_tune_lookup(M, K, N) is None
    assert q.qgemm_path_for(M, K, N) == 0             # built-in: integer GEMV
    q.qgemm_tune_record(M, K, N, 2, 2)                # GEMM, k split <= 2
    assert q.qgemm_tune_lookup(M, K, N) == (2, 2)
    assert q.qgemm_path_for(M, K, N) == 2
    plan = q.qgemm_plan_info(M, K, N, 621)
    assert plan["path"] == 2 and plan["ring"] <= 2    # ring field = k splits for the GEMM
    assert q.qgemm_path_for(2, K, N) == 0             # other shapes keep the built-in choice
    q.qgemm_tune_record(M, K, N, 0, 1)                # integer GEMV, one CTA per SM
    plan = q.qgemm_plan_info(M, K, N, 621)
    assert plan["path"] == 0 and plan["ctas_per_sm"] == 1 and plan["grid"] <= plan["sms"]
    q.qgemm_tune_clear()
    assert q.qgemm_tune_lookup(M, K, N) is None
    assert q.qgemm_plan_info(M, K, N, 621)["ctas_per_sm"] == 2


@pytest.mark.parametrize("M,path,knob", [(5, 0, 1), (17, 1, 0), (1, 2, 3), (1, 0, 3), (1, 1, 1), (4, 7, 0)])
def test_record_refuses_variants_that_cannot_serve_M(M, path, knob):
    with pytest.raises(q.QGemmError):
        q.qgemm_tune_record(M, 4096, 4096, path, knob)


@pytest.mark.parametrize("M", [1, 2, 4, 5, 8, 13, 16, 17, 64, 2048])
def test_workspace_covers_every_candidate(M):
    K, N = 8192, 28672
    base = q.qgemm_workspace_bytes(M, K, N)
    for path, knob in [(0, 1), (0, 2), (1, 0), (2, 1), (2, 2), (2, 4)]:
        try:
            q.qgemm_tune_record(M, K, N, path, knob)
        except q.QGemmError:
            continue
        assert q.qgemm_workspace_bytes(M, K, N) == base   # independent of the choice
    q.qgemm_tune_clear()


def test_set_autotune_validates_mode():
    q.qgemm_set_autotune(0)
    with pytest.raises(q.QGemmError):
        q.qgemm_set_autotune(2)
