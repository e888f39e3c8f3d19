"""The fill reading of the selection (NOSA_FLAG_FILL) against the oracle in the
same reading: Gamma_e is the best of the not-yet-dropped candidates outside
Gamma_q, and a block that no component selects is dropped for good.  Small
seeded cases (device store, offload with fetch counts, empty start, a budget
where Gamma_q often takes pool blocks, k_q = 0) and one full-size layer of the
128K offload workload, whose first step ranks every prefilled candidate."""
import pytest

import bench
from tests import gpu_harness as H
from tests.test_gpu_configs import run_config

pytestmark = pytest.mark.gpu


def _run(sc):
    data = H.unit_data(sc)
    gpu = H.run_gpu(sc, data)
    assert gpu["err"] == 0
    bad = []
    st = H.compare(sc, data, gpu, report=bad)
    assert not bad, bad[:3]
    H.assert_parity(st)
    assert st["diverged"] <= st["cmp"] // 10, st
    return st


def test_fill_gqa8_device_store():
    _run(H.Scenario(B=2, Hq=16, Hkv=2, k_q=4, k_e=12, L0=64 * 37 + 21, steps=70, seed=1, fill=True))


def test_fill_offload_fetch_counts():
    st = _run(H.Scenario(B=2, Hq=8, Hkv=2, k_q=4, k_e=12, L0=64 * 40 + 3, steps=70, offload=True, seed=3,
                         fill=True))
    assert st["fetch_cmp"] > 0


@pytest.mark.parametrize("offload", [False, True])
def test_fill_empty_start(offload):
    """No prefill: the pool is built by the decode appends alone."""
    _run(H.Scenario(B=1, Hq=4, Hkv=2, k_q=2, k_e=6, L0=0, steps=200, offload=offload, seed=4, fill=True))


def test_fill_query_budget_larger_than_agnostic():
    """k_q = 8 > k_e = 3 with single-head groups: Gamma_q often takes pool blocks, so Sel holds
    fewer than k blocks and the pool shrinks and regrows."""
    _run(H.Scenario(B=3, Hq=4, Hkv=4, k_q=8, k_e=3, L0=64 * 25 + 40, steps=120, seed=9, fill=True,
                    lens=[64 * 25 + 40, 64 * 11 + 1, 64 * 30]))


def test_fill_no_query_budget():
    _run(H.Scenario(B=2, Hq=8, Hkv=2, k_q=0, k_e=10, L0=64 * 20 + 5, steps=80, seed=6, fill=True))


def test_fill_offload28_128k_one_layer_micro_batches():
    c = dict(bench.WORKLOADS["offload28-128k"], fill=True)
    st = run_config(c, steps=6, micro=2, name="offload28-128k layer 0, fill reading")
    assert st["fetch_cmp"] > 0
