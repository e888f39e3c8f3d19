"""The largest configurations the library accepts, at parity with the oracle:
the maximum context (max_ctx = 2^20 tokens, 16383 candidate blocks per unit)
with the maximum budgets (k_q = 32, k_e = 256, so 289 blocks attended per
step), in device and offload mode; and the maximum unit count (2048 units,
GQA 8) with every unit compared."""
import pytest

from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def _run(sc, units=None):
    data = H.unit_data(sc)
    gpu = H.run_gpu(sc, data)
    assert gpu["err"] == 0
    bad = []
    st = H.compare(sc, data, gpu, units=units, report=bad)
    assert not bad, bad[:3]
    H.assert_parity(st)
    return st


@pytest.mark.parametrize("offload", [False, True])
def test_max_context_and_max_budgets(offload):
    L0 = (1 << 20) - 128 - 7  # the last steps cross into the final block
    sc = H.Scenario(B=1, Hq=2, Hkv=2, k_q=32, k_e=256, L0=L0, steps=40, offload=offload, seed=31, fused=True)
    assert sc.max_ctx == 1 << 20
    st = _run(sc)
    if offload:
        assert st["fetch_cmp"] > 0


def test_max_units():
    sc = H.Scenario(B=1024, Hq=16, Hkv=2, k_q=4, k_e=6, L0=64 * 5 + 9, steps=6, seed=32, fused=True)
    assert sc.units == 2048
    _run(sc)
