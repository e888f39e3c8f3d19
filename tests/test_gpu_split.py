"""The split decode: nosa_decode_resident attends over Gamma_e + the local block
on a side stream while nosa_select and nosa_cache_sync run, and
nosa_decode_rest attends over the rest of Gamma_q and merges the two softmax
states.  The output must equal the one-pass sparse decode's, i.e. the
oracle's attention over S(t): device store and offload (fetch counts too),
ragged and empty starts, the budget edges k_q = 0 and k_e = 0, the fused head,
and one full-size layer of the 128K offload and 32K device workloads."""
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
    return st


def test_split_gqa8_device_store():
    _run(H.Scenario(B=2, Hq=16, Hkv=2, k_q=4, k_e=12, L0=64 * 37 + 21, steps=70, seed=1, split=True))


def test_split_offload_fetch_counts():
    st = _run(H.Scenario(B=2, Hq=8, Hkv=2, k_q=4, k_e=12, L0=64 * 40 + 3, steps=70, offload=True, seed=3,
                         split=True))
    assert st["fetch_cmp"] > 0


@pytest.mark.parametrize("offload", [False, True])
def test_split_ragged_and_empty(offload):
    _run(H.Scenario(B=3, Hq=8, Hkv=2, k_q=3, k_e=5, L0=0, steps=100, offload=offload, seed=8, split=True,
                    lens=[64 * 12 + 7, 0, 64 * 5]))


@pytest.mark.parametrize("k_q,k_e", [(0, 10), (10, 0)])
def test_split_budget_edges(k_q, k_e):
    _run(H.Scenario(B=2, Hq=4, Hkv=2, k_q=k_q, k_e=k_e, L0=64 * 30 + 9, steps=70, seed=10, split=True))


def test_split_with_fused_head_offload():
    _run(H.Scenario(B=2, Hq=8, Hkv=2, k_q=4, k_e=8, L0=64 * 25 + 50, steps=60, offload=True, seed=13,
                    split=True, head=True))


def test_split_offload28_128k_one_layer_micro_batches():
    c = dict(bench.WORKLOADS["offload28-128k"], split=True)
    st = run_config(c, steps=6, micro=2, name="offload28-128k layer 0, split decode")
    assert st["fetch_cmp"] > 0


def test_split_stack28_32k_one_layer():
    c = dict(bench.WORKLOADS["stack28-32k"], split=True)
    run_config(c, steps=6, name="stack28-32k layer 0, split decode")
