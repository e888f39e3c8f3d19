"""The decode append and the selection in one launch (nosa_append_select):
results identical to nosa_compress_append followed by nosa_select, checked
against the oracle on small cases (device store, offload fetch counts, empty
and ragged starts, block boundaries where Gamma_e changes mid-launch, the fill
reading, bf16 pooled keys, budget edges).  The benchmark workloads use the
fused launch, so the full-size layers of test_gpu_configs cover it at size;
the two full-size cases here run the separate launches instead."""
import pytest

import bench
from tests import gpu_harness as H
from tests.test_gpu_configs import run_config

pytestmark = pytest.mark.gpu


def _run(sc):
    data = H.unit_data(sc)
    gpu = H.run_gpu(sc, data)
    assert gpu["err"] == 0
    assert list(gpu["seq_len"]) == [n + sc.steps for n in sc.lens for _ in range(sc.Hkv)]
    bad = []
    st = H.compare(sc, data, gpu, report=bad)
    assert not bad, bad[:3]
    H.assert_parity(st)
    return st


def test_fused_gqa8_device_store():
    _run(H.Scenario(B=2, Hq=16, Hkv=2, k_q=4, k_e=12, L0=64 * 37 + 21, steps=140, seed=1, fused=True))


def test_fused_offload_fetch_counts():
    st = _run(H.Scenario(B=2, Hq=8, Hkv=2, k_q=4, k_e=12, L0=64 * 40 + 3, steps=140, offload=True, seed=3,
                         fused=True))
    assert st["fetch_cmp"] > 0


@pytest.mark.parametrize("offload", [False, True])
def test_fused_empty_and_ragged(offload):
    _run(H.Scenario(B=3, Hq=4, Hkv=2, k_q=2, k_e=6, L0=0, steps=200, offload=offload, seed=4, fused=True,
                    lens=[0, 64 * 9 + 60, 64 * 3]))


def test_fused_fill_reading():
    _run(H.Scenario(B=2, Hq=8, Hkv=2, k_q=6, k_e=6, L0=64 * 30 + 17, steps=140, seed=5, fused=True, fill=True))


def test_fused_bf16_pooled_keys():
    _run(H.Scenario(B=2, Hq=16, Hkv=2, k_q=8, k_e=8, L0=64 * 33, steps=130, seed=7, fused=True, ck_bf16=True))


@pytest.mark.parametrize("k_q,k_e", [(0, 10), (10, 0), (32, 96)])
def test_fused_budget_edges(k_q, k_e):
    _run(H.Scenario(B=2, Hq=4, Hkv=2, k_q=k_q, k_e=k_e, L0=64 * 140 + 9, steps=70, seed=10, fused=True))


def test_unfused_offload28_128k_one_layer_micro_batches():
    c = dict(bench.WORKLOADS["offload28-128k"], fuse=False)
    st = run_config(c, steps=6, micro=2, name="offload28-128k layer 0, separate append and select")
    assert st["fetch_cmp"] > 0


def test_unfused_stack28_32k_one_layer():
    c = dict(bench.WORKLOADS["stack28-32k"], fuse=False)
    run_config(c, steps=6, name="stack28-32k layer 0, separate append and select")


@pytest.mark.parametrize("offload", [False, True])
def test_layer_decode_step(offload):
    """NosaLayer.decode_step, the one-call step the README shows (the device store: nosa_fused_step;
    the offload store: fused append + select, cache sync, sparse decode)."""
    _run(H.Scenario(B=2, Hq=16, Hkv=2, k_q=4, k_e=12, L0=64 * 21 + 30, steps=70, offload=offload, seed=15,
                    layer_step=True))
