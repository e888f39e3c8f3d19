"""The eviction head fused into append (nosa_compress_append_head): e_j =
sum_h W2[h] softplus(v_j . W1[:, h]) with seeded synthetic weights.  The
logits the GPU stores are compared with the oracle's head (both fp64 with the
same operation order; the two sides' exp/log1p may differ in the last fp64
bit, so a logit may land one fp32 ulp away, rarely), and the whole step runs
at parity with the oracle fed the oracle's own logits: device store, offload,
the fill reading, and one full-size layer of the 128K offload workload."""
import numpy as np
import pytest

import bench
from tests import gpu_harness as H
from tests.test_gpu_configs import run_config

pytestmark = pytest.mark.gpu


def test_head_logits_match_oracle():
    """Ragged prefill (the tiled prefill kernel) and 90 decode steps (the per-warp decode path)."""
    sc = H.Scenario(B=3, Hq=8, Hkv=2, k_q=4, k_e=8, L0=0, steps=90, seed=21, head=True,
                    lens=[64 * 9 + 5, 300, 1])
    data = H.unit_data(sc)
    gpu = H.run_gpu(sc, data)
    assert gpu["err"] == 0
    E = data[2]
    n_exact = n_total = 0
    for u in range(sc.units):
        n = sc.lens[u // sc.Hkv] + sc.steps
        got, want = gpu["e"][u, :n], E[u, :n]
        assert np.all(np.abs(got - want) <= np.spacing(np.abs(want))), u
        n_exact += int(np.sum(got == want))
        n_total += n
    assert n_exact >= n_total - max(1, n_total // 10000), (n_exact, n_total)


def _run(sc):
    data = H.unit_data(sc)
    gpu = H.run_gpu(sc, data)
    assert gpu["err"] == 0
    bad = []
    st = H.compare(sc, data, gpu, report=bad)
    assert not bad, bad[:3]
    H.assert_parity(st)
    return st


def test_head_gqa8_device_store():
    _run(H.Scenario(B=2, Hq=16, Hkv=2, k_q=4, k_e=12, L0=64 * 37 + 21, steps=70, seed=1, head=True))


def test_head_offload_fetch_counts():
    st = _run(H.Scenario(B=2, Hq=8, Hkv=2, k_q=4, k_e=12, L0=64 * 40 + 3, steps=70, offload=True, seed=3,
                         head=True))
    assert st["fetch_cmp"] > 0


def test_head_with_fill_reading():
    _run(H.Scenario(B=2, Hq=8, Hkv=2, k_q=6, k_e=6, L0=64 * 30 + 17, steps=80, seed=5, head=True, fill=True))


def test_head_offload28_128k_one_layer_micro_batches():
    c = dict(bench.WORKLOADS["offload28-128k"], head=True)
    st = run_config(c, steps=6, micro=2, name="offload28-128k layer 0, fused eviction head")
    assert st["fetch_cmp"] > 0
