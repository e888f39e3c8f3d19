"""Pooled keys stored as bf16 (the fp64 sub-block mean rounded once to the
nearest bf16): the stored keys bit-exact against the oracle in the same mode,
and the selection and outputs at parity with it, on small cases and at the
128K-context offload workload's full size.  The fp32 store is checked bit-exact
here too (the mean rounded once to fp32)."""
import numpy as np
import pytest

import bench
import synth
from oracle import OracleUnit
from tests import gpu_harness as H
from tests.test_gpu_configs import run_config

pytestmark = pytest.mark.gpu


def _stored_keys(sc, gpu, u):
    """GPU pooled keys of unit u as float64 [n_sub][128] (fp32 or bf16 storage)."""
    n = int(gpu["seq_len"][u]) // 16
    ck = gpu["ck"].reshape(sc.units, -1, 128)[u, :n]
    if sc.ck_bf16:
        return synth.bf16_to_f32(ck.view(np.uint16)).astype(np.float64)
    return ck.astype(np.float64)


@pytest.mark.parametrize("ck_bf16", [False, True])
def test_stored_pooled_keys_bit_exact(ck_bf16):
    """Prefill (ragged) plus 80 decode steps crossing sub-block and block boundaries: every stored
    pooled key equals the oracle's, bit for bit."""
    sc = H.Scenario(B=3, Hq=8, Hkv=2, k_q=4, k_e=8, L0=0, steps=80, seed=11, lens=[64 * 9 + 5, 64 * 3, 17],
                    ck_bf16=ck_bf16)
    data = H.unit_data(sc)
    gpu = H.run_gpu(sc, data)
    assert gpu["err"] == 0
    K, V, E, _ = data
    for u in range(sc.units):
        b = u // sc.Hkv
        n = sc.lens[b] + sc.steps
        o = OracleUnit(k_q=sc.k_q, k_e=sc.k_e, cap=sc.max_ctx, ck_bf16=ck_bf16)
        o.prefill(K[u, :n], V[u, :n], E[u, :n])
        want = o.ck()
        got = _stored_keys(sc, gpu, u)
        assert got.shape == want.shape
        if not ck_bf16:
            want = want.astype(np.float32).astype(np.float64)
        assert np.array_equal(got, want), (u, np.argwhere(got != want)[:4])


def _run(sc):
    data = H.unit_data(sc)
    gpu = H.run_gpu(sc, data)
    assert gpu["err"] == 0
    bad = []
    st = H.compare(sc, data, gpu, report=bad)
    assert not bad, bad[:3]
    H.assert_parity(st)
    return st


def test_bf16_gqa8_device_store():
    _run(H.Scenario(B=2, Hq=16, Hkv=2, k_q=4, k_e=12, L0=64 * 37 + 21, steps=70, seed=1, ck_bf16=True))


def test_bf16_offload_ragged():
    st = _run(H.Scenario(B=3, Hq=8, Hkv=2, k_q=6, k_e=10, L0=0, steps=70, offload=True, seed=12,
                         lens=[64 * 41 + 3, 64 * 12 + 63, 0], ck_bf16=True))
    assert st["fetch_cmp"] > 0


def test_bf16_offload28_128k_one_layer_micro_batches():
    """Batch 64, 128K context, KV in pinned host memory, two micro-batches: the bf16 variant
    in the benchmark's launch configuration."""
    c = dict(bench.WORKLOADS["offload28-128k"], ck_bf16=True)
    st = run_config(c, steps=6, micro=2, name="offload28-128k layer 0, bf16 pooled keys")
    assert st["fetch_cmp"] > 0
