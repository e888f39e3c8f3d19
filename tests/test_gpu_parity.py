"""Parity of the CUDA path (through the C ABI) with the CPU oracle on small
seeded workloads that span several tiles, cross block boundaries and have
ragged tails.  Tolerances: see tests/gpu_harness.py."""
import pytest

from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def _run(sc, allow_excused=True):
    data = H.unit_data(sc)
    gpu = H.run_gpu(sc, data)
    assert gpu["err"] == 0
    bad = []
    st = H.compare(sc, data, gpu, report=bad)
    assert not bad, bad[:3]
    H.assert_parity(st, allow_excused)
    return st


def test_gqa8_device_store():
    _run(H.Scenario(B=2, Hq=16, Hkv=2, k_q=4, k_e=12, L0=64 * 37 + 21, steps=70, seed=1))


def test_mha_block_boundary_first_step():
    _run(H.Scenario(B=1, Hq=4, Hkv=4, k_q=4, k_e=12, L0=64 * 20, steps=66, seed=2))


def test_offload_fetch_counts():
    st = _run(H.Scenario(B=2, Hq=8, Hkv=2, k_q=4, k_e=12, L0=64 * 40 + 3, steps=70, offload=True, seed=3))
    assert st["fetch_cmp"] > 0


@pytest.mark.parametrize("offload", [False, True])
def test_empty_start_no_prefill(offload):
    _run(H.Scenario(B=1, Hq=4, Hkv=2, k_q=2, k_e=6, L0=0, steps=150, offload=offload, seed=4))


@pytest.mark.parametrize("offload", [False, True])
def test_ragged_prefill(offload):
    _run(H.Scenario(B=3, Hq=8, Hkv=2, k_q=4, k_e=8, L0=0, lens=[37, 64 * 9, 64 * 30 + 5], steps=40,
                    offload=offload, seed=5))


def test_dense_decode():
    _run(H.Scenario(B=2, Hq=16, Hkv=2, k_q=4, k_e=12, L0=64 * 25 + 7, steps=4, seed=6, dense=True))


@pytest.mark.parametrize("k_q,k_e", [(32, 96), (0, 16), (16, 0)])
def test_budget_limits(k_q, k_e):
    _run(H.Scenario(B=1, Hq=16, Hkv=2, k_q=k_q, k_e=k_e, L0=64 * 300 + 11, steps=6, seed=7))


def test_all_blocks_fit_in_budget():
    # fewer candidates than k: every block selected, sparse == dense
    _run(H.Scenario(B=2, Hq=8, Hkv=1, k_q=16, k_e=48, L0=64 * 10 + 30, steps=5, seed=8, dense=True))


@pytest.mark.parametrize("offload", [False, True])
def test_units_split_over_several_ctas(offload):
    # 48 units x 25 selected blocks = 1200 items over 148 decode CTAs: 8 items per CTA, so
    # every unit is streamed by 4 or 5 CTAs and merged from their partial states; ragged lengths
    # leave some units below the budget (padded selections).
    lens = [64 * 30 + 5 + 97 * b for b in range(12)]
    _run(H.Scenario(B=12, Hq=8, Hkv=4, k_q=8, k_e=16, L0=0, steps=24, offload=offload, seed=21, fused=True,
                    lens=lens))


def test_units_merged_from_many_partials():
    # 5 units x 289 items (the largest budget, k_q = 32, k_e = 256) over 148 CTAs: each unit is
    # streamed by about 30 CTAs, and its last contributor merges about 30 partial states.
    _run(H.Scenario(B=5, Hq=8, Hkv=1, k_q=32, k_e=256, L0=64 * 300 + 33, steps=8, seed=22, fused=True))


@pytest.mark.parametrize("Hq,Hkv,offload", [(6, 2, False), (5, 1, True), (12, 2, False), (7, 1, False), (14, 2, True)])
def test_odd_group_sizes(Hq, Hkv, offload):
    # G = 3, 5, 6, 7, 7 query heads per kv head: the score sums G heads, the decode tiles carry
    # G of their 8 head columns, and outputs are strided by G * 128
    _run(H.Scenario(B=2, Hq=Hq, Hkv=Hkv, k_q=4, k_e=10, L0=64 * 26 + 41, steps=40, offload=offload, seed=30 + Hq,
                    fused=True))
