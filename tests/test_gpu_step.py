"""nosa_fused_step (append + select + sparse decode in one launch) against the oracle, through
the C ABI.  The cases cover every team geometry the launch takes -- one CTA per unit (more units
than SMs), two and four CTAs per unit (the one-round merge of few pieces), nine (the one-pass
merge) and 37 or 65 (the general merge) -- short contexts that grow through block boundaries
(Gamma_e refreshed by the append inside the launch), ragged lengths, both pooled-key types, one
budget empty, the largest budgets, and the configurations' own sizes in the benchmark's launch
configuration.  Tolerances and tie handling: tests/gpu_harness.py."""
import pytest
import torch

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
    H.record_stats(f"fused step {sc.B}x{sc.Hkv} L0={sc.L0} kq={sc.k_q} ke={sc.k_e} bf16={sc.ck_bf16}", st)
    return st


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("B,Hq,Hkv", [(2, 16, 2), (8, 16, 2), (1, 8, 1), (37, 8, 1)])
def test_team_geometries(B, Hq, Hkv, bf16):
    # units 4, 16, 1, 37: 37, 9, 65 and 4 CTAs per unit
    _run(H.Scenario(B=B, Hq=Hq, Hkv=Hkv, k_q=16, k_e=48, L0=64 * 90 + 17, steps=12, seed=60 + B, step=True,
                    ck_bf16=bf16))


def test_one_cta_per_unit():
    # 160 units: more than the SMs, so each unit is one CTA (no team waits, several waves)
    _run(H.Scenario(B=80, Hq=8, Hkv=2, k_q=8, k_e=24, L0=64 * 40 + 50, steps=6, seed=61, step=True))


def test_two_ctas_per_unit():
    _run(H.Scenario(B=32, Hq=16, Hkv=2, k_q=16, k_e=48, L0=64 * 70 + 5, steps=8, seed=62, step=True))


@pytest.mark.parametrize("bf16", [False, True])
def test_growth_through_block_boundaries(bf16):
    # a few candidates, fewer than k: Gamma_e fills and is refreshed by the append inside the launch
    _run(H.Scenario(B=2, Hq=8, Hkv=2, k_q=4, k_e=6, L0=64 * 3 + 60, steps=140, seed=63, step=True, ck_bf16=bf16))


def test_empty_start():
    _run(H.Scenario(B=1, Hq=4, Hkv=2, k_q=2, k_e=6, L0=0, steps=150, seed=64, step=True))


def test_ragged_lengths():
    _run(H.Scenario(B=3, Hq=8, Hkv=2, k_q=4, k_e=8, L0=0, lens=[37, 64 * 9, 64 * 30 + 5], steps=40, seed=65,
                    step=True))


@pytest.mark.parametrize("k_q,k_e", [(32, 96), (0, 16), (16, 0), (32, 256)])
def test_budgets(k_q, k_e):
    _run(H.Scenario(B=2, Hq=16, Hkv=2, k_q=k_q, k_e=k_e, L0=64 * 300 + 11, steps=6, seed=66, step=True))


@pytest.mark.parametrize("Hq,Hkv", [(6, 2), (7, 1), (16, 16)])
def test_group_sizes(Hq, Hkv):
    _run(H.Scenario(B=2, Hq=Hq, Hkv=Hkv, k_q=4, k_e=10, L0=64 * 26 + 41, steps=30, seed=67 + Hq, step=True))


def test_matches_separate_launches_bitwise_selection():
    # the same inputs through nosa_append_select + nosa_sparse_decode: identical S(t), Gamma_q and
    # state; outputs equal up to the order of floating-point sums.  bf16 pooled keys: both kernels
    # then sum each score in the same order, so even near-ties must come out the same.
    import numpy as np
    kw = dict(B=4, Hq=16, Hkv=2, k_q=16, k_e=48, L0=64 * 120 + 9, steps=10, seed=68, ck_bf16=True)
    a = H.Scenario(step=True, **kw)
    b = H.Scenario(fused=True, **kw)
    data = H.unit_data(a)
    ga, gb = H.run_gpu(a, data), H.run_gpu(b, data)
    assert ga["err"] == 0 and gb["err"] == 0
    for t in range(a.steps):
        np.testing.assert_array_equal(ga["nsel"][t], gb["nsel"][t])
        np.testing.assert_array_equal(ga["sel"][t], gb["sel"][t])
        np.testing.assert_array_equal(ga["gq"][t], gb["gq"][t])
        np.testing.assert_array_equal(ga["ge"][t], gb["ge"][t])
        np.testing.assert_allclose(ga["out"][t], gb["out"][t], atol=1e-2)
    np.testing.assert_array_equal(ga["seq_len"], gb["seq_len"])
    np.testing.assert_array_equal(ga["ck"], gb["ck"])


def test_refusals():
    import block_sparse_offloadable_b200 as nosa
    for kw, code in ((dict(offload=True), nosa.ERR_UNSUPPORTED), (dict(fill=True), nosa.ERR_UNSUPPORTED)):
        cfg = nosa.make_config(2, 16, 2, 16, 48, 4096, **kw)
        lay = nosa.NosaLayer(cfg)
        q = torch.zeros((2, 16, 128), dtype=torch.int16, device="cuda")
        kv = torch.zeros((4, 1, 128), dtype=torch.int16, device="cuda")
        e = torch.zeros((4, 1), dtype=torch.float32, device="cuda")
        with pytest.raises(nosa.NosaError) as ei:
            lay.fused_step(kv, kv, e, q, torch.empty_like(q))
        assert ei.value.code == code
    # a workspace below nosa_workspace_bytes: refused before any launch, the state untouched
    cfg = nosa.make_config(2, 16, 2, 16, 48, 4096)
    lay = nosa.NosaLayer(cfg)
    q = torch.zeros((2, 16, 128), dtype=torch.int16, device="cuda")
    kv = torch.zeros((4, 1, 128), dtype=torch.int16, device="cuda")
    e = torch.zeros((4, 1), dtype=torch.float32, device="cuda")
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(nosa.NosaError) as ei:
        nosa.nosa_fused_step(cfg, lay.state, kv, kv, e, q, lay.sel, lay.nsel, lay.gq, torch.empty_like(q), small)
    assert ei.value.code == nosa.ERR_CAPACITY
    torch.cuda.synchronize()
    assert lay.seq_len.cpu().tolist() == [0, 0, 0, 0]
