"""Pins of the CPU oracle against what the NOSA pages and the mathematics fix.

Each test is chosen so that a plausible slip (a dropped bias, a wrong pooling
order, a wrong index, a transposed operand, a wrong tie rule) fails it.
The expected values come from closed forms, constructions whose answer is
known by design, or special cases that reduce to textbook softmax attention.
"""
import numpy as np
import pytest

import synth
from oracle import OracleUnit
from tests import cases

FIXTURES = ["maxpool_two_stage.json", "gqa_group_sum.json", "tie_lower_index.json", "evict_two_stage.json",
            "signed_zero_tie.json"]


@pytest.mark.parametrize("name", FIXTURES)
def test_golden_selection(name):
    spec = cases.load_fixture(name)
    K, V, e, q = cases.build_fixture(spec)
    u = OracleUnit(D=spec["D"], G=spec["G"], block=spec["block"], sub=spec["sub"], k_q=spec["k_q"],
                   k_e=spec["k_e"], cap=64 * 64)
    u.prefill(K, V, e)
    z = np.zeros(spec["D"], np.uint16)
    r = u.step(z, z, 0.0, q)
    assert r["gq"].tolist() == spec["expect_gq"]
    if "expect_ge" in spec:
        assert r["ge"].tolist() == spec["expect_ge"]
    assert r["sel"].tolist() == spec["expect_sel"]


def test_tie_two_way_order():
    spec = cases.load_fixture("tie_lower_index.json")
    spec["k_q"] = 2
    K, V, e, q = cases.build_fixture(spec)
    u = OracleUnit(G=1, k_q=2, k_e=0, cap=4096)
    u.prefill(K, V, e)
    z = np.zeros(128, np.uint16)
    assert u.step(z, z, 0.0, q)["gq"].tolist() == [1, 3]


def test_compressed_keys_closed_form():
    """Ramp keys: K[j][d] = (j mod 16)/16 * (+1 even d, -1 odd d) + (sub-block index mod 8)/2.
    The mean over an aligned 16-token sub-block s is +-7.5/16 + (s mod 8)/2 exactly."""
    L, D = 16 * 13 + 5, 128
    j = np.arange(L)
    sign = np.where(np.arange(D) % 2 == 0, 1.0, -1.0)
    K = ((j % 16) / 16.0)[:, None] * sign[None, :] + (((j // 16) % 8) / 2.0)[:, None]
    Kb = cases.f32_to_bf16_bits_exact(K.astype(np.float32))
    u = OracleUnit(k_q=1, k_e=1, cap=4096)
    u.prefill(Kb, Kb, np.zeros(L, np.float32))
    ck = u.ck()
    assert ck.shape == (13, D)
    s = np.arange(13)
    want = 7.5 / 16 * sign[None, :] + ((s % 8) / 2.0)[:, None]
    assert np.array_equal(ck, want)


def test_block_eviction_closed_form():
    """One spike x > 0 in block 1 -> E_1 = x/16; a negative spike in block 2 leaves its max at 0."""
    L = 64 * 4 + 3
    e = np.zeros(L, np.float32)
    e[64 + 37] = 3.0
    e[128 + 5] = -7.0
    z = np.zeros((L, 128), np.uint16)
    u = OracleUnit(k_q=1, k_e=1, cap=4096)
    u.prefill(z, z, e)
    assert u.E().tolist() == [0.0, 3.0 / 16, 0.0, 0.0]


@pytest.mark.parametrize("G", [1, 4])
def test_all_blocks_selected_equals_dense_softmax(G):
    """With k_q >= number of candidates every block is selected, so the sparse
    step must equal textbook softmax(q K^T / sqrt(D) + e) V over all L tokens."""
    L0 = 699  # 10 complete blocks + a 59-token local block; the step adds one
    K, V, e = cases.synthetic_unit(7, 0, 0, 1, L0 + 1)
    q = cases.synthetic_queries(7, 0, 0, 1, G, 1)[0]
    u = OracleUnit(G=G, k_q=16, k_e=4, cap=2048)
    u.prefill(K[:L0], V[:L0], e[:L0])
    r = u.step(K[L0], V[L0], float(e[L0]), q)
    assert r["sel"].tolist() == list(range(11))
    want = cases.textbook_attention(q, K, V, e, np.arange(L0 + 1), 1 / np.sqrt(128))
    np.testing.assert_allclose(r["o"], want, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(u.dense(q), want, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("G", [1, 8])
def test_sparse_step_is_softmax_over_selected_tokens(G):
    L0 = 64 * 45 + 17
    K, V, e = cases.synthetic_unit(11, 2, 1, 0, L0 + 1)
    q = cases.synthetic_queries(11, 2, 1, 0, G, 1)[0]
    u = OracleUnit(G=G, k_q=4, k_e=6, cap=4096)
    u.prefill(K[:L0], V[:L0], e[:L0])
    r = u.step(K[L0], V[L0], float(e[L0]), q)
    sel = r["sel"]
    assert sel[-1] == L0 // 64 and len(sel) <= 4 + 6 + 1
    assert sel[:-1].tolist() == sorted(set(r["gq"].tolist()) | set(r["ge"].tolist()))
    tok = np.concatenate([np.arange(b * 64, min(b * 64 + 64, L0 + 1)) for b in sel])
    want = cases.textbook_attention(q, K, V, e, tok, 1 / np.sqrt(128))
    np.testing.assert_allclose(r["o"], want, rtol=1e-12, atol=1e-15)


def _beats(sa, ia, sb, ib):
    return sa > sb or (sa == sb and ia < ib)


def test_topk_is_the_k_best_by_pairwise_check():
    """Brute force: every selected block beats every unselected candidate."""
    L0 = 64 * 60 + 3
    K, V, e = cases.synthetic_unit(3, 0, 0, 0, L0 + 1)
    q = cases.synthetic_queries(3, 0, 0, 0, 2, 1)[0]
    u = OracleUnit(G=2, k_q=7, k_e=9, cap=8192)
    u.prefill(K[:L0], V[:L0], e[:L0])
    r = u.step(K[L0], V[L0], float(e[L0]), q)
    s, E = r["scores"], u.E()
    nb = r["nb_c"]
    for chosen, score in ((r["gq"], s), (r["ge"], E[:nb])):
        rest = sorted(set(range(nb)) - set(chosen.tolist()))
        for a in chosen:
            for b in rest:
                assert _beats(score[a], a, score[b], b)
    # Gamma_q comes out in rank order
    for a, b in zip(r["gq"][:-1], r["gq"][1:]):
        assert _beats(s[a], a, s[b], b)


def test_locality_bound_is_tight_with_alternating_queries():
    """Gamma_e = blocks 0..5 (highest eviction scores); the query alternates
    between two orthogonal directions that each pick a different pair of
    blocks, so Sel(t) shares exactly the 6 Gamma_e blocks with S(t-1):
    gamma(t) = 6/8 = k_e/k, and exactly the 2 new Gamma_q blocks are fetched."""
    nb, D = 100, 128
    L0 = nb * 64 + 1
    K = np.zeros((L0, D), np.float32)
    for b in (10, 11):
        K[b * 64:(b + 1) * 64, 0] = 1.0
    for b in (20, 21):
        K[b * 64:(b + 1) * 64, 1] = 1.0
    e = np.zeros(L0, np.float32)
    for b, val in zip(range(6), [5.0, 4.0, 3.0, 2.0, 1.5, 1.0]):
        e[b * 64:(b + 1) * 64] = val
    Kb = cases.f32_to_bf16_bits_exact(K)
    u = OracleUnit(G=1, k_q=2, k_e=6, cap=8192)
    u.prefill(Kb, Kb, e)
    qa = np.zeros((1, D), np.float32); qa[0, 0] = 1.0
    qb = np.zeros((1, D), np.float32); qb[0, 1] = 1.0
    z = np.zeros(D, np.uint16)
    for t in range(12):
        q = cases.f32_to_bf16_bits_exact(qa if t % 2 == 0 else qb)
        r = u.step(z, z, 0.0, q)
        assert r["ge"].tolist() == [0, 1, 2, 3, 4, 5]
        assert r["gq"].tolist() == ([10, 11] if t % 2 == 0 else [20, 21])
        if t == 0:
            assert r["n_fetch"] == 2  # the prefill leaves Gamma_e and the local block resident
        else:
            assert r["n_overlap"] == 6 and r["gamma"] == 0.75 and r["n_fetch"] == 2
    assert u.violations()["gamma"] == 0


def test_incremental_eviction_sequence():
    """Blocks complete during decode with eviction scores 1, 3, 2 (prefill),
    then 2.5, 5, 0.5. With k_e = 2: {1,2} -> {1,3} -> {1,4} -> {1,4}; dropped
    blocks never return."""
    D = 128
    Es = [1.0, 3.0, 2.0, 2.5, 5.0, 0.5]
    L_all = 64 * len(Es) + 64
    e = np.zeros(L_all, np.float32)
    for b, val in enumerate(Es):
        e[b * 64:(b + 1) * 64] = val
    z = np.zeros((L_all, D), np.uint16)
    u = OracleUnit(G=1, k_q=0, k_e=2, cap=4096)
    L0 = 3 * 64 + 1
    u.prefill(z[:L0], z[:L0], e[:L0])
    q = np.zeros((1, D), np.uint16)
    expect = {3: [1, 2], 4: [1, 3], 5: [1, 4], 6: [1, 4]}
    seen = {}
    for p in range(L0, 64 * 6 + 1):
        r = u.step(z[p], z[p], float(e[p]), q)
        seen[r["nb_c"]] = r["ge"].tolist()
    assert seen == expect
    v = u.violations()
    assert v["reselect"] == 0 and v["incremental"] == 0


@pytest.mark.parametrize("G,k_q,k_e", [(1, 4, 12), (8, 16, 48)])
def test_invariants_over_many_steps(G, k_q, k_e):
    """Random drifting queries over 150 steps that cross block boundaries:
    gamma(t) >= k_e/k, no re-selection, incremental == brute-force Gamma_e,
    fetches only from fresh Gamma_q blocks."""
    L0, steps = 64 * 70 + 40, 150
    K, V, e = cases.synthetic_unit(5, 1, 0, 1, L0 + steps)
    qs = cases.synthetic_queries(5, 1, 0, 1, G, steps)
    u = OracleUnit(G=G, k_q=k_q, k_e=k_e, cap=8192)
    u.prefill(K[:L0], V[:L0], e[:L0])
    for t in range(steps):
        p = L0 + t
        r = u.step(K[p], V[p], float(e[p]), qs[t])
        if t >= 1:
            assert r["gamma"] >= k_e / (k_q + k_e)
            assert r["n_fetch"] <= k_q
    v = u.violations()
    assert v == {"gamma": 0, "reselect": 0, "incremental": 0, "fetch": 0, "steps": steps}


def test_first_token_and_tiny_context():
    """L = 1 after the append: no candidates, the output is the single value row."""
    K, V, e = cases.synthetic_unit(1, 0, 0, 0, 1)
    q = cases.synthetic_queries(1, 0, 0, 0, 2, 1)[0]
    u = OracleUnit(G=2, k_q=4, k_e=4, cap=128)
    r = u.step(K[0], V[0], float(e[0]), q)
    assert r["sel"].tolist() == [0] and r["nb_c"] == 0
    np.testing.assert_array_equal(r["o"], np.repeat(cases.bf16_bits_to_f64(V[0])[None], 2, 0))


def test_attend_blocks_matches_own_selection():
    L0 = 64 * 30 + 9
    K, V, e = cases.synthetic_unit(21, 0, 0, 0, L0 + 1)
    q = cases.synthetic_queries(21, 0, 0, 0, 2, 1)[0]
    u = OracleUnit(G=2, k_q=3, k_e=5, cap=4096)
    u.prefill(K[:L0], V[:L0], e[:L0])
    r = u.step(K[L0], V[L0], float(e[L0]), q)
    np.testing.assert_array_equal(u.attend_blocks(q, r["sel"]), r["o"])
    tok = np.concatenate([np.arange(b * 64, b * 64 + 64) for b in (2, 7)])
    want = cases.textbook_attention(q, K, V, e, tok, 1 / np.sqrt(128))
    np.testing.assert_allclose(u.attend_blocks(q, [2, 7]), want, rtol=1e-12, atol=1e-15)


def _bf16_neighbours(x):
    """The two bf16 values around x, found by walking the bf16 bit patterns (brute force)."""
    import struct
    f = np.float32(x)
    bits = int(np.frombuffer(struct.pack("<f", f), np.uint32)[0]) >> 16
    cands = []
    for b in range(bits - 2, bits + 3):
        v = np.frombuffer(struct.pack("<I", (b & 0xFFFF) << 16), np.float32)[0]
        if np.isfinite(v):
            cands.append((float(v), b & 0xFFFF))
    return cands


def test_bf16_rounding_is_nearest_ties_to_even():
    """The oracle's bf16 rounding of pooled keys against a brute-force nearest search."""
    import oracle
    rng = np.random.default_rng(0)
    xs = list(rng.normal(0, 0.05, 4000)) + list(rng.normal(0, 3, 1000))
    # exact midpoints between neighbouring bf16 values: ties must go to the even pattern
    xs += [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(0.5 + 2.0 ** -9), 0.0]
    for x in xs:
        got = oracle.round_bf16(x)
        cands = _bf16_neighbours(x)
        best = min(abs(v - x) for v, _ in cands)
        near = [(v, b) for v, b in cands if abs(v - x) == best]
        if len(near) > 1:
            near = [(v, b) for v, b in near if b % 2 == 0]
        assert got == near[0][0], (x, got, near)


def test_bf16_pooled_keys_are_rounded_means():
    """With bf16 pooled keys, each stored mean is the rounded fp64 mean (ramp keys: exact closed form)."""
    import oracle
    L, D = 16 * 5, 128
    j = np.arange(L)
    K = ((j % 16) / 16.0 + 0.01 * (j // 16))[:, None] * np.ones(D)[None, :]
    Kb = np.asarray(synth.bf16_to_f32(np.asarray([np.float32(v).view(np.uint32) >> 16 for v in K.ravel()],
                                                   np.uint16)), np.float32).reshape(L, D)
    Kbits = (Kb.view(np.uint32) >> 16).astype(np.uint16)
    u = OracleUnit(k_q=1, k_e=1, cap=4096, ck_bf16=True)
    u.prefill(Kbits, Kbits, np.zeros(L, np.float32))
    ck = u.ck()
    means = Kb.astype(np.float64).reshape(5, 16, D).mean(axis=1)
    want = np.vectorize(oracle.round_bf16)(means)
    assert np.array_equal(ck, want)
    assert not np.array_equal(ck, means)  # the rounding really happened


def _fixture_query(spec, qspec):
    s = dict(spec, q=qspec)
    return cases.build_fixture(s)[3]


@pytest.mark.parametrize("fill", [True, False])
def test_fill_golden_sequence(fill):
    """Fill reading, hand-derived over four steps: the remainder is filled from the not-yet-dropped
    blocks outside Gamma_q, a dropped block stays dropped, and Sel may hold fewer than k blocks.
    The union reading on the same input differs at the first step."""
    spec = cases.load_fixture("fill_sticky_drop.json")
    K, V, e, _ = cases.build_fixture(spec)
    u = OracleUnit(D=spec["D"], G=spec["G"], block=spec["block"], sub=spec["sub"], k_q=spec["k_q"],
                   k_e=spec["k_e"], cap=64 * 64, fill=fill)
    u.prefill(K, V, e)
    z = np.zeros(spec["D"], np.uint16)
    steps = spec["steps"] if fill else spec["steps"][:1]
    for i, st in enumerate(steps):
        r = u.step(z, z, 0.0, _fixture_query(spec, st["q"]))
        want = st if fill else spec["union_step1"]
        assert r["gq"].tolist() == st["expect_gq"], i
        assert r["ge"].tolist() == want["expect_ge"], i
        assert r["sel"].tolist() == want["expect_sel"], i
    v = u.violations()
    assert v["gamma"] == 0 and v["reselect"] == 0


def test_fill_with_no_query_budget_equals_union():
    """With k_q = 0 nothing is excluded by Gamma_q, so the fill and union readings coincide step by step."""
    L0, steps = 64 * 30 + 9, 140
    K, V, e = cases.synthetic_unit(5, 0, 0, 0, L0 + steps)
    Q = cases.synthetic_queries(5, 0, 0, 0, 2, steps)
    a = OracleUnit(G=2, k_q=0, k_e=7, cap=4096)
    b = OracleUnit(G=2, k_q=0, k_e=7, cap=4096, fill=True)
    a.prefill(K[:L0], V[:L0], e[:L0])
    b.prefill(K[:L0], V[:L0], e[:L0])
    for t in range(steps):
        ra = a.step(K[L0 + t], V[L0 + t], float(e[L0 + t]), Q[t])
        rb = b.step(K[L0 + t], V[L0 + t], float(e[L0 + t]), Q[t])
        assert np.array_equal(ra["sel"], rb["sel"]) and np.array_equal(ra["ge"], rb["ge"]), t
        assert np.array_equal(ra["o"], rb["o"])


@pytest.mark.parametrize("G,k_q,k_e", [(2, 4, 6), (1, 8, 3)])
def test_fill_rules_checked_from_history(G, k_q, k_e):
    """Fill reading, checked step by step against the selection history alone: Gamma_e is disjoint
    from Gamma_q, holds no block that some earlier step left unselected, is the best of the eligible
    blocks by E (ties to the lower id) and is as large as k_e allows; gamma(t) >= k_e/k holds."""
    L0, steps = 64 * 24 + 40, 400
    K, V, e = cases.synthetic_unit(9, 1, 0, 0, L0 + steps)
    Q = cases.synthetic_queries(9, 1, 0, 0, G, steps)
    u = OracleUnit(G=G, k_q=k_q, k_e=k_e, cap=4096, fill=True)
    u.prefill(K[:L0], V[:L0], e[:L0])
    dropped = set()
    shrank = 0
    for t in range(steps):
        r = u.step(K[L0 + t], V[L0 + t], float(e[L0 + t]), Q[t])
        E = u.E()
        nb_c = (u.length - 1) // 64
        gq, ge = set(r["gq"].tolist()), set(r["ge"].tolist())
        assert not (gq & ge)
        assert not (ge & dropped), t
        elig = [b for b in range(nb_c) if b not in gq and b not in dropped]
        assert len(ge) == min(k_e, len(elig))
        shrank += len(gq) + len(ge) < k_q + k_e
        worst = min(ge, key=lambda b: (E[b], -b)) if ge else None
        for b in elig:
            if b not in ge:
                assert (E[b], -b) < (E[worst], -worst), (t, b, worst)
        sel = set(r["sel"].tolist())
        dropped |= {b for b in range(nb_c) if b not in sel}
    v = u.violations()
    assert v["gamma"] == 0 and v["reselect"] == 0 and v["fetch"] == 0
    assert shrank > 0  # the case where Gamma_q takes eligible blocks and Sel holds fewer than k


def test_bf16_pooled_keys_barely_move_the_selection():
    """bf16 rounding of the pooled keys moves few Gamma_q blocks on the synthetic workload (a bound on
    how far the bf16 variant departs from fp32 storage, not a pin of either)."""
    swapped = total = 0
    L0, steps = 8192, 24
    for unit in range(2):
        K, V, e = cases.synthetic_unit(0, 0, unit, 0, L0 + steps)
        Q = cases.synthetic_queries(0, 0, unit, 0, 8, steps)
        a = OracleUnit(G=8, k_q=16, k_e=48, cap=16384)
        b = OracleUnit(G=8, k_q=16, k_e=48, cap=16384, ck_bf16=True)
        a.prefill(K[:L0], V[:L0], e[:L0])
        b.prefill(K[:L0], V[:L0], e[:L0])
        for t in range(steps):
            ra = a.step(K[L0 + t], V[L0 + t], float(e[L0 + t]), Q[t])
            rb = b.step(K[L0 + t], V[L0 + t], float(e[L0 + t]), Q[t])
            swapped += len(set(ra["gq"].tolist()) - set(rb["gq"].tolist()))
            total += len(ra["gq"])
    assert swapped <= 0.01 * total, (swapped, total)


def _bf16_bits(x):
    return (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_evict_head_zero_first_layer_gives_ln2_times_sum():
    """W1 = 0 makes every hidden pre-activation 0 and softplus(0) = ln 2, so e = ln 2 * sum(W2)."""
    import oracle
    _, W2 = synth.head_weights(3, 0, 1)
    V = synth.kv_rows(3, synth.V_STREAM, 0, 0, 0, 0, 5)
    e = oracle.evict_head(V, np.zeros((128, 128), np.float32), W2[0])
    want = np.float32(np.log(2.0) * np.sum(W2[0].astype(np.float64)))
    assert np.all(np.abs(e - want) <= np.spacing(np.abs(want)))


def test_evict_head_single_path_and_orientation():
    """One nonzero W1 entry (row d0, column h0) and W2 = c at h0 only: e_j = c * log(1 + exp(a v_j[d0])).
    A transposed W1 (row h0, column d0) would read a different input dimension."""
    import oracle
    d0, h0, a, c = 5, 77, 3.0, 0.75
    W1 = np.zeros((128, 128), np.float32)
    W1[d0, h0] = a
    W2 = np.zeros(128, np.float32)
    W2[h0] = c
    V = synth.kv_rows(4, synth.V_STREAM, 0, 0, 0, 0, 64)
    vf = synth.bf16_to_f32(V).astype(np.float64)
    want = (c * np.log(1.0 + np.exp(a * vf[:, d0]))).astype(np.float32)
    got = oracle.evict_head(V, W1, W2)
    assert np.all(np.abs(got - want) <= np.spacing(np.abs(want)))
    assert not np.allclose(got, (c * np.log(1.0 + np.exp(a * vf[:, h0]))).astype(np.float32))


def test_evict_head_softplus_extremes():
    """softplus(800) = 800 (a plain log(1+exp) overflows) and softplus(-40) = exp(-40) to within
    1e-17 relative (a plain log(1+exp) gives 0)."""
    import oracle
    W1 = np.zeros((128, 128), np.float32)
    W1[0, 0], W1[0, 1] = 800.0, -40.0
    V = np.zeros((1, 128), np.uint16)
    V[0, 0] = _bf16_bits(1.0)
    for h, want in ((0, 800.0), (1, np.exp(-40.0))):
        W2 = np.zeros(128, np.float32)
        W2[h] = 1.0
        got = oracle.evict_head(V, W1, W2)[0]
        assert got == np.float32(want), (h, got, want)


def test_evict_head_matches_numpy_logaddexp():
    """The head on seeded inputs against NumPy's fp64 matmul and logaddexp(0, z) = softplus(z):
    equal to within one fp32 unit in the last place (the two sum in different orders)."""
    import oracle
    W1, W2 = synth.head_weights(7, 2, 2)
    V = synth.kv_rows(7, synth.V_STREAM, 2, 1, 1, 0, 300)
    vf = synth.bf16_to_f32(V).astype(np.float64)
    for g in range(2):
        want = np.logaddexp(0.0, vf @ W1[g].astype(np.float64)) @ W2[g].astype(np.float64)
        got = oracle.evict_head(V, W1[g], W2[g])
        assert np.all(np.abs(got.astype(np.float64) - want) <= np.spacing(np.abs(want).astype(np.float32))), g
    assert got.std() > 0.2  # the synthetic head is not degenerate


def test_evict_head_is_linear_in_second_layer():
    import oracle
    W1, W2 = synth.head_weights(8, 0, 2)
    V = synth.kv_rows(8, synth.V_STREAM, 0, 0, 0, 0, 50)
    a = oracle.evict_head(V, W1[0], W2[0]).astype(np.float64)
    b = oracle.evict_head(V, W1[0], W2[1]).astype(np.float64)
    ab = oracle.evict_head(V, W1[0], W2[0] + W2[1]).astype(np.float64)
    assert np.allclose(ab, a + b, rtol=0, atol=4e-6)
