"""The device-side generator writes the same bytes as the host-side one."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def test_kv_e_q_bytes_match_host():
    B, Hkv, Hq, p0, T = 2, 3, 6, 1000, 77
    k = torch.empty((B * Hkv, T, 128), dtype=torch.int16, device="cuda")
    v = torch.empty_like(k)
    e = torch.empty((B * Hkv, T), dtype=torch.float32, device="cuda")
    synth.kv_dev(9, synth.K_STREAM, 4, B, Hkv, p0, T, k, seq0=0)
    synth.kv_dev(9, synth.V_STREAM, 4, B, Hkv, p0, T, v)
    synth.e_dev(9, 4, B, Hkv, p0, T, e)
    state = torch.zeros((B * Hq, 128), dtype=torch.float32, device="cuda")
    q = torch.empty((B * Hq, 128), dtype=torch.int16, device="cuda")
    qs = []
    for t in range(5):
        synth.q_dev(9, 4, B, Hq, t, state, q)
        qs.append(q.cpu().numpy().view(np.uint16).copy())
    torch.cuda.synchronize()
    kh, vh, eh = k.cpu().numpy().view(np.uint16), v.cpu().numpy().view(np.uint16), e.cpu().numpy()
    for u in range(B * Hkv):
        b, g = divmod(u, Hkv)
        assert np.array_equal(kh[u], synth.kv_rows(9, synth.K_STREAM, 4, b, g, p0, T))
        assert np.array_equal(vh[u], synth.kv_rows(9, synth.V_STREAM, 4, b, g, p0, T))
        assert np.array_equal(eh[u].view(np.uint32), synth.e_rows(9, 4, b, g, p0, T).view(np.uint32))
    for r in range(B * Hq):
        b, h = divmod(r, Hq)
        want = synth.q_steps(9, 4, b, h, 5)[1]
        for t in range(5):
            assert np.array_equal(qs[t][r], want[t])


def test_sequence_offset_addresses_the_same_rows():
    """Generating sequences 3..4 directly equals rows 3..4 of a batch generated from 0."""
    Hkv, T = 2, 40
    full = torch.empty((6 * Hkv, T, 128), dtype=torch.int16, device="cuda")
    part = torch.empty((2 * Hkv, T, 128), dtype=torch.int16, device="cuda")
    synth.kv_dev(5, synth.V_STREAM, 1, 6, Hkv, 17, T, full)
    synth.kv_dev(5, synth.V_STREAM, 1, 2, Hkv, 17, T, part, seq0=3)
    assert torch.equal(full[3 * Hkv:5 * Hkv], part)
    ef = torch.empty((6 * Hkv, T), dtype=torch.float32, device="cuda")
    ep = torch.empty((2 * Hkv, T), dtype=torch.float32, device="cuda")
    synth.e_dev(5, 1, 6, Hkv, 17, T, ef)
    synth.e_dev(5, 1, 2, Hkv, 17, T, ep, seq0=3)
    assert torch.equal(ef[3 * Hkv:5 * Hkv], ep)
    Hq = 4
    sf = torch.zeros((6 * Hq, 128), dtype=torch.float32, device="cuda")
    sp = torch.zeros((2 * Hq, 128), dtype=torch.float32, device="cuda")
    qf = torch.empty((6 * Hq, 128), dtype=torch.int16, device="cuda")
    qp = torch.empty((2 * Hq, 128), dtype=torch.int16, device="cuda")
    for t in range(3):
        synth.q_dev(5, 1, 6, Hq, t, sf, qf)
        synth.q_dev(5, 1, 2, Hq, t, sp, qp, seq0=3)
        assert torch.equal(qf[3 * Hq:5 * Hq], qp)
