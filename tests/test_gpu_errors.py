"""Error paths on the GPU: device conditions set bits in the state's error word
and leave the state consistent (no fault, no hang); argument checks refuse
bad calls before any launch; a bounded device wait that runs out reports
NOSA_EFLAG_TIMEOUT and the context stays usable."""
import numpy as np
import pytest
import torch

import block_sparse_offloadable_b200 as nosa
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def _rows(n, seed=0):
    g = torch.Generator().manual_seed(seed)
    k = (torch.randn((n, 128), generator=g) / 11.3).to(torch.bfloat16).view(torch.int16)
    return k.cuda()


def _full_layer(fused):
    """A unit pair filled to max_ctx = 128 tokens by a prefill."""
    cfg = nosa.make_config(1, 8, 2, 2, 2, 128)
    lay = nosa.NosaLayer(cfg)
    T = 128
    k = _rows(2 * T, 1).view(2, T, 128)
    v = _rows(2 * T, 2).view(2, T, 128)
    e = torch.zeros((2, T), dtype=torch.float32, device="cuda")
    lay.append(k, v, e, T)
    torch.cuda.synchronize()
    assert lay.read_error() == 0
    return cfg, lay


@pytest.mark.parametrize("fused", [False, True, "step"])
def test_append_past_capacity_sets_the_flag_and_keeps_the_state(fused):
    # separate launches, append + select in one launch, and the whole step in one launch
    cfg, lay = _full_layer(fused)
    kn, vn = _rows(2, 3).view(2, 1, 128), _rows(2, 4).view(2, 1, 128)
    en = torch.zeros((2, 1), dtype=torch.float32, device="cuda")
    q = _rows(8, 5).view(1, 8, 128)
    out = torch.empty((1, 8, 128), dtype=torch.int16, device="cuda")
    if fused == "step":
        lay.fused_step(kn, vn, en, q, out)
    elif fused:
        lay.append_select(kn, vn, en, q)
    else:
        lay.append(kn, vn, en, 1)
        lay.select(q)
    if fused != "step":
        lay.sparse_decode(q, out)
    torch.cuda.synchronize()
    assert lay.read_error(clear=False) & nosa.EFLAG_CAPACITY
    assert lay.seq_len.cpu().tolist() == [128, 128]  # nothing appended
    assert lay.read_error(clear=True) & nosa.EFLAG_CAPACITY
    assert lay.read_error() == 0  # cleared
    assert torch.isfinite(out.view(torch.bfloat16).float()).all()


def test_prefill_into_a_nonempty_unit_sets_the_state_flag():
    cfg, lay = _full_layer(False)
    lay2_k = _rows(2 * 64, 6).view(2, 64, 128)
    e = torch.zeros((2, 64), dtype=torch.float32, device="cuda")
    lay.append(lay2_k, lay2_k, e, 64)
    torch.cuda.synchronize()
    assert lay.read_error() & nosa.EFLAG_STATE
    assert lay.seq_len.cpu().tolist() == [128, 128]


def test_argument_checks_refuse_before_any_launch():
    cfg = nosa.make_config(2, 16, 2, 4, 12, 4096)
    lay = nosa.NosaLayer(cfg)
    q = torch.zeros((2, 16, 128), dtype=torch.int16, device="cuda")
    out = torch.empty_like(q)
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    need = nosa.nosa_workspace_bytes(cfg, nosa.WS_SPARSE_DECODE)
    assert need > 16
    with pytest.raises(nosa.NosaError) as ei:
        nosa.nosa_sparse_decode(cfg, lay.state, q, lay.sel, lay.nsel, None, out, small)
    assert ei.value.code == nosa.ERR_CAPACITY
    with pytest.raises(nosa.NosaError) as ei:
        nosa.nosa_select(cfg, lay.state, q, None, lay.nsel, lay.gq, lay.ws_select)
    assert ei.value.code == nosa.ERR_PTR
    host_q = torch.zeros((2, 16, 128), dtype=torch.int16)  # host memory, not device
    with pytest.raises(nosa.NosaError) as ei:
        nosa.nosa_select(cfg, lay.state, host_q, lay.sel, lay.nsel, lay.gq, lay.ws_select)
    assert ei.value.code == nosa.ERR_PTR
    k = torch.zeros((4, 1, 128), dtype=torch.int16, device="cuda")
    e = torch.zeros((4, 1), dtype=torch.float32, device="cuda")
    with pytest.raises(nosa.NosaError) as ei:  # per-sequence lengths are for a prefill only
        nosa.nosa_compress_append(cfg, lay.state, k, k, e, 1, torch.ones(2, dtype=torch.int32, device="cuda"))
    assert ei.value.code == nosa.ERR_ARG
    with pytest.raises(nosa.NosaError) as ei:
        nosa.nosa_compress_append(cfg, lay.state, k, k, e, 8192)
    assert ei.value.code == nosa.ERR_CAPACITY
    torch.cuda.synchronize()
    assert lay.read_error() == 0 and lay.seq_len.cpu().tolist() == [0, 0, 0, 0]


def test_mode_restrictions():
    off = nosa.make_config(1, 8, 2, 4, 4, 1024, offload=True)
    lay = nosa.NosaLayer(off)
    q = torch.zeros((1, 8, 128), dtype=torch.int16, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(nosa.NosaError) as ei:  # the dense comparator needs the KV store on the device
        lay.dense_decode(q, out)
    assert ei.value.code == nosa.ERR_ARG
    fill = nosa.make_config(1, 8, 2, 4, 4, 1024, fill=True)
    lf = nosa.NosaLayer(fill)
    split = torch.zeros(nosa.nosa_workspace_bytes(fill, nosa.WS_SPLIT), dtype=torch.uint8, device="cuda")
    with pytest.raises(nosa.NosaError) as ei:  # the split decode needs Gamma_e before the select
        nosa.nosa_decode_resident(fill, lf.state, q, split, lf.ws_decode)
    assert ei.value.code == nosa.ERR_UNSUPPORTED
    pageable = torch.zeros(nosa.nosa_state_bytes(off, nosa.BUF_KV_STORE), dtype=torch.uint8)
    with pytest.raises(AssertionError):  # the binding insists on pinned memory; the library checks too
        nosa.NosaLayer(off, host_store=pageable)


def test_bounded_wait_reports_timeout_and_the_context_stays_usable():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    nosa.nosa_check_wait_timeout(err, 1 << 22)  # ~2 ms at the B200's clock
    torch.cuda.synchronize()
    assert int(err.item()) == nosa.EFLAG_TIMEOUT
    # the context still runs the path correctly afterwards
    sc = H.Scenario(B=1, Hq=8, Hkv=2, k_q=4, k_e=4, L0=64 * 8 + 3, steps=4, seed=2, fused=True)
    data = H.unit_data(sc)
    gpu = H.run_gpu(sc, data)
    assert gpu["err"] == 0
    H.assert_parity(H.compare(sc, data, gpu))
