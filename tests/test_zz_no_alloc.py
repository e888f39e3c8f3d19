"""nosa_select_noalloc: the select step for callers that cannot allocate device
memory (its scratch is a fixed array inside the library).  Its results must be
the same as nosa_select's with a caller-provided workspace, on two calls in a
row (the second call finds the first call's leftovers in the shared array).

Kept in its own file, collected last, so that a failure here comes after every
other test has run.  Must pass alone in a fresh process and after the others."""
import numpy as np
import pytest
import torch

import block_sparse_offloadable_b200 as nosa
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,Hq,Hkv,k_q,k_e,L0", [(4, 16, 2, 16, 48, 64 * 300 + 17), (2, 8, 8, 8, 24, 64 * 90 + 63)])
def test_noalloc_select_matches_workspace_select(B, Hq, Hkv, k_q, k_e, L0):
    sc = H.Scenario(B=B, Hq=Hq, Hkv=Hkv, k_q=k_q, k_e=k_e, L0=L0, steps=2, seed=31)
    cfg = sc.cfg()
    need = nosa.nosa_workspace_bytes(cfg, nosa.WS_SELECT)
    assert 0 < need <= nosa.NOALLOC_SELECT_SCRATCH  # the case really uses scratch
    K, V, E, Q = H.unit_data(sc)
    lay = nosa.NosaLayer(cfg)
    lay.append(H._dev16(K[:, :L0]), H._dev16(V[:, :L0]), torch.from_numpy(np.ascontiguousarray(E[:, :L0])).cuda(), L0)
    sel2 = torch.full_like(lay.sel, -7)
    nsel2 = torch.full_like(lay.nsel, -7)
    gq2 = torch.full_like(lay.gq, -7)
    for t in range(2):
        idx = np.arange(sc.units)
        lay.append(H._dev16(K[idx, L0 + t][:, None, :]), H._dev16(V[idx, L0 + t][:, None, :]),
                   torch.from_numpy(np.ascontiguousarray(E[idx, L0 + t][:, None])).cuda(), 1)
        q = H._dev16(Q[t])
        lay.select(q)  # the existing entry point, workspace from the caller
        for rep in range(3):  # two calls in a row on the shared scratch array, then one after a poisoning
            if rep == 2:
                # stale counters and lists, as an interrupted call could leave them: the call must
                # clear what has to start at zero
                nosa.nosa_noalloc_scratch_poison(0x5A)
            sel2.fill_(-7), nsel2.fill_(-7), gq2.fill_(-7)
            nosa.nosa_select_noalloc(cfg, lay.state, q, sel2, nsel2, gq2)
            torch.cuda.synchronize()
            assert torch.equal(nsel2, lay.nsel)
            assert torch.equal(sel2, lay.sel)
            assert torch.equal(gq2, lay.gq)
    assert lay.read_error() == 0


def test_noalloc_rejects_oversize_workspace():
    # 2048 (sequence, kv head) units at 128K context need more select scratch than the
    # fixed array holds; the call is refused before anything is touched or launched
    cfg = nosa.make_config(1024, 16, 2, 16, 48, 131072)
    assert nosa.nosa_validate_config(cfg) == nosa.OK
    assert nosa.nosa_workspace_bytes(cfg, nosa.WS_SELECT) > nosa.NOALLOC_SELECT_SCRATCH
    q = torch.zeros(16, dtype=torch.int16, device="cuda")
    sel = torch.zeros(16, dtype=torch.int32, device="cuda")
    nsel = torch.zeros(16, dtype=torch.int32, device="cuda")
    st = nosa.State()
    with pytest.raises(nosa.NosaError) as ei:
        nosa.nosa_select_noalloc(cfg, st, q, sel, nsel)
    assert ei.value.code == nosa.ERR_CAPACITY


def _captured_nodes(fn):
    """Number of graph nodes that fn() enqueues on a capturing stream (fn's exception is kept)."""
    import ctypes
    g = torch.cuda.CUDAGraph(keep_graph=True)  # the raw graph is kept for inspection, never instantiated
    s = torch.cuda.Stream()
    raised = None
    with torch.cuda.stream(s):
        g.capture_begin(capture_error_mode="thread_local")
        try:
            fn(s)
        except nosa.NosaError as e:
            raised = e
        g.capture_end()
    drv = ctypes.CDLL("libcuda.so.1")
    n = ctypes.c_size_t(0)
    assert drv.cuGraphGetNodes(ctypes.c_void_p(g.raw_cuda_graph()), None, ctypes.byref(n)) == 0
    del g
    return n.value, raised


@pytest.mark.filterwarnings("ignore:The CUDA Graph is empty")  # the refused call's capture is empty by design
def test_noalloc_refused_call_queues_nothing():
    # a missing output pointer is refused with NOSA_ERR_PTR by the checks that precede any work:
    # the call enqueues no node on the (capturing) stream, in particular no clearing of the shared
    # counters; a valid call captured the same way enqueues the clear and the kernel
    sc = H.Scenario(B=4, Hq=16, Hkv=2, k_q=16, k_e=48, L0=64 * 300 + 17, steps=1, seed=32)
    cfg = sc.cfg()
    assert nosa.nosa_workspace_bytes(cfg, nosa.WS_SELECT) > 0
    lay = nosa.NosaLayer(cfg)
    q = torch.zeros((sc.B, sc.Hq, 128), dtype=torch.int16, device="cuda")
    nosa.nosa_noalloc_scratch_poison(0x33)  # the array's address is resolved before any capture
    torch.cuda.synchronize()
    n_bad, err = _captured_nodes(lambda s: nosa.nosa_select_noalloc(cfg, lay.state, q, None, lay.nsel,
                                                                      lay.gq, stream=s))
    assert err is not None and err.code == nosa.ERR_PTR
    assert n_bad == 0
    n_ok, err = _captured_nodes(lambda s: nosa.nosa_select_noalloc(cfg, lay.state, q, lay.sel, lay.nsel,
                                                                     lay.gq, stream=s))
    assert err is None and n_ok >= 2  # the counter clear and the select kernel
    # and the next call, run for real on an empty state, leaves no error
    nosa.nosa_select_noalloc(cfg, lay.state, q, lay.sel, lay.nsel, lay.gq)
    torch.cuda.synchronize()
    assert int(lay.nsel.sum()) == 0 and lay.read_error() == 0
