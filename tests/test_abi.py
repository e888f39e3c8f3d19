"""Host-only checks of the C ABI: the library loads, exports every symbol the
header declares, and its pure host functions (configuration validation,
buffer and workspace sizes, error strings) behave.  No kernel is launched."""
import ctypes
import os
import re

import pytest

import block_sparse_offloadable_b200 as nosa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    nosa.build()
    return nosa.lib()


def test_exports_every_declared_symbol(L):
    hdr = open(os.path.join(ROOT, "include", "nosa.h")).read()
    declared = set(re.findall(r"^\s*(?:int|size_t|const char \*)\s*(nosa_\w+)\s*\(", hdr, re.M))
    assert declared == set(nosa.EXPORTS)
    for name in declared:
        assert getattr(L, name) is not None


def cfg(**kw):
    base = dict(batch=2, heads_q=16, heads_kv=2, k_q=16, k_e=48, max_ctx=8192, offload=False)
    base.update(kw)
    return nosa.make_config(**base)


def test_validate_config(L):
    assert nosa.nosa_validate_config(cfg()) == nosa.OK
    assert nosa.nosa_validate_config(cfg(max_ctx=8190)) == nosa.ERR_ARG
    assert nosa.nosa_validate_config(cfg(heads_q=15)) == nosa.ERR_ARG
    assert nosa.nosa_validate_config(cfg(heads_q=32, heads_kv=2)) == nosa.ERR_UNSUPPORTED  # G = 16
    assert nosa.nosa_validate_config(cfg(k_q=33)) == nosa.ERR_UNSUPPORTED
    assert nosa.nosa_validate_config(cfg(k_q=0, k_e=0)) == nosa.ERR_ARG
    assert nosa.nosa_validate_config(cfg(head_dim=64)) == nosa.ERR_UNSUPPORTED
    assert nosa.nosa_validate_config(cfg(max_ctx=1 << 21)) == nosa.ERR_CAPACITY
    assert nosa.nosa_validate_config(cfg(batch=1024, max_ctx=1 << 20)) == nosa.ERR_CAPACITY
    assert nosa.nosa_validate_config(cfg(ck_bf16=True)) == nosa.OK
    assert nosa.nosa_validate_config(cfg(ck_bf16=True, fill=True)) == nosa.OK
    bad = cfg()
    bad.flags = 4  # an undefined flag bit
    assert nosa.nosa_validate_config(bad) == nosa.ERR_ARG


def test_state_sizes(L):
    c = cfg()
    u, nblk = 4, 8192 // 64
    assert nosa.nosa_state_bytes(c, nosa.BUF_KV_STORE) == u * nblk * 32768
    assert nosa.nosa_state_bytes(c, nosa.BUF_CK) == u * (8192 // 16) * 128 * 4
    assert nosa.nosa_state_bytes(c, nosa.BUF_BLK_EVICT) == u * nblk * 8
    assert nosa.nosa_state_bytes(c, nosa.BUF_GAMMA_E) == u * 48 * 4
    assert nosa.nosa_state_bytes(c, nosa.BUF_CACHE) == 0
    co = cfg(offload=True)
    assert nosa.nosa_state_bytes(co, nosa.BUF_CACHE) == u * (16 + 48 + 2) * 32768
    assert nosa.nosa_state_bytes(co, nosa.BUF_BLOCK_SLOT) == u * nblk * 4
    assert nosa.nosa_state_bytes(cfg(max_ctx=100), nosa.BUF_CK) == 0  # invalid config
    assert nosa.nosa_state_bytes(cfg(ck_bf16=True), nosa.BUF_CK) == u * (8192 // 16) * 128 * 2
    assert nosa.nosa_state_bytes(c, nosa.BUF_POOL) == 0 and nosa.nosa_state_bytes(c, nosa.BUF_POOL_N) == 0
    assert nosa.nosa_state_bytes(cfg(fill=True), nosa.BUF_POOL) == u * nblk * 4
    assert nosa.nosa_state_bytes(cfg(fill=True), nosa.BUF_POOL_N) == u * 4


def _align256(x):
    return (x + 255) // 256 * 256


def _select_chunks(units, nblk, bf16, sms=148, ctas_per_sm=3, stage_blocks=8, max_chunks=64):
    # The select launcher's documented chunk model: n chunks per unit minimise the wave-quantised
    # streaming time plus the depth of the finalizing CTA's merge tree (ceil(n/4) + 1 levels); the
    # chunk length is then rounded up to whole stages.
    work = nblk - 1 if nblk > 1 else 1
    nmax = max(1, min((work + stage_blocks - 1) // stage_blocks, max_chunks))
    ovh, merge = (64, 4) if bf16 else (32, 2)
    slots = sms * ctas_per_sm
    best = min(range(1, nmax + 1),
               key=lambda n: (((units * n + slots - 1) // slots) * ((work + n - 1) // n + ovh)
                              + merge * ((n + 3) // 4 + 1), n))
    per = (work + best - 1) // best
    per = (per + stage_blocks - 1) // stage_blocks * stage_blocks
    return max(1, (nblk - 1 + per - 1) // per)


@pytest.mark.parametrize("bf16", [False, True])
def test_workspace_sizes_follow_the_launch_geometry(L, bf16):
    # select: per-unit counters + one 32-key list per chunk; decode: per-unit counters + two partial
    # states (m[8], l[8], o[8][128] fp32) per decode CTA (one per SM)
    checked = 0
    for batch in (1, 8, 32, 64, 256):
        for heads_kv in (1, 2, 8):
            for ctx in (4096, 16384, 65536, 131072, 1 << 20):
                units = batch * heads_kv
                if units > 2048:
                    continue
                c = cfg(batch=batch, heads_q=heads_kv * 2, heads_kv=heads_kv, max_ctx=ctx, ck_bf16=bf16)
                if nosa.nosa_validate_config(c) != nosa.OK:  # beyond the library's index limits
                    assert nosa.nosa_workspace_bytes(c, nosa.WS_SELECT) == 0
                    continue
                checked += 1
                n = _select_chunks(units, ctx // 64, bf16)
                want = _align256(units * 4) + units * n * 32 * 8 if n > 1 else 0
                assert nosa.nosa_workspace_bytes(c, nosa.WS_SELECT) == want, (batch, heads_kv, ctx, n)
                dec = _align256(units * 4) + 148 * 2 * (2 * 8 + 8 * 128) * 4
                assert nosa.nosa_workspace_bytes(c, nosa.WS_SPARSE_DECODE) == dec
                assert nosa.nosa_workspace_bytes(c, nosa.WS_DENSE_DECODE) == dec
    assert checked >= 70


def test_strerror(L):
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -99):
        assert isinstance(L.nosa_strerror(code), bytes)


def _team(units, max_sel, sms=148):
    return 1 if units > sms else min(sms // units, max_sel)


@pytest.mark.parametrize("bf16", [False, True])
def test_fused_step_workspace(L, bf16):
    # per unit: two counters and two flags; per CTA (units x team size): a 32-key list and a partial
    # state; per unit: k_q slots of Gamma_q outside Gamma_e
    for batch, heads_kv, k_q, k_e in ((1, 1, 16, 48), (8, 2, 16, 48), (32, 2, 16, 48), (80, 2, 8, 24),
                                      (2, 2, 32, 256), (4, 4, 0, 16)):
        c = cfg(batch=batch, heads_q=heads_kv * 4, heads_kv=heads_kv, k_q=k_q, k_e=k_e, ck_bf16=bf16)
        units, max_sel = batch * heads_kv, k_q + k_e + 1
        ctas = units * _team(units, max_sel)
        want = (_align256(units * 16) + _align256(ctas * 32 * 8) + _align256(ctas * (2 * 8 + 8 * 128) * 4) +
                units * max(k_q, 1) * 4)
        assert nosa.nosa_workspace_bytes(c, nosa.WS_FUSED_STEP) == want, (batch, heads_kv)
    # not built for the offload store or the fill reading
    assert nosa.nosa_workspace_bytes(cfg(offload=True), nosa.WS_FUSED_STEP) == 0
    assert nosa.nosa_workspace_bytes(cfg(fill=True), nosa.WS_FUSED_STEP) == 0


def test_fused_step_refuses_before_any_launch(L):
    st = nosa.State()
    P = ctypes.c_void_p

    def call(c, e_new):
        return L.nosa_fused_step(ctypes.byref(c), ctypes.byref(st), P(16), P(16), e_new, P(16), P(16), P(16), None,
                                 P(16), None, 0, None)

    assert call(cfg(offload=True), P(16)) == nosa.ERR_UNSUPPORTED
    assert call(cfg(fill=True), P(16)) == nosa.ERR_UNSUPPORTED
    assert call(cfg(), None) == nosa.ERR_ARG
    assert call(cfg(), P(16)) == nosa.ERR_PTR  # the state's buffers are missing
    bad = cfg()
    bad.k_q = 33
    assert call(bad, P(16)) == nosa.ERR_UNSUPPORTED
