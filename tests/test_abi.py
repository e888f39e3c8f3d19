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


def test_workspace_sizes_cover_chunks(L):
    for c in (cfg(), cfg(batch=64, max_ctx=131072 + 256)):
        for which in (nosa.WS_SELECT, nosa.WS_SPARSE_DECODE, nosa.WS_DENSE_DECODE):
            n = nosa.nosa_workspace_bytes(c, which)
            assert n == 0 or n >= 256


def test_strerror(L):
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -99):
        assert isinstance(L.nosa_strerror(code), bytes)
