"""Python binding of libnosa: the NOSA block-sparse, KV-offloadable decode path on B200.

The functions below carry the C entry points' names (``include/nosa.h``) and
only marshal arguments: torch tensors become raw pointers, the current CUDA
stream becomes the stream argument.  Every step of the path runs in the CUDA
kernels of ``_lib/libnosa.so``; there is no CPU fallback, and importing the
binding on a machine where the library is missing raises.

``NosaLayer`` is a convenience owner of one layer's caller-side buffers (the
library allocates nothing): device state, the KV store (device memory, or
pinned host memory in offload mode), per-step outputs and workspaces.
"""
import ctypes
import os
import subprocess

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_HERE)
LIB_PATH = os.path.join(_HERE, "_lib", "libnosa.so")
_SOURCES = ["nosa_api.cu", "nosa_append.cu", "nosa_select.cu", "nosa_cache.cu", "nosa_decode.cu", "nosa_step.cu",
            "nosa_noalloc.cu", "nosa_diag.cu"]
_HEADERS = ["nosa_common.cuh", "nosa_internal.cuh", "nosa_append_unit.cuh", "nosa_attend.cuh"]
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared"]

OK, ERR_ARG, ERR_CAPACITY, ERR_PTR, ERR_CUDA, ERR_TIMEOUT, ERR_UNSUPPORTED, ERR_DEVICE = 0, -1, -2, -3, -4, -5, -6, -7
EFLAG_CAPACITY, EFLAG_TIMEOUT, EFLAG_NOSLOT, EFLAG_STATE = 1, 2, 4, 8
FLAG_CK_BF16, FLAG_FILL = 1, 2
(BUF_KV_STORE, BUF_EVICT_LOGIT, BUF_CK, BUF_BLK_EVICT, BUF_GAMMA_E, BUF_GAMMA_N, BUF_SEQ_LEN, BUF_CACHE,
 BUF_SLOT_BLOCK, BUF_BLOCK_SLOT, BUF_ERR, BUF_POOL, BUF_POOL_N) = range(13)
WS_SELECT, WS_SPARSE_DECODE, WS_DENSE_DECODE, WS_CACHE_SYNC, WS_SPLIT, WS_FUSED_STEP = 0, 1, 2, 3, 4, 5

# Every extern "C" symbol include/nosa.h declares.
EXPORTS = ["nosa_validate_config", "nosa_state_bytes", "nosa_workspace_bytes", "nosa_state_init",
           "nosa_compress_append", "nosa_compress_append_head", "nosa_select", "nosa_append_select", "nosa_cache_sync", "nosa_sparse_decode",
           "nosa_dense_decode", "nosa_decode_resident", "nosa_decode_rest", "nosa_read_error", "nosa_strerror",
           "nosa_select_noalloc", "nosa_noalloc_scratch_poison", "nosa_check_wait_timeout", "nosa_fused_step"]
NOALLOC_SELECT_SCRATCH = 1 << 20


def build(force=False, verbose=False):
    """Compile libnosa for sm_100a in-tree (nvcc cross-compiles without a GPU)."""
    out = LIB_PATH
    srcs = [os.path.join(_HERE, "csrc", s) for s in _SOURCES]
    deps = srcs + [os.path.join(_HERE, "csrc", h) for h in _HEADERS] + [os.path.join(_ROOT, "include", "nosa.h")]
    if not force and os.path.exists(out) and all(os.path.getmtime(d) <= os.path.getmtime(out) for d in deps):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    cmd = ["nvcc", *NVCC_FLAGS, "-I" + os.path.join(_ROOT, "include"), "-o", out, *srcs]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    return out


class Config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads_q", ctypes.c_int32), ("heads_kv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block", ctypes.c_int32), ("sub_block", ctypes.c_int32),
                ("k_q", ctypes.c_int32), ("k_e", ctypes.c_int32), ("local_blocks", ctypes.c_int32),
                ("offload", ctypes.c_int32), ("max_ctx", ctypes.c_int64), ("scale", ctypes.c_float),
                ("flags", ctypes.c_int32)]


class State(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ["kv_store", "evict_logit", "ck", "blk_evict", "gamma_e", "gamma_n",
                                              "seq_len", "cache", "slot_block", "block_slot", "err", "pool",
                                              "pool_n"]]


_lib = None


def lib():
    """Load libnosa.so; raise if it is missing (there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libnosa is not built ({LIB_PATH}); run block_sparse_offloadable_b200.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, C, S = ctypes.c_void_p, ctypes.POINTER(Config), ctypes.POINTER(State)
        L.nosa_validate_config.argtypes = [C]
        L.nosa_state_bytes.argtypes = [C, ctypes.c_int]
        L.nosa_state_bytes.restype = ctypes.c_size_t
        L.nosa_workspace_bytes.argtypes = [C, ctypes.c_int]
        L.nosa_workspace_bytes.restype = ctypes.c_size_t
        L.nosa_state_init.argtypes = [C, S, P]
        L.nosa_compress_append.argtypes = [C, S, P, P, P, ctypes.c_int32, P, P]
        L.nosa_compress_append_head.argtypes = [C, S, P, P, P, P, ctypes.c_int32, P, P]
        L.nosa_select.argtypes = [C, S, P, P, P, P, P, ctypes.c_size_t, P]
        L.nosa_cache_sync.argtypes = [C, S, P, P, P, P, P, ctypes.c_size_t, P]
        L.nosa_sparse_decode.argtypes = [C, S, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.nosa_append_select.argtypes = [C, S, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.nosa_fused_step.argtypes = [C, S, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.nosa_decode_resident.argtypes = [C, S, P, P, ctypes.c_size_t, P, ctypes.c_size_t, P]
        L.nosa_decode_rest.argtypes = [C, S, P, P, P, ctypes.c_size_t, P, P, ctypes.c_size_t, P]
        L.nosa_dense_decode.argtypes = [C, S, P, P, P, ctypes.c_size_t, P]
        L.nosa_read_error.argtypes = [S, ctypes.POINTER(ctypes.c_uint32), ctypes.c_int, P]
        L.nosa_check_wait_timeout.argtypes = [P, ctypes.c_int64, P]
        L.nosa_select_noalloc.argtypes = [C, S, P, P, P, P, P]
        L.nosa_noalloc_scratch_poison.argtypes = [ctypes.c_uint8, P]
        L.nosa_strerror.argtypes = [ctypes.c_int]
        L.nosa_strerror.restype = ctypes.c_char_p
        _lib = L
    return _lib


class NosaError(RuntimeError):
    def __init__(self, code, what):
        super().__init__(f"{what}: {lib().nosa_strerror(code).decode()} ({code})")
        self.code = code


def _check(code, what):
    if code != OK:
        raise NosaError(code, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_config(batch, heads_q, heads_kv, k_q, k_e, max_ctx, offload=False, head_dim=128, block=64, sub_block=16,
                scale=None, ck_bf16=False, fill=False):
    return Config(batch, heads_q, heads_kv, head_dim, block, sub_block, k_q, k_e, 1, int(bool(offload)),
                  int(max_ctx), float(scale if scale is not None else head_dim ** -0.5),
                  (FLAG_CK_BF16 if ck_bf16 else 0) | (FLAG_FILL if fill else 0))


# ---- the C entry points, one to one -------------------------------------------------

def nosa_validate_config(cfg):
    return lib().nosa_validate_config(ctypes.byref(cfg))


def nosa_state_bytes(cfg, which):
    return lib().nosa_state_bytes(ctypes.byref(cfg), which)


def nosa_workspace_bytes(cfg, which):
    return lib().nosa_workspace_bytes(ctypes.byref(cfg), which)


def nosa_state_init(cfg, st, stream=None):
    _check(lib().nosa_state_init(ctypes.byref(cfg), ctypes.byref(st), _stream(stream)), "nosa_state_init")


def nosa_compress_append(cfg, st, k_new, v_new, e_new, T, lens=None, stream=None):
    _check(lib().nosa_compress_append(ctypes.byref(cfg), ctypes.byref(st), _ptr(k_new), _ptr(v_new), _ptr(e_new),
                                      int(T), _ptr(lens), _stream(stream)), "nosa_compress_append")


def nosa_compress_append_head(cfg, st, k_new, v_new, w1, w2, T, lens=None, stream=None):
    _check(lib().nosa_compress_append_head(ctypes.byref(cfg), ctypes.byref(st), _ptr(k_new), _ptr(v_new), _ptr(w1),
                                           _ptr(w2), int(T), _ptr(lens), _stream(stream)),
           "nosa_compress_append_head")


def nosa_select(cfg, st, q, sel, nsel, gq=None, ws=None, stream=None):
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().nosa_select(ctypes.byref(cfg), ctypes.byref(st), _ptr(q), _ptr(sel), _ptr(nsel), _ptr(gq), _ptr(ws),
                             nbytes, _stream(stream)), "nosa_select")


def nosa_select_noalloc(cfg, st, q, sel, nsel, gq=None, stream=None):
    """nosa_select with its scratch in the library's fixed device array (allocates nothing)."""
    _check(lib().nosa_select_noalloc(ctypes.byref(cfg), ctypes.byref(st), _ptr(q), _ptr(sel), _ptr(nsel), _ptr(gq),
                                     _stream(stream)), "nosa_select_noalloc")


def nosa_noalloc_scratch_poison(byte, stream=None):
    """Test hook: fill nosa_select_noalloc's shared scratch array with `byte` (stale-contents check)."""
    _check(lib().nosa_noalloc_scratch_poison(int(byte) & 0xFF, _stream(stream)), "nosa_noalloc_scratch_poison")


def nosa_cache_sync(cfg, st, sel, nsel, block_table, n_fetched=None, ws=None, stream=None):
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().nosa_cache_sync(ctypes.byref(cfg), ctypes.byref(st), _ptr(sel), _ptr(nsel), _ptr(block_table),
                                 _ptr(n_fetched), _ptr(ws), nbytes, _stream(stream)), "nosa_cache_sync")


def nosa_sparse_decode(cfg, st, q, sel, nsel, block_table, out, ws=None, stream=None):
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().nosa_sparse_decode(ctypes.byref(cfg), ctypes.byref(st), _ptr(q), _ptr(sel), _ptr(nsel),
                                    _ptr(block_table), _ptr(out), _ptr(ws), nbytes, _stream(stream)),
           "nosa_sparse_decode")


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def nosa_append_select(cfg, st, k_new, v_new, e_new, q, sel, nsel, gq=None, ws=None, stream=None):
    _check(lib().nosa_append_select(ctypes.byref(cfg), ctypes.byref(st), _ptr(k_new), _ptr(v_new), _ptr(e_new),
                                    _ptr(q), _ptr(sel), _ptr(nsel), _ptr(gq), _ptr(ws), _nbytes(ws),
                                    _stream(stream)), "nosa_append_select")


def nosa_fused_step(cfg, st, k_new, v_new, e_new, q, sel, nsel, gq, out, ws=None, stream=None):
    _check(lib().nosa_fused_step(ctypes.byref(cfg), ctypes.byref(st), _ptr(k_new), _ptr(v_new), _ptr(e_new),
                                 _ptr(q), _ptr(sel), _ptr(nsel), _ptr(gq), _ptr(out), _ptr(ws), _nbytes(ws),
                                 _stream(stream)), "nosa_fused_step")


def nosa_decode_resident(cfg, st, q, split, ws=None, stream=None):
    _check(lib().nosa_decode_resident(ctypes.byref(cfg), ctypes.byref(st), _ptr(q), _ptr(split), _nbytes(split),
                                      _ptr(ws), _nbytes(ws), _stream(stream)), "nosa_decode_resident")


def nosa_decode_rest(cfg, st, q, gq, split, out, ws=None, stream=None):
    _check(lib().nosa_decode_rest(ctypes.byref(cfg), ctypes.byref(st), _ptr(q), _ptr(gq), _ptr(split),
                                  _nbytes(split), _ptr(out), _ptr(ws), _nbytes(ws), _stream(stream)),
           "nosa_decode_rest")


def nosa_dense_decode(cfg, st, q, out, ws=None, stream=None):
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().nosa_dense_decode(ctypes.byref(cfg), ctypes.byref(st), _ptr(q), _ptr(out), _ptr(ws), nbytes,
                                   _stream(stream)), "nosa_dense_decode")


def nosa_check_wait_timeout(err, max_cycles, stream=None):
    """Run the bounded-wait diagnostic into the device word `err` (a 1-element int32 tensor)."""
    _check(lib().nosa_check_wait_timeout(_ptr(err), int(max_cycles), _stream(stream)), "nosa_check_wait_timeout")


def nosa_read_error(st, clear=True, stream=None):
    flags = ctypes.c_uint32(0)
    rc = lib().nosa_read_error(ctypes.byref(st), ctypes.byref(flags), int(clear), _stream(stream))
    if rc not in (OK, ERR_DEVICE):
        raise NosaError(rc, "nosa_read_error")
    return flags.value


# ---- caller-side buffer owner --------------------------------------------------------

class NosaLayer:
    """Allocates (with torch) every buffer one layer of the path needs and calls the entry points.

    ``host_store``: in offload mode, an existing pinned uint8 tensor to use as the host KV store
    (several layers may share one when their synthetic KV is identical); allocated if None.
    """

    def __init__(self, cfg, device="cuda", host_store=None):
        rc = nosa_validate_config(cfg)
        if rc != OK:
            raise NosaError(rc, "config")
        self.cfg, self.device = cfg, torch.device(device)
        self.units = cfg.batch * cfg.heads_kv
        self.G = cfg.heads_q // cfg.heads_kv
        self.max_sel = cfg.k_q + cfg.k_e + 1
        dev = self.device

        def dbuf(which, dtype=torch.uint8):
            n = nosa_state_bytes(cfg, which)
            if n == 0:
                return None
            return torch.empty(n, dtype=torch.uint8, device=dev).view(dtype)

        if cfg.offload:
            n = nosa_state_bytes(cfg, BUF_KV_STORE)
            if host_store is None:
                host_store = torch.empty(n, dtype=torch.uint8, pin_memory=True)
            assert host_store.is_pinned() and host_store.numel() >= n
            self.kv_store = host_store
        else:
            self.kv_store = dbuf(BUF_KV_STORE)
        self.evict_logit = dbuf(BUF_EVICT_LOGIT, torch.float32)
        self.ck = dbuf(BUF_CK, torch.int16 if cfg.flags & FLAG_CK_BF16 else torch.float32)
        self.blk_evict = dbuf(BUF_BLK_EVICT, torch.float64)
        self.gamma_e = dbuf(BUF_GAMMA_E, torch.int32)
        self.gamma_n = dbuf(BUF_GAMMA_N, torch.int32)
        self.seq_len = dbuf(BUF_SEQ_LEN, torch.int32)
        self.cache = dbuf(BUF_CACHE)
        self.slot_block = dbuf(BUF_SLOT_BLOCK, torch.int32)
        self.block_slot = dbuf(BUF_BLOCK_SLOT, torch.int32)
        self.err = dbuf(BUF_ERR, torch.int32)
        self.pool = dbuf(BUF_POOL, torch.int32)
        self.pool_n = dbuf(BUF_POOL_N, torch.int32)
        self.state = State(*[None if t is None else t.data_ptr() for t in (
            self.kv_store, self.evict_logit, self.ck, self.blk_evict, self.gamma_e, self.gamma_n, self.seq_len,
            self.cache, self.slot_block, self.block_slot, self.err, self.pool, self.pool_n)])
        # per-step outputs and workspaces (zero-filled once, as the library requires)
        self.sel = torch.full((self.units, self.max_sel), -1, dtype=torch.int32, device=dev)
        self.nsel = torch.zeros(self.units, dtype=torch.int32, device=dev)
        self.gq = torch.full((self.units, max(cfg.k_q, 1)), -1, dtype=torch.int32, device=dev)
        self.block_table = torch.full((self.units, self.max_sel), -1, dtype=torch.int32, device=dev)
        self.n_fetched = torch.zeros(self.units, dtype=torch.int32, device=dev)

        def ws(which):
            n = nosa_workspace_bytes(cfg, which)
            return torch.zeros(max(n, 16), dtype=torch.uint8, device=dev) if n else None

        self.ws_select = ws(WS_SELECT)
        self.ws_decode = ws(WS_SPARSE_DECODE)
        self.ws_dense = None if cfg.offload else ws(WS_DENSE_DECODE)
        self.ws_cache = ws(WS_CACHE_SYNC)
        self.split = None if cfg.flags & FLAG_FILL else ws(WS_SPLIT)
        self.ws_step = ws(WS_FUSED_STEP)
        nosa_state_init(cfg, self.state)

    # one decode step = the four calls, in order
    def append(self, k_new, v_new, e_new, T=1, lens=None, stream=None):
        nosa_compress_append(self.cfg, self.state, k_new, v_new, e_new, T, lens, stream)

    def append_head(self, k_new, v_new, w1, w2, T=1, lens=None, stream=None):
        """Append with the eviction logits computed by the fused head (w1 fp32 [Hkv][D][128], w2 [Hkv][128])."""
        nosa_compress_append_head(self.cfg, self.state, k_new, v_new, w1, w2, T, lens, stream)

    def select(self, q, stream=None):
        nosa_select(self.cfg, self.state, q, self.sel, self.nsel, self.gq, self.ws_select, stream)

    def append_select(self, k_new, v_new, e_new, q, stream=None):
        """The decode append (one token) and the selection in one launch."""
        nosa_append_select(self.cfg, self.state, k_new, v_new, e_new, q, self.sel, self.nsel, self.gq,
                           self.ws_select, stream)

    def cache_sync(self, stream=None):
        nosa_cache_sync(self.cfg, self.state, self.sel, self.nsel, self.block_table, self.n_fetched, self.ws_cache,
                        stream)

    def sparse_decode(self, q, out, stream=None):
        bt = self.block_table if self.cfg.offload else None
        nosa_sparse_decode(self.cfg, self.state, q, self.sel, self.nsel, bt, out, self.ws_decode, stream)

    def decode_resident(self, q, stream=None):
        """Attention over Gamma_e + the local block, right after append (may overlap select / cache_sync)."""
        nosa_decode_resident(self.cfg, self.state, q, self.split, self.ws_decode, stream)

    def decode_rest(self, q, out, stream=None):
        """Attention over the rest of Gamma_q, merged with decode_resident's state, into out."""
        nosa_decode_rest(self.cfg, self.state, q, self.gq, self.split, out, self.ws_decode, stream)

    def dense_decode(self, q, out, stream=None):
        nosa_dense_decode(self.cfg, self.state, q, out, self.ws_dense, stream)

    def decode_step(self, k_new, v_new, e_new, q, out, stream=None):
        """One decode step of this layer into `out` (bf16 bits [B][Hq][D]): with the KV store in
        device memory and the union reading, nosa_fused_step (one launch); otherwise append +
        select in one launch, the cache sync (offload), and the sparse decode."""
        if self.ws_step is not None:
            self.fused_step(k_new, v_new, e_new, q, out, stream)
            return
        self.append_select(k_new, v_new, e_new, q, stream)
        if self.cfg.offload:
            self.cache_sync(stream)
        self.sparse_decode(q, out, stream)

    def fused_step(self, k_new, v_new, e_new, q, out, stream=None):
        """One decode step of this layer in one launch (device store, union reading): append,
        select and sparse decode into `out` (bf16 bits [B][Hq][D])."""
        nosa_fused_step(self.cfg, self.state, k_new, v_new, e_new, q, self.sel, self.nsel, self.gq, out,
                        self.ws_step, stream)

    def read_error(self, clear=True, stream=None):
        return nosa_read_error(self.state, clear, stream)
