"""CPU oracle of the NOSA decode step (fp64, single-threaded, plain C).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; the product path never touches it.
It shares no code with the CUDA library.  See ``nosa_oracle.c`` for the
passages of "NOSA: Native and Offloadable Sparse Attention" each step follows.
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "_lib", "libnosa_oracle.so")
_lib = None


def build(force=False):
    """Compile the oracle with gcc (-O2, no fast-math, no FP contraction)."""
    src = os.path.join(_HERE, "nosa_oracle.c")
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(src):
        return _LIB_PATH
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                           "-shared", "-o", _LIB_PATH, src, "-lm"])
    return _LIB_PATH


class Stats(ctypes.Structure):
    _fields_ = [("nb_c", ctypes.c_int32), ("local", ctypes.c_int32), ("n_fetch", ctypes.c_int32),
                ("n_sel", ctypes.c_int32), ("n_overlap", ctypes.c_int32), ("gamma", ctypes.c_double)]


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        L.nosa_oracle_unit_new.restype = P
        L.nosa_oracle_unit_new.argtypes = [ctypes.c_int32] * 6 + [ctypes.c_double, ctypes.c_int64]
        L.nosa_oracle_unit_free.argtypes = [P]
        L.nosa_oracle_prefill.argtypes = [P, P, P, P, ctypes.c_int64]
        L.nosa_oracle_step.argtypes = [P, P, P, ctypes.c_float, P, P, P, P, P, P, P, P, P, P]
        L.nosa_oracle_dense.argtypes = [P, P, P]
        L.nosa_oracle_len.argtypes = [P]
        L.nosa_oracle_len.restype = ctypes.c_int64
        L.nosa_oracle_ck.argtypes = [P]
        L.nosa_oracle_ck.restype = ctypes.POINTER(ctypes.c_double)
        L.nosa_oracle_E.argtypes = [P]
        L.nosa_oracle_E.restype = ctypes.POINTER(ctypes.c_double)
        L.nosa_oracle_violations.argtypes = [P, P]
        L.nosa_oracle_attend_blocks.argtypes = [P, P, P, ctypes.c_int32, P]
        L.nosa_oracle_set_ck_bf16.argtypes = [P, ctypes.c_int32]
        L.nosa_oracle_set_fill.argtypes = [P, ctypes.c_int32]
        L.nosa_oracle_evict_head.argtypes = [P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, P, P, P]
        L.nosa_oracle_round_bf16.argtypes = [ctypes.c_double]
        L.nosa_oracle_round_bf16.restype = ctypes.c_double
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def round_bf16(x):
    """x rounded to the nearest bf16 value, ties to even (the oracle's rounding of pooled keys)."""
    return lib().nosa_oracle_round_bf16(float(x))


def evict_head(V, W1, W2):
    """Eviction logits of value rows V [T][D] (bf16 bits) under one head W1 [D][H], W2 [H] (fp32):
    e_j = sum_h W2[h] softplus(v_j . W1[:, h]), fp64, rounded to fp32."""
    V = np.ascontiguousarray(V, dtype=np.uint16)
    W1 = np.ascontiguousarray(W1, dtype=np.float32)
    W2 = np.ascontiguousarray(W2, dtype=np.float32)
    T, D = V.shape
    H = W2.shape[0]
    assert W1.shape == (D, H)
    e = np.empty(T, np.float32)
    lib().nosa_oracle_evict_head(_p(V), T, D, H, _p(W1), _p(W2), _p(e))
    return e


class OracleUnit:
    """One (sequence, kv head) unit: its KV history, pooled keys and selection state."""

    def __init__(self, D=128, G=1, block=64, sub=16, k_q=16, k_e=48, scale=None, cap=8192, ck_bf16=False,
                 fill=False):
        self.D, self.G, self.block, self.sub, self.k_q, self.k_e = D, G, block, sub, k_q, k_e
        self.scale = 1.0 / np.sqrt(D) if scale is None else float(scale)
        self.cap = cap
        self._u = lib().nosa_oracle_unit_new(D, G, block, sub, k_q, k_e, self.scale, cap)
        if not self._u:
            raise ValueError("oracle: bad unit parameters")
        if ck_bf16:
            lib().nosa_oracle_set_ck_bf16(self._u, 1)
        if fill:
            lib().nosa_oracle_set_fill(self._u, 1)

    def __del__(self):
        if getattr(self, "_u", None) and _lib is not None:
            _lib.nosa_oracle_unit_free(self._u)
            self._u = None

    def prefill(self, K, V, e):
        K = np.ascontiguousarray(K, dtype=np.uint16)
        V = np.ascontiguousarray(V, dtype=np.uint16)
        e = np.ascontiguousarray(e, dtype=np.float32)
        T = K.shape[0]
        assert K.shape == (T, self.D) and V.shape == (T, self.D) and e.shape == (T,)
        rc = lib().nosa_oracle_prefill(self._u, _p(K), _p(V), _p(e), T)
        if rc:
            raise RuntimeError(f"oracle prefill failed ({rc})")

    def step(self, k, v, e, q):
        """Append one token (k, v: [D] bf16 bits; e: float) and decode for q [G][D] bf16 bits."""
        k = np.ascontiguousarray(k, dtype=np.uint16).reshape(self.D)
        v = np.ascontiguousarray(v, dtype=np.uint16).reshape(self.D)
        q = np.ascontiguousarray(q, dtype=np.uint16).reshape(self.G, self.D)
        L_next = self.length + 1
        nb_c = max(0, (L_next - 1) // self.block)
        sel = np.full(self.k_q + self.k_e + 1, -1, np.int32)
        gq = np.full(max(self.k_q, 1), -1, np.int32)
        ge = np.full(max(self.k_e, 1), -1, np.int32)
        scores = np.zeros(max(nb_c, 1), np.float64)
        o = np.zeros((self.G, self.D), np.float64)
        ns, nq, ne = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        st = Stats()
        rc = lib().nosa_oracle_step(self._u, _p(k), _p(v), ctypes.c_float(float(e)), _p(q), _p(sel),
                                    ctypes.byref(ns), _p(gq), ctypes.byref(nq), _p(ge), ctypes.byref(ne),
                                    _p(scores), _p(o), ctypes.byref(st))
        if rc:
            raise RuntimeError(f"oracle step failed ({rc})")
        return {
            "sel": sel[: ns.value].copy(), "gq": gq[: nq.value].copy(), "ge": ge[: ne.value].copy(),
            "scores": scores[:nb_c].copy(), "o": o, "nb_c": st.nb_c, "local": st.local,
            "n_fetch": st.n_fetch, "n_sel": st.n_sel, "n_overlap": st.n_overlap, "gamma": st.gamma,
        }

    def dense(self, q):
        q = np.ascontiguousarray(q, dtype=np.uint16).reshape(self.G, self.D)
        o = np.zeros((self.G, self.D), np.float64)
        lib().nosa_oracle_dense(self._u, _p(q), _p(o))
        return o

    def attend_blocks(self, q, blocks):
        """Attention of q [G][D] (bf16 bits) over the tokens of the given blocks."""
        q = np.ascontiguousarray(q, dtype=np.uint16).reshape(self.G, self.D)
        b = np.ascontiguousarray(blocks, dtype=np.int32)
        o = np.zeros((self.G, self.D), np.float64)
        lib().nosa_oracle_attend_blocks(self._u, _p(q), _p(b), len(b), _p(o))
        return o

    @property
    def length(self):
        return int(lib().nosa_oracle_len(self._u))

    def ck(self):
        n = self.length // self.sub
        return np.ctypeslib.as_array(lib().nosa_oracle_ck(self._u), shape=(self.cap // self.sub * self.D,))[
            : n * self.D].reshape(n, self.D).copy()

    def E(self):
        n = self.length // self.block
        return np.ctypeslib.as_array(lib().nosa_oracle_E(self._u), shape=(self.cap // self.block,))[:n].copy()

    def violations(self):
        out = np.zeros(5, np.int64)
        lib().nosa_oracle_violations(self._u, _p(out))
        return dict(zip(["gamma", "reselect", "incremental", "fetch", "steps"], out.tolist()))
