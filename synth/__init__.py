"""Seeded synthetic inputs for the NOSA decode workloads.

Holds no part of the attention method: only counter-based random draws (see
``nosa_synth.h``).  The CPU build feeds the oracle; the GPU build fills device
memory with the same bytes for large contexts.
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_HOST_SO = os.path.join(_HERE, "_lib", "libnosa_synth_host.so")
_GPU_SO = os.path.join(_HERE, "_lib", "libnosa_synth_gpu.so")
K_STREAM, V_STREAM = 1, 2
_host = None
_gpu = None


def _stale(out, srcs):
    return not os.path.exists(out) or any(os.path.getmtime(s) > os.path.getmtime(out) for s in srcs)


def build(force=False, gpu=True):
    os.makedirs(os.path.join(_HERE, "_lib"), exist_ok=True)
    hdr = os.path.join(_HERE, "nosa_synth.h")
    src = os.path.join(_HERE, "synth_host.c")
    if force or _stale(_HOST_SO, [src, hdr]):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-o",
                               _HOST_SO, src])
    if gpu:
        src = os.path.join(_HERE, "synth_gpu.cu")
        if force or _stale(_GPU_SO, [src, hdr]):
            subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
                                   "-Xcompiler", "-fPIC", "-shared", "-o", _GPU_SO, src])


def host():
    global _host
    if _host is None:
        build(gpu=False)
        L = ctypes.CDLL(_HOST_SO)
        u64, u32, i64, i32, P = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
        L.nosa_synth_kv_rows.argtypes = [u64, u32, u32, u32, u32, u64, i64, i32, P]
        L.nosa_synth_e_rows.argtypes = [u64, u32, u32, u32, u64, i64, P]
        L.nosa_synth_q_steps.argtypes = [u64, u32, u32, u32, i64, i32, P, P]
        L.nosa_synth_head_weights.argtypes = [u64, u32, i32, i32, i32, P, P]
        _host = L
    return _host


def gpu():
    global _gpu
    if _gpu is None:
        build(gpu=True)
        L = ctypes.CDLL(_GPU_SO)
        u64, u32, i64, i32, P = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
        L.nosa_synth_kv_dev.argtypes = [u64, u32, u32, i32, i32, i32, u64, i64, i32, P, P]
        L.nosa_synth_e_dev.argtypes = [u64, u32, i32, i32, i32, u64, i64, P, P]
        L.nosa_synth_q_dev.argtypes = [u64, u32, i32, i32, i32, i64, i32, P, P, P]
        _gpu = L
    return _gpu


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def kv_rows(seed, stream, layer, seq, kvh, p0, T, D=128):
    """K (stream 1) or V (stream 2) rows [T][D] as bf16 bit patterns (uint16)."""
    out = np.empty((T, D), np.uint16)
    host().nosa_synth_kv_rows(seed, stream, layer, seq, kvh, p0, T, D, _p(out))
    return out


def e_rows(seed, layer, seq, kvh, p0, T):
    out = np.empty(T, np.float32)
    host().nosa_synth_e_rows(seed, layer, seq, kvh, p0, T, _p(out))
    return out


def q_steps(seed, layer, seq, qh, n, D=128):
    """Drifting queries of decode steps 0..n-1: (fp32 [n][D], bf16 bits [n][D])."""
    f = np.empty((n, D), np.float32)
    b = np.empty((n, D), np.uint16)
    host().nosa_synth_q_steps(seed, layer, seq, qh, n, D, _p(f), _p(b))
    return f, b


def head_weights(seed, layer, Hkv, D=128, H=128):
    """Synthetic eviction-head weights of one layer: W1 fp32 [Hkv][D][H], W2 fp32 [Hkv][H]."""
    W1 = np.empty((Hkv, D, H), np.float32)
    W2 = np.empty((Hkv, H), np.float32)
    host().nosa_synth_head_weights(seed, layer, Hkv, D, H, _p(W1), _p(W2))
    return W1, W2


def bf16_to_f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---- device-side generation (torch tensors; async on the given CUDA stream) ----

def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"synth {what} failed ({rc})")


def kv_dev(seed, stream, layer, B, Hkv, p0, T, out, cuda_stream=0, D=128, seq0=0):
    """Fill out ([B*Hkv][T][D] bf16, device) with K or V rows of sequences seq0..seq0+B-1,
    positions p0..p0+T-1."""
    _check(gpu().nosa_synth_kv_dev(seed, stream, layer, seq0, B, Hkv, p0, T, D, out.data_ptr(), cuda_stream), "kv")


def e_dev(seed, layer, B, Hkv, p0, T, out, cuda_stream=0, seq0=0):
    _check(gpu().nosa_synth_e_dev(seed, layer, seq0, B, Hkv, p0, T, out.data_ptr(), cuda_stream), "e")


def q_dev(seed, layer, B, Hq, t, state, out, cuda_stream=0, D=128, seq0=0):
    """Advance the fp32 query state [B*Hq][D] to step t and write bf16 queries into out."""
    _check(gpu().nosa_synth_q_dev(seed, layer, seq0, B, Hq, t, D, state.data_ptr(), out.data_ptr(), cuda_stream),
           "q")
