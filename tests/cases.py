"""Input builders shared by the tests: crafted fixtures and seeded synthetic units.

Nothing here computes any part of the method; it only lays out inputs.
"""
import json
import os

import numpy as np

import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def f32_to_bf16_bits_exact(x):
    """Bit pattern of values that are exactly representable in bf16."""
    x = np.asarray(x, np.float32)
    bits = x.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0), "fixture value not exact in bf16"
    return (bits >> 16).astype(np.uint16)


def bf16_bits_to_f64(bits):
    return synth.bf16_to_f32(bits).astype(np.float64)


def load_fixture(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def build_fixture(spec):
    """Prefill arrays (K, V bf16 bits; e fp32) and the query of a crafted spec."""
    D, blk, sub = spec["D"], spec["block"], spec["sub"]
    nblocks = max(len(spec.get("sub_keys", [])), len(spec.get("sub_e", [])))
    L0 = nblocks * blk + spec["local_tokens"]
    K = np.zeros((L0, D), np.float32)
    for b, subs in enumerate(spec.get("sub_keys", [])):
        for s, pairs in enumerate(subs):
            for dim, val in pairs:
                K[b * blk + s * sub: b * blk + (s + 1) * sub, dim] = val
    for pos, dim, val in spec.get("key_spikes", []):
        K[pos, dim] = val
    e = np.zeros(L0, np.float32)
    for b, vals in enumerate(spec.get("sub_e", [])):
        for s, val in enumerate(vals):
            e[b * blk + s * sub: b * blk + (s + 1) * sub] = val
    for pos, val in spec.get("e_spikes", []):
        e[pos] = val
    q = np.zeros((spec["G"], D), np.float32)
    for h, val in enumerate(spec.get("q_all", [])):  # head h: every dim = val
        q[h, :] = val
    for h, pairs in enumerate(spec.get("q", [])):
        for dim, val in pairs:
            q[h, dim] = val
    Kb = f32_to_bf16_bits_exact(K)
    return Kb, Kb.copy(), e, f32_to_bf16_bits_exact(q)


def synthetic_unit(seed, layer, seq, kvh, L, D=128):
    """K, V (bf16 bits [L][D]) and e (fp32 [L]) of one unit, positions 0..L-1."""
    K = synth.kv_rows(seed, synth.K_STREAM, layer, seq, kvh, 0, L, D)
    V = synth.kv_rows(seed, synth.V_STREAM, layer, seq, kvh, 0, L, D)
    e = synth.e_rows(seed, layer, seq, kvh, 0, L)
    return K, V, e


def synthetic_queries(seed, layer, seq, kvh, G, n_steps, D=128):
    """bf16 query bits [n_steps][G][D] of the G q heads of kv head kvh."""
    out = np.empty((n_steps, G, D), np.uint16)
    for g in range(G):
        _, b = synth.q_steps(seed, layer, seq, kvh * G + g, n_steps, D)
        out[:, g, :] = b
    return out


def textbook_attention(q_bits, K_bits, V_bits, e, tokens, scale):
    """softmax(q K^T * scale + e) V over the given token positions, in fp64."""
    q = bf16_bits_to_f64(q_bits)
    K = bf16_bits_to_f64(K_bits[tokens])
    V = bf16_bits_to_f64(V_bits[tokens])
    z = q @ K.T * scale + e[tokens].astype(np.float64)[None, :]
    z -= z.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    return p @ V
