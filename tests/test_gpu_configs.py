"""Parity at the benchmark workloads' full sizes, in the launch configuration bench.py times.

Each test builds bench.Workload for one configuration (one layer of a multi-layer
stack: the per-layer launches are the same), runs decode steps through the C
ABI exactly as the benchmark does (micro-batches on their own streams for the
offload configuration), and checks sampled units -- the first and last
sequence, every kv head -- against the CPU oracle at every step run: selected
sets (near-ties excused and counted), Gamma_e, outputs, and fetch counts.
"""
import json
import os

import numpy as np
import pytest
import torch

import bench
import oracle
import synth
from oracle import OracleUnit
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def record(name, st):
    """Append this workload's parity statistics (exact / excused-tie counts, errors) as one JSON
    line to the file named by NOSA_PARITY_STATS, if that variable is set."""
    path = os.environ.get("NOSA_PARITY_STATS")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": name, **st}) + "\n")


def run_config(c, steps, seqs=None, seed=0, micro=1, dense_step=None, name=None):
    wl = bench.Workload(c, steps, seed=seed, groups=2, layers=1, micro=micro)
    G = c["Hq"] // c["Hkv"]
    seqs = seqs if seqs is not None else sorted({0, c["B"] - 1})
    units = [(b, g) for b in seqs for g in range(c["Hkv"])]
    rec = {(b, g): [] for (b, g) in units}
    dense_out = None
    for t in range(steps):
        wl.cur.copy_(wl.inputs[t])
        wl.launch_step()
        torch.cuda.synchronize()
        for (b, g) in units:
            m, bl = divmod(b, wl.Bm)
            lay = wl.layers[0][m]
            ul = bl * c["Hkv"] + g
            n = int(lay.nsel[ul])
            gn = int(lay.gamma_n[ul])
            rec[(b, g)].append(dict(
                sel=lay.sel[ul, :n].cpu().numpy(), gq=lay.gq[ul].cpu().numpy(),
                ge=lay.gamma_e.view(-1, max(c["k_e"], 1))[ul, :gn].cpu().numpy() if c["k_e"] else None,
                nf=int(lay.n_fetched[ul]) if c["offload"] else None,
                out=synth.bf16_to_f32(wl.out[0, b, g * G:(g + 1) * G].cpu().numpy().view(np.uint16)).astype(
                    np.float64)))
        if dense_step is not None and t == dense_step:
            dense_out = torch.empty_like(wl.out[0])
            for m in range(wl.micro):
                q, _, _, _ = wl.views(wl.cur, 0, m)
                wl.layers[0][m].dense_decode(q, dense_out[m * wl.Bm:(m + 1) * wl.Bm])
            torch.cuda.synchronize()
            dense_out = synth.bf16_to_f32(dense_out.cpu().numpy().view(np.uint16)).astype(np.float64)
    errs = [lay.read_error() for lay in wl.layers[0]]
    assert not any(errs), errs

    st = H.new_stats()
    bad = []
    L0 = c["L"]
    for (b, g) in units:
        K = synth.kv_rows(seed, synth.K_STREAM, wl.kv_layer(0), b, g, 0, L0 + steps)
        V = synth.kv_rows(seed, synth.V_STREAM, wl.kv_layer(0), b, g, 0, L0 + steps)
        if c.get("head"):
            W1, W2 = synth.head_weights(seed, 0, c["Hkv"])
            E = oracle.evict_head(V, W1[g], W2[g])
        else:
            E = synth.e_rows(seed, 0, b, g, 0, L0 + steps)
        Q = np.stack([synth.q_steps(seed, 0, b, g * G + h, steps)[1] for h in range(G)], axis=1)
        o = OracleUnit(G=G, k_q=c["k_q"], k_e=c["k_e"], cap=wl.max_ctx, ck_bf16=c.get("ck_bf16", False),
                       fill=c.get("fill", False))
        o.prefill(K[:L0], V[:L0], E[:L0])
        ok = True
        for t in range(steps):
            r = o.step(K[L0 + t], V[L0 + t], float(E[L0 + t]), Q[t])
            g_ = rec[(b, g)][t]
            ok = H.compare_step(st, o, r, Q[t], g_["sel"], g_["gq"], g_["ge"], g_["out"], c["k_q"], ok,
                                g_["nf"], bad, (t, b, g), c.get("fill", False))
            if dense_out is not None and t == dense_step:
                dref = o.dense(Q[t])
                dg = dense_out[b, g * G:(g + 1) * G]
                st["dense_max_abs"] = max(st["dense_max_abs"], float(np.abs(dg - dref).max()))
                st["dense_max_rel"] = max(st["dense_max_rel"],
                                          float(np.linalg.norm(dg - dref) / np.linalg.norm(dref)))
        v = o.violations()
        assert v["gamma"] == 0 and v["reselect"] == 0 and v["incremental"] == 0 and v["fetch"] == 0, v
    st["mean_abs"] = st["sum_abs"] / max(st["n_out"], 1)
    assert st["cmp"] == len(units) * steps
    record(name or str(c), st)
    assert not bad, bad[:3]
    H.assert_parity(st)
    return st


def test_mha_8k_full():
    """1 layer, batch 1, 16/16 heads, 8K context, 32 steps: every unit, every step."""
    run_config(dict(bench.WORKLOADS["mha-8k"]), steps=32, seqs=[0], name="mha-8k")


def test_gqa_16k_full():
    """1 layer, batch 8, GQA 8:1, 16K context, 128 steps: sequences 0 and 7, every step."""
    run_config(dict(bench.WORKLOADS["gqa-16k"]), steps=128, name="gqa-16k")


def test_stack28_32k_one_layer():
    """Batch 32, GQA 8:1, 32K context (one layer of the 28): 8 steps, plus the dense comparator."""
    run_config(dict(bench.WORKLOADS["stack28-32k"]), steps=8, dense_step=7, name="stack28-32k layer 0")


def test_offload28_128k_one_layer_micro_batches():
    """Batch 64, 128K context, KV in pinned host memory, two micro-batches on two streams."""
    st = run_config(dict(bench.WORKLOADS["offload28-128k"]), steps=6, micro=2, name="offload28-128k layer 0")
    assert st["fetch_cmp"] > 0


@pytest.mark.parametrize("B,L,k,offload", [(256, 131072, 128, False), (32, 32768, 32, True)])
def test_sweep_corners(B, L, k, offload):
    """Sweep corners: the largest device-resident point (batch 256, 128K, k = 128) and an offload point."""
    c = dict(layers=1, B=B, Hq=16, Hkv=2, L=L, k_q=k // 4, k_e=3 * k // 4, steps=64, offload=offload, fuse=True)
    run_config(c, steps=4, micro=2 if offload else 1,
               name=f"sweep B={B} L={L} k={k} {'offload' if offload else 'device'}")
