"""Parity at the benchmark workloads' full sizes, in the launch configuration bench.py times.

Each test builds bench.Workload for one configuration (one layer of a multi-layer
stack: the per-layer launches are the same), runs decode steps through the C
ABI exactly as the benchmark does (micro-batches on their own streams for the
offload configuration), and checks sampled units -- the first and last
sequence, every kv head -- against the CPU oracle at every step run: selected
sets (near-ties excused and counted), Gamma_e, outputs, and fetch counts.
"""

import numpy as np
import pytest
import torch

import bench
import oracle
import synth
from oracle import OracleUnit
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


def run_config(c, steps, seqs=None, seed=0, micro=1, dense_step=None, name=None, layer=0, units=None):
    """Decode `steps` steps of layer `layer` of configuration c as the benchmark launches them;
    check units (seq, kv head) -- by default every kv head of `seqs` (first and last sequence)."""
    wl = bench.Workload(c, steps, seed=seed, groups=2, layers=1, micro=micro, layer0=layer)
    G = c["Hq"] // c["Hkv"]
    seqs = seqs if seqs is not None else sorted({0, c["B"] - 1})
    units = units if units is not None else [(b, g) for b in seqs for g in range(c["Hkv"])]
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
            W1, W2 = synth.head_weights(seed, layer, c["Hkv"])
            E = oracle.evict_head(V, W1[g], W2[g])
        else:
            E = synth.e_rows(seed, layer, b, g, 0, L0 + steps)
        Q = np.stack([synth.q_steps(seed, layer, b, g * G + h, steps)[1] for h in range(G)], axis=1)
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
    H.record_stats(name or str(c), st)
    assert not bad, bad[:3]
    H.assert_parity(st)
    return st


# the device-store configurations run both ways: append + select, then decode (two launches), and
# the fused step (one launch)
PATHS = {"two launches": dict(step=False), "fused step": dict(step=True)}


def _wl(name, path):
    return dict(bench.WORKLOADS[name], **PATHS[path])


@pytest.mark.parametrize("path", sorted(PATHS))
def test_mha_8k_full(path):
    """1 layer, batch 1, 16/16 heads, 8K context, 32 steps: every unit, every step."""
    run_config(_wl("mha-8k", path), steps=32, seqs=[0], name=f"mha-8k {path}")


@pytest.mark.parametrize("path", sorted(PATHS))
def test_gqa_16k_full(path):
    """1 layer, batch 8, GQA 8:1, 16K context, 128 steps: every sequence and kv head, every step."""
    run_config(_wl("gqa-16k", path), steps=128, seqs=list(range(8)), name=f"gqa-16k {path}")


@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("layer", [0, 27])
def test_stack28_32k_layer(layer, path):
    """Batch 32, GQA 8:1, 32K context, layer 0 or 27 of the 28: all 64 decode steps, first and last
    sequence, both kv heads, plus the dense comparator at the last step."""
    run_config(_wl("stack28-32k", path), steps=64, dense_step=63, layer=layer,
               name=f"stack28-32k layer {layer} {path}")


@pytest.mark.parametrize("layer", [0, 27])
def test_offload28_128k_layer_micro_batches(layer):
    """Batch 64, 128K context, KV in pinned host memory (layers 0 and 27 hold the two host KV groups),
    two micro-batches on two streams: all 256 decode steps, first and last sequence, both kv heads."""
    st = run_config(dict(bench.WORKLOADS["offload28-128k"]), steps=256, micro=2, layer=layer,
                    name=f"offload28-128k layer {layer}")
    assert st["fetch_cmp"] > 0


SWEEP_CELLS = sorted({(8, L, k, off) for L in (32768, 131072) for k in (32, 64, 128) for off in (False, True)} |
                     {(B, 131072, 64, off) for B in (1, 8, 32, 128, 256) for off in (False, True)})


@pytest.mark.parametrize("B,L,k,offload", SWEEP_CELLS)
def test_sweep_cell(B, L, k, offload):
    """The sweep (1 layer, 16 q / 2 kv heads, k_e = 0.75 k): every (context, k, device / pinned host)
    cell at batch 8, and every batch at 128K and k = 64, in the launch configuration the sweep times;
    4 decode steps on two sampled units, the first sequence's kv head 0 and the last one's kv head 1."""
    c = dict(layers=1, B=B, Hq=16, Hkv=2, L=L, k_q=k // 4, k_e=3 * k // 4, steps=64, offload=offload, fuse=True,
             step=True)
    run_config(c, steps=4, micro=1, units=[(0, 0), (B - 1, 1)],
               name=f"sweep B={B} L={L} k={k} {'offload' if offload else 'device'}")
