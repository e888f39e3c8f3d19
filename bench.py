"""Benchmark of the NOSA decode hot path on B200 (one JSON line on rank 0).

A step is one decode step of the whole stack: for every layer, append the new
token of every sequence (nosa_compress_append), select (nosa_select), sync the
block cache (nosa_cache_sync, offload mode) and attend (nosa_sparse_decode).
Throughput = sequences x steps / device time.  Default workload (offload28-128k):
28 layers, batch 64, 16 q / 2 kv heads, head_dim 128, 128K context, KV in
pinned host memory with a device cache of local + 64 blocks per (seq, kv head),
k_e = 48, k_q = 16.

    python bench.py [--workload offload28-128k] [--steps K] [--warmup W] [--gpus N] [--impl nosa|reference]

--impl reference times the CPU oracle (the plain fp64 restatement of the
method, single thread) on a bounded sample of the same workload.
N > 1 (torchrun): independent replicas, one per GPU (the decode step has no
exchange between sequences); value = all ranks' tokens / max-over-ranks time.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import block_sparse_offloadable_b200 as nosa  # noqa: E402
import synth  # noqa: E402

METRIC = "sparse decode tokens/s/GPU at 128K ctx; % of HBM and PCIe roofline"
D = 128

# Device-store workloads run each layer's step in one launch (nosa_fused_step; --no-fused-step: the
# two-launch path); the offload workload runs the decode-time append fused into the select launch
# (nosa_append_select), then the cache sync and the decode.  --unfused launches append and select
# separately (and turns the fused step off).
WORKLOADS = {
    # one layer, batch 1, 16 q / 16 kv heads, 8K context, 32 decode steps, KV in device memory
    "mha-8k": dict(layers=1, B=1, Hq=16, Hkv=16, L=8192, k_q=16, k_e=48, steps=32, offload=False, fuse=True,
                   step=True),
    # one layer, batch 8, GQA 16 q / 2 kv heads, 16K context, 128 decode steps, KV in device memory
    "gqa-16k": dict(layers=1, B=8, Hq=16, Hkv=2, L=16384, k_q=16, k_e=48, steps=128, offload=False, fuse=True,
                    step=True),
    # 28-layer stack, batch 32, GQA 16/2, 32K context, 64 decode steps, KV in device memory
    # (its line also carries the library's dense decode on the same inputs)
    "stack28-32k": dict(layers=28, B=32, Hq=16, Hkv=2, L=32768, k_q=16, k_e=48, steps=64, offload=False, fuse=True,
                        step=True, dense_compare=True),
    # 28-layer stack, batch 64, GQA 16/2, 128K context, 256 decode steps, KV in pinned host memory
    "offload28-128k": dict(layers=28, B=64, Hq=16, Hkv=2, L=131072, k_q=16, k_e=48, steps=256, offload=True, fuse=True),
}
DEFAULT_WORKLOAD = "offload28-128k"


def describe(c, groups):
    s = (f"{c['layers']} layers, batch {c['B']}, {c['Hq']} q / {c['Hkv']} kv heads, head_dim 128, "
         f"context {c['L']}, block 64, sub-block 16, k_q={c['k_q']}, k_e={c['k_e']}, local window 1 block, ")
    if c["offload"]:
        s += (f"KV in pinned host memory ({groups} host KV groups shared by layers l mod {groups}), "
              f"device cache = local + {c['k_q'] + c['k_e']} blocks per (seq, kv head)")
    else:
        s += "KV resident in device memory"
    if c.get("ck_bf16"):
        s += ", pooled keys stored bf16"
    if c.get("fill"):
        s += ", fill reading of the selection"
    if c.get("head"):
        s += ", eviction logits from the fused synthetic eviction head"
    if c.get("split"):
        s += ", decode split: Gamma_e + local attended while select and the cache sync run"
    if c.get("step") and not (c["offload"] or c.get("fill") or c.get("head") or c.get("split")):
        s += ", each layer's step (append, select, decode) in one launch"
    elif c.get("fuse"):
        s += ", append and select fused in one launch"
    return s


_PINNED = {}


def pinned(nbytes, key):
    """Pinned host buffer of nbytes, reused across workloads with the same key (pinning is slow)."""
    t = _PINNED.get(key)
    if t is None or t.numel() < nbytes:
        _PINNED.pop(key, None)
        t = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
        _PINNED[key] = t
    return t[:nbytes]


class Workload:
    """All layers of one configuration: state, prefilled context and per-step inputs on the device.

    The batch is split into `micro` micro-batches of consecutive sequences, each with its own
    per-layer state; micro-batch m runs its chain of layers on its own CUDA stream, so one
    micro-batch's host->device fetch overlaps another's HBM-bound select and attention.  Every
    sequence still goes through its layers in order.
    """

    def __init__(self, c, n_steps, seed=0, groups=2, layers=None, device="cuda", micro=1, seq_base=0, dense=False,
                 layer0=0):
        # layer0: index of the first layer built (a test may build one layer deep in the stack)
        self.c, self.seed, self.groups, self.seq_base, self.dense = c, seed, groups, seq_base, dense
        self.layer0 = layer0
        self.L = layers if layers is not None else c["layers"]
        self.B, self.Hq, self.Hkv = c["B"], c["Hq"], c["Hkv"]
        assert self.B % micro == 0, "batch must split evenly into micro-batches"
        self.micro, self.Bm = micro, self.B // micro
        self.units = self.B * self.Hkv
        self.units_m = self.Bm * self.Hkv
        self.n_steps = n_steps
        self.max_ctx = (c["L"] + n_steps + 63) // 64 * 64
        self.cfg = nosa.make_config(self.Bm, self.Hq, self.Hkv, c["k_q"], c["k_e"], self.max_ctx, c["offload"],
                                    ck_bf16=c.get("ck_bf16", False), fill=c.get("fill", False))
        dev = torch.device(device)
        self.host = {}
        if c["offload"]:
            nbytes = nosa.nosa_state_bytes(self.cfg, nosa.BUF_KV_STORE)
            for g in sorted({self.kv_layer(l) for l in range(self.L)}):
                for m in range(micro):
                    self.host[(g, m)] = pinned(nbytes, (g, m))
        self.layers = [[nosa.NosaLayer(self.cfg, dev, self.host[(self.kv_layer(l), m)] if self.host else None)
                        for m in range(micro)] for l in range(self.L)]
        # the fused eviction head: synthetic weights per layer (e is then computed, not an input)
        self.head = bool(c.get("head", False))
        self.split = bool(c.get("split", False))  # decode Gamma_e + local while select / cache sync run
        # append and select in one launch (it takes given logits and feeds the one-pass decode)
        self.fuse = bool(c.get("fuse", False)) and not (self.split or self.head)
        # the whole step of a layer in one launch (device store, union reading, given logits)
        self.step = bool(c.get("step", False)) and not (self.split or self.head or c["offload"] or c.get("fill"))
        self.W = [tuple(torch.from_numpy(w).to(dev) for w in synth.head_weights(seed, self.layer0 + l, self.Hkv))
                  for l in range(self.L)] if self.head else None
        self._prefill(dev)
        self._inputs(dev)

    def kv_layer(self, l):
        """Layer index whose synthetic K/V the l-th built layer holds (host KV groups alias layers)."""
        lg = self.layer0 + l
        return lg % self.groups if self.c["offload"] else lg

    def _prefill(self, dev):
        T = self.c["L"]
        k = torch.empty((self.units_m, T, D), dtype=torch.int16, device=dev)
        v = torch.empty_like(k)
        e = torch.empty((self.units_m, T), dtype=torch.float32, device=dev)
        for l in range(self.L):
            kl = self.kv_layer(l)
            for m, lay in enumerate(self.layers[l]):
                s0 = self.seq_base + m * self.Bm
                synth.kv_dev(self.seed, synth.K_STREAM, kl, self.Bm, self.Hkv, 0, T, k, seq0=s0)
                synth.kv_dev(self.seed, synth.V_STREAM, kl, self.Bm, self.Hkv, 0, T, v, seq0=s0)
                if self.head:
                    lay.append_head(k, v, self.W[l][0], self.W[l][1], T)
                else:
                    synth.e_dev(self.seed, self.layer0 + l, self.Bm, self.Hkv, 0, T, e, seq0=s0)
                    lay.append(k, v, e, T)
        torch.cuda.synchronize()
        del k, v, e

    def _inputs(self, dev):
        """Per-step inputs of every layer and micro-batch, packed so one copy moves a step's inputs."""
        n, Um, L0 = self.n_steps, self.units_m, self.c["L"]
        self.q_bytes = self.Bm * self.Hq * D * 2
        self.kv_bytes = Um * D * 2
        self.e_bytes = 0 if self.head else Um * 4
        self.part_in = self.q_bytes + 2 * self.kv_bytes + self.e_bytes
        self.step_in = self.L * self.micro * self.part_in
        self.inputs = torch.empty((n, self.step_in), dtype=torch.uint8, device=dev)
        qstate = torch.empty((self.Bm * self.Hq, D), dtype=torch.float32, device=dev)
        qt = torch.empty((self.Bm * self.Hq, D), dtype=torch.int16, device=dev)
        kk = torch.empty((Um, n, D), dtype=torch.int16, device=dev)
        vv = torch.empty_like(kk)
        ee = torch.empty((Um, n), dtype=torch.float32, device=dev)
        for l in range(self.L):
            kl = self.kv_layer(l)
            for m in range(self.micro):
                s0 = self.seq_base + m * self.Bm
                synth.kv_dev(self.seed, synth.K_STREAM, kl, self.Bm, self.Hkv, L0, n, kk, seq0=s0)
                synth.kv_dev(self.seed, synth.V_STREAM, kl, self.Bm, self.Hkv, L0, n, vv, seq0=s0)
                if not self.head:
                    synth.e_dev(self.seed, self.layer0 + l, self.Bm, self.Hkv, L0, n, ee, seq0=s0)
                base = (l * self.micro + m) * self.part_in
                for t in range(n):
                    synth.q_dev(self.seed, self.layer0 + l, self.Bm, self.Hq, t, qstate, qt, seq0=s0)
                    row = self.inputs[t]
                    row[base:base + self.q_bytes].view(torch.int16).copy_(qt.view(-1))
                    o = base + self.q_bytes
                    row[o:o + self.kv_bytes].view(torch.int16).copy_(kk[:, t].reshape(-1))
                    o += self.kv_bytes
                    row[o:o + self.kv_bytes].view(torch.int16).copy_(vv[:, t].reshape(-1))
                    o += self.kv_bytes
                    if self.e_bytes:
                        row[o:o + self.e_bytes].view(torch.float32).copy_(ee[:, t])
        self.cur = torch.empty(self.step_in, dtype=torch.uint8, device=dev)
        self.out = torch.empty((self.L, self.B, self.Hq, D), dtype=torch.int16, device=dev)
        self.streams = [torch.cuda.Stream(device=dev) for _ in range(self.micro - 1)]
        self.side = [torch.cuda.Stream(device=dev) for _ in range(self.micro)] if self.split else []
        torch.cuda.synchronize()

    def views(self, buf, l, m=0):
        base = (l * self.micro + m) * self.part_in
        q = buf[base:base + self.q_bytes].view(torch.int16).view(self.Bm, self.Hq, D)
        o = base + self.q_bytes
        k = buf[o:o + self.kv_bytes].view(torch.int16).view(self.units_m, 1, D)
        o += self.kv_bytes
        v = buf[o:o + self.kv_bytes].view(torch.int16).view(self.units_m, 1, D)
        o += self.kv_bytes
        e = buf[o:o + self.e_bytes].view(torch.float32).view(self.units_m, 1) if self.e_bytes else None
        return q, k, v, e

    def out_view(self, l, m, out=None):
        return (self.out if out is None else out)[l, m * self.Bm:(m + 1) * self.Bm]

    def kernel_calls(self, l, m, buf=None, out_buf=None):
        """(name, call) of one layer's step for micro-batch m, in order.  With the split decode,
        ("fork", None) starts the side stream, calls named "resident" run on it, and ("join", None)
        joins it back before the rest of the decode."""
        buf = self.cur if buf is None else buf
        lay = self.layers[l][m]
        q, k, v, e = self.views(buf, l, m)
        out = self.out_view(l, m, out_buf)
        if self.head:
            w1, w2 = self.W[l]
            append = ("append", lambda s: lay.append_head(k, v, w1, w2, 1, None, s))
        else:
            append = ("append", lambda s: lay.append(k, v, e, 1, None, s))
        if self.dense:  # the full-attention comparator: append, then attend to every token
            return [append, ("dense", lambda s: lay.dense_decode(q, out, s))]
        if self.step:
            return [("step", lambda s: lay.fused_step(k, v, e, q, out, s))]
        if self.fuse:
            calls = [("append_select", lambda s: lay.append_select(k, v, e, q, s))]
            if self.c["offload"]:
                calls.append(("cache_sync", lambda s: lay.cache_sync(s)))
            calls.append(("decode", lambda s: lay.sparse_decode(q, out, s)))
            return calls
        calls = [append]
        if self.split:
            calls += [("fork", None), ("resident", lambda s: lay.decode_resident(q, s))]
        calls.append(("select", lambda s: lay.select(q, s)))
        if self.c["offload"]:
            calls.append(("cache_sync", lambda s: lay.cache_sync(s)))
        if self.split:
            calls += [("join", None), ("rest", lambda s: lay.decode_rest(q, out, s))]
        else:
            calls.append(("decode", lambda s: lay.sparse_decode(q, out, s)))
        return calls

    def launch_step(self, buf=None, events=None, out=None):
        """Launch one decode step of every layer and micro-batch.

        With events: everything on the current stream, each call bracketed by CUDA events (the
        per-kernel timing pass).  Otherwise micro-batch m > 0 runs on its own stream, forked from
        and joined back into the current stream."""
        cur = torch.cuda.current_stream()
        if events is not None:
            for l in range(self.L):
                for m in range(self.micro):
                    for name, fn in self.kernel_calls(l, m, buf):
                        if fn is None:
                            continue
                        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        e0.record()
                        fn(cur)
                        e1.record()
                        events.append((name, l, e0, e1))
            return
        streams = [cur] + self.streams
        for s in self.streams:
            s.wait_stream(cur)
        for l in range(self.L):
            for m in range(self.micro):
                for name, fn in self.kernel_calls(l, m, buf, out):
                    if name == "fork":
                        self.side[m].wait_stream(streams[m])
                    elif name == "join":
                        streams[m].wait_stream(self.side[m])
                    else:
                        fn(self.side[m] if name == "resident" else streams[m])
        for s in self.streams:
            cur.wait_stream(s)

    def time_steps(self, warmup, steps, first=0):
        """Device ms per step over `steps` graph-replayed steps (L2 flushed per step if it fits in L2).
        Uses 3 + warmup + steps input steps: 3 eager steps, then `warmup` untimed replays of the captured
        graph (the first replays of a freshly captured graph can run ~0.1 ms slower at the largest
        stores), then the timed replays."""
        t = first
        for _ in range(3):
            self.cur.copy_(self.inputs[t])
            self.launch_step()
            t += 1
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(g, stream=s, capture_error_mode="thread_local"):
            self.launch_step()
        torch.cuda.synchronize()
        for _ in range(warmup):
            self.cur.copy_(self.inputs[t])
            t += 1
            g.replay()
        torch.cuda.synchronize()
        small = step_bytes(self) < 2 * L2_BYTES
        flush = L2Flusher(self.cur.device) if small else None
        ms = 0.0
        for _ in range(steps):
            self.cur.copy_(self.inputs[t])
            t += 1
            if flush is not None:
                flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            ms += e0.elapsed_time(e1)
        del g
        return ms / steps, t

    @property
    def launches_per_step(self):
        # append, select, [cache plan, cache gather], decode (split: resident + rest; fused: append_select;
        # fused step: one launch)
        if self.step:
            return self.L * self.micro
        return self.L * self.micro * ((5 if self.c["offload"] else 3) + (1 if self.split else 0) -
                                      (1 if self.fuse else 0))


# ---------------------------------------------------------------------------------------

L2_BYTES = 126 << 20


class L2Flusher:
    """Writes a buffer twice the size of L2, then reads another one, so the next kernel starts with
    none of its data in L2.  The read leaves L2 holding clean lines: a write alone leaves it full of
    dirty lines, whose write-back would land inside the timed region as traffic the step never made."""

    def __init__(self, dev):
        self.buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        self.buf2 = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        self.sink = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.buf.fill_(1.0)
        torch.sum(self.buf2, 0, out=self.sink)


def ck_elem(c):
    """Bytes per stored pooled-key element: 4 (fp32), or 2 with bf16 pooled keys."""
    return 2 if c.get("ck_bf16") else 4


def step_bytes(wl):
    """Bytes one decode step streams from HBM (pooled keys + selected KV blocks, or all KV for
    the dense comparator), all layers."""
    c = wl.c
    nb = (c["L"] - 1) // 64
    if getattr(wl, "dense", False):
        per_unit = (nb + 1) * (32768 + 256)
    else:
        per_unit = nb * 4 * 128 * ck_elem(c) + (c["k_q"] + c["k_e"] + 1) * (32768 + 256)
    return wl.L * wl.units * per_unit


def algo_bytes(c, U, Bm, Lctx, nsel_mean):
    """Algorithmic bytes per launch of each kernel, for one layer of one micro-batch of Bm sequences
    (U units) at context Lctx, with nsel_mean blocks attended per unit (|S(t)|, the local block
    included).  Select: the pooled keys of the (Lctx - 1) // 64 candidates and the G query heads of each
    unit.  Decode: the K, V and eviction logits of the attended blocks, the queries and the outputs.
    Append: the new K, V rows and logit.  The fused launches add up their parts."""
    nb_c = (Lctx - 1) // 64
    blk = 64 * D * 2 * 2 + 64 * 4  # one block: keys + values (bf16) + eviction logits (fp32)
    a = {
        "select": U * (nb_c * 4 * D * ck_elem(c) + (c["Hq"] // c["Hkv"]) * D * 2),
        "decode": U * nsel_mean * blk + 2 * Bm * c["Hq"] * D * 2,
        "append": U * (2 * D * 2 + 4),
    }
    a["append_select"] = a["select"] + a["append"]
    a["step"] = a["append_select"] + a["decode"]
    n_res = min(c["k_e"], nb_c) + 1  # Gamma_e + the local block
    a["resident"] = U * n_res * blk + Bm * c["Hq"] * D * 2
    a["rest"] = U * max(nsel_mean - n_res, 0) * blk + 2 * Bm * c["Hq"] * D * 2
    return a


def time_idempotent(wl, name, reps, flush=None):
    """Average device time of one launch of a kernel (select, decode, the split decode's resident /
    rest passes, the dense comparator, the fused append + select, or the fused step): a CUDA graph of
    that kernel for every layer, replayed back to back.  All but the fused launches are idempotent;
    a fused launch appends one token per unit per replay, the same work as in a step, so its replays
    time it too."""
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(g, stream=s, capture_error_mode="thread_local"):
        for l in range(wl.L):
            for m in range(wl.micro):
                lay = wl.layers[l][m]
                q, _, _, _ = wl.views(wl.cur, l, m)
                if name == "select":
                    lay.select(q)
                elif name == "append_select":
                    _, k, v, e = wl.views(wl.cur, l, m)
                    lay.append_select(k, v, e, q)
                elif name == "step":
                    _, k, v, e = wl.views(wl.cur, l, m)
                    lay.fused_step(k, v, e, q, wl.out_view(l, m))
                elif name == "resident":
                    lay.decode_resident(q)
                elif name == "rest":
                    lay.decode_rest(q, wl.out_view(l, m))
                elif name == "dense":
                    lay.dense_decode(q, wl.out_view(l, m))
                else:
                    lay.sparse_decode(q, wl.out_view(l, m))
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    total = 0.0
    for _ in range(reps):
        if flush is not None:
            flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        total += e0.elapsed_time(e1)
    del g
    return total / (reps * wl.L * wl.micro)


def measure_pcie_h2d(dev, nbytes=1 << 30):
    h = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    d = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    for _ in range(2):
        d.copy_(h, non_blocking=True)
    torch.cuda.synchronize()
    best = 1e30
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        d.copy_(h, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    del h, d
    return nbytes / (best * 1e-3) / 1e9


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(index), f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        # a timed region of a few ms (the one-layer workloads) can end before the first 200 ms sample:
        # keep sampling until there are a few rows (at most ~1.5 s more)
        for _ in range(15):
            try:
                with open(self.f.name) as fh:
                    if sum(1 for r in fh if r.strip()) >= 3:
                        break
            except OSError:
                break
            time.sleep(0.1)
        self.p.terminate()
        self.p.wait()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[0]))
                mx = float(r[1])
                for name, val in zip(names, r[4:8]):
                    if val.strip() == "Active":
                        reasons.add(name)
            except (ValueError, IndexError):
                pass
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_index(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids) and ids[local_rank].isdigit():
            return int(ids[local_rank])
    return local_rank


def reduce_max_ms(ms, world, device):
    """Device time of the slowest rank (every rank takes part; world 1 returns ms)."""
    if world <= 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(world, batch, steps, ms):
    """Whole-job tokens/s: every rank decodes `batch` sequences per step; time = slowest rank."""
    return world * batch * steps / (ms * 1e-3)


def host_cpu():
    """The host CPU model and its logical core count (the oracle timing runs on one of them)."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"model": model, "logical_cores": os.cpu_count()}


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


# DRAM bytes per launch from an ncu capture (profiles/dram_traffic.json): used only for the
# same workload variant and only while the kernel's sources are unchanged since the capture.
KERNEL_SOURCES = {
    "select": ("nosa_select.cu", "nosa_append_unit.cuh"), "decode": ("nosa_decode.cu", "nosa_attend.cuh"),
    "step": ("nosa_step.cu", "nosa_attend.cuh", "nosa_append_unit.cuh"),
    "cache_sync": ("nosa_cache.cu",), "append": ("nosa_append.cu", "nosa_append_unit.cuh"),
    "append_select": ("nosa_select.cu", "nosa_append_unit.cuh"),
    # kernels that the benchmark's per-kernel pass does not time on its own (prefill, the split
    # decode's passes, the dense comparator, the cache plan): their captures are checked the same way
    "dense": ("nosa_decode.cu", "nosa_attend.cuh"), "resident": ("nosa_decode.cu", "nosa_attend.cuh"),
    "rest": ("nosa_decode.cu", "nosa_attend.cuh"),
    "cache_plan": ("nosa_cache.cu",), "cache_gather": ("nosa_cache.cu",),
    "append_head": ("nosa_append.cu", "nosa_append_unit.cuh"),
    "prefill_store": ("nosa_append.cu", "nosa_append_unit.cuh"),
    "prefill_pool": ("nosa_append.cu", "nosa_append_unit.cuh"),
    "prefill_gamma": ("nosa_append.cu", "nosa_append_unit.cuh"),
    "prefill_head": ("nosa_append.cu", "nosa_append_unit.cuh"),
}


def capture_status():
    """Every committed ncu capture (profiles/dram_traffic.json) and whether the kernel's sources
    still match it: 'current', or 'stale' (its counters no longer describe the code)."""
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            table = json.load(f)
    except (OSError, ValueError):
        return {}
    out = {}
    for e in table.get("captures", []):
        name = e.get("kernel")
        ok = name in KERNEL_SOURCES and e.get("sources_sha256") == sources_sha(name)
        out[f"{name}@{e.get('variant')}"] = "current" if ok else "stale"
    return out


def sources_sha(name):
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_offloadable_b200", "csrc")
    for f in KERNEL_SOURCES[name] + ("nosa_common.cuh", "nosa_internal.cuh"):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def captured_traffic(name, c, args):
    """(bytes per launch, capture note) for kernel `name` on `variant`, or (None, why not)."""
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            table = json.load(f)
    except (OSError, ValueError):
        return None, "no capture"
    variant = traffic_variant(c, args, name)
    for e in table.get("captures", []):
        if e.get("kernel") == name and e.get("variant") == variant:
            if e.get("sources_sha256") != sources_sha(name):
                return None, "kernel changed since the capture"
            return float(e["dram_bytes_per_launch"]), e.get("profile")
    return None, "no capture of this variant"


def traffic_variant(c, args, name):
    """The workload variant a traffic capture of kernel `name` must match: the workload name plus the
    options that change that kernel's work (the layer count does not change a launch)."""
    v = [args.workload]
    for key in ("ck_bf16", "fill", "head", "split"):
        if c.get(key):
            v.append(key)
    if name in ("select", "append") and (not c.get("fuse") or c.get("head") or c.get("split")):
        v.append("unfused")
    return "+".join(v)


# ---------------------------------------------------------------------------------------

def oracle_sample(c, groups, seed, n_units, n_steps, budget_s=25.0):
    """Time the CPU oracle on a deterministic sample of unit-steps of the workload.

    Units: layer 0 / last, seq 0 / last, both kv heads first.  Each sampled unit
    is prefilled (untimed) and stepped n_steps times (timed).  Returns
    (seconds per unit-step, unit-steps timed, description)."""
    import oracle
    G = c["Hq"] // c["Hkv"]
    picks = []
    for l in (0, c["layers"] - 1):
        for b in (0, c["B"] - 1):
            for g in range(c["Hkv"]):
                if (l, b, g) not in picks:
                    picks.append((l, b, g))
    picks = picks[:n_units]
    L0 = c["L"]
    cap = (L0 + n_steps + 63) // 64 * 64
    total_t, count = 0.0, 0
    for (l, b, g) in picks:
        kl = l % groups if c["offload"] else l
        K = synth.kv_rows(seed, synth.K_STREAM, kl, b, g, 0, L0 + n_steps)
        V = synth.kv_rows(seed, synth.V_STREAM, kl, b, g, 0, L0 + n_steps)
        head = synth.head_weights(seed, l, c["Hkv"]) if c.get("head") else None
        if head is not None:  # the prefill's logits come from the head too (untimed)
            E = oracle.evict_head(V[:L0], head[0][g], head[1][g])
        else:
            E = synth.e_rows(seed, l, b, g, 0, L0 + n_steps)
        Q = np.stack([synth.q_steps(seed, l, b, g * G + h, n_steps)[1] for h in range(G)], axis=1)
        u = oracle.OracleUnit(G=G, k_q=c["k_q"], k_e=c["k_e"], cap=cap, ck_bf16=c.get("ck_bf16", False),
                              fill=c.get("fill", False))
        u.prefill(K[:L0], V[:L0], E[:L0])
        for t in range(n_steps):
            t0 = time.perf_counter()
            e_t = (oracle.evict_head(V[L0 + t:L0 + t + 1], head[0][g], head[1][g])[0] if head is not None
                   else E[L0 + t])
            u.step(K[L0 + t], V[L0 + t], float(e_t), Q[t])
            total_t += time.perf_counter() - t0
            count += 1
            if total_t > budget_s:
                break
        if total_t > budget_s:
            break
    desc = (f"{count} unit-steps of units (layer, seq, kv head) in {picks[:max(1, len(picks))]}, "
            f"context {L0}; per-unit-step time x {c['layers'] * c['B'] * c['Hkv']} units per decode step "
            f"(extrapolated, 1 core)")
    return total_t / max(count, 1), count, desc


def run_reference(args, c, rank):
    if rank != 0:
        return
    n_units = 4
    per, count, desc = oracle_sample(c, args.host_groups, args.seed, n_units=n_units,
                                     n_steps=max(1, (args.warmup + args.steps)), budget_s=60.0)
    units_per_step = c["layers"] * c["B"] * c["Hkv"]
    step_s = per * units_per_step
    value = c["B"] / step_s
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{args.workload}: " + describe(c, args.host_groups)},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": desc,
                             "host": host_cpu()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_nosa(args, c, rank, world, dev):
    k_e2e = 0 if args.no_e2e else min(args.steps, 8)
    n_steps = args.warmup + args.steps + args.profile_steps + k_e2e
    assert n_steps <= c["steps"] + 64, "more decode steps than the workload's context margin"
    t_setup = time.time()
    pcie = measure_pcie_h2d(dev) if c["offload"] else None
    micro = args.micro if args.micro else (2 if c["offload"] else 1)
    # replicas: rank r decodes its own sequences r*B .. (r+1)*B-1 (no exchange between sequences)
    wl = Workload(c, n_steps + 8, seed=args.seed, groups=args.host_groups, device=dev, layers=args.layers, micro=micro,
                  seq_base=rank * c["B"])
    setup_s = time.time() - t_setup
    stream = torch.cuda.current_stream()
    step_i = 0

    def feed(t):
        wl.cur.copy_(wl.inputs[t], non_blocking=True)

    graph = None
    if not args.no_graph:
        # capture one step reading the fixed input buffer; each step copies its inputs in first
        feed(0)
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s, capture_error_mode="thread_local"):
            wl.launch_step()
        torch.cuda.synchronize()
        # capturing launched nothing: state is unchanged

    def run_step():
        nonlocal step_i
        feed(step_i)
        if graph is not None:
            graph.replay()
        else:
            wl.launch_step()
        step_i += 1

    for _ in range(args.warmup):
        run_step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = ClockSampler(gpu_index(int(os.environ.get("LOCAL_RANK", 0))))
    time.sleep(0.3)
    small = step_bytes(wl) < 2 * L2_BYTES
    flush = L2Flusher(dev) if small else None
    torch.cuda.synchronize()
    if small:
        # the step's working set fits in L2: flush it before every step, time steps one by one; the
        # step's inputs are staged into the captured graph's input buffer before the timed region
        ms = 0.0
        for _ in range(args.steps):
            feed(step_i)
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            if graph is not None:
                graph.replay()
            else:
                wl.launch_step()
            step_i += 1
            e1.record()
            torch.cuda.synchronize()
            ms += e0.elapsed_time(e1)
    else:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            run_step()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
    clk = clocks.stop()
    ms = reduce_max_ms(ms, world, dev)
    value = aggregate_value(world, c["B"], args.steps, ms)
    launches = wl.launches_per_step * args.steps

    # ---- per-kernel durations (events around every launch, eager) + selection stats ----
    events = []
    fetched, nsel_sum, nsel_n = [], 0, 0
    prev_sel, gammas = None, []
    for _ in range(args.profile_steps):
        feed(step_i)
        # hold the GPU while the host enqueues the whole step, so the events time
        # the kernels back to back rather than host launch gaps
        torch.cuda._sleep(int(4e7))
        wl.launch_step(events=events)
        step_i += 1
        torch.cuda.synchronize()
        all_layers = [lay for per_layer in wl.layers for lay in per_layer]
        if c["offload"]:
            fetched.append(sum(int(lay.n_fetched.sum()) for lay in all_layers))
        for lay in all_layers:
            nsel_sum += int(lay.nsel.sum())
            nsel_n += lay.units
        # locality gamma(t) = |Sel(t) & S(t-1)| / |Sel(t)| (Sel(t): S(t) without the local block)
        cur_sel = [(lay.sel.cpu().numpy(), lay.nsel.cpu().numpy()) for lay in all_layers]
        if prev_sel is not None:
            for (s1, n1), (s0, n0) in zip(cur_sel, prev_sel):
                for u in range(s1.shape[0]):
                    now = set(s1[u, :n1[u] - 1].tolist())
                    if now:
                        gammas.append(len(now & set(s0[u, :n0[u]].tolist())) / len(now))
        prev_sel = cur_sel
    kt = {}
    for name, l, a, b in events:
        kt.setdefault(name, []).append(a.elapsed_time(b))
    # replace the event times (launch included) by graph-replay times: select and decode are
    # idempotent; each replay of the fused append + select appends one more token (the margin of
    # the workload's context covers the 4 replays)
    for name in ("select", "decode", "resident", "rest", "append_select", "step"):
        if name in kt:
            per = time_idempotent(wl, name, reps=3, flush=flush)
            kt[name] = [per] * len(kt[name])
    nsel_mean = nsel_sum / max(nsel_n, 1)
    hbm_peak, peak_kind = load_peaks()
    U, Lctx = wl.units_m, c["L"] + step_i
    algo = algo_bytes(c, U, wl.Bm, Lctx, nsel_mean)
    kern = {}
    for name, ts in kt.items():
        avg = sum(ts) / len(ts)
        kern[name] = {"avg_us": avg * 1e3, "share": sum(ts) / sum(sum(v) for v in kt.values())}
        if name in algo:
            gbs = algo[name] / (avg * 1e-3) / 1e9
            kern[name].update({"bytes": algo[name], "GBps": gbs, "frac_hbm": gbs / hbm_peak})
    pcie_obj = None
    if c["offload"] and fetched:
        fb = sum(fetched) / len(fetched) / (wl.L * wl.micro)  # blocks per launch (layer, micro-batch)
        avg = sum(kt["cache_sync"]) / len(kt["cache_sync"])
        gbs = fb * 32768 / (avg * 1e-3) / 1e9
        kern["cache_sync"].update({"bytes": fb * 32768, "GBps": gbs, "frac_pcie": gbs / pcie})
        step_gbs = sum(fetched) / len(fetched) * 32768 / (ms / args.steps * 1e-3) / 1e9
        pcie_obj = {"fetched_blocks_per_step": sum(fetched) / len(fetched),
                    "fetched_blocks_per_unit_step": fb / U, "achieved_GBps": gbs, "peak_GBps": pcie,
                    "peak": "measured pinned cudaMemcpyAsync H2D, 1 GiB, this box", "frac": gbs / pcie,
                    "step_GBps": step_gbs, "step_frac": step_gbs / pcie,
                    "note": "achieved/frac: the cache sync's own launches, timed one at a time on one stream; "
                            "step_GBps/step_frac: fetched bytes per step over the device-timed step, in which "
                            "the micro-batches' fetches overlap the other micro-batch's select and decode"}
    dom = max(kern, key=lambda k: kern[k]["share"])
    if dom == "cache_sync" and pcie_obj:
        roof = {"bound": "pcie", "kernel": "cache_sync (plan + gather)", "achieved": pcie_obj["achieved_GBps"],
                "peak": pcie, "unit": "GB/s", "frac": pcie_obj["frac"], "traffic": None,
                "peak_source": "measured live: pinned H2D copy"}
    else:
        roof = {"bound": "hbm", "kernel": dom, "achieved": kern[dom]["GBps"], "peak": hbm_peak, "unit": "GB/s",
                "frac": kern[dom]["frac_hbm"], "traffic": None, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json)"}
    hb = max((k for k in kern if "frac_hbm" in kern[k]), key=lambda k: kern[k]["share"])
    roof_hbm = {"bound": "hbm", "kernel": hb, "achieved": kern[hb]["GBps"], "peak": hbm_peak, "unit": "GB/s",
                "frac": kern[hb]["frac_hbm"], "traffic": None}
    for r in (roof, roof_hbm):
        kname = "cache_sync" if r["kernel"].startswith("cache_sync") else r["kernel"]
        if kname in KERNEL_SOURCES:
            r["traffic"], r["traffic_source"] = captured_traffic(kname, c, args)

    # ---- end to end: host inputs -> device, step, outputs -> host, all inside the timed region ----
    # A serving loop.  With at least 1 MB of copies per step: two input/output buffer pairs, each with its
    # own captured step; a copy stream brings step t+1's inputs in and takes step t's outputs out while the
    # compute stream runs step t.  Smaller steps copy in, run and copy out in order on one stream, since
    # the cross-stream waits would cost more than the copies they hide.
    e2e = None
    if k_e2e and rank == 0 and wl.step_in + wl.out.numel() * 2 < (1 << 20):
        hin = torch.empty((k_e2e, wl.step_in), dtype=torch.uint8, pin_memory=True)
        hin.copy_(wl.inputs[step_i:step_i + k_e2e])
        hout = torch.empty((k_e2e,) + tuple(wl.out.shape), dtype=torch.int16, pin_memory=True)
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        w0 = time.perf_counter()
        a0.record()
        for t in range(k_e2e):
            wl.cur.copy_(hin[t], non_blocking=True)
            if graph is not None:
                graph.replay()
            else:
                wl.launch_step()
            hout[t].copy_(wl.out, non_blocking=True)
        a1.record()
        torch.cuda.synchronize()
        wall = time.perf_counter() - w0
        ms_e2e = a0.elapsed_time(a1)
        e2e = {"value": c["B"] * k_e2e / (ms_e2e * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": wl.step_in,
               "d2h_bytes_per_step": wl.out.numel() * 2, "steps": k_e2e, "wall_s": wall,
               "path": "pinned host inputs -> nosa_* C ABI -> pinned host outputs, in order on one stream"}
        step_i += k_e2e
    elif k_e2e and rank == 0:
        hin = torch.empty((k_e2e, wl.step_in), dtype=torch.uint8, pin_memory=True)
        hin.copy_(wl.inputs[step_i:step_i + k_e2e])
        hout = torch.empty((k_e2e,) + tuple(wl.out.shape), dtype=torch.int16, pin_memory=True)
        bufs = [(wl.cur, wl.out), (torch.empty_like(wl.cur), torch.empty_like(wl.out))]
        graphs = [graph, None]
        if graph is not None:
            g2 = torch.cuda.CUDAGraph()
            s2 = torch.cuda.Stream()
            s2.wait_stream(torch.cuda.current_stream())
            with torch.cuda.graph(g2, stream=s2, capture_error_mode="thread_local"):
                wl.launch_step(buf=bufs[1][0], out=bufs[1][1])
            graphs[1] = g2
        torch.cuda.synchronize()
        comp, xfer = torch.cuda.current_stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event(), torch.cuda.Event()]
        ev_done = [torch.cuda.Event(), torch.cuda.Event()]
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        w0 = time.perf_counter()
        a0.record(comp)
        xfer.wait_stream(comp)
        with torch.cuda.stream(xfer):
            bufs[0][0].copy_(hin[0], non_blocking=True)
        ev_in[0].record(xfer)
        for t in range(k_e2e):
            i, j = t % 2, (t + 1) % 2
            if t + 1 < k_e2e:  # pair j was last used by step t-1, whose output copy precedes this on xfer
                with torch.cuda.stream(xfer):
                    bufs[j][0].copy_(hin[t + 1], non_blocking=True)
                ev_in[j].record(xfer)
            comp.wait_event(ev_in[i])
            if graphs[i] is not None:
                graphs[i].replay()
            else:
                wl.launch_step(buf=bufs[i][0], out=bufs[i][1])
            ev_done[i].record(comp)
            xfer.wait_event(ev_done[i])
            with torch.cuda.stream(xfer):
                hout[t].copy_(bufs[i][1], non_blocking=True)
        comp.wait_stream(xfer)
        a1.record(comp)
        torch.cuda.synchronize()
        wall = time.perf_counter() - w0
        ms_e2e = a0.elapsed_time(a1)
        e2e = {"value": c["B"] * k_e2e / (ms_e2e * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": wl.step_in,
               "d2h_bytes_per_step": wl.out.numel() * 2, "steps": k_e2e, "wall_s": wall,
               "path": "pinned host inputs -> nosa_* C ABI -> pinned host outputs; the next step's input copy "
                       "and the previous step's output copy overlap the current step (two buffer pairs)"}
        del graphs
        step_i += k_e2e

    errs = [lay.read_error() for per_layer in wl.layers for lay in per_layer]
    if any(errs):
        raise RuntimeError(f"device error flags set: {errs}")
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        per, count, desc = oracle_sample(c, args.host_groups, args.seed, n_units=4, n_steps=24, budget_s=12.0)
        cv = c["B"] / (per * c["layers"] * c["B"] * c["Hkv"])
        cpu = {"value": cv, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": desc, "host": host_cpu()}
    if rank != 0:
        return None
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded counter-based generator: K,V ~ N(0,1)/sqrt(128) bf16, e ~ N(0,1), drifting q)",
        "config": {"workload": f"{args.workload}: " + describe(c, args.host_groups), "layers": c["layers"],
                   "batch": c["B"], "heads_q": c["Hq"], "heads_kv": c["Hkv"], "context": c["L"], "k_q": c["k_q"],
                   "k_e": c["k_e"], "offload": c["offload"], "pooled_keys": "bf16" if c.get("ck_bf16") else "fp32",
                   "selection": "fill" if c.get("fill") else "union",
                   "eviction_logits": "fused head" if c.get("head") else "input",
                   "decode": "split (resident during select / cache sync, then rest)" if c.get("split") else "one pass", "host_kv_groups": args.host_groups if c["offload"] else None,
                   "cuda_graph": graph is not None, "micro_batches": wl.micro,
                   "l2": ("L2 flushed (256 MB write) before every timed step; steps timed one by one, each "
                          "step's inputs staged on the device before its timed region" if small else
                          f"inputs larger than L2: each step streams {step_bytes(wl) / 1e9:.2f} GB of pooled keys and KV blocks"),
                   "kernel_timing": "select, decode, fused append + select, fused step: CUDA graph of every layer's "
                                    "launch replayed (a fused launch appends a token per replay); append, cache_sync: "
                                    "events per launch"},
        "roofline": roof, "roofline_hbm": roof_hbm, "kernels": kern, "pcie": pcie_obj,
        "mean_selected_blocks": nsel_mean,
        "gamma": ({"mean": float(np.mean(gammas)), "min": float(np.min(gammas)),
                   "floor_k_e_over_k": c["k_e"] / (c["k_q"] + c["k_e"]), "unit_steps": len(gammas)}
                  if gammas else None),
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "ncu_captures": capture_status(),
        "clocks": clk, "setup_s": setup_s,
    }
    return line


def run_dense(args, c, rank, world, dev):
    """The library's dense decode (nosa_dense_decode: every token of the context) on the same
    configuration and the same seeded inputs as the sparse line, graph-replayed the same way."""
    n = 3 + args.warmup + args.steps + 1
    wl = Workload(c, n, seed=args.seed, groups=args.host_groups, device=dev, layers=args.layers, micro=1,
                  seq_base=rank * c["B"], dense=True)
    ms, _ = wl.time_steps(args.warmup, args.steps)
    ms = reduce_max_ms(ms, world, dev)
    small = step_bytes(wl) < 2 * L2_BYTES
    per = time_idempotent(wl, "dense", reps=3, flush=L2Flusher(dev) if small else None)
    Lctx = c["L"] + n
    nbytes = wl.units * ((Lctx + 63) // 64) * (64 * D * 2 * 2 + 64 * 4) + 2 * wl.B * c["Hq"] * D * 2
    hbm_peak, peak_kind = load_peaks()
    gbs = nbytes / (per * 1e-3) / 1e9
    errs = [lay.read_error() for per_layer in wl.layers for lay in per_layer]
    if any(errs):
        raise RuntimeError(f"device error flags set in the dense comparator: {errs}")
    del wl
    torch.cuda.empty_cache()
    return {"value": world * c["B"] / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": args.steps,
            "warmup": args.warmup, "path": "append + nosa_dense_decode over all L tokens, every layer",
            "kernel": {"avg_us": per * 1e3, "bytes": nbytes, "GBps": gbs, "frac_hbm": gbs / hbm_peak,
                       "peak": f"{peak_kind} (MEASURED_PEAKS.json)"}}


SWEEP = dict(batch=(1, 8, 32, 128, 256), context=(32768, 131072), k=(32, 64, 128))


def run_sweep(args, dev):
    """One JSON line per sweep point: 1 layer, 16 q / 2 kv heads, batch x context x k (k_e = 0.75 k),
    KV in device memory and in pinned host memory, against dense decode on identical inputs.
    Every point replays its captured step at least 8 times before timing: with the largest stores
    (batch 256 at 128K, 32 GiB) the first replays of a freshly captured graph run ~0.1 ms slower."""
    steps, warmup = args.steps, max(args.warmup, 8)
    for L in SWEEP["context"]:
        for B in SWEEP["batch"]:
            base = dict(layers=1, B=B, Hq=16, Hkv=2, L=L, k_q=16, k_e=48, steps=3 + warmup + steps,
                        ck_bf16=args.ck_bf16, fuse=not args.unfused, step=not (args.unfused or args.no_fused_step))
            dense = Workload(dict(base, offload=False), 3 + warmup + steps + 1, seed=args.seed, dense=True,
                             device=dev)
            dense_ms, _ = dense.time_steps(warmup, steps)
            del dense
            torch.cuda.empty_cache()
            for k in SWEEP["k"]:
                for offload in (False, True):
                    c = dict(base, k_q=k // 4, k_e=3 * k // 4, offload=offload)
                    wl = Workload(c, 3 + warmup + steps + 1, seed=args.seed, device=dev)
                    ms, _ = wl.time_steps(warmup, steps)
                    errs = [lay.read_error() for per in wl.layers for lay in per]
                    del wl
                    torch.cuda.empty_cache()
                    print(json.dumps({"sweep": {"batch": B, "context": L, "k": k, "k_q": k // 4, "k_e": 3 * k // 4,
                                                "kv": "pinned host" if offload else "device",
                                                "pooled_keys": "bf16" if args.ck_bf16 else "fp32"},
                                      "sparse_tokens_per_s": B / (ms * 1e-3), "sparse_ms_per_step": ms,
                                      "dense_tokens_per_s": B / (dense_ms * 1e-3), "dense_ms_per_step": dense_ms,
                                      "speedup_vs_dense": dense_ms / ms, "steps": steps, "warmup": warmup,
                                      "device_errors": errs}), flush=True)


KQ_SWEEP = dict(k=(64, 128), kq_over_k=(0.0, 0.125, 0.25, 0.375, 0.5))


def run_kq_sweep(args, dev):
    """The k_q/k trade-off (montaan.com summary of 2510.13602, "Tunability": a lower k_q/k raises the
    locality floor k_e/k): one JSON line per (k, k_q, reading) with the measured locality gamma(t),
    the misses fetched per unit and step, |Sel| and the decode throughput.  1 layer, batch 64,
    16 q / 2 kv heads, 128K context, KV in pinned host memory, two micro-batches; k_q <= 32."""
    warmup, steps, stat_steps = args.warmup, args.steps, 16
    for k in KQ_SWEEP["k"]:
        for frac in KQ_SWEEP["kq_over_k"]:
            kq = int(round(frac * k))
            if kq > 32:
                continue
            for fill in (False, True):
                c = dict(layers=1, B=64, Hq=16, Hkv=2, L=131072, k_q=kq, k_e=k - kq, offload=True, fill=fill,
                         ck_bf16=args.ck_bf16, fuse=not args.unfused)
                wl = Workload(c, stat_steps + 3 + warmup + steps + 1, seed=args.seed, device=dev, micro=2)
                prev, gam, miss, nsel = None, [], [], []
                for t in range(stat_steps):
                    wl.cur.copy_(wl.inputs[t])
                    wl.launch_step()
                    torch.cuda.synchronize()
                    now = [(lay.sel.cpu().numpy(), lay.nsel.cpu().numpy(), lay.n_fetched.cpu().numpy())
                           for lay in wl.layers[0]]
                    for m, (sel, ns, nf) in enumerate(now):
                        for u in range(sel.shape[0]):
                            cur = set(sel[u, :ns[u] - 1].tolist())  # Sel(t): S(t) without the local block
                            nsel.append(len(cur))
                            if t > 0:
                                miss.append(int(nf[u]))
                            if prev is not None and cur:
                                before = set(prev[m][0][u, :prev[m][1][u]].tolist())
                                gam.append(len(cur & before) / len(cur))
                    prev = now
                ms, _ = wl.time_steps(warmup, steps, first=stat_steps)
                errs = [lay.read_error() for per in wl.layers for lay in per]
                del wl
                torch.cuda.empty_cache()
                print(json.dumps({"kq_sweep": {"k": k, "k_q": kq, "k_e": k - kq, "kq_over_k": kq / k,
                                               "selection": "fill" if fill else "union",
                                               "pooled_keys": "bf16" if args.ck_bf16 else "fp32"},
                                  "gamma_mean": float(np.mean(gam)), "gamma_min": float(np.min(gam)),
                                  "gamma_floor": (k - kq) / k, "misses_per_unit_step": float(np.mean(miss)),
                                  "sel_per_unit": float(np.mean(nsel)),
                                  "tokens_per_s": c["B"] / (ms * 1e-3), "ms_per_step": ms,
                                  "stat_steps": stat_steps, "steps": steps, "warmup": warmup,
                                  "device_errors": errs}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="nosa", choices=["nosa", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--host-groups", type=int, default=2)
    ap.add_argument("--layers", type=int, default=None, help="override the layer count (profiling captures)")
    ap.add_argument("--micro", type=int, default=0,
                    help="micro-batches on separate streams (default: 2 with offload, else 1)")
    ap.add_argument("--profile-steps", type=int, default=3)
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--dense-only", action="store_true",
                    help="run only the library's dense decode on the workload (for profiling it)")
    ap.add_argument("--no-dense", action="store_true",
                    help="skip the dense-decode comparison of workloads that carry one (stack28-32k)")
    ap.add_argument("--sweep", action="store_true",
                    help="batch x context x k sweep against dense decode (one JSON line per point)")
    ap.add_argument("--ck-bf16", action="store_true", help="store pooled keys as bf16 instead of fp32")
    ap.add_argument("--kq-sweep", action="store_true",
                    help="gamma, misses and throughput against k_q/k, union and fill (one JSON line per point)")
    ap.add_argument("--evict-head", action="store_true",
                    help="compute the eviction logits with the fused synthetic eviction head inside append")
    ap.add_argument("--unfused", action="store_true",
                    help="launch the decode-time append and the select separately (default: one launch)")
    ap.add_argument("--no-fused-step", action="store_true",
                    help="device store: append + select, then decode (two launches) instead of the whole step "
                         "of a layer in one launch")
    ap.add_argument("--split", action="store_true",
                    help="split decode: attend Gamma_e + the local block while select and the cache sync run")
    ap.add_argument("--fill", action="store_true",
                    help="fill reading of the selection: Gamma_e fills the remainder outside Gamma_q")
    args = ap.parse_args()
    c = dict(WORKLOADS[args.workload])
    if args.ck_bf16:
        c["ck_bf16"] = True
    if args.fill:
        c["fill"] = True
    if args.evict_head:
        c["head"] = True
    if args.split:
        c["split"] = True
    if args.unfused:
        c["fuse"] = False
        c["step"] = False
    if args.no_fused_step:
        c["step"] = False
    if args.layers is not None:
        c["layers"] = args.layers
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, c, rank)
        return
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                             device_id=dev)
    nosa.lib()
    if args.sweep:
        run_sweep(args, dev)
        return
    if args.kq_sweep:
        run_kq_sweep(args, dev)
        return
    try:
        if args.dense_only:  # the dense comparator alone (a profiling target)
            dense = run_dense(args, c, rank, world, dev)
            if rank == 0:
                print(json.dumps({"workload": args.workload, "dense": dense}), flush=True)
            return
        line = run_nosa(args, c, rank, world, dev)
        torch.cuda.empty_cache()
        if c.get("dense_compare") and not args.no_dense:
            dense = run_dense(args, c, rank, world, dev)
            if line is not None:
                line["dense"] = dict(dense, sparse_speedup=line["value"] / dense["value"])
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
