"""Host logic of bench.py that needs no GPU: workload descriptions, the
algorithmic byte counts, the variant matching and source check behind the
roofline `traffic` field, and the reference arm's output line."""
import argparse
import json
import os

import pytest

import bench


def _args(workload, **kw):
    a = dict(workload=workload, layers=None, host_groups=2, seed=0, warmup=1, steps=1, gpus=1)
    a.update(kw)
    return argparse.Namespace(**a)


def test_every_workload_uses_the_fused_launch_and_describes_itself():
    # the device-store workloads run each layer's step in one launch, the offload workload the fused
    # append + select (the cache sync runs between the selection and the decode there)
    for name, c in bench.WORKLOADS.items():
        assert c["fuse"] is True
        assert c.get("step", False) is (not c["offload"])
        text = bench.describe(c, 2)
        want = "append and select fused in one launch" if c["offload"] else "(append, select, decode) in one launch"
        assert want in text and f"context {c['L']}" in text
    assert "append and select fused" in bench.describe(dict(bench.WORKLOADS["stack28-32k"], step=False), 2)


def test_step_bytes_match_the_per_unit_formula():
    class W:  # the fields step_bytes reads
        c = dict(bench.WORKLOADS["offload28-128k"])
        L, units, dense = 28, 128, False
    nb = (131072 - 1) // 64
    per_unit = nb * 4 * 128 * 4 + (16 + 48 + 1) * (32768 + 256)
    assert bench.step_bytes(W) == 28 * 128 * per_unit
    W.c = dict(W.c, ck_bf16=True)  # bf16 pooled keys halve the select stream
    assert bench.step_bytes(W) == 28 * 128 * (nb * 4 * 128 * 2 + 65 * (32768 + 256))


def test_traffic_variants_name_what_changes_a_kernel():
    c = dict(bench.WORKLOADS["offload28-128k"])
    a = _args("offload28-128k")
    assert bench.traffic_variant(c, a, "append_select") == "offload28-128k"
    assert bench.traffic_variant(dict(c, ck_bf16=True), a, "append_select") == "offload28-128k+ck_bf16"
    assert bench.traffic_variant(dict(c, fuse=False), a, "select") == "offload28-128k+unfused"
    assert bench.traffic_variant(dict(c, fuse=False), a, "decode") == "offload28-128k"  # decode is the same kernel
    assert bench.traffic_variant(dict(c, head=True), a, "select") == "offload28-128k+head+unfused"


def test_traffic_is_used_only_while_the_sources_match(tmp_path, monkeypatch):
    c = dict(bench.WORKLOADS["stack28-32k"])
    a = _args("stack28-32k")
    table = {"captures": [
        {"kernel": "decode", "variant": "stack28-32k", "dram_bytes_per_launch": 123.0, "profile": "p.md",
         "sources_sha256": bench.sources_sha("decode")},
        {"kernel": "append_select", "variant": "stack28-32k", "dram_bytes_per_launch": 9.0, "profile": "q.md",
         "sources_sha256": "0" * 64},
    ]}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(table))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # sources_sha reads the kernel sources under ROOT: hash the repository's instead
    repo = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    monkeypatch.setattr(bench, "sources_sha", lambda name, _r=repo: _sha_at(_r, name))
    assert bench.captured_traffic("decode", c, a) == (123.0, "p.md")
    assert bench.captured_traffic("append_select", c, a) == (None, "kernel changed since the capture")
    assert bench.captured_traffic("cache_sync", c, a) == (None, "no capture of this variant")


def _sha_at(repo, name):
    import hashlib
    h = hashlib.sha256()
    for f in bench.KERNEL_SOURCES[name] + ("nosa_common.cuh", "nosa_internal.cuh"):
        with open(os.path.join(repo, "block_sparse_offloadable_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def test_committed_traffic_table_is_well_formed():
    with open(os.path.join(bench.ROOT, "profiles", "dram_traffic.json")) as f:
        table = json.load(f)
    for e in table["captures"]:
        assert e["kernel"] in bench.KERNEL_SOURCES
        assert e["dram_bytes_per_launch"] > 0 and len(e["sources_sha256"]) == 64
        assert os.path.exists(os.path.join(bench.ROOT, e["profile"].split(" ")[0]))


def test_reference_arm_prints_one_contract_line(monkeypatch, capsys):
    monkeypatch.setattr(bench, "oracle_sample", lambda *a, **k: (0.01, 5, "sample"))
    c = dict(bench.WORKLOADS["mha-8k"])
    bench.run_reference(_args("mha-8k"), c, rank=0)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "config", "cpu_baseline", "e2e", "impl"):
        assert key in line, key
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["host"]["logical_cores"] >= 1


def test_algorithmic_bytes_per_launch():
    # stack28-32k, one layer: 64 units at 32K + 9 tokens of context, 65 blocks attended per unit
    c = dict(bench.WORKLOADS["stack28-32k"])
    a = bench.algo_bytes(c, U=64, Bm=32, Lctx=32768 + 9, nsel_mean=65.0)
    nb_c = (32768 + 9 - 1) // 64
    assert a["select"] == 64 * (nb_c * 2048 + 8 * 256)  # fp32 pooled keys: 4 x 128 x 4 B per block
    assert a["decode"] == 64 * 65 * (32768 + 256) + 2 * 32 * 16 * 256
    assert a["append"] == 64 * 516
    assert a["step"] == a["select"] + a["append"] + a["decode"]  # the fused step reads each once
    assert abs(a["step"] / 1e6 - 204.9) < 0.1  # 67.2 MB of pooled keys + 137.6 MB of blocks, queries, outputs
    # bf16 pooled keys halve the select stream; the split decode's passes add up to the one-pass decode
    b = bench.algo_bytes(dict(c, ck_bf16=True), U=64, Bm=32, Lctx=32768 + 9, nsel_mean=65.0)
    assert b["select"] - 64 * 8 * 256 == (a["select"] - 64 * 8 * 256) / 2
    assert a["resident"] + a["rest"] == a["decode"] + 32 * 16 * 256
