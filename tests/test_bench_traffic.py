"""bench.py's bookkeeping of recorded DRAM traffic, on CPU: the entry key of a workload, the
kernel whose sources an entry is hashed over, the rule that says which kernel a several-token
step runs, and the round trip from an ncu CSV to profiles/traffic.json and back (in a scratch
copy of the tree, so the committed entries are untouched)."""
import json
import os
import shutil
from dataclasses import replace

import pytest

import bench
from load_balanced_split_step_b200 import workloads as W

CSRC = ("attention.cu", "attention_tcm.cu", "attention_common.cuh", "hpc_common.cuh")


@pytest.fixture()
def scratch_root(tmp_path, monkeypatch):
    """A copy of the kernel sources and an empty profiles/ folder, as bench.ROOT."""
    src = os.path.join(bench.ROOT, "load_balanced_split_step_b200", "csrc")
    dst = tmp_path / "load_balanced_split_step_b200" / "csrc"
    dst.mkdir(parents=True)
    for name in CSRC:
        shutil.copy(os.path.join(src, name), dst / name)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def test_traffic_keys():
    assert bench.traffic_key("heavy", 1) == "heavy"
    assert bench.traffic_key("heavy", 4) == "heavy_q4"
    assert bench.traffic_key("extreme", 2) == "extreme_q2"


def test_each_entry_hashes_its_own_kernel(scratch_root):
    one = {bench.kernel_source_hash(k) for k in ("extreme", "uniform", "heavy", "fp8", "heavy_q2")}
    assert len(one) == 1  # one-token and two-token steps run attention.cu
    q4 = bench.kernel_source_hash("heavy_q4")
    assert q4 not in one
    tcm = scratch_root / "load_balanced_split_step_b200" / "csrc" / "attention_tcm.cu"
    tcm.write_text(tcm.read_text() + "\n// changed\n")
    assert bench.kernel_source_hash("heavy_q4") != q4  # the tcgen05 kernel's entry goes stale
    assert bench.kernel_source_hash("extreme") in one  # the others stay valid
    common = scratch_root / "load_balanced_split_step_b200" / "csrc" / "attention_common.cuh"
    common.write_text(common.read_text() + "\n// changed\n")
    assert bench.kernel_source_hash("extreme") not in one  # a shared header touches every entry


def test_which_kernel_a_several_token_step_runs():
    heavy = W.config_spec("heavy")  # bf16, head_dim 128, 64 / 8 heads
    assert not bench.uses_tcgen05_multi(heavy, "default")  # one token
    assert bench.uses_tcgen05_multi(replace(heavy, q_len=4), "default")
    assert bench.uses_tcgen05_multi(replace(heavy, q_len=3), "default")
    assert not bench.uses_tcgen05_multi(replace(heavy, q_len=2), "default")  # mma.sync by default
    assert bench.uses_tcgen05_multi(replace(heavy, q_len=2), "tcgen05")
    assert not bench.uses_tcgen05_multi(replace(heavy, q_len=4), "mma")
    assert not bench.uses_tcgen05_multi(replace(heavy, q_len=4, kv_dtype="e4m3"), "default")
    assert not bench.uses_tcgen05_multi(replace(heavy, q_len=4, num_heads=128), "default")  # 4 x 16 rows > 32


def _ncu_csv(path, read_bytes, write_bytes):
    rows = ['"ID","Kernel Name","Metric Name","Metric Unit","Metric Value"',
            f'"0","decode_attention_tcm_kernel","dram__bytes_read.sum","byte","{read_bytes:,}"',
            f'"0","decode_attention_tcm_kernel","dram__bytes_write.sum","byte","{write_bytes:,}"']
    path.write_text("==PROF== a line ncu prints first\n" + "\n".join(rows) + "\n")


def test_record_and_load_round_trip(scratch_root):
    csv = scratch_root / "dram.csv"
    _ncu_csv(csv, 1_000_000_000, 4_000_000)
    args = bench.parse_args(["--workload", "heavy", "--requests", "16", "--q-len", "4", "--record-traffic", str(csv)])
    line = bench.record_traffic(args)
    assert line["workload"] == "heavy_q4"
    sample = bench.workload_spec(args)
    full = replace(W.config_spec("heavy"), q_len=4)
    scale = W.algorithmic_bytes(full) / W.algorithmic_bytes(sample)
    assert line["traffic_bytes_per_launch"] == int(round(1_004_000_000 * scale))
    assert line["algorithmic_bytes_full"] == int(W.algorithmic_bytes(full))
    assert line["source_sha256_16"] == bench.kernel_source_hash("heavy_q4")
    assert bench.load_traffic("heavy_q4") == line["traffic_bytes_per_launch"]
    assert bench.load_traffic("heavy") is None  # no entry
    # a changed kernel drops its entry
    tcm = scratch_root / "load_balanced_split_step_b200" / "csrc" / "attention_tcm.cu"
    tcm.write_text(tcm.read_text() + "\n// changed\n")
    assert bench.load_traffic("heavy_q4") is None
    saved = json.loads((scratch_root / "profiles" / "traffic.json").read_text())
    assert set(saved) == {"heavy_q4"}


def test_record_refuses_a_non_default_several_token_kernel(scratch_root):
    csv = scratch_root / "dram.csv"
    _ncu_csv(csv, 1000, 10)
    args = bench.parse_args(["--workload", "heavy", "--requests", "4", "--q-len", "4", "--multi-kernel", "mma",
                             "--record-traffic", str(csv)])
    with pytest.raises(SystemExit):
        bench.record_traffic(args)


def test_committed_entries():
    """profiles/traffic.json holds the five measured workloads: read + write bytes scaled to the
    full size, within 2% of the algorithmic bytes (no re-reads), each with a source hash. (An
    entry whose hash no longer matches the sources is reported as null by the bench.)"""
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        data = json.load(f)
    assert {"extreme", "uniform", "heavy", "fp8", "heavy_q4"} <= set(data)
    for key in ("extreme", "uniform", "heavy", "fp8", "heavy_q4"):
        e = data[key]
        assert len(e["source_sha256_16"]) == 16
        measured = (e["read_bytes"] + e["write_bytes"]) * e["scale_to_full"]
        assert abs(measured - e["traffic_bytes_per_launch"]) <= 1e-6 * measured + 1, key
        ratio = e["traffic_bytes_per_launch"] / e["algorithmic_bytes_full"]
        assert 1.0 <= ratio < 1.02, (key, ratio)
