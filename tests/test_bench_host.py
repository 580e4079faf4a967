"""Host-side pieces of bench.py: the algorithmic byte count the roofline divides
by, and the rule that a recorded DRAM figure is used only for the kernel source
it was taken on.  No GPU is touched."""
import dataclasses
import json
import os

import numpy as np
import pytest

import bench
import sgmv_inputs as gen


def test_tiny_call_bytes_by_hand():
    # segments of 4, 6 and 7 rows have adapters 0, 2 and 1; the 3-row one is -1.
    # Overwrite: x read (16 x 2 B), the slice written (128 x 2 B), three B tiles
    # of 128 x 16 x 2 B, and three int64 metadata vectors of 4 entries.
    p = gen.tiny()
    byts, flops, rows = bench.call_accounting(p, 0)
    assert rows == 17
    assert byts == 17 * (16 * 2 + 128 * 2) + 3 * 128 * 16 * 2 + 3 * 4 * 8
    assert flops == 2 * 128 * 16 * 17


def test_add_mode_reads_the_old_slice_too():
    p = gen.qkv_prefill()
    q = dataclasses.replace(p, add_inputs=not p.add_inputs)
    (b_add, _, rows), (b_over, _, _) = (bench.call_accounting(p, 0), bench.call_accounting(q, 0))
    if not p.add_inputs:
        b_add, b_over = b_over, b_add
    so = bench.DT_SIZE[p.out_dt]
    assert b_add - b_over == rows * p.calls[0].slice_size * so


def test_inactive_and_out_of_range_adapters_move_nothing():
    p = gen.tiny()
    idx = p.lora_idx.copy()
    idx[:] = [-1, 7, -1, -5]          # 7 and -5 are outside [0, 3)
    q = dataclasses.replace(p, lora_idx=idx)
    byts, flops, rows = bench.call_accounting(q, 0)
    assert rows == 0 and flops == 0
    assert byts == 3 * 4 * 8          # the metadata is still read


def test_step_sums_its_calls():
    p = gen.qkv_prefill()
    per_call = [bench.call_accounting(p, c) for c in range(len(p.calls))]
    assert bench.step_accounting(p) == tuple(sum(v[i] for v in per_call) for i in range(3))


@pytest.mark.parametrize("name", sorted(gen.WORKLOADS))
def test_timed_steps_read_their_inputs_from_hbm(name):
    """Workloads whose buffers fit in L2 rotate through copies of them: between two uses of a copy the
    other copies touched exceed L2 (tiny, at a few kilobytes, cannot and says so)."""
    p = gen.WORKLOADS[name]()
    k, enough = bench.l2_copies(p)
    f = bench.footprint_bytes(p)
    assert 1 <= k <= bench.MAX_COPIES
    if k == 1:
        assert f > bench.L2_BYTES
    elif enough:
        assert (k - 1) * f > bench.L2_BYTES and (k - 2) * f <= bench.L2_BYTES
    else:
        assert name == "tiny" and "not an HBM-bound figure" in bench.l2_text(p)
    if name in ("qkv_shrink", "decode_bgmv"):
        assert k > 1 and enough
    if name in ("qkv_prefill", "mlp_mixed", "long_single", "decode_mix"):
        assert k == 1


def test_graph_chunks_keep_the_rotation():
    for period in range(1, bench.MAX_COPIES + 1):
        c = bench.graph_chunk(period)
        assert c % period == 0 and period <= c <= max(bench.STEPS_PER_GRAPH, period)


def test_every_kernel_family_hashes_existing_sources():
    csrc = os.path.join(bench.ROOT, "segmented_gather_gemm_expand_b200", "csrc")
    for family, files in bench.KERNEL_SOURCES.items():
        assert "common.cuh" in files, family
        for fn in files:
            assert os.path.exists(os.path.join(csrc, fn)), (family, fn)
        h = bench.kernel_source_hash(family)
        assert len(h) == 16 and h == bench.kernel_source_hash(family)
    assert bench.kernel_source_hash("tc") != bench.kernel_source_hash("decode")


def _fake_root(tmp_path, source_text):
    csrc = tmp_path / "segmented_gather_gemm_expand_b200" / "csrc"
    csrc.mkdir(parents=True)
    for files in bench.KERNEL_SOURCES.values():
        for fn in files:
            (csrc / fn).write_text(source_text + fn)
    (tmp_path / "profiles").mkdir()
    return tmp_path


def test_recorded_traffic_only_for_the_source_it_was_taken_on(tmp_path, monkeypatch):
    root = _fake_root(tmp_path, "v1 ")
    monkeypatch.setattr(bench, "ROOT", str(root))
    rec = {"qkv_prefill": {"tc": {"dram_read_bytes_per_launch": 100.0, "dram_write_bytes_per_launch": 23.0,
                                  "kernel_source_hash": bench.kernel_source_hash("tc")}}}
    (root / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("qkv_prefill", "tc") == 123.0
    assert bench.recorded_traffic_split("qkv_prefill", "tc") == {"traffic": 123.0, "read": 100.0, "write": 23.0}
    assert bench.recorded_traffic("qkv_prefill", "decode") is None      # no record for that kernel
    assert bench.recorded_traffic("decode_mix", "tc") is None           # nor for that workload
    # a change to a file outside the family keeps the record
    (root / "segmented_gather_gemm_expand_b200" / "csrc" / "bgmv.cuh").write_text("changed")
    assert bench.recorded_traffic("qkv_prefill", "tc") == 123.0
    # a change to the kernel's own source drops it
    (root / "segmented_gather_gemm_expand_b200" / "csrc" / "tc_kernel.cuh").write_text("changed")
    assert bench.recorded_traffic("qkv_prefill", "tc") is None


def test_comment_and_layout_edits_keep_the_record(tmp_path, monkeypatch):
    root = _fake_root(tmp_path, "int v1; ")
    monkeypatch.setattr(bench, "ROOT", str(root))
    rec = {"qkv_prefill": {"tc": {"dram_read_bytes_per_launch": 4.0, "dram_write_bytes_per_launch": 1.0,
                                  "kernel_source_hash": bench.kernel_source_hash("tc")}}}
    (root / "profiles" / "traffic.json").write_text(json.dumps(rec))
    f = root / "segmented_gather_gemm_expand_b200" / "csrc" / "tc_kernel.cuh"
    f.write_text("// a new comment\nint   v1;\n/* another\n one */ tc_kernel.cuh")
    assert bench.recorded_traffic("qkv_prefill", "tc") == 5.0
    f.write_text("int v2; tc_kernel.cuh")
    assert bench.recorded_traffic("qkv_prefill", "tc") is None


def test_code_only_strips_comments():
    assert bench.code_only("a; // b\n/* c\n d */ e;") == "a; e;"


def test_missing_traffic_file_gives_none(tmp_path, monkeypatch):
    root = _fake_root(tmp_path, "v1 ")
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.recorded_traffic("qkv_prefill", "tc") is None


def test_committed_traffic_records_are_well_formed():
    d = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    for workload, kernels in d.items():
        assert workload in gen.WORKLOADS, workload
        for family, e in kernels.items():
            assert family in bench.KERNEL_SOURCES, family
            assert e["dram_read_bytes_per_launch"] > 0 and e["dram_write_bytes_per_launch"] >= 0
            assert len(e["kernel_source_hash"]) == 16
            assert os.path.exists(os.path.join(bench.ROOT, e["source"].split(" ")[0]))


def _json_lines(text):
    return [json.loads(l) for l in text.splitlines() if l.startswith("{")]


def test_reference_arm_prints_one_contract_line():
    # the reference arm times the oracle on the host cores; no GPU is needed
    import subprocess
    import sys
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3",
                        "--cpu-seconds", "1"], cwd=bench.ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["value"] > 0 and d["higher_is_better"] is True and d["steps"] == 1 and d["warmup"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["name"] == "qkv_prefill"
    # the same workload description our arm prints, so the two lines compare like for like
    import numpy as np  # noqa: F401
    p = gen.WORKLOADS["qkv_prefill"](seed=0)
    assert d["config"] == json.loads(json.dumps(bench.workload_config(p, "qkv_prefill", 1)))


def test_reference_arm_under_two_ranks_prints_once():
    import socket
    import subprocess
    import sys
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3", "--cpu-seconds", "1"],
                       cwd=bench.ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1 and lines[0]["impl"] == "reference"
