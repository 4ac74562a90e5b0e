"""Host logic of bench.py that decides which recorded DRAM traffic a bench line
may carry (no GPU).

A traffic figure from an ncu capture is valid only for the kernel source it was
taken on; bench.py keys each entry of profiles/dram_traffic.json by a hash over
the files that kernel is compiled from.  These tests check that the file lists
cover every header each kernel includes, and that an entry is used only while
its hash matches.
"""

from __future__ import annotations

import json
import os
import re

import bench

CSRC = os.path.join(bench.ROOT, "gqa_mqa_kv_b200", "csrc")

# the header holding each kernel family's device code
MAIN = {"split_mma": "split_mma.cuh", "split_tc": "split_tc.cuh", "prefill_tc": "prefill_tc.cuh"}


def _closure(name: str) -> set[str]:
    seen, todo = set(), [name]
    while todo:
        f = todo.pop()
        if f in seen or not os.path.exists(os.path.join(CSRC, f)):
            continue
        seen.add(f)
        with open(os.path.join(CSRC, f)) as fh:
            todo += re.findall(r'#include "([^"]+)"', fh.read())
    return seen


def test_kernel_files_cover_each_kernels_includes():
    assert set(MAIN) == set(bench.KERNEL_FILES)
    for kernel, header in MAIN.items():
        files = set(bench.KERNEL_FILES[kernel])
        missing = _closure(header) - files
        assert not missing, f"{kernel}: {sorted(missing)} not hashed"
        assert "gqa_decode.cu" in files  # the launch code (tensor maps, grid) is part of what was measured


def test_kernel_files_hash_changes_with_a_file(tmp_path, monkeypatch):
    csrc = tmp_path / "gqa_mqa_kv_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in set(sum(bench.KERNEL_FILES.values(), [])):
        with open(os.path.join(CSRC, name), "rb") as f:
            (csrc / name).write_bytes(f.read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    before = {k: bench.kernel_files_hash(k) for k in bench.KERNEL_FILES}
    assert before == {k: bench.kernel_files_hash(k) for k in bench.KERNEL_FILES}  # deterministic
    (csrc / "tcgen05.cuh").write_bytes((csrc / "tcgen05.cuh").read_bytes() + b"\n")
    after = {k: bench.kernel_files_hash(k) for k in bench.KERNEL_FILES}
    assert after["split_mma"] == before["split_mma"]  # does not include tcgen05.cuh
    assert after["split_tc"] != before["split_tc"]
    assert after["prefill_tc"] != before["prefill_tc"]


def test_recorded_traffic_only_while_the_hash_matches(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    table = {
        "_about": "test table",
        "current": {"kernel_family": "split_mma", "kernel_files_hash": "aaaa", "dram_bytes_per_launch": 123},
        "stale": {"kernel_family": "split_tc", "kernel_files_hash": "bbbb", "dram_bytes_per_launch": 456},
    }
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(table))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_files_hash", lambda kernel: {"split_mma": "aaaa", "split_tc": "cccc"}[kernel])
    assert bench.recorded_traffic("current") == 123.0
    assert bench.recorded_traffic("stale") is None
    assert bench.recorded_traffic("absent") is None


def test_committed_traffic_table_is_well_formed():
    with open(os.path.join(bench.ROOT, "profiles", "dram_traffic.json")) as f:
        table = json.load(f)
    for name, ent in table.items():
        if name.startswith("_"):
            continue
        assert ent["kernel_family"] in bench.KERNEL_FILES, name
        assert re.fullmatch(r"[0-9a-f]{16}", ent["kernel_files_hash"]), name
        launches = ent["launches"]
        assert launches and all(x["read"] > 0 and x["write"] >= 0 for x in launches), name
        # the per-launch figure is at least what one captured launch read
        assert ent["dram_bytes_per_launch"] >= min(x["read"] for x in launches), name
