"""Host logic of bench.py that needs no GPU: the launcher's world-size check, and
the committed ncu traffic record, which the bench line reports only while the
kernel sources still hash to the value it was captured on."""
import json
import os
import re
import types

import pytest

import bench

CSRC = os.path.join(bench.ROOT, "relu_linear_attention_attn_b200", "csrc")


def local_includes(header):
    """Every csrc header that `header` pulls in through #include "…", itself included."""
    seen, todo = set(), [header]
    while todo:
        h = todo.pop()
        if h in seen:
            continue
        seen.add(h)
        with open(os.path.join(CSRC, h)) as f:
            todo += re.findall(r'^\s*#include\s+"([^"]+)"', f.read(), re.M)
    return seen


@pytest.mark.parametrize("top, sources", [("tc_kernels.cuh", bench.KERNEL_SOURCES),
                                          ("mixffn_kernels.cuh", bench.MIXFFN_SOURCES)])
def test_traffic_hash_covers_every_included_source(top, sources):
    # a change to any file the kernels compile from must invalidate the record
    hashed = {os.path.basename(s) for s in sources}
    assert local_includes(top) <= hashed


def test_traffic_record_is_used_only_for_its_sources(monkeypatch):
    with open(os.path.join(bench.ROOT, "profiles", "ncu_traffic.json")) as f:
        rec = json.load(f)
    key = "kv_partials_persistent@4096px-b2-overflow"
    r = rec[key]
    kernel, workload = key.split("@")
    monkeypatch.setattr(bench, "kernel_source_hash", lambda sources=None: r["source_hash"])
    assert bench.ncu_traffic(kernel, workload) == r["dram_read_bytes"] + r["dram_write_bytes"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda sources=None: "0" * 16)
    assert bench.ncu_traffic(kernel, workload) is None
    assert bench.ncu_traffic(kernel, "no-such-workload") is None


def test_launcher_world_must_match_gpus(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    with pytest.raises(SystemExit):
        bench.spawn_ranks_if_needed(types.SimpleNamespace(gpus=1))
    bench.spawn_ranks_if_needed(types.SimpleNamespace(gpus=2))     # agrees: no exit
