"""bench.py's byte accounting, checked against the pages' numbers and by hand."""

import json
import os

import numpy as np

import bench
from paged_kv_cache_399_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "page_numbers.json")


def test_kv_bytes_per_token_matches_the_pages():
    data = json.load(open(GOLDEN))
    for row in data["kv_bytes"]:
        per_tok = bench.kv_bytes_per_token(row["layers"], row["kv_heads"], row["head_dim"],
                                           row["bytes_per_value"])
        if "bytes_per_token" in row:
            assert per_tok == row["bytes_per_token"], row["cite"]
        if "gib_per_request" in row:
            assert per_tok * row["context"] / 2 ** 30 == row["gib_per_request"], row["cite"]


def test_decode_bytes_by_hand_and_shared_prefix_counted_once():
    w = workloads.build_workload("t", 5, [16, 20], 1, 4, 2, 64)
    kv = (16 + 20) * 2 * 64 * 2 * 2
    qo = 2 * 2 * 1 * 4 * 64 * 2
    assert bench.decode_bytes(w) == kv + qo + (1 + 2) * 4 + 2 * 4
    g = workloads.build_workload("g", 6, [40, 45], 1, 4, 2, 64, share_groups=[([0, 1], 32)])
    logical = bench.decode_bytes(g, unique=False)
    unique = bench.decode_bytes(g)
    assert logical - unique == 32 * 2 * 64 * 2 * 2   # the 32 shared tokens once, not twice


def test_prefix_sharing_workload_unique_bytes():
    w = workloads.prefix_sharing()
    assert np.all(w.block_tables[0:8, :128] == w.block_tables[0, :128])
    assert bench.decode_bytes(w) < bench.decode_bytes(w, unique=False) / 4


def test_copy_bytes_by_hand_and_fork_workload():
    w = workloads.cow_fork()
    # every pair moves one 16-token block of 8 kv heads x 128 dims (32 KB) in each pool,
    # read once and written once
    assert w.block_bytes == 16 * 8 * 128 * 2
    assert bench.copy_bytes(w) == w.num_pairs * 2 * 2 * 32768
    # the fork copies only partly filled last blocks, once per sample but the first
    src, counts = np.unique(w.mapping[:, 0], return_counts=True)
    assert np.all(counts == 7)
    assert len(set(w.mapping[:, 1].tolist())) == len(w.mapping)
    assert not set(w.mapping[:, 0].tolist()) & set(w.mapping[:, 1].tolist())
    padded = workloads.CopyWorkload("p", 0, 8, 128, 16, 4, np.array([[0, 1], [-1, 2]], dtype=np.int64),
                                    w.key_cache[:4], w.value_cache[:4])
    assert bench.copy_bytes(padded) == 2 * 2 * 32768   # the padding pair moves nothing


def test_copy_traffic_keyed_by_the_copy_sources_only():
    assert bench.source_hash() != bench.source_hash(bench.COPY_SOURCES)
    assert set(bench.DECODE_SOURCES).isdisjoint(bench.COPY_SOURCES)
    csrc = os.path.join(os.path.dirname(bench.__file__), "paged_kv_cache_399_b200", "csrc")
    assert set(bench.DECODE_SOURCES) | set(bench.COPY_SOURCES) | set(bench.FP8_SOURCES) == set(os.listdir(csrc))


def test_reference_arm_prints_the_contract_line(capsys):
    """bench.py --impl reference (the fp64 oracle on host cores) prints one JSON line with
    the contract's keys, for a decode workload and for a copy workload."""
    for wl, steps in (("tiny", 2), ("cow_fork", 1)):
        assert bench.main(["--impl", "reference", "--workload", wl, "--steps", str(steps), "--warmup", "3"]) == 0
        lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
        assert len(lines) == 1
        d = json.loads(lines[0])
        for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                    "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "impl"):
            assert key in d, (wl, key)
        assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
        assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
