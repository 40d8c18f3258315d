"""CPU checks of the bench's accounting, each against a brute-force count over a drawn layout: the
algorithmic bytes of one decode layer (logical, and with a shared prefix's blocks counted once) and
the (query, visible token) pairs of a chunked prefill; the guard that takes a kernel's DRAM traffic
only from a profile summary of the current kernel source and workload; and the end-to-end step's
groups of layers."""
import hashlib
import importlib.util
import os

import numpy as np
import pytest

from paged_kv_cache_470_b200 import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def walk_layout(layout):
    """Every (sequence, token) read through the tables: logical rows, distinct physical rows, and
    distinct table entries per sequence."""
    tables = layout.block_tables.numpy()
    logical, entries, rows = 0, 0, set()
    for b, c in enumerate(layout.context_lens.tolist()):
        t = np.arange(c)
        blk = tables[b, t // 16]
        assert (blk >= 0).all() and (blk < layout.num_blocks).all()
        logical += c
        entries += len(set((t // 16).tolist()))
        rows.update((blk.astype(np.int64) * 16 + t % 16).tolist())
    return logical, len(rows), entries


@pytest.mark.parametrize("cid", [1, 2, 5])
def test_decode_layer_bytes_match_a_walk_of_the_tables(bench, cid):
    cfg = workloads.WORKLOADS[cid]
    layout = workloads.draw_layout(cfg)
    lens = layout.context_lens.tolist()
    share = layout.shares_prefix.tolist()
    logical, unique, entries = walk_layout(layout)
    token = 2 * cfg.Hkv * cfg.D * 2                      # one token's K and V rows of one layer, 16-bit
    lb = bench.layer_bytes(cfg, lens, share, unique_prefix=False)
    lu = bench.layer_bytes(cfg, lens, share, unique_prefix=True)
    assert lb["kv"] == logical * token
    assert lu["kv"] == unique * token
    if cid == 5:
        assert unique < logical                          # the prefix is read by many, stored once
    else:
        assert unique == logical
    B = len(lens)
    assert lb["q_out"] == B * cfg.Hq * cfg.D * 2 * 2     # q read, out written
    assert lb["tables"] == 4 * entries + 4 * B           # table entries read, lengths read
    assert lb["append"] == B * (2 * token + 8)           # new rows read and written, the slot
    assert lb["total"] == lb["kv"] + lb["q_out"] + lb["tables"] + lb["append"]


def brute_pairs(context_lens, chunk_lens):
    total = 0
    for c, n in zip(context_lens, chunk_lens):
        pos = np.arange(c - n, c)                        # the chunk's positions
        total += int(np.less_equal.outer(np.arange(c), pos).sum())
    return total


@pytest.mark.parametrize("key", sorted(workloads.PREFILL_CONFIGS))
def test_prefill_pairs_match_a_causal_mask(bench, key):
    layout = workloads.draw_prefill_layout(workloads.PREFILL_CONFIGS[key])
    c, n = layout.context_lens.tolist(), layout.chunk_lens.tolist()
    assert bench.prefill_pairs(c, n) == brute_pairs(c, n)


def test_prefill_pairs_edge_cases(bench):
    assert bench.prefill_pairs([5], [0]) == 0
    assert bench.prefill_pairs([1], [1]) == 1                 # one token sees itself
    assert bench.prefill_pairs([7], [7]) == 7 * 8 // 2        # a whole prompt: a triangle
    assert bench.prefill_pairs([10, 3], [1, 3]) == 10 + 6     # a decode step, and a short prompt


def test_profiled_traffic_needs_the_current_source_and_workload(bench, tmp_path, monkeypatch):
    src = hashlib.sha256(open(bench.DECODE_SRC, "rb").read()).hexdigest()[:16]
    cfg = workloads.WORKLOADS[2]
    monkeypatch.setattr(bench, "PROFILE_DIR", str(tmp_path))

    def write(h, cid=2, elem="bf16", launch="per_layer"):
        (tmp_path / "p.txt").write_text(f"config_id: {cid}\nelem: {elem}\nlaunch: {launch}\n"
                                        f"decode.cu sha256[:16]: {h}\n"
                                        f"dram_bytes_per_launch: 123456\ndram_bytes_per_layer: 1000\n")
    write(src)
    assert bench.profiled_traffic(cfg, "per_layer") == 123456.0
    assert bench.profiled_traffic(cfg, "layers") is None      # a capture of the other kind of launch
    write(src, launch="layers")
    assert bench.profiled_traffic(cfg, "layers") == 1000.0 * cfg.n_layers   # scaled to the workload's layers
    write("0" * 16)                                           # a capture of another kernel source
    assert bench.profiled_traffic(cfg, "per_layer") is None
    write(src, cid=3)                                         # another workload
    assert bench.profiled_traffic(cfg, "per_layer") is None
    write(src, elem="fp16")                                   # another element type
    assert bench.profiled_traffic(cfg, "per_layer") is None


@pytest.mark.parametrize("L", [1, 2, 3, 4, 5, 7, 8, 24, 32, 80])
def test_e2e_layer_groups_cover_every_layer_once(bench, L):
    """The end-to-end step's groups of layers: contiguous, covering every layer once, none empty, at most 8
    layers, and one layer at each end (its copies cannot overlap a launch) once there are two or more."""
    groups = bench.e2e_groups(L)
    assert groups[0][0] == 0 and groups[-1][1] == L
    assert all(a[1] == b[0] for a, b in zip(groups, groups[1:]))
    sizes = [hi - lo for lo, hi in groups]
    assert all(1 <= sz <= 8 for sz in sizes)
    if L >= 2:
        assert sizes[0] == 1 and sizes[-1] == 1
