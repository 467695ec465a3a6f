"""Host-side arithmetic of bench.py that needs no GPU: the paged-layout study
and the workload naming of the measurement variants."""
import numpy as np

import bench


class _Handle:
    """Stand-in for a cache handle: export_segment returns fixed kept positions."""

    def __init__(self, positions, ring=()):
        self.positions = np.asarray(positions, np.int32)
        self.ring = np.asarray(list(ring) + [-1, -1], np.int32)   # two empty window slots

    def export_segment(self, layer, seq, kv_head):
        return {"pos_c": self.positions, "pos_r": self.ring}


def test_paged_study_counts_blocks_and_partially_dead_ones():
    w = dict(bench.FULL, L=1, Hkv=1)
    # 16-position blocks: positions 0..15 full (1 block), 16..19 (partial), 40 (partial),
    # ring 64..66 (the newest block, still filling: not counted as partially dead)
    h = _Handle(list(range(16)) + [16, 17, 18, 19, 40], ring=[64, 65, 66])
    r = bench.paged_study(h, w, block_sizes=(16,))
    assert r["live_tokens_mean"] == 24
    b = r["block_16"]
    assert b["slots_per_live_token"] == 4 * 16 / 24          # blocks 0, 1, 2, 4
    assert b["partially_dead_block_fraction"] == 2 / 4       # blocks 1 and 2


def test_paged_study_dense_prefix_has_no_dead_space():
    w = dict(bench.FULL, L=1, Hkv=1)
    h = _Handle(range(128))
    r = bench.paged_study(h, w, block_sizes=(32, 64))
    for bs in (32, 64):
        assert r[f"block_{bs}"]["slots_per_live_token"] == 1.0
        assert r[f"block_{bs}"]["partially_dead_block_fraction"] == 0.0


def test_workload_names_mark_the_variants():
    class A:
        layers = None
        prefill = None
        calls = "per-layer"
        compact = "stable"
        score = "random"
        graph = True
    name = bench.workload_name(bench.workload(A))
    for part in ("one attention call per layer", "stable compaction", "random ranking", "single-stream"):
        assert part in name
    class D:
        layers = None
        prefill = None
    base = bench.workload_name(bench.workload(D))
    assert "per layer" not in base and "stable" not in base and "ranking" not in base
