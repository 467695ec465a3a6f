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


def test_block_compaction_replay_counts_moved_rows():
    # blocks of 4 slots by position: 0..7 fill blocks 0 and 1 (block 1 is the
    # tail); then 0, 1, 2 are evicted and 8 arrives (a new tail, block 2).
    # Block 0 keeps 1 live token (< 0.5 x 4): its row moves to the tail.
    hist = [[np.arange(8), np.array([3, 4, 5, 6, 7, 8])]]
    r = bench.block_compaction_study(hist, (4,), (0.5,), row_bytes=100)["block_4_theta_0.5"]
    assert r["initial_rows_moved_per_segment"] == 0
    assert r["rows_moved_per_segment_step"] == 1.0
    assert r["bytes_moved_per_segment_step"] == 200.0
    # after the move: block 1 (4 live) and block 2 (8, 3) hold 2 x 4 slots for 6 live tokens
    assert r["slots_per_live_token"] == 8 / 6
    # a threshold of 0 never compacts; an empty block is freed without moves
    r0 = bench.block_compaction_study([[np.arange(8), np.arange(4, 9)]], (4,), (0.0,), 100)["block_4_theta_0.0"]
    assert r0["rows_moved_per_segment_step"] == 0.0
    assert r0["slots_per_live_token"] == 8 / 5
    # a sparse starting layout is compacted once: blocks 0 and 1 hold one token
    # each (positions 1 and 5), block 2 (the tail) holds 8..11
    ri = bench.block_compaction_study([[np.array([1, 5, 8, 9, 10, 11]), np.array([1, 5, 8, 9, 10, 11, 12])]],
                                      (4,), (0.5,), 100)["block_4_theta_0.5"]
    assert ri["initial_rows_moved_per_segment"] == 2
    assert ri["rows_moved_per_segment_step"] == 0.0


def test_amortised_rate_of_a_run():
    r = bench.amortised_rate(16, 256, step1_ms=7.5, steady_ms=0.35)
    ms = (7.5 + 255 * 0.35) / 256
    assert abs(r["ms_per_step"] - ms) < 1e-12
    assert abs(r["value"] - 16 / (ms * 1e-3)) < 1e-6


def test_config_workloads_and_default_steps():
    class A:
        config = 4
        steps = None
        warmup = 10
    w = bench.workload(A)
    assert (w["L"], w["Hq"], w["Hkv"], w["B"], w["T"], w["V"]) == (64, 40, 8, 32, 512, 152064)
    assert w["pyramidal"] and bench.default_steps(w, A) == 4096 - 10
    A.config = 3
    assert bench.default_steps(bench.workload(A), A) == 3000
    class F:
        config = 5
        batch = 64
        ctx = 131072
        gate = "literal"
    w = bench.workload(F)
    assert (w["B"], w["T"], w["mode"], w["fixed"]) == (64, 131072, "fixed", 2048)
    assert "B=2048 = 4 sinks + 512 window + 1532 top-k" in bench.workload_name(w)
    class G:
        gate = "literal"
    assert "pseudo-code line" in bench.workload_name(bench.workload(G))


def test_oracle_baseline_runs_one_segment_per_process():
    class A:
        config = 1
    w = bench.workload(A)
    r = bench.oracle_sample(w, seconds=0.5, workers=2)
    assert r["cores"] == 2 and r["value"] > 0 and r["unit"] == "tok/s"
    assert "2 single-threaded oracle processes" in r["sample"]
