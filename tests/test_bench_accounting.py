"""The numerators of bench.py's roofline figures, pinned to hand counts.

Every fraction the bench prints divides an algorithmic byte or FLOP count by a
measured time, so the counts themselves are checked here, on the CPU:

* bytes per launch, written out from the tensors each call must read and
  write at the bench's workloads (the same figures the committed profiles
  quote);
* the MMA count of the prefill kernel on small cases worked out tile by
  tile from the order the kernel issues its products (a2 Q K^T, a4 P V, a5
  Q S, a6 K^T V; the segment-sum pass; S as bf16 hi + lo past 32768 tokens);
* the blocked FLOP definitions against their closed forms;
* the recorded DRAM-traffic table: each entry carries a 16-hex-digit source
  hash and a per-launch byte count no smaller than the algorithmic bytes of
  its workload less the share L2 can serve.
"""
import json
import os

import pytest

import bench

D = 128
UNIT = 2 * 128 ** 3  # FLOPs of one 128 x 128 x 128 product


def test_prefill_bytes_at_the_main_workload():
    # q, k, v read and out written: 4 x 32768 x 64 x 128 bf16; one fp32 128 x 128 state per head
    assert bench.prefill_bytes(32768 * 64, 64, 1) == 4 * 32768 * 64 * 128 * 2 + 64 * 128 * 128 * 4
    assert bench.prefill_bytes(32768 * 64, 64, 1) == 2_151_677_952


def test_backward_aggregate_and_decode_bytes():
    assert bench.backward_bytes(32768 * 64) == 3_758_096_384          # q, k, v, dout in; dq, dk, dv out
    assert bench.aggregate_bytes(32768 * 64, 64) == 1_077_936_128      # k, v in; 64 fp32 sums out
    # 256 x 64 states read and written (fp32), q, k, v read and o written (bf16)
    assert bench.decode_bytes(256 * 64) == 256 * 64 * (2 * 128 * 128 * 4 + 4 * 128 * 2) == 2_164_260_864


def test_blocked_flop_definitions():
    th, bk = 1000, 128
    assert bench.prefill_alg_flops(th, bk) == th * (2 * 129 * D + 4 * D * D)
    assert bench.prefill_dense_flops(th, bk) == th * (4 * 128 * D + 4 * D * D)
    # the dense count exceeds the blocked definition by the masked half of each score tile
    assert bench.prefill_dense_flops(th, bk) - bench.prefill_alg_flops(th, bk) == th * 2 * (bk - 1) * D


@pytest.mark.parametrize("lengths,heads,seg,want,block,units", [  # units per head
    # one 128-token tile, one segment, final state wanted: Q K^T, P V, Q S, K^T V
    ([128], 1, 1024, True, 128, 4),
    # ... without the final state the last tile's K^T V is skipped
    ([128], 1, 1024, False, 128, 3),
    # two segments of one tile: the first adds its segment-sum K^T V, not its own a6
    #   segment 0: 3 + 1 (segment sum); segment 1: 4
    ([256], 1, 128, True, 128, 8),
    # a ragged 300-token sequence in one segment: three tiles, a6 after each but the last, plus the final one
    ([300], 2, 1024, True, 128, 3 * 3 + 3),
    # an empty sequence adds nothing
    ([0, 128], 1, 1024, True, 128, 4),
    # 64-row blocks, one tile: Q K^T, P V, Q S twice (once per 64-row block), K^T V in two halves
    ([128], 1, 1024, True, 64, 2 + 2 + 1),
    # 256-row blocks, one full pair: three score steps (Q K^T and P V each), Q S per tile, K^T V per tile
    ([256], 1, 1024, True, 256, 6 + 2 + 2),
    # a segment ending past 32768 tokens reads S as bf16 hi + lo: Q S twice
    ([32768 + 128], 1, 32768 + 128, True, 128, 257 * 2 + 257 * 2 + 257),
])
def test_prefill_mma_units(lengths, heads, seg, want, block, units):
    assert bench.prefill_mma_flops(lengths, heads, seg, want_state=want, block=block) == units * UNIT * heads


def test_prefill_mma_count_at_the_main_workload():
    # 32 segments of 8 tiles per head: 4 units per tile, less the last tile's a6 in the
    # 31 segments with a successor, plus their 8-tile segment-sum passes
    per_head = 32 * 8 * 4 - 31 + 31 * 8
    assert bench.prefill_mma_flops([32768], 64, 1024) == per_head * UNIT * 64


def test_recorded_traffic_table_is_well_formed():
    path = os.path.join(bench.ROOT, "profiles", "dram_traffic.json")
    with open(path) as f:
        rec = json.load(f)
    assert set(rec) <= set(bench.KERNEL_SOURCES)
    alg = {
        "prefill_B1_H64_N32768": bench.prefill_bytes(32768 * 64, 64, 1),
        "backward_B1_H64_N32768": bench.backward_bytes(32768 * 64),
        "prefill_B1_H8_N1048576": bench.prefill_bytes(1048576 * 8, 8, 1),
    }
    for kernel, entries in rec.items():
        for workload, e in entries.items():
            h = e["source_hash"]
            assert len(h) == 16 and all(c in "0123456789abcdef" for c in h), (kernel, workload)
            assert e["bytes_per_launch"] > 0, (kernel, workload)
            if workload in alg:
                # DRAM traffic can undercut the algorithmic bytes only by what L2 keeps between calls
                assert e["bytes_per_launch"] >= 0.9 * alg[workload], (kernel, workload)


def test_source_hash_ignores_comments(tmp_path, monkeypatch):
    src = tmp_path / "linear_attention_blocked_b200" / "csrc"
    src.mkdir(parents=True)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "k", ("a.cuh",))
    (src / "a.cuh").write_text("int x = 1;  // one\n\n// a note\nint y = 2;\n")
    h1 = bench.kernel_source_hash("k")
    (src / "a.cuh").write_text("int x = 1;  // another comment\n// more\nint y = 2;\n")
    assert bench.kernel_source_hash("k") == h1
    (src / "a.cuh").write_text("int x = 1;\nint y = 3;\n")
    assert bench.kernel_source_hash("k") != h1
