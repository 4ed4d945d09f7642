"""Host logic of bench.py on the CPU: the algorithmic-byte model behind every
roofline figure, checked against the bytes counted by hand for the 32k batched
workload (256 (batch, kv-head) pairs, 503 candidate blocks, 25 selected blocks),
and the traffic records' tie to the kernel sources."""

import bench
from workloads import WORKLOADS


def test_byte_model_of_the_32k_batched_workload():
    w = WORKLOADS["batched_needles_32k"]
    pairs, cand, n_sel = 32 * 8, 503, 25          # 32768 tokens: blocks [1, 504) compete
    q_bytes = 32 * 32 * 128 * 2
    bm = bench.byte_model(w, n_sel)
    rec = 9 * 128 * 2                             # mu + 8 columns of U, bf16
    # statistics: one 64 x 128 bf16 block in, one record out, per pair
    assert bm["stats"] == pairs * (64 * 128 * 2 + rec)
    # selection: every candidate record, the queries, the scores written and
    # the selected lists (count + indices)
    assert bm["select"] == pairs * cand * rec + q_bytes + pairs * cand * 4 + pairs * 4 * 26
    assert bm["select"] == 297_485_312
    # decode: K and V of the selected blocks, the queries, the lists, fp32 out + lse
    assert bm["decode"] == (pairs * 25 * 64 * 128 * 2 * 2 + q_bytes + pairs * 4 * 26
                            + 32 * 32 * 129 * 4)
    assert bm["decode"] == 210_532_352


def test_byte_model_with_fp4_records():
    w = WORKLOADS["batched_needles_32k"]
    bm = bench.byte_model(w, 25, rec=800)
    assert bm["select"] == 256 * 503 * 800 + 32 * 32 * 128 * 2 + 256 * 503 * 4 + 256 * 4 * 26
    assert bm["decode"] == bench.byte_model(w, 25)["decode"]


def test_traffic_record_is_dropped_when_the_kernel_changes(monkeypatch):
    real = bench.recorded_traffic("select.cu", "batched_needles_32k")
    monkeypatch.setattr(bench, "source_hash", lambda name: "0" * 16)
    assert bench.recorded_traffic("select.cu", "batched_needles_32k") is None
    assert real is None or real > 0


def test_oracle_baseline_runs_on_several_cores_at_once():
    # two spawn-started processes, each decoding its own (batch, kv-head) pair
    # of a small workload; the rate sums their queries over the slower one's time
    w = WORKLOADS["tiny_4k"].scaled(batch=2)
    value, steps, dt, pairs = bench.oracle_rate(w, 2, steps=3, warmup=1)
    assert steps == 3 and dt > 0 and value > 0
    assert pairs == [(0, 0), (1, 0)]
    one, steps1, _, _ = bench.oracle_rate(w, 1, steps=2, warmup=1)
    assert steps1 == 2 and one > 0
    assert bench.oracle_cores() >= 1
