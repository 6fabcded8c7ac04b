"""Host logic of bench.py that decides what a JSON line reports, on CPU: the
DRAM-traffic record is used only for the kernel source it was taken on, the
committed records are self-consistent, the residual-latency ratio of the
comparator workload honours its noise floor, and the one-launch decode policy
matches the C-ABI's limits."""
import json
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fake_tree(tmp_path, src=b"// kernel v1\n"):
    csrc = tmp_path / "w4a4_rank_gemm_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cuh").write_bytes(src)
    (tmp_path / "profiles").mkdir()
    return csrc


def test_traffic_record_only_for_the_kernel_it_was_taken_on(tmp_path, monkeypatch):
    csrc = _fake_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_hash(["k.cuh"])
    rec = {"w": {"kernel_hash": h, "bytes_per_launch": 1234}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("w", ["k.cuh"]) == 1234
    assert bench.recorded_traffic("other", ["k.cuh"]) is None
    # any change to the source, a comment included, invalidates the record
    (csrc / "k.cuh").write_bytes(b"// kernel v2\n")
    assert bench.kernel_hash(["k.cuh"]) != h
    assert bench.recorded_traffic("w", ["k.cuh"]) is None


def test_traffic_record_missing_or_unreadable(tmp_path, monkeypatch):
    _fake_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("w", ["k.cuh"]) is None
    (tmp_path / "profiles" / "traffic.json").write_text("{not json")
    assert bench.recorded_traffic("w", ["k.cuh"]) is None


def test_committed_traffic_records_are_means_of_their_launches():
    d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    assert d, "no traffic records"
    for name, rec in d.items():
        per = list(rec["per_launch"].values())
        assert rec["bytes_per_launch"] == pytest.approx(sum(per) / len(per), rel=1e-9), name
        assert len(rec["kernel_hash"]) == 16
        assert os.path.exists(os.path.join(ROOT, rec["summary"])), rec["summary"]


def test_residual_ratio_and_noise_floor():
    # a: main 100 us, SERQ adds 4, the comparator adds 20; b: main 50, SERQ 1, comparator 9
    t = {("a", 0): 100.0, ("a", 1): 104.0, ("a", 2): 120.0,
         ("b", 0): 50.0, ("b", 1): 51.0, ("b", 2): 59.0}
    r = bench.residual_summary(t)
    assert list(r["per"]) == ["a", "b"]
    assert r["sum_main"] == 150.0 and r["sum_serq"] == 5.0 and r["sum_two"] == 29.0
    assert r["ratio"] == pytest.approx(29.0 / 5.0) and not r["at_floor"]
    assert r["per"]["a"]["two_factor_residual_us"] == 20.0
    # SERQ's residual below 1% of the main products (here even negative from
    # timing noise): the ratio divides by the floor and says so
    t2 = dict(t)
    t2[("a", 1)], t2[("b", 1)] = 100.2, 49.9
    r2 = bench.residual_summary(t2)
    assert r2["at_floor"]
    assert r2["ratio"] == pytest.approx(29.0 / 1.5)


@pytest.mark.parametrize("decode,grouped,M,K,want", [
    (True, True, 1, 4096, True), (True, True, 8, 4096, True), (True, True, 8, 4097, False),
    (True, True, 9, 4096, False), (True, True, 16, 4096, False), (True, False, 4, 4096, False),
    (False, True, 4, 4096, False), (True, True, 4, 11008, False)])
def test_one_launch_decode_policy(decode, grouped, M, K, want):
    assert bench.fuses_act_quantize(decode, grouped, M, K) is want


def test_one_launch_limits_match_the_header():
    # the policy's M <= 8, K <= 4096 are the limits serq.h documents for the
    # single-launch form of serq_linear_group_act
    h = open(os.path.join(ROOT, "include", "serq.h")).read()
    i = h.index("serq_linear_group_act")
    doc = h[max(0, i - 3000):i + 3000]
    assert "M <= 8" in doc or "M ≤ 8" in doc
    assert "4096" in doc
