"""bench.py's host-side pieces on CPU: the algorithmic byte model the
roofline divides by, the workload string both arms print, the guard that
reports the captured verify traffic only for the kernel code it was captured
on, and the layout of the end-to-end leg's staging buffer."""

import os
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


class _WL:
    B, Hq, Hkv, D, P, S, W, gamma = 1, 16, 2, 256, 64, 4, 4096, 3


def test_algorithmic_bytes_closed_forms():
    n = 1048576
    # verify: K and V of n tokens x 2 KV heads x 256 bf16, the page table,
    # 4 x 16 bf16 query rows and their fp32 outputs (+ lse)
    want = n * 2 * 2 * 256 * 2 + (n // 64) * 4 + 4 * 16 * 256 * 2 + 4 * 16 * 257 * 4
    assert bench.algorithmic_bytes(_WL, "verify", [n]) == want == 2147647744
    # native draft: one query
    assert bench.algorithmic_bytes(_WL, "full", [n]) == n * 2048 + (n // 64) * 4 + 16 * 256 * 2 + 16 * 257 * 4
    # windowed: S + W ring slots (K, V and a tag each), whatever the context
    win = bench.algorithmic_bytes(_WL, "windowed", [n])
    assert win == bench.algorithmic_bytes(_WL, "windowed", [10 * n]) == 4100 * (2048 + 4) + 16 * 256 * 2 + \
        16 * 257 * 4
    # a batch sums its sequences
    assert bench.algorithmic_bytes(_WL, "full", [n, n // 2]) == (bench.algorithmic_bytes(_WL, "full", [n]) +
                                                                bench.algorithmic_bytes(_WL, "full", [n // 2]))


def test_workload_strings():
    assert bench.workload_desc(bench.parse([])) == (
        "1m: batch 1, 16q/2kv heads, D=256, page 64, ctx 1048576, S=4, W=4096, gamma=3, 10 verify layers")
    assert "ctx 789675/895224/279959/897535" in bench.workload_desc(bench.parse(["--config", "ragged4"]))
    assert "ctx 65536" in bench.workload_desc(bench.parse(["--ctx", "65536"]))


def test_recorded_traffic_matches_the_current_kernel():
    # the committed capture belongs to the committed kernel code
    assert bench.kernel_code_hash() == bench.VERIFY_TRAFFIC["sha256"]
    t = bench.verify_traffic(1048580)
    assert t is not None and 1.0 < t / (1048580 * 2048) < 1.02


def test_traffic_guard_follows_the_kernel_code(tmp_path, monkeypatch):
    # a figure recorded against the current sources, 100 bytes per token
    monkeypatch.setitem(bench.VERIFY_TRAFFIC, "sha256", bench.kernel_code_hash())
    monkeypatch.setitem(bench.VERIFY_TRAFFIC, "tokens", 1000)
    monkeypatch.setitem(bench.VERIFY_TRAFFIC, "read_bytes", 100000)
    monkeypatch.setitem(bench.VERIFY_TRAFFIC, "write_bytes", 500)
    assert bench.verify_traffic(4000) == pytest.approx(400500)  # reads scaled by tokens, writes as captured
    # a copy of the sources: a comment edit keeps the figure, a code edit drops it
    for rel in bench.VERIFY_TRAFFIC["sources"]:
        os.makedirs(tmp_path / os.path.dirname(rel), exist_ok=True)
        shutil.copy(os.path.join(ROOT, rel), tmp_path / rel)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    src = tmp_path / bench.VERIFY_TRAFFIC["sources"][0]
    text = src.read_text()
    src.write_text("// a new comment\n" + text)
    assert bench.verify_traffic(4000) == pytest.approx(400500)
    src.write_text(text.replace("kRescaleLog2 = 8.f", "kRescaleLog2 = 7.f"))
    assert bench.verify_traffic(4000) is None
    monkeypatch.setitem(bench.VERIFY_TRAFFIC, "read_bytes", None)
    assert bench.verify_traffic(4000) is None


def test_whole_job_time_per_step():
    assert bench.whole_job_us_per_step(40.0, 10, 1) == pytest.approx(4000.0)
    assert bench.whole_job_us_per_step(40.0, 10, 4) == pytest.approx(1000.0)


def test_staging_layout_slots_are_aligned_and_disjoint():
    shapes = {"q": (3 * 16 * 256, 2), "len": (1, 4), "k": (4 * 2 * 256, 2), "n": (3, 4)}
    offs, total = bench.staging_layout(shapes)
    spans = sorted((offs[k], offs[k] + n * e) for k, (n, e) in shapes.items())
    assert all(o % 256 == 0 for o in offs.values())
    assert all(a_end <= b_start for (_, a_end), (b_start, _) in zip(spans, spans[1:]))
    assert spans[-1][1] <= total < spans[-1][1] + 256
    assert total == sum(-(-n * e // 256) * 256 for n, e in shapes.values())
