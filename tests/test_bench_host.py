"""Host-side helpers of bench.py (no GPU): the head split, the job value of
both multi-GPU modes, the workload overrides and the per-stage algorithmic work."""

import types

import pytest

import bench
from synthetic import WORKLOADS


@pytest.mark.parametrize("world,heads", [(1, 16), (2, 16), (3, 16), (8, 16), (5, 7), (7, 7)])
def test_head_slices_partition_the_heads(world, heads):
    got = [bench.head_slice(world, r, heads) for r in range(world)]
    assert got[0][0] == 0 and got[-1][1] == heads
    for (a0, a1), (b0, b1) in zip(got, got[1:]):
        assert a1 == b0
    sizes = [h1 - h0 for h0, h1 in got]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def test_more_ranks_than_heads_is_refused():
    with pytest.raises(ValueError):
        bench.head_slice(3, 0, 2)


def test_job_value_modes():
    assert bench.job_value(4, 1000, 500.0) == pytest.approx(4 * 1000 / 0.5)
    assert bench.job_value(4, 1000, 500.0, "heads") == pytest.approx(1000 / 0.5)


def test_rank_workloads():
    wl = WORKLOADS["medium"]
    assert bench.rank_workload(wl, 0) == wl
    assert bench.rank_workload(wl, 2).seed == wl.seed + 2000
    assert bench.rank_workload(wl, 2, "heads") == wl


def test_workload_overrides():
    args = types.SimpleNamespace(workload="pages", top_k=128, keep=1)
    wl = bench.chosen_workload(args)
    assert (wl.top_k, wl.keep, wl.n_frames) == (128, 1, 1000)
    cfg = bench.workload_config(wl)
    assert cfg["keep"] == "reference" and cfg["top_k"] == 128 and "frame 0" in cfg["workload"]


def test_stage_work_at_the_pages_workload():
    z = types.SimpleNamespace(T=1_374_000, Tc=105_000, NB=100_000, NS=5000, NK=5000, B0=0)
    work = bench.stage_work(z, 16, 64, 64)
    assert work["compressed_attn"] == ("tensor", 4 * 105_000 ** 2 * 16 * 64, "flop")
    assert work["kept_attn"] == ("tensor", 4 * 1_374_000 * 5000 * 16 * 64, "flop")
    # 1369 valid tokens in 100 blocks per frame: 13.69 per selected block on average
    assert work["selected_gate"][0] == "gather"
    assert work["selected_gate"][1] == 16 * 105_000 * 64 * 1_369_000 // 100_000 * 64 * 2 * 2
    # Q, K, V read once: 3 x 1,374,000 x 16 x 64 x 2 bytes, plus the pooled and kept writes
    assert work["pool"][1] > 3 * 1_374_000 * 16 * 64 * 2


def test_selected_bytes_counts_valid_tokens_of_each_selected_block():
    import torch
    from sparse_global_attention_view_b200 import Shape
    # 6 x 7 grid, P = 4: blocks (0,0) 16 tokens, (0,1) 4 x 3 = 12, (1,0) 2 x 4 = 8, (1,1) 2 x 3 = 6
    shape = Shape(n_frames=2, n_special=1, hp=6, wp=7, n_heads=2, top_k=3)
    sel = torch.tensor([[[0, 1, -1], [4, 7, 3]], [[2, -1, -1], [5, 6, 0]]], dtype=torch.int32)
    tokens = (16 + 12) + (16 + 6 + 6) + 8 + (12 + 8 + 16)
    assert bench.selected_bytes(sel, None, shape) == tokens * 64 * 2 * 2


@pytest.mark.parametrize("world,parallel", [(1, "heads"), (1, "replicas"), (2, "heads"), (8, "heads"),
                                            (4, "replicas")])
def test_both_arms_describe_the_same_config(world, parallel):
    wl = WORKLOADS["pages"]
    cfg = bench.workload_config(wl, bench.l2_note(wl, world, parallel), bench.parallelism_of(wl, world, parallel))
    assert "l2" in cfg and "L2" in cfg["l2"]
    assert cfg["parallelism"].startswith("heads" if (world > 1 and parallel == "heads") else "replicas")


def test_recorded_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    # DRAM bytes from the committed ncu summary count only while the kernel's
    # source is the one they were captured from
    import json
    csrc = tmp_path / "sparse_global_attention_view_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = csrc / "k.cu"
    src.write_text("__global__ void k() {}\n")
    rec = {"k.cu@pages": {"bytes_per_launch": 123, "source_sha": bench.source_hash(str(src))}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("k.cu", "pages") == 123
    assert bench.recorded_traffic("k.cu", "medium") is None
    src.write_text("__global__ void k() { }\n")
    assert bench.recorded_traffic("k.cu", "pages") is None


def test_committed_traffic_matches_the_committed_sources():
    # every record in profiles/traffic.json names a kernel source that exists
    import json
    import os
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    for key, r in rec.items():
        f, wl = key.split("@")
        path = os.path.join(bench.ROOT, "sparse_global_attention_view_b200", "csrc", f)
        assert os.path.exists(path), key
        assert r["bytes_per_launch"] == r["dram_bytes_read"] + r["dram_bytes_write"], key
        assert f in bench.STAGE_SOURCE.values(), key
