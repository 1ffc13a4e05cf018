"""Host-side pieces of bench.py that the reported numbers rest on, on CPU.

* The roofline's algorithmic work counts attended (query row, key) pairs
  from a realised selection (`segment_pairs`).  Here it is checked against
  the oracle's own definition of each query's key set (routed groups plus
  the causal own block), counted one query at a time, and against the
  active-segment restriction that the dK/dV work uses.
* The DRAM traffic it reports comes from a committed ncu summary only while
  that summary was taken on the current kernel sources.
* Routing work is credited only to the kernels whose path a segment takes.
* Both arms describe the same workload in their JSON line.
"""
import importlib.util
import json
import os

import numpy as np
import pytest

from oracle import hga_oracle as orc

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test",
                                                  os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


class W:
    """The fields segment_pairs reads."""
    group_heads = 4
    head_dim = 128


def random_selection(rng, n_kv, n_qb, k_g, q_begin):
    sel = np.full((1, n_kv, n_qb, k_g), -1, np.int32)
    for h in range(n_kv):
        for j in range(n_qb):
            own_blk = (q_begin + 64 * j) // 64
            cands = np.arange(own_blk * 8)          # every group before the own block
            n = min(int(rng.integers(0, k_g + 1)), len(cands))
            sel[0, h, j, :n] = np.sort(rng.choice(cands, n, replace=False))
    return sel


@pytest.mark.parametrize("q_begin", [0, 1024, 4096])
def test_segment_pairs_counts_the_oracle_key_sets(q_begin):
    bench = load_bench()
    rng = np.random.default_rng(q_begin + 7)
    n_kv, n_qb, k_g = 2, 4, 12
    sel = random_selection(rng, n_kv, n_qb, k_g, q_begin)
    all_pairs, act_pairs = bench.segment_pairs(W, sel, q_begin)
    want_all = want_act = 0
    for h in range(n_kv):
        for j in range(n_qb):
            for r in range(64):
                keys = orc.keyset(q_begin, j, r, sel[0, h, j])
                want_all += len(keys) * W.group_heads
                want_act += int((keys >= q_begin).sum()) * W.group_heads
    assert all_pairs == want_all
    assert act_pairs == want_act


def test_measured_traffic_only_for_the_current_sources(tmp_path, monkeypatch):
    bench = load_bench()
    prof = tmp_path / "profiles"
    prof.mkdir()
    entry = {"bytes_per_launch": 1234, "source_hash": bench.source_hash("k")}
    (prof / "dram_traffic.json").write_text(json.dumps({"wl": {"k": entry}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_hash", lambda kernel=None: entry["source_hash"])
    assert bench.measured_traffic("k", "wl") == 1234
    assert bench.measured_traffic("other", "wl") is None
    monkeypatch.setattr(bench, "source_hash", lambda kernel=None: "changed")
    assert bench.measured_traffic("k", "wl") is None


def test_source_hash_follows_each_kernels_own_files(tmp_path, monkeypatch):
    # a kernel's stored figures go stale when its own file, a shared device
    # header or the C header changes, and not when another kernel's does
    bench = load_bench()
    csrc = tmp_path / "hierarchical_routed_sparse_hga_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "include").mkdir()
    names = set(bench.SHARED_SOURCES) | {f for fs in bench.KERNEL_SOURCE.values() for f in fs}
    for f in names:
        (csrc / f).write_text(f)
    (tmp_path / "include" / "hga.h").write_text("h")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    before = {k: bench.source_hash(k) for k in ("attn_bwd_dq_tc", "route_fused", "decode")}
    (csrc / "route.cuh").write_text("route changed")
    after = {k: bench.source_hash(k) for k in before}
    assert after["attn_bwd_dq_tc"] == before["attn_bwd_dq_tc"]
    assert after["route_fused"] != before["route_fused"]
    assert after["decode"] != before["decode"]          # decode includes the routing code
    (csrc / "hga_common.cuh").write_text("common changed")
    assert bench.source_hash("attn_bwd_dq_tc") != before["attn_bwd_dq_tc"]


def test_both_arms_describe_the_same_workload():
    bench = load_bench()
    from hierarchical_routed_sparse_hga_b200 import synth
    w = synth.workloads()["qwen3_fwdbwd_16k"]
    cfg = bench.workload_config("qwen3_fwdbwd_16k", w, 1)
    assert cfg["workload"] == "qwen3_fwdbwd_16k"
    assert (cfg["seq_len"], cfg["seg_len"], cfg["n_q_heads"], cfg["n_kv_heads"],
            cfg["head_dim"]) == (16384, 2048, 32, 8, 128)
    assert cfg["backward"] is True and cfg["parallelism"] == "replicas1"


def test_routing_work_goes_to_the_kernels_that_run():
    # one launch of the fused routing kernel up to 512 candidate blocks, the
    # three long-context kernels beyond; each is credited only with the
    # segments whose path it runs, under the library's own kernel names
    bench = load_bench()
    from hierarchical_routed_sparse_hga_b200 import HGA_K_COUNT, hga_kernel_name
    from hierarchical_routed_sparse_hga_b200 import synth
    names = {hga_kernel_name(k) for k in range(HGA_K_COUNT)}
    three = ("route_qbar", "route_block_topk", "route_select")
    assert set(three) | {"route_fused"} <= names
    w = synth.custom(n_q_heads=32, n_kv_heads=8, head_dim=128, ctx_len=65536, seg_len=2048,
                     topk_blocks=16, topk_groups=64, dtype="bf16", backward=False)
    sel = np.zeros((1, 8, 32, 64), np.int32)
    short = [(14336, sel)]                    # last candidate block 255
    long = [(63488, sel)]                     # last candidate block 1023
    for k in three:
        assert bench.kernel_work(k, w, short)[0] == 0
        assert bench.kernel_work(k, w, long)[0] > 0
    assert bench.kernel_work("route_fused", w, short)[0] > 0
    assert bench.kernel_work("route_fused", w, long)[0] == 0
    # q-bar reads every query row once: Hq x S x d bf16 plus the means written
    assert bench.kernel_work("route_qbar", w, long)[0] == 32 * 2048 * 128 * 2 + 8 * 32 * 128 * 4


def test_profile_cases_reject_an_unknown_case():
    # the profiling driver lists its cases and refuses any other name before
    # touching a GPU
    from hierarchical_routed_sparse_hga_b200 import profile_cases
    assert set(profile_cases.CASES) == {"bench16k", "long128k", "decode", "prepare", "tier",
                                        "simt"}
    with pytest.raises(SystemExit):
        profile_cases.run("no_such_case", None)
    with pytest.raises(SystemExit):
        profile_cases.main([])
