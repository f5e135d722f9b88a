"""bench.py's workload table, on the CPU: the default is the workload the
metric is quoted on, and every --workload choice is a problem the library
accepts (its image tiles into sqrt(B)^L squares)."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_workloads", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_default_workload_is_the_metric_one():
    b = _bench()
    w = b.WORKLOAD
    assert (w["name"], w["H"], w["W"], w["batch"], w["heads"], w["B"], w["L"], w["K"]) == \
        ("px256", 256, 256, 2, 6, 16, 4, 8)
    assert b.METRIC == b.METRIC_PX256


@pytest.mark.parametrize("name", ["px128", "px256", "px256_B64", "px256_K16", "px512"])
def test_every_workload_is_a_valid_problem(name):
    from hierarchical_top_sparse_b200 import llsa
    b = _bench()
    b.select_workload(name)
    w = b.WORKLOAD
    p = llsa.Problem(batch=w["batch"], heads=w["heads"], height=w["H"], width=w["W"], d=w["d"], B=w["B"],
                     L=w["L"], K=w["K"], dtype=llsa.BF16)
    assert llsa.validate(p) == 0
    assert (b.METRIC == b.METRIC_PX256) == (name == "px256")
    assert (b.traffic_record("attn_bwd") is None) or name == "px256"


def test_sweep_points_are_valid_problems_of_equal_size():
    """--sweep: every (N, mode) point is a problem the library accepts, all
    points carry the same number of tokens, LLSA runs the pages' level count
    for the image, the single-level baseline L = 1, and the dense mode keeps
    every block with no enrichment."""
    from hierarchical_top_sparse_b200 import llsa
    b = _bench()
    for side in b.SWEEP_SIDES:
        for mode in ("llsa", "topk_single_level", "dense"):
            p = b.sweep_problem(llsa, side, mode)
            assert llsa.validate(p) == 0, (side, mode)
            assert p.batch * p.heads * p.N == b.SWEEP_TOKENS
            n, kl = llsa.level_sizes(p)
            if mode == "llsa":
                assert p.L == (4 if side >= 256 else 3) and kl[1] == 8 and p.enrich_mask == (1 << p.L) - 1
            elif mode == "topk_single_level":
                assert p.L == 1 and kl[1] == 8 and p.enrich_mask == 1
            else:
                assert p.L == 1 and kl[1] == n[1] and p.enrich_mask == 0
