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
