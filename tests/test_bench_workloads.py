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


def test_roofline_arithmetic_at_256():
    """The compulsory bytes and real-pair FLOPs bench.py divides by, at the
    256 x 256 workload, counted here from the workload itself: 12 slices of
    65536 tokens, d = 64, B = 16, K = 8, four levels of 4096, 256, 16 and 1
    tokens, every level enriched."""
    b = _bench()
    BH, N, d, L, B = 12, 65536, 64, 4, 16
    n = [N, 4096, 256, 16, 1]
    kl = [0, 8, 8, 8, 1]                      # K_4 = min(K, n_4)
    tok = BH * N * d * 2                      # one bf16 tensor
    pyr = BH * (4096 + 256 + 16 + 1) * d * 4  # one fp32 pyramid
    idx = BH * (4096 * 8 + 256 * 8 + 16 * 8 + 1 * 1) * 4
    offs = BH * (4097 + 257 + 17 + 2) * 4
    lse = BH * N * 4
    assert b.algorithmic_bytes("pool", n, kl, BH, N, d, L) == tok + pyr
    assert b.algorithmic_bytes("select", n, kl, BH, N, d, L) == 2 * pyr + idx
    assert b.algorithmic_bytes("attn_fwd", n, kl, BH, N, d, L) == 4 * tok + 2 * pyr + idx + lse
    assert b.algorithmic_bytes("index_transpose", n, kl, BH, N, d, L) == 2 * idx + offs
    assert b.algorithmic_bytes("attn_bwd", n, kl, BH, N, d, L) == 8 * tok + lse + 2 * pyr + 2 * idx + offs
    # 128 fine keys and 8 + 8 + 8 + 1 pooled keys per query
    assert b.keys_per_query(kl, B, L, 0b1111) == 153
    assert b.keys_per_query(kl, B, L, 0) == 128
    pairs = BH * N * 153
    assert b.algorithmic_flops("attn_fwd", kl, BH, N, d, B, L, 0b1111) == pairs * d * 4
    assert b.algorithmic_flops("attn_bwd", kl, BH, N, d, B, L, 0b1111) == pairs * d * 10
    # the figures the profiles quote
    assert round(b.algorithmic_bytes("attn_fwd", n, kl, BH, N, d, L) / 1e6, 1) == 434.3
    assert round(b.algorithmic_bytes("attn_bwd", n, kl, BH, N, d, L) / 1e6, 1) == 838.9
    assert round(pairs * d * 4 / 1e9, 1) == 30.8 and round(pairs * d * 10 / 1e9, 1) == 77.0
