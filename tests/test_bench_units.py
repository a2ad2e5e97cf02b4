"""The benchmark's algorithmic units, counted by hand for the long workload
(PSD feature, d_k = 32, d_v = 64, C = 128, so D = 32 * 33 / 2 = 528), against
the functions bench.py derives its roofline figures from. A change to a count
there moves every reported fraction, so it has to show up here."""

import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_chunked_forward_units():
    """Intra-chunk: the causal half of a 128 x 128 block, 129 / 2 pairs per
    token, each a d_k dot product, a d_v axpy and the weight's square and sum
    (2 * 32 + 2 * 64 + 2 = 194 flop): 12,513. Update: 528 x 64 multiply-adds
    plus 528 adds for z: 68,112. Readout: the same product plus the
    denominator's 528 multiply-adds: 68,640. Bytes: q, k, v in and y out, bf16:
    2 * (32 + 32 + 64 + 64) = 384."""
    flops, nbytes = bench().algorithmic_per_token_head(32, 64, 128, "psd")
    assert flops == 12_513 + 68_112 + 68_640 == 149_265
    assert nbytes == 384


def test_feature_expansion_products():
    """One product per packed feature for phi(k) and one for phi~(q): 2 * 528.
    The first-order feature [1, u] is its input: no products."""
    b = bench()
    assert b.feature_products_per_token_head(32, "psd") == 1_056
    assert b.feature_products_per_token_head(16, "psd") == 2 * 136
    assert b.feature_products_per_token_head(64, "first_order") == 0


def test_floors_order_on_the_long_workload():
    """At the fallback peaks (6.65 TB/s, 1.59 PFLOP/s) and the 1.965 GHz
    clock, one launch of 16 x 131072 token-heads has its tensor floor
    (about 197 us) above its HBM floor (about 121 us), and both above the
    feature expansion's ALU floor (about 59 us)."""
    b = bench()
    th = 16 * 131072
    flops, nbytes = b.algorithmic_per_token_head(32, 64, 128, "psd")
    t_tensor = flops * th / 1.59e15
    t_hbm = nbytes * th / 6.65e12
    t_alu = b.feature_products_per_token_head(32) * th / (148 * 128 * 1.965e9)
    assert 190e-6 < t_tensor < 200e-6
    assert 115e-6 < t_hbm < 125e-6
    assert 55e-6 < t_alu < 65e-6
    assert t_tensor > t_hbm > t_alu


def test_traffic_records_match_the_current_sources():
    """Every DRAM-traffic record in profiles/traffic.json names a kernel the
    bench knows, holds a positive byte count, and is keyed to the hash of
    that kernel's current source files: a kernel edited after its capture
    must be profiled again (the bench would otherwise report its traffic as
    unknown)."""
    import json
    b = bench()
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        records = json.load(f)
    assert records
    for kernel, rec in records.items():
        assert kernel in b.KERNEL_SOURCES, kernel
        assert rec["bytes_per_launch"] > 0, kernel
        assert rec["source_sha"] == b.source_hash(kernel), f"{kernel}: captured on other sources"
