"""bench.py's chunked-chain point (CPU: the timing call is replaced by a
stand-in).  The issued tensor flops per (CTA, 64-token chunk) equal the
kernel's tcgen05.mma issue counts, each product M = 128 rows by N by K = 16:
X^T | Y^T 16 products of N = 128 (2 state parts x 8 k-steps), [K; Q] K^T 8
of N = 64, U^T 24 of N = 64 (6 part products x 4 k-steps), the update 12 of
N = 128 (3 parts x 4 k-steps), U^T M^T 12 of N = 64 (3 part products x 4)."""
import contextlib

import pytest

import bench
import gated_deltanet_tree_verify_b200 as gdn


def _mma_flops(n_products, N):
    return n_products * 2 * 128 * N * 16


def test_issued_flops_match_the_mma_issue_counts():
    issued = (_mma_flops(16, 128) + _mma_flops(8, 64) + _mma_flops(24, 64) + _mma_flops(12, 128)
              + _mma_flops(12, 64))
    assert bench.CHUNK_FLOPS_ISSUED == issued == 26_214_400
    # one part each: X^T | Y^T (N = 128, K = 128), [K; Q] K^T (N = 64, K = 128),
    # U^T (N = 64, K = 64), the update (N = 128, K = 64), U^T M^T (N = 64, K = 64)
    algo = 2 * 128 * (128 * 128 + 64 * 128 + 64 * 64 + 128 * 64 + 64 * 64)
    assert bench.CHUNK_FLOPS_ALGO == algo


def test_roofline_of_a_launch():
    t = 1.25e-3
    r = bench.chunked_tensor_roofline(t, 8, 4096)
    ctas, chunks = 8 * 48, 64
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["issued_gflop"] == pytest.approx(ctas * chunks * bench.CHUNK_FLOPS_ISSUED / 1e9)
    assert r["achieved"] == pytest.approx(ctas * chunks * bench.CHUNK_FLOPS_ISSUED / t / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    assert r["algorithmic"] == pytest.approx(ctas * chunks * bench.CHUNK_FLOPS_ALGO / t / 1e12)
    # a ragged last chunk counts as a whole chunk
    assert bench.chunked_tensor_roofline(t, 8, 4097)["issued_gflop"] == pytest.approx(
        ctas * 65 * bench.CHUNK_FLOPS_ISSUED / 1e9)


def test_point_runs_the_chunked_long_chain(monkeypatch):
    seen = {}

    def fake_verify_point(**kw):
        seen.update(kw)
        with (kw["sampler"] or contextlib.nullcontext()):
            pass
        return 1.27e-3, 2

    monkeypatch.setattr(bench, "_verify_point", fake_verify_point)
    d = bench.run_chunked_point(0)
    assert seen["batch"] == 8 and seen["n_nodes"] == 4096 and seen["tree"] == "chain"
    assert seen["state_dtype"] == "f32" and seen["gate"] == "uniform_a" and seen["min_bytes"] == 0
    assert seen["flags"] == gdn.GDN_FLAG_CHAIN | gdn.GDN_FLAG_PERSIST_LAST | gdn.GDN_FLAG_CHUNKED
    assert d["ms_per_launch"] == pytest.approx(1.27) and d["tokens_per_s"] == pytest.approx(8 * 4096 / 1.27e-3)
    assert d["roofline"] == bench.chunked_tensor_roofline(1.27e-3, 8, 4096)
    assert d["buffer_sets"] == 2 and "clocks" in d and d["workload"] == "long_chain4096_b8_persist_last_f32"
