"""The benchmark's roofline arithmetic against the staged byte and FLOP
formulas, evaluated by hand for the 64K-token workload (B=1, H=8, L=65536,
d=64, bf16 e=2, R=4, m=64):
  forward  per (b, h): L [d e (2 + 4R) + 24 R]            = 65536 * 2400
  backward per (b, h): L [4 d e + 8 + R (4 d e + 16 + 4 d 4)] = 65536 * 6728
  attention FLOPs per token, head, round: 4 (2m) d = 32768 forward,
  5 * 2 (2m) d = 81920 backward; hash: d * n_buckets = 65536."""
import pytest

import bench
from lsh_attention_02_b200 import synth


def test_staged_bytes_and_flops_64k():
    a = bench.algorithmic(synth.WORKLOADS["long_64k"])
    assert 64 * 2 * (2 + 16) + 24 * 4 == 2400
    assert 4 * 64 * 2 + 8 + 4 * (4 * 64 * 2 + 16 + 4 * 64 * 4) == 6728
    assert a["bytes"] == 8 * 65536 * (2400 + 6728) == 4_785_700_864     # 4.79 GB
    assert a["attn_flops"] == 8 * 65536 * 4 * (32768 + 81920)
    assert a["hash_flops"] == 8 * 65536 * 4 * 64 * 1024


def test_forward_only_workload_has_no_backward_bytes():
    w = synth.WORKLOADS["bf16_causal_4k"]                 # B8 H8 L4096 R2, forward only
    a = bench.algorithmic(w)
    assert a["bytes"] == 64 * 4096 * (64 * 2 * (2 + 8) + 24 * 2)
    assert a["attn_flops"] == 64 * 4096 * 2 * 32768


def test_whole_job_rate_counts_every_rank():
    w = synth.WORKLOADS["long_64k"]
    assert bench.whole_job_tokens_per_s(w, 1, 1.0) == 65536 * 1000.0
    assert bench.whole_job_tokens_per_s(w, 4, 2.0) == 4 * 65536 * 500.0


def test_step_roofline_bytes_bound_and_hash_inclusive():
    a = bench.algorithmic(synth.WORKLOADS["long_64k"])
    r = bench.step_roofline(a, 6443.2, 1410.0, 1.65)
    assert r["roofline_ms"] == pytest.approx(4_785_700_864 / 6443.2e9 * 1e3)      # bytes bound: 0.743 ms
    assert r["roofline_ms_with_hash"] == r["roofline_ms"]                        # 377 GFLOP take 0.27 ms
    assert r["frac"] == pytest.approx(r["roofline_ms"] / 1.65)
    h = bench.algorithmic(synth.WORKLOADS["half_million"])                      # nb = 8192: the hash GEMM decides
    rh = bench.step_roofline(h, 6443.2, 1410.0, 2.68)
    assert rh["roofline_ms_with_hash"] == pytest.approx((h["attn_flops"] + h["hash_flops"]) / 1410e12 * 1e3)
    assert rh["roofline_ms_with_hash"] > 3 * rh["roofline_ms"]
