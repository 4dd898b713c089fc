"""The benchmark's roofline arithmetic on the CPU: the algorithmic bytes and FLOPs
of the headline workloads as stated in the documentation, the choice of bound,
and the ncu traffic lookup that goes stale when a kernel's source changes."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_prefill_bytes_of_the_headline_workloads():
    # GDN bf16: q, k, v, o at 2 B x 128, log alpha and beta fp32 scalars: 1032 B per token-head
    gdn = 4 * 4096 * 16
    assert bench.prefill_bytes(2, False, gdn, 128, 128, 64) == gdn * 1032 + 64 * 65536
    assert bench.prefill_bytes(2, False, gdn, 128, 128, 64) == 274726912
    # KDA adds 508 B of per-channel log alpha: 1540 B
    kda = 2 * 8192 * 32
    assert bench.prefill_bytes(2, True, kda, 128, 128, 64) == kda * 1540 + 64 * 65536
    # FG2-GDN adds the per-channel rate: 2048 B
    assert bench.prefill_bytes(2, True, kda, 128, 128, 64, beta_channel=True) == \
        kda * 2048 + 64 * 65536


def test_decode_bytes_and_flops():
    # 2 x 64 KiB of fp32 state per head-step, plus 1032 B of tokens and gates
    assert bench.decode_bytes(256, 32, 128, 128) == 256 * 32 * (2 * 65536 + 1032)
    assert bench.decode_bytes(256, 32, 128, 128) == 1082195968
    assert bench.decode_flops(256, 32, 128, 128) == 256 * 32 * 8 * 128 * 128


def test_prefill_flops_per_token_head():
    # 6 d^2 + 2C(3d + 2d) + C^2 / 3 at d = 128, C = 64: 181.6 kFLOP
    assert bench.prefill_flops(1, 128, 128) == pytest.approx(98304 + 81920 + 4096 / 3)


def test_roofline_takes_the_larger_bound():
    pk = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0}
    # byte-heavy: 6 GB at 6000 GB/s = 1 ms against 1 TFLOP at 1500 TFLOP/s = 0.67 ms
    r = bench.roofline(1.0e12, 6.0e9, 2e-3, pk, "measured")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(3000.0) and r["frac"] == pytest.approx(0.5)
    # flop-heavy
    r = bench.roofline(3.0e12, 6.0e9, 4e-3, pk, "measured")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(750.0) and r["frac"] == pytest.approx(0.5)
    assert r["t_hbm_us"] == pytest.approx(1000.0) and r["t_flop_us"] == pytest.approx(2000.0)


def test_traffic_lookup_goes_stale_with_the_source():
    recs = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))
    key = "chunk_pair_kernel:gdn_prefill_bf16"
    src = "gated_delta_rule_140_b200/csrc/gdn_chunk_pair.cu"
    # the committed capture matches the committed source
    assert bench.traffic_for("chunk_pair_kernel", src, "gdn_prefill_bf16") == \
        recs[key]["bytes_per_launch"]
    # another file in its place (a changed kernel) gives no traffic
    assert bench.traffic_for("chunk_pair_kernel", "gated_delta_rule_140_b200/csrc/gdn_decode.cu",
                             "gdn_prefill_bf16") is None
    # a workload without a capture gives none either
    assert bench.traffic_for("chunk_pair_kernel", src, "no_such_workload") is None
