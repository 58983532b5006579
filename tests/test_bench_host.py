"""Host-side accounting of bench.py for the backward workload (no GPU)."""
import json

import pytest

import bench
from gated_delta_rule_68_b200.workloads import WORKLOADS, make_inputs, make_upstream


def test_backward_bytes_and_flops_by_hand():
    w = WORKLOADS["gdn_bwd_bf16"]
    n = 8 * 2048 * 16                      # head-tokens; Hk = Hv = 16, Dk = Dv = 128
    reads = 4 * n * 128 * 2 + 2 * n * 4    # q, k, v, do in bf16; g, beta in fp32
    writes = 3 * n * 128 * 4 + 2 * n * 4   # dq, dk, dv; dg, dbeta
    states = 3 * 8 * 16 * 128 * 128 * 4    # h0, dhT read; dh0 written
    assert bench.bwd_bytes(w) == reads + writes + states
    assert bench.bwd_flops(w) == 20 * n * 128 * 128
    assert bench.alu_peak_tflops(1965) == pytest.approx(74.45, rel=1e-3)


def test_upstream_gradients_are_seeded_and_shaped():
    w = WORKLOADS["gdn_bwd_bf16"].with_(B=2, T=5, Hk=1, Hv=2, Dk=8, Dv=4)
    a, b = make_upstream(w), make_upstream(w)
    assert a["do"].shape == (2, 5, 2, 4) and a["dhT"].shape == (2, 2, 8, 4)
    assert a["do"].dtype == w.torch_dtype
    assert all(bool((a[n] == b[n]).all()) for n in a)
    assert not bool((make_upstream(w.with_(seed=7))["do"] == a["do"]).all())


def test_backward_reference_arm_prints_one_line(capsys):
    w = WORKLOADS["gdn_bwd_bf16"].with_(T=32, Dk=16, Dv=16)

    class Args:
        warmup, steps = 1, 1
    assert bench.run_bwd_reference(Args, w, 1) == 0
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["metric"] == bench.BWD_METRIC and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_decode_reference_arm_prints_one_line(capsys):
    w = WORKLOADS["decode_bf16"].with_(Dk=16, Dv=16)

    class Args:
        warmup, steps = 1, 2
    assert bench.run_decode_reference(Args, w, 1) == 0
    line = json.loads(capsys.readouterr().out.strip())
    assert line["impl"] == "reference" and line["value"] > 0 and "decode" in line["metric"]


def test_decode_oracle_sample_is_bounded():
    w = WORKLOADS["decode_bf16"].with_(Dk=16, Dv=16)
    cpu = bench.decode_oracle_sample(w, target_s=0.5)
    assert cpu["kind"] == "oracle" and cpu["value"] > 0 and cpu["seconds"] < 5.0


def test_forward_roofline_bytes_match_the_hand_derived_table():
    """The roofline denominators: algorithmic bytes per call (per step for decode) against the
    table derived by hand for the five workloads (q and k once per key head, v and o once
    per value head, g, beta, and h0 and hT once; decode: the state read and written once)."""
    expect_mb = {"gdn_bf16": 287.3, "gva_gdn_bf16": 568.3, "kda_bf16": 1623.2, "decode_bf16": 1619.1}
    for name, mb in expect_mb.items():
        assert bench.algorithmic_bytes(WORKLOADS[name]) / 1e6 == pytest.approx(mb, abs=0.05), name
    # nanochat GDN spelled out: 8 x 2048 tokens, 16 heads of 128, bf16 tensors, fp32 g/beta/states
    n = 8 * 2048 * 16
    by_hand = 4 * n * 128 * 2 + 2 * n * 4 + 2 * 8 * 16 * 128 * 128 * 4
    assert bench.algorithmic_bytes(WORKLOADS["gdn_bf16"]) == by_hand


def test_chunked_backward_tensor_flops_by_hand():
    """Per (unit, 64-token chunk): the forward pass's products (Gram 128x64x128, W and U
    128x64x64 each, R 128x128x64, Qh two 128x64x64, Uh 128x64x64, P 128x128x64, the state
    batch 128x128x128 and 128x64x128), the scan's two (128x128x128, 128x128x64) and the chunk
    kernel's 26.2 Mflop; 4096 chunk units on the nanochat shape."""
    fwd = 2 * (128 * 64 * 128 + 2 * 128 * 64 * 64 + 128 * 128 * 64 + 2 * 128 * 64 * 64 + 128 * 64 * 64
               + 128 * 128 * 64 + 128 * 128 * 128 + 128 * 64 * 128)
    scan = 2 * (128 * 128 * 128 + 128 * 128 * 64)
    chunk = 6400 * 2 * 16 * 8 * 16
    assert bench.bwdc_flops(WORKLOADS["gdn_bwd_bf16"]) == 4096 * (fwd + scan + chunk)
