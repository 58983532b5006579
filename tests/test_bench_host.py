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
