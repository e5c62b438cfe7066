"""CPU checks of bench.py's arithmetic: the algorithmic FLOPs and bytes its
throughput and roofline figures divide by, and the launch count it claims."""

import types

import bench
from mixture_experts_layer_62_b200 import inputs


def test_flops_of_the_prefill_workload():
    # 2 T k 3 d d_ff for the experts + 2 T d E for the router
    cfg = inputs.workload("mixtral_prefill")
    want = 2 * 4096 * 2 * 3 * 4096 * 14336 + 2 * 4096 * 4096 * 8
    assert bench.flops_per_step(cfg) == want
    assert round(want / 1e12, 3) == 2.886
    # GEMM 1/3 and GEMM 2 split the expert FLOPs 2 : 1
    R = 4096 * 2
    assert bench.up_flops(cfg, R) == 2 * R * 4096 * 2 * 14336
    assert bench.down_flops(cfg, R) * 2 == bench.up_flops(cfg, R)
    assert bench.up_flops(cfg, R) + bench.down_flops(cfg, R) + 2 * 4096 * 4096 * 8 == want


def test_flops_with_the_shared_expert():
    cfg = inputs.workload("deepseek_v3")
    T, d, E, k, dff, dfs = 8192, 7168, 256, 8, 2048, 2048
    want = 2 * T * k * 3 * d * dff + 2 * T * d * E + 2 * T * 3 * d * dfs
    assert bench.flops_per_step(cfg) == want
    assert round(want / 1e12, 2) == 6.52


def test_decode_bytes_count_touched_experts_only():
    cfg = inputs.workload("decode_t1")
    st = types.SimpleNamespace(counts=[1, 0, 0, 1, 0, 0, 0, 0])
    b = bench.decode_bytes(cfg, st)
    # two experts' W1, W3, W2 in bf16, the router, one x row and one y row
    assert b == 2 * 3 * 4096 * 14336 * 2 + 4096 * 8 * 2 + 2 * 4096 * 2
    assert round(b / 1e6, 1) == 704.7


def test_stage_bytes_of_the_mixtral_shaped_layer():
    # route: x + W_r + fp32 logits + idx/gate; permute: x + 8192 rows of Xp
    # + pos + row_token; combine: 8192 rows of O + idx/gate + y
    cfg = inputs.workload("mixtral_prefill")
    b = bench.stage_bytes(cfg, 8192)
    assert b["route"] == 4096 * 4096 * 2 + 4096 * 8 * 2 + 4096 * 8 * 4 + 4096 * 2 * 8
    assert b["permute"] == 4096 * 4096 * 2 + 8192 * 4096 * 2 + 4096 * 2 * 4 + 8192 * 4
    assert b["combine"] == 8192 * 4096 * 2 + 4096 * 2 * 8 + 4096 * 4096 * 2
    h = bench.hbm_stages(cfg, 8192, {"route": 0.02, "permute": 0.04, "combine": 0.03}, {"hbm_gbs": 6500.0})
    assert abs(h["combine"]["gbs"] - b["combine"] / 30e-6 / 1e9) < 1e-6
    assert abs(h["combine"]["frac"] - h["combine"]["gbs"] / 6500.0) < 1e-12


def test_launch_counts():
    assert bench.launches_per_forward(inputs.workload("decode_t1")) == 5
    # fused router up to 64 experts: router, scan, gather, GEMM 1/3, GEMM 2, combine
    assert bench.launches_per_forward(inputs.workload("mixtral_prefill")) == 6
    assert bench.launches_per_forward(inputs.workload("mixtral_prefill"), pad_rows=128) == 7
    # wide routers run on the tensor cores: transpose, logits, select
    assert bench.launches_per_forward(inputs.workload("deepseek_v3")) == 8
    # the shared expert rules out the small-batch router
    assert bench.launches_per_forward(dict(inputs.workload("decode_t1"), d_ff_shared=2048)) == 6
    assert bench.launches_per_forward(dict(inputs.workload("decode_t1"), T=0)) == 1
    # fp32 past 64 experts: transpose, CUDA-core logits, select
    assert bench.launches_per_forward(dict(inputs.workload("toy_fp32"), E=72)) == 8


def test_pass_roofline_of_the_deepseek_shaped_layer():
    # 6.52 TFLOP at the bf16 peak against 22.88 GB (all 256 experts touched,
    # the shared expert, the router, x and y) at the HBM peak: compute-bound,
    # 3.91 ms at this machine's measured peaks
    cfg = inputs.workload("deepseek_v3")
    st = types.SimpleNamespace(rows=8192 * 8, counts=[1] * 256)
    peaks = {"bf16_tflops": 1667.2, "hbm_gbs": 6545.3}
    r = bench.pass_roofline(cfg, st, 7.82, peaks)
    assert round(r["flops"] / 1e12, 2) == 6.52
    assert round(r["bytes"] / 1e9, 2) == 22.88
    assert r["bound"] == "tensor" and round(r["roofline_ms"], 2) == 3.91
    assert abs(r["frac"] - 3.91 / 7.82) < 1e-3


def test_every_other_config_is_measured_by_default():
    names = set(bench.EXTRA_WORKLOADS)
    assert {"decode_t1", "decode_t2", "decode_t4", "decode_t8", "deepseek_v3", "skewed_capacity"} <= names


def test_every_gemm_variant_has_a_kernel_name():
    from mixture_experts_layer_62_b200 import GEMM_VARIANTS
    assert set(GEMM_VARIANTS.values()) <= set(bench.KERNEL_NAMES)


def test_clock_samples_are_taken_inside_the_timed_region_only():
    # nvidia-smi lines (timestamp first) before, inside and after the timed
    # region: only the ones inside count, so idle samples around the region
    # cannot hide a power-capped clock under load
    import datetime
    t = datetime.datetime(2026, 1, 2, 3, 4, 5)
    rows = [(1965, "Not Active"), (1965, "Not Active"), (1500, "Active"), (1440, "Active"), (1965, "Not Active")]
    lines = []
    for i, (clk, cap) in enumerate(rows):
        ts = (t + datetime.timedelta(milliseconds=20 * i)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        lines.append(f"{ts}, {clk}, 1965, 900.0, Not Active, Not Active, Not Active, {cap}")
    at = lambda ms: (t + datetime.timedelta(milliseconds=ms)).timestamp()
    inside = bench.ClockSampler.summarise(lines, at(30), at(70))
    assert inside["samples"] == 2 and inside["sm_mhz"] == 1470.0 and inside["reasons"] == ["sw_power_cap"]
    assert bench.ClockSampler.summarise(lines)["samples"] == 5
    none = bench.ClockSampler.summarise(lines, at(200), at(300))
    assert none["samples"] == 0 and none["sm_mhz"] is None
