"""Host-side bookkeeping of bench.py: the algorithmic bytes a step must move
(the roofline's numerator) for the router widths and cache element types."""
import bench
from sparse_decode_attention_basiskv_b200 import synth


def test_algorithmic_bytes_full_router_bf16():
    wl = synth.LLAMA8B_T32K_B16
    T = 32769
    b = bench.algorithmic_bytes(wl, T)
    P = -(-T // 16)
    assert b["route"] == 16 * 8 * T * (64 + 32) * 2
    assert b["attend"] == 16 * 8 * min(128, P) * 16 * (128 + 64) * 2
    assert b["outproj"] == 32 * 64 * 4096 * 2
    assert b["total"] == b["route"] + b["attend"] + b["outproj"] + b["small"]


def test_algorithmic_bytes_narrow_router_and_e4m3():
    T = 32769
    nar = bench.algorithmic_bytes(synth.LLAMA8B_T32K_B16_B16R16, T)
    assert nar["route"] == 16 * 8 * T * (16 + 16) * 2  # the router reads 16 + 16 columns
    f8 = bench.algorithmic_bytes(synth.LLAMA8B_T32K_B16_FP8, T)
    bf = bench.algorithmic_bytes(synth.LLAMA8B_T32K_B16, T)
    assert f8["route"] * 2 == bf["route"] and f8["attend"] * 2 == bf["attend"]
    assert f8["outproj"] == bf["outproj"]  # W' stays bf16
    # the appended token: k, v in as bf16; K, z, e out at one byte each
    no_app = bench.algorithmic_bytes(synth.LLAMA8B_T32K_B16_FP8, T, append=False)
    wl = synth.LLAMA8B_T32K_B16_FP8
    assert f8["small"] - no_app["small"] == (wl.B * wl.Hkv * (2 * wl.d * 2 + wl.d + wl.r_v + wl.r_k)
                                             + wl.Hkv * wl.d * wl.r_v * 2)


def test_sweep_capacity_rule():
    """32 distinct caches while they fit under 150 GB, else as many as fit
    (cycled by layer); the per-layer cache counts every physical page."""
    pts = {(w.B, w.T, w.r_v): w for w in synth.SWEEP}
    assert len(pts) == 24
    small = synth.with_sizes(pts[(8, 32768, 96)], steps=131)
    per = bench.cache_bytes_per_layer(small)
    assert per == 8 * small.pages_capacity() * 8 * 16 * (128 + 96 + 32) * 2
    assert bench.sweep_physical_layers(small) == 32  # 32 x 1.1 GB
    big = synth.with_sizes(pts[(64, 131072, 96)], steps=131)
    assert 34e9 < bench.cache_bytes_per_layer(big) < 35e9
    assert bench.sweep_physical_layers(big) == 4  # floor(150 / 34.4)
    mid = synth.with_sizes(pts[(32, 131072, 64)], steps=131)
    assert bench.sweep_physical_layers(mid) == int(150e9 // bench.cache_bytes_per_layer(mid))
    assert [w.top_k for w in synth.SWEEP if w.T == 131072][0] == 2048
    assert bench.sweep_points("b8_t32k_v64")[0] is pts[(8, 32768, 64)]


def test_both_arms_share_the_config_and_flush_rule():
    """The reference arm and the GPU arm describe the same workload, and
    only steps smaller than twice the L2 are timed with a flush."""
    wl = synth.LLAMA8B_T32K_B16
    gpu_side = bench.bench_config(synth.with_sizes(wl, steps=25), 1, 20, 5)
    ref_side = bench.bench_config(wl, 1, 20, 5)
    assert gpu_side == ref_side
    assert not bench.needs_flush(wl)
    assert bench.needs_flush(synth.LLAMA8B_T4K)  # 37.8 MB a step


def test_step_stats_quantiles():
    st = bench.step_stats([0.001 * i for i in range(1, 101)])  # 1 .. 100 us
    assert st["reps"] == 100
    assert abs(st["median_us"] - 50.5) < 1e-9
    assert abs(st["p10_us"] - 10.9) < 1e-9 and abs(st["p90_us"] - 90.1) < 1e-9
