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
