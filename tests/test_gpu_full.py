"""Parity at the full workload sizes, in the launch configuration the
benchmark times (one fused basiskv_decode per step), checked on sampled
sequences that the oracle recomputes one by one."""
import numpy as np
import pytest
import torch

from oracle import basiskv_oracle as O
from sparse_decode_attention_basiskv_b200 import synth

from harness import (cache_row, Y_ABS, Y_REL, ZE_REL, assert_within, compare_selection, factors_np,
                     gpu_layer, np64, status_clean)

pytestmark = pytest.mark.gpu


def _check_step(pb, layer, y, sel, samples, T_before, k_new=None, v_new=None):
    wl = pb.wl
    f = factors_np(pb)
    W = O.fold_outproj(f["B_V"], f["W_O"], wl.Hq)
    stats = {}
    for b in samples:
        c = {k: np64(v[b]) for k, v in pb.cache.items()}
        kw = {}
        if k_new is not None:
            kw = dict(k_new=np64(k_new[b]), v_new=np64(v_new[b]), A_V=f["A_V"])
        out = O.decode_sequence(np64(pb.q[b]), c["K"], c["Z"], c["E"], T_before, wl.page_size,
                                wl.top_k, f["P_K"], f["U_K"], W, **kw)
        for g in range(wl.Hkv):
            compare_selection(sel[b, g].cpu().numpy(), out["sel"][g], out["near_tie"][g], stats)
            if k_new is not None:
                slot = (layer.block_table[b, T_before // wl.page_size].item(), g,
                        T_before % wl.page_size)
                assert_within(np64(cache_row(layer.Z, wl, "Z", *slot)), out["z_new"][g], ZE_REL,
                          what="z")
                assert_within(np64(cache_row(layer.E, wl, "E", *slot)), out["e_new"][g], ZE_REL,
                          what="e")
        if not out["near_tie"].any():
            assert_within(np64(y[b]), out["y"], Y_REL, Y_ABS, what=f"y b{b}")
    assert stats.get("clean_mismatch", 0) == 0, stats
    return stats


def test_llama8b_t4k_full():
    wl = synth.LLAMA8B_T4K
    pb, layer = gpu_layer(wl)
    sel = torch.empty(wl.B, wl.Hkv, wl.top_k, dtype=torch.int32, device="cuda")
    y = layer.decode(pb.q, sel=sel, max_seq_len=wl.T).clone()
    status_clean()
    _check_step(pb, layer, y, sel, [0], wl.T)


def test_llama8b_t32k_b16_full_with_append():
    """The headline workload: B 16, 32K context, r_v 64, one token appended
    per sequence inside the step."""
    wl = synth.LLAMA8B_T32K_B16
    pb, layer = gpu_layer(wl)
    k_new, v_new = synth.make_tokens(wl, pb.factors, 1, device="cuda")
    k_new, v_new = k_new[:, 0].contiguous(), v_new[:, 0].contiguous()
    sel = torch.empty(wl.B, wl.Hkv, wl.top_k, dtype=torch.int32, device="cuda")
    y = layer.decode(pb.q, k_new, v_new, sel=sel, max_seq_len=wl.T + 1).clone()
    status_clean()
    assert (layer.seq_lens == wl.T + 1).all()
    _check_step(pb, layer, y, sel, [0, 9, 15], wl.T, k_new, v_new)
    # the newest page (holding the appended token) and the sink are always kept
    assert (sel[:, :, 0] == 0).all() and (sel[:, :, -1] == wl.T // wl.page_size).all()


def test_qwen32b_t64k_b8_full():
    wl = synth.with_sizes(synth.QWEN32B_T64K_B8, prefill_tokens=0)
    pb, layer = gpu_layer(wl)
    sel = torch.empty(wl.B, wl.Hkv, wl.top_k, dtype=torch.int32, device="cuda")
    y = layer.decode(pb.q, sel=sel, max_seq_len=wl.T).clone()
    status_clean()
    _check_step(pb, layer, y, sel, [0, 7], wl.T)


def test_sweep_multistep_first_and_last():
    """32-layer sweep shape, sampled: two layers with independent factors,
    several decode steps appending one token each; the oracle carries its own
    cache and is compared on the first and the last step."""
    base = synth.sweep_point(8, 4096, 96, layers=2, steps=4)
    for layer_id in range(base.layers):
        pb = synth.make_problem(base, device="cuda", layer=layer_id)
        from sparse_decode_attention_basiskv_b200.layer import DecodeLayer
        layer = DecodeLayer.from_problem(pb)
        f = factors_np(pb)
        W = O.fold_outproj(f["B_V"], f["W_O"], base.Hq)
        oc = {k: np64(v) for k, v in pb.cache.items()}  # oracle's own cache
        T = base.T
        for step in range(base.steps):
            k_new, v_new = synth.make_tokens(base, pb.factors, 1, device="cuda",
                                             stream_id=100 * layer_id + step)
            k_new, v_new = k_new[:, 0].contiguous(), v_new[:, 0].contiguous()
            q, _ = synth.make_query(base, pb.cache["K"], T, step=step)
            sel = torch.empty(base.B, base.Hkv, base.top_k, dtype=torch.int32, device="cuda")
            y = layer.decode(q, k_new, v_new, sel=sel, max_seq_len=T + 1).clone()
            status_clean()
            for b in range(base.B):
                out = O.decode_sequence(np64(q[b]), oc["K"][b], oc["Z"][b], oc["E"][b], T,
                                        base.page_size, base.top_k, f["P_K"], f["U_K"], W,
                                        k_new=np64(k_new[b]), v_new=np64(v_new[b]),
                                        A_V=f["A_V"])
                for g in range(base.Hkv):
                    oc["Z"][b, g, T] = O.to_bf16(out["z_new"][g])
                    oc["E"][b, g, T] = O.to_bf16(out["e_new"][g])
                    oc["K"][b, g, T] = np64(k_new[b, g])
                if step in (0, base.steps - 1):
                    if not out["near_tie"].any():
                        assert np.array_equal(sel[b].cpu().numpy(), out["sel"])
                        assert_within(np64(y[b]), out["y"], Y_REL, Y_ABS, what=f"y s{step} b{b}")
            T += 1
