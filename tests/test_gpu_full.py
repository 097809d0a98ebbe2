"""Parity at the full workload sizes, in the launch configuration the
benchmark times (one fused basiskv_decode per step), checked on every
sequence, each recomputed by the oracle on its own."""
import numpy as np
import pytest
import torch

from oracle import basiskv_oracle as O
from sparse_decode_attention_basiskv_b200 import synth

from harness import (StepChecker, cache_row, ZE_REL, assert_within, factors_np, gpu_layer, np64,
                     status_clean)

pytestmark = pytest.mark.gpu


def _check_step(pb, layer, y, sel, samples, T_before, k_new=None, v_new=None):
    wl = pb.wl
    f = factors_np(pb)
    W = O.fold_outproj(f["B_V"], f["W_O"], wl.Hq)
    chk = StepChecker(wl, W, wl.name)
    for b in samples:
        c = {k: np64(v[b]) for k, v in pb.cache.items()}
        kw = {}
        if k_new is not None:
            kw = dict(k_new=np64(k_new[b]), v_new=np64(v_new[b]), A_V=f["A_V"])
        out = O.decode_sequence(np64(pb.q[b]), c["K"], c["Z"], c["E"], T_before, wl.page_size,
                                wl.top_k, f["P_K"], f["U_K"], W, **kw)
        if k_new is not None:
            for g in range(wl.Hkv):
                slot = (layer.block_table[b, T_before // wl.page_size].item(), g,
                        T_before % wl.page_size)
                assert_within(np64(cache_row(layer.Z, wl, "Z", *slot)), out["z_new"][g], ZE_REL,
                              what="z")
                assert_within(np64(cache_row(layer.E, wl, "E", *slot)), out["e_new"][g], ZE_REL,
                              what="e")
        chk.check(b, out, sel[b].cpu().numpy(), np64(y[b]), np64(pb.q[b]))
    return chk.report()


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
    _check_step(pb, layer, y, sel, range(wl.B), wl.T, k_new, v_new)
    # the newest page (holding the appended token) and the sink are always kept
    assert (sel[:, :, 0] == 0).all() and (sel[:, :, -1] == wl.T // wl.page_size).all()


def test_qwen32b_t64k_b8_full():
    wl = synth.with_sizes(synth.QWEN32B_T64K_B8, prefill_tokens=0)
    pb, layer = gpu_layer(wl)
    sel = torch.empty(wl.B, wl.Hkv, wl.top_k, dtype=torch.int32, device="cuda")
    y = layer.decode(pb.q, sel=sel, max_seq_len=wl.T).clone()
    status_clean()
    _check_step(pb, layer, y, sel, range(wl.B), wl.T)
