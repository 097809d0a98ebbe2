"""Routing pages of 4 tokens over 16- or 32-token cache pages (Table 10's
adopted Page4; Table 9's budget of routed tokens plus a recent window):
the router scores every 4 tokens, the selection counts 4-token pages, and
the fused step's attention gathers them from the cache pages.  Compared
with the oracle at a page size of 4 (the oracle has no cache pages)."""
import numpy as np
import pytest
import torch

import sparse_decode_attention_basiskv_b200 as bkv
from oracle import basiskv_oracle as O
from sparse_decode_attention_basiskv_b200 import synth

from harness import (S_REL, StepChecker, ZE_REL, assert_e4m3_bracket, assert_within, cache_row,
                     factors_np, gpu_layer, np64, oracle_route, status_clean)

pytestmark = pytest.mark.gpu

P4 = synth.LLAMA8B_T32K_B16_B16R16_PAGE4
CASES = {
    # the pages' B16R16 router at Page4 with a 16-page recent window, ragged tail
    "b16r16_page4": synth.with_sizes(P4, B=4, T=2999, top_k=96),
    # 8-token routing pages
    "b16r16_page8": synth.with_sizes(P4, B=3, T=2001, top_k=64, route_page=8, recent_pages=4),
    # the full-width router (sink + newest routing page) at Page4
    "full_page4": synth.with_sizes(synth.LLAMA8B_T32K_B16, B=2, T=1500, top_k=80, route_page=4),
    # Qwen3-32B shape: 32-token cache pages, 4-token routing pages
    "qwen_b16r16_page4": synth.with_sizes(synth.QWEN32B_T64K_B8, B=2, T=2500, prefill_tokens=0,
                                          top_k=100, route_r_v=16, route_r_k=16, sink_pages=-1,
                                          recent_pages=8, route_page=4),
}


@pytest.fixture(scope="module", params=list(CASES))
def setup(request):
    wl = CASES[request.param]
    pb, layer = gpu_layer(wl)
    return wl, pb, layer


def test_route_scores_and_selection(setup):
    wl, pb, layer = setup
    nr = wl.page_size // wl.sel_page
    scores = torch.full((wl.B, wl.Hkv, layer.dims.max_pages_per_seq * nr), float("nan"),
                        device="cuda")
    sel = torch.empty(wl.B, wl.Hkv, wl.top_k, dtype=torch.int32, device="cuda")
    bkv.basiskv_route(layer.dims, pb.q, layer.seq_lens, wl.T, layer.block_table, layer.P_K,
                      layer.U_K, layer.Z, layer.E, wl.top_k, scores, sel, layer.workspace)
    status_clean()
    chk = StepChecker(wl, None, wl.name + " route")
    P = -(-wl.T // wl.sel_page)
    for b in range(wl.B):
        for g in range(wl.Hkv):
            sc, ref_sel, tie = oracle_route(pb, b, g, wl.T)
            assert len(sc) == P
            assert_within(np64(scores[b, g, :P]), sc, S_REL, what=f"scores b{b} g{g}")
            chk.group(b, g, sel[b, g].cpu().numpy(), sc, ref_sel, tie)
    chk.report()


def test_decode_step_with_append(setup):
    wl, pb, layer = setup
    f = factors_np(pb)
    k_new, v_new = synth.make_tokens(wl, pb.factors, 1, device="cuda")
    k_new, v_new = k_new[:, 0].contiguous(), v_new[:, 0].contiguous()
    sel = torch.empty(wl.B, wl.Hkv, wl.top_k, dtype=torch.int32, device="cuda")
    seq0 = layer.seq_lens.clone()
    y = layer.decode(pb.q, k_new, v_new, sel=sel, max_seq_len=wl.T + 1).clone()
    status_clean()
    assert torch.equal(layer.seq_lens, seq0 + 1)
    W = O.fold_outproj(f["B_V"], f["W_O"], wl.Hq)
    chk = StepChecker(wl, W, wl.name)
    for b in range(wl.B):
        c = {k: np64(v[b]) for k, v in pb.cache.items()}
        out = O.decode_sequence(np64(pb.q[b]), c["K"], c["Z"], c["E"], wl.T, wl.sel_page,
                                wl.top_k, f["P_K"], f["U_K"], W, k_new=np64(k_new[b]),
                                v_new=np64(v_new[b]), A_V=f["A_V"], **wl.router)
        for g in range(wl.Hkv):
            slot = (layer.block_table[b, wl.T // wl.page_size].item(), g, wl.T % wl.page_size)
            assert_within(np64(cache_row(layer.Z, wl, "Z", *slot)), out["z_new"][g], ZE_REL,
                          what="z")
            assert_within(np64(cache_row(layer.E, wl, "E", *slot)), out["e_new"][g], ZE_REL,
                          what="e")
        chk.check(b, out, sel[b].cpu().numpy(), np64(y[b]), np64(pb.q[b]))
    chk.report()
    layer.seq_lens.copy_(seq0)


def test_standalone_attention_refuses_routing_pages(setup):
    wl, pb, layer = setup
    sel = torch.zeros(wl.B, wl.Hkv, wl.top_k, dtype=torch.int32, device="cuda")
    a = torch.empty(wl.B, wl.Hq, wl.r_v, device="cuda")
    with pytest.raises(bkv.BasisKVError) as err:
        bkv.basiskv_attend(layer.dims, pb.q, layer.seq_lens, wl.T, layer.block_table, layer.K,
                           layer.Z, sel, wl.top_k, a, layer.workspace)
    assert err.value.status == bkv.ERR_UNSUPPORTED_SHAPE


def test_page4_full_size():
    """The pages' configuration at the headline size: B 16, 32K context,
    B16R16 router, 512 routed + 16 recent 4-token pages (2048 + 64 tokens),
    one token appended; every sequence checked."""
    wl = P4
    pb, layer = gpu_layer(wl)
    f = factors_np(pb)
    k_new, v_new = synth.make_tokens(wl, pb.factors, 1, device="cuda")
    k_new, v_new = k_new[:, 0].contiguous(), v_new[:, 0].contiguous()
    sel = torch.empty(wl.B, wl.Hkv, wl.top_k, dtype=torch.int32, device="cuda")
    y = layer.decode(pb.q, k_new, v_new, sel=sel, max_seq_len=wl.T + 1).clone()
    status_clean()
    W = O.fold_outproj(f["B_V"], f["W_O"], wl.Hq)
    chk = StepChecker(wl, W, wl.name)
    for b in range(wl.B):
        c = {k: np64(v[b]) for k, v in pb.cache.items()}
        out = O.decode_sequence(np64(pb.q[b]), c["K"], c["Z"], c["E"], wl.T, wl.sel_page,
                                wl.top_k, f["P_K"], f["U_K"], W, k_new=np64(k_new[b]),
                                v_new=np64(v_new[b]), A_V=f["A_V"], **wl.router)
        chk.check(b, out, sel[b].cpu().numpy(), np64(y[b]), np64(pb.q[b]))
    chk.report()
    # the 16 newest routing pages (64 tokens) are the last 16 entries
    P = -(-(wl.T + 1) // wl.sel_page)
    assert (sel[:, :, -16:].cpu() == torch.arange(P - 16, P, dtype=torch.int32)).all()


# Table 13's configuration: B16R16 Page4 over FP8 E4M3 caches
CASES_E4M3 = {
    "b16r16_page4_e4m3": synth.with_sizes(P4, B=4, T=2999, top_k=96, cache_fp8=1),
    "full_page4_e4m3": synth.with_sizes(synth.LLAMA8B_T32K_B16, B=2, T=1500, top_k=80,
                                        route_page=4, cache_fp8=1),
    "qwen_b16r16_page4_e4m3": synth.with_sizes(synth.QWEN32B_T64K_B8, B=2, T=2500,
                                               prefill_tokens=0, top_k=100, route_r_v=16,
                                               route_r_k=16, sink_pages=-1, recent_pages=8,
                                               route_page=4, cache_fp8=1),
}
E4M3_APPEND_TOL = 1e-4  # the decode append: fp32 on the device, fp64 in the oracle


@pytest.mark.parametrize("name", list(CASES_E4M3))
def test_page4_over_e4m3_caches(name):
    """Routing pages over E4M3 caches: the scores of every 4-token routing
    page and the selection, then a fused decode step (its token appended as
    E4M3) against the oracle's own E4M3 step."""
    wl = CASES_E4M3[name]
    pb, layer = gpu_layer(wl)
    assert layer.K.dtype == torch.float8_e4m3fn
    nr = wl.page_size // wl.sel_page
    scores = torch.full((wl.B, wl.Hkv, layer.dims.max_pages_per_seq * nr), float("nan"),
                        device="cuda")
    sel = torch.empty(wl.B, wl.Hkv, wl.top_k, dtype=torch.int32, device="cuda")
    bkv.basiskv_route(layer.dims, pb.q, layer.seq_lens, wl.T, layer.block_table, layer.P_K,
                      layer.U_K, layer.Z, layer.E, wl.top_k, scores, sel, layer.workspace)
    status_clean()
    chk = StepChecker(wl, None, wl.name + " route")
    P = -(-wl.T // wl.sel_page)
    for b in range(wl.B):
        for g in range(wl.Hkv):
            sc, ref_sel, tie = oracle_route(pb, b, g, wl.T)
            assert len(sc) == P
            assert_within(np64(scores[b, g, :P]), sc, S_REL, what=f"scores b{b} g{g}")
            chk.group(b, g, sel[b, g].cpu().numpy(), sc, ref_sel, tie)
    chk.report()

    f = factors_np(pb)
    k_new, v_new = synth.make_tokens(wl, pb.factors, 1, device="cuda")
    k_new, v_new = k_new[:, 0].contiguous(), v_new[:, 0].contiguous()
    y = layer.decode(pb.q, k_new, v_new, sel=sel, max_seq_len=wl.T + 1).clone()
    status_clean()
    W = O.fold_outproj(f["B_V"], f["W_O"], wl.Hq)
    chk = StepChecker(wl, W, wl.name)
    for b in range(wl.B):
        c = {k: np64(v[b]) for k, v in pb.cache.items()}
        out = O.decode_sequence(np64(pb.q[b]), c["K"], c["Z"], c["E"], wl.T, wl.sel_page,
                                wl.top_k, f["P_K"], f["U_K"], W, k_new=np64(k_new[b]),
                                v_new=np64(v_new[b]), A_V=f["A_V"], fp8=True, **wl.router)
        for g in range(wl.Hkv):
            slot = (layer.block_table[b, wl.T // wl.page_size].item(), g, wl.T % wl.page_size)
            z_ref, e_ref = out["z_new"][g], out["e_new"][g]
            assert_e4m3_bracket(np64(cache_row(layer.Z, wl, "Z", *slot)), z_ref,
                                E4M3_APPEND_TOL * np.abs(z_ref).max(), what="z")
            assert_e4m3_bracket(np64(cache_row(layer.E, wl, "E", *slot)), e_ref,
                                E4M3_APPEND_TOL * np.abs(e_ref).max(), what="e")
            np.testing.assert_array_equal(np64(layer.K[slot].float()),
                                          O.to_e4m3(np64(k_new[b, g])))
        chk.check(b, out, sel[b].cpu().numpy(), np64(y[b]), np64(pb.q[b]))
    chk.report()
