"""Parity of the E4M3-cache path (Table 13's FP8 KV format) with the CPU
oracle: the caches hold FP8 E4M3 values, which the oracle reads as exact
numbers, and every append rounds to E4M3 on both sides."""
import numpy as np
import pytest
import torch

import sparse_decode_attention_basiskv_b200 as bkv
from oracle import basiskv_oracle as O
from sparse_decode_attention_basiskv_b200 import synth

from harness import (A_REL, S_REL, Y_ABS, Y_REL, ZE_REL, assert_e4m3_bracket, assert_within,
                     cache_row, StepChecker, factors_np, gpu_layer, np64, oracle_route,
                     status_clean)

pytestmark = pytest.mark.gpu

# decode-time append: fp32 on the device against fp64 in the oracle
Z_APPEND_TOL = 1e-4

SMALL = {
    # the headline layer shape (G 4, r_v 64, page 16)
    "llama_b16_t2k_e4m3": synth.with_sizes(synth.LLAMA8B_T32K_B16_FP8, T=2000, top_k=32),
    # Table 13's Value width (V96), one sequence, ragged tail
    "llama4k_v96_e4m3": synth.with_sizes(synth.LLAMA8B_T4K, T=4000, cache_fp8=1),
    # Qwen3-32B layer shape (G 8, page 32)
    "qwen_b2_t3k_e4m3": synth.with_sizes(synth.QWEN32B_T64K_B8, B=2, T=3000, prefill_tokens=0,
                                         cache_fp8=1),
    # Table 13's router (B16R16) with a recent window of 4 pages, no sink
    "llama_b16r16_b4_t2k_e4m3": synth.with_sizes(synth.LLAMA8B_T32K_B16_B16R16, B=4, T=2000,
                                                 top_k=24, cache_fp8=1),
}


@pytest.fixture(scope="module", params=list(SMALL))
def setup(request):
    wl = SMALL[request.param]
    pb, layer = gpu_layer(wl)
    assert layer.K.dtype == torch.float8_e4m3fn and layer.K.element_size() == 1
    return wl, pb, layer


def test_route_and_select(setup):
    wl, pb, layer = setup
    B, Hkv = wl.B, wl.Hkv
    scores = torch.full((B, Hkv, layer.dims.max_pages_per_seq), float("nan"), device="cuda")
    sel = torch.empty(B, Hkv, wl.top_k, dtype=torch.int32, device="cuda")
    bkv.basiskv_route(layer.dims, pb.q, layer.seq_lens, wl.T, layer.block_table, layer.P_K,
                      layer.U_K, layer.Z, layer.E, wl.top_k, scores, sel, layer.workspace)
    status_clean()
    chk = StepChecker(wl, None, wl.name + " route")
    for b in range(B):
        for g in range(Hkv):
            sc, ref_sel, tie = oracle_route(pb, b, g, wl.T)
            assert_within(np64(scores[b, g, :wl.pages]), sc, S_REL, what=f"scores b{b} g{g}")
            chk.group(b, g, sel[b, g].cpu().numpy(), sc, ref_sel, tie)
    chk.report()


def test_attend_on_oracle_selection(setup):
    wl, pb, layer = setup
    B, Hkv, G = wl.B, wl.Hkv, wl.G
    ref_sel = np.zeros((B, Hkv, wl.top_k), dtype=np.int32)
    for b in range(B):
        for g in range(Hkv):
            ref_sel[b, g] = oracle_route(pb, b, g, wl.T)[1]
    sel = torch.from_numpy(ref_sel).cuda()
    a = torch.empty(B, wl.Hq, wl.r_v, device="cuda")
    bkv.basiskv_attend(layer.dims, pb.q, layer.seq_lens, wl.T, layer.block_table, layer.K,
                       layer.Z, sel, wl.top_k, a, layer.workspace)
    status_clean()
    for b in range(B):
        for g in range(Hkv):
            qg = np64(pb.q[b, g * G:(g + 1) * G])
            ref, _ = O.attend(qg, np64(pb.cache["K"][b, g]), np64(pb.cache["Z"][b, g]),
                              ref_sel[b, g], wl.T, wl.page_size)
            assert_within(np64(a[b, g * G:(g + 1) * G]), ref, A_REL, what=f"a b{b} g{g}")


def test_decode_step_with_append(setup):
    """Fused step over E4M3 caches: the appended K, z and e are stored as
    E4M3, then routing, attention and the out-projection run over T + 1
    tokens; compared with the oracle's own E4M3 append."""
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
        out = O.decode_sequence(np64(pb.q[b]), c["K"], c["Z"], c["E"], wl.T, wl.page_size,
                                wl.top_k, f["P_K"], f["U_K"], W, k_new=np64(k_new[b]),
                                v_new=np64(v_new[b]), A_V=f["A_V"], fp8=True, **wl.router)
        for g in range(wl.Hkv):
            slot = (layer.block_table[b, wl.T // wl.page_size].item(), g, wl.T % wl.page_size)
            z_ref, e_ref = out["z_new"][g], out["e_new"][g]  # unrounded
            assert_e4m3_bracket(np64(cache_row(layer.Z, wl, "Z", *slot)), z_ref,
                                Z_APPEND_TOL * np.abs(z_ref).max(), what="z")
            assert_e4m3_bracket(np64(cache_row(layer.E, wl, "E", *slot)), e_ref,
                                Z_APPEND_TOL * np.abs(e_ref).max(), what="e")
            np.testing.assert_array_equal(np64(layer.K[slot].float()),
                                          O.to_e4m3(np64(k_new[b, g])))
        chk.check(b, out, sel[b].cpu().numpy(), np64(y[b]), np64(pb.q[b]))
    chk.report()
    layer.seq_lens.copy_(seq0)


def test_prefill_chunk_append():
    """A 4096-token prefill chunk (tensor-core path) into E4M3 caches: each
    stored value is the E4M3 rounding of a value within the bf16 path's
    tolerance of the oracle's."""
    wl = synth.with_sizes(synth.QWEN32B_T64K_B8, B=2, T=96, prefill_tokens=4096, cache_fp8=1)
    pb, layer = gpu_layer(wl)
    f = factors_np(pb)
    k, v = synth.make_tokens(wl, pb.factors, 4096, device="cuda", stream_id=99)
    b = 1
    dims1 = bkv.Dims(B=1, Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, hidden=wl.hidden, r_v=wl.r_v,
                     r_k=wl.r_k, page_size=wl.page_size,
                     max_pages_per_seq=layer.dims.max_pages_per_seq,
                     num_phys_pages=layer.dims.num_phys_pages, cache_fp8=1)
    bkv.basiskv_append(dims1, k[b].contiguous(), v[b].contiguous(), 4096, layer.seq_lens[b:],
                       layer.block_table[b], layer.A_V, layer.P_K, layer.U_K, layer.K, layer.Z,
                       layer.E, layer.workspace, W_app=layer.W_app)
    status_clean()
    assert layer.seq_lens.tolist() == [wl.T, wl.T + 4096]
    toks = np.arange(wl.T, wl.T + 4096)
    phys = layer.block_table[b, toks // wl.page_size].long().cpu()
    rows = torch.as_tensor(toks % wl.page_size)
    for g in range(wl.Hkv):
        z_ref, e_ref = O.append_latents(np64(k[b, :, g]), np64(v[b, :, g]), f["A_V"][g],
                                        f["P_K"][g], f["U_K"][g])
        assert_e4m3_bracket(np64(cache_row(layer.Z, wl, "Z", phys, g, rows)), z_ref,
                            ZE_REL * np.abs(z_ref).max(), what="prefill z")
        assert_e4m3_bracket(np64(cache_row(layer.E, wl, "E", phys, g, rows)), e_ref,
                            ZE_REL * np.abs(e_ref).max(), what="prefill e")
        kb = layer.K.view(torch.uint8)[phys, g, rows].view(torch.float8_e4m3fn).float()
        np.testing.assert_array_equal(np64(kb), O.to_e4m3(np64(k[b, :, g])))
