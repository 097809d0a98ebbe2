"""Stage-by-stage parity of the CUDA path (through the C-ABI) with the CPU
oracle, at sizes the oracle finishes in seconds that still span several
tiles and a ragged tail, plus the edge cases of the method."""
import numpy as np
import pytest
import torch

import sparse_decode_attention_basiskv_b200 as bkv
from oracle import basiskv_oracle as O
from sparse_decode_attention_basiskv_b200 import synth
from sparse_decode_attention_basiskv_b200.layer import DecodeLayer

from harness import (A_REL, S_REL, Y_ABS, Y_REL, ZE_REL, assert_e4m3_bracket, assert_within,
                     cache_row,
                     StepChecker,
                     factors_np, gpu_layer, np64, oracle_route, status_clean)

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": synth.TINY,
    "llama4k": synth.LLAMA8B_T4K,
    # the headline layer shape (r_v 64, B 16) at a context the oracle finishes fast
    "llama_b16_t2k": synth.with_sizes(synth.LLAMA8B_T32K_B16, T=2000, top_k=32),
    # the Qwen3-32B layer shape (G 8, page 32) at a short context
    "qwen_b2_t3k": synth.with_sizes(synth.QWEN32B_T64K_B8, B=2, T=3000, prefill_tokens=0),
    # shapes outside the plain-load kernels' lists: page 8 (TMA-ring scoring
    # and attention kernels with their split merge) and r_k 64 (generic scoring)
    "llama_p8_b2_t1500": synth.with_sizes(synth.LLAMA8B_T4K, B=2, T=1500, page_size=8,
                                          top_k=48),
    "llama_rk64_b2_t1500": synth.with_sizes(synth.LLAMA8B_T4K, B=2, T=1500, r_v=64, r_k=64,
                                            top_k=32),
    # the pages' narrow router (16 latent + 16 residual dims) with a recent
    # window of 4 pages and no sink page, at the headline shape
    "llama_b16r16_b4_t2k": synth.with_sizes(synth.LLAMA8B_T32K_B16_B16R16, B=4, T=2000,
                                            top_k=24),
    # a narrow router with the default sink/newest pages, Qwen3-32B shape
    "qwen_b32r16_b2_t3k": synth.with_sizes(synth.QWEN32B_T64K_B8, B=2, T=3000,
                                           prefill_tokens=0, route_r_v=32, route_r_k=16),
}


@pytest.fixture(scope="module", params=list(SMALL))
def setup(request):
    wl = SMALL[request.param]
    pb, layer = gpu_layer(wl)
    return wl, pb, layer


def test_fold_outproj(setup):
    wl, pb, layer = setup
    f = factors_np(pb)
    ref = O.fold_outproj(f["B_V"], f["W_O"], wl.Hq)  # [Hq][r_v][H]
    got = np64(layer.W_fold).reshape(wl.hidden, wl.Hq, wl.r_v).transpose(1, 2, 0)
    tol = 2.0 ** -8 * np.abs(ref) + 1e-5 * np.abs(ref).max()
    assert (np.abs(got - ref) <= tol).all()


def test_route_and_select(setup):
    wl, pb, layer = setup
    B, Hkv = wl.B, wl.Hkv
    scores = torch.full((B, Hkv, layer.dims.max_pages_per_seq), float("nan"), device="cuda")
    sel = torch.empty(B, Hkv, wl.top_k, dtype=torch.int32, device="cuda")
    bkv.basiskv_route(layer.dims, pb.q, layer.seq_lens, wl.T, layer.block_table, layer.P_K,
                      layer.U_K, layer.Z, layer.E, wl.top_k, scores, sel, layer.workspace)
    status_clean()
    P = wl.pages
    chk = StepChecker(wl, None, wl.name + " route")
    for b in range(B):
        for g in range(Hkv):
            sc, ref_sel, tie = oracle_route(pb, b, g, wl.T)
            assert_within(np64(scores[b, g, :P]), sc, S_REL, what=f"scores b{b} g{g}")
            chk.group(b, g, sel[b, g].cpu().numpy(), sc, ref_sel, tie)
    chk.report()


def test_attend_on_oracle_selection(setup):
    wl, pb, layer = setup
    B, Hkv, G = wl.B, wl.Hkv, wl.G
    f = factors_np(pb)
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


def test_outproj(setup):
    wl, pb, layer = setup
    gen = torch.Generator(device="cuda").manual_seed(11)
    a = torch.randn(wl.B, wl.Hq, wl.r_v, generator=gen, device="cuda")
    y = torch.empty(wl.B, wl.hidden, dtype=torch.bfloat16, device="cuda")
    bkv.basiskv_outproj(layer.dims, a, layer.W_fold, y, layer.workspace)
    status_clean()
    f = factors_np(pb)
    W = O.fold_outproj(f["B_V"], f["W_O"], wl.Hq)
    for b in range(wl.B):
        assert_within(np64(y[b]), O.outproj(np64(a[b]), W), Y_REL, Y_ABS, what=f"y b{b}")


def test_decode_step_with_append(setup):
    """Fused step: append one token per sequence, then route, attend and
    out-project over T + 1 tokens; compared with the oracle's own append."""
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
                                v_new=np64(v_new[b]), A_V=f["A_V"], **wl.router)
        # appended state, read back from the paged caches
        for g in range(wl.Hkv):
            slot = (layer.block_table[b, wl.T // wl.page_size].item(), g, wl.T % wl.page_size)
            assert_within(np64(cache_row(layer.Z, wl, "Z", *slot)), out["z_new"][g], ZE_REL,
                          what="z")
            assert_within(np64(cache_row(layer.E, wl, "E", *slot)), out["e_new"][g], ZE_REL,
                          what="e")
            assert torch.equal(layer.K[slot], k_new[b, g])
        chk.check(b, out, sel[b].cpu().numpy(), np64(y[b]), np64(pb.q[b]))
    chk.report()
    # undo the append for the other tests of this module
    layer.seq_lens.copy_(seq0)


def test_ragged_lengths_and_degenerate_pages():
    """Lengths that end mid-page, exactly on a page, inside the first page
    (sink == newest), and contexts with fewer pages than top_k."""
    wl = synth.with_sizes(synth.LLAMA8B_T4K, B=6, T=1200, top_k=16)
    lens = [1, 15, 16, 17, 700, 1200]
    pb, layer = gpu_layer(wl, seq_lens=lens)
    sel = torch.empty(wl.B, wl.Hkv, wl.top_k, dtype=torch.int32, device="cuda")
    y = layer.decode(pb.q, sel=sel, max_seq_len=max(lens)).clone()
    status_clean()
    f = factors_np(pb)
    W = O.fold_outproj(f["B_V"], f["W_O"], wl.Hq)
    chk = StepChecker(wl, W, "ragged")
    for b, T in enumerate(lens):
        c = {k: np64(v[b]) for k, v in pb.cache.items()}
        out = O.decode_sequence(np64(pb.q[b]), c["K"], c["Z"], c["E"], T, wl.page_size,
                                wl.top_k, f["P_K"], f["U_K"], W)
        chk.check(b, out, sel[b].cpu().numpy(), np64(y[b]), np64(pb.q[b]))
    chk.report()
    assert sel[0, 0, 0].item() == 0 and (sel[0, 0, 1:] == -1).all()  # one page


def test_empty_sequence_gives_zero_output():
    """A sequence of length 0 (no append) has no token to attend: its latent
    output, hence its y row, is zero, also after an earlier step left other
    values in the workspace; the other sequence is unaffected."""
    wl = synth.with_sizes(synth.LLAMA8B_T4K, B=2, T=600, top_k=16)
    pb, layer = gpu_layer(wl, seq_lens=[37, 600])
    layer.decode(pb.q, max_seq_len=600)
    layer.seq_lens[0] = 0
    y = torch.full((wl.B, wl.hidden), float("nan"), dtype=torch.bfloat16, device="cuda")
    layer.decode(pb.q, max_seq_len=600, y=y)
    status_clean()
    assert (y[0] == 0).all()
    f = factors_np(pb)
    W = O.fold_outproj(f["B_V"], f["W_O"], wl.Hq)
    c = {k: np64(v[1]) for k, v in pb.cache.items()}
    out = O.decode_sequence(np64(pb.q[1]), c["K"], c["Z"], c["E"], 600, wl.page_size,
                            wl.top_k, f["P_K"], f["U_K"], W)
    sel = torch.empty(wl.B, wl.Hkv, wl.top_k, dtype=torch.int32, device="cuda")
    layer.seq_lens[0] = 0
    y2 = layer.decode(pb.q, sel=sel, max_seq_len=600).clone()
    status_clean()
    assert torch.equal(y2, y)  # the same step again, now with the selection written out
    chk = StepChecker(wl, W, "empty")
    chk.check(1, out, sel[1].cpu().numpy(), np64(y[1]), np64(pb.q[1]))
    chk.report()


def test_dense_when_top_k_covers_context():
    """top_k >= P: every page is attended, so the result is plain attention."""
    wl = synth.with_sizes(synth.TINY, top_k=40)  # 32 pages
    pb, layer = gpu_layer(wl)
    sel = torch.empty(1, 1, 40, dtype=torch.int32, device="cuda")
    y = layer.decode(pb.q, sel=sel, max_seq_len=wl.T).clone()
    status_clean()
    assert sel[0, 0].tolist() == list(range(32)) + [-1] * 8
    f = factors_np(pb)
    W = O.fold_outproj(f["B_V"], f["W_O"], wl.Hq)
    c = {k: np64(v[0]) for k, v in pb.cache.items()}
    out = O.decode_sequence(np64(pb.q[0]), c["K"], c["Z"], c["E"], wl.T, 16, 40, f["P_K"],
                            f["U_K"], W)
    assert_within(np64(y[0]), out["y"], Y_REL, Y_ABS)


def test_route_scores_only_matches_full_call():
    """basiskv_route with sel = NULL computes the same page scores (bit for
    bit) as the full call, and writes no selection."""
    wl = synth.with_sizes(synth.LLAMA8B_T4K, B=2, T=1000, top_k=16)
    pb, layer = gpu_layer(wl)
    d = layer.dims
    sc1 = torch.zeros(2, 8, d.max_pages_per_seq, device="cuda")
    sc2 = torch.zeros_like(sc1)
    sel = torch.empty(2, 8, 16, dtype=torch.int32, device="cuda")
    bkv.basiskv_route(d, pb.q, layer.seq_lens, wl.T, layer.block_table, layer.P_K, layer.U_K,
                      layer.Z, layer.E, 16, sc1, sel, layer.workspace)
    bkv.basiskv_route(d, pb.q, layer.seq_lens, wl.T, layer.block_table, layer.P_K, layer.U_K,
                      layer.Z, layer.E, 16, sc2, None, layer.workspace)
    torch.cuda.synchronize()
    status_clean()
    P = -(-wl.T // wl.page_size)
    assert torch.equal(sc1[:, :, :P], sc2[:, :, :P])


def test_block_table_permutation_invariance():
    """Different physical placements of the same logical pages give
    bit-identical scores, selection and output."""
    wl = synth.with_sizes(synth.LLAMA8B_T4K, B=2, T=1000, top_k=16)
    pb, layer = gpu_layer(wl)
    sc1 = torch.zeros(2, 8, layer.dims.max_pages_per_seq, device="cuda")
    sel1 = torch.empty(2, 8, 16, dtype=torch.int32, device="cuda")
    bkv.basiskv_route(layer.dims, pb.q, layer.seq_lens, wl.T, layer.block_table, layer.P_K,
                      layer.U_K, layer.Z, layer.E, 16, sc1, sel1, layer.workspace)
    y1 = layer.decode(pb.q, max_seq_len=wl.T).clone()
    # a second placement: reverse the physical order
    n = layer.dims.num_phys_pages
    table2 = (n - 1 - layer.block_table).contiguous()
    perm = (n - 1 - torch.arange(n, device="cuda"))
    for name in ("K", "Z", "E"):
        getattr(layer, name).copy_(getattr(layer, name)[perm].clone())
    layer.block_table = table2
    sc2 = torch.zeros_like(sc1)
    sel2 = torch.empty_like(sel1)
    bkv.basiskv_route(layer.dims, pb.q, layer.seq_lens, wl.T, layer.block_table, layer.P_K,
                      layer.U_K, layer.Z, layer.E, 16, sc2, sel2, layer.workspace)
    y2 = layer.decode(pb.q, max_seq_len=wl.T).clone()
    status_clean()
    assert torch.equal(sc1, sc2) and torch.equal(sel1, sel2) and torch.equal(y1, y2)


@pytest.mark.parametrize("prefolded", [True, False], ids=["W_app", "fold_in_call"])
def test_prefill_chunk_append(prefolded):
    """A 4096-token prefill chunk appended to one sequence of the Qwen3-32B
    layer shape (B = 1 view of the batch; the tensor-core path), compared
    token by token; the folded append factor is either built once up front
    or folded inside the call."""
    wl = synth.with_sizes(synth.QWEN32B_T64K_B8, B=2, T=96, prefill_tokens=4096)
    pb, layer = gpu_layer(wl)
    f = factors_np(pb)
    k, v = synth.make_tokens(wl, pb.factors, 4096, device="cuda", stream_id=99)
    b = 1
    dims1 = bkv.Dims(B=1, Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, hidden=wl.hidden, r_v=wl.r_v,
                     r_k=wl.r_k, page_size=wl.page_size,
                     max_pages_per_seq=layer.dims.max_pages_per_seq,
                     num_phys_pages=layer.dims.num_phys_pages)
    bkv.basiskv_append(dims1, k[b].contiguous(), v[b].contiguous(), 4096, layer.seq_lens[b:],
                       layer.block_table[b], layer.A_V, layer.P_K, layer.U_K, layer.K, layer.Z,
                       layer.E, layer.workspace, W_app=layer.W_app if prefolded else None)
    status_clean()
    assert layer.seq_lens.tolist() == [wl.T, wl.T + 4096]
    for g in range(wl.Hkv):
        z_ref, e_ref = O.append_latents(np64(k[b, :, g]), np64(v[b, :, g]), f["A_V"][g],
                                        f["P_K"][g], f["U_K"][g])
        toks = np.arange(wl.T, wl.T + 4096)
        phys = layer.block_table[b, toks // wl.page_size].long().cpu()
        rows = torch.as_tensor(toks % wl.page_size)
        assert_within(np64(cache_row(layer.Z, wl, "Z", phys, g, rows)), z_ref, ZE_REL, what="prefill z")
        assert_within(np64(cache_row(layer.E, wl, "E", phys, g, rows)), e_ref, ZE_REL, what="prefill e")
        assert torch.equal(layer.K[phys, g, rows], k[b, :, g])


# Sequences of different lengths take one chunk each in one call:
# (workload, starting lengths).
RAGGED_PREFILL = {
    "qwen": (synth.with_sizes(synth.QWEN32B_T64K_B8, B=3, T=160, prefill_tokens=200),
             [5, 37, 131]),
    # the narrow router's split tiles (16 latent + 16 residual columns first)
    "llama_b16r16": (synth.with_sizes(synth.LLAMA8B_T32K_B16_B16R16, B=3, T=160, top_k=8,
                                      prefill_tokens=200), [5, 37, 131]),
    "qwen_e4m3": (synth.with_sizes(synth.QWEN32B_T64K_B8, B=3, T=160, prefill_tokens=200,
                                   cache_fp8=1), [5, 37, 131]),
    # the benchmarked launch: eight 4096-token chunks, 2048 (head, M tile)
    # items over the SMs, so every CTA runs many items and reloads W_app
    "qwen_b8_4096": (synth.with_sizes(synth.QWEN32B_T64K_B8, B=8, T=160, prefill_tokens=4096),
                     [96, 101, 3, 64, 77, 32, 0, 159]),
    # other product shapes: d 64 (one k-block per operand, N = 48), r_k 64
    # with N = 160 and 192 (the fewest ring slots), pages of 8 and 32 tokens
    "tiny_d64": (synth.with_sizes(synth.TINY, B=3, T=160, prefill_tokens=200), [5, 37, 131]),
    "llama_v96_k64_p8": (synth.with_sizes(synth.LLAMA8B_T4K, B=2, T=160, r_k=64, page_size=8,
                                          prefill_tokens=700), [13, 150]),
    "llama_v128_k64_p32": (synth.with_sizes(synth.LLAMA8B_T4K, B=2, T=160, r_v=128, r_k=64,
                                            page_size=32, prefill_tokens=700), [0, 77]),
}


@pytest.mark.parametrize("name", list(RAGGED_PREFILL))
def test_prefill_append_ragged_rows(name):
    """Sequences at ragged lengths (5, 37 and 131, say) take a chunk each
    in one tensor-core call (200 tokens: 600 token rows), so M tiles
    straddle sequences and start pages at odd offsets, and the last tile is
    partial.  Every appended row matches the oracle, and no other cache row
    changes."""
    wl, lens0 = RAGGED_PREFILL[name]
    n = wl.prefill_tokens
    pb, layer = gpu_layer(wl, seq_lens=lens0)
    f = factors_np(pb)
    k, v = synth.make_tokens(wl, pb.factors, n, device="cuda", stream_id=7)
    before = {nm: t.clone() for nm, t in (("K", layer.K), ("Z", layer.Z), ("E", layer.E))}
    layer.append(k, v, n)
    status_clean()
    assert layer.seq_lens.tolist() == [x + n for x in lens0]
    fp8 = bool(wl.cache_fp8)
    touched = torch.zeros(layer.K.shape[:3], dtype=torch.bool)  # [phys][Hkv][page row]
    for b, L0 in enumerate(lens0):
        toks = np.arange(L0, L0 + n)
        phys = layer.block_table[b, toks // wl.page_size].long().cpu()
        rows = torch.as_tensor(toks % wl.page_size)
        touched[phys, :, rows] = True
        for g in range(wl.Hkv):
            z_ref, e_ref = O.append_latents(np64(k[b, :, g]), np64(v[b, :, g]), f["A_V"][g],
                                            f["P_K"][g], f["U_K"][g])
            z = np64(cache_row(layer.Z, wl, "Z", phys, g, rows))
            e = np64(cache_row(layer.E, wl, "E", phys, g, rows))
            if fp8:
                assert_e4m3_bracket(z, z_ref, ZE_REL * np.abs(z_ref).max(), what=f"z b{b} g{g}")
                assert_e4m3_bracket(e, e_ref, ZE_REL * np.abs(e_ref).max(), what=f"e b{b} g{g}")
                kb = layer.K.view(torch.uint8)[phys, g, rows].view(torch.float8_e4m3fn).float()
                np.testing.assert_array_equal(np64(kb), O.to_e4m3(np64(k[b, :, g])))
            else:
                assert_within(z, z_ref, ZE_REL, what=f"z b{b} g{g}")
                assert_within(e, e_ref, ZE_REL, what=f"e b{b} g{g}")
                assert torch.equal(layer.K[phys, g, rows], k[b, :, g])
    keep = ~touched.to(layer.K.device)
    lead = wl.tile_lead()
    for nm, t in (("K", layer.K), ("Z", layer.Z), ("E", layer.E)):
        now, old = t.view(torch.uint8) if fp8 else t, before[nm].view(torch.uint8) if fp8 else before[nm]
        if nm != "K":
            now, old = synth.unsplit_tiles(now, lead[nm]), synth.unsplit_tiles(old, lead[nm])
        assert torch.equal(now[keep], old[keep]), f"{nm}: a row outside the appended tokens changed"


def test_device_status_reports_bad_inputs():
    """A block-table entry outside the cache and an append past the
    block-table row are caught by the kernels' own checks: the work is
    skipped and the status word says why."""
    wl = synth.with_sizes(synth.TINY, T=100)
    pb, layer = gpu_layer(wl)
    status_clean()
    layer.block_table[0, 3] = layer.dims.num_phys_pages + 5
    layer.decode(pb.q, max_seq_len=wl.T)
    assert bkv.read_device_status() & bkv.DEV_BAD_PAGE
    assert bkv.read_device_status() == 0  # cleared
    layer.block_table[0, 3] = 3
    cap = layer.dims.max_pages_per_seq * wl.page_size
    layer.seq_lens.fill_(cap)
    k_new, v_new = synth.make_tokens(wl, pb.factors, 1, device="cuda")
    layer.decode(pb.q, k_new[:, 0].contiguous(), v_new[:, 0].contiguous(), max_seq_len=cap)
    assert bkv.read_device_status() & bkv.DEV_OVERFLOW
    assert layer.seq_lens.item() == cap


def test_prefill_append_reports_bad_pages_and_overflow():
    """The tensor-core append's own checks.  A block-table entry outside
    the cache: that page's rows are skipped (the bad-page bit is set) and
    every other row lands.  A chunk that would pass the end of a sequence's
    block-table row: that sequence is skipped whole (the overflow bit) and
    its length is left as it was, while the other sequence appends."""
    wl = synth.with_sizes(synth.QWEN32B_T64K_B8, B=2, T=160, prefill_tokens=400)
    n, S = 200, wl.page_size
    pb, layer = gpu_layer(wl, seq_lens=[5, 37])
    k, v = synth.make_tokens(wl, pb.factors, n, device="cuda", stream_id=5)
    status_clean()
    lp_bad = (5 + 60) // S  # a page inside sequence 0's chunk
    good = int(layer.block_table[0, lp_bad])
    K0 = layer.K[good].clone()
    layer.block_table[0, lp_bad] = layer.dims.num_phys_pages + 7
    layer.append(k, v, n)
    assert bkv.read_device_status() & bkv.DEV_BAD_PAGE
    assert bkv.read_device_status() == 0  # cleared
    layer.block_table[0, lp_bad] = good
    assert torch.equal(layer.K[good], K0), "rows of the bad page were written"
    for b, L0 in enumerate([5, 37]):
        toks = np.arange(L0, L0 + n)
        keep = toks // S != lp_bad if b == 0 else np.ones(n, dtype=bool)
        phys = layer.block_table[b, toks[keep] // S].long().cpu()
        rows = torch.as_tensor(toks[keep] % S)
        assert torch.equal(layer.K[phys, :, rows], k[b, torch.as_tensor(np.nonzero(keep)[0])])
    assert layer.seq_lens.tolist() == [5 + n, 37 + n]
    # sequence 0 now ends 10 tokens before its block-table row does
    cap = layer.dims.max_pages_per_seq * S
    layer.seq_lens[0] = cap - 10
    layer.append(k, v, n)
    assert bkv.read_device_status() & bkv.DEV_OVERFLOW
    assert layer.seq_lens.tolist() == [cap - 10, 37 + 2 * n]
    toks = np.arange(37 + n, 37 + 2 * n)
    phys = layer.block_table[1, toks // S].long().cpu()
    assert torch.equal(layer.K[phys, :, torch.as_tensor(toks % S)], k[1])


@pytest.mark.parametrize("T", [16384, 2048], ids=["p1024", "p128"])
@pytest.mark.parametrize("levels", [1, 3, 64])
def test_selection_with_tied_scores(levels, T):
    """Page scores with many exact ties: z is zero except column 0 of every
    token, which holds one of `levels` values per page, and e is zero, so a
    page's score is one product per head and pages with the same value tie
    exactly (levels = 1: every score equal).  At 1024 pages the threshold's
    bin then holds hundreds of pages (1, 3 levels: the radix select decides)
    or a few (64 levels); at 128 pages every candidate is ranked directly.
    Ties rank by the lower page index on both sides, so the selection must
    equal the oracle's bit for bit, through the selection launch and through
    the fused decode step."""
    wl = synth.with_sizes(synth.LLAMA8B_T32K_B16, B=2, T=T, top_k=64)
    pb = synth.make_problem(wl, device="cuda")
    S, P = wl.page_size, wl.pages
    lvl = torch.arange(P, device="cuda").remainder(levels).float() + 1.0
    z = torch.zeros_like(pb.cache["Z"])
    z[:, :, :P * S, 0] = lvl.repeat_interleave(S).bfloat16()
    pb.cache["Z"] = z
    pb.cache["E"] = torch.zeros_like(pb.cache["E"])
    layer = DecodeLayer.from_problem(pb)
    scores = torch.empty(wl.B, wl.Hkv, layer.dims.max_pages_per_seq, device="cuda")
    sel_r = torch.empty(wl.B, wl.Hkv, wl.top_k, dtype=torch.int32, device="cuda")
    bkv.basiskv_route(layer.dims, pb.q, layer.seq_lens, wl.T, layer.block_table, layer.P_K,
                      layer.U_K, layer.Z, layer.E, wl.top_k, scores, sel_r, layer.workspace)
    sel_d = torch.empty_like(sel_r)
    layer.decode(pb.q, sel=sel_d, max_seq_len=wl.T)
    status_clean()
    for b in range(wl.B):
        for g in range(wl.Hkv):
            _, ref_sel, _ = oracle_route(pb, b, g, wl.T)
            np.testing.assert_array_equal(sel_r[b, g].cpu().numpy(), ref_sel)
            np.testing.assert_array_equal(sel_d[b, g].cpu().numpy(), ref_sel)
