"""A layer stack whose Value width varies per layer (Table 12's per-layer
V ranks): each layer's fused decode step matches the oracle at its own
width, run in order through one DecodeStack."""
import pytest
import torch

from oracle import basiskv_oracle as O
from sparse_decode_attention_basiskv_b200 import synth
from sparse_decode_attention_basiskv_b200.layer import DecodeLayer, DecodeStack

from harness import StepChecker, factors_np, np64, status_clean

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("base,widths", [
    (synth.with_sizes(synth.LLAMA8B_T32K_B16, B=2, T=1500, top_k=24), [32, 64, 128, 96]),
    (synth.with_sizes(synth.QWEN32B_T64K_B8, B=2, T=1200, prefill_tokens=0, top_k=16),
     [64, 32, 96]),
    # E4M3 caches (their scoring instances start at r_v 64)
    (synth.with_sizes(synth.LLAMA8B_T32K_B16_FP8, B=2, T=1500, top_k=24), [96, 64, 128]),
], ids=["llama", "qwen", "llama_e4m3"])
def test_stack_with_per_layer_widths(base, widths):
    wls = synth.stack_layers(base, widths)
    pbs = [synth.make_problem(wl, device="cuda", layer=l) for l, wl in enumerate(wls)]
    stack = DecodeStack([DecodeLayer.from_problem(pb) for pb in pbs])
    assert stack.widths == widths
    toks = [synth.make_tokens(wl, pb.factors, 1, device="cuda", stream_id=l)
            for l, (wl, pb) in enumerate(zip(wls, pbs))]
    ks = [k[:, 0].contiguous() for k, _ in toks]
    vs = [v[:, 0].contiguous() for _, v in toks]
    ys = [y.clone() for y in stack.decode([pb.q for pb in pbs], ks, vs, max_seq_len=base.T + 1)]
    status_clean()
    # the same step of each layer again (lengths reset), with its selection
    # written out: equal outputs, and the selection to check
    for L in stack.layers:
        L.seq_lens.fill_(base.T)
    sels = [torch.empty(wl.B, wl.Hkv, wl.top_k, dtype=torch.int32, device="cuda") for wl in wls]
    for L, pb, k, v, s_, y in zip(stack.layers, pbs, ks, vs, sels, ys):
        assert torch.equal(L.decode(pb.q, k, v, sel=s_, max_seq_len=base.T + 1), y)
    status_clean()
    for l, (wl, pb) in enumerate(zip(wls, pbs)):
        f = factors_np(pb)
        W = O.fold_outproj(f["B_V"], f["W_O"], wl.Hq)
        assert stack.layers[l].seq_lens.tolist() == [base.T + 1] * wl.B
        chk = StepChecker(wl, W, f"layer {l}")
        for b in range(wl.B):
            c = {k: np64(v[b]) for k, v in pb.cache.items()}
            out = O.decode_sequence(np64(pb.q[b]), c["K"], c["Z"], c["E"], wl.T, wl.page_size,
                                    wl.top_k, f["P_K"], f["U_K"], W, k_new=np64(ks[l][b]),
                                    v_new=np64(vs[l][b]), A_V=f["A_V"], fp8=bool(wl.cache_fp8),
                                    **wl.router)
            assert out["a"].shape[1] == widths[l]
            chk.check(b, out, sels[l][b].cpu().numpy(), np64(ys[l][b]), np64(pb.q[b]))
        chk.report()
