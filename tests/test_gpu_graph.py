"""A decode step captured once in a CUDA graph and replayed: the same y,
selection and lengths as the eager calls, step after step (the lengths
advance on the device inside the graph)."""
import pytest
import torch

from sparse_decode_attention_basiskv_b200 import synth
from sparse_decode_attention_basiskv_b200.layer import DecodeLayer, DecodeStack

from harness import status_clean

pytestmark = pytest.mark.gpu


def _steps(wl, n):
    pb = synth.make_problem(wl, device="cuda")
    k, v = synth.make_tokens(wl, pb.factors, n + 1, device="cuda")
    qs = [synth.make_query(wl, pb.cache["K"], wl.T, step=i)[0] for i in range(n + 1)]
    return pb, qs, [k[:, i].contiguous() for i in range(n + 1)], [v[:, i].contiguous() for i in range(n + 1)]


@pytest.mark.parametrize("wl", [synth.with_sizes(synth.LLAMA8B_T4K, B=2, T=1000, top_k=16),
                                synth.with_sizes(synth.LLAMA8B_T32K_B16_FP8, B=2, T=900, top_k=16)],
                         ids=["bf16", "e4m3"])
def test_graph_replay_matches_eager(wl):
    n = 4
    pb, qs, ks, vs = _steps(wl, n)
    eager = DecodeLayer.from_problem(pb)
    graphed = DecodeLayer.from_problem(pb)
    cap = eager.max_seq_len
    ref = []
    for i in range(n + 1):
        ref.append(eager.decode(qs[i], ks[i], vs[i], max_seq_len=cap).clone())
    # the graphed layer: one eager step, then capture and replay the rest
    q_s, k_s, v_s = qs[0].clone(), ks[0].clone(), vs[0].clone()
    y0 = graphed.decode(q_s, k_s, v_s, max_seq_len=cap).clone()
    torch.cuda.synchronize()
    g = graphed.capture(q_s, k_s, v_s, max_seq_len=cap)
    # capture records the step without running it
    assert (graphed.seq_lens == wl.T + 1).all()
    got = [y0]
    for i in range(1, n + 1):
        q_s.copy_(qs[i])
        k_s.copy_(ks[i])
        v_s.copy_(vs[i])
        got.append(g.replay().clone())
    torch.cuda.synchronize()
    status_clean()
    assert torch.equal(graphed.seq_lens, eager.seq_lens)
    for i in range(n + 1):
        assert torch.equal(got[i], ref[i]), f"step {i}"
    for name in ("K", "Z", "E"):
        assert torch.equal(getattr(graphed, name).view(torch.uint8),
                           getattr(eager, name).view(torch.uint8))


def test_stack_graph_replay_matches_eager():
    base = synth.with_sizes(synth.LLAMA8B_T32K_B16, B=2, T=700, top_k=12)
    wls = synth.stack_layers(base, [64, 96, 32])
    pbs = [synth.make_problem(wl, device="cuda", layer=l) for l, wl in enumerate(wls)]
    toks = [synth.make_tokens(wl, pb.factors, 3, device="cuda", stream_id=l)
            for l, (wl, pb) in enumerate(zip(wls, pbs))]
    eager = DecodeStack([DecodeLayer.from_problem(pb) for pb in pbs])
    graphed = DecodeStack([DecodeLayer.from_problem(pb) for pb in pbs])
    cap = min(L.max_seq_len for L in eager.layers)
    qs = [pb.q for pb in pbs]
    ref = []
    for i in range(3):
        ks = [k[:, i].contiguous() for k, _ in toks]
        vs = [v[:, i].contiguous() for _, v in toks]
        ref.append([y.clone() for y in eager.decode(qs, ks, vs, max_seq_len=cap)])
    k_s = [k[:, 0].contiguous() for k, _ in toks]
    v_s = [v[:, 0].contiguous() for _, v in toks]
    got = [[y.clone() for y in graphed.decode(qs, k_s, v_s, max_seq_len=cap)]]
    torch.cuda.synchronize()
    g = graphed.capture(qs, k_s, v_s, max_seq_len=cap)
    for i in (1, 2):
        for l, (k, v) in enumerate(toks):
            k_s[l].copy_(k[:, i])
            v_s[l].copy_(v[:, i])
        got.append([y.clone() for y in g.replay()])
    torch.cuda.synchronize()
    status_clean()
    for i in range(3):
        for l in range(3):
            assert torch.equal(got[i][l], ref[i][l]), f"step {i} layer {l}"
