"""Parity of the 32-layer decode sweep (the Llama-3.1-8B layer shape, top-k
= T/64 pages of 16 tokens, one token appended per sequence per step) at its
largest sizes, in the launch configuration the sweep benchmark times (one
fused basiskv_decode per layer and step).

Per point: two of the 32 layers (their own factors and caches), three
decode steps each.  The oracle carries its own copy of each sampled
sequence's cache (it appends with its own arithmetic every step) and is
compared with the GPU on the first and the last step: appended state, page
selection (bit-exact outside near ties, a valid choice inside them) and y.
These points select up to 2048 of 8192 pages per group, attend over 32K
tokens per group, and run 64 sequences at once."""
import numpy as np
import pytest
import torch

from oracle import basiskv_oracle as O
from sparse_decode_attention_basiskv_b200 import synth
from sparse_decode_attention_basiskv_b200.layer import DecodeLayer

from harness import StepChecker, ZE_REL, assert_within, cache_row, np64, status_clean

pytestmark = pytest.mark.gpu

POINTS = [(1, 131072, 96), (8, 32768, 64), (64, 32768, 96), (32, 131072, 64)]
LAYERS = (0, 31)
STEPS = 3


def _samples(B: int) -> list:
    return sorted({0, B // 2, B - 1})


@pytest.mark.parametrize("B,T,r_v", POINTS, ids=[f"b{b}_t{t // 1024}k_v{r}" for b, t, r in POINTS])
def test_sweep_point_first_and_last_step(B, T, r_v):
    wl = synth.sweep_point(B, T, r_v, layers=32, steps=STEPS)
    assert wl.top_k == T // 64
    samples = _samples(B)
    for layer_id in LAYERS:
        factors = synth.make_factors(wl, layer_id)
        table = synth.block_table(wl)
        paged = synth.make_paged_cache(wl, factors, table.cuda(), "cuda", layer_id)
        keys = synth.PagedKeys(paged["K"], table, wl.page_size)
        queries = [synth.make_query(wl, keys, T, step=s)[0] for s in range(STEPS)]
        layer = DecodeLayer.from_parts(wl, factors, paged, table)
        del paged, keys
        f = {k: np64(v) for k, v in factors.items()}
        W = O.fold_outproj(f["B_V"], f["W_O"], wl.Hq)
        # the oracle's own caches of the sampled sequences (bf16 values held
        # exactly in float32; the oracle's arithmetic promotes to float64)
        oc = {}
        for b in samples:
            c = synth.make_cache(wl, factors, "cuda", layer_id, seqs=[b])
            oc[b] = {k: v[0].float().cpu().numpy() for k, v in c.items()}
            del c
        torch.cuda.empty_cache()
        chk = StepChecker(wl, W, f"{wl.name} layer {layer_id}")
        for step in range(STEPS):
            Tc = T + step
            k_new, v_new = synth.make_tokens(wl, factors, 1, device="cuda",
                                             stream_id=100 * layer_id + step)
            k_new, v_new = k_new[:, 0].contiguous(), v_new[:, 0].contiguous()
            sel = torch.empty(B, wl.Hkv, wl.top_k, dtype=torch.int32, device="cuda")
            y = layer.decode(queries[step], k_new, v_new, sel=sel, max_seq_len=Tc + 1).clone()
            status_clean()
            assert layer.seq_lens.tolist() == [Tc + 1] * B
            compared = step in (0, STEPS - 1)
            for b in samples:
                c = oc[b]
                kb, vb = np64(k_new[b]), np64(v_new[b])
                if compared:
                    q_b = np64(queries[step][b])
                    out = O.decode_sequence(q_b, c["K"], c["Z"], c["E"], Tc, wl.page_size,
                                            wl.top_k, f["P_K"], f["U_K"], W, k_new=kb,
                                            v_new=vb, A_V=f["A_V"])
                    z_new, e_new = out["z_new"], out["e_new"]
                    slot_page = layer.block_table[b, Tc // wl.page_size].item()
                    for g in range(wl.Hkv):
                        slot = (slot_page, g, Tc % wl.page_size)
                        assert_within(np64(cache_row(layer.Z, wl, "Z", *slot)), z_new[g], ZE_REL,
                                      what=f"z step {step} b{b} g{g}")
                        assert_within(np64(cache_row(layer.E, wl, "E", *slot)), e_new[g], ZE_REL,
                                      what=f"e step {step} b{b} g{g}")
                        assert torch.equal(layer.K[slot], k_new[b, g])
                    chk.check(b, out, sel[b].cpu().numpy(), np64(y[b]), q_b)
                    del out
                else:
                    z_new, e_new = zip(*(O.append_latents(kb[g][None], vb[g][None], f["A_V"][g],
                                                          f["P_K"][g], f["U_K"][g])
                                         for g in range(wl.Hkv)))
                    z_new = np.stack([z[0] for z in z_new])
                    e_new = np.stack([e[0] for e in e_new])
                for g in range(wl.Hkv):  # the oracle's own append into its cache
                    c["Z"][g, Tc] = O.to_bf16(z_new[g])
                    c["E"][g, Tc] = O.to_bf16(e_new[g])
                    c["K"][g, Tc] = kb[g]
            # the sink and the newest page (holding this step's token) are kept
            assert (sel[:, :, 0] == 0).all()
            assert (sel[:, :, -1] == Tc // wl.page_size).all()
        chk.report()
        del layer, oc
        torch.cuda.empty_cache()
