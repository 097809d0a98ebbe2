"""CPU checks of the seeded input generators (layout only, no method
arithmetic): the paged-cache generator used for the large sweep workloads
writes exactly what the logical cache paginated through the block table
holds, and the paged key view reads the same keys."""
import torch

from sparse_decode_attention_basiskv_b200 import synth


def _cases():
    base = synth.with_sizes(synth.TINY, B=3, T=200)  # ragged last page
    return [base,
            synth.with_sizes(base, T=192),  # whole pages only
            synth.with_sizes(base, cache_fp8=1),
            synth.with_sizes(synth.LLAMA8B_T4K, B=2, T=100, Hq=8, Hkv=2, hidden=256,
                             route_r_v=16, route_r_k=16, top_k=8)]


def test_paged_cache_matches_paginated_logical_cache():
    for wl in _cases():
        pb = synth.make_problem(wl, layer=3)
        want = pb.paged()
        got = synth.make_paged_cache(wl, pb.factors, pb.table, layer=3)
        for name in ("K", "Z", "E"):
            assert got[name].dtype == want[name].dtype, (wl.name, name)
            a, b = got[name], want[name]
            if a.dtype == torch.float8_e4m3fn:
                a, b = a.view(torch.uint8), b.view(torch.uint8)
            assert torch.equal(a, b), (wl.name, name)


def test_paged_keys_view_reads_logical_keys():
    wl = synth.with_sizes(synth.TINY, B=2, T=200)
    pb = synth.make_problem(wl)
    paged = pb.paged()
    view = synth.PagedKeys(paged["K"], pb.table, wl.page_size)
    for b, g, t in [(0, 0, 0), (1, 0, 17), (1, 0, 199), (0, 0, 63)]:
        assert torch.equal(view[b, g, t], pb.cache["K"][b, g, t])
    q_log, used_log = synth.make_query(wl, pb.cache["K"], wl.T, step=2)
    q_pag, used_pag = synth.make_query(wl, view, wl.T, step=2)
    assert torch.equal(q_log, q_pag) and torch.equal(used_log, used_pag)


def test_tokens_are_dense():
    """The new tokens are handed to the library as raw pointers: both k and
    v come back dense and row-major, whatever layout the einsum that builds
    k picked."""
    wl = synth.with_sizes(synth.TINY, B=2)
    factors = synth.make_factors(wl)
    k, v = synth.make_tokens(wl, factors, 5)
    assert k.shape == v.shape == (2, 5, wl.Hkv, wl.d)
    assert k.is_contiguous() and v.is_contiguous()
