"""Shared helpers for the GPU parity tests: run the CUDA path through the
C-ABI binding and the CPU oracle on the same seeded inputs, and compare.

Tolerances (written out here, used by every test):
* indices (page selection): bit-exact, except (sequence, KV head) slots the
  oracle flags as near ties (its k-th and (k+1)-th float32 scores within
  1e-4 relative), which are counted separately;
* y:      max|y - y_ref| <= 1e-2 * max|y_ref| + 1e-3;
* z, e:   max|x - x_ref| <= 1e-2 * max|x_ref|  (appended state);
* page scores: max|s - s_ref| <= 1e-4 * max|s_ref| per group: fp32
  accumulation over r_v + r_k products per head (relative error ~1e-6),
  loosened to the near-tie window so the two criteria agree;
* a (latent attention output, fp32): max|a - a_ref| <= 1e-3 * max|a_ref|:
  fp32 accumulation and exp2 over at most a few thousand tokens;
* folded W' (bf16): |W - W_ref| <= 2^-8 |W_ref| + 1e-5 max|W_ref|: one bf16
  rounding of an fp32 sum.
"""
from __future__ import annotations

import numpy as np
import torch

import sparse_decode_attention_basiskv_b200 as bkv
from oracle import basiskv_oracle as O
from sparse_decode_attention_basiskv_b200 import synth
from sparse_decode_attention_basiskv_b200.layer import DecodeLayer

Y_REL, Y_ABS = 1e-2, 1e-3
ZE_REL = 1e-2
S_REL = 1e-4
A_REL = 1e-3


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def factors_np(pb) -> dict:
    return {k: np64(v) for k, v in pb.factors.items()}


def within(x, ref, rel, absol=0.0) -> tuple:
    err = float(np.max(np.abs(np.asarray(x) - np.asarray(ref)))) if np.size(ref) else 0.0
    bound = rel * float(np.max(np.abs(ref))) + absol if np.size(ref) else 0.0
    return err <= bound, err, bound


def assert_within(x, ref, rel, absol=0.0, what=""):
    ok, err, bound = within(x, ref, rel, absol)
    assert ok, f"{what}: max err {err:.3e} > bound {bound:.3e}"


def gpu_layer(wl, seq_lens=None):
    pb = synth.make_problem(wl, device="cuda")
    if seq_lens is not None:
        pb.seq_lens = torch.as_tensor(seq_lens, dtype=torch.int32, device="cuda")
    layer = DecodeLayer.from_problem(pb)
    return pb, layer


def oracle_route(pb, b: int, g: int, T: int, cache=None) -> tuple:
    """Oracle scores / selection / near-tie flag of one (sequence, KV head)."""
    wl = pb.wl
    f = factors_np(pb)
    c = pb.cache if cache is None else cache
    qg = np64(pb.q[b, g * wl.G:(g + 1) * wl.G])
    r = wl.router
    sc = O.page_scores(qg, np64(c["Z"][b, g]), np64(c["E"][b, g]), f["P_K"][g], f["U_K"][g], T,
                       wl.page_size, r["r_b"], r["r_q"])
    sel, tie = O.select_pages(sc, wl.top_k, r["n_sink"], r["n_recent"])
    return sc, sel, tie


def compare_selection(gpu_sel: np.ndarray, ref_sel: np.ndarray, tie: bool, stats: dict):
    same = np.array_equal(gpu_sel, ref_sel)
    key = "tie" if tie else "clean"
    stats.setdefault(key, 0)
    stats.setdefault(key + "_mismatch", 0)
    stats[key] += 1
    if not same:
        stats[key + "_mismatch"] += 1
    return same


def status_clean():
    flags = bkv.read_device_status()
    assert flags == 0, f"device status bits {flags:#x}"


def cache_row(paged, wl, name: str, phys: int, g: int, rows):
    """Rows of one (page, KV head) tile of a paged cache in logical column
    order (undoing the narrow router's column split)."""
    lead = wl.tile_lead().get(name, paged.shape[-1])
    fp8 = paged.dtype == torch.float8_e4m3fn
    src = paged.view(torch.uint8) if fp8 else paged  # byte moves only
    tiles = synth.unsplit_tiles(src[phys, g], lead)
    if tiles.dim() == 2:  # one tile
        out = tiles[rows]
    else:
        out = tiles[torch.arange(tiles.shape[0], device=tiles.device),
                    torch.as_tensor(rows).to(tiles.device)]
    return out.view(torch.float8_e4m3fn).float() if fp8 else out


def assert_e4m3_bracket(x, ref, tol, what=""):
    """x (E4M3 values) is the E4M3 rounding of some value within tol
    (elementwise absolute) of ref: to_e4m3(ref - tol) <= x <= to_e4m3(ref +
    tol), to_e4m3 being monotone."""
    x, ref = np.asarray(x, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    lo, hi = O.to_e4m3(ref - tol), O.to_e4m3(ref + tol)
    bad = (x < lo) | (x > hi)
    assert not bad.any(), (f"{what}: {int(bad.sum())} values outside their E4M3 bracket, "
                           f"first x={x[bad][0]} ref={ref[bad][0]}")
