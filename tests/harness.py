"""Shared helpers for the GPU parity tests: run the CUDA path through the
C-ABI binding and the CPU oracle on the same seeded inputs, and compare.

Tolerances (written out here, used by every test):
* indices (page selection): bit-exact, except (sequence, KV head) slots the
  oracle flags as near ties (its k-th and (k+1)-th float32 scores within
  1e-4 relative), which are counted and reported separately; there the GPU's
  selection must equal the oracle's or be another valid choice: the forced
  pages kept, and every page it differs by scored (by the oracle) within
  the near-tie window of the oracle's threshold;
* y:      max|y - y_ref| <= 1e-2 * max|y_ref| + 1e-3, y_ref from the oracle's
  attention on the GPU's selection when a near tie made them differ;
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
                       wl.sel_page, r["r_b"], r["r_q"])
    sel, tie = O.select_pages(sc, wl.top_k, r["n_sink"], r["n_recent"])
    return sc, sel, tie


TIE_REL = 1e-4  # the near-tie window of the selection


class StepChecker:
    """Checks decode steps against the oracle, one sequence at a time.

    check(): every clean group's selection is bit-exact; a near-tie group's
    is bit-exact or another valid choice (see the module docstring); y is
    compared with the oracle's own y, or, where a near tie made a group
    choose differently, with the oracle's attention and out-projection
    recomputed on the GPU's (validated) selection, so no sequence is
    skipped.  report() prints the near-tie counts and asserts that no clean
    group mismatched and that clean groups exist."""

    def __init__(self, wl, W_fold, what: str = ""):
        self.wl, self.W, self.what = wl, W_fold, what
        self.stats = {"groups": 0, "clean": 0, "tie": 0, "clean_mismatch": 0,
                      "tie_other_choice": 0, "y_checked": 0, "y_on_gpu_selection": 0}

    def _valid_alternative(self, gsel: np.ndarray, scores, ref: np.ndarray) -> bool:
        r = self.wl.router
        s = np.asarray(scores, dtype=np.float32).astype(np.float64)
        s[s == 0.0] = 0.0
        P = len(s)
        gs, rs = gsel[gsel >= 0], ref[ref >= 0]
        if len(gs) != len(rs) or not np.array_equal(gsel[len(gs):], ref[len(rs):]):
            return False
        if np.any(np.diff(gs) <= 0) or gs.min() < 0 or gs.max() >= P:
            return False
        forced = set(range(r["n_sink"])) | set(range(P - r["n_recent"], P))
        if not forced <= set(gs.tolist()):
            return False
        chosen = [p for p in rs.tolist() if p not in forced]
        thr = min(s[chosen])
        diff = set(gs.tolist()) ^ set(rs.tolist())
        return all(abs(s[p] - thr) <= TIE_REL * max(abs(s[p]), abs(thr)) for p in diff)

    def group(self, b: int, g: int, gpu_sel: np.ndarray, scores, ref_sel: np.ndarray,
              tie: bool) -> bool:
        """Checks one group's selection against the oracle's (scores, sel,
        near-tie flag); returns True when it is another valid choice."""
        self.stats["groups"] += 1
        self.stats["tie" if tie else "clean"] += 1
        if np.array_equal(gpu_sel, ref_sel):
            return False
        if not tie:
            self.stats["clean_mismatch"] += 1
            raise AssertionError(f"{self.what}: selection of b{b} g{g} differs outside a "
                                 f"near tie: {gpu_sel.tolist()} vs {ref_sel.tolist()}")
        assert self._valid_alternative(gpu_sel, scores, ref_sel), (
            f"{self.what}: near-tie group b{b} g{g} chose an invalid page set")
        self.stats["tie_other_choice"] += 1
        return True

    def selection(self, b: int, out: dict, gpu_sel_b: np.ndarray) -> list:
        """Checks one sequence's groups; returns the groups whose GPU
        selection differs (validly) from the oracle's."""
        return [g for g in range(len(out["sel"]))
                if self.group(b, g, gpu_sel_b[g], out["scores"][g], out["sel"][g],
                              bool(out["near_tie"][g]))]

    def expected(self, out: dict, q_b: np.ndarray, gpu_sel_b: np.ndarray, other: list) -> tuple:
        """(a_ref, y_ref) of one sequence on the GPU's selection."""
        if not other:
            return out["a"], out["y"]
        G, S = self.wl.G, self.wl.sel_page
        a = out["a"].copy()
        for g in other:
            a[g * G:(g + 1) * G], _ = O.attend(q_b[g * G:(g + 1) * G], out["K"][g], out["Z"][g],
                                               gpu_sel_b[g], out["T"], S)
        return a, O.outproj(a, self.W)

    def check(self, b: int, out: dict, gpu_sel_b: np.ndarray, gpu_y_b: np.ndarray,
              q_b: np.ndarray) -> None:
        other = self.selection(b, out, gpu_sel_b)
        _, y_ref = self.expected(out, q_b, gpu_sel_b, other)
        assert_within(gpu_y_b, y_ref, Y_REL, Y_ABS, what=f"{self.what} y b{b}")
        self.stats["y_checked"] += 1
        self.stats["y_on_gpu_selection"] += bool(other)

    def report(self) -> dict:
        st = self.stats
        print(f"[{self.what}] {st['groups']} groups: {st['tie']} near ties "
              f"({st['tie_other_choice']} chose another valid set), {st['clean']} clean; "
              f"y checked on {st['y_checked']} sequences "
              f"({st['y_on_gpu_selection']} on the GPU's selection)")
        assert st["clean_mismatch"] == 0, st
        assert st["clean"] > 0, f"{self.what}: no clean group to compare bit-exactly: {st}"
        return st


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
