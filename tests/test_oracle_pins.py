"""Pins of the CPU oracle against facts that do not come from the oracle.

Each test checks the oracle against brute force, a closed form, an
invariant, or a textbook/library routine (torch's scaled-dot-product
attention with grouped heads), chosen so that a dropped term, a wrong sign,
a wrong index or a transposed operand in the oracle fails at least one.
CPU only; no GPU, no CUDA library.
"""
import itertools

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import basiskv_oracle as O
from sparse_decode_attention_basiskv_b200 import synth


def _orth(rng, n, m):
    q, r = np.linalg.qr(rng.standard_normal((n, m)))
    return q * np.sign(np.diag(r))[None, :]


# ---------------------------------------------------------------- selection
def _dominates(s, c, u):
    return s[c] > s[u] or (s[c] == s[u] and c < u)


@pytest.mark.parametrize("P", range(1, 10))
def test_select_matches_brute_force(P):
    rng = np.random.default_rng(P)
    for trial in range(40):
        # small integers give many exact ties; include signed zeros
        s = rng.integers(-3, 4, size=P).astype(np.float64)
        s[s == 0] = np.where(rng.random(int((s == 0).sum())) < 0.5, -0.0, 0.0)
        for k in range(2, P + 3):
            sel, _ = O.select_pages(s, k)
            got = [int(p) for p in sel if p >= 0]
            assert list(sel[len(got):]) == [-1] * (k - len(got))
            if k >= P:
                assert got == list(range(P))
                continue
            cand = list(range(1, P - 1))
            need = k - 2
            sz = np.where(s == 0, 0.0, s)  # -0 == +0
            valid = []
            for chosen in itertools.combinations(cand, need):
                rest = [u for u in cand if u not in chosen]
                if all(_dominates(sz, c, u) for c in chosen for u in rest):
                    valid.append(sorted({0, P - 1, *chosen}))
            assert len(valid) == 1
            assert got == valid[0]


@pytest.mark.parametrize("P", range(1, 10))
def test_select_sink_and_recent_windows_brute_force(P):
    """The first n_sink and last n_recent pages are forced; the rest of the
    budget goes to the unique dominating set of the middle pages."""
    rng = np.random.default_rng(100 + P)
    for trial in range(15):
        s = rng.integers(-2, 3, size=P).astype(np.float64)
        for n_sink, n_recent in [(0, 1), (1, 2), (2, 1), (2, 3), (0, 3)]:
            for k in range(n_sink + n_recent, P + 2):
                if k < 1:
                    continue
                sel, _ = O.select_pages(s, k, n_sink, n_recent)
                got = [int(p) for p in sel if p >= 0]
                if k >= P:
                    assert got == list(range(P))
                    continue
                forced = set(range(n_sink)) | set(range(P - n_recent, P))
                cand = [p for p in range(P) if p not in forced]
                need = k - len(forced)
                valid = []
                for chosen in itertools.combinations(cand, need):
                    rest = [u for u in cand if u not in chosen]
                    if all(_dominates(s, c, u) for c in chosen for u in rest):
                        valid.append(sorted(forced | set(chosen)))
                assert len(valid) == 1
                assert got == valid[0]


def test_select_near_tie_flag():
    s = np.array([0.0, 5.0, 3.0, 3.0000001, 1.0, 0.0])
    _, tie = O.select_pages(s, 4)  # last chosen 3.0000001 vs rejected 3.0
    assert tie
    _, tie = O.select_pages(np.array([0.0, 5.0, 3.0, 2.0, 1.0, 0.0]), 4)
    assert not tie


# ------------------------------------------------------ append + prediction
def test_khat_exact_when_residual_completes_basis():
    """r_k = d with square orthonormal U_K: khat reproduces k exactly."""
    rng = np.random.default_rng(1)
    d, r_v, n = 16, 6, 9
    A_V = rng.standard_normal((d, r_v))
    P_K = rng.standard_normal((r_v, d))
    U_K = _orth(rng, d, d)
    k, v = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    z, e = O.append_latents(k, v, A_V, P_K, U_K)
    np.testing.assert_allclose(z, v @ A_V, atol=1e-12)
    np.testing.assert_allclose(O.predicted_keys(z, e, P_K, U_K), k, atol=1e-12)


def test_residual_recovers_code_noise_free():
    """k = (v A_V) P_K + e' U_K^T with orthonormal U_K (r_k < d): e == e'."""
    rng = np.random.default_rng(2)
    d, r_v, r_k, n = 32, 8, 5, 7
    A_V = rng.standard_normal((d, r_v))
    P_K = rng.standard_normal((r_v, d))
    U_K = _orth(rng, d, r_k)
    v = rng.standard_normal((n, d))
    ep = rng.standard_normal((n, r_k))
    k = (v @ A_V) @ P_K + ep @ U_K.T
    z, e = O.append_latents(k, v, A_V, P_K, U_K)
    np.testing.assert_allclose(e, ep, atol=1e-12)
    np.testing.assert_allclose(O.predicted_keys(z, e, P_K, U_K), k, atol=1e-12)


def test_identity_factors_closed_form():
    """A_V = I, P_K = I, U_K = I: z = v and e = k - v."""
    rng = np.random.default_rng(3)
    d = 8
    k, v = rng.standard_normal((4, d)), rng.standard_normal((4, d))
    I = np.eye(d)
    z, e = O.append_latents(k, v, I, I, I)
    np.testing.assert_array_equal(z, v)
    np.testing.assert_allclose(e, k - v, atol=1e-15)


# ---------------------------------------------------------------- routing
@pytest.mark.parametrize("r_b,r_q", [(4, 3), (8, 0), (0, 5), (8, 5)])
def test_narrow_router_equals_zeroed_factors(r_b, r_q):
    """A router reading z[:, :r_b] and e[:, :r_q] scores exactly like the
    full router with P_K rows >= r_b and U_K columns >= r_q set to zero."""
    rng = np.random.default_rng(7 + r_b * 10 + r_q)
    d, r_v, r_k, G, T, S = 16, 8, 5, 3, 45, 8
    P_K = rng.standard_normal((r_v, d))
    U_K = _orth(rng, d, r_k)
    z = rng.standard_normal((T, r_v))
    e = rng.standard_normal((T, r_k))
    q = rng.standard_normal((G, d))
    narrow = O.page_scores(q, z, e, P_K, U_K, T, S, r_b, r_q)
    Pz, Uz = P_K.copy(), U_K.copy()
    Pz[r_b:] = 0.0
    Uz[:, r_q:] = 0.0
    np.testing.assert_allclose(narrow, O.page_scores(q, z, e, Pz, Uz, T, S), atol=1e-12)
    full = O.page_scores(q, z, e, P_K, U_K, T, S, r_v, r_k)
    np.testing.assert_array_equal(full, O.page_scores(q, z, e, P_K, U_K, T, S))


def test_narrow_router_ignores_unread_dimensions():
    """Latent dims >= r_b and residual dims >= r_q carry all the signal: the
    narrow router's scores are exactly zero."""
    rng = np.random.default_rng(8)
    d, r_v, r_k, T, S = 16, 8, 6, 30, 8
    z = np.zeros((T, r_v))
    z[:, 4:] = rng.standard_normal((T, 4))
    e = np.zeros((T, r_k))
    e[:, 2:] = rng.standard_normal((T, 4))
    sc = O.page_scores(rng.standard_normal((2, d)), z, e, rng.standard_normal((r_v, d)),
                       _orth(rng, d, r_k), T, S, 4, 2)
    np.testing.assert_array_equal(sc, np.zeros_like(sc))
@pytest.mark.parametrize("T,S", [(37, 8), (32, 8), (5, 16), (64, 16), (39, 4), (3, 4)])
def test_page_scores_closed_form(T, S):
    """khat_t = c_t u and q_h = alpha_h u  =>  score(p) = max_{t,h} alpha_h c_t.

    Slots beyond T carry huge c_t and must not count."""
    rng = np.random.default_rng(T * 100 + S)
    d, r_v, G = 12, 5, 3
    cap = -(-T // S) * S + S
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    c = rng.standard_normal(cap) * 3
    c[T:] = 1e6
    alpha = rng.standard_normal(G)
    P_K = rng.standard_normal((r_v, d))
    U_K = np.eye(d)
    z = rng.standard_normal((cap, r_v))
    e = c[:, None] * u[None, :] - z @ P_K
    q = alpha[:, None] * u[None, :]
    got = O.page_scores(q, z, e, P_K, U_K, T, S)
    P = -(-T // S)
    assert got.shape == (P,)
    for p in range(P):
        want = max(a * c[t] for t in range(p * S, min((p + 1) * S, T))
                   for a in alpha)
        assert abs(got[p] - want) <= 1e-9 * (1 + abs(want))


# -------------------------------------------------------------- attention
def _sdpa_gqa(q, K, V):
    """torch SDPA in float64; q [Hq][d], K [Hkv][n][d], V [Hkv][n][r]."""
    o = F.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(K)[None],
        torch.from_numpy(V)[None], enable_gqa=True)
    return o[0, :, 0].numpy()


@pytest.mark.parametrize("T,S", [(40, 8), (48, 16), (7, 8), (22, 4)])
def test_attend_all_pages_equals_sdpa(T, S):
    rng = np.random.default_rng(T + S)
    G, d, r_v = 4, 16, 6
    q = rng.standard_normal((G, d))
    K = rng.standard_normal((T + S, d))
    z = rng.standard_normal((T + S, r_v))
    P = -(-T // S)
    sel = np.arange(P)
    a, w = O.attend(q, K, z, sel, T, S)
    want = _sdpa_gqa(q, K[None, :T], z[None, :T])
    np.testing.assert_allclose(a, want, atol=1e-12)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-13)
    assert (w >= 0).all()


def test_attend_selected_subset_equals_sdpa_on_subset():
    rng = np.random.default_rng(5)
    G, d, r_v, S, T = 2, 8, 4, 4, 21  # 6 pages, last one partial (1 token)
    q = rng.standard_normal((G, d))
    K = rng.standard_normal((24, d))
    z = rng.standard_normal((24, r_v))
    sel = np.array([0, 2, 5, -1])
    toks = [0, 1, 2, 3, 8, 9, 10, 11, 20]
    a, _ = O.attend(q, K, z, sel, T, S)
    np.testing.assert_allclose(a, _sdpa_gqa(q, K[None, toks], z[None, toks]),
                               atol=1e-12)


def test_attend_equal_keys_gives_mean():
    rng = np.random.default_rng(6)
    S, T = 8, 29
    K = np.tile(rng.standard_normal(16), (32, 1))
    z = rng.standard_normal((32, 3))
    sel = np.array([1, 3])
    a, _ = O.attend(rng.standard_normal((2, 16)), K, z, sel, T, S)
    toks = list(range(8, 16)) + list(range(24, 29))
    np.testing.assert_allclose(a, np.tile(z[toks].mean(0), (2, 1)), atol=1e-12)


# ---------------------------------------------------------- out-projection
def test_dense_value_case_equals_gqa_attention_then_wo():
    """A_V = I, B_V,g = c_g I (r_v = d), every page selected: BasisKV reduces
    to textbook GQA attention (values scaled per KV head) followed by W_O."""
    rng = np.random.default_rng(7)
    Hkv, G, d, H, S, T = 2, 3, 8, 10, 4, 18
    Hq = Hkv * G
    q = rng.standard_normal((Hq, d))
    K = rng.standard_normal((Hkv, 20, d))
    V = O.to_bf16(rng.standard_normal((Hkv, 20, d)))
    cg = np.array([0.5, 2.0])
    A_V = np.stack([np.eye(d)] * Hkv)
    B_V = np.stack([c * np.eye(d) for c in cg])
    W_O = rng.standard_normal((Hq * d, H))
    P_K = rng.standard_normal((Hkv, d, d))
    U_K = np.stack([_orth(rng, d, 3)] * Hkv)
    Z = np.stack([v @ A_V[g] for g, v in enumerate(V)])
    E = rng.standard_normal((Hkv, 20, 3))
    out = O.decode_sequence(q, K, Z, E, T, S, top_k=64, P_K=P_K, U_K=U_K,
                            W_fold=O.fold_outproj(B_V, W_O, Hq))
    o = _sdpa_gqa(q, K[:, :T], cg[:, None, None] * V[:, :T])
    np.testing.assert_allclose(out["y"], o.reshape(-1) @ W_O, atol=1e-10)


def test_fold_matches_unfolded_product():
    rng = np.random.default_rng(8)
    Hkv, G, r_v, d, H = 2, 2, 3, 4, 5
    B_V = rng.standard_normal((Hkv, r_v, d))
    W_O = rng.standard_normal((Hkv * G * d, H))
    a = rng.standard_normal((Hkv * G, r_v))
    y = O.outproj(a, O.fold_outproj(B_V, W_O, Hkv * G))
    want = sum((a[h] @ B_V[h // G]) @ W_O[h * d:(h + 1) * d]
               for h in range(Hkv * G))
    np.testing.assert_allclose(y, want, atol=1e-12)


# -------------------------------------------------- decode-step composition
def test_appended_token_is_routed_and_attended():
    """A new key aligned with a scaled query dominates: the newest page is
    kept and a equals the new token's stored latent."""
    rng = np.random.default_rng(9)
    Hkv, G, d, r_v, r_k, S, T = 1, 2, 16, 4, 4, 8, 31
    A_V = rng.standard_normal((Hkv, d, r_v)) / 4
    P_K = rng.standard_normal((Hkv, r_v, d)) / 2
    U_K = np.stack([_orth(rng, d, r_k)])
    K = rng.standard_normal((Hkv, 40, d))
    Z = rng.standard_normal((Hkv, 40, r_v))
    E = rng.standard_normal((Hkv, 40, r_k))
    u = rng.standard_normal(d)
    k_new = (8 * u / np.linalg.norm(u))[None]
    v_new = rng.standard_normal((Hkv, d))
    q = np.tile(10 * u / np.linalg.norm(u), (G, 1))
    W = O.fold_outproj(rng.standard_normal((Hkv, r_v, d)),
                       rng.standard_normal((G * d, 3)), G)
    out = O.decode_sequence(q, K, Z, E, T, S, 2, P_K, U_K, W, k_new=k_new,
                            v_new=v_new, A_V=A_V)
    assert out["T"] == 32
    assert list(out["sel"][0]) == [0, 3]
    z_stored = O.to_bf16(v_new[0] @ A_V[0])
    np.testing.assert_allclose(out["a"], np.tile(z_stored, (G, 1)), atol=1e-6)


def test_to_bf16_matches_torch_rounding():
    rng = np.random.default_rng(10)
    x = (rng.standard_normal(100000) * 10.0 ** rng.integers(-8, 8, 100000)
         ).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.to_bf16(x), want)


@pytest.mark.parametrize("wl", [synth.TINY, synth.LLAMA8B_T4K],
                         ids=lambda w: w.name)
def test_planted_pages_win_routing(wl):
    """Statistical sanity of the workload + oracle: every page a query was
    planted from is selected."""
    pb = synth.make_problem(wl)
    c = pb.cache
    f = {k: v.double().numpy() for k, v in pb.factors.items()}
    q = pb.q.double().numpy()
    for b in range(wl.B):
        for g in range(wl.Hkv):
            qg = q[b, g * wl.G:(g + 1) * wl.G]
            sc = O.page_scores(qg, c["Z"][b, g].double().numpy(),
                               c["E"][b, g].double().numpy(), f["P_K"][g],
                               f["U_K"][g], wl.T, wl.page_size)
            sel, _ = O.select_pages(sc, wl.top_k)
            want = set(pb.used_pages[b, g * wl.G:(g + 1) * wl.G].reshape(-1).tolist())
            assert want <= set(sel.tolist())


# ---------------------------------------------------------------- FP8 cache
def test_to_e4m3_matches_torch_in_range():
    """Every value of a dense grid over +-448 (ties included) rounds as
    torch's float8_e4m3fn conversion does."""
    rng = np.random.default_rng(12)
    grid = [rng.uniform(-448, 448, 20000), rng.standard_normal(20000),
            rng.standard_normal(5000) * 1e-3]
    # exact halfway points between neighbouring E4M3 values, and the values
    vals = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    vals = np.sort(vals[np.isfinite(vals)])
    grid += [vals, (vals[1:] + vals[:-1]) / 2]
    x = np.concatenate(grid)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(O.to_e4m3(x.astype(np.float32)), ref)


def test_to_e4m3_saturates_and_keeps_steps():
    np.testing.assert_array_equal(O.to_e4m3([500.0, -1e6, 449.0]), [448.0, -448.0, 448.0])
    np.testing.assert_array_equal(O.to_e4m3([2.0 ** -9, 2.0 ** -10, 1.0625, 1.09375]),
                                  [2.0 ** -9, 0.0, 1.0, 1.125])


# ------------------------------------------------- per-layer Value widths
def test_v_rank_schedule_average_and_members():
    from sparse_decode_attention_basiskv_b200 import synth
    for avg in (64, 96):
        w = synth.v_rank_schedule(avg, 32)
        assert len(w) == 32 and sum(w) == 32 * avg
        assert sorted(set(w)) == [avg - 32, avg, avg + 32]
        assert w == synth.v_rank_schedule(avg, 32)  # seeded
    layers = synth.stack_layers(synth.LLAMA8B_T32K_B16, [32, 64, 128])
    assert [L.r_v for L in layers] == [32, 64, 128] and len({L.name for L in layers}) == 3


def test_synthetic_e4m3_caches_hold_e4m3_values():
    """The E4M3 workloads' cache values are E4M3 numbers: the oracle's
    rounding leaves them unchanged (and the filler past the length too)."""
    from sparse_decode_attention_basiskv_b200 import synth
    wl = synth.with_sizes(synth.TINY, T=100, cache_fp8=1)
    pb = synth.make_problem(wl)
    for name in ("K", "Z", "E"):
        x = pb.cache[name].double().numpy()
        np.testing.assert_array_equal(O.to_e4m3(x), x)
    paged = pb.paged()
    assert all(v.dtype == torch.float8_e4m3fn for v in paged.values())


def test_decode_sequence_fp8_stores_and_reads_e4m3_values():
    """The E4M3 branch of the decode step (Table 13's FP8 E4M3 caches): with
    A_V = I the new token's latent is v itself, so the stored z must be
    torch's float8_e4m3fn rounding of v, the stored K torch's rounding of
    k, and a new key that dominates the scores makes a equal that stored
    z; the bf16 branch stores the bf16 roundings instead (the two differ on
    these values, so swapping the branches' roundings fails)."""
    rng = np.random.default_rng(21)
    Hkv, G, d, r_k, S, T = 1, 2, 16, 4, 8, 31
    r_v = d
    A_V = np.eye(d)[None]
    P_K = rng.standard_normal((Hkv, r_v, d)) / 4
    U_K = np.stack([_orth(rng, d, r_k)])
    K = rng.standard_normal((Hkv, 40, d))
    Z = rng.standard_normal((Hkv, 40, r_v))
    E = rng.standard_normal((Hkv, 40, r_k))
    u = rng.standard_normal(d)
    k_new = (8 * u / np.linalg.norm(u))[None] + rng.standard_normal((1, d)) * 1e-2
    v_new = rng.standard_normal((Hkv, d)) * 3
    q = np.tile(10 * u / np.linalg.norm(u), (G, 1))
    W = O.fold_outproj(rng.standard_normal((Hkv, r_v, d)), rng.standard_normal((G * d, 3)), G)

    def torch_round(x, dt):
        return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(dt).double().numpy()

    out8 = O.decode_sequence(q, K, Z, E, T, S, 2, P_K, U_K, W, k_new=k_new, v_new=v_new,
                             A_V=A_V, fp8=True)
    out16 = O.decode_sequence(q, K, Z, E, T, S, 2, P_K, U_K, W, k_new=k_new, v_new=v_new,
                              A_V=A_V)
    z8, k8 = torch_round(v_new[0], torch.float8_e4m3fn), torch_round(k_new[0], torch.float8_e4m3fn)
    z16 = torch_round(v_new[0], torch.bfloat16)
    np.testing.assert_array_equal(out8["Z"][0, T], z8)
    np.testing.assert_array_equal(out8["K"][0, T], k8)
    np.testing.assert_array_equal(out8["E"][0, T],
                                  torch_round(out8["e_new"][0], torch.float8_e4m3fn))
    np.testing.assert_array_equal(out16["Z"][0, T], z16)
    np.testing.assert_array_equal(out16["K"][0, T], k_new[0])
    assert not np.array_equal(z8, z16) and not np.array_equal(k8, k_new[0])
    assert list(out8["sel"][0]) == [0, 3]
    np.testing.assert_allclose(out8["a"], np.tile(z8, (G, 1)), atol=1e-6)
    np.testing.assert_allclose(out16["a"], np.tile(z16, (G, 1)), atol=1e-6)
    # the caches the caller passed are not modified
    assert not np.array_equal(Z[0, T], out8["Z"][0, T])
