"""CPU oracle for the BasisKV decode-attention block — TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this module.  The product path (the C-ABI library and its
Python binding) never calls it, and it shares no code with that path.

It is the plain, slow, obviously correct statement of what the method
computes, in float64 with numpy.  A matrix product from numpy is the only
library primitive; nothing is blocked, fused or reordered.  Every function
works on one (sequence, KV head) group in LOGICAL token order — paging is a
storage detail of the GPU path and does not exist here.

Source: BasisKV, "Value Latents for Communication and Key Routing" (arXiv
2611.02583).  The abstract states the method; Figure 1's caption says the
Value latent is kept in the cache and reused for Key routing with a
Key-specific residual; Table 4 lists the per-token state (compressed Value
of width r_V, residual code of width r_q, exact Key of width d_h) and which
state each phase reads (routing: Value latent + residual; selected
attention: Value latent + exact Key).  The pages print no equations; the
formulas below are the plainest reading of those statements:

  append   z_t = v_t A_V ;  e_t = (k_t - z_t P_K) U_K ;  K_t = k_t
  route    khat_t = z_t P_K + e_t U_K^T ;
           score(page) = max over the page's live tokens and over the query
           heads h of the group of  q_h . khat_t
  select   keep the sink page 0 and the newest page P-1 (more generally
           the first n_sink and the last n_recent pages), then the best
           remaining pages by (score desc, page index asc), k pages in all,
           listed ascending and padded with -1
  attend   s_t = q_h . K_t / sqrt(d) over the selected pages' live tokens;
           p = softmax(s);  a_h = sum_t p_t z_t       (a_h in R^{r_v})
  outproj  y = sum_h a_h W'_h  with  W'_h = B_V,g(h) W_O,h

Precision readings.  Arithmetic is float64.  The cache stores bf16, so the
appended z and e are rounded to bf16 before they are stored (``to_bf16``).
The page choice is an integer decided by floating point: both this oracle
and the GPU take it on float32 scores (the kernel's precision), with -0
mapped to +0 and ties broken by the lower page index.
"""
from __future__ import annotations

import numpy as np


def to_bf16(x) -> np.ndarray:
    """Round to the nearest bfloat16 (ties to even), returned as float64.

    Goes through float32 first; the double rounding differs from a direct
    float64 -> bf16 rounding only on exact float32 half-way cases."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def to_e4m3(x) -> np.ndarray:
    """Round to FP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa
    bits; largest finite 448, subnormal step 2^-9) to nearest even,
    saturating to +-448; returned as float64.  Table 13 of the pages stores
    the caches as FP8 E4M3."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))  # below 2^-6: the subnormal step
    q = 2.0 ** (e - 3)
    r = np.minimum(np.round(a / q) * q, 448.0)  # np.round: half to even
    return np.where(x < 0, -r, r)


# --------------------------------------------------------------------------
# (1) cache append — abstract (the Value is compressed to a latent; a
#     Key-specific residual keeps the part of the Key the latent cannot
#     predict), Table 4 rows.
# --------------------------------------------------------------------------
def append_latents(k: np.ndarray, v: np.ndarray, A_V: np.ndarray,
                   P_K: np.ndarray, U_K: np.ndarray) -> tuple:
    """Value latent and Key residual of new tokens of one KV head.

    k, v : [n][d] new keys / values;  A_V [d][r_v];  P_K [r_v][d];
    U_K [d][r_k].  Returns (z [n][r_v], e [n][r_k]) unrounded; e uses the
    unrounded z.  The cache then stores to_bf16(z), to_bf16(e) and k."""
    z = v @ A_V
    e = (k - z @ P_K) @ U_K
    return z, e


# --------------------------------------------------------------------------
# (2a) routing scores — abstract (the cached Value latent stands in for
#      part of each Key when pages are ranked), Figure 1 caption, Table 4
#      full-context routing column.
# --------------------------------------------------------------------------
def predicted_keys(z: np.ndarray, e: np.ndarray, P_K: np.ndarray,
                   U_K: np.ndarray) -> np.ndarray:
    """khat_t = z_t P_K + e_t U_K^T for every token: [n][d]."""
    return z @ P_K + e @ U_K.T


def page_scores(q_group: np.ndarray, z: np.ndarray, e: np.ndarray,
                P_K: np.ndarray, U_K: np.ndarray, T: int, S: int,
                r_b: int | None = None, r_q: int | None = None) -> np.ndarray:
    """Routing score of every page of one (sequence, KV head) group.

    q_group [G][d] are the group's query heads; z [>=T][r_v], e [>=T][r_k]
    the cached latents in logical order (only t < T is read).  Page p holds
    tokens [p*S, min((p+1)*S, T)).  Returns float64 [P], P = ceil(T/S).

    A narrower router (Table 4: routing reads r_b of the r_V latent
    dimensions and the residual code; Table 9's B16R16 router) reads only
    z[:, :r_b] and e[:, :r_q]: its predicted key is
    z[:, :r_b] P_K[:r_b] + e[:, :r_q] U_K[:, :r_q]^T.  None = full width."""
    r_b = z.shape[1] if r_b is None else r_b
    r_q = e.shape[1] if r_q is None else r_q
    khat = predicted_keys(z[:T, :r_b], e[:T, :r_q], P_K[:r_b], U_K[:, :r_q])
    logits = q_group @ khat.T  # [G][T]
    P = -(-T // S)
    out = np.empty(P)
    for p in range(P):
        out[p] = logits[:, p * S:min((p + 1) * S, T)].max()
    return out


# --------------------------------------------------------------------------
# (2b) page selection — sink + newest always kept; top-k pages (the pages'
#      Table 9 caption uses a routed budget plus a recent window).
# --------------------------------------------------------------------------
def select_pages(scores, top_k: int, n_sink: int = 1, n_recent: int = 1) -> tuple:
    """Choose top_k pages of one group.

    scores: the group's P page scores; they are rounded to float32 here
    because the choice is taken in the kernel's precision.  The first
    n_sink pages and the last n_recent pages are always kept (the default
    keeps the sink page 0 and the newest page; Table 9's budget is a routed
    part plus a recent window); the other top_k - n_sink - n_recent slots go
    to the best remaining pages.  Returns (sel, near_tie): sel is an int32
    array of length top_k, ascending, padded with -1; near_tie is True when
    the last chosen and the first rejected non-forced page have float32
    scores within 1e-4 relative of each other (a slot whose order rounding
    may decide)."""
    s = np.asarray(scores, dtype=np.float32).astype(np.float64)
    s[s == 0.0] = 0.0  # -0 and +0 compare equal and rank by index
    P = len(s)
    sel = np.full(top_k, -1, dtype=np.int32)
    if top_k >= P:
        sel[:P] = np.arange(P)
        return sel, False
    assert n_sink + n_recent <= top_k
    forced = list(range(n_sink)) + list(range(P - n_recent, P))
    need = top_k - len(forced)
    cand = np.arange(n_sink, P - n_recent)
    order = cand[np.lexsort((cand, -s[cand]))]  # score desc, then index asc
    chosen = order[:need]
    near_tie = False
    if len(order) > need and need > 0:
        a, b = s[order[need - 1]], s[order[need]]
        near_tie = bool(abs(a - b) <= 1e-4 * max(abs(a), abs(b)))
    sel[:] = np.sort(np.concatenate([forced, chosen]))
    return sel, near_tie


# --------------------------------------------------------------------------
# (3) exact attention on the selected pages — abstract (exact Keys are read
#     only for the chosen pages), Table 4 selected-attention column (exact
#     Key + Value latent).
# --------------------------------------------------------------------------
def selected_tokens(sel, T: int, S: int) -> np.ndarray:
    toks = [t for p in np.asarray(sel) if p >= 0
            for t in range(p * S, min((p + 1) * S, T))]
    return np.asarray(toks, dtype=np.int64)


def attend(q_group: np.ndarray, K: np.ndarray, z: np.ndarray, sel, T: int,
           S: int) -> tuple:
    """Latent attention output of the group's heads.

    q_group [G][d]; K [>=T][d] exact keys; z [>=T][r_v] Value latents.
    Returns (a [G][r_v], p [G][n]) where p are the softmax weights over the
    selected live tokens (scale 1/sqrt(d))."""
    toks = selected_tokens(sel, T, S)
    d = q_group.shape[1]
    s = (q_group @ K[toks].T) / np.sqrt(d)
    w = np.exp(s - s.max(axis=1, keepdims=True))
    w = w / w.sum(axis=1, keepdims=True)
    return w @ z[toks], w


# --------------------------------------------------------------------------
# (4) latent out-projection — abstract (the Value factor is tied to the
#     output projection), Figure 1 caption (the full output is rebuilt from
#     the latents), Table 1 caption.
# --------------------------------------------------------------------------
def fold_outproj(B_V: np.ndarray, W_O: np.ndarray, Hq: int) -> np.ndarray:
    """W'_h = B_V,g(h) W_O,h for every query head: [Hq][r_v][hidden].

    B_V [Hkv][r_v][d]; W_O [Hq*d][hidden], whose rows h*d..(h+1)*d-1 are
    W_O,h; g(h) = h // (Hq/Hkv)."""
    Hkv, r_v, d = B_V.shape
    G = Hq // Hkv
    return np.stack([B_V[h // G] @ W_O[h * d:(h + 1) * d] for h in range(Hq)])


def outproj(a: np.ndarray, W_fold: np.ndarray) -> np.ndarray:
    """y = sum_h a_h W'_h;  a [Hq][r_v], W_fold [Hq][r_v][hidden] -> [hidden]."""
    y = np.zeros(W_fold.shape[2])
    for h in range(a.shape[0]):
        y += a[h] @ W_fold[h]
    return y


# --------------------------------------------------------------------------
# One decode step of one sequence (all KV heads), composed from the above.
# --------------------------------------------------------------------------
def decode_sequence(q: np.ndarray, K: np.ndarray, Z: np.ndarray, E: np.ndarray,
                    T: int, S: int, top_k: int, P_K: np.ndarray,
                    U_K: np.ndarray, W_fold: np.ndarray,
                    k_new=None, v_new=None, A_V=None, r_b=None, r_q=None,
                    n_sink: int = 1, n_recent: int = 1, fp8: bool = False) -> dict:
    """Decode step for one sequence.

    q [Hq][d]; K [Hkv][cap][d], Z [Hkv][cap][r_v], E [Hkv][cap][r_k] logical
    caches holding T tokens; factors per KV head (A_V [Hkv][d][r_v],
    P_K [Hkv][r_v][d], U_K [Hkv][d][r_k]); W_fold [Hq][r_v][hidden].
    With k_new / v_new ([Hkv][d]) the token is appended first and the step
    attends over T + 1 tokens.  r_b, r_q, n_sink, n_recent: the router's
    widths and the kept pages (page_scores, select_pages).  fp8: the caches
    hold E4M3 values (the appended K, z and e are stored through to_e4m3
    instead of K as given and z, e through to_bf16).  Returns a dict with the
    appended state, the scores, the selection, near-tie flags, a and y, and
    the caches the step read (K, Z, E: with the appended token, if any)."""
    Hkv = K.shape[0]
    Hq = q.shape[0]
    G = Hq // Hkv
    out = {}
    if k_new is not None:
        K, Z, E = K.copy(), Z.copy(), E.copy()
        zs, es = [], []
        for g in range(Hkv):
            z, e = append_latents(k_new[g][None], v_new[g][None], A_V[g],
                                  P_K[g], U_K[g])
            store = to_e4m3 if fp8 else to_bf16
            Z[g, T] = store(z[0])
            E[g, T] = store(e[0])
            K[g, T] = to_e4m3(k_new[g]) if fp8 else k_new[g]
            zs.append(z[0])
            es.append(e[0])
        out["z_new"], out["e_new"] = np.stack(zs), np.stack(es)
        T = T + 1
    scores, sels, ties, a = [], [], [], np.zeros((Hq, Z.shape[2]))
    for g in range(Hkv):
        qg = q[g * G:(g + 1) * G]
        sc = page_scores(qg, Z[g], E[g], P_K[g], U_K[g], T, S, r_b, r_q)
        sel, tie = select_pages(sc, top_k, n_sink, n_recent)
        a[g * G:(g + 1) * G], _ = attend(qg, K[g], Z[g], sel, T, S)
        scores.append(sc)
        sels.append(sel)
        ties.append(tie)
    out.update(T=T, scores=scores, sel=np.stack(sels), near_tie=np.array(ties),
               a=a, y=outproj(a, W_fold), K=K, Z=Z, E=E)
    return out
