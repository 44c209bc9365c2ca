"""fp64 CPU oracle for exact scaled-dot-product attention (test infrastructure).

This module is the *definition* the CUDA kernels are checked against. It is
used only by the tests, by ``__graft_entry__.smoke()`` and by the CPU-baseline
leg of ``bench.py``; the product path never imports it.

Sources (page title, then section):

* "Attention Is O(n²): FlashAttention vs Linear Attention", section
  "Why Attention Is O(n²)": the plain operation ``softmax(Q Kᵀ / sqrt(d)) V``;
  section "Wall-Clock Impact of Tiling": the naive reference that materialises
  the full score matrix.
* "Modern Attention: MQA, GQA, FlashAttention, Sliding Window and RoPE",
  section 3 "FlashAttention: exact, but IO-aware" (running max / running
  denominator, worked example on scores [1, 3]) and section 4
  "Sliding-window attention" (the n = 8, W = 3 mask).
* "Chapter 3: MHA Limitations, MQA, GQA, and FlashAttention", section 3.3
  (query head i reads K/V group i // (H // G)) and section 3.5 (merging two
  partial softmax states by rescaling to the common maximum).

Readings taken where the pages are silent or garbled (all listed in the
design notes):

* ``window_left`` counts the keys strictly before the query's own position,
  so the page's "last W tokens" is ``window_left = W - 1``.
* Causal alignment for ``Nq != Nk`` is bottom-right: query row i sits at key
  position ``qpos(i) = i + Nk - Nq``.
* A window without ``causal`` limits the left side only.
* A row with no allowed key has O = 0 and LSE = -inf.
* LSE is the natural log-sum-exp of the *scaled* scores.
* The merge rule lost from section 3.5 is restated as
  ``m' = max(m_a, m_b)``, ``l' = l_a e^(m_a-m') + l_b e^(m_b-m')``,
  ``acc' = acc_a e^(m_a-m') + acc_b e^(m_b-m')``.

Layouts: Q ``[B, Nq, Hq, d]``, K/V ``[B, Nk, Hkv, d]``, O ``[B, Nq, Hq, d]``,
LSE ``[B, Hq, Nq]``.  Inputs may be any real dtype; they are upcast exactly to
float64 before any arithmetic.
"""

from __future__ import annotations

import math

import numpy as np

NEG_INF = -np.inf


def _f64(x) -> np.ndarray:
    """Exact upcast to float64 (bf16/fp16/fp32 values are all representable)."""
    if hasattr(x, "detach"):  # a torch tensor: go through float32 (exact for bf16)
        x = x.detach().to("cpu").float().numpy()
    return np.asarray(x, dtype=np.float64)


def allowed_mask(Nq: int, Nk: int, causal: bool, window_left: int, rows=None) -> np.ndarray:
    """Boolean ``[Nq, Nk]`` mask of the (query, key) pairs that take part.

    Query row ``i`` sits at key position ``qpos = i + Nk - Nq`` (bottom-right
    alignment). Key ``j`` is allowed when ``j <= qpos`` (if ``causal``) and
    ``j >= qpos - window_left`` (if ``window_left >= 0``). With ``Nq = Nk = 8``,
    ``causal`` and ``window_left = 2`` this is the "last W = 3 tokens" diagram
    of "Modern Attention ...", section 4 "Sliding-window attention".
    ``rows`` (optional) selects query rows: the result is then
    ``[len(rows), Nk]``, the same rows of the full mask.
    """
    i = (np.arange(Nq) if rows is None else np.asarray(rows, dtype=np.int64))[:, None]
    j = np.arange(Nk)[None, :]
    qpos = i + (Nk - Nq)
    ok = np.ones((i.shape[0], Nk), dtype=bool)
    if causal:
        ok &= j <= qpos
    if window_left is not None and window_left >= 0:
        ok &= j >= qpos - window_left
    return ok


def _head_attention(qh, kh, vh, scale, mask):
    """One (batch, query head): materialise S and P, return (O, LSE, P).

    Steps follow the plain definition ("Attention Is O(n²) ...", section
    "Why Attention Is O(n²)"): S = scale * Q Kᵀ; masked entries -> -inf;
    P = softmax over each row (max-subtracted, as in the naive reference of
    section "Wall-Clock Impact of Tiling"); O = P V; LSE = m + ln(sum exp(S - m)).
    """
    S = scale * (qh @ kh.T)                       # [rows, Nk]
    S = np.where(mask, S, NEG_INF)
    m = S.max(axis=1)                             # -inf for a row with no key
    has_key = np.isfinite(m)
    m_safe = np.where(has_key, m, 0.0)
    E = np.exp(S - m_safe[:, None])               # exp(-inf) = 0 for masked keys
    l = E.sum(axis=1)
    P = np.zeros_like(E)
    P[has_key] = E[has_key] / l[has_key, None]
    O = P @ vh
    lse = np.full(m.shape, NEG_INF)
    lse[has_key] = m[has_key] + np.log(l[has_key])
    return O, lse, P


def oracle_attention(q, k, v, causal: bool = False, window_left: int = -1,
                     scale: float | None = None, row_block: int = 512):
    """Exact attention in float64. Returns ``(O [B,Nq,Hq,d], LSE [B,Hq,Nq])``.

    Query head ``hq`` reads K/V head ``hq // (Hq // Hkv)`` ("Chapter 3 ...",
    section 3.3: each K/V group is repeated H // G times). S and P are
    materialised for blocks of ``row_block`` query rows against all ``Nk`` keys.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Hq, d = q.shape
    Bk, Nk, Hkv, dk = k.shape
    assert Bk == B and dk == d and v.shape == k.shape
    assert Hq % Hkv == 0, "query heads must be a multiple of K/V heads"
    group = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    mask = allowed_mask(Nq, Nk, causal, window_left)
    O = np.zeros((B, Nq, Hq, d))
    LSE = np.full((B, Hq, Nq), NEG_INF)
    for b in range(B):
        for hq in range(Hq):
            hk = hq // group
            for r0 in range(0, Nq, row_block):
                r1 = min(r0 + row_block, Nq)
                o, lse, _ = _head_attention(q[b, r0:r1, hq], k[b, :, hk], v[b, :, hk],
                                            scale, mask[r0:r1])
                O[b, r0:r1, hq] = o
                LSE[b, hq, r0:r1] = lse
    return O, LSE


def oracle_attention_rows(q, k, v, b: int, hq: int, rows, causal: bool = False,
                          window_left: int = -1, scale: float | None = None):
    """Selected query rows of one (batch, head): ``(O [len(rows), d], LSE [len(rows)])``.

    Same arithmetic as :func:`oracle_attention`, evaluated only for the listed
    rows so that full-size problems can be checked on sampled outputs.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rows = np.asarray(rows, dtype=np.int64)
    hk = hq // (Hq // Hkv)
    mask = allowed_mask(Nq, Nk, causal, window_left, rows=rows)
    o, lse, _ = _head_attention(q[b, rows, hq], k[b, :, hk], v[b, :, hk], scale, mask)
    return o, lse


def oracle_probabilities(q, k, causal=False, window_left=-1, scale=None, b=0, hq=0):
    """The full probability matrix P ``[Nq, Nk]`` of one (batch, head) (small cases)."""
    q, k = _f64(q), _f64(k)
    _, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    hk = hq // (Hq // Hkv)
    mask = allowed_mask(Nq, Nk, causal, window_left)
    _, _, P = _head_attention(q[b, :, hq], k[b, :, hk], np.zeros((Nk, 1)), scale, mask)
    return P


def oracle_decode(q, k_cache, v_cache, seqlens=None, window_left: int = -1,
                  scale: float | None = None):
    """Single-query decode over a contiguous KV cache.

    ``q [B, Hq, d]``, ``k_cache/v_cache [B, Lmax, Hkv, d]``, ``seqlens [B]``
    (None: all ``Lmax``). The new query's own K/V are already in the cache
    ("Chapter 3 ...", section 3.1: a new token's K/V are appended before it
    attends), so it sits at position ``seqlen - 1`` and sees keys
    ``[max(0, seqlen-1-window_left), seqlen)``. This is exactly the last row of
    causal prefill with ``Nq = 1`` and ``Nk = seqlen``.
    Returns ``(O [B, Hq, d], LSE [B, Hq])``.
    """
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    B, Hq, d = q.shape
    _, Lmax, Hkv, _ = kc.shape
    if seqlens is None:
        seqlens = [Lmax] * B
    seqlens = [int(s) for s in np.asarray(seqlens).reshape(-1)]
    O = np.zeros((B, Hq, d))
    LSE = np.full((B, Hq), NEG_INF)
    for b in range(B):
        L = seqlens[b]
        if L <= 0:
            continue
        o, lse = oracle_attention(q[b:b + 1, None], kc[b:b + 1, :L], vc[b:b + 1, :L],
                                  causal=True, window_left=window_left, scale=scale)
        O[b] = o[0, 0]
        LSE[b] = lse[0, :, 0]
    return O, LSE


def oracle_attention_backward(q, k, v, dout, causal: bool = False, window_left: int = -1,
                              scale: float | None = None):
    """Gradients of the plain definition: ``(dQ [B,Nq,Hq,d], dK, dV [B,Nk,Hkv,d])``.

    The pages state the forward only and note that the saved log-sum-exp is
    what a backward pass reuses ("Chapter 3 ...", section 3.5); the gradients
    here are the exact derivatives of O = P V with P = softmax(scale Q Kᵀ +
    mask), taken step by step:
      dV = Pᵀ dO;  dP = dO Vᵀ;  dS = P * (dP - rowsum(P * dP));
      dQ = scale dS K;  dK = scale dSᵀ Q.
    rowsum(P * dP) equals rowsum(dO * O). With grouped heads a K/V head's
    gradients sum those of its query heads. Rows with no allowed key
    contribute nothing.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    group = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    mask = allowed_mask(Nq, Nk, causal, window_left)
    dQ = np.zeros_like(q)
    dK = np.zeros_like(k)
    dV = np.zeros_like(v)
    for b in range(B):
        for hq in range(Hq):
            hk = hq // group
            _, _, P = _head_attention(q[b, :, hq], k[b, :, hk], v[b, :, hk], scale, mask)
            dO = do[b, :, hq]
            dV[b, :, hk] += P.T @ dO
            dP = dO @ v[b, :, hk].T
            dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
            dQ[b, :, hq] = scale * (dS @ k[b, :, hk])
            dK[b, :, hk] += scale * (dS.T @ q[b, :, hq])
    return dQ, dK, dV


def oracle_attention_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, causal: bool = False,
                            window_left: int = -1, scale: float | None = None):
    """Attention over packed variable-length sequences.

    Sequence ``b`` owns query rows ``[cu_q[b], cu_q[b+1])`` of ``q [total_q,
    Hq, d]`` and keys ``[cu_k[b], cu_k[b+1])`` of ``k, v [total_k, Hkv, d]``
    and attends to its own keys only, with the mask of ``allowed_mask`` taken
    per sequence ("How to Reduce Attention Computation Cost in LLM Training":
    packed sequence boundaries need variable-length kernels). Returns ``(O
    [total_q, Hq, d], LSE [Hq, total_q])``; rows outside every sequence are
    NaN (not computed).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    cq = [int(x) for x in np.asarray(cu_seqlens_q).reshape(-1)]
    ck = [int(x) for x in np.asarray(cu_seqlens_k).reshape(-1)]
    total_q, Hq, d = q.shape
    O = np.full((total_q, Hq, d), np.nan)
    LSE = np.full((Hq, total_q), np.nan)
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        if q1 <= q0:
            continue
        if k1 <= k0:                       # no keys: every row has no allowed key
            O[q0:q1] = 0.0
            LSE[:, q0:q1] = NEG_INF
            continue
        o, lse = oracle_attention(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], causal=causal,
                                  window_left=window_left, scale=scale)
        O[q0:q1] = o[0]
        LSE[:, q0:q1] = lse[0]
    return O, LSE


def paged_to_contiguous(pages, block_table, seqlens=None):
    """Logical per-sequence cache from a paged pool.

    "Inference Engineering", section 2.5 "Optimizing Attention" (the
    PagedAttention paragraph): the cache is split into pages found through a
    lookup table. Logical key ``t`` of sequence ``b`` is row ``t % page_size``
    of page ``block_table[b, t // page_size]``. ``pages [num_pages, page_size,
    Hkv, d]``, ``block_table [B, pages_per_seq]``; keys at or past ``seqlens[b]``
    are left zero and their table entries are not read.
    Returns ``[B, pages_per_seq * page_size, Hkv, d]`` (fp64).
    """
    bt = np.asarray(block_table, dtype=np.int64)
    num_pages, ps, Hkv, d = pages.shape
    B, per_seq = bt.shape
    Lmax = per_seq * ps
    if seqlens is None:
        seqlens = [Lmax] * B
    seqlens = [int(s) for s in np.asarray(seqlens).reshape(-1)]
    out = np.zeros((B, Lmax, Hkv, d))
    for b in range(B):
        for t in range(min(seqlens[b], Lmax)):
            page = int(bt[b, t // ps])
            out[b, t] = _f64(pages[page, t % ps])      # one key row at a time
    return out


def oracle_decode_paged(q, k_pages, v_pages, block_table, seqlens=None, window_left: int = -1,
                        scale: float | None = None):
    """Decode over a paged cache: the plain decode of the logical cache that
    the block table describes (``paged_to_contiguous``). Returns ``(O, LSE)``."""
    kc = paged_to_contiguous(k_pages, block_table, seqlens)
    vc = paged_to_contiguous(v_pages, block_table, seqlens)
    return oracle_decode(q, kc, vc, seqlens, window_left=window_left, scale=scale)


# ---------------------------------------------------------------------------
# Second, independent formulations used only to check the one above.
# ---------------------------------------------------------------------------

def online_softmax(xs):
    """Softmax of a 1-D list in one pass with a running max and denominator.

    "Modern Attention ...", section 3: when a new value raises the maximum, the
    running denominator is rescaled by exp(old_max - new_max). Returns
    ``(probabilities, final_max, denominator)``.
    """
    m, den = -math.inf, 0.0
    for x in xs:
        new_m = max(m, x)
        den = (den * math.exp(m - new_m) if den else 0.0) + math.exp(x - new_m)
        m = new_m
    return [math.exp(x - m) / den for x in xs], m, den


def key_chunk_attention(q, k, v, causal=False, window_left=-1, scale=None, chunk: int = 32):
    """Attention assembled from key chunks, each normalised on its own.

    "Chapter 3 ...", section 3.5: a partial softmax state over one set of keys
    can be merged with the state of another set by rescaling both to their
    common maximum. Here every chunk of ``chunk`` consecutive keys is treated
    as its own small attention problem for all query rows at once, giving a
    normalised output ``O_c`` and its log-sum-exp ``LSE_c`` (a row that sees no
    key of the chunk has ``O_c = 0``, ``LSE_c = -inf``). The chunks are folded
    left to right in that normalised form: the merged log-sum-exp is
    ``log(e^LSE + e^LSE_c)`` and each side's output is weighted by
    ``e^(its LSE - merged LSE)``, which is the section 3.5 rule with the
    denominators carried as logarithms. fp64 throughout; no query blocking.
    Returns ``(O [B,Nq,Hq,d], LSE [B,Hq,Nq])``.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    group = Hq // Hkv
    keep = allowed_mask(Nq, Nk, causal, window_left)
    O = np.zeros((B, Nq, Hq, d))
    LSE = np.full((B, Hq, Nq), NEG_INF)
    for b in range(B):
        for hq in range(Hq):
            kv_head = hq // group
            out = np.zeros((Nq, d))
            lse_run = np.full(Nq, NEG_INF)
            for c0 in range(0, Nk, chunk):
                cols = slice(c0, min(c0 + chunk, Nk))
                logits = np.where(keep[:, cols], scale * (q[b, :, hq] @ k[b, cols, kv_head].T),
                                  NEG_INF)
                seen = keep[:, cols].any(axis=1)
                # the chunk's own log-sum-exp and normalised output
                top = np.where(seen, logits.max(axis=1, initial=NEG_INF), 0.0)
                mass = np.exp(logits - top[:, None]).sum(axis=1)        # >= 1 where seen
                lse_c = np.where(seen, top + np.log(np.where(seen, mass, 1.0)), NEG_INF)
                w_c = np.exp(logits - np.where(seen, lse_c, 0.0)[:, None])   # rows sum to 1
                out_c = w_c @ v[b, cols, kv_head]
                # fold: merged log-sum-exp, then both sides reweighted to it
                both = np.logaddexp(lse_run, lse_c)
                live = np.isfinite(both)
                ref = np.where(live, both, 0.0)
                wa = np.where(np.isfinite(lse_run), np.exp(lse_run - ref), 0.0)
                wb = np.where(np.isfinite(lse_c), np.exp(lse_c - ref), 0.0)
                out = np.where(live[:, None], wa[:, None] * out + wb[:, None] * out_c, 0.0)
                lse_run = both
            O[b, :, hq] = out
            LSE[b, hq] = lse_run
    return O, LSE


def merge_partials(parts):
    """Merge partial softmax states ``[(m, l, acc), ...]`` of disjoint key sets.

    "Chapter 3 ...", section 3.5: the denominators (and the unnormalised
    weighted-V accumulators) are rescaled to the common maximum before adding.
    Returns ``(O, LSE)`` with ``O = acc / l`` and ``LSE = m + ln l`` (O = 0 and
    LSE = -inf when no part saw a key).
    """
    ms = np.array([p[0] for p in parts], dtype=np.float64)
    M = ms.max()
    if not np.isfinite(M):
        d = np.asarray(parts[0][2]).shape
        return np.zeros(d), -np.inf
    L = 0.0
    acc = 0.0
    for m, l, a in parts:
        if np.isfinite(m):
            w = math.exp(m - M)
            L = L + l * w
            acc = acc + np.asarray(a, dtype=np.float64) * w
    return acc / L, M + math.log(L)


def brute_force_attention(q, k, v, causal=False, window_left=-1, scale=None):
    """Pure-Python loops (no NumPy arithmetic) for tiny shapes.

    Nested lists in, nested lists out: ``O[b][i][h][c]`` and ``LSE[b][h][i]``.
    Used to check the NumPy oracle on shapes up to about 8 x 8.
    """
    B, Nq, Hq, d = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Nk, Hkv = len(k[0]), len(k[0][0])
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    group = Hq // Hkv
    O = [[[[0.0] * d for _ in range(Hq)] for _ in range(Nq)] for _ in range(B)]
    LSE = [[[-math.inf] * Nq for _ in range(Hq)] for _ in range(B)]
    for b in range(B):
        for h in range(Hq):
            g = h // group
            for i in range(Nq):
                qpos = i + Nk - Nq
                scores = []
                for j in range(Nk):
                    ok = True
                    if causal and j > qpos:
                        ok = False
                    if window_left >= 0 and j < qpos - window_left:
                        ok = False
                    if ok:
                        s = 0.0
                        for c in range(d):
                            s += float(q[b][i][h][c]) * float(k[b][j][g][c])
                        scores.append((j, s * scale))
                if not scores:
                    continue
                mx = max(s for _, s in scores)
                w = [(j, math.exp(s - mx)) for j, s in scores]
                den = sum(x for _, x in w)
                for c in range(d):
                    O[b][i][h][c] = sum(x * float(v[b][j][g][c]) for j, x in w) / den
                LSE[b][h][i] = mx + math.log(den)
    return O, LSE
