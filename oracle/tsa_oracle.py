"""Plain, slow, fp64 CPU oracle for the prefill attention of Token Sparse Attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import or call it.  It shares no code, table or
helper with the CUDA library under ``long_context_tsa_b200/``; it never
imports that package, and that package never imports this one.

What it computes (each function cites the passage it follows):

* ``score``   -- per-key importance: softmax of the scaled query-key logits
  over the keys, summed over the queries.  Source: "Token Sparse Attention
  Long Context" (skillsdirectory skill page), Step 1, ``TokenScorer.score_tokens``
  with method "entropy".  Readings the page leaves open (stated in the
  design notes): only the last ``window`` queries score (an observation
  window), window query at position p sees keys j <= p (causal), and under
  grouped-query attention the scores of the query heads that share a KV head
  are summed.
* ``select``  -- top-K per KV head.  Source: same page, Step 1,
  ``TokenScorer.select_top_k`` (``torch.topk``) and Step 3 (K clamped to the
  sequence length).  Reading: ties go to the lower index; the kept indices
  are listed ascending, followed by the dropped indices ascending.
* ``coverage_budgets`` -- per-KV-head budget from a token coverage tau:
  the smallest K whose top-K score mass reaches (1 - tau) of the head's total
  mass.  Source: "Token Sparse Attention: Efficient Long-Context Inference
  with Interleaved Token Selection" (sciencestack), the summary's dynamic
  token coverage and Figures 1 and 5 (sparsity set by a coverage tau); the
  skill page's Architecture Overview ("Selection Threshold" deciding K per
  head).  Reading (the pages give no formula): the mass of a token is its
  score, made exact by fixed point -- floor(clamp(s, 0, 256) * 2^S) as an
  integer, S = 55 - ceil(log2 L) so that a head's total stays below 2^63 --
  and the dropped mass may be at most floor(double(M) * tau) of the total M.
* ``attend_block_sparse`` -- ``attend`` restricted further by a mask over
  128 x 128 blocks of the compressed (query, key) space.  Source: the
  sciencestack page, Figures 1 and 5b (Token Sparse Attention composed with a
  block-sparse attention kernel inside the compressed token set).
* ``out_proj_residual`` -- the output projection of the attention output,
  added to the residual.  Source: the skill page, Step 3
  (``SparseAttentionHead.forward``: ``out_proj`` on the attention output of
  the selected tokens, then ``scatter_attention_output`` back to full length);
  the sciencestack page, Figure 3 (outputs scattered back into the full
  sequence layout before the residual connection is added).  Reading: the
  projection is a bias-free linear map of the heads' outputs concatenated per
  position (the multi-head form of the page's single-head ``out_proj``); a row
  dropped by a head's group contributes zero, so projecting the compressed rows
  and scattering them equals projecting the scattered rows; the residual is
  added to every row, as in Figure 3.
* ``drift``   -- representation drift between two hidden-state tensors:
  one minus the mean, over all (batch, position) rows, of the cosine of the
  two rows after each is divided by max(its L2 norm, eps).  Source: the skill
  page, Step 4, ``LayerStabilityAnalyzer.compute_representation_drift``
  (``torch.nn.functional.normalize`` then a dot product per row);
  ``layer_stable`` is the same class's ``is_layer_stable`` window rule.
* ``attend``  -- gather the kept rows of Q, K, V, run softmax attention on the
  compressed tensors with a causal mask by original positions, and scatter the
  result back to full length with zeros at dropped rows.  Source: same page,
  Step 2 (``gather_tokens``, ``scatter_attention_output``) and Step 3
  (``SparseAttentionHead.forward``); "Token Sparse Attention: Efficient
  Long-Context Inference with Interleaved Token Selection" (sciencestack),
  Figure 3 (compress Q/K/V per head, attend, scatter to the full sequence
  layout before the residual add).

All arithmetic is float64 on values widened exactly from the caller's inputs
(each function widens only the slices it reads, to bound memory at long L).
Library primitives (``numpy.matmul``, ``numpy.argsort``) serve as single steps;
there is no blocking or reordering beyond splitting rows into chunks to bound
memory, which does not change any row's arithmetic.

Pins: every function here is checked in ``tests/test_oracle_pins.py`` against
closed forms, invariants, brute force on tiny inputs and PyTorch's own
scaled-dot-product attention.  The pages print no worked numeric example, so
no end-to-end value is pinned by the pages themselves.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "clamp_budgets",
    "score",
    "select",
    "coverage_shift",
    "token_mass",
    "coverage_budgets",
    "attend",
    "attend_rows",
    "attend_accumulate",
    "attend_block_sparse",
    "BLOCK",
    "out_proj_residual",
    "forward",
    "row_cosine",
    "drift",
    "layer_stable",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _scale(d: int, scale) -> float:
    # Step 1 and Step 3 of the skill page divide the logits by the square root
    # of the per-head dimension.
    if scale is None or scale == 0.0:
        return 1.0 / math.sqrt(d)
    return float(scale)


def clamp_budgets(budgets, L: int) -> np.ndarray:
    """Kept-token count per (batch, KV head): ``min(budget, L)``.

    The skill page's Step 3 passes ``k=min(self.k, seq_len)`` to the top-K.
    A budget below 1 has no meaning on the pages and is rejected.
    """
    b = np.asarray(budgets, dtype=np.int64).reshape(-1)
    if np.any(b < 1):
        raise ValueError("every budget must be >= 1")
    return np.minimum(b, L)


def score(q, k, window: int, scale=None) -> np.ndarray:
    """Per-KV-head token importance, shape [B, Hkv, L], float64.

    For query head h (KV group g = h // G, G = Hq // Hkv) and each window query
    at position p in [L - window, L):
        logits_j = scale * q[p] . k[j]           for keys j <= p
        prob_j   = softmax over those keys
    and score_g[j] accumulates prob_j over the window queries of every query
    head in group g.  Follows Step 1 ("entropy": matmul, divide by sqrt(d),
    softmax over keys, sum over queries) with the window / causal / grouping
    readings listed in the module docstring.
    """
    B, Hq, L, D = np.shape(q)
    Hkv = np.shape(k)[1]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    if not 1 <= window <= L:
        raise ValueError("window must be in [1, L]")
    G = Hq // Hkv
    s = _scale(D, scale)
    pos_q = np.arange(L - window, L)
    visible = np.arange(L)[None, :] <= pos_q[:, None]  # [window, L]
    out = np.zeros((B, Hkv, L), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            logits = s * (_f64(q[b, h, L - window:, :]) @ _f64(k[b, g]).T)  # [window, L]
            logits = np.where(visible, logits, -np.inf)
            m = logits.max(axis=1, keepdims=True)
            e = np.exp(logits - m)
            p = e / e.sum(axis=1, keepdims=True)
            out[b, g] += p.sum(axis=0)
    return out


def select(scores, budgets) -> np.ndarray:
    """Per-KV-head permutation of [0, L): kept indices ascending, then dropped ascending.

    ``scores`` is [B, Hkv, L]; values are compared exactly in the dtype given
    (pass float32 scores to reproduce a float32 decision).  The K = min(budget, L)
    largest are kept; among equal values the lower index wins (a stable sort
    on descending value).  Follows ``select_top_k`` (Step 1) with the tie and
    ordering reading stated in the module docstring.  +0.0 and -0.0 compare
    equal, as they do in IEEE arithmetic.
    """
    s = np.asarray(scores)
    if s.ndim != 3:
        raise ValueError("scores must be [B, Hkv, L]")
    if not np.all(np.isfinite(s)):
        raise ValueError("scores must be finite")
    B, Hkv, L = s.shape
    kept = clamp_budgets(budgets, L)
    if kept.size != B * Hkv:
        raise ValueError("one budget per (batch, KV head)")
    perm = np.empty((B, Hkv, L), dtype=np.int64)
    for b in range(B):
        for g in range(Hkv):
            K = int(kept[b * Hkv + g])
            order = np.argsort(-s[b, g], kind="stable")
            perm[b, g, :K] = np.sort(order[:K])
            perm[b, g, K:] = np.sort(order[K:])
    return perm


def coverage_shift(L: int) -> int:
    """Fixed-point shift S of the token masses for sequence length L (L * 256 * 2^S <= 2^63)."""
    return 55 - max(0, math.ceil(math.log2(L)))


def token_mass(scores, L: int) -> np.ndarray:
    """Integer mass floor(clamp(s, 0, 256) * 2^S) of float32 scores, as uint64 (exact).

    NaN counts as 0 (``fmax``); the coverage reading in the module docstring.
    """
    s = np.fmin(np.fmax(np.asarray(scores, dtype=np.float32).astype(np.float64), 0.0), 256.0)
    return np.floor(s * 2.0 ** coverage_shift(L)).astype(np.uint64)


def coverage_budgets(scores, tau: float) -> np.ndarray:
    """Per (b, g) budget K: the fewest top tokens whose mass reaches the coverage target.

    ``scores`` is float32 [B, Hkv, L].  Per head: M = sum of the integer masses,
    D = floor(double(M) * tau) (the mass that may be dropped), target
    T = M - D; K is the smallest k >= 1 such that the k tokens ranked first by
    ``select``'s order (descending score, lower index first on ties) carry
    mass >= T.  With T <= 0 (tau = 1, or no mass at all) K = 1.  Returns int64
    [B * Hkv], ordered like the budgets the other functions take.
    """
    s = np.asarray(scores, dtype=np.float32)
    if s.ndim != 3:
        raise ValueError("scores must be [B, Hkv, L]")
    if not np.all(np.isfinite(s)):
        raise ValueError("scores must be finite")
    if not (0.0 <= tau <= 1.0):
        raise ValueError("tau must lie in [0, 1]")
    B, Hkv, L = s.shape
    out = np.empty(B * Hkv, dtype=np.int64)
    for b in range(B):
        for g in range(Hkv):
            m = token_mass(s[b, g], L)
            M = int(m.sum(dtype=np.uint64))
            D = math.floor(float(M) * tau)
            T = M - D
            if T <= 0:
                out[b * Hkv + g] = 1
                continue
            order = np.argsort(-s[b, g].astype(np.float64), kind="stable")
            prefix = np.cumsum(m[order], dtype=np.uint64)
            out[b * Hkv + g] = int(np.searchsorted(prefix, np.uint64(T), side="left")) + 1
    return out


def attend_rows(q, k, v, perm_bg, K: int, b: int, h: int, G: int, rows, scale=None,
                block_mask_bg=None) -> np.ndarray:
    """Output rows for query head h of batch b at compacted indices ``rows``.

    Compacted row i stands for original position p_i = perm_bg[i] (i < K).
    Its output is  sum_r softmax_r(scale * q[p_i] . k[p_r]) * v[p_r]  over the
    kept rows r whose original position p_r <= p_i (causal by original
    positions).  Returns [len(rows), D] float64.  This is Step 3's
    matmul / softmax / matmul on the gathered tensors of Step 2.

    ``block_mask_bg`` (optional, [nb, nb] of bool, nb >= ceil(K / BLOCK)) adds
    the block-sparse composition: key r is visible to row i only when
    block_mask_bg[i // BLOCK, r // BLOCK] is set as well.  A row that sees no
    key at all outputs zeros.
    """
    D = np.shape(q)[-1]
    s = _scale(D, scale)
    g = h // G
    idx = np.asarray(perm_bg[:K], dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    kh = _f64(k[b, g][idx])  # [K, D]  gathered keys
    vh = _f64(v[b, g][idx])  # [K, D]  gathered values
    out = np.empty((rows.size, D), dtype=np.float64)
    chunk = max(1, (1 << 22) // max(1, K))
    for c0 in range(0, rows.size, chunk):
        rr = rows[c0:c0 + chunk]
        pq = idx[rr]  # original positions of these queries
        qh = _f64(q[b, h][pq])  # [n, D]  gathered queries
        logits = s * (qh @ kh.T)  # [n, K]
        visible = idx[None, :] <= pq[:, None]
        if block_mask_bg is not None:
            bm = np.asarray(block_mask_bg, dtype=bool)
            visible = visible & bm[(rr // BLOCK)[:, None], (np.arange(K) // BLOCK)[None, :]]
        logits = np.where(visible, logits, -np.inf)
        m = logits.max(axis=1, keepdims=True)
        empty = ~np.isfinite(m[:, 0])
        m = np.where(np.isfinite(m), m, 0.0)
        e = np.exp(logits - m)
        den = e.sum(axis=1, keepdims=True)
        p = e / np.where(empty[:, None], 1.0, den)
        out[c0:c0 + chunk] = p @ vh
    return out


# Block size (in compacted positions and keys) of the block-sparse composition.
BLOCK = 128


def attend_block_sparse(q, k, v, perm, budgets, block_mask, scale=None) -> np.ndarray:
    """``attend`` composed with a block mask over the compressed space.

    ``block_mask`` is [B, Hkv, nb, nb] (nb = ceil(L / BLOCK)), nonzero where
    the block of compacted query rows [BLOCK * i, BLOCK * i + BLOCK) may attend
    to the block of compacted keys [BLOCK * j, ...); the causal mask still
    applies inside.  Source: "Token Sparse Attention: Efficient Long-Context
    Inference with Interleaved Token Selection" (sciencestack), Figures 1 and
    5b (the method applied on top of a block-sparse attention kernel inside
    the compressed token set).  Reading: the mask is given per KV group in
    compacted coordinates; rows that see no key output zeros; dropped rows are
    zeros as in ``attend``.
    """
    B, Hq, L, D = np.shape(q)
    Hkv = np.shape(k)[1]
    G = Hq // Hkv
    kept = clamp_budgets(budgets, L)
    perm = np.asarray(perm, dtype=np.int64)
    bm = np.asarray(block_mask) != 0
    out = np.zeros((B, Hq, L, D), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            K = int(kept[b * Hkv + g])
            out[b, h, perm[b, g, :K]] = attend_rows(q, k, v, perm[b, g], K, b, h, G, np.arange(K), scale,
                                                    block_mask_bg=bm[b, g])
    return out


def attend(q, k, v, perm, budgets, scale=None) -> np.ndarray:
    """Full output [B, Hq, L, D] float64: attention on the kept rows, zeros elsewhere.

    Query head h uses the permutation and budget of its KV group h // G.
    The attention output of kept row i is scattered to original position
    perm[b, g, i]; every dropped position holds 0 (Step 2's
    ``scatter_attention_output`` starts from a zero tensor).
    """
    B, Hq, L, D = np.shape(q)
    Hkv = np.shape(k)[1]
    G = Hq // Hkv
    kept = clamp_budgets(budgets, L)
    perm = np.asarray(perm, dtype=np.int64)
    out = np.zeros((B, Hq, L, D), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            K = int(kept[b * Hkv + g])
            rows = np.arange(K)
            out[b, h, perm[b, g, :K]] = attend_rows(q, k, v, perm[b, g], K, b, h, G, rows, scale)
    return out


def attend_accumulate(base, q, k, v, perm, budgets, scale=None) -> np.ndarray:
    """``base`` [B, Hq, L, D] plus the attention output at the kept rows; dropped rows unchanged.

    The skill page's Step 2 ``scatter_add_attention_output`` adds the compressed
    attention output into an existing full-length tensor at the selected
    indices (``full_output[batch, indices] += attention_output``) instead of
    scattering into zeros.
    """
    out = _f64(base).copy()
    B, Hq, L, D = out.shape
    Hkv = np.shape(k)[1]
    G = Hq // Hkv
    kept = clamp_budgets(budgets, L)
    perm = np.asarray(perm, dtype=np.int64)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            K = int(kept[b * Hkv + g])
            out[b, h, perm[b, g, :K]] += attend_rows(q, k, v, perm[b, g], K, b, h, G, np.arange(K), scale)
    return out


def out_proj_residual(x, attn_out, w_o, b: int = 0, rows=None) -> np.ndarray:
    """Residual plus the output projection of the full-length attention output.

    x [B, L, N] is the residual stream, attn_out [B, Hq, L, D] the attention
    output as ``attend`` writes it (zeros at every row a head's KV group
    dropped), w_o [N, Hq * D] the projection weight in the layout of an
    ``nn.Linear`` weight (out_features x in_features), no bias.  For batch
    entry ``b`` and positions ``rows`` (default: all) returns, as float64
    [len(rows), N],
        x[b, p, :] + concat_h(attn_out[b, h, p, :]) @ w_o.T
    -- the skill page's Step 3 ``out_proj`` followed by the scatter back to
    full length, and Figure 3's residual add after the scatter.
    """
    B, Hq, L, D = np.shape(attn_out)
    rows = np.arange(L) if rows is None else np.asarray(rows, dtype=np.int64)
    o = np.transpose(_f64(np.asarray(attn_out)[b][:, rows, :]), (1, 0, 2)).reshape(rows.size, Hq * D)
    return _f64(np.asarray(x)[b][rows]) + o @ _f64(w_o).T


def forward(q, k, v, window: int, budgets, scale=None):
    """Score -> select (on float32-rounded scores) -> attend.  Returns (scores64, perm, out).

    The selection runs on the scores rounded to float32, the precision in
    which the library stores and compares them.
    """
    sc = score(q, k, window, scale)
    perm = select(sc.astype(np.float32), budgets)
    out = attend(q, k, v, perm, budgets, scale)
    return sc, perm, out


# Default of torch.nn.functional.normalize, which the skill page's drift uses.
NORMALIZE_EPS = 1e-12


def row_cosine(h_before, h_after, eps: float = NORMALIZE_EPS) -> np.ndarray:
    """Per-row similarity of [..., hidden] tensors: <a / max(|a|, eps), b / max(|b|, eps)>.

    The skill page, Step 4, ``compute_representation_drift``: both hidden
    states are L2-normalised along the hidden dimension (norm clamped below at
    eps, as ``torch.nn.functional.normalize`` does) and multiplied elementwise,
    then summed over the hidden dimension.
    """
    a = _f64(h_before)
    b = _f64(h_after)
    na = np.maximum(np.sqrt(np.sum(a * a, axis=-1)), eps)
    nb = np.maximum(np.sqrt(np.sum(b * b, axis=-1)), eps)
    return np.sum((a / na[..., None]) * (b / nb[..., None]), axis=-1)


def drift(h_before, h_after, eps: float = NORMALIZE_EPS) -> float:
    """1 - mean of ``row_cosine`` over every (batch, position) row (skill page, Step 4)."""
    return float(1.0 - np.mean(row_cosine(h_before, h_after, eps)))


def layer_stable(history, window: int = 3, threshold: float = 0.1) -> bool:
    """Stability rule of the skill page, Step 4, ``is_layer_stable``.

    ``history`` is the list of drifts so far, the newest last.  With fewer than
    ``window`` entries the layer is not stable; otherwise it is stable when the
    mean of the newest ``window`` drifts is strictly below ``threshold``.
    """
    if len(history) < window:
        return False
    recent = [float(x) for x in history[-window:]]
    return sum(recent) / len(recent) < threshold
