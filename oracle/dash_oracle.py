"""Plain fp64 CPU restatement of the DashAttention forward path (test oracle).

TEST INFRASTRUCTURE ONLY: imported by the test suite, ``smoke()`` and the
CPU-baseline leg of ``bench.py``; never by the product path.

Sources (page titles and sections of the pages on "DashAttention:
Differentiable and Adaptive Sparse Hierarchical Attention"):

* Stage 0, chunk summary -- gist.science technical summary, "Fase 0: Lokale
  Chunk Samenvatting" / "阶段0：局部块摘要": the context is cut into contiguous
  chunks of B keys; a learned query q_bar attends to the keys of each chunk
  with local scaled dot-product attention; q_bar = 0 gives uniform mean
  pooling; a finished chunk's summary is fixed and cached.
* Stage 1, routing -- "Fase 1: Entmax Chunk Routering" / "阶段1": per query,
  logits z_bar against the chunk summaries, w_hat = alpha-entmax(gamma z_bar);
  the support is set by a threshold that depends on the scores (aiexpert.news
  article, method paragraph); under GQA the probabilities of the query heads
  that share a KV head are averaged into one shared support.
* Stage 2, prior-induced sparse softmax -- "Fase 2" / "阶段2": softmax is the
  maximiser of z^T p - KL(p || u); the reference u is replaced by a prior g
  built from the routing weights w with g = 0 wherever w = 0; chunks near the
  diagonal get a separate branch; sigma sets the prior's strength between
  the routing scores and a uniform baseline; the kernel iterates over active
  chunks of a bit-packed mask and adds the routing bias to the logits before
  the softmax.
* alpha-entmax itself is named but not printed by the pages; it is the
  published transformation alpha-entmax(z)_c = [(alpha-1) z_c - tau]_+^(1/(alpha-1))
  with tau chosen so that the output sums to one (Peters, Niculae & Martins,
  "Sparse Sequence-to-Sequence Models", 2019).

Readings where the pages are silent (each is listed in the design notes):

* Stage 0 scale is 1/sqrt(d) (standard SDPA); the value side of the local
  attention is the keys themselves, so the summary lives in key space, which
  is what stage 1 takes logits against.  q_bar is one vector per KV head.
* z_bar_c = q . Kbar_c (raw dot product); gamma carries any scaling.
* Eligible chunks for the query at position i are the complete chunks
  strictly before its own chunk c_i = floor(i / B); if there are none the
  routing row is empty (w = 0, mask = 0).
* Stage 2 bias for key j of block b(j): 0 on the query's own chunk (the
  always-on diagonal branch, causal j <= i); sigma * ln(w_{i,b(j)}) on a routed
  active block (0 when sigma == 0, i.e. g = w**0 = 1); -inf elsewhere.  So
  p_ij is proportional to g_ij * exp(q_i . k_j / sqrt(d)) with g = w_b**sigma,
  the Gibbs maximiser of z^T p - KL(p || g).  Mask bits at or after c_i are
  ignored.
* Decode: the new query is position L-1 of an L-token cache that already
  holds its own key/value; it equals row L-1 of prefill on the same data.
* estimate_diagonal (aiexpert.news article, interface paragraph: a flag for
  a diagonal correction of the alpha-entmax normalisation; gist.science
  summary, Fase 2 "Diagonaal Afhandeling": chunks near the diagonal may have
  no summary): the query's own chunk, whose summary does not exist yet, is
  given an estimated one -- stage 0's learned-query summary over the keys
  the query may see (its chunk's start .. i) -- and joins the entmax as one
  more candidate, so the routed chunks share 1 - w_diag of the mass.  The
  diagonal branch of stage 2 stays on with weight 1 whatever w_diag is;
  w_diag is reported in column c_i of w and never sets a mask bit.
* Top-k routing (the fixed-budget baseline the pages contrast with, NSA and
  InfLLMv2): the coarse score of a chunk is the group mean of the per-head
  softmax of gamma z_bar over the eligible chunks; the k best chunks (equal
  scores: lower index first) are selected, with uniform weights.

What pins each function (``tests/test_oracle.py``):

* ``entmax_bisect``: brute-force support enumeration on n <= 10; alpha = 2
  equals textbook sparsemax; alpha -> 1 approaches softmax; sums to one;
  p > 0 exactly where (alpha-1) z > tau; shift invariance; closed forms for
  two inputs.  ``entmax15_sort`` is pinned the same way and against
  ``entmax_bisect``.
* ``chunk_summary``: q_bar = 0 gives the chunk mean; a large q_bar aligned
  with one key returns that key; summaries lie in the convex hull of the
  chunk's keys; invariant to permuting keys inside a chunk.
* ``route``: G = 1 equals one brute-force entmax per row on hand-computed
  logits; w sums to one on rows with eligible chunks; mask = OR of the
  per-head supports; empty for the first chunk.  With the diagonal
  candidate: a hand-computed sparsemax case (two candidates, B = 2, the
  estimate written out key by key); at the last row of a chunk the estimate
  is the chunk's complete summary, so the weights equal plain routing of the
  same query one position later; the routed chunks and the diagonal sum to
  one; rows of the first chunk give the diagonal weight 1; the mask never
  holds the query's own chunk.
* ``diagonal_summary``: ``chunk_summary`` of the partial chunk (pinned
  through the chunk-end case above and the hand-computed case).
* ``attn_fwd``: all chunks active with sigma = 0 equals dense causal softmax
  attention (torch's fp64 scaled_dot_product_attention); one-hot values
  expose p, which is checked against the variational optimality condition
  of z^T p - KL(p || g); a single active block reduces to a local softmax.
* ``decode``: equals the last row of prefill on the same data (with and
  without the diagonal candidate).
* ``decode_varlen``: each sequence equals the last row of prefill on its own
  prefix; equal lengths reduce to ``decode``; nothing past a sequence's
  length (cache rows, summary rows) changes its result.
* ``route_topk``: with one head per group the selection is the k largest
  logits (softmax is monotone) found by a full sort; k at or above the number
  of eligible chunks selects them all; scores sum to one over the eligible
  chunks; equal scores go to the lower chunk index.
* ``summarize_append``: appending at every chunk boundary of a growing
  cache rebuilds ``chunk_summary`` of the whole cache; rows of sequences not
  at a boundary are left as they were; the paged form equals the contiguous
  one through an identity table.
* ``pack_weights`` / ``unpack_weights`` (the compact routing form): on
  ``route``'s output the round trip returns the dense w and the mask; counts
  are the popcounts of the mask rows; indices ascend and are the set bits;
  each listed weight is the dense w at that chunk (checked element by
  element against a direct scan of the dense rows).
* ``decode_attend`` (stage 2 of a decode step on given routing): with every
  chunk active and w = 1 it is torch's SDPA of each query against its first
  L keys; on ``decode``'s own routing it returns ``decode``'s output; with one
  routed chunk it is a softmax over that chunk (bias sigma ln w) and the
  query's own causal chunk.
* ``decode_paged``: an identity page table over a pool that is the caches
  cut into pages gives ``decode_varlen``; permuting the pool's pages together
  with the table, and rewriting pages no table entry of a sequence's own
  chunks names, change nothing.
"""

import math

import numpy as np


def _f64(a):
    """Any array-like (numpy array, torch tensor incl. bf16) -> fp64 ndarray."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu")
        if hasattr(a, "double"):
            a = a.double()
        a = a.numpy()
    return np.asarray(a, dtype=np.float64)


def _take(a, bi, h0, h1, idx):
    """a[bi, h0:h1][:, idx] for a numpy array or torch tensor, as fp64 (only that slice)."""
    if hasattr(a, "detach"):
        import torch
        return _f64(a[bi, h0:h1][:, torch.as_tensor(np.asarray(idx), dtype=torch.long)])
    return _f64(np.asarray(a)[bi, h0:h1][:, idx])


def _ipow(base, e):
    """base ** e for base >= 0, using exact squaring for the alpha=1.5 case."""
    if e == 2.0:
        return base * base
    if e == 1.0:
        return base
    return np.power(base, e)


# ----------------------------------------------------------------------------
# alpha-entmax
# ----------------------------------------------------------------------------

def entmax_threshold(z, alpha, max_iter=200):
    """tau of alpha-entmax along the last axis, by bisection (fp64).

    Solves sum_c max((alpha-1) z_c - tau, 0) ** (1/(alpha-1)) = 1.  Entries of
    z equal to -inf are not eligible.  Rows without an eligible entry get
    tau = +inf (empty support).  The bracket [max x - 1, max x - n**(1-alpha)]
    holds the root: at the left end the largest entry alone contributes 1, at
    the right end each of the n entries contributes at most 1/n.
    """
    if not alpha > 1.0:
        raise ValueError("alpha must be > 1")
    x = (alpha - 1.0) * _f64(z)
    e = 1.0 / (alpha - 1.0)
    n = np.isfinite(x).sum(axis=-1, keepdims=True).astype(np.float64)
    empty = n == 0
    m = np.where(empty, 0.0, np.max(np.where(np.isfinite(x), x, -np.inf), axis=-1, keepdims=True))
    xs = np.where(np.isfinite(x), x, -np.inf)
    lo = m - 1.0
    hi = m - np.power(np.maximum(n, 1.0), 1.0 - alpha)
    for _ in range(max_iter):
        mid = 0.5 * (lo + hi)
        f = np.sum(_ipow(np.maximum(xs - mid, 0.0), e), axis=-1, keepdims=True) - 1.0
        new_lo = np.where(f >= 0.0, mid, lo)
        new_hi = np.where(f >= 0.0, hi, mid)
        if np.array_equal(new_lo, lo) and np.array_equal(new_hi, hi):
            break
        lo, hi = new_lo, new_hi
    tau = 0.5 * (lo + hi)
    return np.where(empty, np.inf, tau)[..., 0]


def entmax_bisect(z, alpha):
    """alpha-entmax of z along the last axis (fp64), via the bisection threshold."""
    x = (alpha - 1.0) * _f64(z)
    tau = entmax_threshold(z, alpha)
    xs = np.where(np.isfinite(x), x, -np.inf)
    return _ipow(np.maximum(xs - tau[..., None], 0.0), 1.0 / (alpha - 1.0))


def entmax15_sort(z):
    """Exact 1.5-entmax of a 1-D vector by sorting (fp64).

    With x = z / 2 sorted in decreasing order, a support made of the k largest
    entries gives the threshold tau_k = mean_k - sqrt((1 - k var_k) / k), the
    smaller root of sum_{c<=k} (x_c - tau)^2 = 1.  The support is the largest
    k whose tau_k lies strictly below its k-th entry.
    """
    x = 0.5 * _f64(z).reshape(-1)
    x = x[np.isfinite(x)] if not np.all(np.isfinite(x)) else x
    xs = np.sort(x)[::-1]
    k = np.arange(1, xs.size + 1, dtype=np.float64)
    mean = np.cumsum(xs) / k
    meansq = np.cumsum(xs * xs) / k
    delta = (1.0 - k * (meansq - mean * mean)) / k
    tau_k = mean - np.sqrt(np.maximum(delta, 0.0))
    ok = (delta >= 0.0) & (tau_k < xs)
    kstar = int(np.max(np.nonzero(ok)[0])) + 1
    tau = tau_k[kstar - 1]
    xfull = 0.5 * _f64(z).reshape(-1)
    xfull = np.where(np.isfinite(xfull), xfull, -np.inf)
    return np.square(np.maximum(xfull - tau, 0.0)).reshape(np.shape(z)), tau


# ----------------------------------------------------------------------------
# bit-packed masks: bit (c % 32) of word (c // 32) <=> chunk c active
# ----------------------------------------------------------------------------

def pack_mask(active):
    """bool [..., n_c] -> uint32 [..., ceil(n_c / 32)]."""
    active = np.asarray(active, dtype=bool)
    n_c = active.shape[-1]
    n_w = (n_c + 31) // 32
    out = np.zeros(active.shape[:-1] + (n_w,), dtype=np.uint64)
    for c in range(n_c):
        out[..., c // 32] |= active[..., c].astype(np.uint64) << np.uint64(c % 32)
    return out.astype(np.uint32)


def unpack_mask(words, n_c):
    """uint32 [..., n_w] -> bool [..., n_c]."""
    words = np.asarray(words).astype(np.uint64)
    out = np.zeros(words.shape[:-1] + (n_c,), dtype=bool)
    for c in range(n_c):
        out[..., c] = ((words[..., c // 32] >> np.uint64(c % 32)) & np.uint64(1)) == 1
    return out


def pack_weights(w, mask):
    """Compact form of stage 1's output (gist.science summary, Fase 2
    "Implementatie": stage 2 walks the active chunks of a bit-packed mask).

    For every row, the chunks whose mask bit is set, in increasing order, and
    their weights: returns (count [...] int32, index [..., n_c] int32,
    weight [..., n_c] fp64), where only the first count entries of a row of
    index and weight are meaningful (the rest are -1 and 0).
    """
    w = _f64(w)
    n_c = w.shape[-1]
    act = unpack_mask(mask, n_c)
    count = act.sum(axis=-1).astype(np.int32)
    index = np.full(w.shape, -1, dtype=np.int32)
    weight = np.zeros(w.shape)
    flat_a = act.reshape(-1, n_c)
    flat_w = w.reshape(-1, n_c)
    fi = index.reshape(-1, n_c)
    fw = weight.reshape(-1, n_c)
    for r in range(flat_a.shape[0]):
        cs = np.nonzero(flat_a[r])[0]
        fi[r, :cs.size] = cs
        fw[r, :cs.size] = flat_w[r, cs]
    return count, index, weight


def unpack_weights(count, index, weight, n_c):
    """Dense [..., n_c] weights (zero off the listed chunks) and the packed
    mask from the compact form of ``pack_weights``."""
    count = np.asarray(count)
    index = np.asarray(index)
    weight = _f64(weight)
    dense = np.zeros(count.shape + (n_c,))
    fd = dense.reshape(-1, n_c)
    fc, fi, fw = count.reshape(-1), index.reshape(-1, index.shape[-1]), weight.reshape(-1, weight.shape[-1])
    for r in range(fc.size):
        k = int(fc[r])
        fd[r, fi[r, :k]] = fw[r, :k]
    act = np.zeros(dense.shape, dtype=bool)
    fa = act.reshape(-1, n_c)
    for r in range(fc.size):
        fa[r, fi[r, :int(fc[r])]] = True
    return dense, pack_mask(act)


# ----------------------------------------------------------------------------
# Stage 0: chunk summary
# ----------------------------------------------------------------------------

def chunk_summary(K, qbar, B, chunk_begin=0, chunk_end=None):
    """Kbar[b, h, c] = sum_t a_t K[b, h, cB + t] with a = softmax_t(qbar_h . k_t / sqrt(d)).

    K: [b, H_kv, >= chunk_end * B, d]; qbar: [H_kv, d].  Returns fp64
    [b, H_kv, chunk_end - chunk_begin, d] for chunks [chunk_begin, chunk_end).
    """
    K = _f64(K)
    qbar = _f64(qbar)
    b, hkv, n, d = K.shape
    if chunk_end is None:
        chunk_end = n // B
    Kc = K[:, :, chunk_begin * B:chunk_end * B, :].reshape(b, hkv, chunk_end - chunk_begin, B, d)
    s = np.einsum("hd,bhctd->bhct", qbar, Kc) / math.sqrt(d)
    s = s - s.max(axis=-1, keepdims=True)
    a = np.exp(s)
    a = a / a.sum(axis=-1, keepdims=True)
    return np.einsum("bhct,bhctd->bhcd", a, Kc)


# ----------------------------------------------------------------------------
# Stage 1: entmax chunk routing with GQA averaging
# ----------------------------------------------------------------------------

def diagonal_summary(K, qbar, B, i):
    """Estimated summary of the query's own chunk for the query at position i.

    The chunk c_i = floor(i / B) is not complete when its row i is routed, so
    it has no cached summary (gist.science summary, Fase 2 "Diagonaal
    Afhandeling": chunks near the diagonal may have no summary).  The
    estimate is stage 0's learned-query summary taken over the keys the query
    may see, c_i B .. i: ``chunk_summary`` of that partial chunk.  K: [H_kv, >=
    i + 1, d] of one sequence; qbar: [H_kv, d].  Returns fp64 [H_kv, d].
    """
    c_i = i // B
    part = _f64(K)[None, :, c_i * B:i + 1, :]
    return chunk_summary(part, qbar, i + 1 - c_i * B)[0, :, 0, :]


def route(Q, Kbar, alpha, gamma, B, positions=None, near_tol=1e-4, return_heads=False,
          diag=None):
    """Routing weights and active-block mask.

    Q: [b, H_q, N, d]; Kbar: [b, H_kv, n_c, d] (n_c = number of chunk rows
    available).  For each query position i (all of them, or ``positions``):
    z[h, c] = Q[b, h, i] . Kbar[b, h_kv, c] for eligible c < floor(i / B);
    p[h] = alpha-entmax(gamma z[h]); w = mean over the G query heads of the
    KV group; mask bit = (w > 0).

    diag = (K [b, H_kv, N, d], qbar [H_kv, d]) turns on estimate_diagonal
    (aiexpert.news article, interface paragraph: a diagonal correction of the
    alpha-entmax normalisation): the query's own chunk c_i joins the entmax
    as one more candidate, with logit z[h, c_i] = Q[b, h, i] .
    ``diagonal_summary``(i).  Its group-mean weight is written to w[..., c_i];
    the routed chunks c < c_i then share 1 - w[..., c_i].  The mask keeps
    only the routed chunks (bit c_i stays clear: the query's own chunk is
    attended by its own branch in stage 2 whatever its weight).  Rows of the
    first chunk have the diagonal as their only candidate: w[..., 0] = 1.

    Returns (w [b, H_kv, P, n_c] fp64, mask [b, H_kv, P, n_w] uint32,
    near [b, H_kv, P, n_c] bool) where near marks chunks for which some head
    of the group has |(alpha-1) gamma z - tau| < near_tol, i.e. where an
    fp32 implementation may legitimately decide the support bit otherwise.
    With return_heads, also the per-head p [b, H_q, P, n_c].
    """
    b, hq, n, d = Q.shape
    hkv, n_c = Kbar.shape[1], Kbar.shape[2]
    G = hq // hkv
    pos = np.arange(n) if positions is None else np.asarray(positions, dtype=np.int64)
    P = pos.size
    w = np.zeros((b, hkv, P, n_c))
    near = np.zeros((b, hkv, P, n_c), dtype=bool)
    heads = np.zeros((b, hq, P, n_c)) if return_heads else None
    chunk_of = pos // B
    for bi in range(b):
        for g in range(hkv):
            Kb = _f64(Kbar[bi, g])                                      # [n_c, d]
            for c_i in np.unique(chunk_of):
                sel = np.nonzero(chunk_of == c_i)[0]
                ne = int(min(c_i, n_c))
                with_diag = diag is not None and c_i < n_c
                if ne == 0 and not with_diag:
                    continue
                Zq = _take(Q, bi, g * G, (g + 1) * G, pos[sel])          # [G, S, d]
                z = Zq @ Kb[:ne, :].T                                   # [G, S, ne]
                if with_diag:
                    Kd = _take(diag[0], bi, g, g + 1, np.arange(c_i * B, (c_i + 1) * B))[0]
                    est = np.stack([diagonal_summary(Kd[None], _f64(diag[1])[g:g + 1], B,
                                                     int(i) - c_i * B)[0] for i in pos[sel]])
                    zd = np.einsum("gsd,sd->gs", Zq, est)               # [G, S]
                    z = np.concatenate([z, zd[..., None]], axis=-1)     # [G, S, ne + 1]
                p = entmax_bisect(gamma * z, alpha)                     # [G, S, ne (+1)]
                tau = entmax_threshold(gamma * z, alpha)                # [G, S]
                nr = (np.abs((alpha - 1.0) * gamma * z - tau[..., None]) < near_tol).any(axis=0)
                w[bi, g, sel, :ne] = p[..., :ne].mean(axis=0)
                near[bi, g, sel, :ne] = nr[..., :ne]
                if with_diag:
                    w[bi, g, sel, c_i] = p[..., ne].mean(axis=0)
                    near[bi, g, sel, c_i] = nr[..., ne]
                if return_heads:
                    hsl = heads[bi, g * G:(g + 1) * G]
                    hsl[:, sel, :ne] = p[..., :ne]
                    if with_diag:
                        hsl[:, sel, c_i] = p[..., ne]
    routed = w > 0.0
    if diag is not None:
        for k, c_i in enumerate(chunk_of):
            if c_i < n_c:
                routed[:, :, k, c_i] = False
    mask = pack_mask(routed)
    if return_heads:
        return w, mask, near, heads
    return w, mask, near


# ----------------------------------------------------------------------------
# Stage 2: prior-induced block-sparse softmax attention
# ----------------------------------------------------------------------------

def _attend(qg, K, V, w_row, active_row, i, B, sigma):
    """All G heads of one query position against one KV head.

    qg: [G, d]; K, V: [>= i+1, d]; w_row: [n_c]; active_row: bool [n_c].
    Returns o [G, d], lse [G] (natural log of the normaliser of s + bias).
    """
    d = qg.shape[1]
    c_i = i // B
    blocks = [c for c in range(min(c_i, active_row.size)) if active_row[c]]
    idx = [np.arange(c * B, (c + 1) * B) for c in blocks]
    bias = []
    for c in blocks:
        if sigma == 0.0:
            beta = 0.0
        elif w_row[c] > 0.0:
            beta = sigma * math.log(w_row[c])
        else:
            beta = -math.inf
        bias.append(np.full(B, beta))
    idx.append(np.arange(c_i * B, i + 1))         # diagonal branch, causal
    bias.append(np.zeros(i + 1 - c_i * B))
    idx = np.concatenate(idx)
    bias = np.concatenate(bias)
    s = qg @ K[idx].T / math.sqrt(d) + bias[None, :]      # [G, n_keys]
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    o = (e / l) @ V[idx]
    return o, (m + np.log(l))[:, 0]


def attn_fwd(Q, K, V, w, mask, sigma, B, positions=None):
    """O = prior-induced sparse softmax attention, and its log-normaliser.

    Q: [b, H_q, N, d]; K, V: [b, H_kv, N, d]; w: [b, H_kv, P, n_c] and
    mask: [b, H_kv, P, n_w] for the P query positions (all N, or
    ``positions`` in that order).  Returns O [b, H_q, P, d], lse [b, H_q, P].
    """
    w = _f64(w)
    b, hq, n, d = Q.shape
    hkv = K.shape[1]
    G = hq // hkv
    n_c = w.shape[-1]
    active = unpack_mask(mask, n_c)
    pos = np.arange(n) if positions is None else np.asarray(positions, dtype=np.int64)
    O = np.zeros((b, hq, pos.size, d))
    lse = np.zeros((b, hq, pos.size))
    for bi in range(b):
        for g in range(hkv):
            Kf, Vf = _f64(K[bi, g]), _f64(V[bi, g])
            Qg = _take(Q, bi, g * G, (g + 1) * G, pos)                  # [G, P, d]
            for k, i in enumerate(pos):
                o, l = _attend(Qg[:, k, :], Kf, Vf, w[bi, g, k], active[bi, g, k], int(i), B, sigma)
                O[bi, g * G:(g + 1) * G, k] = o
                lse[bi, g * G:(g + 1) * G, k] = l
    return O, lse


# ----------------------------------------------------------------------------
# Decode: one new query per sequence against a cached KV and summary cache
# ----------------------------------------------------------------------------

def decode(q, Kc, Vc, Kbar, L, alpha, gamma, sigma, B, near_tol=1e-4, qbar=None):
    """Single-query step at position L-1 of an L-token cache.

    q: [b, H_q, d]; Kc, Vc: [b, H_kv, >= L, d]; Kbar: [b, H_kv, >= (L-1)//B, d]
    (summaries of complete chunks; only chunks before the query's own are
    read).  Returns (o [b, H_q, d], lse [b, H_q], w [b, H_kv, n_c],
    mask [b, H_kv, n_w], near [b, H_kv, n_c]) with n_c = ceil(L / B).
    With qbar [H_kv, d] given, estimate_diagonal is on, as in ``route``: the
    query's own chunk c_q joins the entmax with the logit of
    ``diagonal_summary`` over the cache rows c_q B .. L - 1, its weight goes
    to w[..., c_q] and its mask bit stays clear.
    """
    q, Kc, Vc, Kbar = _f64(q), _f64(Kc), _f64(Vc), _f64(Kbar)
    b, hq, d = q.shape
    hkv = Kc.shape[1]
    G = hq // hkv
    i = L - 1
    c_q = i // B
    n_c = (L + B - 1) // B
    w = np.zeros((b, hkv, n_c))
    near = np.zeros((b, hkv, n_c), dtype=bool)
    o = np.zeros((b, hq, d))
    lse = np.zeros((b, hq))
    for bi in range(b):
        for g in range(hkv):
            qg = q[bi, g * G:(g + 1) * G]
            z = qg @ Kbar[bi, g, :c_q].T                            # [G, c_q]
            if qbar is not None:
                est = diagonal_summary(Kc[bi, g:g + 1, :L], _f64(qbar)[g:g + 1], B, i)[0]
                z = np.concatenate([z, (qg @ est)[:, None]], axis=1)  # [G, c_q + 1]
            if z.shape[1] > 0:
                p = entmax_bisect(gamma * z, alpha)
                tau = entmax_threshold(gamma * z, alpha)
                w[bi, g, :z.shape[1]] = p.mean(axis=0)
                near[bi, g, :z.shape[1]] = \
                    (np.abs((alpha - 1.0) * gamma * z - tau[:, None]) < near_tol).any(axis=0)
            routed = w[bi, g] > 0.0
            routed[c_q:] = False
            og, lg = _attend(qg, Kc[bi, g, :L], Vc[bi, g, :L], w[bi, g], routed, i, B, sigma)
            o[bi, g * G:(g + 1) * G] = og
            lse[bi, g * G:(g + 1) * G] = lg
    routed = w > 0.0
    routed[..., c_q:] = False
    return o, lse, w, pack_mask(routed), near


def decode_varlen(q, Kc, Vc, Kbar, lens, alpha, gamma, sigma, B, near_tol=1e-4, qbar=None):
    """Decode step for a batch whose sequences hold different numbers of tokens.

    Every sequence takes its own incremental-decoding step (gist.science
    summary, "Belangrijkste Bijdragen" item 4): sequence bi's query sits at
    position lens[bi] - 1 of its own cache, and its result is ``decode`` on its
    first lens[bi] cache rows and the summaries of its complete chunks.  The
    caches share a capacity L_max = Kc.shape[2]; w and near have
    n_c = ceil(L_max / B) columns (zero past the sequence's own), the mask
    ceil(n_c / 32) words.
    """
    q, Kc, Vc, Kbar = _f64(q), _f64(Kc), _f64(Vc), _f64(Kbar)
    b, hq, d = q.shape
    hkv, L_max = Kc.shape[1], Kc.shape[2]
    n_c = (L_max + B - 1) // B
    o = np.zeros((b, hq, d))
    lse = np.zeros((b, hq))
    w = np.zeros((b, hkv, n_c))
    near = np.zeros((b, hkv, n_c), dtype=bool)
    for bi in range(b):
        L = int(lens[bi])
        if not 1 <= L <= L_max:
            raise ValueError(f"cache length {L} outside [1, {L_max}]")
        c_q = (L - 1) // B
        ob, lb, wb, _, nb = decode(q[bi:bi + 1], Kc[bi:bi + 1, :, :L], Vc[bi:bi + 1, :, :L],
                                   Kbar[bi:bi + 1, :, :c_q], L, alpha, gamma, sigma, B, near_tol,
                                   qbar)
        o[bi], lse[bi] = ob[0], lb[0]
        w[bi, :, :wb.shape[2]] = wb[0]
        near[bi, :, :nb.shape[2]] = nb[0]
    routed = w > 0.0
    for bi in range(b):
        routed[bi, :, (int(lens[bi]) - 1) // B:] = False
    return o, lse, w, pack_mask(routed), near


def decode_paged(q, Kpool, Vpool, Kbar, lens, page_table, alpha, gamma, sigma, B, near_tol=1e-4,
                 qbar=None):
    """``decode_varlen`` on caches kept as pages of one chunk each.

    Kpool, Vpool: [n_pages, H_kv, B, d]; page_table[bi, c] is the pool page
    holding chunk c of sequence bi (only chunks below ceil(lens[bi] / B) are
    looked up).  The caches are gathered page by page, with capacity
    page_table.shape[1] * B, and decoded as ``decode_varlen``.
    """
    Kpool, Vpool = _f64(Kpool), _f64(Vpool)
    table = np.asarray(page_table)
    b = table.shape[0]
    n_pages, hkv, Bp, d = Kpool.shape
    if Bp != B:
        raise ValueError("a page holds one chunk of B tokens")
    Kc, Vc = gather_pages(Kpool, Vpool, lens, page_table, B)
    return decode_varlen(q, Kc, Vc, Kbar, lens, alpha, gamma, sigma, B, near_tol, qbar)


def gather_pages(Kpool, Vpool, lens, page_table, B):
    """Contiguous caches [b, H_kv, max_pages * B, d] from one-chunk pages.

    Chunk c of sequence bi (for c below ceil(lens[bi] / B)) is copied from
    page page_table[bi, c]; the rest stays zero.  A page id outside the pool
    raises ValueError.
    """
    Kpool, Vpool = _f64(Kpool), _f64(Vpool)
    table = np.asarray(page_table)
    b = table.shape[0]
    n_pages, hkv, Bp, d = Kpool.shape
    if Bp != B:
        raise ValueError("a page holds one chunk of B tokens")
    cap = table.shape[1] * B
    Kc = np.zeros((b, hkv, cap, d))
    Vc = np.zeros((b, hkv, cap, d))
    for bi in range(b):
        for c in range((int(lens[bi]) + B - 1) // B):
            pg = int(table[bi, c])
            if not 0 <= pg < n_pages:
                raise ValueError(f"page id {pg} outside [0, {n_pages})")
            Kc[bi, :, c * B:(c + 1) * B] = Kpool[pg]
            Vc[bi, :, c * B:(c + 1) * B] = Vpool[pg]
    return Kc, Vc


def decode_attend(q, Kc, Vc, w, mask, lens, sigma, B):
    """Stage 2 alone of a decode step, on given routing weights and mask.

    The prior-induced sparse softmax of gist.science summary "Fase 2" for
    the single query of each sequence (position lens[bi] - 1 of its cache):
    the routed chunks of ``mask`` below the query's own chunk with bias
    sigma * ln w, and the query's own chunk (causal) with bias 0.  This is
    the second half of ``decode`` with its routing replaced by the caller's,
    so a decode kernel's attention output can be compared on the kernel's
    own routing.

    q: [b, H_q, d]; Kc, Vc: [b, H_kv, >= lens, d]; w: [b, H_kv, n_c];
    mask: [b, H_kv, n_w]; lens: per-sequence cache lengths (None: all
    Kc.shape[2]).  Returns (o [b, H_q, d], lse [b, H_q]).
    """
    q, Kc, Vc, w = _f64(q), _f64(Kc), _f64(Vc), _f64(w)
    b, hq, d = q.shape
    hkv, cap = Kc.shape[1], Kc.shape[2]
    G = hq // hkv
    active = unpack_mask(np.asarray(mask), w.shape[-1])
    lens = [cap] * b if lens is None else [int(L) for L in lens]
    o = np.zeros((b, hq, d))
    lse = np.zeros((b, hq))
    for bi in range(b):
        L = lens[bi]
        if not 1 <= L <= cap:
            raise ValueError(f"cache length {L} outside [1, {cap}]")
        for g in range(hkv):
            og, lg = _attend(q[bi, g * G:(g + 1) * G], Kc[bi, g, :L], Vc[bi, g, :L], w[bi, g],
                             active[bi, g], L - 1, B, sigma)
            o[bi, g * G:(g + 1) * G] = og
            lse[bi, g * G:(g + 1) * G] = lg
    return o, lse


def summarize_append(K, qbar, Kbar, lens, B, page_table=None):
    """Summary-cache append for incremental decoding (gist.science summary,
    Fase 0 "Efficiëntie": a chunk's summary is fixed once the chunk is
    complete and is then cached).

    A sequence whose length lens[bi] is a multiple of B has just completed
    chunk c = lens[bi] / B - 1; returns a copy of Kbar [b, H_kv, n, d] with
    that row replaced by the chunk's summary (``chunk_summary`` of its B
    keys).  K is the cache [b, H_kv, >= lens, d], or with page_table the page
    pool [n_pages, H_kv, B, d] (chunk c of sequence bi in page
    page_table[bi, c]).
    """
    K, qbar = _f64(K), _f64(qbar)
    out = _f64(Kbar).copy()
    for bi, L in enumerate(lens):
        L = int(L)
        if L < 1 or L % B:
            continue
        c = L // B - 1
        if page_table is None:
            keys = K[bi:bi + 1, :, c * B:(c + 1) * B]
        else:
            keys = K[int(np.asarray(page_table)[bi, c])][None]
        out[bi, :, c] = chunk_summary(keys, qbar, B)[0, :, 0]
    return out


def route_topk(Q, Kbar, k, gamma, B, positions=None):
    """Fixed-budget top-k routing on the same chunk summaries (the baseline
    the pages contrast with: NSA and InfLLMv2 select the top-k KV blocks by
    coarse attention scores, then run softmax attention on them; gist.science
    summary, "Probleemstelling"; aiexpert.news article, problem paragraph).

    For query position i and KV head g, over the eligible chunks c < floor(i/B):
    score_c = mean over the G query heads of softmax_c(gamma z[h, c]); the k
    chunks with the largest scores are selected (equal scores: lower chunk
    index first; all of them when fewer than k are eligible) and get the
    uniform weight 1 / (number selected).  Returns (w, mask, score) shaped
    like ``route``'s w and mask, score holding the coarse scores.
    """
    b, hq, n, d = Q.shape
    hkv, n_c = Kbar.shape[1], Kbar.shape[2]
    G = hq // hkv
    pos = np.arange(n) if positions is None else np.asarray(positions, dtype=np.int64)
    P = pos.size
    w = np.zeros((b, hkv, P, n_c))
    score = np.zeros((b, hkv, P, n_c))
    for bi in range(b):
        for g in range(hkv):
            Kb = _f64(Kbar[bi, g])
            for j, i in enumerate(pos):
                ne = int(min(i // B, n_c))
                if ne == 0:
                    continue
                z = gamma * (_take(Q, bi, g * G, (g + 1) * G, [i])[:, 0] @ Kb[:ne].T)   # [G, ne]
                e = np.exp(z - z.max(axis=1, keepdims=True))
                s = (e / e.sum(axis=1, keepdims=True)).mean(axis=0)
                order = sorted(range(ne), key=lambda c: (-s[c], c))
                chosen = order[:min(int(k), ne)]
                w[bi, g, j, chosen] = 1.0 / len(chosen)
                score[bi, g, j, :ne] = s
    return w, pack_mask(w > 0.0), score

