"""Pins for the fp64 oracle: each check compares it with something other than itself.

The pages on DashAttention print no worked numeric example, so the pins are
closed forms, brute force on tiny inputs, textbook special cases (sparsemax,
softmax, dense causal attention via torch's own SDPA) and invariants the pages
state (q_bar = 0 gives mean pooling; g = 0 wherever w = 0; GQA heads share one
support; the variational form of the prior-induced softmax).
"""

import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import dash_oracle as O


# ----------------------------------------------------------------------------
# alpha-entmax
# ----------------------------------------------------------------------------

def _brute_entmax(z, alpha):
    """Enumerate supports; keep the one whose own threshold is self-consistent.

    For a candidate support S, tau solves sum_{c in S} ((alpha-1) z_c - tau)^e = 1
    (e = 1/(alpha-1)) with tau below every x_c in S; it is found by a plain
    scalar bisection written here, independent of the oracle.
    """
    x = (alpha - 1.0) * np.asarray(z, dtype=np.float64)
    e = 1.0 / (alpha - 1.0)
    n = x.size
    found = []
    for k in range(1, n + 1):
        for S in itertools.combinations(range(n), k):
            xs = x[list(S)]
            lo, hi = xs.min() - 10.0, xs.min()
            for _ in range(300):
                mid = 0.5 * (lo + hi)
                f = np.sum((xs - mid) ** e) - 1.0
                if f > 0:
                    lo = mid
                else:
                    hi = mid
            tau = 0.5 * (lo + hi)
            inside = np.all(xs > tau)
            outside = np.all(np.delete(x, list(S)) <= tau + 1e-12)
            if inside and outside:
                found.append((S, tau))
    assert len(found) >= 1
    S, tau = found[0]
    p = np.zeros(n)
    p[list(S)] = (x[list(S)] - tau) ** e
    return p


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0, 3.0])
@pytest.mark.parametrize("n", [1, 2, 5, 9])
def test_entmax_matches_brute_force(alpha, n):
    rng = np.random.default_rng(n * 31 + int(alpha * 8))
    for _ in range(4):
        z = rng.normal(scale=2.0, size=n)
        p = oracle.entmax_bisect(z, alpha)
        np.testing.assert_allclose(p, _brute_entmax(z, alpha), atol=1e-9)


def test_entmax15_closed_form_two_inputs():
    # z = (1, 0): x = (1/2, 0); both in the support, (1/2 - t)^2 + t^2 = 1
    # gives t = (1 - sqrt 7) / 4, so p = (((1 + sqrt 7)/4)^2, ((sqrt 7 - 1)/4)^2).
    want = np.array([((1 + math.sqrt(7)) / 4) ** 2, ((math.sqrt(7) - 1) / 4) ** 2])
    np.testing.assert_allclose(oracle.entmax_bisect(np.array([1.0, 0.0]), 1.5), want, atol=1e-13)
    np.testing.assert_allclose(oracle.entmax15_sort(np.array([1.0, 0.0]))[0], want, atol=1e-13)
    # z = (2, 0): x = (1, 0); the top entry alone (t = 0) already sums to one.
    np.testing.assert_allclose(oracle.entmax_bisect(np.array([2.0, 0.0]), 1.5), [1.0, 0.0], atol=1e-13)
    # equal entries: uniform
    np.testing.assert_allclose(oracle.entmax_bisect(np.zeros(4), 1.5), np.full(4, 0.25), atol=1e-13)


def _sparsemax_textbook(z):
    """Sparsemax by sorting (Martins & Astudillo, 2016)."""
    zs = np.sort(z)[::-1]
    cs = np.cumsum(zs)
    k = np.arange(1, z.size + 1)
    kz = k[1 + k * zs > cs].max()
    tau = (cs[kz - 1] - 1.0) / kz
    return np.maximum(z - tau, 0.0)


def test_entmax_alpha2_is_sparsemax():
    rng = np.random.default_rng(7)
    for n in [3, 17, 200]:
        z = rng.normal(size=n)
        np.testing.assert_allclose(oracle.entmax_bisect(z, 2.0), _sparsemax_textbook(z), atol=1e-12)


def test_entmax_alpha_to_one_is_softmax():
    rng = np.random.default_rng(8)
    z = rng.normal(size=50)
    sm = np.exp(z - z.max())
    sm /= sm.sum()
    # the gap to softmax shrinks linearly with alpha - 1
    err3 = np.abs(oracle.entmax_bisect(z, 1.0 + 1e-3) - sm).max()
    err5 = np.abs(oracle.entmax_bisect(z, 1.0 + 1e-5) - sm).max()
    assert err5 < 1e-4
    assert err5 < err3 / 20


@pytest.mark.parametrize("alpha", [1.5, 1.7, 2.0])
def test_entmax_sum_support_shift(alpha):
    rng = np.random.default_rng(9)
    z = rng.normal(scale=3.0, size=(6, 40))
    p = oracle.entmax_bisect(z, alpha)
    tau = O.entmax_threshold(z, alpha)
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-12)
    x = (alpha - 1) * z
    assert np.array_equal(p > 0, x > tau[:, None])
    assert np.all(p >= 0)
    np.testing.assert_allclose(oracle.entmax_bisect(z + 3.7, alpha), p, atol=1e-12)


def test_entmax_masked_entries_and_empty_rows():
    z = np.array([[1.0, -np.inf, 0.5], [-np.inf, -np.inf, -np.inf]])
    p = oracle.entmax_bisect(z, 1.5)
    sub = _brute_entmax(np.array([1.0, 0.5]), 1.5)
    np.testing.assert_allclose(p[0], [sub[0], 0.0, sub[1]], atol=1e-12)
    assert np.all(p[1] == 0)


def test_entmax15_sort_matches_bisect_and_brute():
    rng = np.random.default_rng(10)
    for n in [1, 4, 8]:
        z = rng.normal(scale=1.5, size=n)
        np.testing.assert_allclose(oracle.entmax15_sort(z)[0], _brute_entmax(z, 1.5), atol=1e-10)
    for n in [64, 1000]:
        z = rng.normal(scale=4.0, size=n)
        np.testing.assert_allclose(oracle.entmax15_sort(z)[0], oracle.entmax_bisect(z, 1.5), atol=1e-10)


# ----------------------------------------------------------------------------
# masks
# ----------------------------------------------------------------------------

def test_mask_bit_order():
    active = np.zeros(40, dtype=bool)
    active[[0, 5, 31, 32, 39]] = True
    words = oracle.pack_mask(active)
    assert words.dtype == np.uint32 and words.shape == (2,)
    assert int(words[0]) == (1 << 0) | (1 << 5) | (1 << 31)
    assert int(words[1]) == (1 << 0) | (1 << 7)
    assert np.array_equal(oracle.unpack_mask(words, 40), active)


# ----------------------------------------------------------------------------
# Stage 0
# ----------------------------------------------------------------------------

def test_summary_zero_query_is_mean_pooling():
    rng = np.random.default_rng(11)
    K = rng.normal(size=(2, 3, 256, 32))
    got = oracle.chunk_summary(K, np.zeros((3, 32)), 64)
    np.testing.assert_allclose(got, K.reshape(2, 3, 4, 64, 32).mean(axis=3), atol=1e-13)


def test_summary_is_local_sdpa_over_each_chunk():
    # stage 0 is scaled dot-product attention of one query per KV head over
    # the keys of a chunk, with the keys as values: torch's SDPA per chunk.
    rng = np.random.default_rng(21)
    K = rng.normal(size=(2, 2, 192, 16))
    qb = rng.normal(size=(2, 16))
    got = oracle.chunk_summary(K, qb, 64)
    for b in range(2):
        for h in range(2):
            for c in range(3):
                kc = torch.from_numpy(K[b, h, c * 64:(c + 1) * 64])[None]
                q = torch.from_numpy(qb[h])[None, None]
                ref = torch.nn.functional.scaled_dot_product_attention(q, kc, kc)
                np.testing.assert_allclose(got[b, h, c], ref[0, 0].numpy(), atol=1e-13)


def test_summary_peaked_query_selects_key_and_hull():
    rng = np.random.default_rng(12)
    K = rng.normal(size=(1, 1, 128, 16))
    t = 77  # chunk 1, position 13
    qbar = 200.0 * K[0, 0, t][None, :] / np.linalg.norm(K[0, 0, t])
    # make sure key t is the unique maximiser of qbar . k within its chunk
    K[0, 0, 64:128] *= 0.5
    K[0, 0, t] *= 2.0
    got = oracle.chunk_summary(K, qbar, 64)
    np.testing.assert_allclose(got[0, 0, 1], K[0, 0, t], atol=1e-8)
    # any summary is a convex combination of its chunk's keys
    qb = rng.normal(size=(1, 16))
    S = oracle.chunk_summary(K, qb, 64)
    for _ in range(20):
        u = rng.normal(size=16)
        for c in range(2):
            proj = K[0, 0, c * 64:(c + 1) * 64] @ u
            assert proj.min() - 1e-12 <= S[0, 0, c] @ u <= proj.max() + 1e-12


def test_summary_permutation_invariant_and_range():
    rng = np.random.default_rng(13)
    K = rng.normal(size=(1, 2, 192, 8))
    qb = rng.normal(size=(2, 8))
    perm = rng.permutation(64)
    Kp = K.copy()
    Kp[:, :, 64:128] = K[:, :, 64 + perm]
    np.testing.assert_allclose(oracle.chunk_summary(Kp, qb, 64), oracle.chunk_summary(K, qb, 64), atol=1e-13)
    part = oracle.chunk_summary(K, qb, 64, chunk_begin=1, chunk_end=3)
    np.testing.assert_allclose(part, oracle.chunk_summary(K, qb, 64)[:, :, 1:3], atol=0)


# ----------------------------------------------------------------------------
# Stage 1
# ----------------------------------------------------------------------------

def test_route_single_head_is_plain_entmax():
    rng = np.random.default_rng(14)
    B, n, d = 8, 64, 4
    Q = rng.normal(size=(1, 1, n, d))
    Kbar = rng.normal(size=(1, 1, n // B, d))
    gamma = 0.7
    w, mask, near = oracle.route(Q, Kbar, 1.5, gamma, B)
    for i in range(n):
        ci = i // B
        if ci == 0:
            assert np.all(w[0, 0, i] == 0)
            continue
        z = np.array([sum(Q[0, 0, i, t] * Kbar[0, 0, c, t] for t in range(d)) for c in range(ci)])
        np.testing.assert_allclose(w[0, 0, i, :ci], _brute_entmax(gamma * z, 1.5), atol=1e-9)
        assert np.all(w[0, 0, i, ci:] == 0)
    assert np.array_equal(oracle.unpack_mask(mask, n // B), w > 0)


def test_route_gqa_mean_and_shared_support():
    rng = np.random.default_rng(15)
    B, n, d = 16, 160, 8
    Q = rng.normal(size=(2, 6, n, d))
    Kbar = rng.normal(size=(2, 2, n // B, d))
    w, mask, near, heads = oracle.route(Q, Kbar, 1.5, 1.0, B, return_heads=True)
    G = 3
    for b in range(2):
        for g in range(2):
            hp = heads[b, g * G:(g + 1) * G]
            np.testing.assert_allclose(w[b, g], hp.mean(axis=0), atol=1e-15)
            # the shared support is the union of the member supports
            assert np.array_equal(w[b, g] > 0, (hp > 0).any(axis=0))
            rows = np.arange(n) >= B
            np.testing.assert_allclose(w[b, g, rows].sum(-1), 1.0, atol=1e-12)
    # positions subset reproduces the full result
    pos = [17, 40, 159]
    w2, m2, _ = oracle.route(Q, Kbar, 1.5, 1.0, B, positions=pos)
    np.testing.assert_allclose(w2, w[:, :, pos], atol=0)
    assert np.array_equal(m2, mask[:, :, pos])


def test_pack_weights_against_the_dense_rows():
    rng = np.random.default_rng(45)
    B = 16
    Q = rng.normal(size=(2, 4, 128, 8))
    Kbar = rng.normal(size=(2, 2, 8, 8))
    w, mask, _ = oracle.route(Q, Kbar, 1.5, 1.0, B)
    count, index, weight = oracle.pack_weights(w, mask)
    dense, m2 = oracle.unpack_weights(count, index, weight, 8)
    np.testing.assert_array_equal(dense, w)
    np.testing.assert_array_equal(m2, mask)
    # a direct scan of each dense row, written out here
    for b in range(2):
        for g in range(2):
            for i in range(128):
                cs = [c for c in range(8) if w[b, g, i, c] > 0]
                assert count[b, g, i] == len(cs) == bin(int(mask[b, g, i, 0])).count("1")
                assert list(index[b, g, i, :len(cs)]) == cs
                assert list(weight[b, g, i, :len(cs)]) == [w[b, g, i, c] for c in cs]
                assert (index[b, g, i, len(cs):] == -1).all()
    # rows of the first chunk are empty
    assert not count[:, :, :B].any()


# ----------------------------------------------------------------------------
# estimate_diagonal: the query's own chunk as one more entmax candidate
# ----------------------------------------------------------------------------

def _diag_case(seed, b=1, hq=4, hkv=2, n=96, d=8, B=16):
    rng = np.random.default_rng(seed)
    Q = rng.normal(size=(b, hq, n, d))
    K = rng.normal(size=(b, hkv, n, d))
    qbar = rng.normal(size=(hkv, d)) * 0.5
    return Q, K, qbar, oracle.chunk_summary(K, qbar, B)


def test_route_diag_weights_mask_and_first_chunk():
    B = 16
    Q, K, qbar, Kbar = _diag_case(40, b=2)
    n = Q.shape[2]
    w, mask, _, heads = oracle.route(Q, Kbar, 1.5, 1.0, B, diag=(K, qbar), return_heads=True)
    c_i = np.arange(n) // B
    act = oracle.unpack_mask(mask, Kbar.shape[2])
    for i in range(n):
        # the routed chunks and the diagonal share the unit mass
        np.testing.assert_allclose(w[:, :, i, :c_i[i] + 1].sum(-1), 1.0, atol=1e-12)
        assert not w[:, :, i, c_i[i] + 1:].any()
        # the mask holds the routed chunks only, never the query's own chunk
        assert np.array_equal(act[:, :, i, :c_i[i]], w[:, :, i, :c_i[i]] > 0)
        assert not act[:, :, i, c_i[i]:].any()
    # rows of the first chunk: the diagonal is the only candidate
    np.testing.assert_allclose(w[:, :, :B, 0], 1.0, atol=1e-12)
    np.testing.assert_allclose(heads[:, :, :B, 0], 1.0, atol=1e-12)
    # w is the group mean of the per-head weights, diagonal column included
    np.testing.assert_allclose(w, heads.reshape(2, 2, 2, n, -1).mean(axis=2), atol=1e-15)


def test_route_diag_hand_computed_sparsemax():
    # alpha = 2 (sparsemax), one head, B = 2: for two candidates x0, x1 with
    # |x0 - x1| < 1 the weights are ((x0 - x1 + 1) / 2, (x1 - x0 + 1) / 2)
    rng = np.random.default_rng(41)
    B, d, gamma = 2, 4, 0.3
    Q = rng.normal(size=(1, 1, 4, d))
    K = rng.normal(size=(1, 1, 4, d))
    qbar = rng.normal(size=(1, d))
    Kbar = oracle.chunk_summary(K, qbar, B)
    w, mask, _ = oracle.route(Q, Kbar, 2.0, gamma, B, diag=(K, qbar))
    for i in (2, 3):
        # position 2 sees key 2 alone (estimate = k2); position 3 sees keys 2, 3
        s = np.array([qbar[0] @ K[0, 0, 2], qbar[0] @ K[0, 0, 3]]) / math.sqrt(d)
        a = np.exp(s[: i - 1] - s[: i - 1].max())
        est = (a / a.sum()) @ K[0, 0, 2:i + 1]
        x0 = gamma * (Q[0, 0, i] @ Kbar[0, 0, 0])
        x1 = gamma * (Q[0, 0, i] @ est)
        if abs(x0 - x1) < 1.0:
            want = [(x0 - x1 + 1) / 2, (x1 - x0 + 1) / 2]
        else:
            want = [1.0, 0.0] if x0 > x1 else [0.0, 1.0]
        np.testing.assert_allclose(w[0, 0, i, :2], want, atol=1e-12)
        assert oracle.unpack_mask(mask[0, 0, i], 2)[0] == (want[0] > 0)
    np.testing.assert_allclose(w[0, 0, :2, 0], 1.0, atol=1e-12)


def test_route_diag_at_a_chunk_end_is_plain_routing_a_chunk_later():
    # at the last row of chunk c the estimate covers the whole chunk, i.e. it
    # is the summary K_bar_c; routing there equals plain routing (no diagonal
    # candidate) of the same query one position later, where chunk c has
    # become an eligible chunk
    B = 16
    Q, K, qbar, Kbar = _diag_case(42, n=96)
    for c in (0, 2, 4):
        i = (c + 1) * B - 1
        Q2 = Q.copy()
        Q2[:, :, i + 1] = Q[:, :, i]
        wd, _, _ = oracle.route(Q, Kbar, 1.5, 1.0, B, positions=[i], diag=(K, qbar))
        wp, _, _ = oracle.route(Q2, Kbar, 1.5, 1.0, B, positions=[i + 1])
        np.testing.assert_allclose(wd[:, :, 0, :c + 1], wp[:, :, 0, :c + 1], atol=1e-12)


def test_decode_diag_is_the_last_routed_row():
    B, L = 16, 90
    Q, K, qbar, Kbar = _diag_case(43, b=2, n=96)
    rng = np.random.default_rng(44)
    V = rng.normal(size=K.shape)
    w, mask, _ = oracle.route(Q, Kbar, 1.5, 0.9, B, positions=[L - 1], diag=(K, qbar))
    O, lse = oracle.attn_fwd(Q, K, V, w, mask, 0.7, B, positions=[L - 1])
    o, lse_d, wd, md, _ = oracle.decode(Q[:, :, L - 1], K, V, Kbar, L, 1.5, 0.9, 0.7, B, qbar=qbar)
    n_c = wd.shape[-1]
    np.testing.assert_allclose(wd, w[:, :, 0, :n_c], atol=1e-12)
    assert np.array_equal(oracle.unpack_mask(md, n_c), oracle.unpack_mask(mask[:, :, 0], 6)[..., :n_c])
    np.testing.assert_allclose(o, O[:, :, 0], atol=1e-12)
    np.testing.assert_allclose(lse_d, lse[:, :, 0], atol=1e-12)
    # a length per sequence reduces to the fixed-length call, pages to contiguous
    got = oracle.decode_varlen(Q[:, :, L - 1], K[:, :, :L], V[:, :, :L], Kbar, [L, L], 1.5, 0.9,
                               0.7, B, qbar=qbar)
    for a, b_ in zip(got, (o, lse_d, wd, md)):
        np.testing.assert_array_equal(a, b_)


# ----------------------------------------------------------------------------
# Stage 2
# ----------------------------------------------------------------------------

def _all_active(b, hkv, n, n_c):
    w = np.full((b, hkv, n, n_c), 0.5)
    return w, oracle.pack_mask(np.ones((b, hkv, n, n_c), dtype=bool))


def test_stage2_all_active_sigma0_is_dense_causal_sdpa():
    rng = np.random.default_rng(16)
    b, hq, hkv, n, d, B = 1, 4, 2, 96, 16, 16
    Q, K, V = (rng.normal(size=s) for s in [(b, hq, n, d), (b, hkv, n, d), (b, hkv, n, d)])
    w, mask = _all_active(b, hkv, n, n // B)
    out, lse = oracle.attn_fwd(Q, K, V, w, mask, 0.0, B)
    tq, tk, tv = (torch.from_numpy(a) for a in (Q, K, V))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True, enable_gqa=True)
    np.testing.assert_allclose(out, ref.numpy(), atol=1e-12)
    s = (tq @ tk.repeat_interleave(2, dim=1).transpose(-1, -2)) / math.sqrt(d)
    s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), atol=1e-12)


def test_stage2_uniform_prior_equals_dense_for_any_sigma():
    # w constant over every chunk gives g constant within the query's routed
    # blocks, but the diagonal block keeps weight 1: with w = 1 the prior is
    # uniform everywhere for any sigma.
    rng = np.random.default_rng(17)
    b, hq, hkv, n, d, B = 1, 2, 1, 64, 8, 16
    Q, K, V = (rng.normal(size=s) for s in [(b, hq, n, d), (b, hkv, n, d), (b, hkv, n, d)])
    w = np.ones((b, hkv, n, n // B))
    mask = oracle.pack_mask(w > 0)
    o0, _ = oracle.attn_fwd(Q, K, V, w, mask, 0.0, B)
    o1, _ = oracle.attn_fwd(Q, K, V, w, mask, 1.0, B)
    np.testing.assert_allclose(o1, o0, atol=1e-13)


def _variational_objective(p, s, g):
    """z^T p - KL(p || g) on the support of g (0 log 0 = 0)."""
    nz = p > 0
    return float(p @ s - np.sum(p[nz] * (np.log(p[nz]) - np.log(g[nz]))))


def test_stage2_is_maximiser_of_prior_variational_form():
    # With V = identity rows the output row is the attention distribution p.
    rng = np.random.default_rng(18)
    b, hq, hkv, B = 1, 1, 1, 8
    n = 40
    d = 64                      # >= n, so one-hot value rows fit
    Q = rng.normal(size=(b, hq, n, d)) * 0.5
    K = rng.normal(size=(b, hkv, n, d))
    V = np.zeros((b, hkv, n, d))
    V[0, 0, np.arange(n), np.arange(n)] = 1.0
    n_c = n // B
    w = rng.uniform(0.05, 1.0, size=(b, hkv, n, n_c))
    act = rng.uniform(size=(b, hkv, n, n_c)) < 0.5
    w = np.where(act, w, 0.0)
    sigma = 0.8
    out, _ = oracle.attn_fwd(Q, K, V, w, oracle.pack_mask(act), sigma, B)
    for i in [9, 23, 39]:
        p = out[0, 0, i, :n]
        ci = i // B
        s = K[0, 0, :n] @ Q[0, 0, i] / math.sqrt(d)
        g = np.zeros(n)
        for j in range(i + 1):
            c = j // B
            if c == ci:
                g[j] = 1.0
            elif act[0, 0, i, c]:
                g[j] = w[0, 0, i, c] ** sigma
        g = g / g.sum()
        # g = 0 wherever the routing weight is zero: those keys get no mass
        assert np.all(p[g == 0] < 1e-15)
        np.testing.assert_allclose(p.sum(), 1.0, atol=1e-12)
        best = _variational_objective(p, s, g)
        supp = np.nonzero(g > 0)[0]
        for _ in range(200):
            q = p.copy()
            q[supp] *= np.exp(rng.normal(scale=0.05, size=supp.size))
            q /= q.sum()
            assert _variational_objective(q, s, g) <= best + 1e-12


def test_stage2_single_block_is_local_softmax():
    rng = np.random.default_rng(19)
    b, hq, hkv, n, d, B = 1, 2, 1, 64, 8, 16
    Q, K, V = (rng.normal(size=s) for s in [(b, hq, n, d), (b, hkv, n, d), (b, hkv, n, d)])
    act = np.zeros((b, hkv, n, n // B), dtype=bool)
    act[..., 1] = True
    w = np.where(act, 0.3, 0.0)
    out, _ = oracle.attn_fwd(Q, K, V, w, oracle.pack_mask(act), 2.0, B)
    i = 50                          # chunk 3; routed block 1 plus its own chunk
    keys = list(range(16, 32)) + list(range(48, 51))
    for h in range(2):
        s = K[0, 0, keys] @ Q[0, h, i] / math.sqrt(d)
        s[:16] += 2.0 * math.log(0.3)
        p = np.exp(s - s.max())
        p /= p.sum()
        np.testing.assert_allclose(out[0, h, i], p @ V[0, 0, keys], atol=1e-12)
    # rows in chunks 0 and 1 only see their own chunk
    i = 20
    s = K[0, 0, 16:21] @ Q[0, 0, i] / math.sqrt(d)
    p = np.exp(s - s.max())
    np.testing.assert_allclose(out[0, 0, i], (p / p.sum()) @ V[0, 0, 16:21], atol=1e-12)


# ----------------------------------------------------------------------------
# Decode
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("L", [200, 256, 65])
def test_decode_equals_last_prefill_row(L):
    rng = np.random.default_rng(20 + L)
    b, hq, hkv, d, B = 2, 4, 2, 16, 16
    n = ((L + B - 1) // B) * B
    Q = rng.normal(size=(b, hq, n, d))
    K = rng.normal(size=(b, hkv, n, d))
    V = rng.normal(size=(b, hkv, n, d))
    qbar = rng.normal(size=(hkv, d)) * 0.1
    Kbar = oracle.chunk_summary(K, qbar, B)
    w, mask, _ = oracle.route(Q, Kbar, 1.5, 0.9, B, positions=[L - 1])
    O, lse = oracle.attn_fwd(Q, K, V, w, mask, 0.7, B, positions=[L - 1])
    o, lse_d, wd, md, _ = oracle.decode(Q[:, :, L - 1], K, V, Kbar, L, 1.5, 0.9, 0.7, B)
    np.testing.assert_allclose(o, O[:, :, 0], atol=1e-12)
    np.testing.assert_allclose(lse_d, lse[:, :, 0], atol=1e-12)
    np.testing.assert_allclose(wd, w[:, :, 0, :wd.shape[-1]], atol=0)


def test_decode_attend_dense_is_sdpa_of_the_last_row():
    # every chunk active with w = 1: the prior is uniform over the causal
    # prefix for any sigma, so each sequence's output is torch's SDPA of its
    # query against its first L keys
    rng = np.random.default_rng(25)
    b, hq, hkv, d, B, cap = 3, 4, 2, 16, 16, 160
    lens = [160, 1, 77]
    q = rng.normal(size=(b, hq, d))
    K = rng.normal(size=(b, hkv, cap, d))
    V = rng.normal(size=(b, hkv, cap, d))
    n_c = cap // B
    w = np.ones((b, hkv, n_c))
    mask = oracle.pack_mask(w > 0)
    o, lse = oracle.decode_attend(q, K, V, w, mask, lens, 0.9, B)
    for bi, L in enumerate(lens):
        tq = torch.from_numpy(q[bi][None, :, None, :])
        tk, tv = (torch.from_numpy(a[bi][None, :, :L]) for a in (K, V))
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, enable_gqa=True)
        np.testing.assert_allclose(o[bi], ref[0, :, 0].numpy(), atol=1e-12)
        s = np.einsum("hd,hkd->hk", q[bi], np.repeat(K[bi, :, :L], 2, axis=0)) / math.sqrt(d)
        np.testing.assert_allclose(lse[bi], torch.logsumexp(torch.from_numpy(s), dim=1).numpy(),
                                   atol=1e-12)


def test_decode_attend_on_decode_routing_is_decode_and_prefill_row():
    # fed the routing that decode computes, stage 2 alone gives decode's output,
    # i.e. the last prefill row (itself pinned to dense SDPA and the variational
    # form); fed a different routing it follows that routing instead
    rng = np.random.default_rng(26)
    b, hq, hkv, d, B, L = 2, 4, 2, 16, 16, 150
    Q = rng.normal(size=(b, hq, L, d))
    K = rng.normal(size=(b, hkv, L, d))
    V = rng.normal(size=(b, hkv, L, d))
    Kbar = oracle.chunk_summary(K, rng.normal(size=(hkv, d)) * 0.1, B)
    o, lse, w, mask, _ = oracle.decode(Q[:, :, L - 1], K, V, Kbar, L, 1.5, 0.9, 0.7, B)
    o2, lse2 = oracle.decode_attend(Q[:, :, L - 1], K, V, w, mask, None, 0.7, B)
    np.testing.assert_array_equal(o2, o)
    np.testing.assert_array_equal(lse2, lse)
    # one routed chunk (chunk 2, weight 0.3) plus the query's own chunk 9 (keys 144..149)
    w1 = np.zeros_like(w)
    w1[..., 2] = 0.3
    o3, _ = oracle.decode_attend(Q[:, :, L - 1], K, V, w1, oracle.pack_mask(w1 > 0), None, 2.0, B)
    keys = list(range(32, 48)) + list(range(144, 150))
    for bi in range(b):
        for h in range(hq):
            s = K[bi, h // 2, keys] @ Q[bi, h, L - 1] / math.sqrt(d)
            s[:16] += 2.0 * math.log(0.3)
            p = np.exp(s - s.max())
            np.testing.assert_allclose(o3[bi, h], (p / p.sum()) @ V[bi, h // 2, keys], atol=1e-12)


def _varlen_case(seed, b=3, hq=4, hkv=2, d=16, B=16, L_max=200):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(b, hq, d))
    K = rng.normal(size=(b, hkv, L_max, d))
    V = rng.normal(size=(b, hkv, L_max, d))
    qbar = rng.normal(size=(hkv, d)) * 0.1
    return q, K, V, qbar


def test_decode_varlen_rows_are_last_prefill_rows():
    B, d = 16, 16
    lens = [200, 1, 65, 16, 17]
    q, K, V, qbar = _varlen_case(31, b=len(lens), d=d, B=B)
    Kbar = oracle.chunk_summary(K, qbar, B)
    o, lse, w, mask, _ = oracle.decode_varlen(q, K, V, Kbar, lens, 1.5, 0.9, 0.7, B)
    n_c = (200 + B - 1) // B
    assert w.shape == (len(lens), 2, n_c) and mask.shape == (len(lens), 2, (n_c + 31) // 32)
    for bi, L in enumerate(lens):
        # prefill of this sequence's own prefix (padded to whole chunks), row L - 1
        n = ((L + B - 1) // B) * B
        Qp = np.zeros((1, 4, n, d))
        Qp[0, :, L - 1] = q[bi]
        Kp, Vp = K[bi:bi + 1, :, :n], V[bi:bi + 1, :, :n]
        Kb = oracle.chunk_summary(Kp, qbar, B)
        wp, mp, _ = oracle.route(Qp, Kb, 1.5, 0.9, B, positions=[L - 1])
        Op, lp = oracle.attn_fwd(Qp, Kp, Vp, wp, mp, 0.7, B, positions=[L - 1])
        np.testing.assert_allclose(o[bi], Op[0, :, 0], atol=1e-12)
        np.testing.assert_allclose(lse[bi], lp[0, :, 0], atol=1e-12)
        c_q = (L - 1) // B
        np.testing.assert_allclose(w[bi, :, :c_q], wp[0, :, 0, :c_q], atol=0)
        assert not w[bi, :, c_q:].any()
        assert (oracle.unpack_mask(mask[bi], n_c) == (w[bi] > 0)).all()


def test_decode_varlen_equal_lengths_is_decode():
    B, L = 16, 200
    q, K, V, qbar = _varlen_case(32, B=B, L_max=L)
    Kbar = oracle.chunk_summary(K, qbar, B)
    got = oracle.decode_varlen(q, K, V, Kbar, [L] * 3, 1.5, 0.9, 0.7, B)
    want = oracle.decode(q, K, V, Kbar, L, 1.5, 0.9, 0.7, B)
    for a, b_ in zip(got, want):
        np.testing.assert_array_equal(a, b_)


def test_decode_varlen_ignores_everything_past_each_length():
    B = 16
    lens = [37, 200, 120]
    q, K, V, qbar = _varlen_case(33, B=B)
    Kbar = oracle.chunk_summary(K, qbar, B)
    ref = oracle.decode_varlen(q, K, V, Kbar, lens, 2.0, 0.9, 1.0, B)
    rng = np.random.default_rng(34)
    K2, V2, Kb2 = K.copy(), V.copy(), Kbar.copy()
    for bi, L in enumerate(lens):
        K2[bi, :, L:] += 50.0 * rng.normal(size=K2[bi, :, L:].shape)
        V2[bi, :, L:] -= 50.0
        Kb2[bi, :, (L - 1) // B:] = 1e3
    got = oracle.decode_varlen(q, K2, V2, Kb2, lens, 2.0, 0.9, 1.0, B)
    for a, b_ in zip(got, ref):
        np.testing.assert_array_equal(a, b_)
    with pytest.raises(ValueError):
        oracle.decode_varlen(q, K, V, Kbar, [0, 5, 5], 2.0, 0.9, 1.0, B)


def _pages_of(K, B):
    """[b, h, cap, d] -> pool [b * cap / B, h, B, d] (page of sequence bi, chunk c at bi * n + c)."""
    b, h, cap, d = K.shape
    n = cap // B
    return K.reshape(b, h, n, B, d).transpose(0, 2, 1, 3, 4).reshape(b * n, h, B, d), n


def test_decode_paged_identity_table_is_varlen():
    B, cap = 16, 208
    lens = [200, 1, 16, 17, 208]
    q, K, V, qbar = _varlen_case(35, b=len(lens), B=B, L_max=cap)
    Kbar = oracle.chunk_summary(K, qbar, B)
    Kp, n = _pages_of(K, B)
    Vp, _ = _pages_of(V, B)
    table = np.arange(len(lens) * n).reshape(len(lens), n)
    got = oracle.decode_paged(q, Kp, Vp, Kbar, lens, table, 1.5, 0.9, 0.7, B)
    want = oracle.decode_varlen(q, K, V, Kbar, lens, 1.5, 0.9, 0.7, B)
    for a, b_ in zip(got, want):
        np.testing.assert_array_equal(a, b_)


def test_decode_paged_page_order_and_unused_pages_do_not_matter():
    B, cap = 16, 208
    lens = [150, 33, 208]
    q, K, V, qbar = _varlen_case(36, b=len(lens), B=B, L_max=cap)
    Kbar = oracle.chunk_summary(K, qbar, B)
    Kp, n = _pages_of(K, B)
    Vp, _ = _pages_of(V, B)
    table = np.arange(len(lens) * n).reshape(len(lens), n)
    ref = oracle.decode_paged(q, Kp, Vp, Kbar, lens, table, 2.0, 0.9, 1.0, B)
    rng = np.random.default_rng(37)
    perm = rng.permutation(len(Kp))                       # page j moves to slot perm[j]
    extra = 5                                             # pages nobody references
    Kq = rng.normal(size=(len(Kp) + extra,) + Kp.shape[1:]) * 40.0
    Vq = rng.normal(size=(len(Vp) + extra,) + Vp.shape[1:]) * 40.0
    Kq[perm], Vq[perm] = Kp, Vp
    table2 = perm[table]
    for bi, L in enumerate(lens):                         # entries past a sequence's chunks
        table2[bi, (L + B - 1) // B:] = len(Kp) + bi % extra
    got = oracle.decode_paged(q, Kq, Vq, Kbar, lens, table2, 2.0, 0.9, 1.0, B)
    for a, b_ in zip(got, ref):
        np.testing.assert_array_equal(a, b_)
    bad = table2.copy()
    bad[0, 0] = len(Kq)
    with pytest.raises(ValueError):
        oracle.decode_paged(q, Kq, Vq, Kbar, lens, bad, 2.0, 0.9, 1.0, B)


def test_summarize_append_rebuilds_the_summary_cache():
    # grow three caches token by token; appending at every boundary gives the
    # summaries of the whole cache, computed in one go
    B, cap = 16, 96
    rng = np.random.default_rng(38)
    K = rng.normal(size=(3, 2, cap, 8))
    qbar = rng.normal(size=(2, 8)) * 0.5
    full = oracle.chunk_summary(K, qbar, B)
    kb = np.full_like(full, 7.0)
    lens = np.array([1, 5, 16])
    while True:
        kb = oracle.summarize_append(K, qbar, kb, lens, B)
        if lens.min() == cap:
            break
        lens = np.minimum(lens + 1, cap)
    np.testing.assert_array_equal(kb, full)


def test_summarize_append_touches_only_boundary_sequences_and_pages_agree():
    B, cap = 16, 64
    rng = np.random.default_rng(39)
    K = rng.normal(size=(3, 2, cap, 8))
    qbar = rng.normal(size=(2, 8)) * 0.5
    kb = rng.normal(size=(3, 2, cap // B, 8))
    lens = [32, 33, 64]
    got = oracle.summarize_append(K, qbar, kb, lens, B)
    np.testing.assert_array_equal(got[1], kb[1])                    # not at a boundary
    np.testing.assert_array_equal(got[0, :, [0, 2, 3]], kb[0, :, [0, 2, 3]])
    full = oracle.chunk_summary(K, qbar, B)
    np.testing.assert_array_equal(got[0, :, 1], full[0, :, 1])
    np.testing.assert_array_equal(got[2, :, 3], full[2, :, 3])
    Kp, n = _pages_of(K, B)
    table = np.arange(3 * n).reshape(3, n)
    np.testing.assert_array_equal(oracle.summarize_append(Kp, qbar, kb, lens, B, table), got)


def test_route_topk_single_head_is_k_largest_logits():
    rng = np.random.default_rng(40)
    B, d = 16, 8
    Q = rng.normal(size=(1, 2, 160, d))
    Kbar = rng.normal(size=(1, 2, 10, d))
    for k in (1, 3, 9, 40):
        w, mask, score = oracle.route_topk(Q, Kbar, k, 0.7, B)
        for g in range(2):
            for i in range(160):
                ne = min(i // B, 10)
                sel = np.nonzero(w[0, g, i])[0]
                if ne == 0:
                    assert sel.size == 0
                    continue
                z = Q[0, g, i] @ Kbar[0, g, :ne].T
                want = np.sort(np.argsort(-z, kind="stable")[:min(k, ne)])
                np.testing.assert_array_equal(sel, want)
                np.testing.assert_allclose(w[0, g, i, sel], 1.0 / sel.size)
                np.testing.assert_allclose(score[0, g, i, :ne].sum(), 1.0, atol=1e-12)
                assert (oracle.unpack_mask(mask[0, g, i], 10) == (w[0, g, i] > 0)).all()


def test_route_topk_group_scores_and_ties():
    B, d = 16, 4
    # two heads with mirrored preferences: every chunk gets the same mean
    # score, so the lower indices win
    Kbar = np.zeros((1, 1, 6, d))
    Kbar[0, 0, :, 0] = np.arange(6)
    Q = np.zeros((1, 2, 112, d))
    Q[0, 0, :, 0] = 1.0
    Q[0, 1, :, 0] = -1.0
    w, _, score = oracle.route_topk(Q, Kbar, 2, 1.0, B)
    i = 100                                           # 6 eligible chunks
    z = np.arange(6.0)
    p0 = np.exp(z - z.max()) / np.exp(z - z.max()).sum()
    np.testing.assert_allclose(score[0, 0, i, :6], (p0 + p0[::-1]) / 2, atol=1e-12)
    # scores are symmetric: chunks 0 and 5 tie at the top, then 1 and 4
    assert list(np.nonzero(w[0, 0, i])[0]) == [0, 5]
    w3, _, _ = oracle.route_topk(Q, Kbar, 3, 1.0, B)
    assert list(np.nonzero(w3[0, 0, i])[0]) == [0, 1, 5]

