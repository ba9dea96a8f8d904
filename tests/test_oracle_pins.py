"""Pins of the fp64 oracle against what the pages and mathematics fix (CPU only).

Each test checks the oracle against something other than itself: a table printed on
"CSA And HCA: Definition, State, And Cost Model" (tests/golden), a closed form, an
invariant, a special case that reduces to a library routine (numpy mean / matmul,
torch scaled_dot_product_attention, scipy logsumexp, torch float8 conversion), or
brute force on tiny inputs. They are chosen so that a plausible slip in the oracle
(a dropped term, an off-by-one in a block or window, a swapped stream, a wrong sign)
fails at least one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    out = []
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        out.append([f.strip() for f in line.split("|")])
    return out


def _ints(field):
    return [] if field == "-" else [int(v) for v in field.split(",")]


def _rng(seed):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------------------- visibility


def test_visibility_table_worked_example():
    """Section 6 table: completed CSA (m=4) / HCA (m'=8) entries and local tokens (w=3)."""
    rows = _rows("visibility_m4_m8_w3.txt")
    assert len(rows) == 6
    for t, csa, hca, loc in rows:
        t = int(t)
        assert list(range(O.completed_entries(t, 4))) == _ints(csa), t
        assert list(range(O.completed_entries(t, 8))) == _ints(hca), t
        assert list(O.local_window(t, 3)) == _ints(loc), t


def test_cost_model_counts():
    """Section 8.1 figures: budget crossover, 83.9M FLOPs/query, HCA entry count at 1M."""
    kv = {r[0].split()[0]: float(r[0].split()[1]) for r in _rows("cost_model_flash.txt")}
    m, k, w, H, c = 4, 512, 128, 64, 512
    L = int(kv["csa_full_budget_L"])
    assert O.completed_entries(L - 1, m) == k          # query t = L-1 has exactly k entries
    assert O.completed_entries(L - 2, m) < k
    # candidate list length at a long context equals k + w, giving the printed FLOPs
    rng = _rng(0)
    t = 100_000
    E = O.completed_entries(t, m)
    pool = rng.standard_normal((E, 8))
    local = rng.standard_normal((t + 1, 8))
    idx = rng.permutation(E)[:k]
    A = O.candidates(pool, idx, k, local, t + 1, t, w)
    assert A.shape[0] == k + w
    assert round(4 * H * c * A.shape[0] / 1e6, 1) == kv["main_flops_per_query_millions"]
    assert O.completed_entries(1048575, 128) == int(kv["hca_entries_at_1M"])
    Lx = int(kv["hca_window_crossover_L"])
    assert O.completed_entries(Lx - 1, 128) == w


# ----------------------------------------------------------------------------- compressor


def _compress_inputs(rng, B, n, c, m, S):
    C = rng.standard_normal((B, n, S * c))
    Z = rng.standard_normal((B, n, S * c))
    bias = 0.1 * rng.standard_normal((S, m, c))
    return C, Z, bias


def _changed_entries(base, pert):
    return sorted(set(np.nonzero(np.abs(base - pert).max(axis=(0, 2)) > 0)[0].tolist()))


@pytest.mark.parametrize("field", ["C", "Z"])
def test_overlap_diagram_dependencies(field):
    """Section 2.1 diagram: entry i pools a(block i) and b(block i-1); nothing else."""
    rng = _rng(1)
    m, c, n = 4, 6, 12
    C, Z, bias = _compress_inputs(rng, 1, n, c, m, 2)
    base = O.compress(C, Z, bias, m, overlap=True)
    expect_a, expect_b = {}, {}
    for e, a_tok, b_tok in _rows("overlap_diagram_m4.txt"):
        for tok in _ints(a_tok):
            expect_a.setdefault(tok, []).append(int(e))
        for tok in _ints(b_tok):
            expect_b.setdefault(tok, []).append(int(e))
    for tok in range(n):
        for half, expect in ((0, expect_a), (1, expect_b)):
            X = (C if field == "C" else Z).copy()
            X[0, tok, half * c:(half + 1) * c] += 0.5
            pert = O.compress(X, Z, bias, m, True) if field == "C" else \
                O.compress(C, X, bias, m, True)
            assert _changed_entries(base, pert) == sorted(expect.get(tok, [])), (tok, half)


def test_first_entry_ignores_stream_b():
    """i = 0: the nonexistent preceding block has zero weight (section 2.1)."""
    rng = _rng(2)
    C, Z, bias = _compress_inputs(rng, 2, 16, 5, 4, 2)
    base = O.compress(C, Z, bias, 4, True)
    C2, Z2, b2 = C.copy(), Z.copy(), bias.copy()
    C2[:, :, 5:] = 1e3 * rng.standard_normal(C2[:, :, 5:].shape)
    Z2[:, :, 5:] = 50.0
    b2[1] += 7.0
    out = O.compress(C2, Z2, b2, 4, True)
    np.testing.assert_array_equal(out[:, 0], base[:, 0])
    # and entry 0 is exactly the one-stream (HCA-form) pool of block 0 from stream a
    hca0 = O.compress(C[:, :4, :5], Z[:, :4, :5], bias[:1], 4, False)
    np.testing.assert_allclose(out[:, 0], hca0[:, 0], rtol=0, atol=1e-15)


@pytest.mark.parametrize("overlap,m", [(True, 4), (False, 16), (False, 128)])
def test_weights_sum_to_one(overlap, m):
    """Feature-wise softmax over positions: a constant entry stream pools to itself."""
    rng = _rng(3)
    c, n = 7, 3 * m + 1
    S = 2 if overlap else 1
    _, Z, bias = _compress_inputs(rng, 2, n, c, m, S)
    v = rng.standard_normal(c)
    C = np.tile(np.concatenate([v] * S), (2, n, 1))
    out = O.compress(C, 3 * Z, 10 * bias, m, overlap)
    np.testing.assert_allclose(out, np.broadcast_to(v, out.shape), rtol=0, atol=1e-13)


@pytest.mark.parametrize("overlap,m", [(True, 4), (False, 8)])
def test_uniform_gates_give_block_mean(overlap, m):
    """Constant gate logits and zero bias reduce to plain average pooling (numpy mean)."""
    rng = _rng(4)
    B, c, n = 2, 5, 5 * m + 2
    S = 2 if overlap else 1
    C = rng.standard_normal((B, n, S * c))
    Z = np.full((B, n, S * c), 0.37)
    bias = np.zeros((S, m, c))
    out = O.compress(C, Z, bias, m, overlap)
    E = n // m
    assert out.shape == (B, E, c)
    for i in range(E):
        parts = [C[:, m * i:m * (i + 1), :c]]
        if overlap and i > 0:
            parts.append(C[:, m * (i - 1):m * i, c:])
        ref = np.mean(np.concatenate(parts, axis=1), axis=1)
        np.testing.assert_allclose(out[:, i], ref, rtol=0, atol=1e-14)


def test_dominant_bias_selects_position():
    """A huge positional bias at offset p turns the pool into a gather of token m*i+p."""
    rng = _rng(5)
    m, c, n = 4, 6, 16
    C, Z, bias = _compress_inputs(rng, 1, n, c, m, 2)
    p = 2
    bias[0, p, :] += 200.0
    out = O.compress(C, Z, bias, m, True)
    for i in range(n // m):
        np.testing.assert_allclose(out[0, i], C[0, m * i + p, :c], rtol=0, atol=1e-12)
    # the same bias on stream b selects token m*(i-1)+p of the b half for i > 0
    bias2 = 0.1 * rng.standard_normal((2, m, c))
    bias2[1, p, :] += 200.0
    out2 = O.compress(C, Z, bias2, m, True)
    for i in range(1, n // m):
        np.testing.assert_allclose(out2[0, i], C[0, m * (i - 1) + p, c:], rtol=0, atol=1e-12)


def test_incomplete_trailing_block_never_pooled():
    """floor(n/m) entries; tokens after the last full block change nothing (section 7)."""
    rng = _rng(6)
    m, c, n = 4, 3, 4 * 5 + 3
    C, Z, bias = _compress_inputs(rng, 1, n, c, m, 2)
    out = O.compress(C, Z, bias, m, True)
    assert out.shape[1] == 5
    C[:, 20:] = 1e6
    Z[:, 20:] = 1e3
    np.testing.assert_array_equal(O.compress(C, Z, bias, m, True), out)


def test_channels_independent():
    """Permuting channels of C, Z and the bias permutes the output channels."""
    rng = _rng(7)
    m, c, n = 4, 9, 12
    C, Z, bias = _compress_inputs(rng, 1, n, c, m, 2)
    perm = rng.permutation(c)
    full = np.concatenate([perm, perm + c])
    out = O.compress(C, Z, bias, m, True)
    outp = O.compress(C[:, :, full], Z[:, :, full], bias[:, :, perm], m, True)
    np.testing.assert_allclose(outp, out[:, :, perm], rtol=0, atol=1e-15)


# ----------------------------------------------------------------------------- indexer


def test_index_score_single_head_is_dot_product():
    """n_h^I = 1, w = 1 and positive dot products: I = K q (a matrix-vector product)."""
    rng = _rng(8)
    c_I, m, t = 16, 4, 39
    E = O.completed_entries(t, m)
    q = np.abs(rng.standard_normal((1, c_I)))
    K = np.abs(rng.standard_normal((E + 3, c_I)))
    s = O.index_scores_query(q, np.ones(1), K, t, m)
    assert s.shape == (E,)
    np.testing.assert_allclose(s, K[:E] @ q[0], rtol=1e-13)


def test_index_score_relu_and_linearity():
    """ReLU per head before the weight; linear in w; a one-hot w picks one head."""
    rng = _rng(9)
    H, c_I, m, t = 5, 8, 4, 30
    E = O.completed_entries(t, m)
    q = rng.standard_normal((H, c_I))
    K = rng.standard_normal((E, c_I))
    w1, w2 = rng.random(H), rng.random(H)
    s1 = O.index_scores_query(q, w1, K, t, m)
    s2 = O.index_scores_query(q, w2, K, t, m)
    np.testing.assert_allclose(O.index_scores_query(q, w1 + w2, K, t, m), s1 + s2, rtol=1e-13)
    for h in range(H):
        oh = np.zeros(H)
        oh[h] = 1.0
        d = K @ q[h]
        np.testing.assert_allclose(O.index_scores_query(q, oh, K, t, m), np.where(d > 0, d, 0.0),
                                   rtol=1e-13, atol=1e-15)
    # flipping the sign of a head's query moves mass from the positive to the negative dots
    qn = q.copy()
    qn[0] = -qn[0]
    oh = np.zeros(H)
    oh[0] = 1.0
    a = O.index_scores_query(q, oh, K, t, m)
    b = O.index_scores_query(qn, oh, K, t, m)
    np.testing.assert_allclose(a - b, K @ q[0], rtol=1e-13, atol=1e-15)


def test_index_score_negative_weight_worked_example():
    """The weight multiplies the ReLU of the dot product (it is not inside it): with
    q_0 = (1, 0), q_1 = (0, 1), K_0 = (2, -3), w = (-0.5, 1):
    I_0 = -0.5 * ReLU(2) + 1 * ReLU(-3) = -1."""
    q = np.array([[1.0, 0.0], [0.0, 1.0]])
    K = np.array([[2.0, -3.0]])
    assert O.index_scores_query(q, np.array([-0.5, 1.0]), K, 3, 4).tolist() == [-1.0]


def test_stacked_sequences_read_their_own_rows():
    """Pools and index keys of several sequences stacked row-wise: sequence b reads from
    row kv_row_off[b], so each sequence's result equals the one-sequence call on its own
    rows (and differs from reading sequence 0's rows)."""
    rng = _rng(73)
    H, c, m, w, HI, cI, k, nq = 2, 6, 4, 3, 2, 5, 3, 9
    E = [7, 5]
    off = [0, 7]
    pool = rng.standard_normal((sum(E) + 1, c))
    KI = rng.standard_normal((sum(E) + 1, cI))
    Q = rng.standard_normal((2, nq, H, c))
    local = rng.standard_normal((2, nq, c))
    qI = rng.standard_normal((2, nq, HI, cI))
    wI = rng.random((2, nq, HI))
    pos0 = [4 * E[0] - nq, 4 * E[1] - nq]
    o2, l2 = O.hybrid_attention(Q, pool, off, None, None, local, pos0, w, dense_m=m)
    idx2, cnt2 = O.index_topk(qI, wI, KI, off, pos0, m, k)
    for b in range(2):
        ob, lb = O.hybrid_attention(Q[b:b + 1], pool[off[b]:], [0], None, None, local[b:b + 1],
                                    [pos0[b]], w, dense_m=m)
        np.testing.assert_array_equal(o2[b], ob[0])
        np.testing.assert_array_equal(l2[b], lb[0])
        ib, cb = O.index_topk(qI[b:b + 1], wI[b:b + 1], KI[off[b]:], [0], [pos0[b]], m, k)
        np.testing.assert_array_equal(idx2[b], ib[0])
        np.testing.assert_array_equal(cnt2[b], cb[0])
    o0, _ = O.hybrid_attention(Q[1:2], pool, [0], None, None, local[1:2], [pos0[1]], w, dense_m=m)
    assert not np.allclose(o0[0], o2[1])


def test_index_scores_only_completed_entries():
    rng = _rng(10)
    q = rng.standard_normal((2, 4))
    K = rng.standard_normal((50, 4))
    for t in range(0, 40):
        assert O.index_scores_query(q, np.ones(2), K, t, 4).shape == ((t + 1) // 4,)


@pytest.mark.parametrize("E,k", [(0, 3), (1, 3), (5, 2), (6, 6), (7, 3), (8, 0), (4, 9)])
def test_topk_brute_force(E, k):
    """TopK = the subset of size min(k,E) whose worst member beats every non-member."""
    rng = _rng(11 + E * 10 + k)
    s = np.round(rng.standard_normal(E), 1)             # rounding creates ties
    idx, cnt = O.topk_select(s, k)
    k_eff = min(k, E)
    assert cnt == k_eff and idx.shape == (k,)
    assert (idx[k_eff:] == -1).all()
    chosen = idx[:k_eff].tolist()
    best = None
    for sub in itertools.combinations(range(E), k_eff):
        # lexicographically best subset under (score desc, index asc)
        key = sorted(((-s[j], j) for j in sub))
        if best is None or key < best[0]:
            best = (key, sub)
    assert sorted(chosen) == sorted(best[1])
    # the set is listed in ascending entry order
    assert chosen == sorted(chosen)


def test_topk_ties_prefer_lower_index():
    """Equal scores across the k-th place: the lower entries are taken."""
    s = np.array([1.0, 3.0, 3.0, 2.0, 3.0, 0.5])
    idx, cnt = O.topk_select(s, 4)
    assert idx.tolist() == [1, 2, 3, 4] and cnt == 4
    s = np.array([1.0, 3.0, 2.0, 3.0, 2.0, 0.5, 2.0])     # three 2.0s compete for one place
    idx, cnt = O.topk_select(s, 3)
    assert idx.tolist() == [1, 2, 3] and cnt == 3
    idx, cnt = O.topk_select(np.full(9, 0.25), 4)          # all tied
    assert idx.tolist() == [0, 1, 2, 3] and cnt == 4


def test_index_topk_brute_force_tiny():
    """End-to-end indexer on a tiny case: scores by pure-python loops, ranks by brute force."""
    rng = _rng(12)
    B, nq, H, cI, m, k = 1, 14, 2, 3, 2, 3
    qI = rng.standard_normal((B, nq, H, cI))
    w = rng.random((B, nq, H))
    KI = rng.standard_normal((7, cI))
    idx, counts = O.index_topk(qI, w, KI, [0], [0], m, k)
    for t in range(nq):
        E = (t + 1) // m
        sc = []
        for s in range(E):
            tot = 0.0
            for h in range(H):
                d = sum(qI[0, t, h, j] * KI[s, j] for j in range(cI))
                tot += w[0, t, h] * max(d, 0.0)
            sc.append(tot)
        want = sorted(range(E), key=lambda j: (-sc[j], j))[:k]
        assert counts[0, t] == min(k, E)
        assert idx[0, t, :counts[0, t]].tolist() == sorted(want)


# ----------------------------------------------------------------------------- attention


def _sdpa(q, kv, mask, scale):
    """torch scaled_dot_product_attention in fp64 with a boolean keep-mask."""
    qt = torch.from_numpy(q)
    kt = torch.from_numpy(kv)
    mt = torch.from_numpy(mask)
    return torch.nn.functional.scaled_dot_product_attention(
        qt, kt, kt, attn_mask=mt, scale=scale).numpy()


def test_hca_dense_read_equals_masked_sdpa():
    """HCA = one softmax over [all completed entries ; window] == masked SDPA (library)."""
    rng = _rng(13)
    B, n, H, c, m, w = 1, 70, 3, 8, 8, 5
    C, Z, bias = _compress_inputs(rng, B, n, c, m, 1)
    Q = rng.standard_normal((B, n, H, c))
    local = rng.standard_normal((B, n, c))
    res = O.hca_prefill_layer(C, Z, bias, Q, local, m, w)
    pool = res["pool"][0]
    E = pool.shape[0]
    kv = np.concatenate([pool, local[0]], axis=0)          # [E + n, c]
    mask = np.zeros((n, E + n), dtype=bool)
    for t in range(n):
        mask[t, :(t + 1) // m] = True
        mask[t, E + max(0, t - w + 1):E + t + 1] = True
    scale = 1 / math.sqrt(c)
    for h in range(H):
        ref = _sdpa(Q[0, :, h, :], kv, mask, scale)
        np.testing.assert_allclose(res["O"][0, :, h, :], ref, rtol=1e-12, atol=1e-12)


def test_csa_full_budget_equals_dense_read():
    """CSA with k >= |E_t| selects everything: equal to the dense read at ratio m."""
    rng = _rng(14)
    B, n, H, c, m, w = 1, 40, 2, 6, 4, 3
    Q = rng.standard_normal((B, n, H, c))
    pool = rng.standard_normal((n // m, c))
    local = rng.standard_normal((B, n, c))
    idx = np.full((B, n, 16), -1)
    counts = np.zeros((B, n), dtype=np.int64)
    for t in range(n):
        E = (t + 1) // m
        idx[0, t, :E] = rng.permutation(E)
        counts[0, t] = E
    o1, l1 = O.hybrid_attention(Q, pool, [0], idx, counts, local, [0], w)
    o2, l2 = O.hybrid_attention(Q, pool, [0], None, None, local, [0], w, dense_m=m)
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=1e-13, atol=1e-14)


def test_k_zero_is_sliding_window_attention():
    """k = 0: output is causal sliding-window attention over the local stream (SDPA)."""
    rng = _rng(15)
    B, n, H, c, w = 1, 33, 2, 8, 6
    Q = rng.standard_normal((B, n, H, c))
    local = rng.standard_normal((B, n, c))
    idx = np.zeros((B, n, 0), dtype=np.int64)
    counts = np.zeros((B, n), dtype=np.int64)
    o, _ = O.hybrid_attention(Q, np.zeros((1, c)), [0], idx, counts, local, [0], w)
    mask = np.zeros((n, n), dtype=bool)
    for t in range(n):
        mask[t, max(0, t - w + 1):t + 1] = True
    for h in range(H):
        ref = _sdpa(Q[0, :, h], local[0], mask, 1 / math.sqrt(c))
        np.testing.assert_allclose(o[0, :, h], ref, rtol=1e-12, atol=1e-13)


def test_gathered_and_scatter_mask_forms_agree():
    """[S, S*top_k] gathered-row mask == [S, compressed_len] scatter mask (transformers PR)."""
    rng = _rng(16)
    S, E, k, c, H = 12, 9, 3, 5, 2
    Q = rng.standard_normal((1, S, H, c))
    pool = rng.standard_normal((E, c))
    local = rng.standard_normal((1, S, c))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(S)])        # [S, k]
    scale = 0.7
    # gathered form: keys = pool[idx] for every query laid side by side, mask picks own block
    gathered = pool[idx.reshape(-1)]                                    # [S*k, c]
    mask_g = np.zeros((S, S * k), dtype=bool)
    for t in range(S):
        mask_g[t, t * k:(t + 1) * k] = True
    # scatter form: keys = the pool, mask marks each query's selected columns
    mask_s = np.zeros((S, E), dtype=bool)
    for t in range(S):
        mask_s[t, idx[t]] = True
    o_oracle, _ = O.hybrid_attention(Q, pool, [0], idx[None], np.full((1, S), k), local, [0],
                                     w=0, scale=scale)
    for h in range(H):
        a = _sdpa(Q[0, :, h], gathered, mask_g, scale)
        b = _sdpa(Q[0, :, h], pool, mask_s, scale)
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(o_oracle[0, :, h], a, rtol=1e-12, atol=1e-14)


def test_sink_limits_and_closed_form():
    """Sink: -inf is no sink; +large drives the output to 0; constant rows have a closed form."""
    rng = _rng(17)
    H, c, N = 3, 6, 7
    q = rng.standard_normal((H, c))
    cand = rng.standard_normal((N, c))
    o0, l0 = O.attend_query(q, cand, None)
    o1, l1 = O.attend_query(q, cand, np.full(H, -np.inf))
    np.testing.assert_array_equal(o0, o1)
    np.testing.assert_array_equal(l0, l1)
    o2, _ = O.attend_query(q, cand, np.full(H, 80.0))
    assert np.abs(o2).max() < 1e-25
    # constant candidate rows v: all logits equal z0 = scale q.v
    v = rng.standard_normal(c)
    sink = rng.standard_normal(H)
    scale = 0.3
    o3, l3 = O.attend_query(q, np.tile(v, (N, 1)), sink, scale)
    z0 = scale * (q @ v)
    frac = N * np.exp(z0) / (N * np.exp(z0) + np.exp(sink))
    np.testing.assert_allclose(o3, frac[:, None] * v[None, :], rtol=1e-13)
    np.testing.assert_allclose(l3, np.log(N * np.exp(z0) + np.exp(sink)), rtol=1e-13)


def test_lse_is_logsumexp():
    rng = _rng(18)
    H, c, N = 4, 5, 11
    q = 3 * rng.standard_normal((H, c))
    cand = rng.standard_normal((N, c))
    sink = rng.standard_normal(H)
    _, l = O.attend_query(q, cand, sink, 0.9)
    z = 0.9 * q @ cand.T
    np.testing.assert_allclose(l, logsumexp(np.concatenate([z, sink[:, None]], 1), axis=1),
                               rtol=1e-14)


def test_single_candidate_returns_that_row():
    rng = _rng(19)
    q = rng.standard_normal((2, 4))
    row = rng.standard_normal((1, 4))
    o, l = O.attend_query(q, row, None, 1.0)
    np.testing.assert_allclose(o, np.tile(row, (2, 1)), rtol=0, atol=1e-15)
    np.testing.assert_allclose(l, q @ row[0], rtol=1e-15)


def test_decode_ring_slots_and_position_offset():
    """Decode: query at t = q_pos0 + i reads local slot j mod R; equals prefill at t."""
    rng = _rng(20)
    n, H, c, m, w = 50, 2, 4, 4, 6
    Q = rng.standard_normal((1, n, H, c))
    local = rng.standard_normal((1, n, c))
    pool = rng.standard_normal((n // m + 2, c))
    o_pre, l_pre = O.hybrid_attention(Q, pool, [0], None, None, local, [0], w, dense_m=m)
    t = 45
    R = w
    ring = np.zeros((1, R, c))
    for j in range(t - w + 1, t + 1):
        ring[0, j % R] = local[0, j]
    o_dec, l_dec = O.hybrid_attention(Q[:, t:t + 1], pool, [0], None, None, ring, [t], w,
                                      dense_m=m)
    np.testing.assert_allclose(o_dec[0, 0], o_pre[0, t], rtol=1e-14)
    np.testing.assert_allclose(l_dec[0, 0], l_pre[0, t], rtol=1e-14)


def test_window_only_for_queries_before_first_entry():
    """Queries t < m - 1 have no completed entry: window-only attention."""
    rng = _rng(21)
    n, H, c, m, w = 6, 2, 4, 4, 8
    Q = rng.standard_normal((1, n, H, c))
    local = rng.standard_normal((1, n, c))
    pool = rng.standard_normal((1, c))
    o, _ = O.hybrid_attention(Q, pool, [0], None, None, local, [0], w, dense_m=m)
    for t in range(m - 1):
        ref, _ = O.attend_query(Q[0, t], local[0, :t + 1])
        np.testing.assert_allclose(o[0, t], ref, rtol=1e-15)


# ----------------------------------------------------------------------------- RMSNorm / RoPE


def test_rms_norm_closed_form_and_scale_invariance():
    """RMSNorm output has mean square 1 (up to eps) and ignores a positive scale of its input;
    a constant row a maps to a / sqrt(a^2 + eps)."""
    rng = _rng(80)
    x = rng.standard_normal((4, 512))
    y = O.rms_norm(x, eps=0.0)
    np.testing.assert_allclose((y * y).mean(axis=-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(O.rms_norm(7.5 * x, eps=0.0), y, rtol=1e-13)
    np.testing.assert_allclose(O.rms_norm(np.full((1, 8), 3.0), eps=1e-6), 3.0 / np.sqrt(9.0 + 1e-6),
                               rtol=1e-15)


def test_rope_rotation_properties():
    """rho_p is a rotation of the last 64 channels only: norm preserving, rho_a o rho_b =
    rho_(a+b), its inverse undoes it; in each pair the 2-D rotation by p * base^(-2i/64) maps
    (1, 0) to (cos, sin) of that angle."""
    rng = _rng(81)
    x = rng.standard_normal((3, 512))
    y = O.rope_rotate(x, [3, 40, 1000])
    np.testing.assert_array_equal(y[:, :448], x[:, :448])
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-14)
    np.testing.assert_allclose(O.rope_rotate(O.rope_rotate(x, [3, 40, 1000]), [4, 2, 17]),
                               O.rope_rotate(x, [7, 42, 1017]), rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(O.rope_rotate(y, [3, 40, 1000], inverse=True), x, rtol=1e-12, atol=1e-12)
    e = np.zeros((1, 64))
    e[0, 2 * 5] = 1.0                                        # pair i = 5
    r = O.rope_rotate(e, [9])
    ang = 9 * 10000.0 ** (-2 * 5 / 64)
    np.testing.assert_allclose(r[0, 10:12], [np.cos(ang), np.sin(ang)], rtol=1e-14)
    assert np.count_nonzero(r) == 2


def test_rope_logits_and_output_depend_on_relative_positions():
    """[CSA-DEF] s5.2: q at t against entry j at p_j gives a logit that depends on t - p_j
    only, and the inverse rotation at t puts the output in relative form: shifting the
    query and every entry position by the same amount changes neither the output nor the
    LSE; without the inverse rotation the output would carry the absolute rotation."""
    rng = _rng(82)
    H, c, N, t = 3, 128, 9, 50
    q = rng.standard_normal((H, c))
    ent = rng.standard_normal((N, c))
    pos = np.array([0, 4, 8, 12, 46, 47, 48, 49, 50])          # compressed (m*s) then local
    o1, l1 = O.attend_query_rope(q, t, ent, pos)
    o2, l2 = O.attend_query_rope(q, t + 777, ent, pos + 777)
    np.testing.assert_allclose(o1, o2, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=1e-12)
    # the same attention weights as plain attention over the rotated, normalised inputs
    qn = O.rope_rotate(O.rms_norm(q), np.full(H, t))
    kv = O.rope_rotate(O.rms_norm(ent), pos)
    o_abs, l_abs = O.attend_query(qn, kv)
    np.testing.assert_allclose(l1, l_abs, rtol=1e-14)
    np.testing.assert_allclose(o1[:, :c - 64], o_abs[:, :c - 64], rtol=1e-13)
    assert not np.allclose(o1[:, c - 64:], o_abs[:, c - 64:])


# ----------------------------------------------------------------------------- decode state


@pytest.mark.parametrize("overlap,m,n", [(True, 4, 37), (True, 1, 5), (False, 16, 50), (False, 3, 11)])
def test_decode_state_machine_reproduces_the_compressor(overlap, m, n):
    """[CSA-DEF] s7: feeding tokens one at a time through the bounded tail emits, at
    exactly the tokens whose t + 1 is a multiple of m, the entries the s2.1/s2.2
    compressor pools from the whole stream (a trailing partial block emits nothing)."""
    rng = _rng(40 + m)
    S, c = (2 if overlap else 1), 5
    C = rng.standard_normal((1, n, S * c))
    Z = rng.standard_normal((1, n, S * c))
    bias = 0.1 * rng.standard_normal((S, m, c))
    want = O.compress(C, Z, bias, m, overlap)[0]
    tail = np.zeros((O.tail_slots(m, overlap), 2, S * c))
    got = {}
    for t in range(n):
        e = O.decode_append(tail, C[0, t], Z[0, t], bias, t, m, overlap)
        if e is not None:
            got[t] = e
    assert sorted(got) == [m * (i + 1) - 1 for i in range(n // m)]
    for t, e in got.items():
        np.testing.assert_allclose(e, want[(t + 1) // m - 1], rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("overlap,m", [(True, 4), (False, 8)])
def test_decode_tail_restored_from_a_prefix(overlap, m):
    """An incomplete prefix tail restored from the prefix's last T positions (slot p mod T)
    continues exactly like the uninterrupted stream; the state is T rows whatever n is."""
    rng = _rng(50 + m)
    S, c, n0, n = (2 if overlap else 1), 3, 4 * m + 2, 7 * m + 1
    C = rng.standard_normal((1, n, S * c))
    Z = rng.standard_normal((1, n, S * c))
    bias = 0.1 * rng.standard_normal((S, m, c))
    want = O.compress(C, Z, bias, m, overlap)[0]
    T = O.tail_slots(m, overlap)
    tail = np.full((T, 2, S * c), np.nan)              # anything not restored must not be read
    for p in range(n0 - T, n0):
        tail[p % T, 0], tail[p % T, 1] = C[0, p], Z[0, p]
    for t in range(n0, n):
        e = O.decode_append(tail, C[0, t], Z[0, t], bias, t, m, overlap)
        assert (e is not None) == ((t + 1) % m == 0)
        if e is not None:
            np.testing.assert_allclose(e, want[(t + 1) // m - 1], rtol=1e-13, atol=1e-15)
    assert tail.shape[0] == T


def test_ring_write_keeps_the_window():
    """s7 step 1 into an R-slot ring (R >= w): after token t the ring holds tokens
    t-R+1..t, so the window read through slots j mod R returns tokens max(0,t-w+1)..t."""
    rng = _rng(60)
    n, c, w, R = 23, 4, 5, 7
    kv = rng.standard_normal((n, c))
    ring = np.zeros((R, c))
    for t in range(n):
        O.ring_write(ring, kv[t], t)
        win = O.local_window(t, w)
        np.testing.assert_array_equal(ring[win % R], kv[win])
        held = np.arange(max(0, t - R + 1), t + 1)
        np.testing.assert_array_equal(ring[held % R], kv[held])


# ----------------------------------------------------------------------------- FP4


def test_e2m1_table():
    """OCP microscaling e2m1: 0, 0.5, 1, 1.5, 2, 3, 4, 6."""
    assert O.e2m1_values().tolist() == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e4m3_table_landmarks():
    t = O.e4m3_values()
    assert t[0x7E] == 448.0 and t[0x38] == 1.0 and t[0x01] == 2.0 ** -9
    assert t[0x08] == 2.0 ** -6 and t[0x07] == 7 * 2.0 ** -9
    assert np.all(np.diff(t) > 0)
    # matches torch's float8_e4m3fn decode of every finite non-negative byte
    b = torch.arange(0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn)
    np.testing.assert_array_equal(b.to(torch.float64).numpy(), t)


def test_e4m3_rounding_matches_torch():
    """RNE to E4M3 (in range) agrees with torch's float8_e4m3fn cast on many values."""
    rng = _rng(22)
    v = np.concatenate([
        np.exp(rng.uniform(np.log(2.0 ** -12), np.log(440.0), 20000)),
        O.e4m3_values()[:-1] + np.diff(O.e4m3_values()) / 2,      # exact midpoints
    ]).astype(np.float32)
    ours = O.round_to_table(v.astype(np.float64), O.e4m3_values())
    theirs = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, theirs.astype(np.int64))


# ----------------------------------------------------------------------------- main-KV FP8 entry


def test_main_kv_and_index_key_payloads_reproduce_state_table():
    """Entry payloads taken from the oracle's formats (FP8 codes + bf16 RoPE channels of a
    512-channel main entry; FP4 codes of a 128-channel index key) reproduce the pages'
    persistent-state table and the 736-byte amortised write."""
    rng = _rng(70)
    codes, scales, rope = O.quantize_main_kv_fp8(rng.standard_normal((1, 512)))
    main_b = codes.shape[1] * 1 + rope.shape[1] * 2                  # payload, no scales
    assert main_b == O.main_kv_payload_bytes(512, 64) == 576
    kcodes, _ = O.quantize_fp4(rng.standard_normal((1, 128)))
    index_b = kcodes.shape[1]
    assert index_b == 64
    mib = float(1 << 20)
    rows = [r for r in _rows("state_payload_flash.txt") if len(r) == 6]
    assert len(rows) == 4
    for L, E, main, index, local, total in rows:
        L, E = int(L), int(E)
        assert E == O.completed_entries(L - 1, 4)
        got = (E * main_b / mib, E * index_b / mib, 128 * main_b / mib)
        got = got + (sum(got),)
        for g, want in zip(got, (main, index, local, total)):
            assert round(g, 3) == float(want), (L, g, want)
    (write,) = [r for r in _rows("state_payload_flash.txt") if r[0] == "write_bytes_per_token_layer"]
    assert main_b + (main_b + index_b) / 4 == int(write[1])


def test_main_kv_fp8_rounding_matches_torch_and_layout():
    """FP8 codes are torch's float8_e4m3fn cast of the fp32 quotients x / scale, scale =
    amax / 448 per 64 channels; the last 64 channels are torch's bf16 rounding of x."""
    rng = _rng(71)
    x = (rng.standard_normal((6, 512)) * np.exp(rng.uniform(-8, 8, (6, 1)))).astype(np.float32)
    x[0, :64] = 0.0                                                    # an all-zero group
    x[0, 1:64:2] = -0.0                                                # (with negative zeros)
    x[1, 3] = x[2, 100] = -0.0                                         # -0 in nonzero groups: 0x80
    codes, scales, rope = O.quantize_main_kv_fp8(x)
    assert codes.shape == (6, 448) and scales.shape == (6, 7) and rope.shape == (6, 64)
    assert scales[0, 0] == 0 and (codes[0, :64] == 0).all()            # zero scale: codes 0
    g = x[:, :448].reshape(6, 7, 64)
    want_scale = (np.abs(g).max(axis=-1) / np.float32(448.0)).astype(np.float32)
    np.testing.assert_array_equal(scales, want_scale)
    q = (g / np.where(want_scale > 0, want_scale, 1)[..., None]).astype(np.float32).reshape(6, 448)
    theirs = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    nz = np.repeat(want_scale > 0, 64, axis=1)
    np.testing.assert_array_equal(codes[nz], theirs[nz])
    assert codes[1, 3] == 0x80 and codes[2, 100] == 0x80
    np.testing.assert_array_equal(rope, torch.from_numpy(x[:, 448:]).to(torch.bfloat16).double().numpy())


def test_main_kv_fp8_round_trip_and_error_bound():
    """Entries built from E4M3 values times a power-of-two scale (the group maximum 448)
    come back exactly; random entries come back within half an E4M3 step (2^-4 relative,
    2^-10 scale below the normal range); a negative value that rounds to zero keeps its
    sign bit."""
    rng = _rng(72)
    t4 = O.e4m3_values()
    code = rng.integers(0, 0x7F, (5, 448))
    code[:, ::64] = 0x7E                                             # 448 in every group
    sign = rng.integers(0, 2, (5, 448))
    sc = 2.0 ** rng.integers(-20, 5, (5, 7))
    x = np.where(sign, -1, 1) * t4[code] * np.repeat(sc, 64, axis=1)
    rope = torch.randn(5, 64).to(torch.bfloat16).double().numpy()
    xe = np.concatenate([x, rope], axis=1)
    c2, s2, r2 = O.quantize_main_kv_fp8(xe)
    np.testing.assert_array_equal(O.dequantize_main_kv_fp8(c2, s2, r2), xe)
    y = rng.standard_normal((8, 512)) * 3.0
    y[1, 5] = -1e-12                                                  # underflows in its group
    c3, s3, r3 = O.quantize_main_kv_fp8(y)
    d = O.dequantize_main_kv_fp8(c3, s3, r3)
    s_el = np.repeat(s3.astype(np.float64), 64, axis=1)
    err = np.abs(d[:, :448] - y[:, :448])
    assert (err <= 2.0 ** -4 * np.abs(y[:, :448]) * (1 + 1e-6) + 2.0 ** -10 * s_el * (1 + 1e-6)).all()
    assert c3[1, 5] == 0x80


def test_e2m1_rounding_ties_and_saturation():
    v = np.array([0.0, 0.24, 0.25, 0.26, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 5.01, 6.0, 7.0, 1e9])
    want = [0.0, 0.0, 0.0, 0.5, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, 6.0, 6.0, 6.0]
    got = O.e2m1_values()[O.round_to_table(v, O.e2m1_values())]
    assert got.tolist() == want


def test_fp4_roundtrip_of_representable_values():
    """Values that are e2m1 grid points times an E4M3 scale with amax = 6*scale survive."""
    rng = _rng(23)
    rows = 64
    grid = O.e2m1_values()
    scales = O.e4m3_values()[rng.integers(20, 120, size=(rows, 2))]
    mags = grid[rng.integers(0, 8, size=(rows, 32))]
    mags[:, 0] = 6.0
    mags[:, 16] = 6.0
    sgn = np.where(rng.random((rows, 32)) < 0.5, -1.0, 1.0)
    x = sgn * mags * np.repeat(scales, 16, axis=1)
    codes, sb = O.quantize_fp4(x.astype(np.float32))
    np.testing.assert_array_equal(O.e4m3_values()[sb], scales)
    np.testing.assert_array_equal(O.dequantize_fp4(codes, sb, 32), x)


def test_fp4_error_bound_and_layout():
    """|x - dq(q(x))| <= half the local e2m1 spacing times the scale (plus saturation)."""
    rng = _rng(24)
    x = (rng.standard_normal((40, 64)) / 8).astype(np.float32)
    x[3, :16] = 0.0                                   # all-zero group -> zero scale
    codes, sb = O.quantize_fp4(x)
    assert codes.shape == (40, 32) and sb.shape == (40, 4)
    assert (sb[3, 0] == 0) and (codes[3, :8] == 0).all()
    dq = O.dequantize_fp4(codes, sb, 64)
    s = np.repeat(O.e4m3_values()[sb], 16, axis=1)
    ratio = np.abs(x.astype(np.float64)) / np.where(s > 0, s, 1)
    half_gap = np.where(ratio < 2, 0.25, np.where(ratio < 4, 0.5, 1.0))
    sat = np.maximum(ratio - 6.0, 0)
    assert np.all(np.abs(dq - x) <= (half_gap + sat) * s + 1e-12)
    # nibble order: element 2j is the low nibble of byte j
    one = np.zeros((1, 16), dtype=np.float32)
    one[0, 0], one[0, 1] = 6.0, -3.0                  # scale 1.0, codes 0x7 and 0x8|0x5
    c1, s1 = O.quantize_fp4(one)
    assert s1[0, 0] == 0x38 and c1[0, 0] == (0x7 | (0xD << 4))


def test_fp4_negative_underflow_keeps_sign():
    x = np.zeros((1, 16), dtype=np.float32)
    x[0, 0] = 6.0
    x[0, 1] = -0.2                                   # -0.2 rounds to -0
    c, s = O.quantize_fp4(x)
    assert c[0, 0] == (0x7 | (0x8 << 4))


# ----------------------------------------------------------------------------- the layer chain


def _csa_layer_inputs(rng, B, n, H, c, cI, HI, m):
    C, Z, bias = _compress_inputs(rng, B, n, c, m, 2)
    CI, ZI, biasI = _compress_inputs(rng, B, n, cI, m, 2)
    qI = rng.standard_normal((B, n, HI, cI))
    w = rng.random((B, n, HI))
    Q = rng.standard_normal((B, n, H, c))
    local = rng.standard_normal((B, n, c))
    return dict(C=C, Z=Z, bias=bias, CI=CI, ZI=ZI, biasI=biasI, qI=qI, w=w, Q=Q, local=local)


def _layer(inp, m, k, wwin, **kw):
    return O.csa_prefill_layer(inp["C"], inp["Z"], inp["bias"], inp["CI"], inp["ZI"], inp["biasI"],
                               inp["qI"], inp["w"], inp["Q"], inp["local"], m, k, wwin, **kw)


def test_csa_layer_full_budget_equals_masked_sdpa():
    """Sections 3-5.1: with k >= floor(n/m) TopK keeps every completed entry, so the layer's
    output is one softmax over [all entries s < floor((t+1)/m) ; window] -- masked SDPA
    (library) over the layer's own pool and the local stream, for every sequence."""
    rng = _rng(31)
    B, n, H, c, m, wwin = 2, 45, 3, 8, 4, 6
    inp = _csa_layer_inputs(rng, B, n, H, c, c, 2, m)
    res = _layer(inp, m, n // m + 3, wwin)
    E = n // m
    scale = 1 / math.sqrt(c)
    for b in range(B):
        assert (res["counts"][b] == [(t + 1) // m for t in range(n)]).all()
        kv = np.concatenate([res["pool"][b], inp["local"][b]], axis=0)
        mask = np.zeros((n, E + n), dtype=bool)
        for t in range(n):
            mask[t, :(t + 1) // m] = True
            mask[t, E + max(0, t - wwin + 1):E + t + 1] = True
        for h in range(H):
            ref = _sdpa(inp["Q"][b, :, h], kv, mask, scale)
            np.testing.assert_allclose(res["O"][b, :, h], ref, rtol=1e-11, atol=1e-12)


def test_csa_layer_indexer_reads_only_its_own_stream():
    """Section 3.1: the indexer scores separate index keys K^I (a second compressor instance
    over its own stream), not the main entries. Changing the main stream C leaves every
    selection unchanged and changes the output; changing stream b of the index stream in
    block 0 (pooled only into index key 1, by the overlap of section 2.1) changes some
    selection. Main and index widths are equal here, so feeding the main pool to the indexer
    would run and be caught by value."""
    rng = _rng(32)
    B, n, H, c, m, k, wwin = 2, 64, 2, 8, 4, 3, 5
    inp = _csa_layer_inputs(rng, B, n, H, c, c, 2, m)
    base = _layer(inp, m, k, wwin)
    pert = dict(inp, C=inp["C"] + 3.0 * rng.standard_normal(inp["C"].shape))
    r1 = _layer(pert, m, k, wwin)
    np.testing.assert_array_equal(r1["idx"], base["idx"])
    assert np.abs(r1["O"] - base["O"]).max() > 1e-3
    CI = inp["CI"].copy()
    CI[:, :m, c:] = 5.0 + 5.0 * rng.standard_normal(CI[:, :m, c:].shape)
    r2 = _layer(dict(inp, CI=CI), m, k, wwin)
    changed = np.nonzero((r2["idx"] != base["idx"]).any(axis=-1))
    assert len(changed[0]) > 0
    # only queries that can see index key 1 (t >= 2m - 1) may change
    assert changed[1].min() >= 2 * m - 1


def _fp4_grid_rows(rng, rows, cols, exp):
    """Rows whose 16-element groups are e2m1 grid points times 2^exp with one element at 6
    (so amax / 6 = 2^exp is the exact E4M3 scale and quantisation is the identity)."""
    grid = O.e2m1_values()
    mags = grid[rng.integers(0, 8, size=(rows, cols))]
    mags[:, ::16] = 6.0
    sgn = np.where(rng.random((rows, cols)) < 0.5, -1.0, 1.0)
    return sgn * mags * 2.0 ** exp


def test_csa_layer_fp4_is_exact_on_representable_operands():
    """Section 8 precision table (indexer in FP4): quantisation is the identity on operands
    that are already FP4 values with exact E4M3 block scales, so the FP4 layer selects what
    the unquantised layer selects. The index keys are made representable by constant blocks:
    every position pooled into key i carries the same row, and softmax weights sum to one."""
    rng = _rng(33)
    B, n, H, c, cI, HI, m, k, wwin = 1, 48, 2, 8, 32, 3, 4, 3, 4
    inp = _csa_layer_inputs(rng, B, n, H, c, cI, HI, m)
    E = n // m
    u = _fp4_grid_rows(rng, E + 1, cI, -3)                 # key i = row u[i]
    CI = np.empty((B, n, 2 * cI))
    for j in range(E):
        CI[0, m * j:m * (j + 1), :cI] = u[j]               # stream a of block j -> key j
        CI[0, m * j:m * (j + 1), cI:] = u[j + 1]           # stream b of block j -> key j + 1
    qI = _fp4_grid_rows(rng, B * n * HI, cI, -2).reshape(B, n, HI, cI)
    inp = dict(inp, CI=CI, qI=qI)
    r32 = _layer(inp, m, k, wwin)
    r4 = _layer(inp, m, k, wwin, index_fp4=True)
    np.testing.assert_allclose(r32["KI"][0], u[:E], rtol=1e-15, atol=0)
    np.testing.assert_array_equal(r4["KI"][0], u[:E])
    np.testing.assert_array_equal(r4["idx"], r32["idx"])
    np.testing.assert_allclose(r4["O"], r32["O"], rtol=1e-13, atol=1e-14)


def test_csa_layer_fp4_scores_the_quantised_operands():
    """The FP4 layer's selection is the TopK (brute force here) of the scores of the
    quantise -> dequantise images of both q^I and K^I; the quantiser and the compressor
    are pinned on their own above, so this pins how the layer wires them."""
    rng = _rng(34)
    B, n, H, c, cI, HI, m, k, wwin = 1, 40, 2, 8, 32, 3, 4, 4, 4
    inp = _csa_layer_inputs(rng, B, n, H, c, cI, HI, m)
    res = _layer(inp, m, k, wwin, index_fp4=True)
    KI = O.compress(inp["CI"], inp["ZI"], inp["biasI"], m, True)[0]
    kc, ks = O.quantize_fp4(KI)
    K4 = O.dequantize_fp4(kc, ks, cI)
    qc, qs = O.quantize_fp4(inp["qI"].reshape(-1, cI))
    q4 = O.dequantize_fp4(qc, qs, cI).reshape(n, HI, cI)
    differs = 0
    for t in range(n):
        E = (t + 1) // m
        sc = [sum(inp["w"][0, t, h] * max(float(q4[t, h] @ K4[s]), 0.0) for h in range(HI))
              for s in range(E)]
        want = sorted(sorted(range(E), key=lambda j: (-sc[j], j))[:k])
        assert res["idx"][0, t, :res["counts"][0, t]].tolist() == want, t
        sc32 = [sum(inp["w"][0, t, h] * max(float(inp["qI"][0, t, h] @ KI[s]), 0.0)
                    for h in range(HI)) for s in range(E)]
        differs += int(sorted(sorted(range(E), key=lambda j: (-sc32[j], j))[:k]) != want)
    # the quantisation is visible: some query selects differently than unquantised scores
    assert differs > 0
