"""GPU parity: dsv4_index_topk (indexer scores + per-query TopK) against the fp64 oracle.

Stage-isolated: q^I, w and K^I come from the seeded generator (FP4 operands are
quantised by the oracle), so both sides score the same bytes.
"""
import numpy as np
import pytest
import torch

import oracle as O
from parity_util import check_topk_query, sample_positions
from workloads import Generator, preset

pytestmark = pytest.mark.gpu


def _inputs(shape, nq, rows, seed):
    g = Generator(seed)
    qI, w = g.index_queries(shape, nq)
    KI = g.index_keys(shape, rows)
    return qI, w, KI


def _score_bound(qI64, w64, KI64, t, m):
    """Worst-case fp32 accumulation bound per entry: 2e-5 * sum_h |w_h| sum_d |q_hd k_sd|."""
    E = (t + 1) // m
    mag = np.abs(qI64) @ np.abs(KI64[:E]).T            # [H_I, E]
    return 2e-5 * (np.abs(w64) @ mag) + 1e-30


def _run_and_check(dsv4, qI, w, KI, offs, pos0, m, k, positions, qI_sc=None, KI_sc=None,
                   qI64=None, KI64=None, c_I=None, what=""):
    B, nq = w.shape[:2]
    max_e = max((int(p0) + nq) // m for p0 in pos0)
    scores = torch.full((B, nq, max(max_e, 1)), float("nan"), device="cuda")
    idx, counts = dsv4.dsv4_index_topk(
        qI.cuda(), w.cuda(), KI.cuda(), torch.tensor(offs, dtype=torch.int64).cuda(),
        torch.tensor(pos0, dtype=torch.int32).cuda(), m, k, max_e,
        qI_scales=None if qI_sc is None else qI_sc.cuda(),
        KI_scales=None if KI_sc is None else KI_sc.cuda(), c_I=c_I, scores_out=scores)
    # the same request through the workspace path must give identical indices
    idx2, counts2 = dsv4.dsv4_index_topk(
        qI.cuda(), w.cuda(), KI.cuda(), torch.tensor(offs, dtype=torch.int64).cuda(),
        torch.tensor(pos0, dtype=torch.int32).cuda(), m, k, max_e,
        qI_scales=None if qI_sc is None else qI_sc.cuda(),
        KI_scales=None if KI_sc is None else KI_sc.cuda(), c_I=c_I)
    dsv4.dsv4_check_errors()
    assert torch.equal(idx, idx2) and torch.equal(counts, counts2)
    idx, counts, scores = idx.cpu().numpy(), counts.cpu().numpy(), scores.cpu().numpy()
    qI64 = O.as_f64(qI) if qI64 is None else qI64
    KI64 = O.as_f64(KI) if KI64 is None else KI64
    w64 = O.as_f64(w)
    ties = 0
    for b, i in positions:
        t = int(pos0[b]) + i
        s64 = O.index_scores_query(qI64[b, i], w64[b, i], KI64[offs[b]:], t, m)
        bound = _score_bound(qI64[b, i], w64[b, i], KI64[offs[b]:], t, m)
        ties += check_topk_query(idx[b, i], counts[b, i], s64, k, scores[b, i], bound,
                                 f"{what} b={b} t={t}")
    return ties


def test_index_tiny_fp32(dsv4):
    shape = preset("tiny_csa")
    qI, w, KI = _inputs(shape, shape.n, shape.n // shape.m, 0)
    pos = [(0, i) for i in range(shape.n)]
    _run_and_check(dsv4, qI, w, KI, [0], [0], shape.m, shape.k, pos, what="tiny")


@pytest.fixture(params=["tensor_cores", "cuda_cores"])
def index_path(request, monkeypatch):
    """Run a case on the tcgen05 score kernel (bf16, H_I=64, c_I=128) and the CUDA-core one."""
    monkeypatch.setenv("DSV4_FORCE_SIMT", "1" if request.param == "cuda_cores" else "0")
    return request.param


@pytest.mark.parametrize("n,k,HI,cI", [(300, 8, 4, 32), (523, 64, 8, 64), (97, 200, 2, 16),
                                       (4 * 300 + 3, 128, 64, 128), (4 * 5000 + 2, 300, 64, 128),
                                       (7, 4, 64, 128)])
def test_index_ragged_bf16(dsv4, index_path, n, k, HI, cI):
    shape = preset("flash_csa_prefill", n=n, k=k, H_I=HI, c_I=cI)
    qI, w, KI = _inputs(shape, n, n // 4, n + k)
    if n <= 2000:
        pos = [(0, i) for i in range(n)]
    else:
        pos = [(0, t) for t in sample_positions(n, 4, extra=[4 * 4096 - 1, 4 * 4096, 4 * k])]
    _run_and_check(dsv4, qI, w, KI, [0], [0], 4, k, pos, what=f"{index_path} n={n} k={k}")


@pytest.mark.parametrize("n,k,HI,cI", [(4 * 600 + 1, 64, 64, 128), (523, 16, 8, 64)])
def test_index_mixed_sign_weights(dsv4, index_path, n, k, HI, cI):
    """Head weights of both signs (the score is a weighted sum of per-head ReLUs, so it can
    be negative): the selection still follows the fp64 scores."""
    shape = preset("flash_csa_prefill", n=n, k=k, H_I=HI, c_I=cI)
    qI, w, KI = _inputs(shape, n, n // 4, 5 * n + k)
    w = 2.0 * w - 1.0
    pos = [(0, t) for t in sample_positions(n, 4, extra=[4 * k - 1, 4 * k, n - 1], count=64)]
    _run_and_check(dsv4, qI, w, KI, [0], [0], 4, k, pos, what=f"{index_path} mixed-sign n={n}")


def test_index_mixed_sign_weights_long_rows(dsv4):
    """Decode rows longer than 16384 entries (the threshold top-k) with head weights of
    both signs: negative scores pass through the key transform and the histograms."""
    shape = preset("flash_csa_prefill", B=2)
    lens = [4 * 20000 + 3, 4 * 17000]
    rows = [L // 4 for L in lens]
    offs = list(np.concatenate([[0], np.cumsum(rows)[:-1]]).astype(np.int64))
    g = Generator(33)
    qI, w = g.index_queries(shape, 1)
    w = 2.0 * w - 1.0
    KI = g.index_keys(shape, int(sum(rows)) + 1)
    pos0 = [L - 1 for L in lens]
    _run_and_check(dsv4, qI, w, KI, offs, pos0, 4, 512, [(0, 0), (1, 0)], what="mixed-sign long")


def test_index_batched_offsets_decode_like(dsv4, index_path):
    """Several sequences stacked in one key pool, one query each at the sequence end."""
    shape = preset("flash_csa_prefill", B=5)
    lens = [7, 130, 2048 + 3, 4097, 1]
    rows = [L // 4 for L in lens]
    offs = list(np.concatenate([[0], np.cumsum(rows)[:-1]]).astype(np.int64))
    g = Generator(9)
    qI, w = g.index_queries(shape, 1)
    KI = g.index_keys(shape, int(sum(rows)) + 1)
    pos0 = [L - 1 for L in lens]
    _run_and_check(dsv4, qI, w, KI, offs, pos0, 4, 512, [(b, 0) for b in range(5)],
                   what="decode-like")


def test_index_long_rows_radix_path(dsv4):
    """Rows far longer than k (radix select) with many exact ties (quantised keys)."""
    shape = preset("flash_csa_prefill", H_I=4, c_I=16)
    g = Generator(11)
    E = 20000
    KI = (g.normal("KI", (E + 1, 16), 1.0) * 2).round().clamp(-3, 3).to(torch.bfloat16)
    qI = (g.normal("qI", (1, 2, 4, 16), 1.0)).round().to(torch.bfloat16)
    w = torch.ones(1, 2, 4)
    pos0 = [4 * E - 2]
    _run_and_check(dsv4, qI, w, KI, [0], pos0, 4, 1000, [(0, 0), (0, 1)], what="radix ties")


@pytest.mark.parametrize("kind", ["few_values", "all_equal", "mostly_zero"])
def test_index_short_rows_ties(dsv4, kind):
    """Rows of at most 2048 entries (the select that keeps each thread's keys in registers and
    stops its radix passes once a bin is taken whole) whose scores take a few distinct values,
    a single value, or are zero for most entries (ReLU of negative dot products) with the k-th
    place among the zeros. Integer-valued operands keep every score exact on both sides."""
    g = Generator(13)
    E = 1800
    qI = (g.normal("qI", (1, 3, 4, 16), 1.0)).round().to(torch.bfloat16)
    if kind == "few_values":
        KI = (g.normal("KI", (E + 1, 16), 1.0) * 2).round().clamp(-3, 3).to(torch.bfloat16)
    elif kind == "all_equal":
        KI = torch.ones(E + 1, 16).to(torch.bfloat16)
    else:
        qI = qI.abs()
        KI = -(g.normal("KI", (E + 1, 16), 1.0).abs() * 2).round().clamp(1, 3)
        KI[::17] = -KI[::17]                       # about 106 entries with positive scores
        KI = KI.to(torch.bfloat16)
    w = torch.ones(1, 3, 4)
    pos0 = [4 * E - 3]                             # E_t = E - 1, E - 1, E
    _run_and_check(dsv4, qI, w, KI, [0], pos0, 4, 300, [(0, 0), (0, 1), (0, 2)],
                   what=f"short-row {kind}")


def test_index_decode_long_contexts(dsv4):
    """Decode over long contexts: one query per sequence, rows of 17.5k-75k entries (the
    workspace path: histograms of the top 16 key bits, a filter pass, then a select among
    the boundary candidates)."""
    shape = preset("flash_csa_prefill", B=3)
    lens = [300001, 131075, 70003]
    rows = [L // 4 for L in lens]
    offs = list(np.concatenate([[0], np.cumsum(rows)[:-1]]).astype(np.int64))
    g = Generator(21)
    qI, w = g.index_queries(shape, 1)
    KI = g.index_keys(shape, int(sum(rows)) + 1)
    pos0 = [L - 1 for L in lens]
    _run_and_check(dsv4, qI, w, KI, offs, pos0, 4, 512, [(b, 0) for b in range(3)],
                   what="decode long")


def test_index_decode_mixed_lengths_dynamic_units(dsv4):
    """Decode batch with rows from no entries to ~50k: the score kernel's persistent CTAs draw
    (row, 4096-entry chunk) units from a counter over the rows' dense unit list, so empty rows,
    rows shorter than one chunk, exact multiples of a chunk and ragged last chunks all occur."""
    rng = np.random.default_rng(5)
    lens = [1, 3, 4, 7, 4 * 4096, 4 * 4096 + 3, 4 * 4097, 4 * 8192 + 2] + \
        [int(x) for x in rng.integers(8, 4 * 50000, 16)]
    shape = preset("flash_csa_prefill", B=len(lens))
    rows = [L // 4 for L in lens]
    offs = list(np.concatenate([[0], np.cumsum(rows)[:-1]]).astype(np.int64))
    g = Generator(41)
    qI, w = g.index_queries(shape, 1)
    KI = g.index_keys(shape, int(sum(rows)) + 1)
    pos0 = [L - 1 for L in lens]
    _run_and_check(dsv4, qI, w, KI, offs, pos0, 4, 512, [(b, 0) for b in range(len(lens))],
                   what="decode mixed")


def test_index_decode_concentrated_scores_two_levels(dsv4):
    """Long decode rows whose scores all lie within a few per cent of each other: the bin of
    the top 11 key bits holding the k-th largest score holds nearly the whole row, so the
    threshold takes the second histogram level (key bits 20..13)."""
    shape = preset("flash_csa_prefill", B=2)
    lens = [4 * 40000 + 1, 4 * 23000 + 2]
    rows = [L // 4 for L in lens]
    offs = list(np.concatenate([[0], np.cumsum(rows)[:-1]]).astype(np.int64))
    g = Generator(43)
    base = g.normal("base", (1, 128), 128 ** -0.5)
    KI = (base + 0.05 * g.normal("KI", (int(sum(rows)) + 1, 128), 128 ** -0.5)).to(torch.bfloat16)
    qI = (base.reshape(1, 1, 1, 128) + 0.05 * g.normal("qI", (2, 1, 64, 128), 128 ** -0.5))
    qI = qI.to(torch.bfloat16)
    w = g.uniform("wI", (2, 1, 64), 0.5, 1.0)
    pos0 = [L - 1 for L in lens]
    s64 = O.index_scores_query(O.as_f64(qI)[0, 0], O.as_f64(w)[0, 0], O.as_f64(KI), pos0[0], 4)
    top = np.sort(s64)[::-1]
    assert top[0] < 1.2 * top[-1]                      # one quarter-octave bin or two
    _run_and_check(dsv4, qI, w, KI, offs, pos0, 4, 512, [(0, 0), (1, 0)], what="concentrated")


def test_index_many_long_rows(dsv4):
    """More than 1024 queries whose rows exceed 16384 entries: the workspace path selects per
    16384-entry segment and merges the candidates (the threshold pipeline serves requests with
    few rows, as in decode)."""
    shape = preset("flash_csa_prefill", H_I=4, c_I=16)
    nq, E0 = 1100, 17000
    pos0 = [4 * E0]
    g = Generator(31)
    qI, w = g.index_queries(shape, nq)
    KI = g.index_keys(shape, (pos0[0] + nq) // 4 + 1)
    _run_and_check(dsv4, qI, w, KI, [0], pos0, 4, 256, [(0, i) for i in (0, 1, 547, 1099)],
                   what="many long rows")


def test_index_flash_full_sampled(dsv4, index_path):
    """V4-Flash shape: n=8192, H_I=64, c_I=128, k=512; every query run, a sample compared."""
    shape = preset("flash_csa_prefill")
    qI, w, KI = _inputs(shape, shape.n, shape.n // shape.m, 1)
    pos = [(0, t) for t in sample_positions(shape.n, 4, extra=[2046, 2047, 2048, 2051, 4095])]
    _run_and_check(dsv4, qI, w, KI, [0], [0], 4, 512, pos, what="flash")


def test_index_fp4(dsv4, index_path):
    """FP4 operands (e2m1 + E4M3 per 16): the oracle scores the same dequantised values. The
    tensor-core path scores an exact bf16 expansion; the CUDA-core path decodes per element."""
    shape = preset("pro_csa_prefill", n=4 * 700 + 1)
    n, E = shape.n, shape.n // 4
    qI, w, KI = _inputs(shape, n, E, 2)
    qc, qs = O.quantize_fp4(qI.float().reshape(-1, 128))
    kc, ks = O.quantize_fp4(KI.float())
    qI64 = O.dequantize_fp4(qc, qs, 128).reshape(1, n, 64, 128)
    KI64 = O.dequantize_fp4(kc, ks, 128)
    qc_t = torch.from_numpy(qc).reshape(1, n, 64, 64)
    pos = [(0, t) for t in sample_positions(n, 4, extra=[1023, 1024, 2799])]
    _run_and_check(dsv4, qc_t, w, torch.from_numpy(kc), [0], [0], 4, 256, pos,
                   qI_sc=torch.from_numpy(qs), KI_sc=torch.from_numpy(ks), qI64=qI64,
                   KI64=KI64, c_I=128, what=f"fp4 {index_path}")


def _fp4_decode_case(lens, seed, k, pad_front=0):
    """One query per sequence at its end; FP4 q^I and K^I (the oracle's quantiser), keys of
    sequence b from row pad_front + sum(rows before b) of one pool."""
    shape = preset("pro_csa_prefill", B=len(lens))
    rows = [L // 4 for L in lens]
    offs = list((pad_front + np.concatenate([[0], np.cumsum(rows)[:-1]])).astype(np.int64))
    total = pad_front + int(sum(rows))
    qI, w, KI = _inputs(shape, 1, total, seed)
    qc, qs = O.quantize_fp4(qI.float().reshape(-1, 128))
    kc, ks = O.quantize_fp4(KI.float())
    qI64 = O.dequantize_fp4(qc, qs, 128).reshape(len(lens), 1, 64, 128)
    KI64 = O.dequantize_fp4(kc, ks, 128)
    qc_t = torch.from_numpy(qc).reshape(len(lens), 1, 64, 64)
    return dict(qI=qc_t, w=w, KI=torch.from_numpy(kc), offs=offs, pos0=[L - 1 for L in lens],
                m=4, k=k, positions=[(b, 0) for b in range(len(lens))],
                qI_sc=torch.from_numpy(qs), KI_sc=torch.from_numpy(ks), qI64=qI64, KI64=KI64,
                c_I=128)


def test_index_fp4_decode_long_rows(dsv4):
    """FP4 decode over long rows: the score kernel reads e2m1 codes and E4M3 scales of the key
    pool and expands them itself (threshold top-k, dynamically scheduled units). The pool
    starts two rows in, so most sequences start at odd rows (scale pairs straddle their
    blocks), and has an odd row count (its last row's scales are read on their own)."""
    lens = [4 * 20001 + 3, 4 * 17000, 4 * 3000 + 1, 4 * 40000 + 2]
    case = _fp4_decode_case(lens, 51, 512, pad_front=2)
    assert case["KI"].shape[0] % 2 == 1 and sum(o % 2 for o in case["offs"]) >= 2
    _run_and_check(dsv4, what="fp4 decode long", **case)


def test_index_fp4_decode_short_rows(dsv4):
    """FP4 decode over rows shorter than the threshold top-k's (one CTA per unit), including
    a row of one entry and the pool's last row."""
    lens = [4 * 3 + 1, 4 * 129, 4 * 1000 + 2, 4 * 4097 + 3, 7]
    case = _fp4_decode_case(lens, 52, 256)
    _run_and_check(dsv4, what="fp4 decode short", **case)


def test_index_k_zero_and_short(dsv4):
    shape = preset("tiny_csa")
    qI, w, KI = _inputs(shape, 10, 2, 4)
    idx, counts = dsv4.dsv4_index_topk(qI.cuda(), w.cuda(), KI.cuda(),
                                       torch.zeros(1, dtype=torch.int64).cuda(),
                                       torch.zeros(1, dtype=torch.int32).cuda(), 4, 0, 2)
    assert idx.numel() == 0 and (counts.cpu() == 0).all()
