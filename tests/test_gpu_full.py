"""GPU parity at the full benchmark sizes, on sampled outputs.

The kernels run on whole requests shaped like the benchmarked workloads, through the same
calls and workspaces the benchmark makes; the fp64 oracle evaluates sampled queries (and
sampled decode sequences) from the same seeded inputs. Inputs are drawn on the GPU by the
seeded generator; the oracle receives CPU copies of just the rows it reads.

Every attention case runs at two input scales: "model" draws Q and the KV rows at
N(0,1)/sqrt(c) as the workloads do (near-uniform softmax, |O| ~ 1e-3..1e-2), and "unit"
draws them at N(0,1) (logits of std 1, |O| ~ 0.1), where a wrong row set, a dropped block or
a zeroed output moves O far beyond the tolerance. Both are also held to the norm-wise bf16
bound (max |diff| <= 1e-2 * max |oracle|), and the observed errors are printed.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from parity_util import assert_close, check_topk_query, sample_positions
from workloads import DECODE_BATCH, Generator, preset

pytestmark = pytest.mark.gpu


class _Rows:
    """Q-like accessor over the sampled queries' rows, copied from the device."""

    def __init__(self, Q, positions):
        self.shape = tuple(Q.shape)
        self.rows = {p: Q[p].float().cpu() for p in positions}

    def __getitem__(self, key):
        return self.rows[key]


def _compare(Og, Lg, Or, Lr, positions, what):
    bi = tuple(torch.tensor(positions).T.to(Og.device))
    assert_close(Og[bi].float().cpu(), Or, "bf16", what + " O", verbose=True)
    assert_close(Lg[bi].float().cpu(), Lr, "bf16", what + " LSE", verbose=True)


SCALES = {"model": None, "unit": 1.0}


def _std(scale, c):
    return 1 / math.sqrt(c) if SCALES[scale] is None else SCALES[scale]


@pytest.mark.parametrize("scale", list(SCALES))
def test_attn_hca_prefill_full_sampled(dsv4, scale):
    """V4-Flash HCA layer prefill: B=2, n=65536, H=64, c=512, m'=128 dense + w=128."""
    s = preset("flash_hca_prefill")
    B, n, H, c, m, w = s.B, s.n, s.H, s.c, s.m, s.w
    g = Generator(41, device="cuda")
    std = _std(scale, c)
    rows = [n // m + 1] * B
    offs = np.concatenate([[0], np.cumsum(rows)[:-1]]).astype(np.int64)
    Q = g.normal("Q", (B, n, H, c), std, torch.bfloat16)
    pool = g.normal("pool", (int(sum(rows)), c), std, torch.bfloat16)
    local = g.normal("local", (B, n, c), std, torch.bfloat16)
    pos0 = [0] * B
    Og, Lg = dsv4.dsv4_hybrid_sparse_attn(Q, pool, torch.from_numpy(offs).cuda(), None, None, local,
                                          torch.zeros(B, dtype=torch.int32, device="cuda"), m, w,
                                          None, 1 / math.sqrt(c))
    dsv4.dsv4_check_errors()
    positions = [(b, t) for b in range(B)
                 for t in sample_positions(n, m, extra=[127, 128, 129, 4095, 65535], count=6, seed=b)]
    Or, Lr = O.hybrid_attention(_Rows(Q, positions), pool.cpu(), offs, None, None, local.cpu(),
                                pos0, w, None, 1 / math.sqrt(c), dense_m=m, queries=positions)
    _compare(Og, Lg, Or, Lr, positions, f"hca prefill full ({scale})")
    del Q, pool, local, Og, Lg


@pytest.mark.parametrize("scale", list(SCALES))
def test_attn_pro_prefill_full_sampled(dsv4, scale):
    """V4-Pro CSA layer prefill attention: n=131072, H=128 (two head groups), k=1024, w=128,
    random valid index sets over the completed entries."""
    s = preset("pro_csa_prefill")
    n, H, c, m, w, k = s.n, s.H, s.c, s.m, s.w, s.k
    g = Generator(43, device="cuda")
    std = _std(scale, c)
    E = n // m
    Q = g.normal("Q", (1, n, H, c), std, torch.bfloat16)
    pool = g.normal("pool", (E + 1, c), std, torch.bfloat16)
    local = g.normal("local", (1, n, c), std, torch.bfloat16)
    vis = (torch.arange(n, device="cuda") + 1) // m
    idx, counts = g.random_index_sets(vis, k)
    idx, counts = idx.reshape(1, n, k), counts.reshape(1, n)
    Og, Lg = dsv4.dsv4_hybrid_sparse_attn(Q, pool, torch.zeros(1, dtype=torch.int64, device="cuda"), idx,
                                          counts, local, torch.zeros(1, dtype=torch.int32, device="cuda"),
                                          m, w, None, 1 / math.sqrt(c))
    dsv4.dsv4_check_errors()
    positions = [(0, t) for t in sample_positions(n, m, extra=[4 * 1024 - 1, 4 * 1024, 131071], count=12)]
    idx_c = {p: idx[p].cpu() for p in positions}
    cnt_c = {p: counts[p].cpu() for p in positions}

    class _Sel:
        def __getitem__(self, key):
            return idx_c[key]

    class _Cnt:
        def __getitem__(self, key):
            return cnt_c[key]

    Or, Lr = O.hybrid_attention(_Rows(Q, positions), pool.cpu(), [0], _Sel(), _Cnt(), local.cpu(), [0], w,
                                None, 1 / math.sqrt(c), queries=positions)
    _compare(Og, Lg, Or, Lr, positions, f"pro prefill full ({scale})")
    del Q, pool, local, Og, Lg


def _decode_batch():
    """The batched-decode workload: 64 sequences, seeded context lengths in [131072, 1048576]."""
    D = DECODE_BATCH
    L = torch.randint(D["L_lo"], D["L_hi"] + 1, (D["B"],), generator=torch.Generator().manual_seed(47))
    return D, L


def test_decode_index_topk_full_sampled(dsv4):
    """Decode indexer top-k over all completed entries (131k-1M contexts, k=512), through the
    workspace path the benchmark uses; sampled sequences against the fp64 scores."""
    D, L = _decode_batch()
    B, k, HI, cI, m = D["B"], D["k"], D["H_I"], D["c_I"], D["m_csa"]
    E = (L // m).tolist()
    offs = np.concatenate([[0], np.cumsum(E)[:-1]]).astype(np.int64)
    g = Generator(48, device="cuda")
    shape = preset("flash_csa_prefill", B=B)
    KI = g.index_keys(shape, int(sum(E)) + 1)
    qI, w = g.index_queries(shape, 1)
    pos0 = (L - 1).to(torch.int32)
    maxE = max(E)
    ws = torch.empty(dsv4.dsv4_index_topk_workspace_size(B, 1, maxE, k), dtype=torch.uint8, device="cuda")
    idx, counts = dsv4.dsv4_index_topk(qI, w, KI, torch.from_numpy(offs).cuda(), pos0.cuda(), m, k, maxE,
                                       workspace=ws)
    dsv4.dsv4_check_errors()
    idx, counts = idx.cpu().numpy(), counts.cpu().numpy()
    order = np.argsort(E)
    for b in (int(order[0]), int(order[len(order) // 2]), int(order[-1])):
        t = int(pos0[b])
        KIb = O.as_f64(KI[int(offs[b]):int(offs[b]) + E[b]].cpu())
        s64 = O.index_scores_query(qI[b, 0].cpu(), w[b, 0].cpu(), KIb, t, m)
        check_topk_query(idx[b, 0], counts[b, 0], s64, k, what=f"decode index b={b} L={int(L[b])}")


@pytest.mark.parametrize("scale", list(SCALES))
@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_decode_attention_full_sampled(dsv4, kind, scale):
    """Decode attention of the CSA (k + w rows) and HCA (dense + w rows) layers at the batch
    shape, with the split-list workspace the benchmark passes; sampled sequences."""
    D, L = _decode_batch()
    B, H, c, k, w = D["B"], D["H"], D["c"], D["k"], D["w"]
    m = D["m_csa"] if kind == "csa" else D["m_hca"]
    E = (L // m).tolist()
    offs = np.concatenate([[0], np.cumsum(E)[:-1]]).astype(np.int64)
    g = Generator(49, device="cuda")
    std = _std(scale, c)
    pool = g.normal("pool", (int(sum(E)) + 1, c), std, torch.bfloat16)
    Q = g.normal("Q", (B, 1, H, c), std, torch.bfloat16)
    local = g.normal("local", (B, w, c), std, torch.bfloat16)
    sink = g.normal("sink", (H,), 1.0) if kind == "csa" else None
    pos0 = (L - 1).to(torch.int32)
    if kind == "csa":
        idx, counts = g.random_index_sets(torch.tensor(E), k)
        idx, counts = idx.reshape(B, 1, k), counts.reshape(B, 1)
    else:
        idx = counts = None
    aws = torch.empty(max(1, dsv4.dsv4_hybrid_sparse_attn_workspace_size(B, 1, H, c)), dtype=torch.uint8,
                      device="cuda")
    Og, Lg = dsv4.dsv4_hybrid_sparse_attn(Q, pool, torch.from_numpy(offs).cuda(), idx, counts, local,
                                          pos0.cuda(), m, w, sink, 1 / math.sqrt(c), workspace=aws)
    dsv4.dsv4_check_errors()
    order = np.argsort(E)
    for b in (int(order[0]), int(order[len(order) // 2]), int(order[-1])):
        # the oracle reads this sequence's pool rows and local ring only
        pool_b = pool[int(offs[b]):int(offs[b]) + E[b] + 1].cpu()
        Or, Lr = O.hybrid_attention(
            _Rows(Q[b:b + 1], [(0, 0)]), pool_b, [0],
            None if idx is None else idx[b:b + 1].cpu().numpy(),
            None if counts is None else counts[b:b + 1].cpu().numpy(),
            local[b:b + 1].cpu(), [int(pos0[b])], w, None if sink is None else sink.cpu(),
            1 / math.sqrt(c), dense_m=m if kind == "hca" else 0, queries=[(0, 0)])
        assert_close(Og[b, 0].float().cpu(), Or[0], "bf16", f"decode {kind} ({scale}) b={b} O",
                     verbose=True)
        assert_close(Lg[b, 0].float().cpu(), Lr[0], "bf16", f"decode {kind} ({scale}) b={b} LSE",
                     verbose=True)


def test_index_pro_fp4_full_sampled(dsv4):
    """V4-Pro indexer at full size: 131072 queries over up to 32768 entries, k=1024, FP4
    operands. The device quantises q^I and K^I with dsv4_quantize_fp4 and scores them through
    the benchmark's call and workspace; the oracle quantises the same bf16 rows with its own
    quantiser and scores the dequantised values in fp64 for sampled queries."""
    s = preset("pro_csa_prefill")
    n, m, k, HI, cI = s.n, s.m, s.k, s.H_I, s.c_I
    E = n // m
    g = Generator(51, device="cuda")
    qI, w = g.index_queries(s, n)
    KI = g.index_keys(s, E)
    qc, qs = dsv4.dsv4_quantize_fp4(qI.reshape(-1, cI))
    kc, ks = dsv4.dsv4_quantize_fp4(KI)
    ws = torch.empty(dsv4.dsv4_index_topk_workspace_size_ex(dsv4.FP4, 1, n, HI, cI, E, k, E),
                     dtype=torch.uint8, device="cuda")
    zero64 = torch.zeros(1, dtype=torch.int64, device="cuda")
    zero32 = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx, counts = dsv4.dsv4_index_topk(qc.view(1, n, HI, cI // 2), w, kc, zero64, zero32, m, k, E,
                                       qI_scales=qs, KI_scales=ks, c_I=cI, workspace=ws)
    dsv4.dsv4_check_errors()
    idx, counts = idx.cpu().numpy(), counts.cpu().numpy()
    kc64, ks64 = O.quantize_fp4(KI.float().cpu())
    KI64 = O.dequantize_fp4(kc64, ks64, cI)
    for t in sample_positions(n, m, extra=[4 * k - 1, 4 * k, 4 * 16384 + 3, n - 1], count=4):
        qct, qst = O.quantize_fp4(qI[0, t].float().cpu())
        q64 = O.dequantize_fp4(qct, qst, cI)
        s64 = O.index_scores_query(q64, w[0, t].cpu(), KI64, t, m)
        check_topk_query(idx[0, t], counts[0, t], s64, k, what=f"pro fp4 index t={t}")
