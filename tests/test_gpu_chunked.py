"""GPU parity of chunked prefill with a start position and of context-parallel prefill.

"CSA And HCA: Definition, State, And Cost Model", s1/s5.1 (what a query at position t sees)
and s11 (long prefill split into ranges); pypto-lib PR #834's "Performance" workload (128
tokens at start position 896) is the chunk shape used here, at V4-Flash widths.

* Attention of query chunks that start at q_pos0 > 0 (different per sequence) over a local
  ring of R >= w + nq - 1 slots, against the fp64 oracle.
* A CSA layer prefilled as a prefix [0, 896) and then a chunk [896, 1024) -- the chunk's
  compressor takes the one-block halo, its queries the window halo and the prefix's
  entries -- against the oracle's full prefill of all 1024 tokens for the chunk's queries.
* Context-parallel prefill emulated on one GPU: two ranks of 512 tokens each run the
  per-rank steps (halo compression, entries of both ranks gathered, index TopK and
  attention of the rank's own queries); every output equals single-pass prefill on the GPU
  bit for bit, for a CSA and an HCA layer. (The collectives themselves are covered by the
  gloo test on the CPU; this run has one GPU.)
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from compressed_sparse_mqa_dsv4_b200 import cp
from parity_util import assert_close, check_topk_query
from workloads import Generator, preset

pytestmark = pytest.mark.gpu


def test_attention_chunks_with_start_positions(dsv4):
    B, nq, H, c, m, w, k = 2, 128, 64, 512, 4, 128, 64
    pos0 = [896, 1001]
    R = 256                                            # >= w + nq - 1 = 255
    g = Generator(61)
    E = [(p + nq) // m for p in pos0]
    offs = np.concatenate([[0], np.cumsum([e + 1 for e in E])[:-1]]).astype(np.int64)
    Q = g.normal("Q", (B, nq, H, c), 1.0, torch.bfloat16)
    pool = g.normal("pool", (int(sum(E)) + B, c), 1.0, torch.bfloat16)
    local = g.normal("local", (B, R, c), 1.0, torch.bfloat16)
    sink = g.normal("sink", (H,), 1.0)
    vis = torch.tensor([[(p + i + 1) // m for i in range(nq)] for p in pos0]).reshape(-1)
    idx, counts = g.random_index_sets(vis, k)
    idx, counts = idx.reshape(B, nq, k), counts.reshape(B, nq)
    Og, Lg = dsv4.dsv4_hybrid_sparse_attn(Q.cuda(), pool.cuda(), torch.from_numpy(offs).cuda(), idx.cuda(),
                                          counts.cuda(), local.cuda(),
                                          torch.tensor(pos0, dtype=torch.int32).cuda(), m, w, sink.cuda(),
                                          1 / math.sqrt(c))
    dsv4.dsv4_check_errors()
    qs = [(b, i) for b in range(B) for i in (0, 1, 3, 64, 126, 127)]
    Or, Lr = O.hybrid_attention(Q, pool, offs, idx.numpy(), counts.numpy(), local, pos0, w, sink,
                                1 / math.sqrt(c), queries=qs)
    bi = tuple(np.array(qs).T)
    assert_close(Og.cpu()[bi], Or, "bf16", "chunk attention O", verbose=True)
    assert_close(Lg.cpu()[bi], Lr, "bf16", "chunk attention LSE", verbose=True)


def _flash_inputs(n, seed):
    s = preset("flash_csa_prefill", n=n, k=64)
    g = Generator(seed)
    C, Z, bias = g.compressor_inputs(s, "main")
    CI, ZI, biasI = g.compressor_inputs(s, "index")
    qI, w = g.index_queries(s)
    # unit-scale queries and local rows: logits of std ~1, so a wrong row set shows
    Q = g.normal("Qu", (1, n, s.H, s.c), 1.0, torch.bfloat16)
    local = g.normal("Lu", (1, n, s.c), 1.0, torch.bfloat16)
    sink = g.sink(s)
    return s, dict(C=C, Z=Z, bias=bias, CI=CI, ZI=ZI, biasI=biasI, qI=qI, w=w, Q=Q, local=local,
                   sink=sink)


def test_chunked_prefill_matches_full_prefill_oracle(dsv4):
    n, p0 = 1024, 896
    s, x = _flash_inputs(n, 62)
    d = {k_: (v.cuda() if v is not None else None) for k_, v in x.items()}
    m, k, wwin = s.m, s.k, s.w
    E = n // m
    # prefix [0, p0): the cache this chunk extends
    pool = torch.empty(1, E, s.c, dtype=torch.bfloat16, device="cuda")
    KI = torch.empty(1, E, s.c_I, dtype=torch.bfloat16, device="cuda")
    dsv4.dsv4_compress(d["C"][:, :p0].contiguous(), d["Z"][:, :p0].contiguous(), d["bias"], m, True,
                       out=pool[:, :p0 // m])
    dsv4.dsv4_compress(d["CI"][:, :p0].contiguous(), d["ZI"][:, :p0].contiguous(), d["biasI"], m, True,
                       out=KI[:, :p0 // m])
    # the chunk [p0, n): halo compression, then index top-k and attention from position p0
    sl = slice(p0, n)
    pool[:, p0 // m:] = cp.compress_range(d["C"][:, sl], d["Z"][:, sl], d["bias"], m, True, p0,
                                          d["C"][:, p0 - m:p0], d["Z"][:, p0 - m:p0])
    KI[:, p0 // m:] = cp.compress_range(d["CI"][:, sl], d["ZI"][:, sl], d["biasI"], m, True, p0,
                                        d["CI"][:, p0 - m:p0], d["ZI"][:, p0 - m:p0])
    Og, Lg, idx, cnt = cp.prefill_range(
        Q=d["Q"][:, sl].contiguous(), local=d["local"][:, sl].contiguous(), p0=p0, m=m, wwin=wwin,
        pool=pool.view(E, s.c), KI=KI.view(E, s.c_I), qI=d["qI"][:, sl].contiguous(),
        w=d["w"][:, sl].contiguous(), k=k, sink=d["sink"], local_halo=d["local"][:, :p0])
    dsv4.dsv4_check_errors()
    queries = [(0, t) for t in (896, 897, 899, 900, 960, 1000, 1022, 1023)]
    ref = O.csa_prefill_layer(x["C"], x["Z"], x["bias"], x["CI"], x["ZI"], x["biasI"], x["qI"], x["w"],
                              x["Q"], x["local"], m, k, wwin, sink=x["sink"], queries=queries)
    assert_close(pool, ref["pool"], "bf16", "pool (prefix + chunk)", verbose=True)
    assert_close(KI, ref["KI"], "bf16", "index keys (prefix + chunk)", verbose=True)
    # the GPU's own pools in fp64 give the scores its selection should follow
    KI64 = O.as_f64(KI[0].cpu())
    same = []
    for q_n, (_, t) in enumerate(queries):
        i = t - p0
        sc = O.index_scores_query(x["qI"][0, t], x["w"][0, t], KI64, t, m)
        check_topk_query(idx[0, i].cpu().numpy(), int(cnt[0, i]), sc, k, what=f"chunk t={t}")
        if set(idx[0, i, :int(cnt[0, i])].tolist()) == set(ref["idx"][0, t, :ref["counts"][0, t]].tolist()):
            same.append(q_n)
    assert len(same) >= len(queries) - 1
    rows = [queries[q][1] - p0 for q in same]
    assert_close(Og[0, rows].cpu(), ref["O"][same], "bf16", "chunk O vs full prefill", verbose=True)
    assert_close(Lg[0, rows].cpu(), ref["LSE"][same], "bf16", "chunk LSE vs full prefill", verbose=True)


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_context_parallel_emulated_equals_single_pass(dsv4, kind):
    n, W = 1024, 2
    if kind == "csa":
        s, x = _flash_inputs(n, 63)
    else:
        s = preset("flash_hca_prefill", B=1, n=n)
        g = Generator(64)
        C, Z, bias = g.compressor_inputs(s, "main")
        x = dict(C=C, Z=Z, bias=bias, Q=g.normal("Qu", (1, n, s.H, s.c), 1.0, torch.bfloat16),
                 local=g.normal("Lu", (1, n, s.c), 1.0, torch.bfloat16), sink=None)
    d = {k_: (v.cuda() if v is not None else None) for k_, v in x.items()}
    m, wwin, ov = s.m, s.w, kind == "csa"
    E = n // m
    # single pass
    pool1 = dsv4.dsv4_compress(d["C"], d["Z"], d["bias"], m, ov)
    KI1 = dsv4.dsv4_compress(d["CI"], d["ZI"], d["biasI"], m, True) if ov else None
    O1, L1, i1, c1 = cp.prefill_range(Q=d["Q"], local=d["local"], p0=0, m=m, wwin=wwin,
                                      pool=pool1.view(E, -1),
                                      KI=None if KI1 is None else KI1.view(E, -1),
                                      qI=d.get("qI"), w=d.get("w"), k=s.k, sink=d["sink"])
    # two ranks of n/W tokens: the per-rank steps of cp_prefill with the exchanges done by hand
    sh = n // W
    ents, kents = [], []
    for r in range(W):
        sl = slice(r * sh, (r + 1) * sh)
        halo = (d["C"][:, r * sh - m:r * sh], d["Z"][:, r * sh - m:r * sh]) if r else (None, None)
        ents.append(cp.compress_range(d["C"][:, sl], d["Z"][:, sl], d["bias"], m, ov, r * sh, *halo))
        if ov:
            hI = (d["CI"][:, r * sh - m:r * sh], d["ZI"][:, r * sh - m:r * sh]) if r else (None, None)
            kents.append(cp.compress_range(d["CI"][:, sl], d["ZI"][:, sl], d["biasI"], m, True, r * sh, *hI))
    pool = torch.cat(ents, dim=1)                       # the all-gather of cp_prefill
    KI = torch.cat(kents, dim=1) if ov else None
    assert torch.equal(pool, pool1)
    if ov:
        assert torch.equal(KI, KI1)
    for r in range(W):
        sl = slice(r * sh, (r + 1) * sh)
        Or, Lr, ir, cr = cp.prefill_range(
            Q=d["Q"][:, sl].contiguous(), local=d["local"][:, sl].contiguous(), p0=r * sh, m=m, wwin=wwin,
            pool=pool.view(E, -1), KI=None if KI is None else KI.view(E, -1),
            qI=None if not ov else d["qI"][:, sl].contiguous(), w=None if not ov else d["w"][:, sl].contiguous(),
            k=s.k, sink=d["sink"], local_halo=d["local"][:, :r * sh] if r else None)
        dsv4.dsv4_check_errors()
        if ov:
            assert torch.equal(cr, c1[:, sl]) and torch.equal(ir, i1[:, sl]), f"rank {r} top-k"
        assert torch.equal(Or, O1[:, sl]), f"rank {r} O"
        assert torch.equal(Lr, L1[:, sl]), f"rank {r} LSE"
