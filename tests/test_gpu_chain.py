"""GPU end-to-end: compress -> index top-k -> hybrid attention vs the oracle's own chain.

The tiny fp32 CSA/HCA layers run whole on both sides: the GPU chain feeds its own
compressed pools and top-k sets forward; the oracle chain does the same in fp64. Queries
whose top-k sets differ only by ties are excluded from the output comparison (their
candidate lists differ legitimately); every other query must match.
"""
import numpy as np
import pytest
import torch

import oracle as O
from parity_util import assert_close, check_topk_query
from workloads import Generator, preset

pytestmark = pytest.mark.gpu


def test_chain_tiny_csa_fp32(dsv4):
    s = preset("tiny_csa")
    g = Generator(0)
    C, Z, bias = g.compressor_inputs(s, "main")
    CI, ZI, biasI = g.compressor_inputs(s, "index")
    qI, w = g.index_queries(s)
    Q = g.queries(s)
    local = g.local_kv(s)
    ref = O.csa_prefill_layer(C, Z, bias, CI, ZI, biasI, qI, w, Q, local, s.m, s.k, s.w)
    pool = dsv4.dsv4_compress(C.cuda(), Z.cuda(), bias.cuda(), s.m, True)
    KI = dsv4.dsv4_compress(CI.cuda(), ZI.cuda(), biasI.cuda(), s.m, True)
    E = s.n // s.m
    off = torch.zeros(1, dtype=torch.int64, device="cuda")
    pos0 = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx, counts = dsv4.dsv4_index_topk(qI.cuda(), w.cuda(), KI.reshape(E, -1), off, pos0, s.m,
                                       s.k, E)
    O_, L_ = dsv4.dsv4_hybrid_sparse_attn(Q.cuda(), pool.reshape(E, -1), off, idx, counts,
                                          local.cuda(), pos0, s.m, s.w)
    dsv4.dsv4_check_errors()
    assert_close(pool, ref["pool"], "f32", "pool")
    assert_close(KI, ref["KI"], "f32", "index keys")
    idx_c, cnt_c = idx.cpu().numpy(), counts.cpu().numpy()
    qI64, w64, KI64 = O.as_f64(qI), O.as_f64(w), ref["KI"][0]
    same = []
    for t in range(s.n):
        sc = O.index_scores_query(qI64[0, t], w64[0, t], KI64, t, s.m)
        check_topk_query(idx_c[0, t], cnt_c[0, t], sc, s.k, what=f"t={t}")
        if set(idx_c[0, t, :cnt_c[0, t]].tolist()) == set(ref["idx"][0, t, :ref["counts"][0, t]].tolist()):
            same.append(t)
    assert len(same) >= s.n - 2
    assert_close(O_.cpu()[0, same], ref["O"][0, same], "f32", "O")
    assert_close(L_.cpu()[0, same], ref["LSE"][0, same], "f32", "LSE")


def test_chain_tiny_hca_fp32(dsv4):
    s = preset("tiny_hca")
    g = Generator(1)
    C, Z, bias = g.compressor_inputs(s, "main")
    Q = g.queries(s)
    local = g.local_kv(s)
    ref = O.hca_prefill_layer(C, Z, bias, Q, local, s.m, s.w)
    pool = dsv4.dsv4_compress(C.cuda(), Z.cuda(), bias.cuda(), s.m, False)
    E = s.n // s.m
    off = torch.zeros(1, dtype=torch.int64, device="cuda")
    pos0 = torch.zeros(1, dtype=torch.int32, device="cuda")
    O_, L_ = dsv4.dsv4_hybrid_sparse_attn(Q.cuda(), pool.reshape(E, -1), off, None, None,
                                          local.cuda(), pos0, s.m, s.w)
    dsv4.dsv4_check_errors()
    assert_close(O_, ref["O"], "f32", "O")
    assert_close(L_, ref["LSE"], "f32", "LSE")
