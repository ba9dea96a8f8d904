"""GPU test of dsv4_index_topk_noalloc, the indexer top-k for callers that cannot allocate.

Some callers cannot call cudaMalloc (a runtime that only hands out pre-planned buffers,
plain C code without a device allocator, a serving loop where an allocation could
synchronise the device). dsv4_index_topk_noalloc serves them from a fixed scratch array
inside the library. This test calls it through the C ABI (ctypes, raw device pointers)
twice in a row and checks both results against the workspace-based dsv4_index_topk on
the same inputs. The scratch is reused between the two calls, so the second call also
shows that leftover contents do not leak into a result.

The file name sorts last so that a run stopping at the first failure has already run
every other test.
"""
import ctypes

import pytest
import torch

from workloads import Generator, preset

pytestmark = pytest.mark.gpu


def _noalloc(lib):
    f = lib.dsv4_index_topk_noalloc
    P, I, L = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    f.restype = I
    f.argtypes = [I, P, P, P, P, P, L, P, P, I, I, I, I, I, I, I, P, P, P]
    return f


def test_noalloc_matches_workspace_entry_point(dsv4):
    f = _noalloc(dsv4.lib)
    s = preset("flash_csa_prefill")                 # n=8192: 8 chunks of the 8 MiB scratch
    g = Generator(21)
    qI, w = g.index_queries(s)
    E = s.n // s.m
    KI = g.index_keys(s, E).cuda()
    qI, w = qI.cuda(), w.cuda()
    off = torch.zeros(1, dtype=torch.int64, device="cuda")
    pos0 = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref_idx, ref_cnt = dsv4.dsv4_index_topk(qI, w, KI, off, pos0, s.m, s.k, E)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        idx = torch.full((1, s.n, s.k), -7, dtype=torch.int32, device="cuda")
        cnt = torch.full((1, s.n), -7, dtype=torch.int32, device="cuda")
        st = f(dsv4.BF16, qI.data_ptr(), None, w.data_ptr(), KI.data_ptr(), None, E,
               off.data_ptr(), pos0.data_ptr(), 1, s.n, s.H_I, s.c_I, s.m, s.k, E,
               idx.data_ptr(), cnt.data_ptr(), stream)
        assert st == 0, dsv4.lib.dsv4_last_error_message()
        dsv4.dsv4_check_errors()
        # same kernels, query-independent results: the indices agree exactly
        assert torch.equal(cnt, ref_cnt), f"call {call}: counts differ"
        assert torch.equal(idx, ref_idx), f"call {call}: indices differ"


def test_noalloc_rejects_rows_beyond_the_scratch(dsv4):
    f = _noalloc(dsv4.lib)
    too_many = (8 << 20) // 4 + 4
    st = f(dsv4.BF16, ctypes.c_void_p(16), None, ctypes.c_void_p(16), ctypes.c_void_p(16), None,
           too_many, ctypes.c_void_p(16), ctypes.c_void_p(16), 1, 1, 64, 128, 4, 512, too_many,
           ctypes.c_void_p(16), ctypes.c_void_p(16), None)
    assert st == 1                                  # DSV4_ERR_INVALID_ARG, nothing enqueued
    assert b"scratch limit" in dsv4.lib.dsv4_last_error_message()


def test_noalloc_fp4_operands_match_workspace_entry_point(dsv4):
    """FP4 operands with a key pool small enough that the exact bf16 expansion of K^I fits
    in the fixed scratch beside the score rows: the same tensor-core path as the workspace
    entry point, so the indices agree exactly, on two calls in a row."""
    f = _noalloc(dsv4.lib)
    s = preset("flash_csa_prefill", n=4096)
    g = Generator(22, device="cuda")
    E = s.n // s.m
    qI, w = g.index_queries(s)
    KI = g.index_keys(s, E)
    qc, qs = dsv4.dsv4_quantize_fp4(qI.reshape(-1, s.c_I))
    kc, ks = dsv4.dsv4_quantize_fp4(KI)
    off = torch.zeros(1, dtype=torch.int64, device="cuda")
    pos0 = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref_idx, ref_cnt = dsv4.dsv4_index_topk(qc.view(1, s.n, s.H_I, s.c_I // 2), w, kc, off, pos0, s.m,
                                            s.k, E, qI_scales=qs, KI_scales=ks, c_I=s.c_I)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        idx = torch.full((1, s.n, s.k), -7, dtype=torch.int32, device="cuda")
        cnt = torch.full((1, s.n), -7, dtype=torch.int32, device="cuda")
        st = f(dsv4.FP4, qc.data_ptr(), qs.data_ptr(), w.data_ptr(), kc.data_ptr(), ks.data_ptr(), E,
               off.data_ptr(), pos0.data_ptr(), 1, s.n, s.H_I, s.c_I, s.m, s.k, E,
               idx.data_ptr(), cnt.data_ptr(), stream)
        assert st == 0, dsv4.lib.dsv4_last_error_message()
        dsv4.dsv4_check_errors()
        assert torch.equal(cnt, ref_cnt), f"call {call}: counts differ"
        assert torch.equal(idx, ref_idx), f"call {call}: indices differ"


def test_noalloc_long_rows_and_large_fp4_pool(dsv4):
    """Decode-length rows (one query per sequence over 40k-90k entries, beyond the one-CTA
    top-k) and a FP4 key pool far larger than a bf16 expansion in the fixed scratch could
    hold (decode requests expand the FP4 keys inside the score kernel): checked against the
    fp64 oracle under the stated tie rule, on two calls in a row."""
    import numpy as np
    import oracle as O
    from parity_util import check_topk_query
    f = _noalloc(dsv4.lib)
    s = preset("flash_csa_prefill")
    g = Generator(23, device="cuda")
    lens = [160001, 240000, 361003]
    E = [L // s.m for L in lens]
    B, k = len(lens), s.k
    offs = np.concatenate([[0], np.cumsum(E)[:-1]]).astype(np.int64)
    KI = g.index_keys(s, int(sum(E)))
    qI, w = g.index_queries(preset("flash_csa_prefill", B=B), 1)
    pos0 = torch.tensor([L - 1 for L in lens], dtype=torch.int32, device="cuda")
    off = torch.from_numpy(offs).cuda()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for fmt in ("bf16", "fp4"):
        if fmt == "fp4":
            qc, qs = dsv4.dsv4_quantize_fp4(qI.reshape(-1, s.c_I))
            kc, ks = dsv4.dsv4_quantize_fp4(KI)
            args = (dsv4.FP4, qc.data_ptr(), qs.data_ptr(), kc.data_ptr(), ks.data_ptr())
            K64 = O.dequantize_fp4(*O.quantize_fp4(KI.float().cpu()), s.c_I)
            q64 = [O.dequantize_fp4(*O.quantize_fp4(qI[b, 0].float().cpu()), s.c_I) for b in range(B)]
        else:
            args = (dsv4.BF16, qI.data_ptr(), None, KI.data_ptr(), None)
            K64 = O.as_f64(KI.cpu())
            q64 = [qI[b, 0].cpu() for b in range(B)]
        for call in range(2):
            idx = torch.full((B, 1, k), -7, dtype=torch.int32, device="cuda")
            cnt = torch.full((B, 1), -7, dtype=torch.int32, device="cuda")
            st = f(args[0], args[1], args[2], w.data_ptr(), args[3], args[4], int(sum(E)),
                   off.data_ptr(), pos0.data_ptr(), B, 1, s.H_I, s.c_I, s.m, k, max(E),
                   idx.data_ptr(), cnt.data_ptr(), stream)
            assert st == 0, dsv4.lib.dsv4_last_error_message()
            dsv4.dsv4_check_errors()
            ih, ch = idx.cpu().numpy(), cnt.cpu().numpy()
            for b in range(B):
                s64 = O.index_scores_query(q64[b], w[b, 0].cpu(), K64[int(offs[b]):int(offs[b]) + E[b]],
                                           lens[b] - 1, s.m)
                check_topk_query(ih[b, 0], ch[b, 0], s64, k, what=f"{fmt} call {call} b={b}")
