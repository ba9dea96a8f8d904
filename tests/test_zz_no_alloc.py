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
