"""CPU checks of the C ABI: the library loads, exports every declared symbol, and rejects
bad arguments on the host before touching a device. No kernel is launched here."""
import ctypes
import glob
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "compressed_sparse_mqa_dsv4_b200", "libdsv4.so")


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(dsv4_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):       # the package itself refuses to import without it
        subprocess.run([sys.executable, os.path.join(ROOT, "compressed_sparse_mqa_dsv4_b200", "build.py")],
                       check=True)
    return ctypes.CDLL(LIB)


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_status_strings_and_version(lib):
    lib.dsv4_status_string.restype = ctypes.c_char_p
    for s in range(7):
        assert lib.dsv4_status_string(s)
    assert lib.dsv4_status_string(99) == b"unknown status"
    assert lib.dsv4_abi_version() == 1


def test_host_validation_rejects_bad_arguments(lib):
    lib.dsv4_last_error_message.restype = ctypes.c_char_p
    P = ctypes.c_void_p
    # dsv4_compress with m = 0
    assert lib.dsv4_compress(1, P(16), P(16), P(16), P(16), 1, 8, 8, 0, 1, None) == 1
    assert b"bad sizes" in lib.dsv4_last_error_message()
    # empty request is a no-op (no launch)
    assert lib.dsv4_compress(1, None, None, None, None, 0, 8, 8, 4, 1, None) == 0
    # FP4 quantiser needs cols % 16 == 0
    assert lib.dsv4_quantize_fp4(P(16), P(16), P(16), ctypes.c_int64(4), 24, None) == 1
    # attention: w < 1 rejected
    args = [1, P(16), P(16), ctypes.c_int64(4), P(16), None, None, 0, P(16), 8, P(16), 1, 1, 64,
            512, 4, 0, None, ctypes.c_float(1.0), P(16), None, None, ctypes.c_size_t(0), None]
    assert lib.dsv4_hybrid_sparse_attn(*args) == 1
    # decode state: m = 0 rejected; B = 0 is a no-op; a ring of R = 0 slots rejected
    lib.dsv4_compress_decode.restype = ctypes.c_int
    assert lib.dsv4_compress_decode(1, P(16), P(16), P(16), P(16), P(16), P(16), ctypes.c_int64(4),
                                    P(16), 1, 8, 0, 1, None) == 1
    assert lib.dsv4_compress_decode(1, None, None, None, None, None, None, ctypes.c_int64(0), None,
                                    0, 8, 4, 1, None) == 0
    lib.dsv4_ring_write.restype = ctypes.c_int
    assert lib.dsv4_ring_write(1, P(16), P(16), 0, P(16), 1, 8, None) == 1
    # index top-k: k above the supported maximum
    lib.dsv4_index_topk.restype = ctypes.c_int
    a = [1, P(16), None, P(16), P(16), None, ctypes.c_int64(1), P(16), P(16), 1, 1, 64, 128, 4,
         5000, 8, P(16), P(16), None, ctypes.c_int64(0), P(256), ctypes.c_size_t(1 << 20), None]
    assert lib.dsv4_index_topk(*a) == 1


def test_workspace_size_is_bounded(lib):
    lib.dsv4_index_topk_workspace_size.restype = ctypes.c_size_t
    small = lib.dsv4_index_topk_workspace_size(1, 8192, 2048, 512)
    assert small == 8192 * 2048 * 4
    big = lib.dsv4_index_topk_workspace_size(1, 131072, 32768, 1024)
    assert 0 < big <= (256 << 20) and big % 256 == 0


def _r256(x):
    return (x + 255) // 256 * 256


@pytest.mark.parametrize("B,nq,E,k", [(64, 1, 262144, 512), (1, 4, 16385, 512), (1, 1024, 40000, 4096)])
def test_workspace_size_threshold_topk_rows(lib, B, nq, E, k):
    """Requests of at most 1024 rows longer than 16384 entries: score rows plus the threshold
    top-k region of 8448 bytes + round256(4k) + 64 KiB per row, as the header states."""
    f = lib.dsv4_index_topk_workspace_size
    f.restype = ctypes.c_size_t
    rows = B * nq
    per = 4 * ((E + 3) // 4 * 4) + 8448 + _r256(4 * k) + 65536
    rows = min(rows, (256 << 20) // per)
    want = _r256(rows * 4 * ((E + 3) // 4 * 4)) + _r256(rows * (8448 + _r256(4 * k) + 65536))
    assert f(B, nq, E, k) == want


@pytest.mark.parametrize("B,nq,E,k", [(1, 1100, 17000, 256), (1, 2048, 32768, 1024)])
def test_workspace_size_segment_topk_rows(lib, B, nq, E, k):
    """More than 1024 long rows: score rows plus 8k bytes per 16384-entry segment per row."""
    f = lib.dsv4_index_topk_workspace_size
    f.restype = ctypes.c_size_t
    nseg = (E + 16383) // 16384
    cand = nseg * k * 8
    per = 4 * ((E + 3) // 4 * 4) + cand
    rows = min(B * nq, (256 << 20) // per)
    want = _r256(rows * 4 * ((E + 3) // 4 * 4)) + _r256(rows * cand)
    assert f(B, nq, E, k) == want


def test_workspace_size_short_rows_and_empty(lib):
    f = lib.dsv4_index_topk_workspace_size
    f.restype = ctypes.c_size_t
    assert f(1, 2048, 16384, 512) == 2048 * 16384 * 4            # no top-k region
    assert f(1, 8192, 16384, 512) == 256 << 20                    # chunks of 4096 rows
    assert f(0, 8, 100, 4) == 0 and f(2, 0, 100, 4) == 0



def test_decode_job_layout_and_host_validation(lib):
    """dsv4_decode_job as the binding builds it (96 bytes: six ints, eight pointers, one
    int64), and host validation of dsv4_decode_state before anything is enqueued."""
    import compressed_sparse_mqa_dsv4_b200 as dsv4
    J = dsv4._DecodeJob
    assert ctypes.sizeof(J) == 96 and J.x_new.offset == 24 and J.pool_rows.offset == 88
    bad = (J * 1)(J(kind=7, c=8))
    assert lib.dsv4_decode_state(1, bad, 1, ctypes.c_void_p(16), 1, None) == 1
    assert b"kind 7" in lib.dsv4_last_error_message()
    too_many = (J * 33)()
    assert lib.dsv4_decode_state(1, too_many, 33, ctypes.c_void_p(16), 1, None) == 1
    ring_no_out = (J * 1)(J(kind=0, c=8, R=4, x_new=16))
    assert lib.dsv4_decode_state(1, ring_no_out, 1, ctypes.c_void_p(16), 1, None) == 1
    assert lib.dsv4_decode_state(1, bad, 1, ctypes.c_void_p(16), 0, None) == 0   # B == 0: no-op
    fp4_odd = (J * 1)(J(kind=3, c=24, m=4, overlap=1, x_new=16, z_new=16, bias=16, tail=16, out=16,
                        out_scales=16, pool_row_off=16, pool_rows=8))
    assert lib.dsv4_decode_state(1, fp4_odd, 1, ctypes.c_void_p(16), 1, None) == 1     # c % 16
    fp8_rope = (J * 1)(J(kind=2, c=512, m=4, overlap=1, rope_dims=63, x_new=16, z_new=16, bias=16,
                         tail=16, out=16, out_scales=16, out_rope=16, pool_row_off=16, pool_rows=8))
    assert lib.dsv4_decode_state(1, fp8_rope, 1, ctypes.c_void_p(16), 1, None) == 1    # odd rope
