"""CPU checks of the Python binding: it marshals arguments only. Host tensors, wrong dtypes,
non-contiguous views and mismatched state shapes are refused before the library is called,
so there is no CPU path to fall back to; the exported names match the C entry points.
"""
import inspect
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if not os.path.exists(os.path.join(ROOT, "compressed_sparse_mqa_dsv4_b200", "libdsv4.so")):
    subprocess.run([sys.executable, os.path.join(ROOT, "compressed_sparse_mqa_dsv4_b200", "build.py")],
                   check=True)

import compressed_sparse_mqa_dsv4_b200 as dsv4  # noqa: E402


def test_every_public_function_is_a_library_entry_point_or_size_helper():
    for name in dsv4.__all__:
        obj = getattr(dsv4, name)
        if name.startswith("dsv4_"):
            assert hasattr(dsv4.lib, name), f"{name} has no C entry point of the same name"
            assert inspect.isfunction(obj)


@pytest.mark.parametrize("call", [
    lambda: dsv4.dsv4_compress(torch.zeros(1, 8, 16), torch.zeros(1, 8, 16),
                               torch.zeros(2, 4, 8), 4, True),
    lambda: dsv4.dsv4_quantize_fp4(torch.zeros(4, 32, dtype=torch.bfloat16)),
    lambda: dsv4.dsv4_ring_write(torch.zeros(2, 8), torch.zeros(2, 4, 8),
                                 torch.zeros(2, dtype=torch.int32)),
    lambda: dsv4.dsv4_compress_decode(torch.zeros(2, 16), torch.zeros(2, 16), torch.zeros(2, 4, 8),
                                      torch.zeros(2, 8, 2, 16), torch.zeros(4, 8),
                                      torch.zeros(2, dtype=torch.int64),
                                      torch.zeros(2, dtype=torch.int32), 4, True),
    lambda: dsv4.dsv4_index_topk(torch.zeros(1, 4, 2, 32), torch.zeros(1, 4, 2), torch.zeros(8, 32),
                                 torch.zeros(1, dtype=torch.int64), torch.zeros(1, dtype=torch.int32),
                                 4, 2, 8),
    lambda: dsv4.dsv4_hybrid_sparse_attn(torch.zeros(1, 4, 2, 16), torch.zeros(8, 16),
                                         torch.zeros(1, dtype=torch.int64), None, None,
                                         torch.zeros(1, 4, 16), torch.zeros(1, dtype=torch.int32),
                                         4, 2),
])
def test_host_tensors_are_refused(call):
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        call()


class _FakeCuda:
    """Stands in for a device tensor in the checks that run before any pointer is used."""

    def __init__(self, t):
        self._t = t
        self.is_cuda = True
        self.dtype = t.dtype
        self.shape = t.shape

    def is_contiguous(self):
        return self._t.is_contiguous()

    def numel(self):
        return self._t.numel()


def test_decode_state_shape_and_dtype_checks():
    B, c, m = 2, 8, 4
    C = _FakeCuda(torch.zeros(B, 2 * c))
    bias = _FakeCuda(torch.zeros(2, m, c))
    off = _FakeCuda(torch.zeros(B, dtype=torch.int64))
    pos = _FakeCuda(torch.zeros(B, dtype=torch.int32))
    pool = _FakeCuda(torch.zeros(4, c))
    wrong_tail = _FakeCuda(torch.zeros(B, m, 2, 2 * c))          # a CSA tail has 2m slots
    with pytest.raises(ValueError, match="tail must be"):
        dsv4.dsv4_compress_decode(C, C, bias, wrong_tail, pool, off, pos, m, True)
    with pytest.raises(ValueError, match="Z_new must be"):
        dsv4.dsv4_compress_decode(C, _FakeCuda(torch.zeros(B, 2 * c, dtype=torch.bfloat16)), bias,
                                  wrong_tail, pool, off, pos, m, True)
    with pytest.raises(ValueError, match="pos must be"):
        dsv4.dsv4_ring_write(_FakeCuda(torch.zeros(B, c)), _FakeCuda(torch.zeros(B, 4, c)),
                             _FakeCuda(torch.zeros(B, dtype=torch.int64)))
    assert dsv4.decode_tail_shape(B, c, m, True) == (B, 2 * m, 2, 2 * c)
    assert dsv4.decode_tail_shape(B, c, 128, False) == (B, 128, 2, c)


def test_non_contiguous_views_are_refused():
    x = _FakeCuda(torch.zeros(4, 32, dtype=torch.bfloat16).t())
    with pytest.raises(ValueError, match="must be contiguous"):
        dsv4.dsv4_quantize_fp4(x)


def _header_declarations():
    import re
    text = open(os.path.join(ROOT, "include", "dsv4.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    decls = {}
    for ret, name, params in re.findall(r"\b(int|size_t|const char\*)\s+(dsv4_[a-z0-9_]+)\s*\(([^)]*)\)\s*;",
                                        text, flags=re.S):
        ps = [p.strip() for p in params.replace("\n", " ").split(",") if p.strip()]
        decls[name] = (ret, [] if ps == ["void"] else ps)
    return decls


def _ctype_for(param: str):
    import ctypes
    p = " ".join(param.split())
    if "*" in p:
        return (ctypes.c_void_p, ctypes.c_char_p)
    t = p.rsplit(" ", 1)[0]
    return {"int": (ctypes.c_int,), "int64_t": (ctypes.c_int64,), "size_t": (ctypes.c_size_t,),
            "float": (ctypes.c_float,)}[t]


def test_binding_argtypes_match_the_header():
    """Every entry point the binding declares has as many ctypes arguments as the header's
    parameters, each of the same width (a 64-bit size passed as a 32-bit int would be read
    with garbage upper bits), and the matching return type."""
    import ctypes
    decls = _header_declarations()
    assert len(decls) >= 12
    checked = 0
    for name, (ret, params) in decls.items():
        fn = getattr(dsv4.lib, name)
        want_ret = {"int": ctypes.c_int, "size_t": ctypes.c_size_t, "const char*": ctypes.c_char_p}[ret]
        assert fn.restype == want_ret, f"{name}: restype {fn.restype} for {ret}"
        if fn.argtypes is None:
            assert name == "dsv4_abi_version" or not params, f"{name}: argtypes not declared"
            continue
        assert len(fn.argtypes) == len(params), f"{name}: {len(fn.argtypes)} ctypes args, {len(params)} in the header"
        for i, (have, p) in enumerate(zip(fn.argtypes, params)):
            struct_ptr = "*" in p and isinstance(have, type) and issubclass(have, ctypes._Pointer)
            assert have in _ctype_for(p) or struct_ptr, f"{name} arg {i} ({p}): {have}"
        checked += 1
    assert checked >= 10


def test_packed_decode_job_checks():
    """The FP8 / FP4 compressor jobs of dsv4_decode_state check their pool shapes and dtypes
    before any pointer is taken."""
    B, c, cI, m, rd = 2, 576, 128, 4, 64
    C = _FakeCuda(torch.zeros(B, 2 * c, dtype=torch.bfloat16))
    bias = _FakeCuda(torch.zeros(2, m, c))
    tail = _FakeCuda(torch.zeros(B, 2 * m, 2, 2 * c, dtype=torch.bfloat16))
    off = _FakeCuda(torch.zeros(B, dtype=torch.int64))
    codes = _FakeCuda(torch.zeros(8, c - rd, dtype=torch.uint8))
    scales = _FakeCuda(torch.zeros(8, (c - rd) // 64))
    rope = _FakeCuda(torch.zeros(8, rd, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="codes rows must have"):
        dsv4.decode_compress_fp8_job(C, C, bias, tail, _FakeCuda(torch.zeros(8, c, dtype=torch.uint8)),
                                     scales, rope, off, m, True, rd)
    with pytest.raises(ValueError, match="rope must be given"):
        dsv4.decode_compress_fp8_job(C, C, bias, tail, codes, scales, None, off, m, True, rd)
    with pytest.raises(ValueError, match="scales must be"):
        dsv4.decode_compress_fp8_job(C, C, bias, tail, codes, _FakeCuda(torch.zeros(8, 7, dtype=torch.uint8)),
                                     rope, off, m, True, rd)
    with pytest.raises(ValueError, match="tail must be"):
        dsv4.decode_compress_fp8_job(C, C, bias, _FakeCuda(torch.zeros(B, m, 2, 2 * c, dtype=torch.bfloat16)),
                                     codes, scales, rope, off, m, True, rd)
    CI = _FakeCuda(torch.zeros(B, 2 * cI, dtype=torch.bfloat16))
    biasI = _FakeCuda(torch.zeros(2, m, cI))
    tailI = _FakeCuda(torch.zeros(B, 2 * m, 2, 2 * cI, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="FP4 pool rows"):
        dsv4.decode_compress_fp4_job(CI, CI, biasI, tailI, _FakeCuda(torch.zeros(8, cI // 2, dtype=torch.uint8)),
                                     _FakeCuda(torch.zeros(8, cI // 32, dtype=torch.uint8)), off, m, True)
    with pytest.raises(ValueError, match="scales must be"):
        dsv4.decode_compress_fp4_job(CI, CI, biasI, tailI, _FakeCuda(torch.zeros(8, cI // 2, dtype=torch.uint8)),
                                     _FakeCuda(torch.zeros(8, cI // 16)), off, m, True)
