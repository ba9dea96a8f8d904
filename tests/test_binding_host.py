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
