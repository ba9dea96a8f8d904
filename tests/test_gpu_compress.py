"""GPU parity: dsv4_compress (CSA overlap / HCA) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from parity_util import assert_close
from workloads import Generator, preset

pytestmark = pytest.mark.gpu


def _run(dsv4, shape, which="main", n=None, seed=0):
    g = Generator(seed)
    C, Z, bias = g.compressor_inputs(shape, which, n=n)
    overlap = shape.kind == "csa"
    out = dsv4.dsv4_compress(C.cuda(), Z.cuda(), bias.cuda(), shape.m, overlap)
    ref = O.compress(C, Z, bias, shape.m, overlap)
    return out, ref


@pytest.mark.parametrize("name,which", [("tiny_csa", "main"), ("tiny_csa", "index"),
                                        ("tiny_hca", "main")])
def test_compress_tiny_fp32(dsv4, name, which):
    out, ref = _run(dsv4, preset(name), which)
    assert out.shape == ref.shape
    assert_close(out, ref, "f32", f"{name}/{which}")


@pytest.mark.parametrize("n", [0, 3, 4, 5, 4 * 37 + 3, 1000])
@pytest.mark.parametrize("c", [512, 128, 24, 12])
def test_compress_ragged_bf16(dsv4, n, c):
    shape = preset("flash_csa_prefill", B=2, n=n, c=c, c_I=c)
    out, ref = _run(dsv4, shape, "main", seed=n + c)
    assert out.shape == ref.shape
    if ref.size:
        assert_close(out, ref, "bf16", f"csa n={n} c={c}")


@pytest.mark.parametrize("m", [128, 16, 1, 3])
def test_compress_hca_ratios(dsv4, m):
    shape = preset("flash_hca_prefill", B=2, n=m * 9 + m // 2, m=m, c=256)
    out, ref = _run(dsv4, shape, "main", seed=m)
    assert_close(out, ref, "bf16", f"hca m={m}")


def test_compress_fp32_scalar_path(dsv4):
    """c not a multiple of the 16-byte vector takes the scalar kernel."""
    shape = preset("tiny_csa", c=7, n=41)
    out, ref = _run(dsv4, shape, "main")
    assert_close(out, ref, "f32", "scalar path")


def test_compress_flash_full(dsv4):
    """V4-Flash CSA main (c=512) and index-key (c_I=128) compressors at n=8192."""
    shape = preset("flash_csa_prefill")
    for which in ("main", "index"):
        out, ref = _run(dsv4, shape, which)
        assert_close(out, ref, "bf16", f"flash {which}")


def test_compress_hca_full(dsv4):
    """V4-Flash HCA compressor at batch 2, n=65536, m'=128."""
    out, ref = _run(dsv4, preset("flash_hca_prefill"), "main")
    assert out.shape == (2, 512, 512)
    assert_close(out, ref, "bf16", "hca full")


def test_compress_large_logits(dsv4):
    """Gate logits far from 0 (+-60) stay finite and exact (max subtraction per channel)."""
    shape = preset("tiny_csa", n=64)
    g = Generator(5)
    C, Z, bias = g.compressor_inputs(shape)
    Z = Z * 60
    out = dsv4.dsv4_compress(C.cuda(), Z.cuda(), bias.cuda(), 4, True)
    ref = O.compress(C, Z, bias, 4, True)
    assert_close(out, ref, "f32", "large logits")
