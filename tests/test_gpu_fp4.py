"""GPU parity: dsv4_quantize_fp4 codes and scale bytes are bit-exact with the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from workloads import Generator

pytestmark = pytest.mark.gpu


def _cmp(dsv4, x_bf16):
    codes, scales = dsv4.dsv4_quantize_fp4(x_bf16.cuda())
    rc, rs = O.quantize_fp4(x_bf16.float())
    np.testing.assert_array_equal(scales.cpu().numpy(), rs)
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)


@pytest.mark.parametrize("rows,cols", [(1, 16), (7, 64), (1000, 128), (64 * 33, 128)])
def test_fp4_random(dsv4, rows, cols):
    x = Generator(rows).normal("x", (rows, cols), 1 / np.sqrt(cols), torch.bfloat16)
    _cmp(dsv4, x)


def test_fp4_edge_values(dsv4):
    """Zero groups, ties of the e2m1 grid, subnormal and saturated scales, signed zeros."""
    rows = []
    rows.append([0.0] * 16)                                        # zero scale
    rows.append([6.0, -3.0, 0.25 * 1, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -2.5,
                 -5.0, 0.1, -0.1, 4.0])                            # ties at scale 1
    rows.append([0.05] + [0.01] * 15)                              # subnormal E4M3 scale
    rows.append([1e-3] + [3e-4] * 15)                              # scale rounds to 0
    rows.append([3000.0, -2900.0] + [1.0] * 14)                    # scale saturates at 448
    rows.append([-0.0] * 8 + [6.0] + [-1e-9] * 7)                  # signed zeros
    rows.append([2.0 ** -12] * 16)                                 # scale rounds to 0 -> codes 0
    x = torch.tensor(rows, dtype=torch.float32).to(torch.bfloat16)
    _cmp(dsv4, x)


def test_fp4_index_shapes(dsv4):
    """Indexer operands at V4 shape: q^I rows (n*H_I, 128) and keys (E, 128)."""
    g = Generator(3)
    q = g.normal("q", (2048 * 64, 128), 1 / np.sqrt(128), torch.bfloat16)
    _cmp(dsv4, q)
