"""GPU parity of the production main-KV entry ("CSA And HCA: Definition, State, And Cost
Model", s8 precision table: 448 FP8 + 64 bf16 RoPE channels per entry) against the oracle's
quantize_main_kv_fp8 / dequantize_main_kv_fp8.

* Quantisation: codes and scales bit-exact (rounding decided in fp32 on both sides), edge
  groups included (all zero, -0 codes, subnormal codes, saturation, exact ties).
* Expansion to bf16: bit-exact against the oracle's exact value rounded to bf16.
* Quantise on emission: the decode compressor's FP8 entries equal the quantisation of the
  bf16 entries the bf16 decode compressor emits for the same token stream, bit for bit.
* Decode attention over an FP8 pool: against the oracle attending over the exactly
  dequantised rows (bf16 tolerance), and bit-identical to the bf16 kernel over the
  expanded pool.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from parity_util import assert_close
from workloads import Generator

pytestmark = pytest.mark.gpu


def _rows_with_edges(g, rows, c, dtype):
    x = g.normal("x", (rows, c), 1.0, torch.float32)
    x[0, :64] = 0.0                                  # zero group: zero scale, zero codes
    x[1, :64] = 0.0
    x[1, 0], x[1, 1] = 448.0, -4e-4                  # -4e-4 / scale rounds to -0: code 0x80
    x[2, :64] = torch.linspace(-1, 1, 64)           # tiny codes around zero
    x[2, 5] = 448.0 * 2 ** -9 * 3                    # subnormal E4M3 range after scaling
    x[3, 64:128] = 1e-30                             # subnormal-scale group
    x[4, 128:192] *= 1e4
    return x.to(dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantize_main_kv_bit_exact(dsv4, dtype):
    g = Generator(81)
    x = _rows_with_edges(g, 300, 512, dtype)
    codes, scales, rope = dsv4.dsv4_quantize_main_kv(x.cuda())
    dsv4.dsv4_check_errors()
    c_ref, s_ref, r_ref = O.quantize_main_kv_fp8(x.float())
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), s_ref.astype(np.float32).view(np.uint32))
    assert np.array_equal(rope.float().cpu().double().numpy(), r_ref)
    assert codes[1, 1].item() == 0x80 and (codes[0, :64] == 0).all()


def test_dequantize_main_kv_bit_exact(dsv4):
    g = Generator(82)
    x = _rows_with_edges(g, 200, 512, torch.bfloat16)
    codes, scales, rope = dsv4.dsv4_quantize_main_kv(x.cuda())
    out = dsv4.dsv4_dequantize_main_kv(codes, scales, rope)
    dsv4.dsv4_check_errors()
    exact = O.dequantize_main_kv_fp8(codes.cpu().numpy(), scales.cpu().numpy(), rope.float().cpu().numpy())
    want = torch.from_numpy(exact).to(torch.bfloat16)          # round to nearest even, once
    assert torch.equal(out.cpu(), want)


@pytest.mark.parametrize("overlap,m", [(True, 4), (False, 128)])
def test_emission_quantises_the_bf16_entry(dsv4, overlap, m):
    B, c, rope = 3, 512, 64
    S = 2 if overlap else 1
    g = Generator(83 + m)
    n0 = [0, 5 * m + 1, 2 * m]
    steps = 2 * m + 3
    C = [g.normal(f"C{b}", (n0[b] + steps, S * c), 1.0, torch.bfloat16) for b in range(B)]
    Z = [g.normal(f"Z{b}", (n0[b] + steps, S * c), 1.0, torch.bfloat16) for b in range(B)]
    bias = g.normal("bias", (S, m, c), 0.1).cuda()
    E = [(n0[b] + steps) // m for b in range(B)]
    off = torch.tensor(np.concatenate([[0], np.cumsum(E)[:-1]]), dtype=torch.int64).cuda()
    rows = int(sum(E))
    T = S * m

    def tail0():
        t = torch.zeros(B, T, 2, S * c, dtype=torch.bfloat16)
        for b in range(B):
            for p in range(max(0, n0[b] - T), n0[b]):
                t[b, p % T, 0], t[b, p % T, 1] = C[b][p], Z[b][p]
        return t.cuda()

    tail_a, tail_b = tail0(), tail0()
    pool = torch.zeros(rows, c, dtype=torch.bfloat16, device="cuda")
    codes = torch.zeros(rows, c - rope, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(rows, (c - rope) // 64, dtype=torch.float32, device="cuda")
    rp = torch.zeros(rows, rope, dtype=torch.bfloat16, device="cuda")
    emitted = []
    for s in range(steps):
        pos = torch.tensor([n0[b] + s for b in range(B)], dtype=torch.int32, device="cuda")
        Cn = torch.stack([C[b][n0[b] + s] for b in range(B)]).cuda()
        Zn = torch.stack([Z[b][n0[b] + s] for b in range(B)]).cuda()
        dsv4.dsv4_compress_decode(Cn, Zn, bias, tail_a, pool, off, pos, m, overlap)
        dsv4.dsv4_compress_decode_fp8(Cn, Zn, bias, tail_b, codes, scales, rp, off, pos, m, overlap)
        for b in range(B):
            if (n0[b] + s + 1) % m == 0:
                emitted.append(int(off[b]) + (n0[b] + s + 1) // m - 1)
    dsv4.dsv4_check_errors()
    assert len(emitted) >= 3
    ev = torch.tensor(emitted)
    c_ref, s_ref, r_ref = O.quantize_main_kv_fp8(pool[ev.cuda()].float().cpu())
    assert np.array_equal(codes[ev.cuda()].cpu().numpy(), c_ref)
    assert np.array_equal(scales[ev.cuda()].cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(rp[ev.cuda()].float().cpu().double().numpy(), r_ref)


def test_decode_attention_over_fp8_pool(dsv4):
    B, H, c, k, w, m = 8, 64, 512, 512, 128, 4
    lens = [1, 5, 129, 2048, 4096 + 3, 20000, 70001, 262144]
    g = Generator(84)
    E = [L // m for L in lens]
    offs = np.concatenate([[0], np.cumsum([e + 1 for e in E])[:-1]]).astype(np.int64)
    rows = int(sum(E)) + B
    x = g.normal("pool", (rows, c), 1.0, torch.bfloat16).cuda()
    codes, scales, rope = dsv4.dsv4_quantize_main_kv(x)
    Q = g.normal("Q", (B, 1, H, c), 1.0, torch.bfloat16).cuda()
    local = g.normal("local", (B, w, c), 1.0, torch.bfloat16).cuda()
    sink = g.normal("sink", (H,), 1.0).cuda()
    idx, cnt = g.random_index_sets(torch.tensor(E), k)
    idx, cnt = idx.reshape(B, 1, k).cuda(), cnt.reshape(B, 1).cuda()
    idx[2, 0, 0] = -5 if cnt[2, 0] > 0 else idx[2, 0, 0]      # an invalid selection: skipped, reported
    pos0 = torch.tensor([L - 1 for L in lens], dtype=torch.int32).cuda()
    off = torch.from_numpy(offs).cuda()
    Og, Lg = dsv4.dsv4_hybrid_sparse_attn_fp8(Q, codes, scales, rope, off, idx, cnt, local, pos0, m, w, sink)
    with pytest.raises(dsv4.DSV4Error) as ei:
        dsv4.dsv4_check_errors()
    assert ei.value.status == 5
    # the same rows expanded to bf16, attended by the bf16 kernel: bit-identical
    pool16 = dsv4.dsv4_dequantize_main_kv(codes, scales, rope)
    Ob, Lb = dsv4.dsv4_hybrid_sparse_attn(Q, pool16, off, idx, cnt, local, pos0, m, w, sink)
    with pytest.raises(dsv4.DSV4Error):
        dsv4.dsv4_check_errors()
    assert torch.equal(Og, Ob) and torch.equal(Lg, Lb)
    # the oracle over the exact dequantised rows (the invalid selection left out)
    exact = O.dequantize_main_kv_fp8(codes.cpu().numpy(), scales.cpu().numpy(), rope.float().cpu().numpy())
    idx_o, cnt_o = idx.cpu().numpy().copy(), cnt.cpu().numpy().copy()
    if cnt_o[2, 0] > 0:
        idx_o[2, 0, :cnt_o[2, 0] - 1] = idx_o[2, 0, 1:cnt_o[2, 0]]
        cnt_o[2, 0] -= 1
    qs = [(b, 0) for b in range(B)]
    Or, Lr = O.hybrid_attention(Q.cpu(), exact, offs, idx_o, cnt_o, local.cpu(), pos0.cpu().numpy(), w,
                                sink.cpu(), 1 / math.sqrt(c), queries=qs)
    assert_close(Og[:, 0].cpu(), Or, "bf16", "fp8 pool decode O", verbose=True)
    assert_close(Lg[:, 0].cpu(), Lr, "bf16", "fp8 pool decode LSE", verbose=True)
