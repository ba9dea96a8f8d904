"""GPU parity of the s5.2 contract of "CSA And HCA: Definition, State, And Cost Model":
RMS normalisation of query heads and KV entries, RoPE on their last 64 channels at their
positions (query t, compressed entry s at m*s, local entry j at j), and the inverse
rotation of the output's last 64 channels at t -- against the oracle's rms_norm /
rope_rotate / attend_query_rope.

The rows are normalised and rotated by dsv4_norm_rope; the inverse rotation of O is fused
into the attention kernels (dsv4_hybrid_sparse_attn_rope): the tensor-core epilogue for
prefill, the split-list combine for decode, and the CUDA-core kernel.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from parity_util import assert_close
from workloads import Generator

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("norm,inverse", [(True, False), (False, True), (False, False)])
def test_norm_rope_rows(dsv4, dtype, norm, inverse):
    g = Generator(71)
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    rows, c, H = 96, 512, 4
    x = g.normal("x", (rows, c), 1.0, dt)
    pos = torch.tensor([0, 1, 7, 4096, 131071, 1 << 20, 1048575 + 4096, 999983] * 3, dtype=torch.int32)
    y = x.clone().cuda()
    dsv4.dsv4_norm_rope(y, pos.cuda(), rows_per_pos=H, rope=64, norm=norm, inverse=inverse)
    dsv4.dsv4_check_errors()
    ref = O.rms_norm(x) if norm else O.as_f64(x)
    ref = O.rope_rotate(ref, np.repeat(pos.numpy(), H), 64, inverse=inverse)
    assert_close(y.cpu(), ref, dtype, f"norm_rope norm={norm} inverse={inverse}", verbose=True)


def _rope_case(dsv4, *, B, nq, pos0, R, m, k, dense, split, seed, simt, monkeypatch):
    H, c, w = 64, 512, 128
    monkeypatch.setenv("DSV4_FORCE_SIMT", "1" if simt else "0")
    g = Generator(seed)
    E = [(p + nq) // m for p in pos0]
    offs = np.concatenate([[0], np.cumsum([e + 1 for e in E])[:-1]]).astype(np.int64)
    Qr = g.normal("Q", (B, nq, H, c), 1.0, torch.bfloat16)           # raw rows
    poolr = g.normal("pool", (int(sum(E)) + B, c), 1.0, torch.bfloat16)
    localr = g.normal("local", (B, R, c), 1.0, torch.bfloat16)
    sink = g.normal("sink", (H,), 1.0)
    # GPU: normalise and rotate every row at its position, then attend with inverse RoPE
    Q = Qr.cuda()
    qpos = torch.tensor([p + i for p in pos0 for i in range(nq)], dtype=torch.int32).cuda()
    dsv4.dsv4_norm_rope(Q, qpos, rows_per_pos=H)
    pool = poolr.cuda()
    ppos = torch.cat([torch.arange(e + 1) * m for e in E]).to(torch.int32).cuda()
    dsv4.dsv4_norm_rope(pool, ppos)
    local = localr.cuda()
    # ring slot r of sequence b holds the position j = r (mod R) nearest below the last query
    lpos = []
    for p in pos0:
        last = p + nq - 1
        lpos += [last - ((last - r) % R) for r in range(R)]
    lpos_t = torch.tensor(lpos, dtype=torch.int32)
    dsv4.dsv4_norm_rope(local, lpos_t.cuda())
    if dense:
        idx = counts = None
    else:
        vis = torch.tensor([[(p + i + 1) // m for i in range(nq)] for p in pos0]).reshape(-1)
        idx, counts = g.random_index_sets(vis, k)
        idx, counts = idx.reshape(B, nq, k), counts.reshape(B, nq)
    ws = None
    if split:
        ws = torch.empty(max(1, dsv4.dsv4_hybrid_sparse_attn_workspace_size(B, nq, H, c)), dtype=torch.uint8,
                         device="cuda")
    Og, Lg = dsv4.dsv4_hybrid_sparse_attn(Q, pool, torch.from_numpy(offs).cuda(),
                                          None if dense else idx.cuda(), None if dense else counts.cuda(),
                                          local, torch.tensor(pos0, dtype=torch.int32).cuda(), m, w,
                                          sink.cuda(), 1 / math.sqrt(c), workspace=ws, rope_dims=64)
    dsv4.dsv4_check_errors()
    # oracle: the s5.2 contract on the raw rows
    lp = lpos_t.numpy().reshape(B, R)
    for b in range(B):
        for i in sorted({0, nq // 2, nq - 1}):
            t = pos0[b] + i
            if dense:
                sel = np.arange((t + 1) // m)
            else:
                sel = idx[b, i, :int(counts[b, i])].numpy().astype(np.int64)
            win = np.arange(max(0, t - w + 1), t + 1)
            ent = np.concatenate([O.as_f64(poolr[int(offs[b]) + sel]), O.as_f64(localr[b, win % R])])
            epos = np.concatenate([sel * m, win])
            assert (lp[b, win % R] == win).all()
            o, lse = O.attend_query_rope(Qr[b, i], t, ent, epos, sink, 1 / math.sqrt(c))
            assert_close(Og[b, i].cpu(), o, "bf16", f"rope O b={b} t={t}", verbose=(i == 0))
            assert_close(Lg[b, i].cpu(), lse, "bf16", f"rope LSE b={b} t={t}")


@pytest.mark.parametrize("path", ["tensor_cores", "cuda_cores"])
def test_rope_contract_prefill_chunk(dsv4, path, monkeypatch):
    """Flash shapes, 200 queries from position 4000 (CSA, random selections of up to 512)."""
    _rope_case(dsv4, B=1, nq=200, pos0=[4000], R=512, m=4, k=512, dense=False, split=False,
               seed=72, simt=path == "cuda_cores", monkeypatch=monkeypatch)


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_rope_contract_decode_split(dsv4, kind, monkeypatch):
    """Decode at contexts near 2^20 (split candidate lists merged by the combine kernel)."""
    pos = [1048575, 700001, 131071, 5000]
    _rope_case(dsv4, B=4, nq=1, pos0=pos, R=128, m=4 if kind == "csa" else 128, k=512,
               dense=kind == "hca", split=True, seed=73, simt=False, monkeypatch=monkeypatch)
