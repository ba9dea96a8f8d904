"""GPU parity of the incremental decode state ("CSA And HCA: Definition, State, And Cost
Model", s7): the ring slot write and the compressor state machine, against the oracle's
state machine on the same seeded token streams, and a whole CSA decode step (ring write,
both compressor states, index top-k, attention) against the oracle chain.
"""
import numpy as np
import pytest
import torch

import oracle as O
from parity_util import assert_close, check_topk_query
from workloads import Generator

pytestmark = pytest.mark.gpu


def _streams(seed, n_tot, S, c, m, dtype):
    g = Generator(seed)
    C = [g.normal(f"C{b}", (n, S * c), 1.0, dtype) for b, n in enumerate(n_tot)]
    Z = [g.normal(f"Z{b}", (n, S * c), 1.0, dtype) for b, n in enumerate(n_tot)]
    bias = g.normal("bias", (S, m, c), 0.1)
    return C, Z, bias


def _restore_tail(C, Z, n0, S, m, c, dtype):
    """Tail state after prefixes of n0[b] tokens: slot p mod T holds position p's rows."""
    T = S * m
    tail = torch.zeros(len(n0), T, 2, S * c, dtype=dtype)
    for b, n in enumerate(n0):
        for p in range(max(0, n - T), n):
            tail[b, p % T, 0], tail[b, p % T, 1] = C[b][p], Z[b][p]
    return tail


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("overlap,m,c", [(True, 4, 512), (True, 4, 128), (False, 128, 512),
                                         (False, 16, 64), (True, 1, 24), (False, 3, 40)])
def test_compress_decode_matches_oracle(dsv4, dtype, overlap, m, c):
    """Three sequences (empty, ragged and block-aligned prefixes) each take one token per
    call across at least two block boundaries; pool rows of entries completed during the
    calls match the oracle's state machine, no other row is touched."""
    S = 2 if overlap else 1
    n0 = [0, 5 * m + 2, 3 * m]
    steps = 2 * m + 3
    n_tot = [a + steps for a in n0]
    C, Z, bias = _streams(7 + m + c, n_tot, S, c, m, dtype)
    E_tot = [n // m for n in n_tot]
    off = np.concatenate([[0], np.cumsum(E_tot)[:-1]]).astype(np.int64)
    sentinel = 1024.0                       # exact in bf16 and fp32
    pool = torch.full((sum(E_tot) + 1, c), sentinel, dtype=dtype, device="cuda")
    tail = _restore_tail(C, Z, n0, S, m, c, dtype).cuda()
    off_d = torch.from_numpy(off).cuda()
    bias_d = bias.cuda()
    for s in range(steps):
        pos = torch.tensor([a + s for a in n0], dtype=torch.int32, device="cuda")
        C_new = torch.stack([C[b][n0[b] + s] for b in range(3)]).cuda()
        Z_new = torch.stack([Z[b][n0[b] + s] for b in range(3)]).cuda()
        dsv4.dsv4_compress_decode(C_new, Z_new, bias_d, tail, pool, off_d, pos, m, overlap)
    dsv4.dsv4_check_errors()
    got = pool.cpu().double().numpy()
    kind = "f32" if dtype == torch.float32 else "bf16"
    for b in range(3):
        st = np.zeros((S * m, 2, S * c))
        want = {}
        for t in range(n_tot[b]):
            e = O.decode_append(st, C[b][t], Z[b][t], bias, t, m, overlap)
            if e is not None:
                want[(t + 1) // m - 1] = e
        first = n0[b] // m                  # entries completed by the prefix
        for i in range(E_tot[b]):
            row = got[off[b] + i]
            if i >= first:
                assert_close(torch.from_numpy(row), want[i], kind, f"b={b} entry {i}")
            else:
                assert (row == sentinel).all(), f"b={b}: prefix entry {i} was written"
    assert (got[-1] == sentinel).all()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("overlap,m,c", [(True, 4, 512), (False, 128, 512), (False, 3, 40)])
def test_compress_decode_equals_prefill_compress(dsv4, dtype, overlap, m, c):
    """Entries completed token by token equal, to the last unit in the last place, the
    ones the prefill compressor computes from the whole stream (same fp32 arithmetic in
    the same position order)."""
    S = 2 if overlap else 1
    n = 3 * m + 1
    C, Z, bias = _streams(99 + m, [n], S, c, m, dtype)
    pool = torch.zeros(n // m, c, dtype=dtype, device="cuda")
    tail = torch.zeros(dsv4.decode_tail_shape(1, c, m, overlap), dtype=dtype, device="cuda")
    off = torch.zeros(1, dtype=torch.int64, device="cuda")
    bias_d = bias.cuda()
    for t in range(n):
        dsv4.dsv4_compress_decode(C[0][t:t + 1].cuda(), Z[0][t:t + 1].cuda(), bias_d, tail, pool,
                                  off, torch.tensor([t], dtype=torch.int32, device="cuda"), m,
                                  overlap)
    ref = dsv4.dsv4_compress(C[0][None].cuda(), Z[0][None].cuda(), bias_d, m, overlap)[0]
    dsv4.dsv4_check_errors()
    a, r = pool.double(), ref.double()
    ulp = 2.0 ** -7 if dtype == torch.bfloat16 else 2.0 ** -22
    assert ((a - r).abs() <= ulp * r.abs() + 1e-30).all()


@pytest.mark.parametrize("dtype,c", [(torch.bfloat16, 512), (torch.float32, 40)])
def test_ring_write(dsv4, dtype, c):
    """Slot pos[b] mod R of each sequence's ring takes the new entry; nothing else changes."""
    B, R = 5, 16
    g = Generator(5)
    local = g.normal("local", (B, R, c), 1.0, dtype).cuda()
    kv = g.normal("kv", (B, c), 1.0, dtype).cuda()
    pos = torch.tensor([0, 15, 16, 37, 1000003], dtype=torch.int32)
    want = local.clone()
    for b in range(B):
        want[b, int(pos[b]) % R] = kv[b]
    dsv4.dsv4_ring_write(kv, local, pos.cuda())
    dsv4.dsv4_check_errors()
    assert torch.equal(local, want)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_state_one_launch_equals_separate_calls(dsv4, dtype):
    """A token's whole state update in one dsv4_decode_state launch (ring writes and the
    compressors of a CSA layer -- main and index keys -- and of an HCA layer, over several
    tokens crossing block boundaries) leaves rings, tails and pools bit-identical to the
    separate dsv4_ring_write / dsv4_compress_decode calls."""
    B, c, cI, R = 3, 128, 32, 8
    n0 = [0, 4 * 33 + 1, 128 * 2 - 3]
    steps = 9
    g = Generator(61)
    layers = [("csa", c, 4, True), ("csa_index", cI, 4, True), ("hca", c, 128, False)]
    state = {}
    for name, ch, m, ov in layers:
        S = 2 if ov else 1
        E = [(a + steps) // m + 1 for a in n0]
        off = torch.tensor(np.concatenate([[0], np.cumsum(E)[:-1]]), dtype=torch.int64)
        state[name] = dict(
            ch=ch, m=m, ov=ov, S=S, off=off.cuda(),
            bias=g.normal(f"bias_{name}", (S, m, ch), 0.1).cuda(),
            tail=g.normal(f"tail_{name}", (B, S * m, 2, S * ch), 1.0, dtype).cuda(),
            pool=g.normal(f"pool_{name}", (sum(E), ch), 1.0, dtype).cuda())
    local = g.normal("local", (B, R, c), 1.0, dtype).cuda()
    ref = {k: {x: v[x].clone() for x in ("tail", "pool")} for k, v in state.items()}
    ref_local = local.clone()
    for s in range(steps):
        pos = torch.tensor([a + s for a in n0], dtype=torch.int32, device="cuda")
        kv = g.normal(f"kv{s}", (B, c), 1.0, dtype).cuda()
        news = {name: (g.normal(f"C{s}{name}", (B, st["S"] * st["ch"]), 1.0, dtype).cuda(),
                       g.normal(f"Z{s}{name}", (B, st["S"] * st["ch"]), 1.0, dtype).cuda())
                for name, st in state.items()}
        jobs = [dsv4.decode_ring_job(kv, local)]
        for name, st in state.items():
            jobs.append(dsv4.decode_compress_job(*news[name], st["bias"], st["tail"], st["pool"],
                                                 st["off"], st["m"], st["ov"]))
        dsv4.dsv4_decode_state(jobs, pos)
        dsv4.dsv4_ring_write(kv, ref_local, pos)
        for name, st in state.items():
            dsv4.dsv4_compress_decode(*news[name], st["bias"], ref[name]["tail"], ref[name]["pool"],
                                      st["off"], pos, st["m"], st["ov"])
    dsv4.dsv4_check_errors()
    assert torch.equal(local, ref_local)
    for name in state:
        assert torch.equal(state[name]["tail"], ref[name]["tail"]), name
        assert torch.equal(state[name]["pool"], ref[name]["pool"]), name


def test_csa_decode_step_chain_fp32(dsv4):
    """Whole CSA decode steps of two sequences (prefixes of 37 and 64 tokens, 9 new tokens
    each): ring write, main and index compressor states, index top-k over the grown pools,
    attention over selected entries ++ window; against the oracle running the same state
    machine and chain in fp64. Queries whose top-k sets differ only by ties are excluded
    from the output comparison."""
    B, H, c, m, w, k, HI, cI, R = 2, 4, 64, 4, 16, 8, 2, 32, 16
    n0, steps = [37, 64], 9
    n_tot = [a + steps for a in n0]
    g = Generator(3)
    C, Z, bias = _streams(11, n_tot, 2, c, m, torch.float32)
    CI, ZI, biasI = _streams(12, n_tot, 2, cI, m, torch.float32)
    kv = [g.normal(f"kv{b}", (n, c), 1.0) for b, n in enumerate(n_tot)]
    Q = [g.normal(f"Q{b}", (n, H, c), c ** -0.5) for b, n in enumerate(n_tot)]
    qI = [g.normal(f"qI{b}", (n, HI, cI), cI ** -0.5) for b, n in enumerate(n_tot)]
    wI = [torch.rand(n, HI, generator=torch.Generator().manual_seed(13 + b)) for b, n in enumerate(n_tot)]
    E_max = [n // m for n in n_tot]
    off = np.concatenate([[0], np.cumsum(E_max)[:-1]]).astype(np.int64)
    off_d = torch.from_numpy(off).cuda()
    # device state after the prefixes: pools from the prefill compressor, tails, rings
    pool = torch.zeros(sum(E_max) + 1, c, device="cuda")
    KIp = torch.zeros(sum(E_max) + 1, cI, device="cuda")
    local = torch.zeros(B, R, c, device="cuda")
    for b in range(B):
        e0 = n0[b] // m
        pool[off[b]:off[b] + e0] = dsv4.dsv4_compress(C[b][None, :n0[b]].cuda(), Z[b][None, :n0[b]].cuda(),
                                                      bias.cuda(), m, True)[0]
        KIp[off[b]:off[b] + e0] = dsv4.dsv4_compress(CI[b][None, :n0[b]].cuda(), ZI[b][None, :n0[b]].cuda(),
                                                     biasI.cuda(), m, True)[0]
        for p in range(max(0, n0[b] - R), n0[b]):
            local[b, p % R] = kv[b][p].cuda()
    tail = _restore_tail(C, Z, n0, 2, m, c, torch.float32).cuda()
    tailI = _restore_tail(CI, ZI, n0, 2, m, cI, torch.float32).cuda()
    # oracle state: the same prefixes through its own state machine
    o_pool = [np.zeros((E_max[b], c)) for b in range(B)]
    o_KI = [np.zeros((E_max[b], cI)) for b in range(B)]
    o_tail = [np.zeros((2 * m, 2, 2 * c)) for _ in range(B)]
    o_tailI = [np.zeros((2 * m, 2, 2 * cI)) for _ in range(B)]
    o_ring = [np.zeros((R, c)) for _ in range(B)]

    def o_token(b, t):
        O.ring_write(o_ring[b], kv[b][t], t)
        e = O.decode_append(o_tail[b], C[b][t], Z[b][t], bias, t, m, True)
        eI = O.decode_append(o_tailI[b], CI[b][t], ZI[b][t], biasI, t, m, True)
        if e is not None:
            o_pool[b][(t + 1) // m - 1], o_KI[b][(t + 1) // m - 1] = e, eI

    for b in range(B):
        for t in range(n0[b]):
            o_token(b, t)
    bias_d, biasI_d = bias.cuda(), biasI.cuda()
    compared = 0
    for s in range(steps):
        ts = [a + s for a in n0]
        pos = torch.tensor(ts, dtype=torch.int32, device="cuda")
        dsv4.dsv4_ring_write(torch.stack([kv[b][ts[b]] for b in range(B)]).cuda(), local, pos)
        dsv4.dsv4_compress_decode(torch.stack([C[b][ts[b]] for b in range(B)]).cuda(),
                                  torch.stack([Z[b][ts[b]] for b in range(B)]).cuda(), bias_d, tail,
                                  pool, off_d, pos, m, True)
        dsv4.dsv4_compress_decode(torch.stack([CI[b][ts[b]] for b in range(B)]).cuda(),
                                  torch.stack([ZI[b][ts[b]] for b in range(B)]).cuda(), biasI_d,
                                  tailI, KIp, off_d, pos, m, True)
        qI_s = torch.stack([qI[b][ts[b]] for b in range(B)])[:, None].cuda()
        w_s = torch.stack([wI[b][ts[b]] for b in range(B)])[:, None].cuda()
        Q_s = torch.stack([Q[b][ts[b]] for b in range(B)])[:, None].cuda()
        emax = max((t + 1) // m for t in ts)
        idx, counts = dsv4.dsv4_index_topk(qI_s, w_s, KIp, off_d, pos, m, k, emax)
        Og, Lg = dsv4.dsv4_hybrid_sparse_attn(Q_s, pool, off_d, idx, counts, local, pos, m, w)
        dsv4.dsv4_check_errors()
        idx_c, cnt_c = idx.cpu().numpy(), counts.cpu().numpy()
        for b in range(B):
            t = ts[b]
            o_token(b, t)
            E_t = (t + 1) // m
            sc = O.index_scores_query(qI[b][t], wI[b][t], o_KI[b][:E_t], t, m)
            check_topk_query(idx_c[b, 0], cnt_c[b, 0], sc, k, what=f"b={b} t={t}")
            o_idx, o_cnt = O.topk_select(sc, k)
            if set(idx_c[b, 0, :cnt_c[b, 0]].tolist()) != set(o_idx[:o_cnt].tolist()):
                continue
            cand = O.candidates(o_pool[b], o_idx, o_cnt, o_ring[b], R, t, w)
            o_ref, l_ref = O.attend_query(Q[b][t], cand)
            assert_close(Og[b, 0], o_ref, "f32", f"O b={b} t={t}")
            assert_close(Lg[b, 0], l_ref, "f32", f"LSE b={b} t={t}")
            compared += 1
    assert compared >= 2 * steps - 2


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_state_packed_emission(dsv4, dtype):
    """The fused state update emitting straight into the production pools: the CSA main-KV
    compressor into an FP8 pool (codes, scales, bf16 RoPE tail) and the index-key compressor
    into an FP4 pool (e2m1 codes, E4M3 scales), beside an HCA compressor into a plain pool.
    Over tokens crossing block boundaries, the FP8 pool is bit-identical to the one
    dsv4_compress_decode_fp8 writes, and the FP4 pool holds exactly the oracle's FP4
    quantisation of the entries dsv4_compress_decode emits (rounded to dtype first); rows not
    completed stay untouched."""
    B, c, cI, rd = 3, 576, 128, 64
    n0 = [0, 4 * 21 + 2, 128 - 3]
    steps = 11
    g = Generator(67)
    E = [(a + steps) // 4 + 1 for a in n0]
    off = torch.tensor(np.concatenate([[0], np.cumsum(E)[:-1]]), dtype=torch.int64).cuda()
    rows = sum(E)
    b_main, b_idx = g.normal("b_main", (2, 4, c), 0.1).cuda(), g.normal("b_idx", (2, 4, cI), 0.1).cuda()
    t_main = g.normal("t_main", (B, 8, 2, 2 * c), 1.0, dtype).cuda()
    t_idx = g.normal("t_idx", (B, 8, 2, 2 * cI), 1.0, dtype).cuda()
    codes8 = torch.full((rows, c - rd), 0x5A, dtype=torch.uint8, device="cuda")
    scales8 = torch.full((rows, (c - rd) // 64), -1.0, device="cuda")
    rope8 = torch.full((rows, rd), -7.0, dtype=torch.bfloat16, device="cuda")
    codes4 = torch.full((rows, cI // 2), 0xA5, dtype=torch.uint8, device="cuda")
    scales4 = torch.full((rows, cI // 16), 0x3C, dtype=torch.uint8, device="cuda")
    ref8 = (codes8.clone(), scales8.clone(), rope8.clone())
    ref_tmain, ref_tidx = t_main.clone(), t_idx.clone()
    plain_idx = torch.full((rows, cI), 1024.0, dtype=dtype, device="cuda")  # sentinel rows
    for s in range(steps):
        pos = torch.tensor([a + s for a in n0], dtype=torch.int32, device="cuda")
        Cm, Zm = (g.normal(f"{n}m{s}", (B, 2 * c), 1.0, dtype).cuda() for n in "CZ")
        Ci, Zi = (g.normal(f"{n}i{s}", (B, 2 * cI), 1.0, dtype).cuda() for n in "CZ")
        jobs = [dsv4.decode_compress_fp8_job(Cm, Zm, b_main, t_main, codes8, scales8, rope8, off, 4,
                                             True, rd),
                dsv4.decode_compress_fp4_job(Ci, Zi, b_idx, t_idx, codes4, scales4, off, 4, True)]
        dsv4.dsv4_decode_state(jobs, pos)
        dsv4.dsv4_compress_decode_fp8(Cm, Zm, b_main, ref_tmain, *ref8, off, pos, 4, True)
        dsv4.dsv4_compress_decode(Ci, Zi, b_idx, ref_tidx, plain_idx, off, pos, 4, True)
    dsv4.dsv4_check_errors()
    assert torch.equal(t_main, ref_tmain) and torch.equal(t_idx, ref_tidx)
    for got, want, name in zip((codes8, scales8, rope8), ref8, ("codes", "scales", "rope")):
        assert torch.equal(got, want), f"FP8 {name}"
    written = (plain_idx != 1024.0).any(dim=1).cpu().numpy()
    assert written.sum() == sum((a + steps) // 4 - a // 4 for a in n0)
    rc, rs = O.quantize_fp4(plain_idx.float().cpu()[written])
    gc, gs = codes4.cpu().numpy(), scales4.cpu().numpy()
    np.testing.assert_array_equal(gs[written], rs)
    np.testing.assert_array_equal(gc[written], rc)
    assert (gc[~written] == 0xA5).all() and (gs[~written] == 0x3C).all()
