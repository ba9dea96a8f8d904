"""A decode step captured once in a CUDA graph and replayed gives what the same calls give
when launched one by one: every call of the path only enqueues work on the caller's stream
(no host synchronisation, allocation or host-side decision on device data), so a serving loop
can replay a token's whole step as one graph. The step: the fused state update of a CSA and an
HCA layer, the CSA index top-k (threshold pipeline with dynamically scheduled score units, over
bf16 and over FP4 keys) and attention of both layers (split lists for HCA).
"""
import math

import numpy as np
import pytest
import torch

from workloads import Generator

pytestmark = pytest.mark.gpu


def _setup(dsv4, fp4):
    g = Generator(71, device="cuda")
    B, H, c, k, w, HI, cI = 6, 64, 512, 256, 32, 64, 128
    L = torch.tensor([70001, 133, 90003, 4 * 16384 + 7, 20000, 999], dtype=torch.int64)
    E4, E128 = (L // 4).tolist(), (L // 128).tolist()
    off4 = torch.tensor(np.concatenate([[0], np.cumsum(E4)[:-1]]), dtype=torch.int64, device="cuda")
    off128 = torch.tensor(np.concatenate([[0], np.cumsum(E128)[:-1]]), dtype=torch.int64, device="cuda")
    pos = (L - 1).to(torch.int32).cuda()
    t = dict(B=B, H=H, c=c, k=k, w=w, HI=HI, cI=cI, pos=pos, off4=off4, off128=off128,
             maxE=max(E4))
    t["pool4"] = g.normal("pool4", (sum(E4) + 1, c), c ** -0.5, torch.bfloat16)
    t["pool128"] = g.normal("pool128", (sum(E128) + 1, c), c ** -0.5, torch.bfloat16)
    KI = g.normal("KI", (sum(E4) + 1, cI), cI ** -0.5, torch.bfloat16)
    qI = g.normal("qI", (B, 1, HI, cI), cI ** -0.5, torch.bfloat16)
    if fp4:
        t["KI"], t["KI_sc"] = dsv4.dsv4_quantize_fp4(KI)
        qc, t["qI_sc"] = dsv4.dsv4_quantize_fp4(qI.reshape(-1, cI))
        t["qI"] = qc.view(B, 1, HI, cI // 2)
        qd = dsv4.FP4
    else:
        t["KI"], t["qI"], t["KI_sc"], t["qI_sc"] = KI, qI, None, None
        qd = dsv4.BF16
    t["wI"] = g.uniform("wI", (B, 1, HI))
    t["Q"] = g.normal("Q", (B, 1, H, c), c ** -0.5, torch.bfloat16)
    t["local"] = g.normal("local", (B, w, c), c ** -0.5, torch.bfloat16)
    t["sink"] = g.normal("sink", (H,), 1.0)
    t["kv"] = g.normal("kv", (B, c), c ** -0.5, torch.bfloat16)
    t["C4"], t["Z4"] = g.normal("C4", (B, 2 * c), 1.0, torch.bfloat16), g.normal("Z4", (B, 2 * c), 1.0, torch.bfloat16)
    t["C128"], t["Z128"] = g.normal("C128", (B, c), 1.0, torch.bfloat16), g.normal("Z128", (B, c), 1.0, torch.bfloat16)
    t["b4"], t["b128"] = g.normal("b4", (2, 4, c), 0.1), g.normal("b128", (1, 128, c), 0.1)
    t["tail4"] = g.normal("tail4", dsv4.decode_tail_shape(B, c, 4, True), 1.0, torch.bfloat16)
    t["tail128"] = g.normal("tail128", dsv4.decode_tail_shape(B, c, 128, False), 1.0, torch.bfloat16)
    t["ws"] = torch.empty(dsv4.dsv4_index_topk_workspace_size_ex(qd, B, 1, HI, cI, t["maxE"], k,
                                                                   t["KI"].shape[0]),
                          dtype=torch.uint8, device="cuda")
    t["aws"] = torch.empty(max(1, dsv4.dsv4_hybrid_sparse_attn_workspace_size(B, 1, H, c)),
                           dtype=torch.uint8, device="cuda")
    t["idx"] = torch.empty(B, 1, k, dtype=torch.int32, device="cuda")
    t["cnt"] = torch.empty(B, 1, dtype=torch.int32, device="cuda")
    t["O4"], t["O128"] = torch.empty_like(t["Q"]), torch.empty_like(t["Q"])
    t["lse4"], t["lse128"] = (torch.empty(B, 1, H, device="cuda") for _ in range(2))
    return t


def _step(dsv4, t):
    """State update (ring + CSA and HCA compressors, one launch), then index top-k and the
    two attention layers. Every output is written into preallocated buffers."""
    jobs = [dsv4.decode_ring_job(t["kv"], t["local"]),
            dsv4.decode_compress_job(t["C4"], t["Z4"], t["b4"], t["tail4"], t["pool4"], t["off4"], 4, True),
            dsv4.decode_compress_job(t["C128"], t["Z128"], t["b128"], t["tail128"], t["pool128"],
                                     t["off128"], 128, False)]
    dsv4.dsv4_decode_state(jobs, t["pos"])
    dsv4.dsv4_index_topk(t["qI"], t["wI"], t["KI"], t["off4"], t["pos"], 4, t["k"], t["maxE"],
                         qI_scales=t["qI_sc"], KI_scales=t["KI_sc"], c_I=t["cI"], idx=t["idx"],
                         counts=t["cnt"], workspace=t["ws"])
    dsv4.dsv4_hybrid_sparse_attn(t["Q"], t["pool4"], t["off4"], t["idx"], t["cnt"], t["local"], t["pos"], 4,
                                 t["w"], t["sink"], 1 / math.sqrt(t["c"]), O=t["O4"], lse=t["lse4"],
                                 workspace=t["aws"])
    dsv4.dsv4_hybrid_sparse_attn(t["Q"], t["pool128"], t["off128"], None, None, t["local"], t["pos"], 128,
                                 t["w"], None, 1 / math.sqrt(t["c"]), O=t["O128"], lse=t["lse128"],
                                 workspace=t["aws"])


OUTS = ("idx", "cnt", "O4", "lse4", "O128", "lse128", "local", "tail4", "tail128", "pool4", "pool128")


@pytest.mark.parametrize("fp4", [False, True])
def test_decode_step_graph_replay_equals_eager(dsv4, fp4):
    t = _setup(dsv4, fp4)
    start = {n: t[n].clone() for n in ("local", "tail4", "tail128", "pool4", "pool128")}
    _step(dsv4, t)                                  # eager (also sets kernel attributes)
    torch.cuda.synchronize()
    dsv4.dsv4_check_errors()
    eager = {n: t[n].clone() for n in OUTS}
    for n, v in start.items():                      # the state update runs again from the start
        t[n].copy_(v)
    for n in ("idx", "cnt", "O4", "lse4", "O128", "lse128"):
        t[n].zero_()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            _step(dsv4, t)
    torch.cuda.current_stream().wait_stream(side)
    for n, v in start.items():                      # capture enqueued nothing; reset anyway
        t[n].copy_(v)
    graph.replay()
    torch.cuda.synchronize()
    dsv4.dsv4_check_errors()
    for n in OUTS:
        assert torch.equal(t[n], eager[n]), f"{n} differs after graph replay (fp4={fp4})"
    del graph
