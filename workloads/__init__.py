"""Seeded synthetic inputs for the DeepSeek-V4 hybrid CSA/HCA attention hot path.

This module is shared by the CUDA path's tests/bench and by the fp64 oracle's
tests. It draws random numbers and arranges them into the shapes the method
consumes; it holds none of the method's arithmetic (no visibility rule, no
pooling, no scoring, no softmax). Anything that depends on the method -- for
example how many compressed entries a query may see -- is passed in by the
caller.

Recipe (every tensor has its own derived seed, so any subset of tensors can be
regenerated independently and in any order):

* normal(std)  = torch.randn(..) * std, drawn in fp32, then cast to the
  storage dtype (bf16 rounding is round-to-nearest-even, done by torch).
* uniform(lo, hi) = lo + (hi - lo) * torch.rand(..), fp32.
* "Activations" (compressor entry streams C, local shared-KV rows, main
  queries Q, indexer queries q^I, decode pools) are N(0,1)/sqrt(dim) for the
  V4-shaped configurations and N(0,1) for the tiny configuration, except
  that Q of the tiny configuration is N(0,1)/sqrt(c) as its description
  states.
* Gate logits Z are N(0,1) everywhere; positional biases are N(0, 0.1^2)
  (0.1 read as the standard deviation); indexer head weights w ~ U(0,1);
  sink logits ~ N(0,1) where a configuration has a sink.

The five named presets follow the V4-Flash / V4-Pro shapes of the
"CSA And HCA: Definition, State, And Cost Model" page (section 1, table of
published configurations).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

__all__ = [
    "LayerShape", "PRESETS", "preset", "Generator",
]


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Shape and dtype description of one attention layer invocation."""
    name: str
    kind: str                 # "csa" or "hca"
    dtype: str                # "f32" or "bf16": storage dtype of C, Z, Q, local, pools
    B: int                    # batch (sequences)
    n: int                    # tokens per sequence (prefill)
    H: int                    # main query heads n_h
    c: int                    # shared KV / head dim
    m: int                    # compression ratio (m for CSA, m' for HCA)
    w: int                    # local window
    k: int = 0                # CSA top-k
    H_I: int = 0              # indexer heads n_h^I
    c_I: int = 0              # indexer dim c^I
    index_fp4: bool = False   # indexer operands quantised to FP4 (e2m1 + E4M3 per 16)
    sink: bool = False        # per-head sink logit present
    act_scaled: bool = True   # activations scaled by 1/sqrt(dim)

    @property
    def overlap(self) -> int:
        return 1 if self.kind == "csa" else 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.c)


# The five workloads. Sizes are the V4 shapes; the tiny one is a small CSA+HCA pair.
PRESETS = {
    # tiny fp32 CSA layer and HCA layer (m'=16), batch 1, n=256
    "tiny_csa": LayerShape("tiny_csa", "csa", "f32", B=1, n=256, H=4, c=64, m=4, w=16,
                           k=8, H_I=2, c_I=32, act_scaled=False),
    "tiny_hca": LayerShape("tiny_hca", "hca", "f32", B=1, n=256, H=4, c=64, m=16, w=16,
                           act_scaled=False),
    # V4-Flash CSA prefill, bf16, n=8192, sink
    "flash_csa_prefill": LayerShape("flash_csa_prefill", "csa", "bf16", B=1, n=8192, H=64,
                                    c=512, m=4, w=128, k=512, H_I=64, c_I=128, sink=True),
    # V4-Flash HCA prefill, bf16, batch 2, n=65536, m'=128
    "flash_hca_prefill": LayerShape("flash_hca_prefill", "hca", "bf16", B=2, n=65536, H=64,
                                    c=512, m=128, w=128),
    # V4-Pro CSA prefill, n=131072, H=128, k=1024, FP4 indexer
    "pro_csa_prefill": LayerShape("pro_csa_prefill", "csa", "bf16", B=1, n=131072, H=128,
                                  c=512, m=4, w=128, k=1024, H_I=64, c_I=128,
                                  index_fp4=True),
}


def preset(name: str, **overrides) -> LayerShape:
    """A named preset, optionally with fields replaced (e.g. a smaller n)."""
    return dataclasses.replace(PRESETS[name], **overrides)


# Batched decode: 64 sequences, context lengths uniform in [131072, 1048576],
# four layers alternating CSA (m=4) and HCA (m'=128), V4-Flash shapes.
DECODE_BATCH = dict(B=64, L_lo=131072, L_hi=1048576, H=64, c=512, k=512, w=128,
                    H_I=64, c_I=128, m_csa=4, m_hca=128,
                    layers=("csa", "hca", "csa", "hca"))


_TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


class Generator:
    """Deterministic tensor factory: tensor `tag` of seed `seed` is always the same.

    device: where the tensor is drawn ("cpu" or "cuda"). The same (seed, tag) gives
    different bytes on the two devices (different torch RNG engines), so a test must
    draw on one device and copy.
    """

    def __init__(self, seed: int = 0, device: str = "cpu"):
        self.seed = int(seed)
        self.device = device

    def _gen(self, tag: str) -> torch.Generator:
        # stable 63-bit sub-seed from (seed, tag)
        h = 1469598103934665603
        for ch in f"{self.seed}:{tag}".encode():
            h = ((h ^ ch) * 1099511628211) & ((1 << 63) - 1)
        g = torch.Generator(device=self.device)
        g.manual_seed(h)
        return g

    def normal(self, tag: str, shape: Sequence[int], std: float = 1.0,
               dtype: torch.dtype = torch.float32) -> torch.Tensor:
        x = torch.randn(*shape, generator=self._gen(tag), device=self.device,
                        dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        return x.to(dtype)

    def uniform(self, tag: str, shape: Sequence[int], lo: float = 0.0, hi: float = 1.0,
                dtype: torch.dtype = torch.float32) -> torch.Tensor:
        x = torch.rand(*shape, generator=self._gen(tag), device=self.device,
                       dtype=torch.float32)
        return (x * (hi - lo) + lo).to(dtype)

    def randint(self, tag: str, shape: Sequence[int], lo: int, hi: int) -> torch.Tensor:
        """Integers uniform in [lo, hi] inclusive (int64)."""
        return torch.randint(lo, hi + 1, tuple(shape), generator=self._gen(tag),
                             device=self.device, dtype=torch.int64)

    # ------------------------------------------------------------------ layer inputs
    def compressor_inputs(self, shape: LayerShape, which: str = "main", n: Optional[int] = None):
        """Entry stream C, gate logits Z and positional bias for one compressor instance.

        which="main": width c (CSA: two streams a|b -> 2c columns; HCA: c columns).
        which="index": the CSA indexer-key instance, width c_I, two streams.
        Returns (C [B,n,S*width] storage dtype, Z [B,n,S*width] storage dtype,
        bias [S,m,width] fp32) with S = 2 for CSA, 1 for HCA.
        """
        n = shape.n if n is None else n
        width = shape.c if which == "main" else shape.c_I
        S = 2 if shape.kind == "csa" else 1
        dt = _TORCH_DTYPE[shape.dtype]
        std = (1.0 / math.sqrt(width)) if shape.act_scaled else 1.0
        C = self.normal(f"{which}.C", (shape.B, n, S * width), std, dt)
        Z = self.normal(f"{which}.Z", (shape.B, n, S * width), 1.0, dt)
        bias = self.normal(f"{which}.bias", (S, shape.m, width), 0.1, torch.float32)
        return C, Z, bias

    def queries(self, shape: LayerShape, nq: Optional[int] = None) -> torch.Tensor:
        """Main queries Q [B, nq, H, c] (storage dtype)."""
        nq = shape.n if nq is None else nq
        std = 1.0 / math.sqrt(shape.c)
        return self.normal("Q", (shape.B, nq, shape.H, shape.c), std, _TORCH_DTYPE[shape.dtype])

    def local_kv(self, shape: LayerShape, R: Optional[int] = None) -> torch.Tensor:
        """Uncompressed local shared-KV rows [B, R, c] (R = n for prefill)."""
        R = shape.n if R is None else R
        std = (1.0 / math.sqrt(shape.c)) if shape.act_scaled else 1.0
        return self.normal("local", (shape.B, R, shape.c), std, _TORCH_DTYPE[shape.dtype])

    def index_queries(self, shape: LayerShape, nq: Optional[int] = None):
        """Indexer queries q^I [B, nq, H_I, c_I] (bf16 for bf16 layers) and weights w [B,nq,H_I] fp32."""
        nq = shape.n if nq is None else nq
        std = (1.0 / math.sqrt(shape.c_I)) if shape.act_scaled else 1.0
        qI = self.normal("qI", (shape.B, nq, shape.H_I, shape.c_I), std, _TORCH_DTYPE[shape.dtype])
        w = self.uniform("wI", (shape.B, nq, shape.H_I), 0.0, 1.0)
        return qI, w

    def index_keys(self, shape: LayerShape, rows: int) -> torch.Tensor:
        """Free-standing indexer keys K^I [rows, c_I] (for stage-isolated index tests)."""
        std = (1.0 / math.sqrt(shape.c_I)) if shape.act_scaled else 1.0
        return self.normal("KI", (rows, shape.c_I), std, _TORCH_DTYPE[shape.dtype])

    def pool(self, shape: LayerShape, rows: int, tag: str = "pool") -> torch.Tensor:
        """Free-standing compressed main pool [rows, c] (for stage-isolated attention tests)."""
        std = (1.0 / math.sqrt(shape.c)) if shape.act_scaled else 1.0
        return self.normal(tag, (rows, shape.c), std, _TORCH_DTYPE[shape.dtype])

    def sink(self, shape: LayerShape) -> Optional[torch.Tensor]:
        return self.normal("sink", (shape.H,), 1.0) if shape.sink else None

    # ------------------------------------------------------------------ index sets
    def random_index_sets(self, visible: torch.Tensor, k: int, tag: str = "idx"):
        """Random candidate sets for stage-isolated attention tests.

        visible: int tensor [Q] -- how many entries each query may choose from (the
        caller computes it). For each query, draws a uniformly random subset of size
        min(k, visible) of [0, visible), in random order, padded with -1, on the
        generator's device. Returns (idx int32 [Q, k], counts int32 [Q]).
        """
        dev = self.device
        visible = visible.to(torch.int64).reshape(-1).to(dev)
        Qn = visible.numel()
        idx = torch.full((Qn, k), -1, dtype=torch.int32, device=dev)
        counts = torch.minimum(visible, torch.tensor(k, device=dev)).to(torch.int32)
        if k == 0 or Qn == 0:
            return idx, counts
        emax = int(visible.max().item()) if Qn else 0
        if emax == 0:
            return idx, counts
        g = self._gen(tag)
        chunk = max(1, (1 << 24) // max(emax, 1))
        for q0 in range(0, Qn, chunk):
            q1 = min(Qn, q0 + chunk)
            r = torch.rand(q1 - q0, emax, generator=g, device=dev)
            cols = torch.arange(emax, device=dev).unsqueeze(0)
            r = torch.where(cols < visible[q0:q1].unsqueeze(1), r, torch.full_like(r, 2.0))
            kk = min(k, emax)
            order = torch.argsort(r, dim=1)[:, :kk].to(torch.int32)
            keep = torch.arange(kk, device=dev).unsqueeze(0) < counts[q0:q1].unsqueeze(1)
            idx[q0:q1, :kk] = torch.where(keep, order, torch.full_like(order, -1))
        return idx, counts
