"""Python binding of libdsv4 (the C ABI declared in include/dsv4.h).

Argument marshalling only: every function takes torch tensors that already live on
the CUDA device, checks dtype / shape / contiguity, allocates missing outputs with
torch (device memory is PyTorch's job here), and calls the C entry point of the same
name on the current torch stream. All arithmetic happens in the library's CUDA
kernels. If the library is missing, importing this package fails loudly; there is no
CPU fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

__all__ = [
    "DSV4Error", "lib", "LIB_PATH", "F32", "BF16", "FP4",
    "dsv4_compress", "dsv4_compress_decode", "dsv4_ring_write", "decode_tail_shape",
    "dsv4_decode_state", "decode_ring_job", "decode_compress_job", "decode_compress_fp8_job",
    "decode_compress_fp4_job",
    "dsv4_quantize_fp4", "dsv4_index_topk", "dsv4_index_topk_workspace_size",
    "dsv4_index_topk_workspace_size_ex",
    "dsv4_hybrid_sparse_attn", "dsv4_hybrid_sparse_attn_workspace_size", "dsv4_check_errors",
    "dsv4_norm_rope", "dsv4_quantize_main_kv", "dsv4_dequantize_main_kv",
    "dsv4_compress_decode_fp8", "dsv4_hybrid_sparse_attn_fp8",
    "dsv4_hybrid_sparse_attn_fp8_workspace_size",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdsv4.so")
F32, BF16, FP4 = 0, 1, 2

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libdsv4.so not found at {LIB_PATH}: build it with "
        "`python compressed_sparse_mqa_dsv4_b200/build.py` (nvcc, sm_100a)")

lib = ctypes.CDLL(LIB_PATH)

_P, _I, _L, _F, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
lib.dsv4_abi_version.restype = _I
lib.dsv4_status_string.restype = ctypes.c_char_p
lib.dsv4_status_string.argtypes = [_I]
lib.dsv4_last_error_message.restype = ctypes.c_char_p
lib.dsv4_check_errors.restype = _I
lib.dsv4_check_errors.argtypes = [_P]
lib.dsv4_compress.restype = _I
lib.dsv4_compress.argtypes = [_I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]
lib.dsv4_compress_decode.restype = _I
lib.dsv4_compress_decode.argtypes = [_I, _P, _P, _P, _P, _P, _P, _L, _P, _I, _I, _I, _I, _P]
lib.dsv4_ring_write.restype = _I
lib.dsv4_ring_write.argtypes = [_I, _P, _P, _I, _P, _I, _I, _P]


class _DecodeJob(ctypes.Structure):
    """dsv4_decode_job of include/dsv4.h."""
    _fields_ = [("kind", ctypes.c_int), ("c", ctypes.c_int), ("m", ctypes.c_int),
                ("overlap", ctypes.c_int), ("R", ctypes.c_int), ("rope_dims", ctypes.c_int),
                ("x_new", ctypes.c_void_p), ("z_new", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("tail", ctypes.c_void_p), ("out", ctypes.c_void_p), ("out_scales", ctypes.c_void_p),
                ("out_rope", ctypes.c_void_p), ("pool_row_off", ctypes.c_void_p),
                ("pool_rows", ctypes.c_int64)]


DECODE_MAX_JOBS = 32
lib.dsv4_decode_state.restype = _I
lib.dsv4_decode_state.argtypes = [_I, ctypes.POINTER(_DecodeJob), _I, _P, _I, _P]
lib.dsv4_quantize_fp4.restype = _I
lib.dsv4_quantize_fp4.argtypes = [_P, _P, _P, _L, _I, _P]
lib.dsv4_index_topk_workspace_size.restype = _S
lib.dsv4_index_topk_workspace_size.argtypes = [_I, _I, _I, _I]
lib.dsv4_index_topk_workspace_size_ex.restype = _S
lib.dsv4_index_topk_workspace_size_ex.argtypes = [_I, _I, _I, _I, _I, _I, _I, _L]
lib.dsv4_index_topk.restype = _I
lib.dsv4_index_topk.argtypes = [_I, _P, _P, _P, _P, _P, _L, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                _P, _P, _P, _L, _P, _S, _P]
lib.dsv4_index_topk_noalloc.restype = _I
lib.dsv4_index_topk_noalloc.argtypes = [_I, _P, _P, _P, _P, _P, _L, _P, _P, _I, _I, _I, _I, _I, _I,
                                        _I, _P, _P, _P]
lib.dsv4_hybrid_sparse_attn.restype = _I
lib.dsv4_hybrid_sparse_attn.argtypes = [_I, _P, _P, _L, _P, _P, _P, _I, _P, _I, _P, _I, _I, _I,
                                        _I, _I, _I, _P, _F, _P, _P, _P, _S, _P]
lib.dsv4_hybrid_sparse_attn_rope.restype = _I
lib.dsv4_hybrid_sparse_attn_rope.argtypes = lib.dsv4_hybrid_sparse_attn.argtypes[:-1] + [_I, _P]
lib.dsv4_norm_rope.restype = _I
lib.dsv4_norm_rope.argtypes = [_I, _P, _P, _L, _I, _I, _I, _I, _I, _F, _P]
lib.dsv4_quantize_main_kv.restype = _I
lib.dsv4_quantize_main_kv.argtypes = [_I, _P, _P, _P, _P, _L, _I, _I, _P]
lib.dsv4_dequantize_main_kv.restype = _I
lib.dsv4_dequantize_main_kv.argtypes = [_P, _P, _P, _P, _L, _I, _I, _P]
lib.dsv4_compress_decode_fp8.restype = _I
lib.dsv4_compress_decode_fp8.argtypes = [_I, _P, _P, _P, _P, _P, _P, _P, _I, _P, _L, _P, _I, _I, _I,
                                         _I, _P]
lib.dsv4_hybrid_sparse_attn_fp8_workspace_size.restype = _S
lib.dsv4_hybrid_sparse_attn_fp8_workspace_size.argtypes = [_I, _I, _I, _I]
lib.dsv4_hybrid_sparse_attn_fp8.restype = _I
lib.dsv4_hybrid_sparse_attn_fp8.argtypes = [_P, _P, _P, _P, _L, _P, _P, _P, _I, _P, _I, _P, _I, _I,
                                            _I, _I, _I, _I, _P, _F, _P, _P, _P, _S, _P]
lib.dsv4_hybrid_sparse_attn_workspace_size.restype = _S
lib.dsv4_hybrid_sparse_attn_workspace_size.argtypes = [_I, _I, _I, _I]


class DSV4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.dsv4_last_error_message().decode(errors="replace")
        name = lib.dsv4_status_string(status).decode()
        super().__init__(f"{where}: {name} ({status}): {msg}")


def _check(status: int, where: str):
    if status != 0:
        raise DSV4Error(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def _code(dtype: torch.dtype) -> int:
    if dtype == torch.float32:
        return F32
    if dtype == torch.bfloat16:
        return BF16
    raise ValueError(f"unsupported dtype {dtype}")


def dsv4_compress(C: torch.Tensor, Z: torch.Tensor, bias: torch.Tensor, m: int, overlap: bool,
                  out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Compressor: C, Z [B, n, S*c], bias fp32 [S, m, c] -> out [B, n//m, c]."""
    _dev(C, "C"), _dev(Z, "Z", C.dtype), _dev(bias, "bias", torch.float32)
    B, n, width = C.shape
    S = 2 if overlap else 1
    c = width // S
    if out is None:
        out = torch.empty(B, n // m, c, dtype=C.dtype, device=C.device)
    _dev(out, "out", C.dtype)
    _check(lib.dsv4_compress(_code(C.dtype), _ptr(C), _ptr(Z), _ptr(bias), _ptr(out), B, n, c, m,
                             1 if overlap else 0, _stream(stream)), "dsv4_compress")
    return out


def decode_tail_shape(B: int, c: int, m: int, overlap: bool):
    """Shape of the compressor tail state of dsv4_compress_decode: [B, S*m, 2, S*c]."""
    S = 2 if overlap else 1
    return (B, S * m, 2, S * c)


def dsv4_compress_decode(C_new: torch.Tensor, Z_new: torch.Tensor, bias: torch.Tensor,
                         tail: torch.Tensor, pool: torch.Tensor, pool_row_off: torch.Tensor,
                         pos: torch.Tensor, m: int, overlap: bool, stream=None) -> None:
    """One decode token per sequence: C_new, Z_new [B, S*c] into the tail
    [B, S*m, 2, S*c]; completed entries are written to pool [rows, c] in place."""
    _dev(C_new, "C_new"), _dev(Z_new, "Z_new", C_new.dtype), _dev(bias, "bias", torch.float32)
    B, width = C_new.shape
    S = 2 if overlap else 1
    c = width // S
    _dev(tail, "tail", C_new.dtype), _dev(pool, "pool", C_new.dtype)
    _dev(pool_row_off, "pool_row_off", torch.int64), _dev(pos, "pos", torch.int32)
    if tuple(tail.shape) != decode_tail_shape(B, c, m, overlap):
        raise ValueError(f"tail must be {decode_tail_shape(B, c, m, overlap)}, got {tuple(tail.shape)}")
    if pool.shape[-1] != c:
        raise ValueError(f"pool rows must have {c} channels")
    _check(lib.dsv4_compress_decode(_code(C_new.dtype), _ptr(C_new), _ptr(Z_new), _ptr(bias),
                                    _ptr(tail), _ptr(pool), _ptr(pool_row_off),
                                    pool.numel() // c, _ptr(pos), B, c, m, 1 if overlap else 0,
                                    _stream(stream)), "dsv4_compress_decode")


def dsv4_ring_write(kv_new: torch.Tensor, local: torch.Tensor, pos: torch.Tensor,
                    stream=None) -> None:
    """kv_new [B, c] into slot pos[b] mod R of local [B, R, c], in place."""
    _dev(kv_new, "kv_new"), _dev(local, "local", kv_new.dtype), _dev(pos, "pos", torch.int32)
    B, c = kv_new.shape
    if local.shape[0] != B or local.shape[2] != c:
        raise ValueError(f"local must be [{B}, R, {c}]")
    _check(lib.dsv4_ring_write(_code(kv_new.dtype), _ptr(kv_new), _ptr(local), local.shape[1],
                               _ptr(pos), B, c, _stream(stream)), "dsv4_ring_write")


def decode_ring_job(kv_new: torch.Tensor, local: torch.Tensor):
    """A dsv4_decode_state job: the dsv4_ring_write of kv_new [B, c] into local [B, R, c]."""
    _dev(kv_new, "kv_new"), _dev(local, "local", kv_new.dtype)
    B, c = kv_new.shape
    if local.shape[0] != B or local.shape[2] != c:
        raise ValueError(f"local must be [{B}, R, {c}]")
    job = _DecodeJob(kind=0, c=c, m=0, overlap=0, R=local.shape[1], rope_dims=0,
                     x_new=kv_new.data_ptr(), z_new=None, bias=None, tail=None, out=local.data_ptr(),
                     pool_row_off=None, pool_rows=0)
    return job, kv_new.dtype, B, (kv_new, local)


def decode_compress_job(C_new: torch.Tensor, Z_new: torch.Tensor, bias: torch.Tensor,
                        tail: torch.Tensor, pool: torch.Tensor, pool_row_off: torch.Tensor,
                        m: int, overlap: bool):
    """A dsv4_decode_state job: the dsv4_compress_decode of one compressor (same arguments)."""
    _dev(C_new, "C_new"), _dev(Z_new, "Z_new", C_new.dtype), _dev(bias, "bias", torch.float32)
    B, width = C_new.shape
    S = 2 if overlap else 1
    c = width // S
    _dev(tail, "tail", C_new.dtype), _dev(pool, "pool", C_new.dtype)
    _dev(pool_row_off, "pool_row_off", torch.int64)
    if tuple(tail.shape) != decode_tail_shape(B, c, m, overlap):
        raise ValueError(f"tail must be {decode_tail_shape(B, c, m, overlap)}, got {tuple(tail.shape)}")
    if pool.shape[-1] != c:
        raise ValueError(f"pool rows must have {c} channels")
    job = _DecodeJob(kind=1, c=c, m=m, overlap=1 if overlap else 0, R=0, rope_dims=0,
                     x_new=C_new.data_ptr(), z_new=Z_new.data_ptr(), bias=bias.data_ptr(), tail=tail.data_ptr(),
                     out=pool.data_ptr(), pool_row_off=pool_row_off.data_ptr(), pool_rows=pool.numel() // c)
    return job, C_new.dtype, B, (C_new, Z_new, bias, tail, pool, pool_row_off)


def _compress_common(C_new, Z_new, bias, tail, pool_row_off, m, overlap):
    _dev(C_new, "C_new"), _dev(Z_new, "Z_new", C_new.dtype), _dev(bias, "bias", torch.float32)
    B, width = C_new.shape
    c = width // (2 if overlap else 1)
    _dev(tail, "tail", C_new.dtype), _dev(pool_row_off, "pool_row_off", torch.int64)
    if tuple(tail.shape) != decode_tail_shape(B, c, m, overlap):
        raise ValueError(f"tail must be {decode_tail_shape(B, c, m, overlap)}, got {tuple(tail.shape)}")
    return B, c


def decode_compress_fp8_job(C_new: torch.Tensor, Z_new: torch.Tensor, bias: torch.Tensor,
                            tail: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
                            rope: Optional[torch.Tensor], pool_row_off: torch.Tensor, m: int,
                            overlap: bool, rope_dims: int = 64):
    """A dsv4_decode_state job: the compressor token of dsv4_compress_decode_fp8 (the entry into
    the FP8 main-KV pool: codes uint8 [rows, c - rope_dims], scales fp32 [rows, (c-rope)/64],
    rope bf16 [rows, rope_dims])."""
    B, c = _compress_common(C_new, Z_new, bias, tail, pool_row_off, m, overlap)
    _dev(codes, "codes", torch.uint8), _dev(scales, "scales", torch.float32)
    if rope_dims:
        if rope is None:
            raise ValueError(f"rope must be given for rope_dims={rope_dims}")
        _dev(rope, "rope", torch.bfloat16)
    if codes.shape[-1] != c - rope_dims:
        raise ValueError(f"codes rows must have {c - rope_dims} bytes")
    job = _DecodeJob(kind=2, c=c, m=m, overlap=1 if overlap else 0, R=0, rope_dims=rope_dims,
                     x_new=C_new.data_ptr(), z_new=Z_new.data_ptr(), bias=bias.data_ptr(),
                     tail=tail.data_ptr(), out=codes.data_ptr(), out_scales=scales.data_ptr(),
                     out_rope=rope.data_ptr() if rope_dims else None,
                     pool_row_off=pool_row_off.data_ptr(), pool_rows=codes.shape[0])
    return job, C_new.dtype, B, (C_new, Z_new, bias, tail, codes, scales, rope, pool_row_off)


def decode_compress_fp4_job(C_new: torch.Tensor, Z_new: torch.Tensor, bias: torch.Tensor,
                            tail: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
                            pool_row_off: torch.Tensor, m: int, overlap: bool):
    """A dsv4_decode_state job: the compressor token with the entry emitted into an FP4 pool
    (the index keys: codes uint8 [rows, c/2], E4M3 scales uint8 [rows, c/16]), rounded to the
    input dtype and quantised as dsv4_quantize_fp4 quantises that row."""
    B, c = _compress_common(C_new, Z_new, bias, tail, pool_row_off, m, overlap)
    _dev(codes, "codes", torch.uint8), _dev(scales, "scales", torch.uint8)
    if codes.shape[-1] != c // 2 or scales.shape[-1] != c // 16:
        raise ValueError(f"FP4 pool rows must be {c // 2} code bytes and {c // 16} scales")
    job = _DecodeJob(kind=3, c=c, m=m, overlap=1 if overlap else 0, R=0, rope_dims=0,
                     x_new=C_new.data_ptr(), z_new=Z_new.data_ptr(), bias=bias.data_ptr(),
                     tail=tail.data_ptr(), out=codes.data_ptr(), out_scales=scales.data_ptr(),
                     out_rope=None, pool_row_off=pool_row_off.data_ptr(), pool_rows=codes.shape[0])
    return job, C_new.dtype, B, (C_new, Z_new, bias, tail, codes, scales, pool_row_off)


def dsv4_decode_state(jobs, pos: torch.Tensor, stream=None) -> None:
    """One launch for a token's ring writes and compressor states: `jobs` from decode_ring_job,
    decode_compress_job, decode_compress_fp8_job or decode_compress_fp4_job (same dtype and
    batch; no two jobs writing the same memory), pos int32 [B]."""
    _dev(pos, "pos", torch.int32)
    if not jobs:
        return
    if len(jobs) > DECODE_MAX_JOBS:
        raise ValueError(f"at most {DECODE_MAX_JOBS} jobs per call")
    dtypes = {j[1] for j in jobs}
    batches = {j[2] for j in jobs}
    if len(dtypes) != 1 or batches != {pos.shape[0]}:
        raise ValueError("jobs must share one dtype and the batch of pos")
    arr = (_DecodeJob * len(jobs))(*[j[0] for j in jobs])
    _check(lib.dsv4_decode_state(_code(next(iter(dtypes))), arr, len(jobs), _ptr(pos), pos.shape[0],
                                 _stream(stream)), "dsv4_decode_state")


def dsv4_quantize_fp4(x: torch.Tensor, codes: Optional[torch.Tensor] = None,
                      scales: Optional[torch.Tensor] = None, stream=None):
    """bf16 [rows, cols] -> (codes uint8 [rows, cols/2], scales uint8 [rows, cols/16])."""
    _dev(x, "x", torch.bfloat16)
    cols = x.shape[-1]
    rows = x.numel() // max(cols, 1)
    if codes is None:
        codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(rows, cols // 16, dtype=torch.uint8, device=x.device)
    _check(lib.dsv4_quantize_fp4(_ptr(x), _ptr(codes), _ptr(scales), rows, cols, _stream(stream)),
           "dsv4_quantize_fp4")
    return codes, scales


def dsv4_index_topk_workspace_size(B: int, nq: int, max_entries: int, k: int) -> int:
    return int(lib.dsv4_index_topk_workspace_size(B, nq, max_entries, k))


def dsv4_index_topk_workspace_size_ex(qdtype: int, B: int, nq: int, H_I: int, c_I: int,
                                      max_entries: int, k: int, ki_rows: int) -> int:
    return int(lib.dsv4_index_topk_workspace_size_ex(qdtype, B, nq, H_I, c_I, max_entries, k,
                                                     ki_rows))


def dsv4_index_topk(qI: torch.Tensor, w: torch.Tensor, KI: torch.Tensor,
                    kv_row_off: torch.Tensor, q_pos0: torch.Tensor, m: int, k: int,
                    max_entries: int, qI_scales: Optional[torch.Tensor] = None,
                    KI_scales: Optional[torch.Tensor] = None, H_I: Optional[int] = None,
                    c_I: Optional[int] = None, idx: Optional[torch.Tensor] = None,
                    counts: Optional[torch.Tensor] = None,
                    scores_out: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None, stream=None):
    """Indexer scores + TopK. Returns (idx int32 [B, nq, k], counts int32 [B, nq]).

    qI: [B, nq, H_I, c_I] fp32/bf16, or FP4 codes uint8 [B, nq, H_I, c_I/2] with qI_scales.
    KI: [rows, c_I] fp32/bf16, or FP4 codes uint8 [rows, c_I/2] with KI_scales.
    """
    fp4 = qI.dtype == torch.uint8
    _dev(qI, "qI"), _dev(w, "w", torch.float32), _dev(KI, "KI", qI.dtype)
    _dev(kv_row_off, "kv_row_off", torch.int64), _dev(q_pos0, "q_pos0", torch.int32)
    B, nq = qI.shape[0], qI.shape[1]
    H_I = qI.shape[2] if H_I is None else H_I
    c_I = (qI.shape[3] * (2 if fp4 else 1)) if c_I is None else c_I
    qd = FP4 if fp4 else _code(qI.dtype)
    if fp4:
        _dev(qI_scales, "qI_scales", torch.uint8), _dev(KI_scales, "KI_scales", torch.uint8)
    ki_rows = KI.shape[0]
    if idx is None:
        idx = torch.empty(B, nq, k, dtype=torch.int32, device=qI.device)
    if counts is None:
        counts = torch.empty(B, nq, dtype=torch.int32, device=qI.device)
    scores_ld = 0
    if scores_out is not None:
        _dev(scores_out, "scores_out", torch.float32)
        scores_ld = scores_out.shape[-1]
    ws_bytes = dsv4_index_topk_workspace_size_ex(qd, B, nq, H_I, c_I, max_entries, k, ki_rows)
    if scores_out is not None and fp4:
        # room for the bf16 expansion of K^I and of every query's q^I (one chunk)
        ws_bytes = ki_rows * c_I * 2 + B * nq * H_I * c_I * 2 + 1024
    elif scores_out is not None:
        ws_bytes = 0
    if ws_bytes and (workspace is None or workspace.numel() < ws_bytes):
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=qI.device)
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(lib.dsv4_index_topk(qd, _ptr(qI), _ptr(qI_scales), _ptr(w), _ptr(KI), _ptr(KI_scales),
                               ki_rows, _ptr(kv_row_off), _ptr(q_pos0), B, nq, H_I, c_I, m, k,
                               max_entries, _ptr(idx), _ptr(counts), _ptr(scores_out), scores_ld,
                               _ptr(workspace), ws_bytes, _stream(stream)), "dsv4_index_topk")
    return idx, counts


def dsv4_hybrid_sparse_attn(Q: torch.Tensor, pool: torch.Tensor, kv_row_off: torch.Tensor,
                            idx: Optional[torch.Tensor], counts: Optional[torch.Tensor],
                            local: torch.Tensor, q_pos0: torch.Tensor, m: int, w: int,
                            sink: Optional[torch.Tensor] = None, scale: Optional[float] = None,
                            O: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                            want_lse: bool = True, workspace: Optional[torch.Tensor] = None,
                            rope_dims: int = 0, stream=None):
    """Hybrid shared-KV MQA. Q [B, nq, H, c]; pool [rows, c]; local [B, R, c].

    idx/counts: int32 [B, nq, k] / [B, nq] (CSA) or None (HCA dense read with ratio m).
    Returns (O [B, nq, H, c], lse fp32 [B, nq, H] or None).
    workspace: uint8 device scratch for split candidate lists (decode); allocated here when
    the request would use it and none is given.
    rope_dims > 0: the output's last rope_dims channels are rotated back by each query's
    position (dsv4_hybrid_sparse_attn_rope).
    """
    _dev(Q, "Q"), _dev(pool, "pool", Q.dtype), _dev(local, "local", Q.dtype)
    _dev(kv_row_off, "kv_row_off", torch.int64), _dev(q_pos0, "q_pos0", torch.int32)
    B, nq, H, c = Q.shape
    R = local.shape[1]
    k = 0
    idx_p = None
    if idx is not None:
        _dev(idx, "idx", torch.int32), _dev(counts, "counts", torch.int32)
        k = idx.shape[-1]
        # k == 0 (window only): torch gives an empty tensor a NULL pointer, which the ABI
        # reads as the dense mode; hand over a valid pointer that is never dereferenced.
        idx_p = _ptr(idx) if idx.numel() > 0 else _ptr(counts)
    if sink is not None:
        _dev(sink, "sink", torch.float32)
    if scale is None:
        scale = 1.0 / math.sqrt(c)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None and want_lse:
        lse = torch.empty(B, nq, H, dtype=torch.float32, device=Q.device)
    ws_bytes = dsv4_hybrid_sparse_attn_workspace_size(B, nq, H, c)
    if ws_bytes and (workspace is None or workspace.numel() < ws_bytes):
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=Q.device)
    ws_bytes = workspace.numel() if workspace is not None else 0
    args = (_code(Q.dtype), _ptr(Q), _ptr(pool), pool.shape[0], _ptr(kv_row_off), idx_p,
            _ptr(counts), k, _ptr(local), R, _ptr(q_pos0), B, nq, H, c, m, w, _ptr(sink),
            float(scale), _ptr(O), _ptr(lse), _ptr(workspace), ws_bytes)
    if rope_dims:
        _check(lib.dsv4_hybrid_sparse_attn_rope(*args, rope_dims, _stream(stream)),
               "dsv4_hybrid_sparse_attn_rope")
    else:
        _check(lib.dsv4_hybrid_sparse_attn(*args, _stream(stream)), "dsv4_hybrid_sparse_attn")
    return O, lse


def dsv4_norm_rope(x: torch.Tensor, pos: torch.Tensor, rows_per_pos: int = 1, rope: int = 64,
                   norm: bool = True, inverse: bool = False, eps: float = 1e-6,
                   stream=None) -> torch.Tensor:
    """In place on x [..., c]: RMS-normalise each row (norm) and rotate its last `rope`
    channels by pos[row // rows_per_pos] (inverse: by minus the angle). Returns x."""
    _dev(x, "x"), _dev(pos, "pos", torch.int32)
    c = x.shape[-1]
    rows = x.numel() // max(c, 1)
    _check(lib.dsv4_norm_rope(_code(x.dtype), _ptr(x), _ptr(pos), rows, rows_per_pos, c, rope,
                              1 if norm else 0, 1 if inverse else 0, float(eps), _stream(stream)),
           "dsv4_norm_rope")
    return x


def dsv4_hybrid_sparse_attn_workspace_size(B: int, nq: int, H: int, c: int) -> int:
    return int(lib.dsv4_hybrid_sparse_attn_workspace_size(B, nq, H, c))


def dsv4_check_errors(stream=None):
    """Synchronise the stream and raise DSV4Error if a kernel flagged a device-side error."""
    _check(lib.dsv4_check_errors(_stream(stream)), "dsv4_check_errors")


# ----------------------------------------------------------------------------- FP8 main-KV entries


def dsv4_quantize_main_kv(x: torch.Tensor, rope: int = 64, stream=None):
    """x [rows, c] (fp32 / bf16) -> (codes uint8 [rows, c-rope], scales fp32 [rows, (c-rope)/64],
    rope bf16 [rows, rope]): the FP8 main-KV entry format."""
    _dev(x, "x")
    c = x.shape[-1]
    rows = x.numel() // max(c, 1)
    codes = torch.empty(rows, c - rope, dtype=torch.uint8, device=x.device)
    scales = torch.empty(rows, (c - rope) // 64, dtype=torch.float32, device=x.device)
    rp = torch.empty(rows, rope, dtype=torch.bfloat16, device=x.device)
    _check(lib.dsv4_quantize_main_kv(_code(x.dtype), _ptr(x), _ptr(codes), _ptr(scales), _ptr(rp),
                                     rows, c, rope, _stream(stream)), "dsv4_quantize_main_kv")
    return codes, scales, rp


def dsv4_dequantize_main_kv(codes: torch.Tensor, scales: torch.Tensor, rope: torch.Tensor,
                            out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """FP8 entries -> bf16 rows [rows, c]."""
    _dev(codes, "codes", torch.uint8), _dev(scales, "scales", torch.float32)
    _dev(rope, "rope", torch.bfloat16)
    rows, nf = codes.shape
    r = rope.shape[-1]
    if out is None:
        out = torch.empty(rows, nf + r, dtype=torch.bfloat16, device=codes.device)
    _check(lib.dsv4_dequantize_main_kv(_ptr(codes), _ptr(scales), _ptr(rope), _ptr(out), rows, nf + r,
                                       r, _stream(stream)), "dsv4_dequantize_main_kv")
    return out


def dsv4_compress_decode_fp8(C_new, Z_new, bias, tail, codes, scales, rope, pool_row_off, pos, m: int,
                             overlap: bool, stream=None) -> None:
    """dsv4_compress_decode emitting completed entries into an FP8 pool (codes, scales, rope)."""
    _dev(C_new, "C_new"), _dev(Z_new, "Z_new", C_new.dtype), _dev(bias, "bias", torch.float32)
    _dev(tail, "tail", C_new.dtype), _dev(codes, "codes", torch.uint8)
    _dev(scales, "scales", torch.float32), _dev(rope, "rope", torch.bfloat16)
    _dev(pool_row_off, "pool_row_off", torch.int64), _dev(pos, "pos", torch.int32)
    B, width = C_new.shape
    S = 2 if overlap else 1
    c = width // S
    if tuple(tail.shape) != decode_tail_shape(B, c, m, overlap):
        raise ValueError(f"tail must be {decode_tail_shape(B, c, m, overlap)}")
    _check(lib.dsv4_compress_decode_fp8(_code(C_new.dtype), _ptr(C_new), _ptr(Z_new), _ptr(bias),
                                        _ptr(tail), _ptr(codes), _ptr(scales), _ptr(rope),
                                        rope.shape[-1], _ptr(pool_row_off), codes.shape[0], _ptr(pos),
                                        B, c, m, 1 if overlap else 0, _stream(stream)),
           "dsv4_compress_decode_fp8")


def dsv4_hybrid_sparse_attn_fp8_workspace_size(B: int, H: int, c: int, k: int) -> int:
    return int(lib.dsv4_hybrid_sparse_attn_fp8_workspace_size(B, H, c, k))


def dsv4_hybrid_sparse_attn_fp8(Q, codes, scales, rope, kv_row_off, idx, counts, local, q_pos0,
                                m: int, w: int, sink=None, scale=None, O=None, lse=None,
                                workspace=None, stream=None):
    """Decode attention over an FP8 pool. Q [B, 1, H, c] bf16; (codes, scales, rope) the pool;
    idx/counts [B, 1, k] / [B, 1]; local [B, R, c] bf16. Returns (O, lse)."""
    _dev(Q, "Q", torch.bfloat16), _dev(local, "local", torch.bfloat16)
    _dev(codes, "codes", torch.uint8), _dev(scales, "scales", torch.float32)
    _dev(rope, "rope", torch.bfloat16), _dev(idx, "idx", torch.int32), _dev(counts, "counts", torch.int32)
    _dev(kv_row_off, "kv_row_off", torch.int64), _dev(q_pos0, "q_pos0", torch.int32)
    B, nq, H, c = Q.shape
    if nq != 1:
        raise ValueError("dsv4_hybrid_sparse_attn_fp8 takes one query per sequence")
    k = idx.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(c)
    if O is None:
        O = torch.empty_like(Q)
    if lse is None:
        lse = torch.empty(B, 1, H, dtype=torch.float32, device=Q.device)
    need = dsv4_hybrid_sparse_attn_fp8_workspace_size(B, H, c, k)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=Q.device)
    _check(lib.dsv4_hybrid_sparse_attn_fp8(_ptr(Q), _ptr(codes), _ptr(scales), _ptr(rope), codes.shape[0],
                                           _ptr(kv_row_off), _ptr(idx), _ptr(counts), k, _ptr(local),
                                           local.shape[1], _ptr(q_pos0), B, H, c, rope.shape[-1], m, w,
                                           _ptr(sink), float(scale), _ptr(O), _ptr(lse), _ptr(workspace),
                                           workspace.numel(), _stream(stream)),
           "dsv4_hybrid_sparse_attn_fp8")
    return O, lse
