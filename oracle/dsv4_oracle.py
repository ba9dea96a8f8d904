"""fp64 CPU oracle for the DeepSeek-V4 hybrid CSA/HCA attention hot path.

TEST INFRASTRUCTURE. This module is the plain, slow, obviously-correct statement of
what the hot path computes. Only the test suite, the smoke check and the benchmark's
CPU-baseline leg may import it; the product library never does, and it shares no code
with the CUDA kernels.

Everything is computed in float64 (numpy). Storage formats are decoded exactly
(bf16 -> fp32 -> fp64 is exact; an FP4 e2m1 code times its E4M3 scale is exact).
Library primitives used as single steps: numpy matmul, exp/log, sqrt, cos/sin, max, lexsort.

Sources (page title, then section / equation):
  [CSA-DEF] "CSA And HCA: Definition, State, And Cost Model"
      s1  completed-entry set E_t^(r) = {s | 0 <= s < floor((t+1)/r)}
      s2.1 CSA overlapping two-stream compressor (the [S^a; S^b] softmax equation and
           the C_i^Comp sum); i = 0 pads the preceding block with zero weight
      s2.2 HCA non-overlapping one-stream compressor
      s3.1 lightning-indexer score I_{t,s} and TopK over E_t^(m)
      s3.2 / s4 shared-KV MQA (each entry is both key and value for every head)
      s5.1 local window L_t = {max(0,t-w+1)..t} and ONE candidate list / softmax
      s5.2 logit scaled by 1/sqrt(c)
      s5.2 RMSNorm of query heads and the shared KV head; RoPE on the last 64 channels
           (query at t, compressed entry s at m*s, local entry j at j); inverse RoPE
           of the output's last 64 channels at t
      s5.3 sink logit z'_h in the denominator only
      s7  incremental decode state machine (local ring slot per token, bounded
          compressor tail, entry emitted when (t+1) is a multiple of the ratio)
      s8  precision table (MXFP4 indexer operands; main KV entries of 448 FP8 + 64 bf16
          RoPE channels, 576-byte payload) and the per-layer persistent-state table
  [PR-MASK] huggingface/transformers PR #45892 discussion: [S, S*top_k] gathered
      mask vs [S, compressed_len] scatter mask give identical attention.
  [PYPTO] pypto-lib PR #834: per-query compressed counts (cmp_counts).

Readings taken where the pages are silent (each is also listed in the design notes):
  * CSA input halves: columns [0, c) are stream a (current block), [c, 2c) are
    stream b (preceding block); bias[0] = B^a, bias[1] = B^b, each [m, c].
  * i = 0: the preceding block is excluded from the softmax (weight exactly 0).
  * Trailing incomplete block: never pooled; a sequence of n tokens has floor(n/m)
    entries.
  * Top-k: S_t is a set: the k_eff = min(k, |E_t|) largest scores, ties going to the
    lower entry index, listed in ascending entry order; the k - k_eff unused slots hold -1.
  * Softmax scale is an explicit parameter (default 1/sqrt(c)).
  * No de-duplication between compressed and local candidates (different objects).
  * FP4: e2m1 codes with one E4M3 scale per 16 consecutive elements (NVFP4-style),
    scale = RNE_e4m3(amax / 6) computed from fp32 amax/6, code = RNE_e2m1(x / scale)
    from the fp32 quotient, saturating at +-6; a zero scale gives zero codes.
    The sign bit follows IEEE rounding (a negative value that rounds to zero is -0,
    code 0x8). Two codes per byte, element 2j in the low nibble.
  * RMSNorm without a learned gain, eps = 1e-6; RoPE on adjacent channel pairs of the
    last 64 channels with base 10000 (the pages fix the rotated channels and positions).
  * Main-KV FP8 entries: the RoPE channels are the last 64; the FP8 channels carry one
    fp32 scale per 64 channels, scale = amax / 448 (the pages leave the scale metadata
    open).
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------- helpers


def as_f64(x) -> np.ndarray:
    """Exact decode of a torch tensor / numpy array (fp32, bf16, fp64) to float64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------- [CSA-DEF] s1, s5.1


def completed_entries(t: int, r: int) -> int:
    """|E_t^(r)|: query t sees compressed entries s in [0, floor((t+1)/r))  ([CSA-DEF] s1)."""
    return (t + 1) // r


def local_window(t: int, w: int) -> np.ndarray:
    """L_t = {max(0, t-w+1), ..., t}  ([CSA-DEF] s5.1)."""
    return np.arange(max(0, t - w + 1), t + 1)


# ----------------------------------------------------------------------------- [CSA-DEF] s2


def _pool_entry(logits: np.ndarray, values: np.ndarray) -> np.ndarray:
    """Feature-wise softmax over positions (axis -2), then the weighted sum of values.

    logits, values: [..., positions, channels]. One independent softmax per channel
    ([CSA-DEF] s2: "normalized over positions independently for every feature channel").
    """
    mu = logits.max(axis=-2, keepdims=True)
    e = np.exp(logits - mu)
    s = e / e.sum(axis=-2, keepdims=True)
    return (s * values).sum(axis=-2)


def compress(C, Z, bias, m: int, overlap: bool) -> np.ndarray:
    """Learned compressor ([CSA-DEF] s2.1 for overlap=True, s2.2 for overlap=False).

    C, Z : [B, n, S*c]  entry stream(s) and gate logits; S = 2 (CSA: a | b) or 1 (HCA)
    bias : [S, m, c]    positional bias B^a (and B^b)
    returns [B, floor(n/m), c]

    Entry i pools the current block {m*i .. m*i+m-1} from stream a with bias B^a and,
    for CSA with i > 0, the preceding block {m*(i-1) .. m*i-1} from stream b with
    bias B^b, under ONE softmax over all those positions per channel.
    """
    C = as_f64(C)
    Z = as_f64(Z)
    bias = as_f64(bias)
    B, n, width = C.shape
    c = width // 2 if overlap else width
    E = n // m
    out = np.zeros((B, E, c))
    for i in range(E):
        cur = slice(m * i, m * (i + 1))
        logits = [Z[:, cur, :c] + bias[0]]
        values = [C[:, cur, :c]]
        if overlap and i > 0:
            prev = slice(m * (i - 1), m * i)
            logits.append(Z[:, prev, c:2 * c] + bias[1])
            values.append(C[:, prev, c:2 * c])
        out[:, i, :] = _pool_entry(np.concatenate(logits, axis=1),
                                   np.concatenate(values, axis=1))
    return out


# ----------------------------------------------------------------------------- [CSA-DEF] s3.1


def index_scores_query(qI, w, KI, t: int, m: int) -> np.ndarray:
    """I_{t,s} = sum_h w_{t,h} ReLU(q^I_{t,h} . K^I_s) for s in E_t^(m)  ([CSA-DEF] s3.1).

    qI [H_I, c_I], w [H_I], KI [rows >= |E_t|, c_I] (this sequence's keys) -> [|E_t|].
    """
    qI = as_f64(qI)
    w = as_f64(w)
    KI = as_f64(KI)
    E_t = completed_entries(t, m)
    dots = qI @ KI[:E_t].T                    # [H_I, E_t]
    return w @ np.maximum(dots, 0.0)          # [E_t]


def topk_select(scores: np.ndarray, k: int):
    """TopK over the eligible entries ([CSA-DEF] s3.1), with the tie/padding reading.

    S_t is a set: the min(k, len) entries with the largest scores, equal scores at the
    threshold going to the lower entry index. Returns (idx int32 [k], count) with the
    selected entries in ascending entry order; unused slots are -1.
    """
    scores = np.asarray(scores, dtype=np.float64)
    E = scores.shape[0]
    k_eff = min(k, E)
    order = np.lexsort((np.arange(E), -scores))   # primary: -score, secondary: index
    idx = np.full(k, -1, dtype=np.int32)
    idx[:k_eff] = np.sort(order[:k_eff])
    return idx, k_eff


# ----------------------------------------------------------------------------- [CSA-DEF] s3.2-s5.3


def attend_query(q, cand, sink=None, scale: float = None):
    """One shared-KV MQA step for one query over one candidate list.

    q    [H, c]   query heads
    cand [N, c]   candidate entries A_t (compressed entries ++ local entries); each row is
                  both the key and the value for every head ([CSA-DEF] s3.2)
    sink [H] or None: per-head sink logit z'_h, in the denominator only ([CSA-DEF] s5.3)
    scale: logit scale, default 1/sqrt(c) ([CSA-DEF] s5.2)
    returns (o [H, c], lse [H]) with lse = log(sum_j exp(z_j) + exp(z'_h)).
    """
    q = as_f64(q)
    cand = as_f64(cand)
    H, c = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(c)
    z = scale * (q @ cand.T)                          # [H, N]
    mu = z.max(axis=1) if cand.shape[0] else np.full(H, -np.inf)
    if sink is not None:
        sink = as_f64(sink)
        mu = np.maximum(mu, sink)
    e = np.exp(z - mu[:, None])
    den = e.sum(axis=1)
    if sink is not None:
        den = den + np.exp(sink - mu)
    o = (e @ cand) / den[:, None]
    lse = mu + np.log(den)
    return o, lse


def candidates(pool_seq, idx_row, count, local_seq, R: int, t: int, w: int,
               dense_m: int = 0) -> np.ndarray:
    """Build A_t ([CSA-DEF] s5.1): compressed part then local part.

    pool_seq : [rows, c] this sequence's compressed pool
    idx_row  : [k] selected entries (CSA) -- ignored when dense_m > 0
    count    : number of valid leading entries of idx_row
    dense_m  : > 0 for the HCA dense read of all E_t^(dense_m) entries ([CSA-DEF] s4)
    local_seq: [R, c] local ring; local entry j lives in slot j mod R
    """
    if dense_m > 0:
        comp = np.arange(completed_entries(t, dense_m))
    else:
        comp = np.asarray(idx_row[:count], dtype=np.int64)
    loc = local_window(t, w) % R
    return np.concatenate([pool_seq[comp], local_seq[loc]], axis=0)


def hybrid_attention(Q, pool, kv_row_off, idx, counts, local, q_pos0, w: int,
                     sink=None, scale=None, dense_m: int = 0, queries=None):
    """Hybrid sparse attention over (selected | all completed) entries ++ local window.

    Q        [B, nq, H, c]
    pool     [rows, c]; sequence b's entries start at row kv_row_off[b]
    idx      [B, nq, k] int (CSA) or None (dense HCA read with ratio dense_m)
    counts   [B, nq] valid entries per query (CSA) or None
    local    [B, R, c] local ring (R = n for prefill; slot = position mod R)
    q_pos0   [B]: query i of sequence b sits at position t = q_pos0[b] + i
    queries  optional list of (b, i) pairs to evaluate
    returns (O [B, nq, H, c], LSE [B, nq, H]) for all queries, or, when `queries` is
    given, (O [len(queries), H, c], LSE [len(queries), H]) in the order listed.
    """
    pool = as_f64(pool)
    local = as_f64(local)
    B, nq, H, c = Q.shape
    R = local.shape[1]
    listed = queries is not None
    if not listed:
        queries = [(b, i) for b in range(B) for i in range(nq)]
    O = np.empty((len(queries), H, c))
    LSE = np.empty((len(queries), H))
    for q_n, (b, i) in enumerate(queries):
        t = int(q_pos0[b]) + i
        base = int(kv_row_off[b])
        pool_seq = pool[base:]
        row = None if idx is None else np.asarray(idx[b, i])
        cnt = 0 if counts is None else int(counts[b, i])
        A = candidates(pool_seq, row, cnt, local[b], R, t, w, dense_m)
        O[q_n], LSE[q_n] = attend_query(as_f64(Q[b, i]), A, sink, scale)
    if not listed:
        return O.reshape(B, nq, H, c), LSE.reshape(B, nq, H)
    return O, LSE


def index_topk(qI, w, KI, kv_row_off, q_pos0, m: int, k: int, queries=None,
               with_scores: bool = False):
    """Indexer scores + TopK for every query ([CSA-DEF] s3.1).

    qI [B, nq, H_I, c_I], w [B, nq, H_I], KI [rows, c_I] with sequence b's keys from
    row kv_row_off[b]. Returns idx int32 [B, nq, k], counts int32 [B, nq] (and, when
    with_scores, a dict (b, i) -> fp64 score vector over E_t).
    """
    KI = as_f64(KI)
    B, nq = qI.shape[:2]
    idx = np.full((B, nq, k), -1, dtype=np.int32)
    counts = np.zeros((B, nq), dtype=np.int32)
    scores = {}
    if queries is None:
        queries = [(b, i) for b in range(B) for i in range(nq)]
    for b, i in queries:
        t = int(q_pos0[b]) + i
        s = index_scores_query(as_f64(qI[b, i]), as_f64(w[b, i]), KI[int(kv_row_off[b]):], t, m)
        idx[b, i], counts[b, i] = topk_select(s, k)
        if with_scores:
            scores[(b, i)] = s
    return (idx, counts, scores) if with_scores else (idx, counts)


# ----------------------------------------------------------------------------- FP4 ([CSA-DEF] s3.1, s8)


def e4m3_values() -> np.ndarray:
    """Decoded value of every non-negative E4M3 (fn) byte 0x00..0x7E, from the bit layout.

    Layout s.eeee.mmm, exponent bias 7; exponent field 0 is subnormal (m/8 * 2^-6);
    0x7F is NaN and is excluded. Largest finite value 0x7E = 1.75 * 2^8 = 448.
    """
    vals = []
    for code in range(0x7F):
        e, mant = code >> 3, code & 7
        if e == 0:
            vals.append(mant / 8.0 * 2.0 ** -6)
        else:
            vals.append((1.0 + mant / 8.0) * 2.0 ** (e - 7))
    return np.array(vals)


def e2m1_values() -> np.ndarray:
    """Decoded value of the non-negative e2m1 codes 0..7: s.ee.m, bias 1, subnormal at e=0."""
    vals = []
    for code in range(8):
        e, mant = code >> 1, code & 1
        vals.append(mant * 0.5 if e == 0 else (1.0 + mant / 2.0) * 2.0 ** (e - 1))
    return np.array(vals)


def round_to_table(v: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Round non-negative v to the nearest table value, ties to the even code.

    table is increasing, so code order is value order; values above the last entry
    saturate to it. Distances are compared exactly (all quantities are dyadic).
    """
    v = np.asarray(v, dtype=np.float64)
    hi = np.searchsorted(table, v, side="left")          # first table value >= v
    hi = np.clip(hi, 0, len(table) - 1)
    lo = np.clip(hi - 1, 0, len(table) - 1)
    d_lo = np.abs(v - table[lo])
    d_hi = np.abs(table[hi] - v)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(v >= table[-1], len(table) - 1, code)  # saturate
    return code.astype(np.int64)


def quantize_fp4(x):
    """Quantise rows to FP4 e2m1 with one E4M3 scale per 16 consecutive elements.

    x: [rows, cols] (cols % 16 == 0), any float dtype; values are taken as fp32.
    Returns (codes uint8 [rows, cols/2], scales uint8 [rows, cols/16]).
    """
    x32 = np.asarray(as_f64(x), dtype=np.float32)
    rows, cols = x32.shape
    g = x32.reshape(rows, cols // 16, 16)
    amax = np.abs(g).max(axis=-1)                                 # exact
    s32 = (amax / np.float32(6.0)).astype(np.float32)             # fp32 division
    t4 = e4m3_values()
    sbyte = round_to_table(np.minimum(s32.astype(np.float64), t4[-1]), t4)
    sval = t4[sbyte].astype(np.float32)                           # decoded scale, exact
    safe = np.where(sval > 0, sval, np.float32(1.0)).astype(np.float32)
    q32 = (g / safe[..., None]).astype(np.float32)                # fp32 division
    t2 = e2m1_values()
    mag = round_to_table(np.abs(q32).astype(np.float64), t2)
    sign = np.signbit(q32)            # IEEE: the sign survives rounding to zero
    code = (mag | (sign.astype(np.int64) << 3))
    code = np.where(sval[..., None] > 0, code, 0).reshape(rows, cols)
    packed = (code[:, 0::2] | (code[:, 1::2] << 4)).astype(np.uint8)
    return packed, sbyte.astype(np.uint8)


def dequantize_fp4(codes, scales, cols: int) -> np.ndarray:
    """Exact fp64 value of packed e2m1 codes times their E4M3 scales -> [rows, cols]."""
    codes = np.asarray(codes, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    rows = codes.shape[0]
    nib = np.empty((rows, cols), dtype=np.int64)
    nib[:, 0::2] = codes & 0xF
    nib[:, 1::2] = codes >> 4
    t2 = e2m1_values()
    mag = t2[nib & 7]
    val = np.where(nib & 8, -mag, mag)
    t4 = e4m3_values()
    s = t4[scales.astype(np.int64) & 0x7F]
    return val * np.repeat(s, 16, axis=1)


# ----------------------------------------------------------------------------- [CSA-DEF] s5.2


def rms_norm(x, eps: float = 1e-6) -> np.ndarray:
    """RMS normalisation over the last axis ([CSA-DEF] s5.2: every query head and the shared
    KV head, right before core attention): x / sqrt(mean(x^2) + eps). Reading: no learned
    gain (a per-channel gain would be an upstream weight), eps = 1e-6."""
    x = as_f64(x)
    return x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps)


def rope_rotate(x, pos, rope: int = 64, base: float = 10000.0, inverse: bool = False):
    """rho_p of [CSA-DEF] s5.2 on the last `rope` channels of x [..., c]: channel pairs
    (c - rope + 2i, c - rope + 2i + 1) rotate by the angle p * base^(-2i / rope); the other
    channels are unchanged; inverse=True rotates by minus the angle. `pos` broadcasts over
    the leading axes of x. Reading: adjacent channel pairs and base 10000 (the pages fix
    only which channels rotate and the positions)."""
    x = np.array(as_f64(x), copy=True)
    c = x.shape[-1]
    half = rope // 2
    freq = base ** (-2.0 * np.arange(half) / rope)                  # [rope/2]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * freq       # [..., rope/2]
    if inverse:
        ang = -ang
    a = x[..., c - rope::2].copy()
    b = x[..., c - rope + 1::2].copy()
    cs, sn = np.cos(ang), np.sin(ang)
    x[..., c - rope::2] = a * cs - b * sn
    x[..., c - rope + 1::2] = a * sn + b * cs
    return x


def attend_query_rope(q, t: int, entries, entry_pos, sink=None, scale: float = None,
                      rope: int = 64):
    """One query's core attention with the s5.2 contract: the query heads q [H, c] and the
    candidate entries [N, c] are RMS-normalised, q is rotated at its position t and entry j
    at entry_pos[j] (compressed entry s: m*s for CSA, m'*s for HCA; local entry j: j), one
    softmax as in attend_query, and the output's last `rope` channels are rotated back at t
    (inverse RoPE). Returns (o [H, c], lse [H])."""
    qn = rope_rotate(rms_norm(q), np.full(as_f64(q).shape[0], t), rope)
    kv = rope_rotate(rms_norm(entries), np.asarray(entry_pos), rope)
    o, lse = attend_query(qn, kv, sink, scale)
    return rope_rotate(o, np.full(o.shape[0], t), rope, inverse=True), lse


# ----------------------------------------------------------------------------- main-KV cache entry ([CSA-DEF] s8)


def main_kv_payload_bytes(c: int = 512, rope: int = 64) -> int:
    """Payload of one production main (or local) KV entry ([CSA-DEF] s8 precision table):
    the c - rope non-RoPE channels in FP8 (1 byte) and the rope RoPE channels in bf16."""
    return (c - rope) * 1 + rope * 2


def quantize_main_kv_fp8(x, rope: int = 64, group: int = 64):
    """Production main-KV entry format ([CSA-DEF] s8): channels [0, c - rope) in FP8 E4M3,
    channels [c - rope, c) (the RoPE part) kept in bf16.

    The pages leave the FP8 scale metadata open; reading: one fp32 scale per `group`
    consecutive FP8 channels, scale = fp32(amax / 448) (448 = the largest E4M3 value),
    code = RNE_E4M3(fp32(x / scale)) saturating at 448, IEEE sign (a negative value that
    rounds to zero keeps its sign), zero scale -> zero codes.
    x: [rows, c], values taken as fp32 (bf16 inputs are exact).
    Returns (codes uint8 [rows, c - rope] = sign << 7 | magnitude code,
             scales float32 [rows, (c - rope) / group], rope float64 [rows, rope] (the bf16
             value of each RoPE channel)).
    """
    x32 = np.asarray(as_f64(x), dtype=np.float32)
    rows, c = x32.shape
    nf = c - rope
    assert nf % group == 0, "FP8 channels must split into whole groups"
    g = x32[:, :nf].reshape(rows, nf // group, group)
    amax = np.abs(g).max(axis=-1)
    scale = (amax / np.float32(448.0)).astype(np.float32)               # fp32 division
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    q = (g / safe[..., None]).astype(np.float32)                          # fp32 division
    t4 = e4m3_values()
    mag = round_to_table(np.abs(q).astype(np.float64), t4)
    code = mag | (np.signbit(q).astype(np.int64) << 7)
    code = np.where(scale[..., None] > 0, code, 0).reshape(rows, nf)
    rope_vals = round_bf16(x32[:, nf:])
    return code.astype(np.uint8), scale, rope_vals


def round_bf16(x32: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even) and return them as
    float64: keep the top 16 bits of the fp32 pattern after adding the rounding bias."""
    u = np.asarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = 0x7FFF + ((u >> 16) & 1)
    r = ((u + bias) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def dequantize_main_kv_fp8(codes, scales, rope_vals, group: int = 64) -> np.ndarray:
    """Exact fp64 value of a production main-KV entry: E4M3 value x its group scale, then
    the bf16 RoPE channels -> [rows, c]."""
    codes = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    t4 = e4m3_values()
    mag = t4[codes & 0x7F]
    val = np.where(codes & 0x80, -mag, mag)
    s = np.repeat(np.asarray(scales, dtype=np.float32).astype(np.float64), group, axis=1)
    return np.concatenate([val * s, np.asarray(rope_vals, dtype=np.float64)], axis=1)


# ----------------------------------------------------------------------------- [CSA-DEF] s7


def tail_slots(m: int, overlap: bool) -> int:
    """Rows of the bounded compressor tail ([CSA-DEF] s7 state table): the current block,
    plus for CSA the preceding block, whose stream-b half the next entry pools."""
    return 2 * m if overlap else m


def decode_append(tail, C_row, Z_row, bias, t: int, m: int, overlap: bool):
    """One token of the compressor state machine ([CSA-DEF] s7, steps 2-4).

    tail  float64 [T, 2, S*c], T = tail_slots(m, overlap): slot p mod T holds the C row
          (tail[., 0]) and the Z row (tail[., 1]) of position p. Position t's rows are
          written in place.
    Returns the completed entry [c] when t + 1 is a multiple of m (it is entry
    (t+1)/m - 1 and is eligible for the block's final token), else None: an incomplete
    block exposes no entry. The entry is the s2.1 / s2.2 softmax over the block's
    positions (stream a, bias[0]) and, for CSA after the first block, the preceding
    block's positions (stream b, bias[1]).
    """
    T = tail.shape[0]
    tail[t % T, 0] = as_f64(C_row)
    tail[t % T, 1] = as_f64(Z_row)
    if (t + 1) % m != 0:
        return None
    i = (t + 1) // m - 1
    width = tail.shape[2]
    c = width // 2 if overlap else width
    bias = as_f64(bias)
    pooled = [(m * i + p, 0, bias[0][p]) for p in range(m)]
    if overlap and i > 0:
        pooled += [(m * (i - 1) + p, 1, bias[1][p]) for p in range(m)]
    logits = np.stack([tail[pos % T, 1, half * c:(half + 1) * c] + b for pos, half, b in pooled])
    values = np.stack([tail[pos % T, 0, half * c:(half + 1) * c] for pos, half, _ in pooled])
    top = logits.max(axis=0)
    e = np.exp(logits - top)
    return (e * values).sum(axis=0) / e.sum(axis=0)


def ring_write(local, kv_row, t: int) -> None:
    """[CSA-DEF] s7 step 1: the token's shared-KV entry overwrites ring slot t mod R."""
    local[t % local.shape[0]] = as_f64(kv_row)


# ----------------------------------------------------------------------------- layer chains


def csa_prefill_layer(C, Z, bias, CI, ZI, biasI, qI, w, Q, local, m: int, k: int, wwin: int,
                      sink=None, scale=None, queries=None, index_fp4: bool = False):
    """One CSA prefill layer: compress (main, index keys) -> scores -> TopK -> attention.

    index_fp4: quantise q^I and K^I with quantize_fp4 before scoring (the FP4 indexer of
    [CSA-DEF] s3.1 / s8); the scores are then taken over the dequantised values in fp64.
    All sequences start at position 0 (q_pos0 = 0, R = n).
    Returns a dict with the pools, idx, counts, O, LSE.
    """
    pool = compress(C, Z, bias, m, overlap=True)         # [B, E, c]
    KI = compress(CI, ZI, biasI, m, overlap=True)        # [B, E, c_I]
    B, E = pool.shape[:2]
    qI64 = as_f64(qI)
    if index_fp4:
        Bq, nq, HI, cI = qI64.shape
        qc, qs = quantize_fp4(qI64.reshape(-1, cI))
        qI64 = dequantize_fp4(qc, qs, cI).reshape(Bq, nq, HI, cI)
        kc, ks = quantize_fp4(KI.reshape(-1, KI.shape[-1]))
        KI = dequantize_fp4(kc, ks, KI.shape[-1]).reshape(KI.shape)
    off = np.arange(B) * E
    pos0 = np.zeros(B, dtype=np.int64)
    idx, counts = index_topk(qI64, w, KI.reshape(B * E, -1), off, pos0, m, k, queries)
    O, LSE = hybrid_attention(Q, pool.reshape(B * E, -1), off, idx, counts, local, pos0,
                              wwin, sink, scale, 0, queries)
    return dict(pool=pool, KI=KI, idx=idx, counts=counts, O=O, LSE=LSE)


def hca_prefill_layer(C, Z, bias, Q, local, m: int, wwin: int, sink=None, scale=None,
                      queries=None):
    """One HCA prefill layer: compress (m') -> dense read over completed entries ++ window."""
    pool = compress(C, Z, bias, m, overlap=False)
    B, E = pool.shape[:2]
    off = np.arange(B) * E
    pos0 = np.zeros(B, dtype=np.int64)
    O, LSE = hybrid_attention(Q, pool.reshape(B * E, -1), off, None, None, local, pos0,
                              wwin, sink, scale, m, queries)
    return dict(pool=pool, O=O, LSE=LSE)
