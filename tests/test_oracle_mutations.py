"""The oracle's pins catch plausible slips (CPU only).

Each case plants one mistake in a temporary copy of the oracle package: a swapped stream,
a dropped or misplaced bias, a visibility, window or block bound off by one, ReLU after
the head sum, a dropped sink or scale, a wrong tie order, a wrong E4M3/e2m1 table entry
or nibble order, ... Then it runs the pin tests against that copy. Every planted mistake
must make at least one pin fail, and the unchanged copy must pass. The repository's own
oracle is never modified.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_SRC = os.path.join(ROOT, "oracle", "dsv4_oracle.py")

# name -> (text in the oracle, text planted instead)
SLIPS = {
    "compress: streams a and b swapped":
        ("logits = [Z[:, cur, :c] + bias[0]]", "logits = [Z[:, cur, c:2*c] + bias[0]]"),
    "compress: bias of stream b dropped":
        ("logits.append(Z[:, prev, c:2 * c] + bias[1])", "logits.append(Z[:, prev, c:2 * c])"),
    "compress: stream b takes bias a":
        ("logits.append(Z[:, prev, c:2 * c] + bias[1])", "logits.append(Z[:, prev, c:2 * c] + bias[0])"),
    "compress: wrong preceding block":
        ("prev = slice(m * (i - 1), m * i)", "prev = slice(m * i, m * (i + 1))"),
    "compress: softmax over channels instead of positions":
        ("s = e / e.sum(axis=-2, keepdims=True)", "s = e / e.sum(axis=-1, keepdims=True)"),
    "visibility: one entry early":
        ("return (t + 1) // r", "return t // r"),
    "window: one position too many":
        ("return np.arange(max(0, t - w + 1), t + 1)", "return np.arange(max(0, t - w), t + 1)"),
    "indexer: ReLU after the head sum":
        ("return w @ np.maximum(dots, 0.0)", "return np.maximum(w @ dots, 0.0)"),
    "indexer: one entry past the completed ones":
        ("dots = qI @ KI[:E_t].T", "dots = qI @ KI[:E_t + 1].T"),
    "indexer: weight inside the ReLU":
        ("return w @ np.maximum(dots, 0.0)", "return np.maximum(w[:, None] * dots, 0.0).sum(axis=0)"),
    "indexer: sequence key offset ignored":
        ("KI[int(kv_row_off[b]):], t, m)", "KI, t, m)"),
    "attention: sequence pool offset ignored":
        ("pool_seq = pool[base:]", "pool_seq = pool"),
    "fp8 main KV: zero-scale group keeps sign codes":
        ("code = np.where(scale[..., None] > 0, code, 0).reshape(rows, nf)", "code = code.reshape(rows, nf)"),
    "fp8 main KV: sign of -0 dropped":
        ("code = mag | (np.signbit(q).astype(np.int64) << 7)", "code = mag | ((q < 0).astype(np.int64) << 7)"),
    "rope: rotation sign":
        ("x[..., c - rope::2] = a * cs - b * sn", "x[..., c - rope::2] = a * cs + b * sn"),
    "rope: frequency exponent":
        ("freq = base ** (-2.0 * np.arange(half) / rope)", "freq = base ** (-1.0 * np.arange(half) / rope)"),
    "rope: output not rotated back":
        ("return rope_rotate(o, np.full(o.shape[0], t), rope, inverse=True), lse", "return o, lse"),
    "rms norm: sum instead of mean":
        ("return x / np.sqrt((x * x).mean(axis=-1, keepdims=True) + eps)",
         "return x / np.sqrt((x * x).sum(axis=-1, keepdims=True) + eps)"),
    "rope: entries rotated at the query position":
        ("kv = rope_rotate(rms_norm(entries), np.asarray(entry_pos), rope)",
         "kv = rope_rotate(rms_norm(entries), np.full(len(entry_pos), t), rope)"),
    "topk: ties to the higher entry":
        ("order = np.lexsort((np.arange(E), -scores))", "order = np.lexsort((-np.arange(E), -scores))"),
    "topk: selection not in ascending entry order":
        ("idx[:k_eff] = np.sort(order[:k_eff])", "idx[:k_eff] = order[:k_eff]"),
    "attention: sink dropped from the denominator":
        ("den = den + np.exp(sink - mu)", "den = den"),
    "attention: logit scale dropped":
        ("z = scale * (q @ cand.T)", "z = (q @ cand.T)"),
    "attention: default scale 1/c":
        ("scale = 1.0 / np.sqrt(c)", "scale = 1.0 / c"),
    "attention: LSE without the running max":
        ("lse = mu + np.log(den)", "lse = np.log(den)"),
    "attention: local ring slot off by one":
        ("loc = local_window(t, w) % R", "loc = (local_window(t, w) + 1) % R"),
    "attention: HCA dense read one entry too many":
        ("comp = np.arange(completed_entries(t, dense_m))", "comp = np.arange(completed_entries(t, dense_m) + 1)"),
    "decode: entry emitted one token early":
        ("if (t + 1) % m != 0:\n        return None", "if t % m != 0:\n        return None"),
    "decode: preceding block read from stream a":
        ("pooled += [(m * (i - 1) + p, 1, bias[1][p])", "pooled += [(m * (i - 1) + p, 0, bias[1][p])"),
    "decode: ring slot off by one":
        ("local[t % local.shape[0]] = as_f64(kv_row)", "local[(t + 1) % local.shape[0]] = as_f64(kv_row)"),
    "fp8 main KV: scale amax/240":
        ("scale = (amax / np.float32(448.0)).astype(np.float32)",
         "scale = (amax / np.float32(240.0)).astype(np.float32)"),
    "fp8 main KV: RoPE channels taken from the front":
        ("rope_vals = round_bf16(x32[:, nf:])", "rope_vals = round_bf16(x32[:, :rope])"),
    "fp8 main KV: bf16 rounding truncates":
        ("bias = 0x7FFF + ((u >> 16) & 1)", "bias = 0 * u"),
    "fp4: E4M3 exponent bias 8":
        ("vals.append((1.0 + mant / 8.0) * 2.0 ** (e - 7))", "vals.append((1.0 + mant / 8.0) * 2.0 ** (e - 8))"),
    "fp4: e2m1 subnormal 0.25":
        ("vals.append(mant * 0.5 if e == 0", "vals.append(mant * 0.25 if e == 0"),
    "fp4: nibble order swapped":
        ("packed = (code[:, 0::2] | (code[:, 1::2] << 4)).astype(np.uint8)",
         "packed = (code[:, 1::2] | (code[:, 0::2] << 4)).astype(np.uint8)"),
    "fp4: block scale amax/4":
        ("s32 = (amax / np.float32(6.0)).astype(np.float32)", "s32 = (amax / np.float32(4.0)).astype(np.float32)"),
    "csa layer: main pool fed to the indexer":
        ("idx, counts = index_topk(qI64, w, KI.reshape(B * E, -1)",
         "idx, counts = index_topk(qI64, w, pool.reshape(B * E, -1)"),
    "csa layer: index keys compressed without overlap":
        ("KI = compress(CI, ZI, biasI, m, overlap=True)",
         "KI = compress(CI[..., :CI.shape[-1] // 2], ZI[..., :ZI.shape[-1] // 2], biasI[:1], m, overlap=False)"),
    "csa layer: FP4 branch leaves the keys unquantised":
        ("KI = dequantize_fp4(kc, ks, KI.shape[-1]).reshape(KI.shape)", "KI = KI.reshape(KI.shape)"),
    "csa layer: FP4 branch leaves the queries unquantised":
        ("qI64 = dequantize_fp4(qc, qs, cI).reshape(Bq, nq, HI, cI)", "qI64 = qI64.reshape(Bq, nq, HI, cI)"),
    "csa layer: attention window one position wider":
        ("O, LSE = hybrid_attention(Q, pool.reshape(B * E, -1), off, idx, counts, local, pos0,\n                              wwin, sink, scale, 0, queries)",
         "O, LSE = hybrid_attention(Q, pool.reshape(B * E, -1), off, idx, counts, local, pos0,\n                              wwin + 1, sink, scale, 0, queries)"),
    "fp4: sign lost on rounding to zero":
        ("code = (mag | (sign.astype(np.int64) << 3))",
         "code = (mag | ((sign & (mag > 0)).astype(np.int64) << 3))"),
}


def _run_pins(tmp, name, planted):
    """Copy the oracle package and the pin tests under tmp/name, plant the slip (if any),
    run the pins there; returns pytest's exit code and the last line of its output."""
    d = os.path.join(tmp, name)
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(d, "oracle"),
                    ignore=shutil.ignore_patterns("__pycache__", "*.so", "*.o"))
    os.makedirs(os.path.join(d, "tests"))
    for f in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(d, "tests", f))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(d, "tests", "golden"))
    if planted is not None:
        src_path = os.path.join(d, "oracle", "dsv4_oracle.py")
        src = open(src_path).read()
        before, after = planted
        src = src.replace(before, after, 1)
        open(src_path, "w").write(src)
    env = dict(os.environ, PYTHONDONTWRITEBYTECODE="1")
    env.pop("PYTHONPATH", None)
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-x", "-q",
                        "-p", "no:cacheprovider"], cwd=d, env=env, capture_output=True, text=True,
                       timeout=600)
    lines = (r.stdout or r.stderr).strip().splitlines()
    return r.returncode, lines[-1] if lines else ""


def test_every_planted_slip_fails_a_pin(tmp_path):
    src = open(ORACLE_SRC).read()
    for name, (before, _) in SLIPS.items():
        assert src.count(before) == 1, f"oracle text for '{name}' not found once: update the slip"
    cases = [("unchanged", None)] + [(f"slip{n}", SLIPS[k]) for n, k in enumerate(SLIPS)]
    names = ["unchanged"] + list(SLIPS)
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda c: _run_pins(str(tmp_path), *c), cases))
    rc0, last0 = results[0]
    assert rc0 == 0, f"the unchanged oracle copy fails its pins: {last0}"
    missed = [f"{n} ({last})" for n, (rc, last) in zip(names[1:], results[1:]) if rc != 1]
    assert not missed, "slips not caught by any pin (exit code != 1): " + "; ".join(missed)
