"""Mutation check of the oracle's pins: each entry plants one plausible
mistake in a copy of the oracle (a dropped term, a wrong sign or direction,
the wrong rounding, a moved bit, a wrong index) and runs the pin suite
(`test_oracle_pins.py`) against that copy; every planted mistake must make a
pin fail. The unmodified copy must pass. CPU only; the repository's own
oracle is never modified."""
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (what the mistake is, exact text in oracle/wq_oracle.py, replacement).
# Not listed, because it is no mistake: computing the stored fold's quotient
# in fp64 instead of fp32 before the fp16 rounding gives the same fp16 value
# for every pair of fp16 operands (test_fold_fp16_is_the_correctly_rounded_
# quotient_exhaustive), so no pin can tell the two apart.
MUTANTS = [
    ("symmetric codes rounded down instead of to nearest",
     "qs = np.clip(np.rint(wg / sf), -qmax - 1, qmax)", "qs = np.clip(np.floor(wg / sf), -qmax - 1, qmax)"),
    ("asymmetric zero point with the wrong sign",
     "zero = np.clip(np.rint(-mn / sf32), 0, Q)", "zero = np.clip(np.rint(mn / sf32), 0, Q)"),
    ("fp16 step rounded to nearest instead of up",
     "h[below] = np.nextafter(h[below], np.float16(np.inf))", "h[below] = h[below]"),
    ("asymmetric range without 0",
     "mn = np.minimum(wg.min(axis=2), np.float32(0))", "mn = wg.min(axis=2)"),
    ("symmetric qmax off by one",
     "qmax = (1 << (bits - 1)) - 1\n        amax", "qmax = (1 << (bits - 1))\n        amax"),
    ("dequantize adds the zero point",
     "return ((q - z) * s).reshape(N, K)", "return ((q + z) * s).reshape(N, K)"),
    ("4-bit packing puts odd channels in the even slots",
     "words |= c[:, :, 2 * j + 1] << np.uint32(4 * (j + 4))", "words |= c[:, :, 2 * j + 1] << np.uint32(4 * j)"),
    ("3-bit packing moves channel 30's bit",
     "words[:, :, t] |= ((c[:, :, 30] >> np.uint32(t)) & 1) << np.uint32(15)",
     "words[:, :, t] |= ((c[:, :, 30] >> np.uint32(t)) & 1) << np.uint32(14)"),
    ("matmul reference with the output rows reversed",
     "return np.asarray(X16, dtype=np.float64) @ D.T", "return np.asarray(X16, dtype=np.float64) @ D[::-1].T"),
    ("activation statistic without the absolute value",
     "return np.abs(X.astype(np.float64)).sum(axis=0) / float(T)", "return X.astype(np.float64).sum(axis=0) / float(T)"),
    ("AWQ candidates with the exponent 1 - alpha",
     "out[j] = np.power(m, float(a)).astype(np.float16)", "out[j] = np.power(m, 1.0 - float(a)).astype(np.float16)"),
    ("AWQ error scales down by multiplying",
     "return W16.astype(np.float64) - Dq / s16.astype(np.float64)[None, :]",
     "return W16.astype(np.float64) - Dq * s16.astype(np.float64)[None, :]"),
    ("AWQ search keeps the largest loss",
     "best = int(np.argmin(losses))", "best = int(np.argmax(losses))"),
    ("AWQ loss sums |XE| instead of its square",
     "total += float(np.sum(P * P))", "total += float(np.sum(np.abs(P)))"),
    ("norm fold multiplies by s",
     "return gamma.astype(np.float64) / s.astype(np.float64)", "return gamma.astype(np.float64) * s.astype(np.float64)"),
    ("stored norm fold multiplies by s",
     "return (gamma.astype(np.float32) / s.astype(np.float32)).astype(np.float16)",
     "return (gamma.astype(np.float32) * s.astype(np.float32)).astype(np.float16)"),
    ("block fold applies s_o to o_proj's rows instead of v_proj's",
     'out["wv"], _ = awq_fold_into_linear_rows(out["wv"], s_o)', 'out["wo"], _ = awq_fold_into_linear_rows(out["wo"], s_o)'),
    ("decoder block without the MLP residual",
     "return y + ((g / (1.0 + np.exp(-g))) * u) @ p[\"wd\"].T", "return ((g / (1.0 + np.exp(-g))) * u) @ p[\"wd\"].T"),
    ("GPTQ error feedback with the wrong sign",
     "W[:, i + 1:b1] -= np.outer(err, G[i, i + 1:b1])", "W[:, i + 1:b1] += np.outer(err, G[i, i + 1:b1])"),
    ("GPTQ without the lazy block update",
     "W[:, b1:] -= Err @ G[b0:b1, b1:]", "W[:, b1:] -= 0.0 * (Err @ G[b0:b1, b1:])"),
    ("GPTQ error not divided by the factor's diagonal",
     "err = (W[:, i] - deq) / G[i, i]", "err = (W[:, i] - deq)"),
    ("GPTQ Hessian without the damping",
     "H += damp * np.mean(np.diag(H)) * np.eye(H.shape[0])", "H += 0.0 * np.eye(H.shape[0])"),
    ("GPTQ Hessian without the factor 2",
     "H = 2.0 * (X.T @ X)", "H = (X.T @ X)"),
    ("int8 absmax with 128 levels",
     "mult = 127.0 / np.max(np.abs(X))", "mult = 128.0 / np.max(np.abs(X))"),
    ("int8 zero point with the wrong sign",
     "zp = np.rint(-mult * np.min(X) - 128.0)", "zp = np.rint(mult * np.min(X) - 128.0)"),
    ("W4A8 activation codes rounded down",
     "q = np.clip(np.rint(x * mult[:, :, None]), -127, 127)", "q = np.clip(np.floor(x * mult[:, :, None]), -127, 127)"),
    ("W4A8 scale multiplies by the activation multiplier",
     "scale = steps.astype(np.float64)[None, :, :] / mult.astype(np.float64)[:, None, :]",
     "scale = steps.astype(np.float64)[None, :, :] * mult.astype(np.float64)[:, None, :]"),
    ("asymmetric codes subtract the zero point",
     "q = np.rint(wg / sf32[:, :, None]).astype(np.int32) + zero[:, :, None]",
     "q = np.rint(wg / sf32[:, :, None]).astype(np.int32) - zero[:, :, None]"),
    ("asymmetric Q off by one", "        Q = (1 << bits) - 1\n        mn", "        Q = (1 << bits)\n        mn"),
    ("asymmetric all-zero group without the step-1 rule",
     "step_h = np.where(r == 0, np.float16(1.0), step_h)", "step_h = step_h"),
    ("symmetric all-zero group without the step-1 rule",
     "step_h = np.where(amax == 0, np.float16(1.0), step_h)", "step_h = step_h"),
    ("4-bit unpack keeps 3 bits",
     "out[:, :, 2 * j] = (w >> np.uint32(4 * j)) & 0xF", "out[:, :, 2 * j] = (w >> np.uint32(4 * j)) & 0x7"),
    ("alpha grid divided by n - 1",
     "return np.arange(n_alpha, dtype=np.float64) / float(n_alpha)",
     "return np.arange(n_alpha, dtype=np.float64) / float(n_alpha - 1)"),
    ("no floor on mu", "m = np.maximum(np.asarray(mu, dtype=np.float64), MU_FLOOR)",
     "m = np.asarray(mu, dtype=np.float64)"),
    ("AWQ loss over the first linear only",
     "        total += float(np.sum(P * P))\n    return total",
     "        total += float(np.sum(P * P))\n        break\n    return total"),
    ("linear fold leaves the bias", "bf = None if b is None else np.asarray(b, dtype=np.float64) / s64",
     "bf = None if b is None else np.asarray(b, dtype=np.float64)"),
    ("GPTQ code with the zero point's sign flipped",
     "q = np.rint(w32 / sf).astype(np.int32) + zero_h.astype(np.int32)",
     "q = np.rint(w32 / sf).astype(np.int32) - zero_h.astype(np.int32)"),
    ("GPTQ group parameters from the original weights",
     "gc, gs, gz = quantize_groups_f32(W[:, i:i + group].astype(np.float32), bits, group, symmetric)",
     "gc, gs, gz = quantize_groups_f32(np.asarray(W16)[:, i:i + group].astype(np.float32), bits, group, symmetric)"),
    ("GPTQ keeps the weights of dead channels", "    W[:, dead] = 0.0\n", "    pass\n"),
    ("W4A8 all-zero activation group with multiplier 0",
     "mult = np.where(amax == 0, np.float32(1.0), np.float32(127.0)",
     "mult = np.where(amax == 0, np.float32(0.0), np.float32(127.0)"),
    ("W4A8 without the zero point",
     "qw = codes.astype(np.int64).reshape(N, G, group) - zeros.astype(np.int64)[:, :, None]",
     "qw = codes.astype(np.int64).reshape(N, G, group)"),
]


def run_pins(old, new):
    """Run the pin suite against a copy of the oracle with `old` replaced by
    `new` (None: unmodified). Returns (exit code, output tail)."""
    with tempfile.TemporaryDirectory() as tmp:
        shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(tmp, "oracle"),
                        ignore=shutil.ignore_patterns("__pycache__"))
        shutil.copytree(os.path.join(ROOT, "synth"), os.path.join(tmp, "synth"),
                        ignore=shutil.ignore_patterns("__pycache__"))
        os.makedirs(os.path.join(tmp, "tests"))
        for f in ("conftest.py", "test_oracle_pins.py"):
            shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(tmp, "tests", f))
        shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(tmp, "tests", "golden"),
                        ignore=shutil.ignore_patterns("__pycache__"))
        if old is not None:
            p = os.path.join(tmp, "oracle", "wq_oracle.py")
            src = open(p).read()
            assert src.count(old) == 1, f"mutation site not unique: {old!r}"
            with open(p, "w") as f:
                f.write(src.replace(old, new))
        r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                            os.path.join(tmp, "tests", "test_oracle_pins.py")],
                           cwd=tmp, capture_output=True, text=True, timeout=300,
                           env={**os.environ, "PYTHONDONTWRITEBYTECODE": "1"})
        return r.returncode, (r.stdout + r.stderr)[-600:]


def test_unmodified_copy_passes():
    rc, out = run_pins(None, None)
    assert rc == 0, out


def test_every_planted_mistake_fails_a_pin():
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda m: (m[0], run_pins(m[1], m[2])), MUTANTS))
    survivors = [name for name, (rc, _) in results if rc == 0]
    assert survivors == [], f"mistakes no pin catches: {survivors}"
    # exit code 1: a pin failed (2 would be a collection error, not a catch)
    broken = [(name, out) for name, (rc, out) in results if rc != 1]
    assert broken == [], broken
