"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source, in a
temporary directory on the CPU, builds it, and runs the pin suites of its
area against the copy (the `orc` fixture loads it through FP8Q_ORACLE_DIR).
At least one pin must fail.  The mistakes are the kind a restatement of the pages'
formulas could make: a dropped term, a wrong rounding, a swapped formula, a
wrong index, a reordered epilogue.  Every planted index stays inside its
array, so a mutated oracle reads only what it owns.
"""
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE = os.path.join(ROOT, "oracle")
sys.path.insert(0, ROOT)
from oracle import CFLAGS  # noqa: E402  (the flags the oracle itself builds with)
CASTS = ["tests/test_oracle_method.py", "tests/test_oracle_rules.py"]
CODECS = ["tests/test_oracle_codecs.py"]
PRODUCTS = ["tests/test_oracle_scaled_mm.py"]

MUTATIONS = [
    ("per-token clamp dropped (DeepEP 5 Utils: amax.clamp(1e-4))", CASTS,
     "            if (amax < clampmin)\n                amax = clampmin;",
     "            (void)clampmin;"),
    ("e4m3fn encode saturates at 448 instead of giving NaN (torch's .to(float8_e4m3fn))", CODECS,
     "return (uint8_t)((c > 0x7Eu ? 0x7Fu : c) | sign);",
     "return (uint8_t)((c > 0x7Eu ? 0x7Eu : c) | sign);"),
    ("per-token groups start one element apart instead of one group apart", CASTS,
     "            int64_t base = r * n + g * group;",
     "            int64_t base = r * n + g;"),
    ("fp8 encode rounds ties away from zero instead of to even", CODECS,
     "if (rem > half || (rem == half && (kept & 1u)))",
     "if (rem >= half)"),
    ("per-channel keeps a zero amax (ColossalAI: torch.where(amax > 0, amax, 1))", CASTS,
     "        amax = amax > 0.0f ? amax : 1.0f;\n        float scale = scale_of(amax, fmax, rule);\n        scale_inv[r]",
     "        float scale = scale_of(amax, fmax, rule);\n        scale_inv[r]"),
    ("per-token scale_inv written as 1 / scale instead of amax / 448", CASTS,
     "scale_inv[r * G + g] = scale_inv_of(amax, fmax, rule);",
     "scale_inv[r * G + g] = 1.0f / scale;"),
    ("per-tensor scale_inv written as amax / FMAX instead of 1 / scale", CASTS,
     "    scale_inv[0] = 1.0f / scale;   /* `1.0 / scale` is one rounding under both rules */",
     "    scale_inv[0] = amax / fmax;"),
    ("block dequant takes the row block's index for the column block", CASTS,
     "float sc = s[(i / block) * nb + j / block];",
     "float sc = s[(i / block) * nb + (i / block) % nb];"),
    ("per-tensor product drops the bias", PRODUCTS,
     "            if (bias) v = v + bias[n];\n            store_elem(out, yt, m * N + n, v);",
     "            store_elem(out, yt, m * N + n, v);"),
    ("per-tensor product adds the bias before the scale", PRODUCTS,
     "            float v = acc * s;\n            if (bias) v = v + bias[n];",
     "            float v = acc;\n            if (bias) v = v + bias[n];\n            v = v * s;"),
    ("fine-grained product walks the weight's k-blocks backwards", PRODUCTS,
     "const float s = sa[m * kb + j] * sb[(n / bb) * kb + j];",
     "const float s = sa[m * kb + j] * sb[(n / bb) * kb + (kb - 1 - j)];"),
    ("fine-grained product takes another row's activation scales", PRODUCTS,
     "        const float* sar = sa + m * ka;",
     "        const float* sar = sa + (M - 1 - m) * ka;"),
]


def _caught(tmp, name, pins, old, new):
    """Builds the copy with the planted mistake and runs its area's pins; returns (caught, log)."""
    src = open(os.path.join(ORACLE, "fp8q_oracle.c")).read()
    if src.count(old) != 1:
        return False, f"the text to mutate for '{name}' is not unique in the oracle"
    os.makedirs(tmp)
    for fn in ("__init__.py", "fp8q_oracle.h"):
        shutil.copy(os.path.join(ORACLE, fn), os.path.join(tmp, fn))
    with open(os.path.join(tmp, "fp8q_oracle.c"), "w") as f:
        f.write(src.replace(old, new))
    # the mutated copy must build: a pin run that fails only because the copy does not
    # compile would prove nothing
    b = subprocess.run(["gcc", *CFLAGS, "-o", os.path.join(tmp, "libfp8q_oracle.so"),
                        os.path.join(tmp, "fp8q_oracle.c"), "-lm"], capture_output=True, text=True)
    if b.returncode != 0:
        return False, f"the copy with '{name}' does not build:\n{b.stderr[-2000:]}"
    env = dict(os.environ, FP8Q_ORACLE_DIR=tmp)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "not gpu", *pins], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    return r.returncode == 1 and " failed" in r.stdout, r.stdout[-3000:]


def test_every_planted_mistake_fails_a_pin(tmp_path):
    with cf.ThreadPoolExecutor(max_workers=len(MUTATIONS)) as ex:
        futs = {m[0]: ex.submit(_caught, str(tmp_path / f"m{i}"), *m) for i, m in enumerate(MUTATIONS)}
        results = {name: f.result() for name, f in futs.items()}
    missed = {name: log for name, (ok, log) in results.items() if not ok}
    assert not missed, "no pin caught:\n" + "\n\n".join(f"{n}\n{log}" for n, log in missed.items())
