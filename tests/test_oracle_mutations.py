"""The oracle's pins catch plausible mistakes (CPU, no GPU).

Each case plants one mistake in a copy of the oracle's C++ source: a flipped sign, a
dropped term, a wrong index, an off-by-one mask.  It builds that copy and runs the
oracle's pins against it in a fresh interpreter.  At least one pin must fail.  The
stored regression output (tests/golden) is left out, since the oracle wrote it itself:
every mistake must be caught by a check that stands apart from the oracle.  A control
case builds the unchanged source the same way, and every pin must pass on it.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "hspec_oracle.cpp")
HDR = os.path.join(ROOT, "oracle", "hspec_oracle.h")
PINS = ["tests/test_oracle_pins.py", "tests/test_oracle_step_pins.py", "tests/test_oracle_verify_pins.py"]

# (what the mistake is, the correct line, the mistaken line)
MUTATIONS = [
    ("dt_bias added with the wrong sign",
     "softplus(row[2 * HP + 2 * N + h] + (double)L.dt_bias[h])",
     "softplus(row[2 * HP + 2 * N + h] - (double)L.dt_bias[h])"),
    ("RoPE position without the context offset",
     "long pos = (long)ctx + j;",
     "long pos = j;"),
    ("B read from the C columns of the in-projection",
     "Bm[(size_t)j * N + n] = row[2 * HP + n];",
     "Bm[(size_t)j * N + n] = row[2 * HP + N + n];"),
    ("GQA maps query head h to kv head h % Hkv",
     "int g = h / G;",
     "int g = h % Hkv;"),
    ("dt dropped from the input term of the recurrence",
     "s = decay * s + d_t * xv * B[(size_t)t * N + n];",
     "s = decay * s + xv * B[(size_t)t * N + n];"),
    ("D skip term dropped from y",
     "y[((size_t)t * H + hh) * P + p] = acc + Dv[hh] * x[((size_t)t * H + hh) * P + p];",
     "y[((size_t)t * H + hh) * P + p] = acc;"),
    ("softmax without the 1/sqrt(D) scale",
     "s[t] = acc * scale;",
     "s[t] = acc;"),
    ("causal block mask off by one",
     "int visible = causal_block ? ctx + j + 1 : T;",
     "int visible = causal_block ? ctx + j : T;"),
    ("state decay exp(-dt A) instead of exp(dt A)",
     "double decay = std::exp(d_t * A[hh]);",
     "double decay = std::exp(-d_t * A[hh]);"),
    ("RMSNorm weight dropped",
     "out[i] = x[i] * inv * (double)w[i];",
     "out[i] = x[i] * inv;"),
    ("page slot of token t taken as (t + 1) % page",
     "size_t src = ((size_t)pg * page + t % page) * row;",
     "size_t src = ((size_t)pg * page + (t + 1) % page) * row;"),
    ("injected state read as [H][N][P] instead of [H][P][N]",
     "h[i] = h0 ? h0[(size_t)hh * P * N + i] : 0.0;",
     "h[i] = h0 ? h0[(size_t)hh * P * N + (i % N) * P + i / N] : 0.0;"),
    ("LM-head argmax tie won by the highest id",
     "if (lg[v] > lg[best]) best = v;",
     "if (lg[v] >= lg[best]) best = v;"),
    ("verification lets a NaN logit win",
     "if (std::isnan(x)) continue;",
     "if (false) continue;"),
    ("verification returns the last accepted token instead of the target's next one",
     "next_token[c] = t[a];",
     "next_token[c] = t[a > 0 ? a - 1 : 0];"),
    ("verification advances the context by the accepted drafts only",
     "if (ctx_lens) ctx_lens[c] += a + 1;",
     "if (ctx_lens) ctx_lens[c] += a;"),
    ("reduced draft head returns the draft row instead of the target id",
     "reduced ? io->draft_to_target[am[j]] : am[j]",
     "am[j]"),
]


def _run_pins(tmp_path, source):
    work = tmp_path / "src"
    work.mkdir()
    (work / "hspec_oracle.cpp").write_text(source)
    shutil.copy(HDR, work / "hspec_oracle.h")
    lib = tmp_path / "liboracle.so"
    subprocess.run(["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", str(work / "hspec_oracle.cpp"),
                    "-o", str(lib)], check=True, capture_output=True)
    env = dict(os.environ, HSPEC_ORACLE_LIB=str(lib), OMP_NUM_THREADS="4")
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu",
                           *PINS], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)


def test_unchanged_copy_passes_every_pin(tmp_path):
    r = _run_pins(tmp_path, open(SRC).read())
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]


@pytest.mark.parametrize("what,good,bad", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_fails_a_pin(tmp_path, what, good, bad):
    src = open(SRC).read()
    assert src.count(good) == 1, f"the line to mutate is not unique in the oracle: {good}"
    r = _run_pins(tmp_path, src.replace(good, bad))
    assert r.returncode == 1, f"no pin failed with the mistake '{what}':\n{r.stdout[-1500:]}"
