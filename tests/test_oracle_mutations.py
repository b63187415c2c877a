"""The oracle's pins must reject a wrong oracle. Each case plants one plausible
mistake (a dropped term, a wrong sign, exponent or index, a transposed operand)
in a copy of the oracle's C source, compiles it on the CPU, and runs the pin
suite against it (tests/test_oracle_pins.py, through LA_ORACLE_LIBRARY): at
least one pin must fail. The unmutated copy, built the same way, must pass."""
import os
import subprocess
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SOURCE = os.path.join(ROOT, "oracle", "lightning_oracle.c")

# (what the mistake is, text in the source, replacement, which occurrence)
MUTATIONS = [
    ("definition: carried state decays i instead of i+1 steps",
     "i+1 steps of decay */\n            const double dq = exp(-s * (double)(i + 1));",
     "i+1 steps of decay */\n            const double dq = exp(-s * (double)(i));", 0),
    ("definition: the diagonal term dropped",
     "for (size_t j = 0; j <= i; ++j) {", "for (size_t j = 0; j < i; ++j) {", 0),
    ("definition: decay with the wrong sign",
     "const double w = exp(-s * (double)(i - j)) * qk;", "const double w = exp(s * (double)(i - j)) * qk;", 0),
    ("blockwise: the inter-block term dropped",
     "Ot[i * d + c] = intra + inter;", "Ot[i * d + c] = intra;", 0),
    ("blockwise: key decay one step off",
     "exp(-s * (double)(m - 1 - j))) * Vt[j * d + c];", "exp(-s * (double)(m - j))) * Vt[j * d + c];", 0),
    ("blockwise: full-block decay on a short last block",
     "const double dblock = exp(-s * (double)m);", "const double dblock = exp(-s * (double)B);", 0),
    ("recurrence: state update transposed",
     "S[r * d + c] = decay * S[r * d + c] + ki[r] * vi[c];",
     "S[r * d + c] = decay * S[r * d + c] + ki[c] * vi[r];", 0),
    ("snapshots: state update transposed",
     "S[r * d + c] = decay * S[r * d + c] + ki[r] * vi[c];",
     "S[r * d + c] = decay * S[r * d + c] + ki[c] * vi[r];", 1),
    ("backward: the state gradient decays one step too many",
     "const double carry = (jj + 1 == L) ? 1.0 : decay;", "const double carry = decay;", 0),
    ("decode: the state not decayed",
     "S[r * d + c] = decay * S[r * d + c] + kr * widen(v, dtype, base + c);",
     "S[r * d + c] = S[r * d + c] + kr * widen(v, dtype, base + c);", 0),
    ("norm_gate: sigmoid of -g",
     "/ (1.0 + exp(-gv));", "/ (1.0 + exp(gv));", 0),
    ("norm_gate: per-head mean divided by all channels",
     "ss / (double)group + eps", "ss / (double)N + eps", 0),
    ("rope: not a rotation",
     "out[i] = x[i] * cs - x[i + half] * sn;", "out[i] = x[i] * cs + x[i + half] * sn;", 0),
    ("gqa decode: the new token's value read from the cache",
     "acc[c] += w * (p < P ? widen(v_cache", "acc[c] += w * (p <= P ? widen(v_cache", 0),
    ("gqa prefill: query rotated one position late",
     "ROPE_NEW(qr, i);", "ROPE_NEW(qr, i + 1);", 0),
    ("gqa prefill: a query does not see its own key",
     "const long P = (long)start + i;", "const long P = (long)start + i - 1;", 0),
    ("blockwise: query decay one step short",
     "const double dq = exp(-s * (double)(i + 1)); /* query decay d_q[i] */",
     "const double dq = exp(-s * (double)(i)); /* query decay d_q[i] */", 0),
    ("backward: dk from the transposed gradient state",
     "acc += R[r * d + c] * V[jj * d + c];", "acc += R[c * d + r] * V[jj * d + c];", 0),
    ("backward: the state-in gradient not decayed",
     "const double f = L > 0 ? decay : 1.0;", "const double f = 1.0;", 0),
    ("decode: the output read from k",
     "const double qr = widen(q, dtype, base + r);", "const double qr = widen(k, dtype, base + r);", 0),
    ("norm_gate: eps added outside the square root",
     "1.0 / sqrt(ss / (double)group + eps);", "1.0 / (sqrt(ss / (double)group) + eps);", 0),
    ("norm_gate: the weight of the head's channel only",
     "(double)gamma[n] * x * inv", "(double)gamma[n % d] * x * inv", 0),
    ("rope: frequencies halved",
     "pow(base, -2.0 * i / (double)rot)", "pow(base, -1.0 * i / (double)rot)", 0),
    ("gqa decode: KV head by modulo instead of by group",
     "hk = h / group;", "hk = h % kv_heads;", 0),
    ("gqa prefill: scores not scaled",
     "sc[p] = scale * dot;", "sc[p] = dot;", 1),
]


def _build_copy(tmp_path, text):
    src = tmp_path / "oracle_copy.c"
    lib = tmp_path / "liboracle_copy.so"
    src.write_text(text)
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-o", str(lib),
                    str(src), "-lm"], check=True)
    return str(lib)


def _pins_pass(lib):
    env = dict(os.environ, LA_ORACLE_LIBRARY=lib, OMP_NUM_THREADS="4")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.join(HERE, "test_oracle_pins.py"), "-x", "-q",
                        "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode == 0, r.stdout[-2000:]


def _mutate(text, old, new, occurrence):
    assert text.count(old) > occurrence, "mutation anchor not found: " + old
    at = -1
    for _ in range(occurrence + 1):
        at = text.index(old, at + 1)
    return text[:at] + new + text[at + len(old):]


def test_the_unmutated_copy_passes_the_pins(tmp_path):
    ok, out = _pins_pass(_build_copy(tmp_path, open(SOURCE).read()))
    assert ok, out


@pytest.mark.parametrize("what,old,new,occurrence", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_a_planted_mistake_fails_a_pin(tmp_path, what, old, new, occurrence):
    lib = _build_copy(tmp_path, _mutate(open(SOURCE).read(), old, new, occurrence))
    ok, out = _pins_pass(lib)
    assert not ok, "every pin passes with the planted mistake: " + what
