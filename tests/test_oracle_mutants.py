"""The oracle's pins catch plausible mistakes.  Each case below plants one mistake in a copy of
the oracle's C source (a dropped term, a wrong sign, a wrong or transposed operand, a missing
sum over the broadcast rows), builds that copy in a scratch tree and runs the pin tests
(test_oracle.py, test_oracle_pwa.py, test_oracle_pair_bias.py) against it: at least one pin
must fail.  The unchanged copy must pass them all, so that a failure means the mistake was
found and not that the scratch tree is broken.  Nothing here touches the repository's own
oracle build."""
import os
import re
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_TESTS = ["tests/test_oracle.py", "tests/test_oracle_pwa.py", "tests/test_oracle_pair_bias.py"]

# name: (text in pba_oracle.c, the mistaken text)
MUTANTS = {
    # attention forward
    "bias_scaled_with_the_dot_product": (
        "s[j] = scale * dot + (bias ? bias[(size_t)i * Nk + j] : 0.0);",
        "s[j] = scale * (dot + (bias ? bias[(size_t)i * Nk + j] : 0.0));"),
    "masked_keys_in_the_normaliser": (
        "if (!keep || keep[j]) z += exp(s[j] - m);",
        "z += exp(s[j] - m);"),
    "lse_without_the_row_max": ("return m + log(z);", "return log(z);"),
    "gate_dropped_from_out": ("out[(size_t)i * C + c] = gate * o;", "out[(size_t)i * C + c] = o;"),
    # attention backward
    "dgate_without_one_minus_sigmoid": (
        "dg[e] = g ? dout[e] * o[e] * sg * (1.0 - sg) : 0.0;",
        "dg[e] = g ? dout[e] * o[e] * sg : 0.0;"),
    "D_without_the_P_weight": ("D += P[(size_t)i * Nk + j] * acc;", "D += acc;"),
    "dS_sign_of_D": ("* (dP[(size_t)i * Nk + j] - D);", "* (dP[(size_t)i * Nk + j] + D);"),
    "dq_without_scale": ("dq[(size_t)i * C + c] = scale * acc;", "dq[(size_t)i * C + c] = acc;"),
    "dk_from_k_instead_of_q": (
        "acck += dS[(size_t)i * Nk + j] * q[(size_t)i * C + c];",
        "acck += dS[(size_t)i * Nk + j] * k[(size_t)j * C + c];"),
    "dv_from_ungated_dout": (
        "accv += P[(size_t)i * Nk + j] * dOa[(size_t)i * C + c];",
        "accv += P[(size_t)i * Nk + j] * dout[(size_t)i * C + c];"),
    "dbias_not_summed_over_rows": (
        "if (dbh) for (size_t e = 0; e < (size_t)Nq * Nk; ++e) dbh[e] += dss[e];",
        "if (dbh) for (size_t e = 0; e < (size_t)Nq * Nk; ++e) dbh[e] = dss[e];"),
    "dbias_row_not_summed_over_rows": (
        "dbias_row[j] += p[j] * (dP[j] - D);", "dbias_row[j] = p[j] * (dP[j] - D);"),
    # pair-weighted averaging
    "pwa_lse_without_the_row_max": ("*lse = m + log(l);", "*lse = log(l);"),
    "pwa_gate_dropped": ("out[e] = g ? sigmoid(g[e]) * o : o;", "out[e] = o;"),
    "pwa_dgate_without_one_minus_sigmoid": (
        "if (g && dg) dg[e] = dout[e] * o * s * (1.0 - s);",
        "if (g && dg) dg[e] = dout[e] * o * s;"),
    "pwa_dv_with_transposed_weights": (
        "for (int i = 0; i < N; ++i) a += w[(size_t)i * N + j] * doa",
        "for (int i = 0; i < N; ++i) a += w[(size_t)j * N + i] * doa"),
    "pwa_dbias_without_the_row_centring": (
        "= w[(size_t)i * N + j] * (dw[j] - r);", "= w[(size_t)i * N + j] * dw[j];"),
    # pair-bias prologue
    "layernorm_unbiased_variance": ("var /= Cz;", "var /= (Cz - 1);"),
    "layernorm_eps_outside_the_root": ("*sigma = sqrt(var + eps);", "*sigma = sqrt(var) + eps;"),
    "projection_without_beta": (
        "s += (gamma[c] * xh[c] + beta[c]) * w[(size_t)c * H + h];",
        "s += gamma[c] * xh[c] * w[(size_t)c * H + h];"),
    "dw_from_the_normalised_row": ("dw[(size_t)c * H + h] += y * g[h];", "dw[(size_t)c * H + h] += xh[c] * g[h];"),
    "dgamma_without_xh": ("dgamma[c] += s * xh[c];", "dgamma[c] += s;"),
    "dz_without_the_projection_term": (
        "dzr[c] = (gamma[c] * dy[c] - m1 - xh[c] * m2) / sigma;",
        "dzr[c] = (gamma[c] * dy[c] - m1) / sigma;"),
}


def _source():
    with open(os.path.join(ROOT, "oracle", "pba_oracle.c")) as f:
        return f.read()


def _scratch_tree(dst, src_text):
    """oracle/ (with the given C source, built), pba_inputs/ and the pin tests under dst."""
    ign = shutil.ignore_patterns("*.so", "*.tmp*", "__pycache__")
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dst, "oracle"), ignore=ign)
    shutil.copytree(os.path.join(ROOT, "pba_inputs"), os.path.join(dst, "pba_inputs"), ignore=ign)
    os.makedirs(os.path.join(dst, "tests"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dst, "tests", "golden"))
    for name in ["conftest.py", "pba_testlib.py"] + [os.path.basename(p) for p in PIN_TESTS]:
        shutil.copy(os.path.join(ROOT, "tests", name), os.path.join(dst, "tests", name))
    with open(os.path.join(dst, "oracle", "pba_oracle.c"), "w") as f:
        f.write(src_text)
    env = dict(os.environ, PYTHONDONTWRITEBYTECODE="1")
    subprocess.run([sys.executable, "-c", "import oracle; oracle.build(force=True)"], cwd=dst,
                   env=env, check=True, capture_output=True, timeout=300)


def _run_pins(dst):
    env = dict(os.environ, OMP_NUM_THREADS="2", PYTHONDONTWRITEBYTECODE="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        "-m", "not gpu"] + PIN_TESTS,
                       cwd=dst, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, (r.stdout + r.stderr).strip().splitlines()[-1:]


def _case(tmp_root, name, src_text):
    dst = os.path.join(tmp_root, name)
    _scratch_tree(dst, src_text)
    return name, _run_pins(dst)


def test_every_planted_mistake_fails_a_pin(tmp_path):
    src = _source()
    cases = {"unchanged": src}
    for name, (old, new) in MUTANTS.items():
        assert src.count(old) == 1, "%s: the text to change must occur exactly once" % name
        cases[name] = src.replace(old, new)
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with ThreadPoolExecutor(workers) as ex:
        results = dict(ex.map(lambda kv: _case(str(tmp_path), *kv), cases.items()))
    rc, tail = results.pop("unchanged")
    assert rc == 0, "the unchanged oracle copy must pass its pins: %s" % tail
    missed = [n for n, (rc, tail) in results.items()
              if rc != 1 or not any(re.search(r"\b1 failed\b", t) for t in tail)]
    assert not missed, "mistakes no pin caught: %s" % ", ".join(
        "%s (%s)" % (n, results[n][1]) for n in missed)
