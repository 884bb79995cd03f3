"""The oracle's pins catch plausible mistakes.

Each case copies the oracle into a temporary directory, plants one mistake in
the copy's C source (the real oracle is never touched), lets the copy compile
itself, and runs the pin tests (tests/test_oracle_pins.py) against it: at least
one pin must fail.  An unplanted copy must pass, so that a failure means the
mistake was caught and not that the copy is broken.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (what the oracle computes, the plausible mistake) as (original text, planted text)
MUTATIONS = {
    "transposed transition": (
        "A[m * dk + j] = alpha_m * (eye - beta * k[m] * k[j]);",
        "A[j * dk + m] = alpha_m * (eye - beta * k[m] * k[j]);"),
    "gate on the value side": (
        "double alpha_m = exp(p->gate == LQO_GATE_SCALAR ? g[0] : g[m]);",
        "double alpha_m = exp(p->gate == LQO_GATE_SCALAR ? g[0] : g[j % dk]);"),
    "dropped beta in the write": (
        "Sn[i * dk + j] = acc + beta * v[i] * k[j];",
        "Sn[i * dk + j] = acc + v[i] * k[j];"),
    "output read before the update": (
        "    memcpy(S, Sn, sizeof(double) * dv * dk);\n    /* o_t = S_t q_t */",
        "    /* o_t = S_t q_t */"),
    "smoothing without the square root": (
        "s[j] = (smooth && m > 0.0f) ? sqrtf(m) : 1.0f;",
        "s[j] = (smooth && m > 0.0f) ? m : 1.0f;"),
    "row scale over 128": (
        "sigma[i] = mx / 127.0f;",
        "sigma[i] = mx / 128.0f;"),
    "codes truncated, not rounded": (
        "code = rintf((R[i * dk + j] * rs[j]) * rho);",
        "code = truncf((R[i * dk + j] * rs[j]) * rho);"),
    "columns ranked before the rows are zeroed": (
        "            R[i * dk + j] = 0.0f;\n        }\n    }\n    /* 1b.",
        "        }\n    }\n    /* 1b."),
    "flush one token early": (
        "(t + 1) % p->window == 0",
        "t % p->window == 0"),
    "row compensators left out of the decoded state": (
        "for (int j = 0; j < dk; ++j) S[i * dk + j] += (double)comp_vec[c * dk + j];",
        "(void)i;"),
    "column compensators left out of the decoded state": (
        "for (int i = 0; i < dv; ++i) S[i * dk + j] += (double)comp_vec[n_rows * dk + c * dv + i];",
        "(void)j;"),
    "max-abs ranking as the default": (
        "if (select == LQO_SELECT_L2) acc = acc + a * a;\n            else if (a > acc) acc = a;\n"
        "        }\n        score[i] = acc;",
        "if (a > acc) acc = a;\n        }\n        score[i] = acc;"),
    "smoothing factors not applied when decoding": (
        "S[i * dk + j] = (double)sigma[i] * (double)Q[i * dk + j] * (double)s[j];",
        "S[i * dk + j] = (double)sigma[i] * (double)Q[i * dk + j];"),
    "smoothing multiplied in where it should divide": (
        "for (int j = 0; j < dk; ++j) rs[j] = 1.0f / s[j];",
        "for (int j = 0; j < dk; ++j) rs[j] = s[j];"),
    "row scale applied as a division by 127/M": (
        "code = rintf((R[i * dk + j] * rs[j]) * rho);",
        "code = rintf((R[i * dk + j] * rs[j]) / rho);"),
    "smoothing in the naive mode": (
        "const int sm = naive ? 0 : p->smooth;",
        "const int sm = p->smooth;"),
}


def _copy_and_run(dest, mutation=None):
    """Copy the oracle and its pin tests to dest, plant the mutation, run the pins."""
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(dest, "oracle"),
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    # the seeded input generators some pins draw from (no kernels are needed)
    pkg = "recurrent_state_quantization_lq_b200"
    shutil.copytree(os.path.join(ROOT, pkg), os.path.join(dest, pkg),
                    ignore=shutil.ignore_patterns("*.so", "__pycache__", "csrc", "_build"))
    os.makedirs(os.path.join(dest, "tests"))
    for name in ("test_oracle_pins.py", "conftest.py"):
        shutil.copy(os.path.join(ROOT, "tests", name), os.path.join(dest, "tests", name))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(dest, "tests", "golden"))
    shutil.copy(os.path.join(ROOT, "pytest.ini"), dest)
    if mutation is not None:
        src = os.path.join(dest, "oracle", "lq_oracle.c")
        with open(src) as f:
            text = f.read()
        original, planted = mutation
        assert text.count(original) == 1, "the mutation's anchor is no longer in the oracle source"
        with open(src, "w") as f:
            f.write(text.replace(original, planted))
    return subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                           "tests/test_oracle_pins.py"], cwd=dest, capture_output=True, text=True, timeout=600)


def test_unplanted_copy_passes(tmp_path):
    r = _copy_and_run(str(tmp_path))
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, name):
    r = _copy_and_run(str(tmp_path), MUTATIONS[name])
    assert r.returncode == 1, (name, r.stdout[-2000:] + r.stderr[-2000:])   # 1: some pin failed
