"""The oracle's pins catch plausible mistakes (CPU only).  Each case copies the
oracle into a temporary package, plants one mistake in its C source (a wrong
table entry, bias, index, sign, tie rule, dropped term or swapped operand;
where the same step is written at two sites, at both),
builds it and runs tests/test_oracle_pins.py against that copy in a
subprocess: the pins must fail.  An unmodified copy must pass them, and the
subprocess must import the copy, not the repository's oracle."""
import concurrent.futures
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

MUTANTS = {
    "codebook entry": ("{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0}", "{0.0, 0.5, 1.0, 1.5, 2.0, 2.5, 4.0, 6.0}"),
    "E4M3 exponent bias": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);", "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "E4M3 subnormal step": ("v = ldexp((double)m / 8.0, -6);", "v = ldexp((double)m / 8.0, -7);"),
    "nibble order": ("return (i & 1) ? (uint8_t)(b >> 4) : (uint8_t)(b & 15);",
                     "return (i & 1) ? (uint8_t)(b & 15) : (uint8_t)(b >> 4);"),
    "transcode global exponent": ("int g = have ? kmax - 8 : 0;", "int g = have ? kmax - 7 : 0;"),
    "group score drops its second term": ("gscore[g] = (i2 < 0) ? c[i1] : c[i1] + c[i2];", "gscore[g] = c[i1];"),
    "group ties to the higher index": ("(best < 0 || gscore[g] > gscore[best])", "(best < 0 || gscore[g] >= gscore[best])"),
    "expert ties to the higher index": ("!taken[e] && (best < 0 || c[e] > c[best])) best = e;",
                                        "!taken[e] && (best < 0 || c[e] >= c[best])) best = e;"),
    "renormalised weights without rsf": ("renormalize ? (sj / S) * rsf : sj * rsf", "renormalize ? (sj / S) : sj * rsf"),
    "weights from the biased score": ("float sj = s[topk_ids", "float sj = c[topk_ids"),
    "quantiser scale divisor": ("float v = amax / 6.0f;", "float v = amax / 4.0f;"),
    "E2M1 ties to the odd code": ("double d = fabs(E2M1_MAGNITUDE[c] - a);\n        if (d < best_d || (d == best_d && (c & 1) == 0))",
                                  "double d = fabs(E2M1_MAGNITUDE[c] - a);\n        if (d < best_d || (d == best_d && (c & 1) == 1))"),
    "E4M3 ties to the odd code": ("double d = fabs(orc_e4m3_value((uint8_t)c) - a);\n        if (d < best_d || (d == best_d && (c & 1) == 0))",
                                  "double d = fabs(orc_e4m3_value((uint8_t)c) - a);\n        if (d < best_d || (d == best_d && (c & 1) == 1))"),
    "E2M1 drops the sign of zero": ("return (uint8_t)(signbit(x) ? (best | 8) : best);", "return (uint8_t)(x < 0 ? (best | 8) : best);"),
    "SiLU sign": ("return g / (1.0 + exp(-g));", "return g / (1.0 + exp(g));"),
    "gate and up swapped": ("a[i] = silu(g) * u;", "a[i] = silu(u) * g;"),
    "down weight row index": ("const int64_t r = (int64_t)e * H + h;", "const int64_t r = (int64_t)e * H + (H - 1 - h);",
                              2),
    "block scale index": ("orc_e4m3_value(sf[k / 16]) * global;", "orc_e4m3_value(sf[k / 32]) * global;"),
    "combine drops the routing weight": ("o[h] += (double)wts[q] * y;", "o[h] += y;"),
    "permutation not stable": ("        for (int64_t p = 0; p < P; ++p)\n            if (topk_ids[p] == e) {",
                               "        for (int64_t p = P - 1; p >= 0; --p)\n            if (topk_ids[p] == e) {"),
    "MXFP8 scale exponent": ("X = ex - 1 - 8;", "X = ex - 1 - 7;"),
    "compact spread limit": ("emax - e_of[b] > 14) ok = 0;", "emax - e_of[b] > 15) ok = 0;"),
    "transcode spread limit": ("else if (have && kmax - kmin > 17) status = 1;", "else if (have && kmax - kmin > 18) status = 1;"),
    "transcode zero test on the sign bit": ("if (nibble(c + b * 16, i) & 7) zero = 0;", "if (nibble(c + b * 16, i)) zero = 0;",
                                            2),
    "transcode second half scale": ("so[2 * b + 1] = byte; /* second 16-code half */",
                                    "so[2 * b + 1] = byte ? (uint8_t)(byte - 8) : 0; /* second 16-code half */"),
    "exp series drops a term": ("    p = fmaf(p, r, (float)(1.0 / 6.0));\n", ""),
    "exp reduction sign": ("float r = fmaf(-n, ln2_hi, y);", "float r = fmaf(n, ln2_hi, y);"),
    "sigmoid negative branch": ("return e / (1.0f + e);", "return 1.0f / (1.0f + e);"),
    "quantiser ignores the global": ("            v = v / gs;\n", ""),
    "router logits transposed operand": ("const double b = (double)w[(int64_t)e * H + h];",
                                         "const double b = (double)w[(int64_t)h * E + e];"),
    "E8M0 bias": ("return ldexp(1.0, (int)byte - 127);", "return ldexp(1.0, (int)byte - 128);"),
    "MXFP8 element scaling direction": ("orc_e4m3_rne_satfinite(ldexpf(xb[i], -X));", "orc_e4m3_rne_satfinite(ldexpf(xb[i], X));"),
    "compact decode nibble order": ("const int n = (b & 1) ? (byte >> 4) : (byte & 15);",
                                    "const int n = (b & 1) ? (byte & 15) : (byte >> 4);"),
    "one group too few kept": ("for (int r = 0; r < topk_group; ++r) {", "for (int r = 0; r + 1 < topk_group; ++r) {"),
    "renormalisation sum drops the last weight": ("for (int j = 0; j < top_k; ++j) S = S + s[",
                                                  "for (int j = 0; j + 1 < top_k; ++j) S = S + s["),
    "permutation offsets shifted": ("offsets[e + 1] = offsets[e] + counts[e];", "offsets[e + 1] = offsets[e] + counts[E - 1 - e];"),
    "W4A16 intermediate not rounded to BF16": (
        "for (int i = 0; i < I; ++i) a[i] = (double)orc_bf16_to_float(orc_float_to_bf16((float)a[i]));",
        "for (int i = 0; i < I; ++i) a[i] = (double)(float)a[i];"),
    "intermediate quantised with the input global": ("orc_quantize_f32(a32, 1, I, act_global_mid, aq, as);",
                                                     "orc_quantize_f32(a32, 1, I, act_global, aq, as);"),
    "compact field sign": ("int lo = zero_of[2 * j] ? 15 : emax - e_of[2 * j];",
                           "int lo = zero_of[2 * j] ? 15 : e_of[2 * j] - emax;"),
}


def _copy_oracle(dst, mutation):
    pkg = os.path.join(dst, "oracle")
    os.makedirs(pkg)
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), pkg)
    src = open(os.path.join(ROOT, "oracle", "nvfp4_oracle.c")).read()
    if mutation is not None:
        old, new, sites = (*mutation, 1) if len(mutation) == 2 else mutation
        assert src.count(old) == sites, f"mutation site count changed: {old!r}"
        src = src.replace(old, new)
    open(os.path.join(pkg, "nvfp4_oracle.c"), "w").write(src)


def _env(dst):
    return dict(os.environ, PYTHONPATH=os.pathsep.join([dst, ROOT]), OMP_NUM_THREADS="2")


def _run_pins(dst):
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu", PINS]
    r = subprocess.run(cmd, cwd=dst, env=_env(dst), capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    base = tmp_path_factory.mktemp("oracle_mutants")
    cases = {"(unmodified)": None, **MUTANTS}
    dirs = {}
    for i, (name, mut) in enumerate(cases.items()):
        d = str(base / f"m{i}")
        _copy_oracle(d, mut)
        dirs[name] = d
    # the subprocess imports the copy
    d0 = dirs["(unmodified)"]
    where = subprocess.run([sys.executable, "-c", "import oracle; print(oracle.__file__)"], cwd=d0, env=_env(d0),
                           capture_output=True, text=True, timeout=120).stdout.strip()
    assert where.startswith(d0), where
    with concurrent.futures.ThreadPoolExecutor(max_workers=max(2, min(8, os.cpu_count() or 2))) as ex:
        futs = {name: ex.submit(_run_pins, d) for name, d in dirs.items()}
        return {name: f.result() for name, f in futs.items()}


def test_unmodified_copy_passes_the_pins(outcomes):
    rc, out = outcomes["(unmodified)"]
    assert rc == 0, out


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistake_fails_a_pin(outcomes, name):
    rc, out = outcomes[name]
    assert rc == 1, f"{name}: pins passed (exit {rc})\n{out}"
