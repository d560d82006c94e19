"""Plants mistakes in copies of the oracle (on the CPU) and checks that the
pins catch each one: a pin suite that passes a broken oracle pins nothing.

Each mutant is compiled from a mutated copy of the oracle source into a
temporary directory, and the pin suite is run against it in a subprocess; the
run must fail. The shipped oracle is never modified.
"""

import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "tgd_oracle.cpp")

# (name, original text, mutated text): each is a plausible slip.
MUTANTS = [
    ("adam_dropped_1_minus_beta1", "m[1] = (float)(b1 * m[1] + (1 - b1) * g.im);",
     "m[1] = (float)(b1 * m[1] + g.im);"),
    ("no_bias_correction", "const double bc1 = 1 - std::pow(h.b1, s)", "const double bc1 = 1.0 + 0 * s"),
    ("weight_update_sign", "cd nv = {wv.re * decay - h.lr * X[e].re",
     "cd nv = {wv.re * decay + h.lr * X[e].re"),
    ("projection_transposed_U", "cd c = proj ? conj(U[ki * rn + jo]) : U[jo * rn + ki];",
     "cd c = proj ? conj(U[(jo * rn + ki) % (In * rn)]) : U[jo * rn + ki];"),
    ("expand_conjugated", "cd c = proj ? conj(U[ki * rn + jo]) : U[jo * rn + ki];",
     "cd c = proj ? conj(U[ki * rn + jo]) : conj(U[jo * rn + ki]);"),
    ("gram_missing_conj", "cd p = x1[b] * conj(x2[b]);", "cd p = x1[b] * x2[b];"),
    ("key_without_fma", "float k = std::fma(re, re, im2);", "float rr = re * re; float k = rr + im2;"),
    ("scatter_off_by_one", "X[*it - base] = X[*it - base] + sparse_upd[j];",
     "X[(*it - base + 1) % (Ia * Ib)] = X[(*it - base + 1) % (Ia * Ib)] + sparse_upd[j];"),
    ("jacobi_row_sign", "A[p * n + j] = {c * xp.re - s * xq.re, c * xp.im - s * xq.im};",
     "A[p * n + j] = {c * xp.re + s * xq.re, c * xp.im + s * xq.im};"),
    ("mask_not_applied", "X[e] = in_omega[base + e] ? cd{0, 0} : load_elem(g, h.gdt, base + e);",
     "X[e] = load_elem(g, h.gdt, base + e);"),
    ("bias_correction_step_off_by_one", "const double s = (double)(h.t + 1);",
     "const double s = (double)(h.t + 2);"),
    ("decay_applied_after_update",
     "cd nv = {wv.re * decay - h.lr * X[e].re, wv.im * decay - h.lr * X[e].im};",
     "cd nv = {(wv.re - h.lr * X[e].re) * decay, (wv.im - h.lr * X[e].im) * decay};"),
    ("sparse_scale_dropped",
     "    cd u = adam_update(gj, &h.sp_m[j * mc], &h.sp_v[j * vc], h, bc1, bc2);\n"
     "    sparse_upd[j] = {h.o.sparse_scale * u.re, h.o.sparse_scale * u.im};",
     "    cd u = adam_update(gj, &h.sp_m[j * mc], &h.sp_v[j * vc], h, bc1, bc2);\n"
     "    sparse_upd[j] = {u.re, u.im};"),
    ("moment_reset_ignored", "if (h.o.moments_on_refresh == 1) {", "if (h.o.moments_on_refresh == 7) {"),
    ("view_as_real_v_uses_abs2", "v[1] = (float)(b2 * v[1] + (1 - b2) * g.im * g.im);",
     "v[1] = (float)(b2 * v[1] + (1 - b2) * abs2(g));"),
    ("refresh_schedule_off_by_one", "if (h.o.auto_refresh && h.T > 0 && h.t % h.T == 0) refresh(h, g);",
     "if (h.o.auto_refresh && h.T > 0 && (h.t + 1) % h.T == 0) refresh(h, g);"),
    ("random_draw_ignores_ordinal", "uint64_t s = sm_mix(seed + (ordinal + 1) * SM_GAMMA);",
     "uint64_t s = sm_mix(seed + SM_GAMMA);"),
    ("eigenvalues_ascending", "[&](int64_t a, int64_t b) { return A[a * n + a].re > A[b * n + b].re; });",
     "[&](int64_t a, int64_t b) { return A[a * n + a].re < A[b * n + b].re; });"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, name
    with tempfile.TemporaryDirectory() as d:
        mut = os.path.join(d, "mutant.cpp")
        so = os.path.join(d, "mutant.so")
        open(mut, "w").write(src.replace(old, new))
        subprocess.run(["g++", "-O1", "-std=c++17", "-fPIC", "-shared", "-pthread",
                        "-ffp-contract=off", "-o", so, mut], check=True)
        env = dict(os.environ, TGD_ORACLE_LIB=so, TGD_ORACLE_THREADS="2")
        r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                            os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                           env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
        assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"
