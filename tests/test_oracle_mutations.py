"""The oracle's pins must catch plausible mistakes.

Each case below plants one mistake in a copy of ``oracle/dsa3d_oracle.c`` (on the CPU only),
builds it, and runs the pin suites (attention, and the layer's convolution and offset network)
against that copy; the suites must fail.  This checks that the
pins fix the oracle rather than merely agreeing with it.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "dsa3d_oracle.c")

MUTANTS = {
    "scale_1_over_dh": ("double scale = 1.0 / sqrt((double)dh);\n    int64_t p[3], b[3];\n    coords(P, n, p);\n    decode_t d = decode(P, h, n);\n    double m",
                        "double scale = 1.0 / (double)dh;\n    int64_t p[3], b[3];\n    coords(P, n, p);\n    decode_t d = decode(P, h, n);\n    double m"),
    "no_upper_face_rule": ("if (b[a] == D - 1 && d->f[a] != 0.0f) valid = 0;", ""),
    "swapped_corner_weight": ("w *= ca ? (double)f[a] : 1.0 - (double)f[a];\n    }\n    return w;\n}\nstatic",
                              "w *= ca ? 1.0 - (double)f[a] : (double)f[a];\n    }\n    return w;\n}\nstatic"),
    "uncentred_window": ("uvw[2] = tau % P->kw - rw;", "uvw[2] = tau % P->kw;"),
    "dropped_D": ("double dS = Pt * (dP - D);", "double dS = Pt * dP;"),
    "dropped_value_offset_term": ("doff[a] += scale * dS * qk + Pt * ov;", "doff[a] += scale * dS * qk;"),
    "flipped_derivative_sign": ("if (a == axis) w *= ca ? 1.0 : -1.0;", "if (a == axis) w *= ca ? -1.0 : 1.0;"),
    "dk_missing_scale": ("double gk = w * scale * S.dS[tau];", "double gk = w * S.dS[tau];"),
    "transposed_coords": ("p[1] = (n / P->Wp) % P->Hp;", "p[1] = (n / P->Hp) % P->Wp;"),
    "lse_without_log_l": ("return m + log(l);", "return m;"),
    "no_carry": ("if (fr == 1.0f) {", "if (0) {"),
    "dv_uses_dS": ("double gv = w * S.P[tau];", "double gv = w * S.dS[tau];"),
    "dq_uses_vtil": ("dq[e] += scale * dS * S->ktil[e];", "dq[e] += scale * dS * S->vtil[e];"),
    "per_tap_offsets_read_tap_0": ("* P->n_off + tau) * 3);", "* P->n_off + 0) * 3);"),
    "per_tap_gradient_not_per_tap": ("double *doff = doff_all + (P->n_off > 1 ? 3 * tau : 0);",
                                     "double *doff = doff_all;"),
    "dwconv_convolution_not_correlation": (
        "const int64_t ts = t0 + u - rt, ys = y0 + v - rh, xs = x0 + ww - rw;\n"
        "                        if (ts < 0 || ts >= F || ys < 0 || ys >= Hp || xs < 0 || xs >= Wp) continue;\n"
        "                        const int64_t src = (ts * Hp + ys) * Wp + xs;\n                        acc",
        "const int64_t ts = t0 - u + rt, ys = y0 - v + rh, xs = x0 - ww + rw;\n"
        "                        if (ts < 0 || ts >= F || ys < 0 || ys >= Hp || xs < 0 || xs >= Wp) continue;\n"
        "                        const int64_t src = (ts * Hp + ys) * Wp + xs;\n                        acc"),
    "dwconv_bias_dropped": ("double acc = b ? (double)b[c] : 0.0;", "double acc = 0.0;"),
    "dwconv_dw_wrong_source": ("dw[wi] += g * rd(x, io, src * C + c);", "dw[wi] += g * rd(x, io, n * C + c);"),
    "dwconv_dx_wrong_target": ("dx[src * C + c] += (double)w[wi] * g;", "dx[n * C + c] += (double)w[wi] * g;"),
    "dwconv_db_dropped": ("            db[c] += g;\n", ""),
}
PIN_FILES = ["test_oracle_pins.py", "test_oracle_layer_pins.py"]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", "-std=c11",
                    "-o", str(lib), str(mut), "-lm"], check=True)
    env = dict(os.environ, DSA3D_ORACLE_LIB=str(lib), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        *(os.path.join(ROOT, "tests", f) for f in PIN_FILES)],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins accepted the planted mistake {name}:\n{r.stdout[-2000:]}"
