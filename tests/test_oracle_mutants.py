"""Mutation tests of the oracle's pins.

Each case plants one plausible mistake in a copy of the oracle's C source (a
dropped term, a wrong sign, a swapped index, a transposed operand, an
off-by-one, a wrong order), compiles that copy into a scratch library and
runs the pin tests of the part it touches against it.  The pins must fail.
A control compiles the unmodified source the same way, and its pins must
pass.  So a pin suite that cannot tell the definition from a near miss of it
shows up here.

Mistakes are planted in the oracle only, on the CPU.
"""
import concurrent.futures as cf
import os
import re
import subprocess
import sys

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

SWITCH = ["test_oracle_switch.py"]
BUILD = ["test_oracle_build.py", "test_oracle_build_random.py"]
ATTN = ["test_oracle_attention.py", "test_oracle_attention_random.py"]
SMOOTH = ["test_oracle_smooth.py", "test_oracle_attention_random.py"]
LOCAL = ["test_oracle_local.py", "test_oracle_attention_random.py"]
VERLET = ["test_oracle_verlet.py"]

# (name, pin files, text of the definition, the planted mistake)
MUTANTS = [
    # the switch and its cosine (cosine switch from r_on to rcut)
    ("taylor_sign", SWITCH,
     "c[k] = -c[k - 1] / div;", "c[k] = c[k - 1] / div;"),
    ("taylor_factorial", SWITCH,
     "double div = (double)((2 * k) * (2 * k + 1));", "double div = (double)((2 * k) * (2 * k - 1));"),
    ("taylor_truncated", SWITCH,
     "#define ORC_NTAYLOR 12", "#define ORC_NTAYLOR 6"),
    ("cos_phase", SWITCH,
     "double t = u - 0.5;", "double t = u + 0.5;"),
    ("switch_half_dropped", SWITCH,
     "return 0.5 * one_plus;", "return one_plus;"),
    ("switch_scaled_by_rcut", SWITCH,
     "double u = num / den;", "double u = num / rcut;"),
    ("switch_onset", SWITCH,
     "if (r < r_on) return 1.0;", "if (r < r_on) return 0.5;"),
    # the neighbour set, its cap and its order
    ("vector_sign", BUILD,
     "v[c] = xs - xi[c];", "v[c] = xi[c] - xs;"),
    ("cutoff_inclusive", BUILD,
     "if (r2 < g->rc2) {", "if (r2 <= g->rc2) {"),
    ("self_images_dropped", BUILD,
     "if (j == i && S[0] == 0 && S[1] == 0 && S[2] == 0) continue;", "if (j == i) continue;"),
    ("image_range_minimum_image", BUILD,
     "g->reach[k] = rcut / h;", "g->reach[k] = 0.5 * rcut / h;"),
    ("negative_images_dropped", BUILD,
     "lo[k] = (int)ceil(-df - g->reach[k] - 1e-6);", "lo[k] = (int)ceil(-df - 1e-6);"),
    ("shift_wrong_box_row", BUILD,
     "double p1 = s1 * g->a[1][c];", "double p1 = s1 * g->a[0][c];"),
    ("r2_term_dropped", BUILD,
     "r2 = r2 + t2;", "r2 = r2 + 0.0 * t2;"),
    ("cap_keeps_farthest", BUILD,
     "if (a->r2 < b->r2) return -1;\n    if (a->r2 > b->r2) return 1;",
     "if (a->r2 > b->r2) return -1;\n    if (a->r2 < b->r2) return 1;"),
    ("cap_tie_break_reversed", BUILD,
     "if (a->j != b->j) return a->j < b->j ? -1 : 1;\n    for (int k = 0; k < 3; ++k)\n"
     "        if (a->S[k] != b->S[k]) return a->S[k] < b->S[k] ? -1 : 1;\n    return 0;\n}\n\n"
     "/* canonical",
     "if (a->j != b->j) return a->j > b->j ? -1 : 1;\n    for (int k = 0; k < 3; ++k)\n"
     "        if (a->S[k] != b->S[k]) return a->S[k] > b->S[k] ? -1 : 1;\n    return 0;\n}\n\n"
     "/* canonical"),
    ("cap_off_by_one", BUILD + VERLET,
     "buf->len = nnei_max;", "buf->len = nnei_max - 1;"),
    ("canonical_shift_order_reversed", BUILD,
     "if (a->S[k] != b->S[k]) return a->S[k] < b->S[k] ? -1 : 1;\n    return 0;\n}\n\n"
     "/* Fractional",
     "if (a->S[k] != b->S[k]) return a->S[k] > b->S[k] ? -1 : 1;\n    return 0;\n}\n\n"
     "/* Fractional"),
    ("canonical_sort_skipped", BUILD + VERLET,
     "qsort(buf->buf, (size_t)buf->len, sizeof(orc_cand), cmp_canon);", ";"),
    ("dist_is_r2", BUILD,
     "double r = sqrt(r2);", "double r = r2;"),
    # Verlet-list reuse
    ("refine_cutoff_inclusive", VERLET,
     "if (c.r2 < g->rc2)", "if (c.r2 <= g->rc2)"),
    ("refine_shift_dropped", VERLET,
     "c.S[2] = cand_shift[3 * p + 2];", "c.S[2] = 0;"),
    ("refine_source_as_centre", VERLET,
     "c.r2 = edge_vec(g, x + 3 * i, x + 3 * (int64_t)c.j, c.S, v);",
     "c.r2 = edge_vec(g, x + 3 * (int64_t)c.j, x + 3 * i, c.S, v);"),
    ("refine_reads_next_row", VERLET,
     "for (int64_t p = cand_ptr[i]; p < cand_ptr[i + 1]; ++p) {",
     "for (int64_t p = cand_ptr[i]; p < cand_ptr[i + 1] - 1; ++p) {"),
    # block-dense attention
    ("projection_transposed", ATTN + SMOOTH,
     "acc = acc + x[a * c + k] * W[(int64_t)k * c + m];",
     "acc = acc + x[a * c + k] * W[(int64_t)m * c + k];"),
    ("logit_scale_d", ATTN,
     "double l = ((s[a] * s[b]) * dot) / rsd;\n            P[a * n + b] = l;",
     "double l = ((s[a] * s[b]) * dot) / (double)d;\n            P[a * n + b] = l;"),
    ("logit_query_switch_dropped", ATTN,
     "double l = ((s[a] * s[b]) * dot) / rsd;\n            P[a * n + b] = l;",
     "double l = (s[b] * dot) / rsd;\n            P[a * n + b] = l;"),
    ("logit_key_is_query_row", ATTN,
     "for (int t = 0; t < d; ++t) dot = dot + Q[a * c + h * d + t] * K[b * c + h * d + t];",
     "for (int t = 0; t < d; ++t) dot = dot + Q[a * c + h * d + t] * K[a * c + h * d + t];"),
    ("logit_head_slice", ATTN,
     "for (int t = 0; t < d; ++t) dot = dot + Q[a * c + h * d + t] * K[b * c + h * d + t];",
     "for (int t = 0; t < d; ++t) dot = dot + Q[a * c + t] * K[b * c + t];"),
    ("softmax_max_not_subtracted", ATTN,
     "double e = exp(P[a * n + b] - m);", "double e = exp(P[a * n + b]);"),
    ("softmax_not_normalised", ATTN,
     "for (int64_t b = 0; b < n; ++b) P[a * n + b] = P[a * n + b] / z;",
     "for (int64_t b = 0; b < n; ++b) P[a * n + b] = P[a * n + b] / 1.0;"),
    ("av_map_transposed", ATTN,
     "acc = acc + P[a * n + b] * V[b * c + h * d + t];",
     "acc = acc + P[b * n + a] * V[b * c + h * d + t];"),
    ("av_value_head_slice", ATTN,
     "acc = acc + P[a * n + b] * V[b * c + h * d + t];",
     "acc = acc + P[a * n + b] * V[b * c + t];"),
    # slot-occupancy attention
    ("smooth_phantom_sign", SMOOTH,
     "if (phi > 0) z = z + (double)phi * exp(-m);", "if (phi > 0) z = z + (double)phi * exp(m);"),
    ("smooth_phantoms_dropped", SMOOTH,
     "if (phi > 0) z = z + (double)phi * exp(-m);", "if (phi > 0) z = z + 0.0 * exp(-m);"),
    ("smooth_phantom_count", SMOOTH,
     "int64_t phi = nnei_max - n;", "int64_t phi = nnei_max - n - 1;"),
    ("smooth_one_switch", SMOOTH,
     "double l = ((s[a] * s[b]) * dot) / rsd;\n                        E[b] = l;",
     "double l = (s[b] * dot) / rsd;\n                        E[b] = l;"),
    # local attention
    ("local_query_from_edge", LOCAL,
     "project(1, c, H + i * c, Wq, q);", "project(1, c, G + base * c, Wq, q);"),
    ("local_switch_dropped", LOCAL,
     "double l = (sw[base + b] * dot) / rsd;", "double l = dot / rsd;"),
    ("local_not_normalised", LOCAL,
     "acc = acc + (P[b] / z) * V[b * c + h * d + t];", "acc = acc + P[b] * V[b * c + h * d + t];"),
    ("local_empty_row_not_zeroed", LOCAL,
     "for (int m = 0; m < c; ++m) out[i * c + m] = 0.0;\n            if (n <= 0) continue;",
     "if (n <= 0) continue;\n            for (int m = 0; m < c; ++m) out[i * c + m] = 0.0;"),
]

# the same for the oracle's Python side (oracle/__init__.py): the layer chain,
# its fp32 rounding and the CSR's scalar outputs
PY_MUTANTS = [
    ("forward_layers_not_chained", ATTN,
     "        g = o\n", "        g = np.asarray(G0)\n"),
    ("forward_fp32_output_not_rounded", ATTN,
     "            o = o.astype(np.float32)\n", "            o = o.astype(np.float64)\n"),
    ("forward_fp32_switch_not_rounded", ATTN,
     "        sw = sw.astype(np.float32).astype(np.float64)\n", "        sw = sw\n"),
    ("n_truncated_inclusive", BUILD,
     "np.count_nonzero(raw > nnei_max))}\n\n\ndef verlet_candidates(",
     "np.count_nonzero(raw >= nnei_max))}\n\n\ndef verlet_candidates("),
    ("refine_n_truncated_inclusive", VERLET,
     "np.count_nonzero(raw > nnei_max))}\n\n\ndef centre(",
     "np.count_nonzero(raw >= nnei_max))}\n\n\ndef centre("),
    ("verlet_criterion_strict", VERLET,
     "return 2.0 * max_displacement(coords, coords_ref) >= float(skin)",
     "return 2.0 * max_displacement(coords, coords_ref) > float(skin)"),
    ("verlet_list_without_skin", VERLET,
     "    r = float(rcut) + float(skin)\n", "    r = float(rcut)\n"),
]

ALL_PINS = sorted({f for _, files, _, _ in MUTANTS + PY_MUTANTS for f in files})


def _compile(src_text, path):
    c_path = path + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", *oracle.CFLAGS, "-o", path, c_path, "-lm"], check=True,
                   capture_output=True, timeout=120)


# runs pytest with a given file standing in for oracle/__init__.py (loaded as
# the package "oracle" before the tests import it)
_WITH_PACKAGE = (
    "import importlib.util, sys\n"
    "init, args = sys.argv[1], sys.argv[2:]\n"
    "spec = importlib.util.spec_from_file_location('oracle', init)\n"
    "mod = importlib.util.module_from_spec(spec)\n"
    "sys.modules['oracle'] = mod\n"
    "spec.loader.exec_module(mod)\n"
    "import pytest\n"
    "sys.exit(pytest.main(args))\n")


def _run_pins(lib, files, init=None):
    env = dict(os.environ, MLG_ORACLE_LIB=lib, OMP_NUM_THREADS="2",
               PYTHONDONTWRITEBYTECODE="1")
    args = [*[os.path.join(HERE, f) for f in files], "-x", "-q", "-m", "not gpu", "-p",
            "no:cacheprovider"]
    if init is None:
        cmd = [sys.executable, "-m", "pytest", *args]
    else:
        cmd = [sys.executable, "-c", _WITH_PACKAGE, init, *args]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    return r.returncode, (r.stdout + r.stderr)[-1500:]


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    src = open(oracle._SRC).read()
    tmp = str(tmp_path_factory.mktemp("mutants"))
    jobs = {"control": (src, ALL_PINS)}
    for name, files, old, new in MUTANTS:
        assert src.count(old) == 1, f"{name}: the definition's text is not unique in the source"
        jobs[name] = (src.replace(old, new), files)

    lib0 = oracle.build()
    py_src = open(os.path.join(os.path.dirname(oracle._SRC), "__init__.py")).read()
    for name, files, old, new in PY_MUTANTS:
        assert py_src.count(old) == 1, f"{name}: the definition's text is not unique in the source"
        jobs[name] = (py_src.replace(old, new), files)
    # the unmodified Python side through the same stand-in path
    jobs["py_control"] = (py_src, ALL_PINS)
    py_names = {m[0] for m in PY_MUTANTS} | {"py_control"}

    def one(item):
        name, (text, files) = item
        if name in py_names:
            pkg = os.path.join(tmp, f"py_{name}")
            os.makedirs(pkg, exist_ok=True)
            init = os.path.join(pkg, "__init__.py")
            with open(init, "w") as f:
                f.write(text)
            return name, _run_pins(lib0, files, init)
        lib = os.path.join(tmp, f"lib_{name}.so")
        _compile(text, lib)
        return name, _run_pins(lib, files)

    with cf.ThreadPoolExecutor(max_workers=max(2, min(8, (os.cpu_count() or 2) // 2))) as ex:
        return dict(ex.map(one, jobs.items()))


@pytest.mark.parametrize("name", ["control", "py_control"])
def test_control_passes(outcomes, name):
    rc, tail = outcomes[name]
    assert rc == 0, tail


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS + PY_MUTANTS])
def test_mutant_is_caught(outcomes, name):
    rc, tail = outcomes[name]
    # caught: pytest ran and a pin failed, or the mutant crashed (a signal);
    # an error before the pins ran (exit 1 without a failed test) is not
    caught = (rc == 1 and re.search(r"\b\d+ failed\b", tail)) or rc < 0
    assert caught, f"mutant {name} survived the pins (rc {rc}):\n{tail}"
