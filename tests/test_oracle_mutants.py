"""Mutation tests of the oracle's pins (CPU).

Each mutant is a copy of the oracle with one plausible mistake planted in it:
a wrong exponent bias or tie rule in the formats, a dropped term or a missing
scale in the indexer, a reversed order in the selection, a transposed index or
a missing normalisation in the attention, an off-by-one in the window or the
pool, a reordered layer schedule. The pin tests (tests/test_oracle_formats.py,
test_oracle_selection.py, test_oracle_attention.py) run against each mutant in
a subprocess and must fail; the unmutated copy, built the same way, must pass.
A mistake that no pin catches would leave that part of the oracle unchecked.
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_DIR = os.path.join(ROOT, "oracle")
C_SRC = os.path.join(ORACLE_DIR, "csa2_oracle.c")
PY_SRC = os.path.join(ORACLE_DIR, "__init__.py")
PINS = {
    "formats": os.path.join(ROOT, "tests", "test_oracle_formats.py"),
    "selection": os.path.join(ROOT, "tests", "test_oracle_selection.py"),
    "attention": os.path.join(ROOT, "tests", "test_oracle_attention.py"),
}

# (name, text in csa2_oracle.c, replacement, which occurrence (1-based), pin files)
C_MUTANTS = [
    ("e4m3 exponent bias 8", "mag = (1.0 + m / 8.0) * ldexp(1.0, e - 7);",
     "mag = (1.0 + m / 8.0) * ldexp(1.0, e - 8);", 1, ["formats"]),
    ("e4m3 subnormal step 2^-10", "mag = m * ldexp(1.0, -9);", "mag = m * ldexp(1.0, -10);", 1,
     ["formats"]),
    ("e4m3 ties to the larger code",
     "if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {", "if (d <= best_d) {", 1,
     ["formats"]),
    ("e2m1 mantissa weight 1/4", "(1.0 + m / 2.0) * ldexp(1.0, e - 1)",
     "(1.0 + m / 4.0) * ldexp(1.0, e - 1)", 1, ["formats"]),
    ("e2m1 ties to the larger code",
     "if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {", "if (d <= best_d) {", 2,
     ["formats"]),
    ("e2m1 drops the sign of a zero", "return (uint8_t)(best | (signbit(v) ? 0x8 : 0));",
     "return (uint8_t)(best | (v < 0 && best ? 0x8 : 0));", 1, ["formats"]),
    ("fp4 scale amax/4", "float s_f = amax / 6.0f;", "float s_f = amax / 4.0f;", 1, ["formats"]),
    ("fp4 nibble order swapped",
     "packed[r * (C / 2) + (g * 16 + c) / 2] = (uint8_t)(code[0] | (code[1] << 4));",
     "packed[r * (C / 2) + (g * 16 + c) / 2] = (uint8_t)(code[1] | (code[0] << 4));", 1,
     ["formats"]),
    ("fp4 dequantize drops the element sign",
     "double s = orc_e4m3_value(sf[r * (C / 16) + c / 16]);\n            out[r * C + c] = orc_e2m1_value(code) * s;",
     "double s = orc_e4m3_value(sf[r * (C / 16) + c / 16]);\n            out[r * C + c] = orc_e2m1_value(code & 7) * s;",
     1, ["formats"]),
    ("fp4 dequantize takes the wrong group's scale",
     "double s = orc_e4m3_value(sf[r * (C / 16) + c / 16]);",
     "double s = orc_e4m3_value(sf[r * (C / 16) + c / 32]);", 1, ["formats"]),
    ("mx shared exponent minus 1", "int e = (ex - 1) - 2;", "int e = (ex - 1) - 1;", 1, ["formats"]),
    ("index dots drop the first term",
     "for (int i = 0; i < HD; i++)\n            acc += (int64_t)q[i] * (int64_t)k[t * HD + i];\n        S[t] = acc;",
     "for (int i = 1; i < HD; i++)\n            acc += (int64_t)q[i] * (int64_t)k[t * HD + i];\n        S[t] = acc;",
     1, ["selection"]),
    ("index score drops the key scale", "score[t] = s * kscale[t];", "score[t] = s;", 1,
     ["selection"]),
    ("index score truncates above 2^24", "float s = (float)acc; /* round to nearest even */",
     "float s = (acc > 16777216 || acc < -16777216) ? (float)(acc - acc % 4) : (float)acc;", 1,
     ["selection"]),
    ("block max misses the last token",
     "for (int64_t t = 8 * j + 1; t < 8 * j + 8 && t < n_visible; t++)",
     "for (int64_t t = 8 * j + 1; t < 8 * j + 7 && t < n_visible; t++)", 1, ["selection"]),
    ("block count rounds down", "int64_t nblk = (n_visible + 7) / 8;", "int64_t nblk = n_visible / 8;",
     1, ["selection"]),
    ("ties go to the higher position",
     "    if (x->p < y->p) return -1;\n    if (x->p > y->p) return 1;",
     "    if (x->p > y->p) return -1;\n    if (x->p < y->p) return 1;", 1, ["selection"]),
    ("lowest scores first", "    if (x->s > y->s) return -1;\n    if (x->s < y->s) return 1;",
     "    if (x->s < y->s) return -1;\n    if (x->s > y->s) return 1;", 1, ["selection"]),
    ("selection left in rank order", "    qsort(out, (size_t)m, sizeof(int64_t), orc_cmp_i64);\n", "", 1,
     ["selection"]),
    ("attention without the softmax scale", "logit[j] = scale * dot;", "logit[j] = dot;", 1,
     ["attention"]),
    ("attention without the normalisation", "out[h * C + c] = acc / z;", "out[h * C + c] = acc;", 1,
     ["attention"]),
    ("attention reads keys transposed",
     "dot += (double)bf16_to_float(q[h * C + c]) * kv[j * C + c];",
     "dot += (double)bf16_to_float(q[h * C + c]) * kv[c * n + j];", 1, ["attention"]),
    ("attention values shifted by a channel", "acc += logit[j] * kv[j * C + c];",
     "acc += logit[j] * kv[j * C + (c + 1) % C];", 1, ["attention"]),
    ("mx zero block takes exponent 0", "    if (amax == 0.0)\n        return -127;",
     "    if (amax == 0.0)\n        return 0;", 1, ["formats"]),
    ("mx exponent clamped at -126", "    if (e < -127)\n        e = -127;",
     "    if (e < -126)\n        e = -126;", 1, ["formats"]),
    ("e4m3 code 0x7F read as 480", "    if (e == 0xF && m == 0x7)\n        return NAN;\n", "", 1,
     ["formats"]),
    ("e4m3 saturates at 240", "    if (ax > 448.0)\n        ax = 448.0;", "    if (ax > 240.0)\n        ax = 240.0;",
     1, ["formats"]),
    ("zero-scale group keeps the sign of zeros",
     "                    if (s == 0.0f) {\n                        code[u] = 0;",
     "                    if (s == 0.0f) {\n                        code[u] = signbit(xv) ? 0x8 : 0;", 1,
     ["formats"]),
    ("mx elements scaled one exponent low",
     "double v = ldexp((double)bf16_to_float(xr[g * 32 + c + u]), -e);",
     "double v = ldexp((double)bf16_to_float(xr[g * 32 + c + u]), -e - 1);", 1, ["formats"]),
    ("mx dequantize takes the wrong block's scale", "double s = orc_e8m0_value(sf[r * (C / 32) + c / 32]);",
     "double s = orc_e8m0_value(sf[r * (C / 32) + c / 64]);", 1, ["formats"]),
    ("index score overflow not rejected",
     "        if (acc > INT32_MAX || acc < INT32_MIN) {\n            out_of_range = 1;\n            continue;\n        }\n",
     "", 1, ["selection"]),
    ("block max ignores the first token", "        float m = score[8 * j];",
     "        float m = score[8 * j + 1 < n_visible ? 8 * j + 1 : 8 * j];", 1, ["selection"]),
    ("selection padded with 0", "        out[i] = -1;", "        out[i] = 0;", 1, ["selection"]),
    ("fp4 element by reciprocal multiply", "float v = xv / s; /* fp32 IEEE division */",
     "float v = xv * (1.0f / s);", 1, ["formats"]),
]

# Mutants that change the arithmetic but not a single output over the oracle's
# input domain (bf16 values), so no pin can catch them. Each is built and
# checked to give the unmutated oracle's bytes on every input of the step it
# changes; if that ever stopped holding, it would belong in C_MUTANTS.
#   fp4 scale by reciprocal multiply: fp32(amax * fp32(1/6)) differs from
#   fp32(amax / 6) for some bf16 amax (about 10,600 of 32,640), but never by
#   enough to change the E4M3 code it rounds to: an E4M3 midpoint m has at most
#   5 significant bits, so amax / 6 lands on it only when amax = 6 m exactly,
#   where both forms give m.
EQUIVALENT_C_MUTANTS = [
    ("fp4 scale by reciprocal multiply", "float s_f = amax / 6.0f; /* fp32 IEEE division */",
     "float s_f = amax * (1.0f / 6.0f);", 1),
]

# (name, text in oracle/__init__.py, replacement, pin files)
PY_MUTANTS = [
    ("window starts one position early", "lo = max(0, q_pos - n_win + 1, swa_pos0)",
     "lo = max(0, q_pos - n_win, swa_pos0)", ["attention"]),
    ("pool keeps an invisible position", "return pos[pos < n_visible]",
     "return pos[np.minimum(pos, n_visible - 1) < n_visible]", ["selection"]),
    ("pool of half the blocks",
     "pool = topk(blk, np.arange(blk.size, dtype=np.int64), pool_blocks)",
     "pool = topk(blk, np.arange(blk.size, dtype=np.int64), pool_blocks // 2)", ["selection"]),
    ("decoder groups reordered", "[REINDEX, REUSE, REUSE, REUSE] * 4",
     "[REUSE, REINDEX, REUSE, REUSE] * 4", ["selection"]),
    ("Reindex rescoring with the first layer's query",
     "top, _, _ = reindex_layer(q_idx_of(l), k_idx, k_scale, pool, n_visible)",
     "top, _, _ = reindex_layer(q_idx_of(0), k_idx, k_scale, pool, n_visible)", ["selection"]),
    ("bf16 read one bit low", "u = np.ascontiguousarray(x_bf16, dtype=np.uint16).astype(np.uint32) << 16",
     "u = np.ascontiguousarray(x_bf16, dtype=np.uint16).astype(np.uint32) << 15", ["attention"]),
    ("window ends one position early", "hi = min(q_pos, swa_pos0 + swa_rows - 1)",
     "hi = min(q_pos - 1, swa_pos0 + swa_rows - 1)", ["attention"]),
    ("Full top-k one short", "top = topk(tok[ppos], ppos, k_top)", "top = topk(tok[ppos], ppos, k_top - 1)",
     ["selection"]),
    ("Reindex key scales doubled", "sc = index_scores(q_idx, k_idx[ppos], k_scale[ppos])",
     "sc = index_scores(q_idx, k_idx[ppos], k_scale[ppos] * 2)", ["selection"]),
    ("attention drops selected position 0", "sel = sel[sel >= 0]", "sel = sel[sel > 0]", ["attention"]),
    ("stack returns the pool reversed", "            pools[l] = pool", "            pools[l] = pool[::-1].copy()",
     ["selection"]),
]


def _replace_nth(text, old, new, n):
    count = text.count(old)
    assert count >= n, f"mutation site not found ({count} occurrences): {old!r}"
    start = -1
    for _ in range(n):
        start = text.index(old, start + 1)
    return text[:start] + new + text[start + len(old):]


def _compile(src_text, out_dir):
    os.makedirs(out_dir, exist_ok=True)
    c = os.path.join(out_dir, "csa2_oracle.c")
    so = os.path.join(out_dir, "libcsa2_oracle.so")
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", "-o", so,
                           c, "-lm"])
    return so


def _run_pins(files, lib, oracle_pkg_parent=None):
    """Exit status of the pin tests run against oracle library `lib` (and,
    with oracle_pkg_parent, against the oracle package found there)."""
    env = dict(os.environ, CSA2_ORACLE_LIB=lib)
    args = [PINS[f] for f in files] + ["-x", "-q", "-p", "no:cacheprovider", "-m", "not gpu"]
    pre = f"sys.path.insert(0, {oracle_pkg_parent!r}); import oracle; " if oracle_pkg_parent else ""
    code = (f"import sys; {pre}sys.path.insert(0, {ROOT!r}); import pytest; "
            f"sys.exit(pytest.main({args!r}))")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    return r.returncode


def _workers():
    return max(1, min(8, os.cpu_count() or 1))


def test_unmutated_copy_passes_the_pins(tmp_path):
    lib = _compile(open(C_SRC).read(), str(tmp_path / "clean"))
    assert _run_pins(list(PINS), lib) == 0


def test_every_c_mutant_fails_a_pin(tmp_path):
    src = open(C_SRC).read()

    def one(i):
        name, old, new, nth, files = C_MUTANTS[i]
        lib = _compile(_replace_nth(src, old, new, nth), str(tmp_path / f"m{i}"))
        return name, _run_pins(files, lib)

    with concurrent.futures.ThreadPoolExecutor(_workers()) as ex:
        results = list(ex.map(one, range(len(C_MUTANTS))))
    survivors = [name for name, rc in results if rc == 0]
    assert not survivors, f"mutants no pin catches: {survivors}"


def test_every_python_mutant_fails_a_pin(tmp_path):
    from oracle import build
    lib = build()
    src = open(PY_SRC).read()

    def one(i):
        name, old, new, files = PY_MUTANTS[i]
        pkg = tmp_path / f"p{i}" / "oracle"
        pkg.mkdir(parents=True)
        (pkg / "__init__.py").write_text(_replace_nth(src, old, new, 1))
        shutil.copy(C_SRC, pkg / "csa2_oracle.c")
        return name, _run_pins(files, lib, str(pkg.parent))

    with concurrent.futures.ThreadPoolExecutor(_workers()) as ex:
        results = list(ex.map(one, range(len(PY_MUTANTS))))
    survivors = [name for name, rc in results if rc == 0]
    assert not survivors, f"mutants no pin catches: {survivors}"


@pytest.mark.parametrize("name,old,new,nth", EQUIVALENT_C_MUTANTS, ids=[m[0] for m in EQUIVALENT_C_MUTANTS])
def test_equivalent_mutant_changes_no_output(tmp_path, name, old, new, nth):
    """The mutant's FP4 bytes and scales equal the oracle's for a group of
    every finite bf16 amax (both signs)."""
    src = open(C_SRC).read()
    lib = _compile(_replace_nth(src, old, new, nth), str(tmp_path / "eq"))
    code = (f"import sys; sys.path.insert(0, {ROOT!r}); sys.path.insert(0, {os.path.join(ROOT, 'tests')!r}); "
            "import numpy as np, oracle, test_oracle_formats as F; "
            "g = F.every_bf16_amax_groups(); p, s = oracle.fp4_quantize(g); "
            "np.save(sys.argv[1], np.concatenate([p, s], axis=1))")
    outs = []
    for i, l in enumerate([lib, oracle_lib()]):
        f = str(tmp_path / f"out{i}.npy")
        subprocess.check_call([sys.executable, "-c", code, f], cwd=ROOT, env=dict(os.environ, CSA2_ORACLE_LIB=l),
                              timeout=600)
        outs.append(__import__("numpy").load(f))
    assert (outs[0] == outs[1]).all(), name


def oracle_lib():
    from oracle import build
    return build()


@pytest.mark.parametrize("name,old,new,nth,files", C_MUTANTS, ids=[m[0] for m in C_MUTANTS])
def test_c_mutation_site_is_in_the_source(name, old, new, nth, files):
    assert open(C_SRC).read().count(old) >= nth, name


@pytest.mark.parametrize("name,old,new,files", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_python_mutation_site_is_in_the_source(name, old, new, files):
    assert open(PY_SRC).read().count(old) == 1, name
