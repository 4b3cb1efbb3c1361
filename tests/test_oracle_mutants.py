"""The oracle's pins catch plausible mistakes: each mutant below is oracle.c
with one deliberate error (a flipped tie rule, a dropped term, a wrong
rounding, a swapped operand, a reversed order), compiled on the CPU into a
temporary library; the pin tests of the stage it breaks must fail against it,
while the same tests pass against an unmutated copy built the same way."""
import concurrent.futures as cf
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")
T_FMT = "tests/test_oracle_formats.py"
T_STG = "tests/test_oracle_stages.py"
T_DSP = "tests/test_oracle_dispatch.py"
T_PRJ = "tests/test_oracle_router_projection.py"
T_FAR = "tests/test_oracle_finalize_ar.py"

MUTANTS = [
    ("route: equal scores go to the higher id", T_STG, "route",
     [("return (a->e > b->e) - (a->e < b->e);", "return (a->e < b->e) - (a->e > b->e);")]),
    ("route: weights renormalised over k - 1 picks", T_STG, "route",
     [("for (int j = 0; j < k; ++j) S = S + s[cand[j].e];", "for (int j = 1; j < k; ++j) S = S + s[cand[j].e];")]),
    ("route: the selection bias left in the weights", T_STG, "route",
     [("w_row[j] = s[cand[j].e] / S;", "w_row[j] = cand[j].c / S;")]),
    ("sigmoid of +x", T_FMT, "sigmoid or exp",
     [("float e = oc_exp(-x);", "float e = oc_exp(x);")]),
    ("exp: a Taylor term dropped", T_FMT, "exp",
     [("p = fmaf(p, r, (float)(1.0 / 720.0));", "p = fmaf(p, r, 0.0f);")]),
    ("E2M1: the tie at 0.75 rounds down", T_FMT, "e2m1",
     [("c += (m >= 0.75f);", "c += (m > 0.75f);")]),
    ("E4M3: ties to the odd code", T_FMT, "e4m3",
     [("(d == best_d && (c & 1) == 0)", "(d == best_d && (c & 1) == 1)")]),
    ("BF16: ties away from zero", T_FMT, "bf16",
     [("u += 0x7fffu + keep_lsb;", "u += 0x8000u;")]),
    ("sum of squares: an odd block folded into its neighbour", T_FMT, "sumsq",
     [("if (nb & 1) lev[m++] = lev[nb - 1];", "if (nb & 1) lev[m - 1] = lev[m - 1] + lev[nb - 1];")]),
    ("inverse RMS without eps", T_FMT, "inv_rms",
     [("float d = mean + eps;", "float d = mean;")]),
    ("norm: the gain centre dropped", T_STG, "norm or gain",
     [("float g = gc + oc_bf16_to_f32(w[h]);", "float g = oc_bf16_to_f32(w[h]);")]),
    ("norm: a BF16 rounding before the inverse RMS", T_STG, "norm",
     [("y[h] = oc_bf16_rn(t * inv);", "y[h] = oc_bf16_rn(oc_bf16_to_f32(oc_bf16_rn(t)) * inv);")]),
    ("quant: block scale from amax / 4", T_STG, "norm_quant",
     [("const float r6 = (float)(1.0 / 6.0);", "const float r6 = (float)(1.0 / 4.0);")]),
    ("quant: nibbles swapped", T_STG, "norm_quant",
     [("packed8[i] = (uint8_t)((codes[2 * i] & 0x0f) | (codes[2 * i + 1] << 4));",
       "packed8[i] = (uint8_t)((codes[2 * i + 1] & 0x0f) | (codes[2 * i] << 4));")]),
    ("combine: slots past the end read", T_STG, "combine",
     [("            if (r < 0 || r >= R) continue;\n            const uint16_t* row = expert_out",
       "            if (r < 0) continue;\n            const uint16_t* row = expert_out")]),
    ("combine: the first slot unweighted", T_STG, "combine",
     [("acc[h] = fmaf(wj, oc_bf16_to_f32(y[h]), acc[h]);\n        }\n        for (int h = 0; h < H; ++h) out",
       "acc[h] = fmaf(j == 0 ? 1.0f : wj, oc_bf16_to_f32(y[h]), acc[h]);\n        }\n        for (int h = 0; h < H; ++h) out")]),
    ("join: alpha and beta swapped", T_STG, "join",
     [("float a = alpha * r[h];\n            float b = beta * n;", "float a = beta * r[h];\n            float b = alpha * n;")]),
    ("dispatch: an expert's rows in reverse entry order", T_DSP, "",
     [("int64_t r = next[e]++;", "int64_t r = offsets[e + 1] - 1 - (next[e]++ - offsets[e]);")]),
    ("projection: the scale dropped", T_PRJ, "",
     [("out64[(size_t)t * E + e] = (double)scale * s;", "out64[(size_t)t * E + e] = s;")]),
    ("finalize: partials added in reverse rank order", T_FAR, "",
     [("        for (int r = 0; r < world; ++r) {\n            for (int h = 0; h < H; ++h) acc[h] = 0.0f;",
       "        for (int rr = 0; rr < world; ++rr) {\n            const int r = world - 1 - rr;\n"
       "            for (int h = 0; h < H; ++h) acc[h] = 0.0f;"),
      ("s[h] = (r == 0) ? acc[h] : s[h] + acc[h];", "s[h] = (rr == 0) ? acc[h] : s[h] + acc[h];")]),
]


def _build(src_text, path):
    c = path + ".c"
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", *oracle.CFLAGS, c, "-o", path, "-lm"], check=True, capture_output=True)


def _run_pins(lib, test_file, kexpr):
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider", "-m", "not gpu", test_file]
    if kexpr:
        cmd += ["-k", kexpr]
    env = dict(os.environ, MB_ORACLE_LIB=lib)
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_every_mutant_fails_its_stage_pins(tmp_path):
    text = open(SRC).read()
    jobs = []
    control = str(tmp_path / "control.so")
    _build(text, control)
    for i, (what, test_file, kexpr, edits) in enumerate(MUTANTS):
        mutated = text
        for old, new in edits:
            assert mutated.count(old) == 1, f"{what}: the text to mutate is not in oracle.c once"
            mutated = mutated.replace(old, new)
        lib = str(tmp_path / f"mutant{i}.so")
        _build(mutated, lib)
        jobs.append((what, lib, test_file, kexpr))
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 2)) as ex:
        # the unmutated copy passes the same selections
        ctrl = {(f, k): ex.submit(_run_pins, control, f, k) for _, _, f, k in jobs}
        runs = [(what, ex.submit(_run_pins, lib, f, k)) for what, lib, f, k in jobs]
        for (f, k), fut in ctrl.items():
            r = fut.result()
            assert r.returncode == 0, f"unmutated oracle fails {f} -k {k!r}:\n{r.stdout[-2000:]}"
        survived = [what for what, fut in runs if fut.result().returncode == 0]
    assert not survived, f"mutants that no pin caught: {survived}"
