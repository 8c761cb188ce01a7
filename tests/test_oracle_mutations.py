"""Mutation check of the oracle's pins: each entry below plants one plausible mistake in
oracle/hifa4_oracle.c (a wrong rounding tie, a dropped term, a flipped sign, a wrong
index, a transposed operand), in a copy of the sources, and the oracle's CPU pins
(tests/test_oracle_*.py) must fail on it.  The unmutated copy must pass.  By default a
representative subset runs (about a minute); HIFA4_ALL_MUTATIONS=1 runs every entry."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join("oracle", "hifa4_oracle.c")

MUTATIONS = [
    ("e2m1 ties to odd", "(c & 1) == 0 && (best & 1) == 1", "(c & 1) == 1 && (best & 1) == 0"),
    ("e2m1 saturation drops the sign", "if (a >= 6.0f) return sign | 7;", "if (a >= 6.0f) return 7;"),
    ("e2m1 twice table 3 -> 2.5", "{0, 1, 2, 3, 4, 6, 8, 12}", "{0, 1, 2, 3, 4, 5, 8, 12}"),
    ("e4m3 subnormal exponent", "ldexpf((float)m, -9)", "ldexpf((float)m, -10)"),
    ("e4m3 units exponent", "((int64_t)(8 + m) << (e - 1))", "((int64_t)(8 + m) << e)"),
    ("e4m3 ties to odd", "return (uint8_t)((lo & 1) ? hi : lo);", "return (uint8_t)((lo & 1) ? lo : hi);"),
    ("e4m3 saturates to NaN", "if (x >= 448.0f) return 0x7E;", "if (x >= 448.0f) return 0x7F;"),
    ("exp2 clamp -126", "float xc = fmaxf(x, -127.0f);", "float xc = fmaxf(x, -126.0f);"),
    ("exp2 coefficient c1", "#define EXP2_C1 0x1.63e65ap-1f", "#define EXP2_C1 0x1.65e65ap-1f"),
    ("exp2 drops the cubic term", "float p = fmaf(fmaf(fmaf(EXP2_C3, f, EXP2_C2), f, EXP2_C1), f, 1.0f);",
     "float p = fmaf(fmaf(EXP2_C2, f, EXP2_C1), f, 1.0f);"),
    ("exp2 quadratic fit", "float p = fmaf(fmaf(fmaf(EXP2_C3, f, EXP2_C2), f, EXP2_C1), f, 1.0f);",
     "float p = fmaf(fmaf(0x1.51d9ccp-2f, f, 0x1.54f8d6p-1f), f, 1.0f);"),
    ("linear-mantissa P_hat", "float sigma = ldexpf(e4m3_value(sc), k2);\n",
     "float sigma = ldexpf(e4m3_value(sc), k2);\n"
     "                for (int e = 0; e < 16; ++e) {\n"
     "                    double pr = Pf[blk * 16 + e];\n"
     "                    if (!(pr > 0.0) || !(sigma > 0.0f)) { code[e] = 0; continue; }\n"
     "                    double z = log2(pr / sigma) - 73.0 / 1024.0, fl = floor(z);\n"
     "                    code[e] = e2m1_encode((float)ldexp(1.0 + (z - fl), (int)fl));\n"
     "                }\n"),
    ("block scale 1/4", "uint8_t sc = e4m3_encode_pos(ldexpf(amax * (1.0f / 6.0f), -k));", "uint8_t sc = e4m3_encode_pos(ldexpf(amax * (1.0f / 4.0f), -k));"),
    ("block R halved", "float R = (sigma == 0.0f) ? 0.0f : 1.0f / sigma;", "float R = (sigma == 0.0f) ? 0.0f : 0.5f / sigma;"),
    ("row packing nibble order", "codes[r * (d / 2) + blk * 8 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));\n        }\n    }\n}\n\n/* Rotate-half", "codes[r * (d / 2) + blk * 8 + i] = (uint8_t)(c[2 * i + 1] | (c[2 * i] << 4));\n        }\n    }\n}\n\n/* Rotate-half"),
    ("row quantiser group index", "int g = h / grp;\n        const uint16_t* xr", "int g = h % Hkv;\n        const uint16_t* xr"),
    ("smoothing divides", "v[i] = scale ? xv * scale[g * d + blk * 16 + i] : xv;\n            }\n            quant16(v, c, &scales[r * (d / 16) + blk]);\n            for (int i = 0; i < 8; ++i)\n                codes[r * (d / 2) + blk * 8 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));\n        }\n    }\n}\n\n/* Rotate", "v[i] = scale ? xv / scale[g * d + blk * 16 + i] : xv;\n            }\n            quant16(v, c, &scales[r * (d / 16) + blk]);\n            for (int i = 0; i < 8; ++i)\n                codes[r * (d / 2) + blk * 8 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));\n        }\n    }\n}\n\n/* Rotate"),
    ("V blocks along channels", "x[i] = bf16_to_f32(vh[(size_t)(blk * 16 + i) * d + c]);", "x[i] = bf16_to_f32(vh[(size_t)c * N + blk * 16 + i]);"),
    ("rope minus sign", "o[i] = a - b;", "o[i] = a + b;"),
    ("rope cos and sin swapped", "float a = x1 * c, b = x2 * sn;", "float a = x1 * sn, b = x2 * c;"),
    ("S accumulation RN instead of RZ", "else if (model == 3) acc = units_to_f32_rz(f32_to_units(acc) + t);", "else if (model == 3) acc = units_to_f32(f32_to_units(acc) + t);"),
    ("S uses the Q scale twice", "return isum * e4m3_units(as) * e4m3_units(bs);", "return isum * e4m3_units(as) * e4m3_units(as);"),
    ("causal mask includes the diagonal", "valid[kk] = a->dec_nq ? (key <= pos) : !(a->causal && key > i);", "valid[kk] = a->dec_nq ? (key <= pos) : !(a->causal && key >= i);"),
    ("m not rounded to fp16", "mnew16 = fmaxf(m16, f16_round(mu));", "mnew16 = fmaxf(m16, mu);"),
    ("alpha sign", "float alpha = (m16 == -INFINITY) ? 0.0f : own_exp2(m16 - mnew16);", "float alpha = (m16 == -INFINITY) ? 0.0f : own_exp2(mnew16 - m16);"),
    ("l not rescaled", "l16 = f16_round(fmaf(alpha, l16, (float)r));", "l16 = f16_round(fmaf(1.0f, l16, (float)r));"),
    ("normaliser from P (not P_hat)", "r += a->l_from_p ? P[kk] : Ph[kk];", "r += a->l_from_p ? Ph[kk] : P[kk];"),
    ("epilogue off by one", "float o = O32[x] / l16;", "float o = O32[x] / (l16 + 1.0f);"),
    ("P ignores m", "Pf[kk] = own_exp2(fmaf(Sf[kk], c, -mref));", "Pf[kk] = own_exp2(fmaf(Sf[kk], c, 0.0f));"),
    ("two-level R without 2^-k", "float sigma = ldexpf(e4m3_value(sc), k);", "float sigma = e4m3_value(sc);"),
    ("GQA kv head index", "const int g = h / (a->Hq / a->Hkv);", "const int g = h % a->Hkv;"),
    ("V scale of the next block", "e4m3_value(a->vs[vr * (Nk / 16) + key / 16]);", "e4m3_value(a->vs[vr * (Nk / 16) + (key / 16 + 1) % (Nk / 16)]);"),
    ("O accumulation drops half of PV", "O32[x] = (float)((double)O32[x] + pv[x]);", "O32[x] = (float)((double)O32[x] + 0.5 * pv[x]);"),
    ("O not rescaled", "if (m16 != -INFINITY && alpha != 1.0f) O32[x] = alpha * O32[x];", "if (m16 != -INFINITY && alpha != 1.0f) O32[x] = O32[x];"),
    ("merge weight sign", "float w = (mp[sp] == -INFINITY) ? 0.0f : own_exp2(mp[sp] - m);", "float w = (mp[sp] == -INFINITY) ? 0.0f : own_exp2(m - mp[sp]);"),
    ("merge l unweighted", "L = fmaf(w, lp[sp], L);", "L = lp[sp] + L;"),
    ("decode position", "(long long)Nk - a->dec_nq + (i % a->dec_nq)", "(long long)Nk - a->dec_nq + (i / a->dec_nq)"),
    ("decode output row map", "(bkv % Hkv) * G + hi) * nq + t;", "(bkv % Hkv) + hi * Hkv) * nq + t;"),
    ("calibration ratio inverted", "sv = (float)pow((double)ak / (double)aq, alpha);", "sv = (float)pow((double)aq / (double)ak, alpha);"),
    ("calibration query-head index", "qcal + (((size_t)b * Hq + (size_t)g * grp + hh) * N) * d;", "qcal + (((size_t)b * Hq + (size_t)g + hh * Hkv) * N) * d;"),
    ("two-level offset 9", "k2 = (ex - 1) - 10;", "k2 = (ex - 1) - 9;"),
    ("bf16 rounding ties away", "u += 0x7FFFu + ((u >> 16) & 1u);", "u += 0x8000u;"),
    ("bruteforce scale 1/d", "s[key] = acc / sqrt((double)d);", "s[key] = acc / (double)d;"),
    ("exact loop uses e^x", "P[kk] = valid[kk] ? exp2(S[kk] * cd - mnew64) : 0.0;", "P[kk] = valid[kk] ? exp(S[kk] * cd - mnew64) : 0.0;"),
    ("rotated rows: smoothing divides", "v[i] = scale ? xv * scale[g * d + blk * 16 + i] : xv;\n            }\n            quant16(v, c, &scales[r * (d / 16) + blk]);\n            for (int i = 0; i < 8; ++i)\n                codes[r * (d / 2) + blk * 8 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));\n        }\n    }\n}\n\n/* V^T", "v[i] = scale ? xv / scale[g * d + blk * 16 + i] : xv;\n            }\n            quant16(v, c, &scales[r * (d / 16) + blk]);\n            for (int i = 0; i < 8; ++i)\n                codes[r * (d / 2) + blk * 8 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));\n        }\n    }\n}\n\n/* V^T"),
    ("rotated rows: group index", "int g = h / grp;\n        const float* xr", "int g = h % Hkv;\n        const float* xr"),
    ("two-level clamp -30", "if (p_t == 0.0f || k2 < -40) k2 = -40;", "if (p_t == 0.0f || k2 < -30) k2 = -30;"),
    ("two-level without the clamp", "if (p_t == 0.0f || k2 < -40) k2 = -40;", "if (p_t == 0.0f) k2 = -40;"),
    ("two-level scale without 2^k", "float sigma = ldexpf(e4m3_value(sc), k2);", "float sigma = e4m3_value(sc);"),
    ("causal loop skips the diagonal tile", "int ntiles = a->causal ? i / bc + 1 : N / bc;", "int ntiles = a->causal ? (i + 1) / bc : N / bc;"),
    ("exact loop alpha sign", "double alpha = (mo == -INFINITY) ? 0.0 : exp2(mo - mn);", "double alpha = (mo == -INFINITY) ? 0.0 : exp2(mn - mo);"),
    ("trace records P_hat as P", "out->tr_p[(j - jstart) * bc + kk] = (float)P[kk];", "out->tr_p[(j - jstart) * bc + kk] = (float)Ph[kk];"),
    ("E2M1 magnitude 3 -> 2.5", "{0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f}", "{0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 2.5f, 4.0f, 6.0f}"),
    ("merge O unweighted", "O[x] = fmaf(w, op[sp][x], O[x]);", "O[x] = op[sp][x] + O[x];"),
    ("decode output off by one", "float inv = (L > 0.0f) ? 1.0f / L : 0.0f;", "float inv = (L > 0.0f) ? 1.0f / (L + 1.0f) : 0.0f;"),
]

# one per area: formats, exp2, P_hat rule, block quantiser, packing, GEMM accumulation,
# running max, normaliser, merge, calibration, output rounding
DEFAULT = {"e4m3 ties to odd", "exp2 quadratic fit", "linear-mantissa P_hat", "block R halved",
           "row packing nibble order", "S accumulation RN instead of RZ", "m not rounded to fp16",
           "normaliser from P (not P_hat)", "merge weight sign", "calibration ratio inverted",
           "bf16 rounding ties away"}
SELECTED = [m for m in MUTATIONS if os.environ.get("HIFA4_ALL_MUTATIONS") or m[0] in DEFAULT]


def _copy(dst):
    for sub in ("oracle", "tests", "bit_flashattention_b200"):
        shutil.copytree(os.path.join(ROOT, sub), os.path.join(dst, sub),
                        ignore=shutil.ignore_patterns("*.so", "__pycache__", "csrc", "test_gpu_*", "test_zz_*"))


def _pins_pass(dst):
    tests = sorted(os.path.join("tests", f) for f in os.listdir(os.path.join(dst, "tests"))
                   if f.startswith("test_oracle_") and f != "test_oracle_mutations.py")
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *tests],
                       cwd=dst, capture_output=True, text=True, timeout=900, env=env)
    return r.returncode == 0, r.stdout[-2000:]


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    """{name: (pattern found once, pins pass, output tail)} for the unmutated copy
    ("unmutated") and every selected mutation, run a few at a time."""
    from concurrent.futures import ThreadPoolExecutor

    def work(job):
        name, old, new = job
        dst = str(tmp_path_factory.mktemp("mutant"))
        _copy(dst)
        found = True
        if old is not None:
            p = os.path.join(dst, SRC)
            s = open(p).read()
            found = s.count(old) == 1
            if not found:
                return name, (False, True, "")
            open(p, "w").write(s.replace(old, new))
        ok, out = _pins_pass(dst)
        shutil.rmtree(dst, ignore_errors=True)
        return name, (found, ok, out)

    jobs = [("unmutated", None, None)] + SELECTED
    tmp_path_factory.getbasetemp()            # create the base directory before the threads do
    with ThreadPoolExecutor(max_workers=max(1, min(4, (os.cpu_count() or 2) // 2))) as ex:
        return dict(ex.map(work, jobs))


def test_unmutated_copy_passes(outcomes):
    found, ok, out = outcomes["unmutated"]
    assert ok, out


@pytest.mark.parametrize("name", [m[0] for m in SELECTED])
def test_mutation_is_caught(outcomes, name):
    found, ok, _ = outcomes[name]
    assert found, f"the pattern of {name!r} no longer matches the oracle"
    assert not ok, f"no pin fails when the oracle has: {name}"
