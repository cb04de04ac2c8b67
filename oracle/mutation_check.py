"""Plant one plausible mistake at a time in a copy of the oracle and check
that the CPU pins catch it (test infrastructure only).

Each mutation replaces one exact fragment of rq_oracle.c in a temporary copy
of `oracle/` and `tests/`, rebuilds that copy's liboracle.so and runs
tests/test_oracle_pins.py there.  A mutation that leaves every pin green is
reported as SURVIVED and the script exits 1.  The repository's own files are
never touched.

    python oracle/mutation_check.py            # all mutations
    python oracle/mutation_check.py -k cr      # names containing "cr"
"""
import argparse
import os
import shutil
import subprocess
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

# (name, fragment of rq_oracle.c, replacement)
MUTATIONS = [
    ("fwht sign swap",
     "                v[j + h] = a - b;\n            }\n    float cd",
     "                v[j + h] = b - a;\n            }\n    float cd"),
    ("no sign flip", "        v[i] = D[i] < 0 ? -r[i] : r[i];", "        v[i] = r[i];"),
    ("cd dropped", "        y[i] = v[i] * cd;", "        y[i] = v[i];"),
    ("outer 2^(b-1)", "const float outer = (float)half - 0.5f;",
     "const float outer = (float)half;"),
    ("round instead of floor", "float fl = floorf(u);", "float fl = rintf(u);"),
    ("scale mean", "double s = num / den;", "double s = num / (double)g;"),
    ("level offset",
     "int lvl = 2 * c - (nlev - 1);\n        num += (double)y[i]",
     "int lvl = 2 * c - nlev;\n        num += (double)y[i]"),
    ("pack shift",
     "words[j / per] |= (uint32_t)codes[j] << (bits * (j % per));",
     "words[j / per] |= (uint32_t)codes[j] << (bits * (per - 1 - j % per));"),
    ("residual reversed",
     "r[i] = orq_bf16_to_f32(x[i]) - orq_bf16_to_f32(ref[i]);",
     "r[i] = orq_bf16_to_f32(ref[i]) - orq_bf16_to_f32(x[i]);"),
    ("recon no transpose",
     "acc += R[(size_t)i * d + j] * yhat[i];     /* (R^T yhat)_j */",
     "acc += R[(size_t)j * d + i] * yhat[i];"),
    ("softmax no max", "z[t] = exp(z[t] - m);", "z[t] = exp(z[t]);"),
    ("splitmix shift", "z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;",
     "z = (z ^ (z >> 28)) * 0x94D049BB133111EBull;"),
    ("sign top bit", "D[i] = (orq_splitmix64(seed, (uint64_t)i) >> 63) ? -1 : 1;",
     "D[i] = (orq_splitmix64(seed, (uint64_t)i) & 1) ? -1 : 1;"),
    ("zero inv rule", "const float inv = (amax < FLT_MIN) ? 0.0f : outer / amax;",
     "const float inv = outer / amax;"),
    # compressed reference: residual base, reference levels, reconstruction
    ("cr residual against rotated bf16 reference",
     "z[k * g + i] = s * (float)(2 * c[k * g + i] - rtop);",
     "z[k * g + i] = y[k * g + i];"),
    ("cr reference level offset",
     "z[k * g + i] = s * (float)(2 * c[k * g + i] - rtop);",
     "z[k * g + i] = s * (float)(2 * c[k * g + i] - rtop - 1);"),
    ("cr residual not subtracted", "            y[i] = y[i] - z[i];", "            y[i] = y[i];"),
    ("cr reconstruction drops the loop",
     "            w[i] += orq_f16_to_f64(scales[k]) * (2 * c[i] - top);",
     "            w[i] += 0.0;"),
    ("cr reconstruction no transpose",
     "            acc += R[(size_t)i * d + j] * w[i];",
     "            acc += R[(size_t)j * d + i] * w[i];"),
]


def run_one(name, old, new, tmp, timeout):
    src_path = os.path.join(tmp, "oracle", "rq_oracle.c")
    orig = open(os.path.join(HERE, "rq_oracle.c")).read()
    if orig.count(old) < 1:
        return "FRAGMENT NOT FOUND"
    with open(src_path, "w") as f:
        f.write(orig.replace(old, new, 1))
    subprocess.run([sys.executable, os.path.join(tmp, "oracle", "build.py"), "--force"],
                   check=True, stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-q", "-x",
                        "-p", "no:cacheprovider"], cwd=tmp, capture_output=True, text=True,
                       timeout=timeout)
    tail = (r.stdout.strip().splitlines() or ["?"])[-1]
    return ("caught: " if r.returncode != 0 else "SURVIVED: ") + tail


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("-k", default="", help="run the mutations whose name contains this")
    ap.add_argument("--timeout", type=int, default=900)
    args = ap.parse_args()
    survived = 0
    with tempfile.TemporaryDirectory(prefix="oracle_mut_") as tmp:
        shutil.copytree(HERE, os.path.join(tmp, "oracle"),
                        ignore=shutil.ignore_patterns("*.so", "__pycache__"))
        shutil.copytree(os.path.join(ROOT, "tests"), os.path.join(tmp, "tests"),
                        ignore=shutil.ignore_patterns("__pycache__"))
        shutil.copy(os.path.join(ROOT, "pytest.ini"), tmp)
        for name, old, new in MUTATIONS:
            if args.k not in name:
                continue
            verdict = run_one(name, old, new, tmp, args.timeout)
            survived += not verdict.startswith("caught")
            print(f"{name:48s} {verdict}", flush=True)
    sys.exit(1 if survived else 0)


if __name__ == "__main__":
    main()
