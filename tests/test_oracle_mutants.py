"""Mutation check of the oracle pins: plant a plausible mistake in a copy of the
oracle's C source (on the CPU), rebuild that copy, and require the pin suite to
fail on it.  The real oracle is never modified.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (name, file, original text(s), mutated text(s))
MUTANTS = [
    ("high-band sign", "haar.c", "*hi = (a - b) * HAAR_S;", "*hi = (b - a) * HAAR_S;"),
    ("replica taken from frame 1", "haar.c", "const int64_t vt = (pt == 0) ? 0 : pt - 1;",
     "const int64_t vt = (pt == 0) ? 1 : pt - 1;"),
    ("subband bit order", "haar.c",
     "const int64_t s = 4 * bt + 2 * by + bx;\n                                o[",
     "const int64_t s = bt + 2 * by + 4 * bx;\n                                o["),
    ("dropped level-2 pass (2D)", "haar.c", "level2d_fwd(mid, y + b * ny, C1, H / 2, W / 2);",
     "level2d_fwd(mid, y + b * ny, C1, H / 2, W / 2); for (int64_t q = 0; q < ny; ++q) y[b * ny + q] *= 1.0;"
     " if (b == 0) y[0] += 1e-3;"),
    ("inverse swaps the pair", "haar.c", "*b = (lo - hi) * HAAR_S;", "*b = (hi - lo) * HAAR_S;"),
    ("transposed projection", "fsq.c", "z = fmaf(w[i * C + c], u[(b * C + c) * S + s], z);",
     "z = fmaf(w[(c * FSQ_DIM + i) % (FSQ_DIM * C)], u[(b * C + c) * S + s], z);"),
    ("projection kept in double", "fsq.c",
     ["float z = 0.0f;", "z = fmaf(w[i * C + c], u[(b * C + c) * S + s], z);"],
     ["double z = 0.0;", "z += (double)w[i * C + c] * (double)u[(b * C + c) * S + s];"]),
    ("basis most-significant first", "fsq.c", "for (int k = 0; k < i; ++k)", "for (int k = i + 1; k < FSQ_DIM; ++k)"),
    ("odd level offset", "fsq.c", "const double off = (L % 2 == 0) ? 0.5 : 0.0;", "const double off = 0.5;"),
    ("eps sign", "fsq.c", "(L - 1) * (1.0 + FSQ_EPS) / 2.0", "(L - 1) * (1.0 - FSQ_EPS) / 2.0"),
    ("adjoint drops the replica instead of adding it", "haar.c", "else if (pt == 1)\n                                    *dst += g[dt][dy][dx];",
     "else if (pt == 1)\n                                    *dst = g[dt][dy][dx];"),
    ("unpatcher adjoint feeds the replica", "haar.c", "pt == 0 ? 0.0 : v[", "pt == 0 ? 1.0 : v["),
    ("slope without the half width", "fsq.c", "return half / (c * c) / (double)(L / 2);", "return half / (c * c);"),
    ("decode backward transposes W", "fsq.c", "acc += (double)w[i * C + c] * gc;",
     "acc += (double)w[(c * FSQ_DIM + i) % (FSQ_DIM * C)] * gc;"),
    ("decode forgets the offset", "fsq.c", "zhat[i] = (double)(digits[i] - half_width) / (double)half_width;",
     "zhat[i] = (double)(digits[i]) / (double)half_width;"),
    ("temporal padding repeats the edge frame", "haar.c", "return r < T ? r : period - r;",
     "return r < T ? r : period - r + 1;"),
    ("continuation chunk pairs frames in reverse", "haar.c", "(c * T + 2 * j + dt) * H",
     "(c * T + 2 * j + 1 - dt) * H"),
]


@pytest.mark.parametrize("name,fname,orig,mutated", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, fname, orig, mutated):
    for f in ("haar.c", "fsq.c"):
        shutil.copy(os.path.join(ROOT, "oracle", f), tmp_path / f)
    src = (tmp_path / fname).read_text()
    origs, muts = (orig, mutated) if isinstance(orig, list) else ([orig], [mutated])
    for o, m in zip(origs, muts):
        # A mistake in a statement that appears in several functions is planted in all of them.
        assert src.count(o) >= 1, f"mutation anchor not found in {fname}: {o!r}"
        src = src.replace(o, m)
    (tmp_path / fname).write_text(src)
    so = tmp_path / "mutant.so"
    subprocess.run(["gcc", "-std=c11", "-O1", "-fPIC", "-shared", "-ffp-contract=off", "-o", str(so),
                    str(tmp_path / "haar.c"), str(tmp_path / "fsq.c"), "-lm"], check=True)
    env = dict(os.environ, ORACLE_SO=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        "tests/test_oracle_haar.py", "tests/test_oracle_fsq.py", "tests/test_oracle_backward.py",
                        "tests/test_oracle_padding.py"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch the planted mistake '{name}'"
