"""Planted mistakes in the oracle are caught by its pins.

Each case copies the oracle into a temporary tree, plants one plausible mistake in
oracle.c (a dropped term or scale, a wrong sign, a transposed operand, an index
error, a wrong offset, bit order, codebook entry or scale in a weight code), and runs the pins of
test_oracle.py against that copy in a subprocess: at least one pin must fail (pytest
exit status 1, a failed test, not a crash or a collection error).  An unchanged copy
run the same way must pass.  Every planted mistake keeps its indices inside the
arrays, so a mutant fails an assertion rather than memory.
"""
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {  # name: (text of oracle.c, replacement)
    "h_without_s": ("h[i * d_out + n] = base + s * lora;", "h[i * d_out + n] = base + lora;"),
    "h_without_lowrank": ("h[i * d_out + n] = base + s * lora;", "h[i * d_out + n] = base + 0.0 * lora;"),
    "dx_wrong_sign": ("dX[i * d_in + k] = base[k] + s * lora;", "dX[i * d_in + k] = base[k] - s * lora;"),
    "g_transposed_B": ("acc += bf16_to_f64(dY[m * d_out + n]) * bf16_to_f64(B[n * r + j]);",
                       "acc += bf16_to_f64(dY[m * d_out + n]) * bf16_to_f64(B[j * d_out + n]);"),
    "xa_index_error": ("acc += bf16_to_f64(x[m * d_in + k]) * bf16_to_f64(A[j * d_in + k]);",
                       "acc += bf16_to_f64(x[m * d_in + k]) * bf16_to_f64(A[j * d_in + (d_in - 1 - k)]);"),
    "db_without_s": ("dB[n * r + j] = s * acc[(n - n0) * r + j];", "dB[n * r + j] = acc[(n - n0) * r + j];"),
    "da_transposed": ("dA[j * d_in + k] = s * acc[(k - k0) * r + j];", "dA[k * r + j] = s * acc[(k - k0) * r + j];"),
    "q4_offset": ("(double)(code - 8)", "(double)(code - 7)"),
    "q4_nibble_order": ("(k % 2 == 0) ? (byte & 0x0F) : (byte >> 4)", "(k % 2 == 1) ? (byte & 0x0F) : (byte >> 4)"),
    "q4_scale_block": ("(double)(code - 8) * bf16_to_f64(sc[k / Q4_BLOCK])",
                       "(double)(code - 8) * bf16_to_f64(sc[k / Q4_BLOCK / 2])"),
    "fp8_exponent_bias": ("ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 8.0, e - 8)"),
    "fp8_subnormal_step": ("ldexp((double)m, -9)", "ldexp((double)m, -10)"),
    "fp8_row_scale": ("bf16_to_f64(W->scale[n])", "bf16_to_f64(W->scale[0])"),
    "codebook_reversed": ("row[k] = g_codebook[code] * bf16_to_f64(sc[k / Q4_BLOCK]);",
                          "row[k] = g_codebook[15 - code] * bf16_to_f64(sc[k / Q4_BLOCK]);"),
    "codebook_without_scale": ("row[k] = g_codebook[code] * bf16_to_f64(sc[k / Q4_BLOCK]);",
                               "row[k] = g_codebook[code];"),
}


def _tree(base, name, mutation):
    d = os.path.join(base, name)
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(d, "oracle"),
                    ignore=shutil.ignore_patterns("*.so", "*.tmp", "__pycache__"))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(d, "tests", "golden"))
    for f in ("test_oracle.py", "conftest.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(d, "tests", f))
    if mutation:
        old, new = mutation
        path = os.path.join(d, "oracle", "oracle.c")
        src = open(path).read()
        assert src.count(old) == 1, f"{name}: the text to change must occur exactly once"
        with open(path, "w") as fh:
            fh.write(src.replace(old, new))
    return d


def _run(d):
    # the copy's conftest puts its own root first on sys.path, so `import oracle` loads
    # the copy; the package under test comes from the repository
    env = dict(os.environ, PYTHONPATH=d + os.pathsep + ROOT, OMP_NUM_THREADS="2")
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                           os.path.join(d, "tests", "test_oracle.py")],
                          cwd=d, env=env, capture_output=True, text=True, timeout=900)


def test_planted_mistakes_fail_the_pins(tmp_path):
    cases = [("control", None)] + list(MUTANTS.items())
    trees = {name: _tree(str(tmp_path), name, m) for name, m in cases}
    with ThreadPoolExecutor(max_workers=4) as ex:
        results = dict(zip(trees, ex.map(_run, trees.values())))
    control = results.pop("control")
    assert control.returncode == 0, "the unchanged copy must pass:\n" + control.stdout[-3000:]
    missed = {n: r.returncode for n, r in results.items() if r.returncode != 1}
    assert not missed, f"mutants not caught by a failing pin (exit status): {missed}\n" + "\n".join(
        results[n].stdout[-800:] for n in missed)
