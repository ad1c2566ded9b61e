"""The oracle's pins must catch plausible mistakes.

Each case copies the oracle's C source, plants one mistake (a dropped term, a
wrong sign, index or constant), builds the copy with gcc on the CPU and runs
the pin tests against it in a fresh process; the pins must fail.
"""
import concurrent.futures
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "sp_oracle.c")

MUTANTS = {
    "bias dropped": (
        "double v = y[j] + (bias ? ld(bias, j, c->dtype) : 0.0);",
        "double v = y[j];"),
    "dropout not rescaled": (
        "v = keep ? v * scale : 0.0;", "v = keep ? v : 0.0;"),
    "wrong philox output word": (
        "return u[j & 3] >= orc_drop_threshold(p);",
        "return u[(j + 1) & 3] >= orc_drop_threshold(p);"),
    "philox multipliers swapped": (
        "uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)x0;",
        "uint64_t p0 = (uint64_t)PHILOX_M1 * (uint64_t)x0;"),
    "philox second key word not bumped": (
        "k1 += PHILOX_W1;", "k1 += 0u;"),
    "rounding ties away from zero": (
        "double r = nearbyint(scaled);", "double r = round(scaled);"),
    "unbiased variance": (
        "var += (x[j] - mean) * (x[j] - mean);\n        var /= (double)h;",
        "var += (x[j] - mean) * (x[j] - mean);\n        var /= (double)(h - 1);"),
    "eps outside the square root": (
        "rstd = 1.0 / sqrt(var + (double)c->eps);",
        "rstd = 1.0 / (sqrt(var) + (double)c->eps);"),
    "beta dropped": (
        "o[j] = orc_round((x[j] - mean) * rstd * ld(gamma, j, c->dtype) + b,",
        "o[j] = orc_round((x[j] - mean) * rstd * ld(gamma, j, c->dtype) + 0*b,"),
    "rms gamma dropped": (
        "o[j] = orc_round(x[j] * rstd * ld(gamma, j, c->dtype), c->dtype);",
        "o[j] = orc_round(x[j] * rstd, c->dtype);"),
    "reduce-scatter ignores the rank": (
        "int64_t n = (int64_t)rank * per + i;", "int64_t n = i;"),
    "all-gather in reverse order": (
        "out[(int64_t)r * shard_rows * h + i] = shards[r][i];",
        "out[(int64_t)(t - 1 - r) * shard_rows * h + i] = shards[r][i];"),
    "layernorm backward drops mean(g)": (
        "? rstd * (g - mg - xhat[j] * mgx)", "? rstd * (g - xhat[j] * mgx)"),
    "layernorm backward sign": (
        "? rstd * (g - mg - xhat[j] * mgx)", "? rstd * (g - mg + xhat[j] * mgx)"),
    "rmsnorm backward drops the projection": (
        ": rstd * (g - xhat[j] * mgx);", ": rstd * g;"),
    "dbias sums before dropout": (
        "if (dbias) dbias[j] += dz[j];", "if (dbias) dbias[j] += dr;"),
    "dropout backward not rescaled": (
        "dz[j] = keep ? dr * scale : 0.0;", "dz[j] = keep ? dr : 0.0;"),
    "residual-stream gradient dropped": (
        "double dr = dx + (drnext ? ld(drnext, row * h + j, c->res_dtype) : 0.0);",
        "double dr = dx;"),
    "dgamma without xhat": (
        "dgamma[j] += dn[j] * xhat[j];", "dgamma[j] += dn[j];"),
    "A_TP attention term not divided by t": (
        "coeff = 10.0 + 24.0 / (double)t + attn / (double)t;",
        "coeff = 10.0 + 24.0 / (double)t + attn;"),
    "norm reads the unrounded residual sum": (
        "        x[j] = r;\n",
        "        x[j] = ld(resid, rrow * h + j, c->res_dtype) + v;\n"),
    "entry norm drops beta": (
        "o[j] = (xr[j] - mu) * rs * ld(gamma, j, c->dtype) + b;",
        "o[j] = (xr[j] - mu) * rs * ld(gamma, j, c->dtype) + 0 * b;"),
    "entry norm uses the unbiased variance": (
        "var += (xr[j] - mu) * (xr[j] - mu);\n                var /= (double)h;",
        "var += (xr[j] - mu) * (xr[j] - mu);\n                var /= (double)(h - 1);"),
    "residual sum stored in the I/O dtype": (
        "double r = orc_round(ld(resid, rrow * h + j, c->res_dtype) + v, c->res_dtype);",
        "double r = orc_round(ld(resid, rrow * h + j, c->res_dtype) + v, c->dtype);"),
    "residual gradient stored in the I/O dtype": (
        "st(dres_in, row * h + j, c->res_dtype, dr);",
        "st(dres_in, row * h + j, c->dtype, dr);"),
    "entry mean stored at the rank-local row": (
        "if (mean) mean[n] = mu;", "if (mean) mean[i] = mu;"),
    "entry rstd stored at the rank-local row": (
        "if (rstd) rstd[n] = rs;", "if (rstd) rstd[i] = rs;"),
    "row-chunk shares: dbeta reported as dgamma": (
        "if (dgamma) dgamma[j] = acc[j];", "if (dgamma) dgamma[j] = acc[h + j];"),
    "row-parallel linear drops the last rank": (
        "            for (int k = 0; k < t; ++k) {\n                double part = 0.0;",
        "            for (int k = 0; k < t - 1; ++k) {\n                double part = 0.0;"),
    "row-parallel linear reads the weight transposed": (
        "part += ld(x, n * f + i, ORC_BF16) * ld(w, j * f + i, ORC_BF16);",
        "part += ld(x, n * f + i, ORC_BF16) * ld(w, i * h + j, ORC_BF16);"),
    "column-parallel linear skips the all-gather order": (
        "orc_all_gather(t, shard_rows, h, (const double* const*)sh, X);",
        "for (int64_t q = 0; q < N * h; ++q) X[q] = sh[0][q % (shard_rows * h)];"),
    "ring attention skips the last ring step": (
        "            for (int i = 0; i < t; ++i) {\n                const int64_t blk = ((int64_t)r - i + t) % t;\n                /* the block's scores",
        "            for (int i = 0; i < t - 1; ++i) {\n                const int64_t blk = ((int64_t)r - i + t) % t;\n                /* the block's scores"),
    "ring attention does not rescale the values when the maximum grows": (
        "                l *= alpha;\n                for (int64_t c = 0; c < d; ++c) o[c] *= alpha;\n                for (int64_t jj = 0; jj < per; ++jj) {\n                    const int64_t j = blk * per + jj;\n                    const double p = exp(sc[jj] - mnew);\n                    l += p;\n                    for (int64_t c = 0; c < d; ++c) o[c] += p * ld(v, base",
        "                l *= alpha;\n                for (int64_t jj = 0; jj < per; ++jj) {\n                    const int64_t j = blk * per + jj;\n                    const double p = exp(sc[jj] - mnew);\n                    l += p;\n                    for (int64_t c = 0; c < d; ++c) o[c] += p * ld(v, base"),
    "ring attention ignores the scale": (
        "                    sc[jj] = scale * acc;\n                    if (sc[jj] > bmax) bmax = sc[jj];\n                }\n                /* fold",
        "                    sc[jj] = acc;\n                    if (sc[jj] > bmax) bmax = sc[jj];\n                }\n                /* fold"),
    "ring volume without (t-1)/t": (
        "double phase = (double)(t - 1) / (double)t * V;",
        "double phase = V;"),
}


def _run_mutant(name, workdir):
    find, repl = MUTANTS[name]
    src = open(SRC).read()
    if src.count(find) != 1:
        return name, None, f"mutation site not unique/found: {name}"
    d = os.path.join(workdir, name.replace(" ", "_"))
    os.makedirs(d, exist_ok=True)
    mut_c = os.path.join(d, "mutant.c")
    with open(mut_c, "w") as f:
        f.write(src.replace(find, repl))
    lib = os.path.join(d, "libmutant.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared",
                    "-ffp-contract=off", "-o", lib, mut_c, "-lm"], check=True)
    env = dict(os.environ, SP_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q",
                        "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True,
                       timeout=900)
    return name, r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def mutant_results():
    with tempfile.TemporaryDirectory() as tmp:
        with concurrent.futures.ThreadPoolExecutor(
                max_workers=max(2, os.cpu_count() or 2)) as ex:
            futs = [ex.submit(_run_mutant, n, tmp) for n in MUTANTS]
            return {n: (rc, out) for n, rc, out in
                    (f.result() for f in futs)}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, mutant_results):
    rc, out = mutant_results[name]
    assert rc is not None, out
    assert rc != 0, f"pins did not catch: {name}\n{out}"
