"""Plant plausible mistakes in copies of the oracle (on the CPU) and require that at
least one pin catches each of them.  Every mutation keeps all memory accesses in
bounds, so a mutant can only compute wrong values, never crash."""
import os
import shutil
import subprocess
import tempfile

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "vq_oracle.c")

MUTANTS = {
    "msb_first_bits": ("uint32_t bit = (row[p / 8] >> (p % 8)) & 1u;",
                       "uint32_t bit = (row[p / 8] >> (7 - p % 8)) & 1u;"),
    "dropped_scale": ("w[c] = s * v;", "w[c] = v; (void)s;"),
    "codebook_transposed": ("float v = orc_half_to_float(cb[(int64_t)code * W->d + c % W->d]);",
                            "float v = orc_half_to_float(cb[(int64_t)(c % W->d) * (1 << W->bits) + code]);"),
    "subvector_index": ("uint32_t code = orc_code_at(row, c / W->d, W->bits);",
                        "uint32_t code = orc_code_at(row, c % W->d, W->bits);"),
    "scale_group_128": ("float s = orc_half_to_float(srow[c / 64]);",
                        "float s = orc_half_to_float(srow[c / 128]);"),
    "silu_sign": ("h[i] = g / (1.0 + exp(-g)) * u;", "h[i] = g / (1.0 + exp(g)) * u;"),
    "dropped_route_weight": ("for (int64_t c = 0; c < hidden; c++) yt[c] += wt * o[c];",
                             "for (int64_t c = 0; c < hidden; c++) yt[c] += o[c]; (void)wt;"),
    "x_transposed": ("acc += (double)w[c] * orc_x_at(x, xt, m * x_row_stride + c);\n                y[m",
                     "acc += (double)w[c] * orc_x_at(x, xt, c * M + m);\n                y[m"),
    "half_subnormal": ("v = ldexp((double)frac, -24);", "v = ldexp((double)frac, -25);"),
    "bf16_bias": ("v = ldexp((double)(128 + frac), expo - 134);",
                  "v = ldexp((double)(128 + frac), expo - 133);"),
    "row_bytes_floor": ("return ((ncodes + 31) / 32) * 4 * (int64_t)bits;",
                        "return (ncodes / 32 + 1) * 4 * (int64_t)bits;"),
    "fp32_accumulate": ("double acc = 0.0;\n                for (int64_t c = 0; c < W->cols; c++)\n"
                        "                    acc += (double)w[c] * orc_x_at(x, xt, m * x_row_stride + c);",
                        "float acc = 0.0f;\n                for (int64_t c = 0; c < W->cols; c++)\n"
                        "                    acc += w[c] * (float)orc_x_at(x, xt, m * x_row_stride + c);"),
    "uncounted_bad_id": ("{ bad++; continue; }", "{ continue; }"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique/found"
    tmp = tempfile.mkdtemp(prefix="orc_mut_")
    try:
        c = os.path.join(tmp, "m.c")
        so = os.path.join(tmp, "libm.so")
        with open(c, "w") as f:
            f.write(src.replace(old, new))
        subprocess.run(["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC",
                        "-shared", "-o", so, c, "-lm"], check=True)
        L = oracle.load(so)
        caught = []
        for pin in ALL_PINS:
            try:
                pin(L)
            except AssertionError:
                caught.append(pin.__name__)
        assert caught, f"no pin catches mutant {name}"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
