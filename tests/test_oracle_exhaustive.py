"""Exhaustive pins of the oracle's scalar rules, each against a rule written independently in a
small C program built here with OpenMP and linked with the oracle's library.

Round-to-nearest-even onto the grids, over every FP32 bit pattern in [0, 8] (and every 17th
pattern in [-8, -0]).

The rule: a value at or above the grid's largest magnitude saturates to it; below, it is
rounded half-to-even on the grid step that holds there -- E2M1 steps 0.5 below 2, 1 in [2, 4),
2 in [4, 6); E1M2 step 0.5; INT4 step 1 -- and the result is looked up in the grid the pages
print ("当你的 GPU 学不会算账", sections "E2M1：一块刻度不均的尺子" and "UFP4：换一把尺子";
"低精度量化技术：IF4…", section 2.2: INT4 at most 7). On a tie, the half-to-even step count is
the even code (reading R5). The checker shares nothing with the oracle's nearest-point search.

The MX shared exponent (reading R10, the OCP MX rule floor(log2 amax) - 2 clamped to
[-127, 127]) over every positive finite float, from the float's exponent field; and FP32 to
bfloat16 round-to-nearest-even over every finite float, by the carry-add on the bit pattern.
"""
import os
import subprocess

import pytest

import oracle as O
from oracle import build as oracle_build

CHECKER = r'''
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
uint8_t orc_round_rtne(int grid, float v);
int orc_mx_exponent(float amax);
uint16_t orc_f32_to_bf16(float f);

static const double E2M1[8] = {0, 0.5, 1, 1.5, 2, 3, 4, 6};   /* the printed E2M1 grid */

static int e2m1_code(double m) {
  for (int c = 0; c < 8; ++c) if (E2M1[c] == m) return c;
  return -1;
}

/* kind 0: E2M1, 1: E1M2, 2: INT4 */
static double rule(int kind, double a) {
  if (kind == 1) return fmin(rint(2 * a) / 2, 3.5);
  if (kind == 2) return fmin(rint(a), 7.0);
  double step = a < 2 ? 0.5 : (a < 4 ? 1.0 : 2.0);
  return fmin(rint(a / step) * step, 6.0);
}

/* floor(log2 a) - 2 from the exponent field (subnormals: below 2^-126, so clamped), clamped */
static int mx_rule(uint32_t u) {
  const int E = (int)(u >> 23);
  const int e = E == 0 ? -200 : E - 127 - 2;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

/* round half to even on the 16 dropped bits: add 0x7FFF plus the kept LSB, keep the top half */
static uint16_t bf16_rule(uint32_t u) { return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16); }

static int scalar_rules(const char* which) {
  long long bad = 0, checked = 0;
  if (strcmp(which, "mx") == 0) {
    #pragma omp parallel for reduction(+:bad, checked) schedule(static, 1 << 20)
    for (long long p = 1; p < 0x7F800000LL; ++p) {
      float a;
      const uint32_t u = (uint32_t)p;
      memcpy(&a, &u, 4);
      if (orc_mx_exponent(a) != mx_rule(u)) ++bad;
      ++checked;
    }
  } else {
    #pragma omp parallel for reduction(+:bad, checked) schedule(static, 1 << 20)
    for (long long p = 0; p < 0x100000000LL; ++p) {
      const uint32_t u = (uint32_t)p;
      if ((u & 0x7F800000u) == 0x7F800000u) continue;                 /* inf / NaN */
      if ((u & 0x7FFFFFFFu) >= 0x7F7F8000u) continue;                 /* rounds past FLT_MAX */
      float f;
      memcpy(&f, &u, 4);
      if (orc_f32_to_bf16(f) != bf16_rule(u)) ++bad;
      ++checked;
    }
  }
  printf("%lld %lld\n", bad, checked);
  return 0;
}

int main(int argc, char** argv) {
  if (argc == 2) return scalar_rules(argv[1]);
  const int kind = atoi(argv[1]), grid = atoi(argv[2]);
  const uint32_t last = 0x41000000u;   /* 8.0f */
  long long bad = 0, checked = 0;
  #pragma omp parallel for reduction(+:bad, checked) schedule(static, 1 << 20)
  for (long long p = 0; p <= (long long)last; ++p) {
    float a;
    const uint32_t u = (uint32_t)p;
    memcpy(&a, &u, 4);
    const double m = rule(kind, (double)a);
    const int code = kind == 0 ? e2m1_code(m) : (kind == 1 ? (int)(2 * m) : (int)m);
    if (orc_round_rtne(grid, a) != (uint8_t)code) ++bad;
    ++checked;
    if (p % 17 == 0) {
      /* sign-magnitude grids keep the sign bit (also on zero); INT4 is two's complement */
      const uint8_t neg = kind == 2 ? (uint8_t)((-code) & 0xF) : (uint8_t)(8 | code);
      if (orc_round_rtne(grid, -a) != neg) ++bad;
      ++checked;
    }
  }
  printf("%lld %lld\n", bad, checked);
  return 0;
}
'''


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    d = tmp_path_factory.mktemp("rtne_checker")
    src, exe = d / "checker.c", d / "checker"
    src.write_text(CHECKER)
    libdir = os.path.dirname(oracle_build.build())
    subprocess.run(["gcc", "-O2", "-fopenmp", str(src), "-L", libdir, "-loracle",
                    "-Wl,-rpath," + libdir, "-lm", "-o", str(exe)], check=True)
    return str(exe)


@pytest.mark.slow
@pytest.mark.parametrize("kind,grid", [(0, O.GRID_E2M1), (1, O.GRID_E1M2), (2, O.GRID_INT4)],
                         ids=["E2M1", "E1M2", "INT4"])
def test_rtne_every_float_in_range(checker, kind, grid):
    out = subprocess.run([checker, str(kind), str(grid)], capture_output=True, text=True,
                         check=True, timeout=600).stdout.split()
    bad, checked = int(out[0]), int(out[1])
    assert checked > 0x41000000
    assert bad == 0


@pytest.mark.slow
@pytest.mark.parametrize("which,count", [
    ("mx", 0x7F800000 - 1),                       # every positive finite float
    ("bf16", 2 ** 32 - 2 ** 24 - 2 ** 16),        # every finite float not rounding past FLT_MAX
])
def test_scalar_rules_every_float(checker, which, count):
    out = subprocess.run([checker, which], capture_output=True, text=True, check=True,
                         timeout=600).stdout.split()
    bad, checked = int(out[0]), int(out[1])
    assert checked == count
    assert bad == 0
