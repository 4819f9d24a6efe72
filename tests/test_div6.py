"""The NVFP4 attention kernel (each P' vector's scale code) and the NVFP4
quantiser (each Q/K/V vector's scale code) form amax / 6 with one multiply by
RN(1/6) and one fma correction with the exact residual (div6_rn in
quantize_nvfp4.cuh; Markstein's residual correction of a reciprocal product,
IBM J. Res. Dev. 34(1), 1990).  The scale codes must be those of
the IEEE-rounded quotient, so the identity is checked here for EVERY finite
non-negative fp32 x whose quotient is normal (smaller quotients are below half
the smallest E4M3 subnormal and give code 0 either way), with the C library's
exact fmaf standing in for the GPU's fused multiply-add."""
import subprocess

SRC = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
int main(void) {
  const float c = 1.0f / 6.0f;
  if (c != 0x1.555556p-3f) return 2;                  /* RN(1/6), as in the kernel */
  uint64_t bad = 0, n = 0;
  for (uint32_t u = 0; u < 0x7F800000u; ++u) {
    float x;
    memcpy(&x, &u, 4);
    const float ref = x / 6.0f;
    if (ref < 0x1p-126f) continue;
    const float q0 = x * c;
    const float q1 = fmaf(fmaf(-q0, 6.0f, x), c, q0);
    if (memcmp(&ref, &q1, 4) != 0) ++bad;
    ++n;
  }
  printf("%llu %llu\n", (unsigned long long)n, (unsigned long long)bad);
  return bad != 0;
}
"""


def test_div6_correctly_rounded_for_all_normal_quotients(tmp_path):
    src = tmp_path / "div6.c"
    src.write_text(SRC)
    exe = tmp_path / "div6"
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", str(src), "-o", str(exe),
                    "-lm"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    n, bad = map(int, r.stdout.split())
    assert r.returncode == 0 and bad == 0
    assert n > 2_000_000_000          # every normal quotient was checked
