"""The kernels' multiply-shift division (Granlund & Montgomery) against the hardware
divide, compiled on the host from the same header: every divisor up to 4096 against
dense small numerators and random numerators up to 2^31 - 1."""
import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "gqa_exact_attention_b200", "csrc")

PROG = r'''
#include <cstdio>
#include <cstdint>
#include <random>
#define __host__
#define __device__
#include "fast_divmod.h"
int main() {
    std::mt19937 rng(12345);
    long long bad = 0;
    for (uint32_t d = 1; d <= 4096; ++d) {
        gqa::FastDiv f = gqa::make_fastdiv(d);
        for (uint32_t n = 0; n < 20000; ++n) {
            uint32_t q, r; gqa::fastdivmod(n, f, q, r);
            if (q != n / d || r != n % d) ++bad;
        }
        for (int k = 0; k < 2000; ++k) {
            uint32_t n = rng() & 0x7FFFFFFFu;
            if (gqa::fastdiv(n, f) != n / d) ++bad;
        }
        uint32_t edge[3] = {0x7FFFFFFFu, 0x7FFFFFFFu - d, (0x7FFFFFFFu / d) * d};
        for (uint32_t n : edge) if (gqa::fastdiv(n, f) != n / d) ++bad;
    }
    std::printf("%lld\n", bad);
    return bad != 0;
}
'''


def test_fastdiv_exhaustive(tmp_path):
    src = tmp_path / "t.cpp"
    src.write_text(PROG)
    exe = tmp_path / "t"
    subprocess.run(["g++", "-O2", "-std=c++17", "-I", CSRC, str(src), "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip() == "0", r.stdout
