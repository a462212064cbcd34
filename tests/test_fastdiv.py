"""Multiply-shift division of the row kernels (host and device share one definition in
csrc/csa_internal.h): compiled here with the host compiler and checked exhaustively against
integer division on the divisors and numerators the kernels meet (head counts, sequence
lengths up to 2^20, row indices below 2^31), including every numerator that sits next to a
multiple of the divisor near the top of the range."""
import os
import pathlib
import subprocess
import tempfile

ROOT = pathlib.Path(__file__).resolve().parents[1]

DRIVER = r"""
#include <stdio.h>
#include <initializer_list>
#include <vector_types.h>
#include "csa_internal.h"
using namespace csa;
static int check(uint32_t d, uint32_t n) {
    const FastDiv f = make_fastdiv(d);
    if (fastdiv(n, f) != n / d) { printf("FAIL d=%u n=%u got=%u\n", d, n, fastdiv(n, f)); return 1; }
    return 0;
}
int main() {
    int bad = 0;
    const uint32_t top = 0x7fffffffu;
    for (uint32_t d = 1; d <= 4096 && !bad; ++d) {
        for (uint32_t n = 0; n < 20000; ++n) bad |= check(d, n);
        for (uint32_t q = top / d - 3; q <= top / d; ++q)        // around the last multiples
            for (int e = -1; e <= 1; ++e) {
                const long long n = (long long)q * d + e;
                if (n >= 0 && n <= (long long)top) bad |= check(d, (uint32_t)n);
            }
        uint64_t x = 0x9e3779b97f4a7c15ull * d;                   // pseudo-random numerators
        for (int i = 0; i < 2000; ++i) {
            x ^= x << 13; x ^= x >> 7; x ^= x << 17;
            bad |= check(d, (uint32_t)(x & top));
        }
    }
    for (uint32_t l = 12; l <= 20 && !bad; ++l)                   // long sequences
        for (uint32_t d : {(1u << l) - 1, 1u << l, (1u << l) + 1, 3u << (l - 2), 1000u * l + 7})
            for (uint32_t n : {0u, d - 1, d, 2 * d - 1, top - 1, top, top / d * d, top / d * d - 1})
                bad |= check(d, n);
    printf(bad ? "FAIL\n" : "ok\n");
    return bad;
}
"""


def test_fastdiv_matches_integer_division():
    with tempfile.TemporaryDirectory() as tmp:
        src = pathlib.Path(tmp) / "fastdiv_check.cc"
        exe = pathlib.Path(tmp) / "fastdiv_check"
        src.write_text(DRIVER)
        cuda_inc = pathlib.Path(os.environ.get("CUDA_HOME", "/usr/local/cuda")) / "include"
        subprocess.run(["g++", "-O2", "-std=c++17", "-I", str(cuda_inc), "-I", str(ROOT / "include"),
                        "-I", str(ROOT / "causal_self_attention_gqa_b200" / "csrc"), str(src), "-o", str(exe)],
                       check=True)
        out = subprocess.run([str(exe)], capture_output=True, text=True)
        assert out.returncode == 0 and out.stdout.strip().endswith("ok"), out.stdout[-500:]
