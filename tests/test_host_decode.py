"""White-box checks of the host FFN's number-format code against the oracle.

The host half of the miss split decodes weights with vector code (E4M3 through
exact fp16 images, E2M1 through a magnitude table) and rounds activations with
scalar code (E4M3, E2M1).  The FFN-level tests compare whole outputs within the
dtype bars, which a wrong decode of a rare code (an E4M3 subnormal, say) could
hide in.  Here a small harness, compiled with g++ around the library's source,
decodes every E4M3 code and every packed E2M1 byte and rounds a set of values
that includes every midpoint; each result must equal the oracle's exactly.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "expert_offloaded_edge_b200", "csrc")

HARNESS = r"""
#include "ftm_host_ffn.cpp"
#include <cstdio>
#include <cstdlib>

__attribute__((target("avx2,fma,f16c"))) static void decode_all() {
  alignas(32) uint8_t codes[256];
  for (int i = 0; i < 256; ++i) codes[i] = static_cast<uint8_t>(i);
  for (int c = 0; c < 256; c += 32) {
    __m256 v[4];
    ftm::e4m3x32(codes + c, v);
    float f[32];
    for (int k = 0; k < 4; ++k) _mm256_storeu_ps(f + 8 * k, v[k]);
    for (int j = 0; j < 32; ++j) std::printf("e4m3 %d %a\n", c + j, f[j]);
  }
  for (int c = 0; c < 256; c += 4) {   // 4 bytes = 8 codes, element 2j in the low nibble of byte j
    float f[8];
    _mm256_storeu_ps(f, ftm::e2m1x8(codes + c));
    for (int j = 0; j < 8; ++j) std::printf("e2m1 %d %d %a\n", c + j / 2, j % 2, f[j]);
  }
}

int main(int argc, char** argv) {
  if (!ftm::g_f16c) { std::printf("skip\n"); return 0; }
  decode_all();
  FILE* in = std::fopen(argv[1], "r");
  float v;
  while (std::fscanf(in, "%a", &v) == 1)
    std::printf("round %a %a %a\n", v, ftm::e4m3_round(v), ftm::e2m1_round(v));
  std::fclose(in);
  return 0;
}
"""


def _values():
    """Non-negative test values: every E4M3 and E2M1 value, every midpoint
    between neighbours, the points one ulp either side of each midpoint, values
    past the saturation points, and random values over the whole range."""
    e4 = sorted({oracle.e4m3_value(c) for c in range(0x7F)})
    e2 = sorted({oracle.e2m1_value(c) for c in range(8)})
    pts = set()
    for grid in (e4, e2):
        pts.update(grid)
        for a, b in zip(grid, grid[1:]):
            m = np.float32((a + b) / 2)
            pts.update([float(m), float(np.nextafter(m, np.float32(0))), float(np.nextafter(m, np.float32(1e9)))])
    pts.update([448.0, 460.0, 464.0, 1000.0, 6.0, 7.0, 1e30, 2.0 ** -10, 2.0 ** -11])
    rng = np.random.default_rng(5)
    pts.update(float(v) for v in np.float32(np.exp(rng.uniform(np.log(1e-4), np.log(600.0), 2000))))
    return sorted(float(np.float32(p)) for p in pts)


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp("host_decode")
    src = d / "harness.cpp"
    src.write_text(HARNESS)
    exe = d / "harness"
    subprocess.check_call([gxx, "-O2", "-std=c++17", "-I", os.path.join(ROOT, "include"), "-I", CSRC, str(src),
                           "-o", str(exe), "-pthread"])
    vals = d / "values.txt"
    vals.write_text("\n".join(float(v).hex() for v in _values()) + "\n")
    out = subprocess.check_output([str(exe), str(vals)], text=True)
    if out.strip() == "skip":
        pytest.skip("CPU without AVX2/FMA/F16C")
    return out.splitlines()


def test_e4m3_vector_decode_every_code(harness):
    got = {int(p[1]): float.fromhex(p[2]) for p in (ln.split() for ln in harness) if p[0] == "e4m3"}
    assert len(got) == 256
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            assert got[c] == (-480.0 if c & 0x80 else 480.0)   # NaN codes, absent from weights
        else:
            assert got[c] == oracle.e4m3_value(c), hex(c)


def test_e2m1_vector_decode_every_nibble(harness):
    got = [(int(p[1]), int(p[2]), float.fromhex(p[3])) for p in (ln.split() for ln in harness) if p[0] == "e2m1"]
    assert len(got) == 512
    for byte, hi, v in got:
        nib = (byte >> 4) if hi else (byte & 15)
        assert v == oracle.e2m1_value(nib), (byte, hi)


def test_scalar_rounding_matches_the_oracle_encoders(harness):
    rows = [p for p in (ln.split() for ln in harness) if p[0] == "round"]
    assert len(rows) > 2000
    for _, a, r4, r2 in rows:
        v = float.fromhex(a)
        assert float.fromhex(r4) == oracle.e4m3_value(oracle.e4m3_encode(v)), ("e4m3", v)
        assert float.fromhex(r2) == oracle.e2m1_value(oracle.e2m1_encode(v)), ("e2m1", v)
