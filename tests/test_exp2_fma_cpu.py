"""The FMA-pipe 2^x used for part of the prefill softmax, checked on the CPU.

The scalar form in ``csrc/exp2_fma.cuh`` is plain float32 arithmetic (adds, fused
multiply-adds, one integer add), which a host compiler evaluates with the same IEEE
rounding as the GPU; it is built here with g++ and compared with 2^x in float64 over every
argument range the softmax produces: relative error within the polynomial's bound where the
result is normal, about 2^-125 (and never more) for arguments below -125 and for -inf.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "paged_kv_cache_465_b200", "csrc")

PROG = r"""
#include <cstdio>
#include <cstdlib>
#include <vector>
#include "exp2_fma.cuh"
int main(int argc, char** argv) {
  FILE* f = fopen(argv[1], "rb");
  std::vector<float> x;
  float v;
  while (fread(&v, 4, 1, f) == 1) x.push_back(v);
  fclose(f);
  FILE* g = fopen(argv[2], "wb");
  for (float a : x) { float y = pa::exp2_fma(a); fwrite(&y, 4, 1, g); }
  fclose(g);
  return 0;
}
"""


@pytest.fixture(scope="module")
def run(tmp_path_factory):
    cxx = shutil.which("g++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    d = tmp_path_factory.mktemp("exp2")
    src = d / "prog.cpp"
    src.write_text(PROG)
    exe = d / "prog"
    subprocess.run([cxx, "-O2", "-ffp-contract=off", "-std=c++17", "-I", CSRC, str(src), "-o",
                    str(exe)], check=True, capture_output=True)

    def call(x):
        x = np.ascontiguousarray(x, dtype=np.float32)
        (d / "in.bin").write_bytes(x.tobytes())
        subprocess.run([str(exe), str(d / "in.bin"), str(d / "out.bin")], check=True)
        return np.frombuffer((d / "out.bin").read_bytes(), dtype=np.float32)
    return call


def test_relative_error_within_the_polynomial_bound(run):
    rng = np.random.default_rng(5)
    x = np.concatenate([
        rng.uniform(-125, 127.49, 2_000_000),
        rng.uniform(-30, 8, 2_000_000),                 # the softmax's usual range (x <= 8)
        np.arange(-125, 128, dtype=np.float64),          # integers: f = 0
        np.arange(-125, 127) + 0.5,                      # ties of the rounding to j
        np.arange(-125, 127) + 0.5 - 2.0 ** -16,
        [0.0, -0.0, 1e-40, -1e-40, 2.0 ** -149, 8.0, 7.999999],
    ]).astype(np.float32)
    y = run(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert np.all(np.isfinite(y)) and np.all(y > 0)
    assert rel.max() < 7.6e-5, (rel.max(), x[np.argmax(rel)])
    # the error is the polynomial's on the reduced argument: both signs occur (no bias)
    sgn = np.sign(y - ref)
    assert (sgn > 0).mean() > 0.2 and (sgn < 0).mean() > 0.2


def test_small_arguments_and_minus_infinity(run):
    x = np.array([-125.0, -125.5, -126.0, -200.0, -1e30, -np.inf], np.float32)
    y = run(x).astype(np.float64)
    assert np.all(y > 0) and np.all(y <= 2.0 ** -124)
    assert np.all(y[1:] == y[0])            # everything below -125 is clamped to -125


def test_agrees_with_the_exponent_for_powers_of_two(run):
    j = np.arange(-125, 128)
    y = run(j.astype(np.float32)).astype(np.float64)
    # 2^j times the polynomial's value at f = 0 (its constant term), exactly
    c0 = np.float64(np.float32(0.9999280571937561))
    assert np.array_equal(y, c0 * np.exp2(j.astype(np.float64)))
