"""Exhaustive check of the quantiser's division-free inner loop.

The quantiser normalises each weight by its block absmax with one reciprocal
per block and a corrected quotient per element, and finds the code from a
bucket table (csrc/nf4_quant.cuh).  tests/cuda/check_quotient.cu runs both
over every bfloat16 pair (x, a) the fast path can meet and compares against
CUDA's correctly rounded division and a plain threshold count: the codes (from
the floor-indexed table and from the centred table the quantiser uses) must
agree for every pair and the quotients bit for bit wherever they can matter.
"""
import os
import subprocess
import tempfile

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_fast_quotient_and_bucket_code_exhaustive():
    from bit_nf4_quantised_codebook_b200 import api, build
    build.build()
    _, thr = api.qlora_build_codebook()
    hexes = [format(int(np.float32(t).view(np.uint32)), "08x") for t in thr]
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "check_quotient")
        subprocess.run([build.nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                        "-I", os.path.join(ROOT, "bit_nf4_quantised_codebook_b200", "csrc"),
                        os.path.join(ROOT, "tests", "cuda", "check_quotient.cu"), "-o", exe], check=True)
        out = subprocess.run([exe] + hexes, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    fields = dict(kv.split("=") for kv in out.stdout.split())
    assert int(fields["pairs"]) > 10 ** 9
    assert int(fields["bad_code"]) == 0, out.stdout
    assert int(fields["bad_quotient"]) == 0, out.stdout
    assert int(fields["bad_centred"]) == 0, out.stdout
