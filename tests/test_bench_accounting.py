"""The byte counts bench.py divides by, checked against the sizes the library
itself reports for the stored formats (host calls, no GPU) and against the
oracle's storage accounting."""
import ctypes
import itertools

import pytest

import bench
from oracle import formats as F
from oracle import nf4


@pytest.fixture(scope="module")
def api():
    from bit_nf4_quantised_codebook_b200 import build
    build.build()
    from bit_nf4_quantised_codebook_b200 import api as a
    return a


def test_format_stored_bytes_match_library_sizes(api):
    L = api.lib()
    for (cb, block, dq), (n, k) in itertools.product(
            itertools.product(bench.FORMAT_CODEBOOKS, bench.FORMAT_BLOCKS, bench.FORMAT_DQ),
            [(4096, 4096), (40, 1536), (11008, 4096)]):
        f = api._Format(api.CODEBOOKS[cb], block, api.DQ_MODES[dq])
        a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
        assert L.qlora_format_sizes(ctypes.byref(f), n, k, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)) == 0
        mean = 0 if dq == "none" else 4
        assert bench.format_stored_bytes(n, k, block, dq) == a.value + b.value + c.value + mean
        bits = F.storage_bits_per_weight(block, dq, n, k)
        assert abs(8 * bench.format_stored_bytes(n, k, block, dq) / (n * k) - bits) < 1e-12


def test_merge_bytes(api):
    for _, n, k in bench.MERGE_SHAPES:
        cb, qb, sb = api.qlora_nf4_sizes(n, k)
        packed = cb + qb + sb + 4
        assert packed == nf4.storage_bytes(n, k)
        assert bench.merge_bytes(n, k, 64) == 2 * packed + 2 * 64 * (k + n)
        nb = n * k // 64
        assert bench.merge_kernel_bytes(n, k, 64) == packed + 2 * 64 * (k + n) + n * k // 2 + 4 * nb


def test_adamw_bytes_per_parameter():
    # read p, g, m, v (float32); write p, m, v (float32) and the bfloat16 copy
    assert bench.ADAMW_BYTES_PER_PARAM == 4 * 4 + 3 * 4 + 2


def test_fused_gemm_bytes_and_per_shape_traffic():
    """The fused GEMMs' algorithmic bytes count the stored weight as the library
    sizes it, and a layer set's DRAM traffic is the sum of its linears'
    per-shape captures (q, k, v, o share one shape, gate and up another), or
    None once a shape is missing or the kernel sources differ from the capture's."""
    for c in bench.layer_cases("proj7b"):
        f, b = bench.fused_bytes(c)
        packed = nf4.storage_bytes(c.N, c.K)
        assert f == 2 * c.M * c.K + packed + 2 * c.M * c.r + 2 * c.r * c.N + 2 * c.M * c.N
        assert b == 2 * c.M * c.N + packed + 2 * c.M * c.r + 2 * c.K * c.r + 2 * c.M * c.K
    cases = bench.layer_cases("shapes_65b")
    shapes = {(c.N, c.K) for c in cases}
    assert shapes == {(8192, 8192), (22016, 8192), (8192, 22016)}
    sha = bench.kernel_sources_sha1()
    table = {"sources_sha1": sha}
    for n, (N, K) in enumerate(sorted(shapes)):
        table[("shapes_65b", N, K, "fwd")] = 1000 * (n + 1)
        table[("shapes_65b", N, K, "bwd")] = 7 * (n + 1)
    # sorted shapes: (8192, 8192) x4 -> 1, (8192, 22016) x1 -> 2, (22016, 8192) x2 -> 3
    assert bench.fused_traffic("shapes_65b", cases, "fwd", table) == 1000 * (4 * 1 + 1 * 2 + 2 * 3)
    assert bench.fused_traffic("shapes_65b", cases, "bwd", table) == 7 * (4 * 1 + 1 * 2 + 2 * 3)
    one = [c for c in cases if c.name.split("_")[1] == "gate"]
    assert bench.fused_traffic("shapes_65b", one, "fwd", table) == 3000
    del table[("shapes_65b", 8192, 22016, "bwd")]
    assert bench.fused_traffic("shapes_65b", cases, "bwd", table) is None
    table["sources_sha1"] = "0" * 40
    assert bench.fused_traffic("shapes_65b", cases, "fwd", table) is None
