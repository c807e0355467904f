"""The allocation-free quantiser entry point (qlora_quantize_noalloc).

Some callers cannot allocate device memory — e.g. a plugin interface that
passes input and output buffers but offers no allocator, or a runtime whose
memory plan forbids new allocations mid-step — so they cannot provide the
workspace qlora_quantize needs.  qlora_quantize_noalloc keeps that scratch in
a static device array inside the library instead.  This test calls it through
the C ABI twice in a row (two different weights, so the second call must not
depend on what the first left in the shared array) and checks that each result
equals the workspace-based qlora_quantize bit for bit, the tolerance every
quantiser test here uses.  It also checks that a weight over the array's limit
is rejected before anything is launched.  Kept in its own file, named to be
collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_nf4_quantised_codebook_b200 import inputs

pytestmark = pytest.mark.gpu


def _api():
    from bit_nf4_quantised_codebook_b200 import build
    build.build()
    from bit_nf4_quantised_codebook_b200 import api
    return api


def _same(a, b):
    assert torch.equal(a.codes, b.codes), "packed codes differ"
    assert torch.equal(a.c2q, b.c2q), "E4M3 block constants differ"
    assert torch.equal(a.c1.view(torch.int32), b.c1.view(torch.int32)), "group scales differ"
    assert torch.equal(a.mean[:1].view(torch.int32), b.mean[:1].view(torch.int32)), "mean differs"


def test_noalloc_matches_workspace_quantiser_on_two_calls():
    api = _api()
    shapes = [(1024, 4096, 41), (768, 11008, 42)]   # second: more blocks, groups straddling rows
    for n, k, seed in shapes:
        W = api.bits_to_tensor(inputs.weight_bf16(n, k, 0.02, seed, 0.001))
        err = api.new_error_word()
        ref = api.qlora_quantize(W, dev_err=err)
        out = api.alloc_weight(n, k)
        api.qlora_quantize_noalloc(W, out, dev_err=err)
        torch.cuda.synchronize()
        assert int(err[0].item()) == 0
        _same(out, ref)


def test_noalloc_rejects_weights_over_the_limit():
    api = _api()
    L = api.lib()
    n, k = 16384, 8192                                  # 2^27 weights > 2^26
    buf = torch.empty(64, dtype=torch.uint8, device="cuda")
    p = buf.data_ptr()
    w = api._Weight(n, k, p, p, p, p)
    st = L.qlora_quantize_noalloc(p, ctypes.byref(w), None, None)
    assert st == 7 and b"static scratch" in L.qlora_status_string(st)
