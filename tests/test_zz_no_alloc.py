"""The allocation-free quantiser entry point (qlora_quantize_noalloc).

Some callers cannot allocate device memory — e.g. a plugin interface that
passes input and output buffers but offers no allocator, or a runtime whose
memory plan forbids new allocations mid-step — so they cannot provide the
workspace qlora_quantize needs.  qlora_quantize_noalloc keeps that scratch in
a static device array inside the library instead.  This test calls it through
the C ABI twice in a row (two different weights, so the second call must not
depend on what the first left in the shared array) and checks that each result
equals the workspace-based qlora_quantize bit for bit, the tolerance every
quantiser test here uses, and the first also equals the CPU oracle directly.
A weight at the array's limit (8192 x 8192, after a smaller call has left its
contents in the array) must match too, and one row over the limit is rejected
before anything is launched.  Kept in its own file, named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_nf4_quantised_codebook_b200 import inputs
from oracle import nf4

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
    for i, (n, k, seed) in enumerate(shapes):
        wb = inputs.weight_bf16(n, k, 0.02, seed, 0.001)
        W = api.bits_to_tensor(wb)
        err = api.new_error_word()
        ref = api.qlora_quantize(W, dev_err=err)
        out = api.alloc_weight(n, k)
        api.qlora_quantize_noalloc(W, out, dev_err=err)
        torch.cuda.synchronize()
        assert int(err[0].item()) == 0
        _same(out, ref)
        if i == 0:  # and the CPU oracle, directly
            want = nf4.quantize_nf4(wb)
            assert np.array_equal(out.codes.cpu().numpy(), want["codes"])
            assert np.array_equal(out.c2q.cpu().numpy(), want["c2q"])
            assert np.array_equal(out.c1.cpu().numpy(), want["c1"])
            assert out.mean.cpu().numpy()[0] == want["mean"]


def test_noalloc_at_the_limit_after_a_smaller_call():
    """N*K = 2^26 uses every absmax slot and group sum of the array and the mean
    tree's global-memory levels; the smaller call before it leaves its own values
    in the array."""
    api = _api()
    err = api.new_error_word()
    for n, k, seed in [(512, 4096, 43), (8192, 8192, 44)]:
        W = api.bits_to_tensor(inputs.weight_bf16(n, k, 0.02, seed, 0.001))
        out = api.alloc_weight(n, k)
        api.qlora_quantize_noalloc(W, out, dev_err=err)
        ref = api.qlora_quantize(W, dev_err=err)
        torch.cuda.synchronize()
        assert int(err[0].item()) == 0
        _same(out, ref)


def test_noalloc_rejects_weights_over_the_limit():
    api = _api()
    L = api.lib()
    buf = torch.empty(64, dtype=torch.uint8, device="cuda")
    p = buf.data_ptr()
    for n, k in [(8193, 8192), (16384, 8192)]:          # one row over 2^26 weights, and 2^27
        w = api._Weight(n, k, p, p, p, p)
        st = L.qlora_quantize_noalloc(p, ctypes.byref(w), None, None)
        assert st == 7 and b"static scratch" in L.qlora_status_string(st)
