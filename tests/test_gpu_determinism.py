"""Run-to-run determinism of the linear layer on the GPU.

The library's reductions all run in a fixed order, so repeating a forward or
backward on the same inputs must give the same bits every time.  These tests
repeat each call 30 times back to back on one stream — the way a training
loop issues them, with each launch allowed to overlap the previous one's tail —
and compare every output with the first.  Shapes: the CTA-pair path (4096
tokens; a square and both rectangular LLaMA-7B projections), the one-CTA path
(100 tokens) and the small-M path (16 tokens).
"""
import pytest
import torch

from bit_nf4_quantised_codebook_b200 import inputs

pytestmark = pytest.mark.gpu

REPS = 30


def _api():
    from bit_nf4_quantised_codebook_b200 import build
    build.build()
    from bit_nf4_quantised_codebook_b200 import api
    return api


def _case(name, M, N, K):
    return inputs.LinearCase(name, M=M, N=N, K=K, r=64, alpha=16.0, w_std=0.02, a_std=0.01, b_std=0.01)


CASES = [_case("det_q", 4096, 4096, 4096), _case("det_gate", 4096, 11008, 4096),
         _case("det_down", 4096, 4096, 11008), _case("det_m100", 100, 8192, 8192),
         _case("det_m16", 16, 8192, 8192)]


@pytest.mark.parametrize("case", CASES, ids=[c.name for c in CASES])
def test_repeated_calls_are_bit_identical(case):
    api = _api()
    dev = torch.device("cuda", 0)
    q = api.qlora_quantize(api.bits_to_tensor(case.W(), dev))
    X, A, B, dY = (api.bits_to_tensor(getattr(case, k)(), dev) for k in ("X", "A", "B", "dY"))
    err = api.new_error_word(dev)
    Y = torch.empty(case.M, case.N, dtype=torch.bfloat16, device=dev)
    sT = torch.empty(case.M, case.r, dtype=torch.bfloat16, device=dev)
    dX = torch.empty(case.M, case.K, dtype=torch.bfloat16, device=dev)
    dA = torch.empty(case.K, case.r, dtype=torch.float32, device=dev)
    dB = torch.empty(case.r, case.N, dtype=torch.float32, device=dev)
    first = None
    differs = []
    for rep in range(REPS):
        api.qlora_linear_forward(q, X, A, B, case.s, Y=Y, T_save=sT, dev_err=err)
        api.qlora_linear_backward(q, X, dY, A, B, case.s, T_saved=sT, dX=dX, dA=dA, dB=dB, dev_err=err)
        out = [t.clone() for t in (Y, sT, dX, dA, dB)]
        if first is None:
            first = out
        else:
            differs += [(rep, name) for name, a, b in zip(("Y", "sT", "dX", "dA", "dB"), out, first)
                        if not torch.equal(a, b)]
    torch.cuda.synchronize()
    assert int(err[0].item()) == 0
    assert not differs, f"outputs changed between repetitions: {differs[:8]}"
