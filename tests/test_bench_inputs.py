"""bench.py's input plumbing on CPU: tensors drawn in spawned worker processes
are the bits the seeded recipe gives in this process, and linears that the
recipe makes identical share one generated tensor."""
import numpy as np

import bench
from bit_nf4_quantised_codebook_b200 import inputs


def test_parallel_generation_matches_the_recipe():
    c = inputs.LinearCase("g", M=48, N=96, K=128, r=8, alpha=16.0, w_std=0.02, a_std=0.05, b_std=0.05,
                          outlier_frac=0.01, seed=7)
    req = {bench.tensor_key(k, c): (k, c) for k in ("W", "X", "A", "B", "dY")}
    par = bench.generate(req, workers=2)
    for kind in ("W", "X", "A", "B", "dY"):
        assert np.array_equal(par[bench.tensor_key(kind, c)], getattr(c, kind)()), kind


def test_identical_linears_share_tensors():
    q, k, v, o, gate, up, down = inputs.shapes_65b()
    assert bench.tensor_key("W", q) == bench.tensor_key("W", k) == bench.tensor_key("W", o)
    assert bench.tensor_key("W", gate) == bench.tensor_key("W", up) != bench.tensor_key("W", q)
    assert bench.tensor_key("X", q) == bench.tensor_key("X", gate) != bench.tensor_key("X", down)
    assert bench.tensor_key("dY", q) == bench.tensor_key("dY", down) != bench.tensor_key("dY", gate)


def test_layer_set_flops():
    """Summed over the seven linears: 3.439e12 (LLaMA-7B layer) and 2.702e13 (65B shapes) flop per fwd+bwd."""
    f7 = sum(c.flops_fwd() + c.flops_bwd() for c in bench.layer_cases("llama7b_layer"))
    f65 = sum(c.flops_fwd() + c.flops_bwd() for c in bench.layer_cases("shapes_65b"))
    assert abs(f7 - 3.439e12) / 3.439e12 < 1e-3
    assert abs(f65 - 2.702e13) / 2.702e13 < 1e-3
    for c in bench.layer_cases("shapes_65b"):
        f, b = bench.fused_flops(c)
        assert f + b < c.flops_fwd() + c.flops_bwd()
