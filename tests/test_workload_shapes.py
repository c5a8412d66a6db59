"""The synthetic workloads have the shapes of Jamba's Mamba layer as the pages
print them (tests/golden/jamba_layer_shapes.json), and the generators follow
the stated recipe (CPU only)."""
import json
import math
import os

import torch

from selective_state_space_26_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "jamba_layer_shapes.json")


def _g(key):
    with open(GOLDEN) as f:
        return json.load(f)[key]["value"]


def test_jamba_sized_workloads_match_the_pages():
    d_inner = _g("d_model") * _g("expansion")
    for name, w in synth.WORKLOADS.items():
        if "tiny" in name:
            continue
        assert w.d_inner == d_inner, name
        assert w.d_state == _g("d_state"), name
        assert w.batch * w.seqlen <= _g("max_context_tokens") * 16, name
    longest = max(w.seqlen for w in synth.WORKLOADS.values())
    assert longest == _g("max_context_tokens")


def test_delta_bias_centres_delta_on_log_uniform_dt0():
    bias = synth.dt_bias_for(8192, 1).double()
    dt0 = torch.log1p(torch.exp(bias))   # softplus(bias): the step size at zero noise
    assert float(dt0.min()) >= 1e-3 * (1 - 1e-6) and float(dt0.max()) <= 1e-1 * (1 + 1e-6)
    # log-uniform on [1e-3, 1e-1]: log10(dt0) uniform on [-3, -1]
    l = torch.log10(dt0)
    assert abs(float(l.mean()) + 2.0) < 0.03
    assert abs(float(l.std()) - 2.0 / math.sqrt(12.0)) < 0.03


def test_A_and_state_recipes():
    A = synth.make_A(8, 16)
    assert torch.equal(A[3], -torch.arange(1, 17, dtype=torch.float32))
    st = synth.decode_state(4, 256, 16, 7)
    assert st.dtype == torch.float32 and abs(float(st.std()) - 0.1) < 0.005


def test_projection_inputs_follow_their_recipe():
    """dt_low arrives as two bf16 planes whose sum is dt_low to ~2^-16 relative;
    W_dt stays inside +-R^-1/2; W_x has std ~d_inner^-1/2 so projected entries
    are ~N(0, 1); norm weights lie in [0.5, 1.5]; the draws are seeded."""
    di = synth.dt_proj_inputs(64, 512, 256, seed=7, device="cpu")
    rec = di.hi.double() + di.lo.double()
    rel = (rec - di.dt_low.double()).abs() / di.dt_low.double().abs().clamp_min(1e-30)
    assert float(rel.max()) <= 2.0 ** -16
    assert float(di.W_dt.float().abs().max()) <= 256 ** -0.5
    again = synth.dt_proj_inputs(64, 512, 256, seed=7, device="cpu")
    assert torch.equal(again.hi, di.hi) and torch.equal(again.W_dt, di.W_dt)
    xi = synth.x_proj_inputs(32, 4096, 256, 16, seed=8, device="cpu")
    assert xi.W_x.shape == (288, 4096) and xi.u.dtype == torch.bfloat16
    assert abs(float(xi.W_x.float().std()) * math.sqrt(4096) - 1.0) < 0.05
    proj = xi.u.float() @ xi.W_x.float().T
    assert 0.9 < float(proj.std()) < 1.1
    for w in (xi.w_dt, xi.w_B, xi.w_C):
        assert w.dtype == torch.float32 and float(w.min()) >= 0.5 and float(w.max()) <= 1.5
