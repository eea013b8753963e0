"""The allocation-free timestep embedding against the allocating entry point.

af_timestep_embed_noalloc serves callers that cannot allocate device memory
(their memory is budgeted by another allocator, or cudaMalloc would stall a
latency-critical loop, or they may only allocate at start-up); it keeps its
intermediates in one fixed device array instead of an af_scratch.  This test
calls it twice in a row through the C ABI and checks each result against
af_timestep_embed on the same inputs: both run the same kernels on the same
inputs, so the results must be identical bit for bit (the timestep-embedding
parity test holds af_timestep_embed itself to the oracle); the second call must
not be disturbed by what the first one left in the shared array.  It also checks that an
oversized batch is refused.  It lives in its own file, collected last, so a
run that stops at the first failure has already run every other test; it
needs nothing from the other tests.
"""
import numpy as np
import pytest
import torch

import oracle as O
from helpers import af_config, draw_weights, full_config, to_f32, upload

pytestmark = pytest.mark.gpu


def test_noalloc_timestep_embed_matches_allocating_entry():
    import diffusion_transformer_denoising_auraflow_b200 as af
    cfg = full_config()
    names = [n for n, _ in O.weight_specs(cfg) if n.startswith("time_step_proj")]
    w = af.Weights(af_config(cfg))
    upload(w, draw_weights(cfg, 51, names))
    s = af.Scratch(w, 4, 64, 8)
    t1 = to_f32(np.array([0.0, 0.25, 0.5, 1.0], np.float32))
    t2 = to_f32(np.array([0.9, 0.123, 0.77, 0.001], np.float32))
    got1 = torch.full((4, 3072), float("nan"), device="cuda")
    got2 = torch.full((4, 3072), float("nan"), device="cuda")
    af.timestep_embed_noalloc(w, t1, got1)      # two calls in a row
    af.timestep_embed_noalloc(w, t2, got2)
    ref1 = torch.empty(4, 3072, device="cuda")
    ref2 = torch.empty(4, 3072, device="cuda")
    af.timestep_embed(w, s, t1, ref1)
    af.timestep_embed(w, s, t2, ref2)
    s.sync()
    assert torch.equal(got1, ref1)
    assert torch.equal(got2, ref2)
    # batch too large for the fixed array: refused before any launch
    big = torch.zeros(32, device="cuda")
    out = torch.zeros(32, 3072, device="cuda")
    with pytest.raises(af.AFError) as ei:
        af.timestep_embed_noalloc(w, big, out)
    assert ei.value.status == 2
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0
