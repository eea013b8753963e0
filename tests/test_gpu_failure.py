"""Failure detection on the GPU, without a GPU fault.

Every wait of the device pipelines is bounded; a wait that runs out records
the timeout in the scratch's error word, the kernel frees its TMEM and
returns, and af_sync reports AF_ERR_TIMEOUT.  af_check_wait_timeout runs that
path on purpose (an mbarrier phase that nothing completes, a 20 ms limit):
the report must arrive, be cleared by the report, and leave the context
usable for the tensor-core kernels, which allocate TMEM again.
"""
import time

import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import af_config, tiny_config, to_bf16, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def af():
    import diffusion_transformer_denoising_auraflow_b200 as m
    assert torch.cuda.is_available()
    return m


def _linear_ok(af, M, N, K, seed):
    A = synth.normal(seed, f"fA{M}_{N}_{K}", (M, K), 1.0)
    W = synth.normal(seed + 1, f"fW{M}_{N}_{K}", (N, K), 0.02)
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    af.linear(to_bf16(A), to_bf16(W), C)
    torch.cuda.synchronize()
    ref = A.astype(np.float64) @ W.astype(np.float64).T
    return O.rel_l2(to_np(C), ref)


def test_wait_timeout_is_reported_and_the_context_stays_usable(af):
    w = af.Weights(af_config(tiny_config()))
    s = af.Scratch(w, 1, 64, 8)
    s.sync()                                  # nothing pending
    t0 = time.monotonic()
    s.check_wait_timeout(20_000_000)
    with pytest.raises(af.AFError) as e:
        s.sync()
    elapsed = time.monotonic() - t0
    assert e.value.status == 6                # AF_ERR_TIMEOUT
    assert 0.015 < elapsed < 5.0, elapsed     # the wait ran to its limit, and no further
    s.sync()                                  # the report cleared the word
    # TMEM was released: the 1-CTA and the CTA-pair GEMMs allocate it again
    assert _linear_ok(af, 300, 520, 256, 31) < 3e-3
    assert _linear_ok(af, 1100, 776, 520, 33) < 3e-3
    s.sync()
    # and the check can be repeated
    s.check_wait_timeout(5_000_000)
    with pytest.raises(af.AFError) as e:
        s.sync()
    assert e.value.status == 6
    s.sync()
