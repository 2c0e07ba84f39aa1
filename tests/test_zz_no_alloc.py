"""The residual + LayerNorm GEMM entry point that allocates no device memory.

It serves callers that cannot allocate while running (a real-time audio thread,
a runtime whose device memory is laid out in advance).  Its output must match
the allocating entry point's (albert_test_gemm, epilogue 2) within the
single-kernel tolerance, on two calls in a row with different data (the calls
share one static scratch array), and it must reject M beyond its 2048-row limit
without writing.  This file is collected last so that a stop-at-first-failure
run has already run every other test.
"""
import numpy as np
import pytest
import torch

import synth
import transformer_encoder_albert_b200 as tea

pytestmark = pytest.mark.gpu


def _case(M, K, seed):
    r = np.random.default_rng(seed)
    bf = lambda a: torch.tensor(synth.bf16_round(np.asarray(a, np.float32))).cuda().to(torch.bfloat16)
    f32 = lambda a: torch.tensor(np.asarray(a, np.float32)).cuda()
    return dict(A=bf(r.normal(0, 1, (M, K))), W=bf(r.normal(0, 0.05, (768, K))),
                bias=f32(r.normal(0, 0.1, 768)), R=bf(r.normal(0.3, 1.0, (M, 768))),
                ln_g=f32(1 + r.normal(0, 0.1, 768)), ln_b=f32(r.normal(0, 0.1, 768)))


def _close(got, ref):
    got, ref = got.float().cpu().numpy(), ref.float().cpu().numpy()
    scale = np.max(np.abs(ref))
    assert np.all(np.abs(got - ref) <= 8e-3 * np.abs(ref) + 2e-3 * scale)


def test_noalloc_matches_allocating_entry_on_two_calls_in_a_row():
    for M, K, seed in ((1000, 768, 1), (2048, 2048, 2)):
        c = _case(M, K, seed)
        ref = torch.empty(M, 768, device="cuda", dtype=torch.bfloat16)
        assert tea.test_gemm(c["A"], c["W"], c["bias"], ref, 2, R=c["R"], ln_g=c["ln_g"],
                             ln_b=c["ln_b"], eps=1e-12) == 0
        got = torch.full((M, 768), 5.0, device="cuda", dtype=torch.bfloat16)
        assert tea.gemm_residual_ln_noalloc(c["A"], c["W"], c["bias"], c["R"], c["ln_g"], c["ln_b"],
                                            got, eps=1e-12) == 0
        _close(got, ref)


def test_noalloc_rejects_rows_beyond_its_static_scratch():
    c = _case(2049, 768, 3)
    Y = torch.full((2049, 768), 5.0, device="cuda", dtype=torch.bfloat16)
    rc = tea.gemm_residual_ln_noalloc(c["A"], c["W"], c["bias"], c["R"], c["ln_g"], c["ln_b"], Y)
    assert rc == 3  # ALBERT_ERR_SHAPE
    torch.cuda.synchronize()
    assert torch.all(Y == 5.0)
