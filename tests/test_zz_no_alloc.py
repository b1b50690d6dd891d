"""The allocation-free fit entry point against the workspace fit.

Callers such as an inference-engine plugin bound to a memory plan fixed before
execution, or a latency-critical loop that cannot take cudaMalloc's implicit
synchronisation, cannot allocate device memory during a call; for them the library
exports sparsepr_fit_residual_noalloc, whose scratch is a fixed static device array.
This test calls it twice in a row through the C ABI (different inputs each time, so a
stale result from the first call would show) and compares each result with the
workspace entry point on the same inputs, at the fit test's tolerance.  It must pass in
a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

import free_block_sparse_response_b200 as spr

pytestmark = pytest.mark.gpu

TOL_FIT = 1e-5   # same bound as the fit-kernel parity test


def _probe_problem(seed, heads, p, d):
    """Probe outputs whose residual is a noisy affine function of the sparse output."""
    rng = np.random.default_rng(seed)
    xs = rng.normal(size=(1, heads, p, d))
    m_true = rng.normal(size=(heads, d, d)) * 0.05
    dp = xs + np.einsum("hij,bhpj->bhpi", m_true, xs) + 0.3 + 0.01 * rng.normal(size=xs.shape)
    return (torch.from_numpy(xs).float().cuda().contiguous(), torch.from_numpy(dp).float().cuda().contiguous())


def _rel(a, b):
    return float((a.double() - b.double()).norm() / b.double().norm())


def test_noalloc_fit_matches_workspace_fit_twice():
    from free_block_sparse_response_b200.build import build
    build()
    heads, p, d = 6, 256, 128
    cfg = spr.SparsePRConfig(n_probe=p, rank=32, ridge_lambda=1e-3)
    ws = spr.new_workspace(1, heads, 4 * p, d, cfg, torch.device("cuda"))
    m = torch.empty(1, heads, d, d, device="cuda")
    beta = torch.empty(1, heads, d, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call, seed in enumerate((11, 12)):
        xs, dp = _probe_problem(seed, heads, p, d)
        m_ref, b_ref = spr.fit_residual(xs, dp, cfg, ws)
        spr.check(ws)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        spr.fit_residual_noalloc(xs, dp, cfg, m, beta, status=status)
        torch.cuda.synchronize()
        free_after = torch.cuda.mem_get_info()[0]
        if call == 1:   # the first call may load the library module that holds the array
            assert free_after == free_before, "the no-allocation call changed free device memory"
        assert int(status.item()) == spr.OK, f"call {call}: device status"
        assert _rel(m, m_ref) <= TOL_FIT, f"call {call}: M"
        assert _rel(beta, b_ref) <= TOL_FIT, f"call {call}: beta"


def test_noalloc_fit_zero_weights_fall_back_to_uniform_and_report():
    """Caller weights that sum to zero: like the workspace fit, the call records
    INVALID_ARG in its status and fits the heads with uniform weights, so M and beta
    equal the uniform-weight fit of the same probes."""
    heads, p, d = 2, 128, 128
    cfg = spr.SparsePRConfig(n_probe=p, rank=16, ridge_lambda=1e-3)
    cfg_u = spr.SparsePRConfig(n_probe=p, rank=16, ridge_lambda=1e-3, weight_mode=spr.WEIGHT_UNIFORM)
    xs, dp = _probe_problem(13, heads, p, d)
    zero_w = torch.zeros(1, heads, p, device="cuda")
    ws = spr.new_workspace(1, heads, 4 * p, d, cfg, torch.device("cuda"))
    m_ref, b_ref = spr.fit_residual(xs, dp, cfg_u, ws)
    spr.check(ws)
    m = torch.empty(1, heads, d, d, device="cuda")
    beta = torch.empty(1, heads, d, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    spr.fit_residual_noalloc(xs, dp, cfg, m, beta, weights=zero_w, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == spr.ERR_INVALID_ARG
    assert _rel(m, m_ref) <= TOL_FIT and _rel(beta, b_ref) <= TOL_FIT
    # the next call starts from a clear status word
    spr.fit_residual_noalloc(xs, dp, cfg_u, m, beta, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == spr.OK


def test_noalloc_fit_rejects_sizes_beyond_its_scratch():
    heads, p, d = 64, 256, 128      # 64 * 516 KiB > 32 MiB
    cfg = spr.SparsePRConfig(n_probe=p)
    xs = torch.zeros(1, heads, p, d, device="cuda")
    m = torch.empty(1, heads, d, d, device="cuda")
    beta = torch.empty(1, heads, d, device="cuda")
    with pytest.raises(spr.SparsePRError) as ei:
        spr.fit_residual_noalloc(xs, xs, cfg, m, beta)
    assert ei.value.code == spr.ERR_UNSUPPORTED
    assert "fixed array" in str(ei.value)
