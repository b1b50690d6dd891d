"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
function include/sparsepr.h declares, and its host arithmetic and argument checks
behave (no kernel is launched here)."""
import ctypes
import os
import re

import pytest

import free_block_sparse_response_b200 as spr
from oracle import sparsepr_oracle as O

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "sparsepr.h")


@pytest.fixture(scope="module")
def L():
    from free_block_sparse_response_b200.build import build
    build()
    return spr.lib()


def test_header_declarations_are_exported(L):
    text = open(HEADER).read()
    declared = set(re.findall(r"SPARSEPR_API\s+[\w\s\*]+?\b(sparsepr_\w+)\s*\(", text))
    assert declared == set(spr.EXPORTED_SYMBOLS)
    for name in declared:
        assert getattr(L, name) is not None


def test_route_k_and_groups_match_oracle(L):
    for n, b, rho, p in [(1024, 64, 0.25, 32), (8192, 128, 0.22, 64), (75600, 128, 0.22, 256),
                         (118800, 128, 0.22, 256), (32760, 128, 0.26, 512), (1000, 64, 0.0, 3),
                         (1000, 64, 5.0, 3), (777, 64, 0.3, 0), (128, 128, 1.0, 0)]:
        assert spr.route_k(n, b, rho, p) == O.route_k(n, b, rho, p)
        assert spr.num_groups(n, b) == O.n_groups(n, b)


def test_workspace_size_positive_and_rejects_bad_sizes(L):
    cfg = spr.SparsePRConfig()
    assert spr.workspace_size(1, 40, 75600, 128, cfg) > 40 * 75600 * 591 * 4
    assert L.sparsepr_workspace_size(1, 1, 100, 96, ctypes.byref(cfg.c())) == 0
    bad = spr.SparsePRConfig(block=48)
    assert L.sparsepr_workspace_size(1, 1, 100, 64, ctypes.byref(bad.c())) == 0


def test_argument_errors_return_codes_without_launching(L):
    cfg = spr.SparsePRConfig(block=128).c()
    # unsupported head dim: rejected before any device work
    rc = L.sparsepr_partition(None, None, spr.BF16, 1, 1, 100, 96, ctypes.byref(cfg), None, None, None, None,
                              None, None, None, None)
    assert rc == spr.ERR_UNSUPPORTED
    assert b"head dim" in L.sparsepr_last_error()
    rc = L.sparsepr_partition(None, None, 7, 1, 1, 100, 128, ctypes.byref(cfg), None, None, None, None, None,
                              None, None, None)
    assert rc == spr.ERR_INVALID_ARG
    rc = L.sparsepr_sparse_attn(None, None, None, spr.BF16, 1, 1, 100, 128, 128, None, None, None, None, None, 1,
                                0.0, None, None, None)
    assert rc == spr.ERR_INVALID_ARG
    rc = L.sparsepr_fit_residual(None, None, None, 1, 1, 128, 64, -1.0, 8, 0, None, None, None, None)
    assert rc == spr.ERR_INVALID_ARG
    rc = L.sparsepr_test_topk(None, 1, 4, 4, 5, None, None, None)
    assert rc == spr.ERR_INVALID_ARG
    # an unknown partition rule is refused before anything is launched (the non-null
    # pointers below are never dereferenced on the host)
    bad = spr.SparsePRConfig(partition_mode=7).c()
    fake = ctypes.c_void_p(256)
    rc = L.sparsepr_partition(fake, fake, spr.BF16, 1, 1, 1024, 128, ctypes.byref(bad), None, fake, fake, fake, fake,
                              fake, fake, None)
    assert rc == spr.ERR_INVALID_ARG
    assert b"partition_mode" in L.sparsepr_last_error()
    bad = spr.SparsePRConfig(route_budget=5).c()
    k_out = ctypes.c_int32(0)
    rc = L.sparsepr_route(fake, fake, fake, 1, 1, 1024, ctypes.byref(bad), fake, ctypes.byref(k_out), None, fake, None)
    assert rc == spr.ERR_INVALID_ARG
    assert b"route_budget" in L.sparsepr_last_error()
    bad = spr.SparsePRConfig(route_budget=spr.BUDGET_GLOBAL, density=float("nan")).c()
    rc = L.sparsepr_route(fake, fake, fake, 1, 1, 1024, ctypes.byref(bad), fake, ctypes.byref(k_out), None, fake, None)
    assert rc == spr.ERR_INVALID_ARG
    assert b"density" in L.sparsepr_last_error()


def test_params_struct_layout():
    assert ctypes.sizeof(spr.sparsepr._CParams) == 56
    assert spr.sparsepr._CParams.density.offset == 24
    assert spr.sparsepr._CParams.scale.offset == 40
    assert spr.sparsepr._CParams.partition_mode.offset == 44
    assert spr.sparsepr._CParams.route_scores.offset == 48
    assert spr.sparsepr._CParams.route_budget.offset == 52


def test_python_wrappers_refuse_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 64, 64)
    with pytest.raises(ValueError):
        spr.dense_attn(q, q, q, block=64)


def test_misaligned_inputs_are_refused(L):
    """Q, K and V are read with 16-byte vector and TMA loads: a start off a 16-byte
    boundary is refused before anything is launched (pointers never dereferenced)."""
    cfg = spr.SparsePRConfig(block=128).c()
    ok, odd = ctypes.c_void_p(256), ctypes.c_void_p(256 + 8)
    rc = L.sparsepr_partition(ok, odd, spr.BF16, 1, 1, 1024, 128, ctypes.byref(cfg), None, ok, ok, ok, ok, ok, ok,
                              None)
    assert rc == spr.ERR_INVALID_ARG
    assert b"16-byte" in L.sparsepr_last_error()
    rc = L.sparsepr_sparse_attn(odd, ok, ok, spr.BF16, 1, 1, 1024, 128, 128, ok, ok, ok, ok, ok, 1, 0.0, ok, ok,
                                None)
    assert rc == spr.ERR_INVALID_ARG
    rc = L.sparsepr_probe_dense(ok, ok, odd, spr.BF16, 1, 1, 1024, 128, 128, ok, 8, ok, ok, ok, ok, 1, 0.0, ok, ok,
                                ok, None)
    assert rc == spr.ERR_INVALID_ARG


def test_one_call_entries_refuse_bad_arguments(L):
    """The one-call entries check their arguments before anything is launched."""
    cfg = spr.SparsePRConfig(block=128, n_probe=0).c()
    ok = ctypes.c_void_p(256)
    assert L.sparsepr_call_workspace_size(spr.BF16, 1, 2, 1024, 128, ctypes.byref(cfg)) == 0  # n_probe = 0
    rc = L.sparsepr_attention(ok, ok, ok, spr.BF16, 1, 2, 1024, 128, ctypes.byref(cfg), ok, ok, None)
    assert rc == spr.ERR_INVALID_ARG
    good = spr.SparsePRConfig(block=128, n_sampled=64, n_probe=16).c()
    assert L.sparsepr_call_workspace_size(spr.BF16, 1, 2, 1024, 128, ctypes.byref(good)) > \
        L.sparsepr_workspace_size(1, 2, 1024, 128, ctypes.byref(good))
    assert L.sparsepr_host_workspace_size(spr.BF16, 1, 2, 1024, 128, ctypes.byref(good), 0) == 0
    rc = L.sparsepr_attention_host(ok, ok, ok, spr.BF16, 1, 2, 1024, 128, ctypes.byref(good), ok, 0, ok, None, None)
    assert rc == spr.ERR_INVALID_ARG and b"groups" in L.sparsepr_last_error()
    s = ctypes.c_void_p(4096)
    rc = L.sparsepr_attention_host(ok, ok, ok, spr.BF16, 1, 2, 1024, 128, ctypes.byref(good), ok, 2, ok, s, s)
    assert rc == spr.ERR_INVALID_ARG and b"copy stream" in L.sparsepr_last_error()


def test_call_workspace_holds_full_route_rows_under_the_global_budget():
    """The one-call workspace sizes the route for k groups per block under the uniform
    budget and for all G groups (rows padded with -1) under the global budget."""
    L = spr.lib()
    uni = spr.SparsePRConfig(block=128, n_sampled=512, n_probe=256, density=0.22)
    glo = spr.SparsePRConfig(block=128, n_sampled=512, n_probe=256, density=0.22, route_budget=spr.BUDGET_GLOBAL)
    n, h = 75600, 2
    g = spr.num_groups(n, 128)
    k = spr.route_k(n, 128, 0.22, 256)
    a = int(L.sparsepr_call_workspace_size(spr.BF16, 1, h, n, 128, ctypes.byref(uni.c())))
    b = int(L.sparsepr_call_workspace_size(spr.BF16, 1, h, n, 128, ctypes.byref(glo.c())))
    assert a > 0 and b > a
    assert b - a >= 4 * h * g * (g - k)  # the extra route columns, before alignment
    assert b - a <= 4 * h * g * (g - k) + 4096
