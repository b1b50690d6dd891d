"""Failure detection: a bounded device wait that runs out reports SPARSEPR_ERR_TIMEOUT.

Every spin-wait in the library gives up after a bound and records a timeout in the
workspace's status word instead of hanging.  The test build libsparsepr_waittest.so is
the same source with the cooperative capacity fill's grid-barrier bound cut to zero, so
an ordinary partition call on the Small workload makes that wait run out: the fill
blocks take their error path and return (the barrier guards no asynchronous copy or
tensor-core work, so nothing is left in flight), the call completes, and
sparsepr_check reports the timeout.  The same GPU then runs a normal-build call in a
fresh workspace, which must still pass its checks: the context stays usable.
"""
import ctypes

import numpy as np
import pytest
import torch

import free_block_sparse_response_b200 as spr
from free_block_sparse_response_b200 import sparsepr as binding
from free_block_sparse_response_b200.build import WAITTEST_LIB_PATH, build
from synthetic import CONFIGS, make_inputs

pytestmark = pytest.mark.gpu


def _cfg(w):
    return spr.SparsePRConfig(block=w.block, n_sampled=w.n_sampled, n_probe=w.n_probe,
                              kmeans_iters=w.kmeans_iters, rank=w.rank, density=w.density,
                              ridge_lambda=w.ridge_lambda)


def test_fill_grid_barrier_timeout_is_reported_and_context_survives():
    build()
    build(variant="waittest")
    short = binding.load_library(WAITTEST_LIB_PATH)
    w = CONFIGS["small"]
    cfg = _cfg(w)
    q, k, v = (t.cuda() for t in make_inputs(w, 0, heads=2))
    bt, h, n, d = q.shape
    g = spr.num_groups(n, w.block)
    ws = spr.new_workspace(bt, h, n, d, cfg, q.device)
    outs = [torch.empty(bt, h, g * w.block, dtype=torch.int32, device="cuda"),
            torch.empty(bt, h, g, dtype=torch.int32, device="cuda"),
            torch.empty(bt, h, g * w.block, dtype=torch.int32, device="cuda"),
            torch.empty(bt, h, g, dtype=torch.int32, device="cuda"),
            torch.empty(bt, h, g, g, dtype=torch.float32, device="cuda")]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = short.sparsepr_partition(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), spr.BF16, bt, h, n,
                                  d, ctypes.byref(cfg.c()), None, *(ctypes.c_void_p(t.data_ptr()) for t in outs),
                                  ctypes.c_void_p(ws.data_ptr()), stream)
    assert rc == spr.OK, "the call itself is valid; the timeout is a device-side outcome"
    assert short.sparsepr_check(ctypes.c_void_p(ws.data_ptr()), stream) == spr.ERR_TIMEOUT
    # the partition state stays in bounds after the aborted fill (tokens in [0, N) or -1)
    perm = outs[0].cpu().numpy()
    assert ((perm >= -1) & (perm < n)).all() and (outs[1].cpu().numpy() <= w.block).all()
    # a normal build's call on the same GPU, fresh workspace: completes with no error
    o, parts = spr.attention(q, k, v, cfg, return_parts=True)
    spr.check(parts["ws"])
    assert torch.isfinite(o.float()).all()
    sizes = parts["partition"].key_gsize.cpu().numpy()
    assert (sizes.sum(axis=-1) == n).all()
    want = parts["probe_out"][0, 0].to(o.dtype)
    assert torch.equal(o[0, 0][parts["probe_idx"][0, 0].long()], want)
