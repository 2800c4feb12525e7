"""Failure detection on the GPU without a fault: a bounded device wait that
runs out reports through the device error word, and the context stays usable.

Every wait in the library's kernels is bounded; when one expires, the kernel
records a site code in the error word, leaves its loops and returns, and
tp_check_error reports TP_ERR_TIMEOUT.  tp_selftest_wait_timeout drives
exactly that path with a barrier that nothing completes and a short limit.
"""
import time

import pytest
import torch

import tensor_transformer_layer_column_b200 as tl
from gpu_util import assert_no_device_error, dev, dims_of, require_gpu
from oracle import mlp as omlp
from parity import check
from synth import make_inputs, to_f64, workload
from tensor_transformer_layer_column_b200.sublayer import ShardedMLP

pytestmark = pytest.mark.gpu

SELFTEST_CODE = 0x0F1


def test_expired_wait_is_reported_and_cleared():
    require_gpu()
    assert_no_device_error()
    t0 = time.perf_counter()
    tl.selftest_wait_timeout(50_000_000)          # 50 ms
    code = tl.check_error()
    elapsed = time.perf_counter() - t0
    assert code == SELFTEST_CODE
    assert 0.04 <= elapsed < 5.0                  # the wait ran to its limit, then returned
    assert tl.check_error() == 0                  # tp_check_error cleared the word


def test_context_usable_after_expired_wait():
    """After a timed-out wait the same context still computes correctly."""
    require_gpu()
    tl.selftest_wait_timeout(10_000_000)
    assert tl.check_error() == SELFTEST_CODE
    w = workload("mlp_fwd_T128_D256_F1024_t2")
    inp = make_inputs(w, with_dy=False)
    g = dev(inp)
    m = ShardedMLP(dims_of(w), g["w1"], g["b1"], g["w2"], g["b2"])
    o = m.forward(g["x"])
    torch.cuda.synchronize()
    assert_no_device_error()
    y, _, _ = omlp.mlp_fwd(*(to_f64(inp[k]) for k in ("x", "w1", "b1", "w2", "b2")))
    check("y", o["y"], y)
