"""Failure detection on the GPU without a fault: a bounded device wait that
runs out reports through the device error word, and the context stays usable.

Every wait in the library's kernels is bounded; when one expires, the kernel
records a site code in the error word, leaves its loops and returns, and
tp_check_error reports TP_ERR_TIMEOUT.  tp_selftest_wait_timeout drives
exactly that path with a barrier that nothing completes and a short limit.

A value that overflows fp16 where the attention sublayer stores fp16 ("The
attention heads split": qkv holds the shard's projections) is recorded the
same way and reported as TP_ERR_RANGE; inputs scaled past the fp16 range
drive it without any fault.
"""
import time

import pytest
import torch

import tensor_transformer_layer_column_b200 as tl
from gpu_util import assert_no_device_error, dev, dims_of, require_gpu
from oracle import attention as oatt
from oracle import mlp as omlp
from parity import check
from synth import Workload, make_inputs, to_f64, workload
from tensor_transformer_layer_column_b200.sublayer import ShardedAttention, ShardedMLP

pytestmark = pytest.mark.gpu

SELFTEST_CODE = 0x0F1
RANGE_CODE = 0x301
TP_ERR_TIMEOUT, TP_ERR_RANGE = 6, 7


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


def test_status_names_the_kind_of_error():
    require_gpu()
    tl.selftest_wait_timeout(10_000_000)
    assert tl.check_status() == (TP_ERR_TIMEOUT, SELFTEST_CODE)
    assert tl.check_status() == (0, 0)
    assert tl.lib().tp_status_string(TP_ERR_RANGE) == b"TP_ERR_RANGE"


def test_fp16_overflow_in_qkv_is_reported_as_a_range_error():
    """Wqkv ~ N(0, 2000^2) keeps Wqkv itself inside fp16 (|w| < 65504) but puts
    about 4 % of qkv = x Wqkv (std 2000 * sqrt(256) = 32000) beyond 65504.
    The QKV product's epilogue records 0x301; tp_check_error reports
    TP_ERR_RANGE with that code and clears it; the same context then computes
    an unscaled attention forward that matches the oracle."""
    require_gpu()
    assert_no_device_error()
    w = Workload("range", "attn_fwd", batch=1, seq=64, hidden=256, heads=4, head_dim=64, t=2)
    inp = make_inputs(w)
    big = dict(inp)
    big["wqkv"] = (inp["wqkv"].float() * 1e5).to(torch.bfloat16)     # 0.02 * 1e5 = 2000
    assert float(big["wqkv"].float().abs().max()) < 65504.0
    g = dev(big)
    m = ShardedAttention(dims_of(w), g["wqkv"], g["bqkv"], g["wout"], g["bout"])
    m.forward(g["x"])
    assert tl.check_status() == (TP_ERR_RANGE, RANGE_CODE)
    assert tl.check_status() == (0, 0)

    g = dev(inp)
    m = ShardedAttention(dims_of(w), g["wqkv"], g["bqkv"], g["wout"], g["bout"])
    o = m.forward(g["x"])
    torch.cuda.synchronize()
    assert_no_device_error()
    x, wqkv, bqkv, wout, bout = (to_f64(inp[k]) for k in ("x", "wqkv", "bqkv", "wout", "bout"))
    y, _ = oatt.attn_fwd(x, wqkv, bqkv, wout, bout, w.batch, w.heads, w.causal)
    check("y", o["y"], y)
