"""The C-ABI library loads on any host and exports every symbol include/*.h declares.

No compute calls: these run without a GPU.
"""
import ctypes
import glob
import os
import re

import pytest

import tensor_transformer_layer_column_b200 as tl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"\b(tp_[a-z0-9_]+)\s*\(", src):
            names.add(m.group(1))
    return names


def test_header_declares_the_boundary():
    want = {"tp_mlp_fwd", "tp_mlp_bwd", "tp_attn_fwd", "tp_attn_bwd", "tp_layer_fwd",
            "tp_layer_bwd", "tp_shard_cols", "tp_shard_rows", "tp_shard_qkv_heads",
            "tp_workspace_size", "tp_status_string"}
    assert want <= _declared()


@pytest.fixture(scope="module", autouse=True)
def built_library():
    if not os.path.exists(tl.lib_path):
        from tensor_transformer_layer_column_b200 import build
        build.build()


def test_library_exports_every_declared_symbol():
    handle = ctypes.CDLL(tl.lib_path)
    missing = [n for n in sorted(_declared()) if not hasattr(handle, n)]
    assert not missing, missing
    assert set(tl.EXPORTED_SYMBOLS) == _declared()


def test_host_validation_without_gpu():
    lib = tl.lib()
    assert tl.version().startswith("tplayer-b200")
    assert lib.tp_status_string(4) == b"TP_ERR_WORKSPACE"
    ok = tl.Dims.of(4, 2048, 4096, 16384, 32, 128, 8)
    assert tl.workspace_size(tl.OP_LAYER_BWD, ok) > 0
    assert tl.workspace_size(tl.OP_MLP_FWD, ok) == 0
    # Invalid dims give size 0 (H % t, D != H*dh, unsupported t, dh).
    for bad in (tl.Dims.of(1, 8, 4096, 16384, 30, 128, 8), tl.Dims.of(1, 8, 4096, 16384, 32, 64, 8),
                tl.Dims.of(1, 8, 4096, 16384, 32, 128, 3), tl.Dims.of(1, 8, 4096, 16384, 16, 256, 8)):
        assert tl.workspace_size(tl.OP_LAYER_BWD, bad) == 0
    # Arguments are checked before anything touches a device: these return
    # without a GPU.
    d = tl.Dims.of(1, 8, 256, 1024, 0, 0, 2)
    st = lib.tp_mlp_fwd(ctypes.byref(d), None, None, None, None, None, None, None, None, None,
                        None, 0, None)
    assert st == 1  # TP_ERR_INVALID_ARG: null pointers
    d3 = tl.Dims.of(1, 8, 256, 1024, 0, 0, 3)
    st = lib.tp_mlp_fwd(ctypes.byref(d3), 16, 16, None, 16, None, None, 16, 16, 16, None, 0, None)
    assert st == 2  # TP_ERR_UNSUPPORTED: t = 3
    st = lib.tp_mlp_fwd(ctypes.byref(d), 24, 16, None, 16, None, None, 16, 16, 16, None, 0, None)
    assert st == 3  # TP_ERR_MISALIGNED: x not 16-byte aligned
    st = lib.tp_mlp_bwd(ctypes.byref(d), 16, 16, 16, 16, 16, 16, None, 16, 16, 16, None, None,
                        None, 0, None)
    assert st == 4  # TP_ERR_WORKSPACE
    da = tl.Dims.of(1, 8, 512, 0, 4, 128, 8)
    st = lib.tp_attn_fwd(ctypes.byref(da), 16, 16, None, 16, None, None, 16, 16, 16, 16, None, 0,
                         None)
    assert st == 1  # TP_ERR_INVALID_ARG: heads % t != 0
    assert lib.tp_trace_begin(None, None, None, -1) == 1
    assert lib.tp_trace_end() == 0


def test_recompute_entry_points_host_side():
    """Workspace sizes and argument checks of the recomputation entry points (no GPU).

    The recomputing backward needs the saved activations' bytes on top of the
    ordinary backward workspace, since it rebuilds them there; the forward
    that saves nothing holds them in its workspace instead of caller buffers.
    """
    lib = tl.lib()
    B, S, D, F, H, dh, t = 4, 2048, 4096, 16384, 32, 128, 8
    d = tl.Dims.of(B, S, D, F, H, dh, t)
    T = B * S
    acts = (T * D * 2 + 2 * T * 4 + T * 3 * D * 2 + T * D * 2 + B * H * S * 4 + 2 * T * D * 2
            + 2 * T * 4 + 2 * T * F * 2)
    bwd = tl.workspace_size(tl.OP_LAYER_BWD, d)
    rec = tl.workspace_size(tl.OP_LAYER_BWD_RECOMPUTE, d)
    assert acts <= rec - bwd <= acts + 16 * 256
    fwd = tl.workspace_size(tl.OP_LAYER_FWD, d)
    nos = tl.workspace_size(tl.OP_LAYER_FWD_NOSAVE, d)
    assert acts <= nos - fwd <= acts + 16 * 256
    bad = tl.Dims.of(1, 8, 4096, 16384, 30, 128, 8)
    assert tl.workspace_size(tl.OP_LAYER_BWD_RECOMPUTE, bad) == 0
    small = tl.Dims.of(1, 8, 256, 1024, 2, 128, 2)
    p = tl.LayerParams()
    st = lib.tp_layer_fwd_nosave(ctypes.byref(small), 16, ctypes.byref(p), 16, None, 0, None)
    assert st == 1  # TP_ERR_INVALID_ARG: parameter pointers missing
    g = tl.LayerGrads()
    st = lib.tp_layer_bwd_recompute(ctypes.byref(small), 16, ctypes.byref(p), 16, 16,
                                    ctypes.byref(g), None, 0, None)
    assert st == 1


def test_selftest_limit_checked_on_host():
    lib = tl.lib()
    assert lib.tp_selftest_wait_timeout(0, None) == 1            # below 1 ms
    assert lib.tp_selftest_wait_timeout(20_000_000_000, None) == 1   # above 10 s


def test_size_limits_reported_on_host():
    lib = tl.lib()
    big = tl.Dims.of(65536, 32768, 4096, 16384, 32, 128, 8)      # batch*seq = 2^31
    assert tl.workspace_size(tl.OP_LAYER_BWD, big) == 0
    st = lib.tp_mlp_fwd(ctypes.byref(big), 16, 16, None, 16, None, None, 16, 16, 16, None, 0, None)
    assert st == 2  # TP_ERR_UNSUPPORTED
    wide = tl.Dims.of(1, 8, 16384, 65536, 128, 128, 8)             # layer LayerNorm limit
    p = tl.LayerParams()
    st = lib.tp_layer_fwd_nosave(ctypes.byref(wide), 16, ctypes.byref(p), 16, None, 0, None)
    assert st == 2


def test_layer_forward_accepts_null_activations_at_zero_tokens():
    """torch gives NULL for empty tensors: with batch*seq == 0 the layer
    forwards need no activation buffers and return before touching a device."""
    lib = tl.lib()
    d = tl.Dims.of(0, 64, 256, 1024, 2, 128, 2)
    p = tl.LayerParams(ln1_g=16, ln1_b=16, wqkv=16, wout=16, ln2_g=16, ln2_b=16, w1=16, w2=16)
    assert lib.tp_layer_fwd(ctypes.byref(d), None, ctypes.byref(p), ctypes.byref(tl.LayerActs()),
                            None, None, 0, None) == 0
    assert lib.tp_postln_layer_fwd(ctypes.byref(d), None, ctypes.byref(p),
                                   ctypes.byref(tl.PostLNActs()), None, None, 0, None) == 0
    d1 = tl.Dims.of(1, 64, 256, 1024, 2, 128, 2)   # with tokens the buffers are required
    assert lib.tp_layer_fwd(ctypes.byref(d1), None, ctypes.byref(p), ctypes.byref(tl.LayerActs()),
                            None, None, 0, None) == 1


def test_ds_limit_sizes_the_attention_backward_workspace():
    # dS^T of all heads (fp16, S rounded up to 128) is part of the attention
    # backward's workspace exactly when it fits under the limit.
    d = tl.Dims.of(2, 300, 512, 0, 4, 128, 4)
    prev = tl.attn_set_ds_limit(0)
    try:
        assert prev == 4 << 30
        without = tl.workspace_size(tl.OP_ATTN_BWD, d)
        s_pad = 384
        need = 2 * 4 * s_pad * s_pad * 2
        assert tl.attn_set_ds_limit(need) == 0
        with_ds = tl.workspace_size(tl.OP_ATTN_BWD, d)
        assert with_ds - without == need
        tl.attn_set_ds_limit(need - 1)
        assert tl.workspace_size(tl.OP_ATTN_BWD, d) == without
    finally:
        tl.attn_set_ds_limit(prev)


def test_ds_limit_enters_the_layer_backward_workspace():
    # The layer backward shares one region between the MLP and attention
    # backwards (the larger of the two); at c5 the attention part with dS^T
    # (1.07 GB) is the larger, without it the MLP's.
    d = tl.Dims.of(4, 2048, 4096, 16384, 32, 128, 8)
    prev = tl.attn_set_ds_limit(0)
    try:
        without = tl.workspace_size(tl.OP_LAYER_BWD, d)
        tl.attn_set_ds_limit(prev)
        with_ds = tl.workspace_size(tl.OP_LAYER_BWD, d)
    finally:
        tl.attn_set_ds_limit(prev)
    dst = 4 * 32 * 2048 * 2048 * 2
    assert without < with_ds <= without + dst
    assert tl.workspace_size(tl.OP_LAYER_FWD, d) > 0
