"""The workspace-free LayerNorm backward against the workspace entry point.

tp_layernorm_bwd_noalloc exists for callers that cannot allocate device
memory where they run the backward (allocator callbacks, fixed memory
budgets); its scratch is a static array inside the library, shared by every
call on a device.  Two calls in a row, with different inputs, must each match
tp_layernorm_bwd within the tolerance the parity tests use, so that nothing a
call leaves in the shared array leaks into the next one.
"""
import numpy as np
import pytest
import torch

import tensor_transformer_layer_column_b200 as tl
from parity import check

pytestmark = pytest.mark.gpu


def _inputs(rows, D, seed):
    g = torch.Generator().manual_seed(seed)
    bf = torch.bfloat16
    x = (torch.randn(rows, D, generator=g) * 1.5 + 0.3).to(bf).cuda()
    gam = (1 + 0.1 * torch.randn(D, generator=g)).to(bf).cuda()
    bet = (0.1 * torch.randn(D, generator=g)).to(bf).cuda()
    dy = torch.randn(rows, D, generator=g).to(bf).cuda()
    dres = torch.randn(rows, D, generator=g).to(bf).cuda()
    y = torch.empty_like(x)
    mean = torch.empty(rows, dtype=torch.float32, device="cuda")
    rstd = torch.empty_like(mean)
    tl.layernorm_fwd(x, gam, bet, rows, D, 1e-5, y, mean, rstd)
    return x, gam, dy, dres, mean, rstd


def _f64(t):
    return t.to(torch.float64).cpu().numpy()


@pytest.mark.parametrize("rows,D", [(8192, 4096), (1000, 8192)])
def test_noalloc_matches_workspace_entry_point_twice(rows, D):
    if not torch.cuda.is_available() or torch.cuda.get_device_capability()[0] != 10:
        pytest.skip("needs an sm_100 device")
    for call, seed in enumerate((1, 2)):
        x, gam, dy, dres, mean, rstd = _inputs(rows, D, seed)
        dx_a, dg_a, db_a = torch.empty_like(x), torch.empty_like(gam), torch.empty_like(gam)
        ws = torch.empty(tl.layernorm_bwd_workspace_size(rows, D), dtype=torch.uint8,
                         device="cuda")
        tl.layernorm_bwd(dy, x, gam, mean, rstd, dres, rows, D, dx_a, dg_a, db_a, ws)
        dx_b, dg_b, db_b = torch.empty_like(x), torch.empty_like(gam), torch.empty_like(gam)
        tl.layernorm_bwd_noalloc(dy, x, gam, mean, rstd, dres, rows, D, dx_b, dg_b, db_b)
        torch.cuda.synchronize()
        assert tl.check_error() == 0
        check(f"dx (call {call})", dx_b, _f64(dx_a))
        check(f"dgamma (call {call})", dg_b, _f64(dg_a))
        check(f"dbeta (call {call})", db_b, _f64(db_a))


def test_noalloc_rejects_rows_wider_than_its_limit():
    if not torch.cuda.is_available() or torch.cuda.get_device_capability()[0] != 10:
        pytest.skip("needs an sm_100 device")
    st = tl.lib().tp_layernorm_bwd_noalloc(16, 16, 16, 16, 16, None, 4, 8200, 16, None, None, None)
    assert st == 2   # TP_ERR_UNSUPPORTED: D beyond 8192
