"""The workspace-free LayerNorm backward against the workspace entry point.

tp_layernorm_bwd_noalloc exists for callers that cannot allocate device
memory where they run the backward (allocator callbacks, fixed memory
budgets); its scratch is a static array inside the library, shared by every
call on a device.  Two calls in a row, with different inputs, must each give
the same dx as tp_layernorm_bwd bit for bit, and dgamma / dbeta within the
parity tolerance of the fp64 oracle, so that nothing a call leaves in the
shared array leaks into the next one.
"""
import pytest
import torch

import tensor_transformer_layer_column_b200 as tl
from oracle import core as ocore
from parity import check

pytestmark = pytest.mark.gpu


def _require_gpu():
    if not torch.cuda.is_available() or torch.cuda.get_device_capability()[0] != 10:
        pytest.skip("needs an sm_100 device")


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
    if rows:
        tl.layernorm_fwd(x, gam, bet, rows, D, 1e-5, y, mean, rstd)
    return x, gam, dy, dres, mean, rstd


def _f64(t):
    return t.to(torch.float64).cpu().numpy()


@pytest.mark.parametrize("rows,D", [(8192, 4096), (1000, 8192), (300, 1024)])
def test_noalloc_matches_workspace_entry_point_twice(rows, D):
    _require_gpu()
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
        # dx depends on one row only: the same kernel arithmetic, bit for bit.
        assert torch.equal(dx_b, dx_a), f"dx differs from tp_layernorm_bwd (call {call})"
        # dgamma / dbeta against the fp64 oracle, from the same mean and rstd.
        _, dg_r, db_r = ocore.layernorm_bwd(_f64(dy), _f64(x), _f64(gam), _f64(mean), _f64(rstd))
        check(f"dgamma (call {call})", dg_b, dg_r)
        check(f"dbeta (call {call})", db_b, db_r)
        if D * 2 * tl_blocks(rows) <= (1 << 20):
            # Both paths group rows alike while the array holds every block.
            assert torch.equal(dg_b, dg_a) and torch.equal(db_b, db_a)


def tl_blocks(rows):
    """Row blocks of the LayerNorm backward: 2 per SM, at most one per row."""
    return max(1, min(rows, 2 * torch.cuda.get_device_properties(0).multi_processor_count))


def test_noalloc_zero_rows_zeroes_the_parameter_gradients():
    _require_gpu()
    D = 512
    x, gam, dy, dres, mean, rstd = _inputs(8, D, 3)
    dg = torch.full_like(gam, 7.0)
    db = torch.full_like(gam, 7.0)
    dx = torch.empty_like(x)
    tl.layernorm_bwd_noalloc(dy, x, gam, mean, rstd, None, 0, D, dx, dg, db)
    torch.cuda.synchronize()
    assert tl.check_error() == 0
    assert not dg.any() and not db.any()


def test_noalloc_rejects_rows_wider_than_its_limit():
    _require_gpu()
    st = tl.lib().tp_layernorm_bwd_noalloc(16, 16, 16, 16, 16, None, 4, 8200, 16, None, None, None)
    assert st == 2   # TP_ERR_UNSUPPORTED: D beyond 8192
