"""Parity of the CUDA LayerNorm (pre-LN building block) with the fp64 oracle."""
import numpy as np
import pytest
import torch

import tensor_transformer_layer_column_b200 as tl
from gpu_util import require_gpu
from oracle import core
from parity import check

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows,D", [(1, 256), (333, 1024), (1000, 4096), (64, 8192), (257, 264)])
def test_layernorm_fwd_bwd(rows, D):
    require_gpu()
    g = torch.Generator().manual_seed(rows + D)
    bf = torch.bfloat16
    x = (torch.randn(rows, D, generator=g) * 2 + 0.5).to(bf)
    gam = (1 + 0.1 * torch.randn(D, generator=g)).to(bf)
    bet = (0.1 * torch.randn(D, generator=g)).to(bf)
    dy = torch.randn(rows, D, generator=g).to(bf)
    dres = torch.randn(rows, D, generator=g).to(bf)
    xd, gd, bd, dyd, drd = (v.cuda() for v in (x, gam, bet, dy, dres))
    y = torch.empty_like(xd)
    mean = torch.empty(rows, dtype=torch.float32, device="cuda")
    rstd = torch.empty_like(mean)
    tl.layernorm_fwd(xd, gd, bd, rows, D, 1e-5, y, mean, rstd)
    f = lambda v: v.to(torch.float64).numpy()
    yr, mr, rr = core.layernorm_fwd(f(x), f(gam), f(bet), 1e-5)
    check("y", y, yr)
    check("mean", mean, mr)
    check("rstd", rstd, rr)
    ws = torch.empty(tl.layernorm_bwd_workspace_size(rows, D), dtype=torch.uint8, device="cuda")
    dx = torch.empty_like(xd)
    dg = torch.empty_like(gd)
    db = torch.empty_like(bd)
    tl.layernorm_bwd(dyd, xd, gd, mean, rstd, drd, rows, D, dx, dg, db, ws)
    dxr, dgr, dbr = core.layernorm_bwd(f(dy), f(x), f(gam), mr, rr)
    check("dx", dx, dxr + f(dres))
    check("dgamma", dg, dgr)
    check("dbeta", db, dbr)
    assert tl.check_error() == 0


@pytest.mark.parametrize("rows,D,offset", [(300, 4096, 0.0), (77, 1000, 100.0), (5, 8192, -30.0)])
def test_layernorm_fwd_f16_output_and_offset_rows(rows, D, offset):
    """tp_layernorm_fwd_f16 (the fp16 output that feeds the attention
    products) against the oracle, on rows whose mean is far from zero: the
    per-thread mean / M2 combination must not lose the variance to
    cancellation."""
    require_gpu()
    g = torch.Generator().manual_seed(rows * 7 + D)
    bf = torch.bfloat16
    x = (torch.randn(rows, D, generator=g) + offset).to(bf)
    gam = (1 + 0.1 * torch.randn(D, generator=g)).to(bf)
    bet = (0.1 * torch.randn(D, generator=g)).to(bf)
    y = torch.empty(rows, D, dtype=torch.float16, device="cuda")
    mean = torch.empty(rows, dtype=torch.float32, device="cuda")
    rstd = torch.empty_like(mean)
    tl.layernorm_fwd_f16(x.cuda(), gam.cuda(), bet.cuda(), rows, D, 1e-5, y, mean, rstd)
    f = lambda v: v.to(torch.float64).numpy()
    yr, mr, rr = core.layernorm_fwd(f(x), f(gam), f(bet), 1e-5)
    check("y", y, yr)
    check("mean", mean, mr)
    check("rstd", rstd, rr)
    assert tl.check_error() == 0
