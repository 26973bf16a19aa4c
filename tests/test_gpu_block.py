"""The full Naju block (norm, projections, conv, scan, modulation, residual)
against the fp64 block oracle: forward output, input gradient and every
parameter gradient (fp32 activations; the GEMMs are torch fp32)."""
import numpy as np
import pytest
import torch

from discrete_selective_ssm_b200.block import NajuBlock, init_params
from oracle import block as ob
from naju_check import TOL_F32, assert_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("coupled", [False, True])
@pytest.mark.parametrize("N", [16, 64])
def test_block_parity(coupled, N):
    Bt, L, dm, di = 2, 150, 48, 72
    params = init_params(dm, di, N, seed=5 + N)
    blk = NajuBlock(dm, di, N, "cuda", dtype=torch.float32, params=params, coupled=coupled)
    gen = torch.Generator().manual_seed(6)
    x = torch.randn(Bt, L, dm, generator=gen)
    dout = torch.randn(Bt, L, dm, generator=gen)
    out, ctx = blk.forward(x.cuda())
    dx, g = blk.backward(ctx, dout.cuda())
    torch.cuda.synchronize()
    ro, cache = ob.block_fwd(x.numpy(), {k: v.numpy() for k, v in params.items()}, coupled)
    rdx, rg = ob.block_bwd(cache, dout.numpy(), coupled)
    assert_close(out, ro, TOL_F32, name="out")
    assert_close(dx, rdx, TOL_F32, name="dx")
    for k in ob.PARAMS:
        if coupled and k in ("W_b", "b_b"):
            assert float(g[k].abs().max()) == 0.0
            continue
        assert_close(g[k], rg[k], TOL_F32, name=k)
