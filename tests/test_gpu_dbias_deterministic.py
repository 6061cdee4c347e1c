"""GPU: masked_attn_bwd_deterministic gives dbias that is bitwise the same on
every call and agrees with the float64 oracle's reduction onto the bias
shape, for every way a bias broadcasts (batch, a group's heads or all heads,
the queries), on the tensor-core kernels (head dim 64 and 128) and the fp32
kernels; and the partial-sum workspace is checked before anything runs."""
import numpy as np
import pytest
import torch

import structured_mask_attention_analytic_b200 as sma
import workloads as wl
from oracle import attention as at
from oracle import attention_grad as ag
from tests._helpers import f64

pytestmark = pytest.mark.gpu

B, H, KVH, LQ, LK = 2, 8, 2, 300, 400
KP = 512  # key dim of the bias, 128-rounded
# Gradient agreement as in the other backward tests: relative to m = max(1,
# max |ref|), max-abs <= 2.5e-2 m and mean-abs <= 2.5e-3 m (bf16 operands),
# 1e-4 m / 1e-5 m for fp32 operands.
TOL = {"bf16": (2.5e-2, 2.5e-3), "fp32": (1e-4, 1e-5)}

SHAPES = [(B, KVH, 1, KP), (B, H, 1, KP), (1, 1, 1, KP), (1, KVH, LQ, KP), (B, 1, LQ, KP),
          (B, H, LQ, KP)]


def _close(name, got, ref, dtype):
    g = f64(got)
    m = max(1.0, float(np.abs(ref).max()))
    err = np.abs(g - ref)
    tmax, tmean = TOL[dtype]
    assert np.isfinite(g).all(), f"{name}: non-finite"
    assert err.max() <= tmax * m, f"{name}: max abs err {err.max():.3e} (scale {m:.2f})"
    assert err.mean() <= tmean * m, f"{name}: mean abs err {err.mean():.3e} (scale {m:.2f})"


@pytest.mark.parametrize("bshape", SHAPES, ids=str)
@pytest.mark.parametrize("D,dtype", [(128, "bf16"), (64, "bf16"), (64, "fp32")])
def test_deterministic_dbias(bshape, D, dtype):
    rng = wl.rng_for(71)
    q = wl.normal(rng, (B, LQ, H, D), dtype)
    k = wl.normal(rng, (B, LK, KVH, D), dtype)
    v = wl.normal(rng, (B, LK, KVH, D), dtype)
    do = wl.normal(rng, (B, LQ, H, D), dtype)
    mask = torch.from_numpy(rng.random((B, KVH, 1, KP)) < 0.8)
    bias = wl.normal(rng, bshape, dtype)
    qc, kc, vc, dc, mc, bc = (t.cuda() for t in (q, k, v, do, mask, bias))
    out, lse = sma.masked_attn_fwd(qc, kc, vc, mc, bc, True)
    dbs = []
    for _ in range(3):
        dq, dk, dv, db = sma.masked_attn_bwd(qc, kc, vc, out, lse, dc, mc, bc, True, return_dbias=True,
                                             deterministic=True)
        dbs.append(db.clone())
    torch.cuda.synchronize()
    assert sma.device_status() == 0
    for other in dbs[1:]:
        assert torch.equal(dbs[0], other), "dbias differs between calls"
    keep = at.aux_view(mask.numpy(), H, KVH, LK) & at.causal_keep(LQ, LK)[None, None]
    bb = at.aux_view(f64(bias), H, KVH, LK)
    rq, rk, rv, rdb = ag.attention_grad(f64(q), f64(k), f64(v), f64(do), keep=keep, bias=bb,
                                        dbias_shape=bshape, workers=8)
    _close("dbias", dbs[0], rdb, dtype)
    _close("dq", dq, rq, dtype)
    _close("dk", dk, rk, dtype)
    assert (dbs[0][..., LK:] == 0).all()


def test_partial_workspace_too_small_is_rejected():
    rng = wl.rng_for(72)
    q = wl.normal(rng, (B, LQ, H, 128), "bf16").cuda()
    k = wl.normal(rng, (B, LK, KVH, 128), "bf16").cuda()
    v = wl.normal(rng, (B, LK, KVH, 128), "bf16").cuda()
    do = wl.normal(rng, (B, LQ, H, 128), "bf16").cuda()
    bias = wl.normal(rng, (B, KVH, 1, KP), "bf16").cuda()
    out, lse = sma.masked_attn_fwd(q, k, v, None, bias, False)
    need = sma.masked_attn_bwd_dbias_workspace_size(torch.bfloat16, B, H, KVH, LQ, 128, list(bias.shape))
    assert need == B * H * ((LQ + 63) // 64) * KP * 4
    small = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError, match="workspace"):
        sma.masked_attn_bwd(q, k, v, out, lse, do, None, bias, False, return_dbias=True, deterministic=True,
                            dbias_workspace=small)
    torch.cuda.synchronize()
    assert sma.device_status() == 0
