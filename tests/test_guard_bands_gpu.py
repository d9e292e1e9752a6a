"""Guard bands: no kernel writes outside the outputs it is given.

Each output is a view into the middle of a larger buffer whose margins hold a
sentinel pattern; after the call (and a sync) the margins must be unchanged.
The views are placed at awkward offsets (2-byte phases for bf16) so the ragged
row ends and the vector stores next to the buffer ends are exercised, on both
CE kernels (row kernel and ring pipeline), the forward-only and selective
outputs, the VJP and the linear cross-entropy.
"""
import numpy as np
import pytest
import torch

import gh_synth
import lm_head_cross_gh_b200 as gh
from ce_check import to_device

pytestmark = pytest.mark.gpu

GUARD = 4099  # elements of margin on each side
SENTINEL16 = 0x7BCD  # a finite bf16 pattern no kernel writes
SENTINEL32 = 123456.5


def guarded(shape, dtype, offset=0):
    n = int(np.prod(shape))
    if dtype == torch.bfloat16:
        buf = torch.full((n + 2 * GUARD + offset,), SENTINEL16, dtype=torch.int16, device="cuda")
        view = buf[GUARD + offset:GUARD + offset + n].view(torch.bfloat16).view(*shape)
    else:
        buf = torch.full((n + 2 * GUARD + offset,), SENTINEL32, dtype=dtype, device="cuda")
        view = buf[GUARD + offset:GUARD + offset + n].view(*shape)
    return buf, view, (GUARD + offset, GUARD + offset + n)


def margins_intact(buf, span, dtype):
    torch.cuda.synchronize()
    lo, hi = span
    a = buf.cpu().numpy()
    want = SENTINEL16 if dtype == torch.bfloat16 else SENTINEL32
    return bool((a[:lo] == want).all() and (a[hi:] == want).all())


@pytest.mark.parametrize("path", ["rows", "ring"])
@pytest.mark.parametrize("dtype,V,offset", [("bf16", 50257, 3), ("bf16", 9, 1), ("f32", 1025, 1), ("bf16", 262147, 5)])
def test_ce_outputs_stay_in_bounds(cuda_device, monkeypatch, path, dtype, V, offset):
    monkeypatch.setenv("GH_CE_PATH", path)
    B = 33 if V < 100000 else 3
    p = gh_synth.ce_normal(B, V, 3.0, dtype=dtype, ignore_frac=0.2, z_loss=1e-4, seed=V)
    x, t = to_device(p)
    tdt = x.dtype
    gbuf, g, gspan = guarded((B, V), tdt, offset)
    lbuf, loss, lspan = guarded((1,), torch.float32, 0)
    gh.gh_ce_fwd_bwd(x, t, p.ignore_index, "mean", 1e-4, grad=g, loss=loss.view(()))
    assert margins_intact(gbuf, gspan, tdt) and margins_intact(lbuf, lspan, torch.float32)
    rbuf, rl, rspan = guarded((B,), torch.float32, 1)
    gh.gh_ce_fwd(x, t, p.ignore_index, "sum", 0.0, row_loss=rl)
    assert margins_intact(rbuf, rspan, torch.float32)
    sbuf, sel, sspan = guarded((B,), torch.float32, 2)
    gh.gh_selective_log_softmax(x, torch.clamp(t, min=0), out=sel)
    assert margins_intact(sbuf, sspan, torch.float32)
    vbuf, vg, vspan = guarded((B, V), tdt, offset + 1)
    gh.gh_ce_vjp(x, t, rl, torch.ones(B, device="cuda"), p.ignore_index, grad=vg)
    assert margins_intact(vbuf, vspan, tdt)


def test_linear_ce_outputs_stay_in_bounds(cuda_device):
    p = gh_synth.linear_ce_normal(300, 64, 1000, chunk=128, ignore_frac=0.05, seed=1)
    X = torch.from_numpy(p.inputs.view(np.int16)).cuda().view(torch.bfloat16)
    W = torch.from_numpy(p.weight.view(np.int16)).cuda().view(torch.bfloat16)
    t = torch.from_numpy(p.targets).cuda()
    # TMA needs 16-byte aligned outputs: offsets in whole 8-element steps
    xbuf, dX, xspan = guarded(tuple(X.shape), torch.bfloat16, 8 - GUARD % 8)
    wbuf, dW, wspan = guarded(tuple(W.shape), torch.bfloat16, 8 - GUARD % 8)
    for accum in ("fp32", "weight"):
        gh.gh_linear_ce(X, W, t, -100, "mean", 1e-4, 128, accum, grad_inputs=dX, grad_weight=dW)
        assert margins_intact(xbuf, xspan, torch.bfloat16) and margins_intact(wbuf, wspan, torch.bfloat16)
