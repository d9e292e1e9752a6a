"""Host-only checks of the C ABI: the library loads, exports every function the
header declares, and rejects bad arguments before touching the GPU."""
import ctypes
import os

import pytest

import lm_head_cross_gh_b200 as gh


@pytest.fixture(scope="module")
def L():
    from lm_head_cross_gh_b200 import _build
    _build.build()
    return gh.lib()


def test_every_declared_symbol_is_exported(L):
    names = gh.header_symbols()
    assert set(names) >= {"gh_ce_fwd_bwd", "gh_linear_ce", "gh_get_device_status", "gh_status_string",
                          "gh_version"}
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/gh.h but not exported"


def test_status_strings_and_version(L):
    assert gh.gh_version().startswith("gh ")
    seen = set()
    for code in range(7):
        s = gh.status_string(code)
        assert s and s != "unknown status"
        seen.add(s)
    assert len(seen) == 7
    assert gh.status_string(99) == "unknown status"


FAKE = 0x7F0000000000  # a well-aligned non-null address; never dereferenced


@pytest.mark.parametrize("kw,expect", [
    (dict(B=-1), gh.GH_ERR_INVALID_ARG),
    (dict(V=0), gh.GH_ERR_INVALID_ARG),
    (dict(V=1 << 31), gh.GH_ERR_INVALID_ARG),
    (dict(dtype=7), gh.GH_ERR_INVALID_ARG),
    (dict(reduction=5), gh.GH_ERR_INVALID_ARG),
    (dict(z=float("nan")), gh.GH_ERR_INVALID_ARG),
    (dict(z=float("inf")), gh.GH_ERR_INVALID_ARG),
    (dict(logits=None), gh.GH_ERR_INVALID_ARG),
    (dict(targets=None), gh.GH_ERR_INVALID_ARG),
    (dict(grad=None), gh.GH_ERR_INVALID_ARG),
    (dict(loss=None), gh.GH_ERR_INVALID_ARG),
    (dict(logits=FAKE + 1), gh.GH_ERR_INVALID_ARG),         # misaligned for bf16
    (dict(targets=FAKE + 4), gh.GH_ERR_INVALID_ARG),        # int64 misaligned
    (dict(grad=FAKE + 64), gh.GH_ERR_INVALID_ARG),          # partial overlap with logits
])
def test_ce_rejects_bad_arguments_on_host(L, kw, expect):
    a = dict(logits=FAKE, targets=FAKE + (1 << 32), B=16, V=100, dtype=gh.GH_BF16, ii=-100, reduction=0,
             z=0.0, loss=FAKE + (2 << 32), grad=FAKE + (3 << 32))
    a.update(kw)
    st = L.gh_ce_fwd_bwd(a["logits"], a["targets"], a["B"], a["V"], a["dtype"], a["ii"], a["reduction"],
                         a["z"], a["loss"], a["grad"], None)
    assert st == expect


@pytest.mark.parametrize("kw", [
    dict(N=-1), dict(D=0), dict(D=12), dict(V=0), dict(accum=3), dict(reduction=2), dict(z=float("nan")),
    dict(inputs=None), dict(weight=None), dict(targets=None), dict(loss=None), dict(dX=None), dict(dW=None),
    dict(inputs=FAKE + 8), dict(weight=FAKE + 2),
])
def test_linear_ce_rejects_bad_arguments_on_host(L, kw):
    a = dict(inputs=FAKE, weight=FAKE + (1 << 32), targets=FAKE + (2 << 32), N=64, D=64, V=100, chunk=0,
             accum=0, ii=-100, reduction=0, z=0.0, loss=FAKE + (3 << 32), dX=FAKE + (4 << 32),
             dW=FAKE + (5 << 32))
    a.update(kw)
    st = L.gh_linear_ce(a["inputs"], a["weight"], a["targets"], a["N"], a["D"], a["V"], a["chunk"],
                        a["accum"], a["ii"], a["reduction"], a["z"], a["loss"], a["dX"], a["dW"], None)
    assert st == gh.GH_ERR_INVALID_ARG


def test_python_binding_validates_before_calling():
    import torch
    x = torch.zeros(4, 8)
    t = torch.zeros(4, dtype=torch.int64)
    with pytest.raises(ValueError):
        gh.gh_ce_fwd_bwd(x, t)  # CPU tensors are refused; no CPU fallback exists
