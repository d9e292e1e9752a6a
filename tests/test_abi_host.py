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


def test_newer_entry_points_reject_bad_arguments_on_host(L):
    bad = gh.GH_ERR_INVALID_ARG
    lg, tg, out = FAKE, FAKE + (1 << 32), FAKE + (2 << 32)
    # gh_ce_fwd
    assert L.gh_ce_fwd(lg, tg, -1, 100, gh.GH_BF16, -100, 0, 0.0, out, None, None) == bad
    assert L.gh_ce_fwd(lg, tg, 16, 100, gh.GH_BF16, -100, 0, 0.0, None, None, None) == bad
    assert L.gh_ce_fwd(lg, tg, 16, 100, gh.GH_BF16, -100, 0, 0.0, out, out + 2, None) == bad  # row_loss misaligned
    # gh_selective_log_softmax
    assert L.gh_selective_log_softmax(lg, tg, 16, 0, gh.GH_BF16, out, None) == bad
    assert L.gh_selective_log_softmax(lg, None, 16, 100, gh.GH_BF16, out, None) == bad
    assert L.gh_selective_log_softmax(lg, tg, 16, 100, 9, out, None) == bad
    # gh_ce_vjp
    assert L.gh_ce_vjp(lg, tg, 16, 100, gh.GH_BF16, -100, None, out, FAKE + (3 << 32), None) == bad
    assert L.gh_ce_vjp(lg, tg, 16, 100, gh.GH_BF16, -100, out, out, lg + 64, None) == bad  # partial overlap
    # gh_count_valid
    assert L.gh_count_valid(tg, -1, 100, -100, out, None) == bad
    assert L.gh_count_valid(tg, 16, 100, -100, out + 4, None) == bad
    # shard entry points need an aligned total count
    assert L.gh_ce_fwd_bwd_shard(lg, tg, 16, 100, gh.GH_BF16, -100, 0, 0.0, None, out, FAKE + (3 << 32),
                                 None) == bad
    assert L.gh_linear_ce_shard(lg, FAKE + (4 << 32), tg, 64, 64, 100, 0, 0, -100, 0, 0.0, out + 4, out,
                                FAKE + (5 << 32), FAKE + (6 << 32), None) == bad
    # gh_chunked_linear_loss needs a callback
    assert L.gh_chunked_linear_loss(lg, FAKE + (4 << 32), 64, 64, 100, 0, 0, gh.CHUNK_LOSS_FN(), None, out,
                                    FAKE + (5 << 32), FAKE + (6 << 32), None) == bad


def test_plain_c_program_uses_the_header_and_library(L, tmp_path):
    """include/gh.h compiles as C99 with warnings as errors, and a C program
    linked against libgh.so gets every host-side refusal the header promises
    (tests/abi_c_check.c), with no GPU and no Python in between."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc") or shutil.which("cc")
    if gcc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(gh.LIB_PATH)
    exe = str(tmp_path / "abi_c_check")
    build = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                            "-I", os.path.join(root, "include"), os.path.join(root, "tests", "abi_c_check.c"),
                            "-o", exe, "-L", libdir, "-lgh", "-Wl,-rpath," + libdir, "-lm"],
                           capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "0 failed checks" in run.stdout
