"""The data-parallel cross-entropy's collective steps on two gloo ranks (CPU).

Each rank holds half of a batch.  The library's shard entry points are
replaced by float64 PyTorch stand-ins with the same contract (count the valid
targets; divide by the total count passed in), so what runs here is exactly
the wrapper's sequence of all-reduces: the valid counts summed before the
shard call, the losses and the weight gradients summed after it.  Every rank
must then hold the full batch's mean loss, its own rows of the full batch's
input/logits gradient, and the full weight gradient.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _HostOps:
    """float64 stand-ins for gh_count_valid / gh_ce_fwd_bwd_shard / gh_linear_ce_shard."""

    @staticmethod
    def gh_count_valid(t, V, ii):
        return torch.tensor((t != ii).sum().item(), dtype=torch.int64)

    @staticmethod
    def _rows(x, t, ii, z):
        valid = t != ii
        tt = torch.where(valid, t, torch.zeros_like(t))
        lse = torch.logsumexp(x, dim=1)
        rl = torch.where(valid, lse - x.gather(1, tt[:, None])[:, 0] + z * lse * lse, torch.zeros_like(lse))
        g = torch.softmax(x, dim=1) * (1 + 2 * z * lse)[:, None]
        g[torch.arange(x.shape[0]), tt] -= 1.0
        return rl, g * valid[:, None]

    @classmethod
    def gh_ce_fwd_bwd_shard(cls, x, t, n, ii, reduction, z):
        rl, g = cls._rows(x, t, ii, z)
        scale = 1.0 / max(int(n), 1) if reduction == "mean" else 1.0
        return (rl.sum() * scale).reshape(()), g * scale

    @classmethod
    def gh_linear_ce_shard(cls, X, W, t, n, ii, reduction, z, chunk, accum):
        loss, G = cls.gh_ce_fwd_bwd_shard(X @ W.T, t, n, ii, reduction, z)
        return loss, G @ W, G.T @ X

    slices_seen = []

    @classmethod
    def gh_linear_ce_shard_f32(cls, X, W, t, n, ii, reduction, z, chunk, *, grad_weight_f32=None,
                               on_slice=None, dw_slices=1, max_sms=0):
        """bf16 inputs; the shard's weight gradient as an unrounded fp32 sum.
        With on_slice: the rows of the gradient handed over in dw_slices
        consecutive ranges, in order, once each range is written."""
        X64, W64 = X.double(), W.double()
        loss, G = cls.gh_ce_fwd_bwd_shard(X64 @ W64.T, t, n, ii, reduction, z)
        dW = (G.T @ X64).float()
        if grad_weight_f32 is None:
            grad_weight_f32 = dW
        else:
            grad_weight_f32.copy_(dW)
        if on_slice is not None:
            V = W.shape[0]
            k = min(dw_slices, V)
            for s in range(k):
                v0, v1 = V * s // k, V * (s + 1) // k
                cls.slices_seen.append((v0, v1))
                on_slice(v0, v1)
        return loss.float(), (G @ W64).to(X.dtype), grad_weight_f32

    @staticmethod
    def gh_cast_f32_to_bf16(src):
        return src.to(torch.bfloat16)


def _batch(seed=0, N=24, D=6, V=17):
    g = torch.Generator().manual_seed(seed)
    X = torch.randn(N, D, generator=g, dtype=torch.float64)
    W = torch.randn(V, D, generator=g, dtype=torch.float64) * 0.3
    t = torch.randint(0, V, (N,), generator=g)
    t[::5] = -100
    t[1] = -100  # more ignored rows on rank 0 than on rank 1
    return X, W, t


def _plain(t):
    """A tensor as a numpy copy for the result queue: a torch tensor put on a
    multiprocessing queue travels as a shared file descriptor, which the
    parent can no longer fetch once the rank has exited."""
    return t.detach().float().numpy().copy() if t.dtype == torch.bfloat16 else t.detach().numpy().copy()


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    from lm_head_cross_gh_b200 import functional as GF
    dist.init_process_group("gloo", rank=rank, world_size=world)
    X, W, t = _batch()
    rows = slice(rank * 12, (rank + 1) * 12)
    # standalone CE on the logits shard
    logits = (X @ W.T)[rows].clone().requires_grad_(True)
    loss = GF.data_parallel_cross_entropy(logits, t[rows], -100, "mean", 1e-3, ops=_HostOps)
    loss.backward()
    # linear CE with a replicated weight
    Xs = X[rows].clone().requires_grad_(True)
    Wr = W.clone().requires_grad_(True)
    lin = GF.data_parallel_chunked_linear_cross_entropy(Xs, Wr, t[rows], -100, "mean", 1e-3,
                                                        grad_weight_accum_dtype="weight", ops=_HostOps)
    lin.backward()
    out.put((rank, loss.item(), _plain(logits.grad), lin.item(), _plain(Xs.grad), _plain(Wr.grad)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_data_parallel_cross_entropy():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the full batch on one process, same stand-in arithmetic
    X, W, t = _batch()
    Xf, Wf = X.clone().requires_grad_(True), W.clone().requires_grad_(True)
    n = int((t != -100).sum())
    lf, Gf = _HostOps.gh_ce_fwd_bwd_shard(X @ W.T, t, n, -100, "mean", 1e-3)
    for rank, loss, glog, lin, gx, gw in res:
        glog, gx, gw = torch.from_numpy(glog), torch.from_numpy(gx), torch.from_numpy(gw)
        rows = slice(rank * 12, (rank + 1) * 12)
        assert loss == pytest.approx(lf.item(), rel=1e-12)
        assert torch.allclose(glog, Gf[rows], rtol=1e-12, atol=1e-15)
        assert lin == pytest.approx(lf.item(), rel=1e-12)
        assert torch.allclose(gx, (Gf @ W)[rows], rtol=1e-10, atol=1e-13)
        assert torch.allclose(gw, Gf.T @ X, rtol=1e-10, atol=1e-13)


def _rank_main_fp32(rank, world, port, out):
    """bf16 inputs and weight with fp32 weight-gradient accumulation: each rank's
    fp32 accumulator is all-reduced in fp32 and the sum rounded once."""
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    from lm_head_cross_gh_b200 import functional as GF
    dist.init_process_group("gloo", rank=rank, world_size=world)
    X, W, t = _batch(seed=3, N=40, D=16, V=33)
    rows = slice(rank * 20, (rank + 1) * 20)
    Xs = X[rows].to(torch.bfloat16).requires_grad_(True)
    Wr = W.to(torch.bfloat16).requires_grad_(True)
    lin = GF.data_parallel_chunked_linear_cross_entropy(Xs, Wr, t[rows], -100, "mean", 1e-3,
                                                        grad_weight_accum_dtype="fp32", ops=_HostOps,
                                                        overlap_slices=3)
    lin.backward()
    out.put((rank, lin.item(), str(Wr.grad.dtype), _plain(Wr.grad), list(_HostOps.slices_seen)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_fp32_weight_gradient_is_rounded_once():
    """'fp32' accumulation across ranks: the weight gradient every rank holds is
    bf16(fp32 partial of rank 0 + fp32 partial of rank 1), one rounding of the
    fp32 sum, not a sum of bf16-rounded partials."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main_fp32, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    X, W, t = _batch(seed=3, N=40, D=16, V=33)
    Xb, Wb = X.to(torch.bfloat16), W.to(torch.bfloat16)
    n = torch.tensor(int((t != -100).sum()))
    parts = [_HostOps.gh_linear_ce_shard_f32(Xb[r * 20:(r + 1) * 20], Wb, t[r * 20:(r + 1) * 20], n, -100, "mean",
                                             1e-3, 0)[2] for r in range(2)]
    once = (parts[0] + parts[1]).to(torch.bfloat16)
    twice = (parts[0].to(torch.bfloat16) + parts[1].to(torch.bfloat16))
    assert not torch.equal(once, twice)  # the two readings differ on this batch
    for rank, lin, gw_dtype, gw, seen in res:
        assert gw_dtype == str(torch.bfloat16)
        gw = torch.from_numpy(gw).to(torch.bfloat16)  # bf16 -> fp32 -> bf16 is exact
        # every range of weight rows was summed over the ranks (each by its own
        # asynchronous all-reduce) before the single rounding
        assert seen == [(0, 11), (11, 22), (22, 33)], rank
        assert torch.equal(gw, once), rank
