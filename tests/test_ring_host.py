"""Ring (context-parallel) attention: the schedule and the exchanges over gloo ranks on CPU.

The ring driver (exact_attention_159_b200/ring.py) is run by 2 and 3 gloo ranks with an fp64
CPU stand-in for the per-chunk kernels (test infrastructure, below): the stand-in computes
each chunk's attention with the oracle, and the chunk backward from the definition with the
rows' global LSE and D.  What is checked is the ring itself -- which chunk each rank holds
at each step, which blocks the causal mask skips, the log-sum-exp merge and the return of
the dK / dV accumulators to their owners -- against the oracle on the whole sequence, to
fp64 rounding.  The kernels are checked on their own by the GPU tests.
"""
import os

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import oracle as OR


class Fp64Backend:
    """The per-chunk steps in fp64 on CPU (tensors B x H x n x d, float64)."""

    def fwd(self, q, k, v, scale, causal):
        B, H = q.shape[:2]
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:-1], dtype=torch.float64)
        for b in range(B):
            for h in range(H):
                ob, lb = OR.fwd(q[b, h].numpy(), k[b, h].numpy(), v[b, h].numpy(), scale, causal, nthreads=1)
                o[b, h] = torch.from_numpy(ob)
                lse[b, h] = torch.from_numpy(lb)
        return o, lse

    def bwd(self, q, k, v, o, do, lse, scale, causal):
        # the chunk's share of the gradients, P from the rows' global LSE and D from the global O
        s = scale * torch.einsum("bhid,bhjd->bhij", q, k)
        if causal:
            n = q.shape[2]
            s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), -float("inf"))
        p = torch.exp(s - lse[..., None])
        dp = torch.einsum("bhid,bhjd->bhij", do, v)
        dsum = (do * o).sum(-1, keepdim=True)
        ds = p * (dp - dsum)
        return (scale * torch.einsum("bhij,bhjd->bhid", ds, k), scale * torch.einsum("bhij,bhid->bhjd", ds, q),
                torch.einsum("bhij,bhid->bhjd", p, do))

    def merge(self, o_part, lse_part, o_acc, lse_acc, first):
        if first:
            o_acc.copy_(o_part)
            lse_acc.copy_(lse_part)
            return
        l_new = torch.logaddexp(lse_acc, lse_part)
        o_acc.copy_(torch.exp(lse_acc - l_new)[..., None] * o_acc + torch.exp(lse_part - l_new)[..., None] * o_part)
        lse_acc.copy_(l_new)

    def accumulate(self, acc, x, first):
        if first:
            acc.copy_(x)
        else:
            acc.add_(x)

    def to_bf16(self, x):
        return x.clone()

    def f32_like(self, t):
        return torch.empty(t.shape, dtype=torch.float64)

    def lse_like(self, q):
        return torch.empty(q.shape[:-1], dtype=torch.float64)


def _inputs(B, H, N, d, seed):
    r = np.random.default_rng(seed)
    return [torch.from_numpy(r.standard_normal((B, H, N, d))) for _ in range(4)]  # q, k, v, do


def _worker(rank, world, port, causal, out):
    import torch.distributed as dist
    from exact_attention_159_b200 import ring
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, n, d = 1, 2, 8, 8
        q, k, v, do = _inputs(B, H, n * world, d, seed=7)
        sl = slice(rank * n, (rank + 1) * n)
        qc, kc, vc, doc = (t[:, :, sl].contiguous() for t in (q, k, v, do))
        be = Fp64Backend()
        o, lse = ring.ring_attention_fwd(qc, kc, vc, 0.4, causal, backend=be)
        dq, dk, dv = ring.ring_attention_bwd(qc, kc, vc, o, doc, lse, 0.4, causal, backend=be)
        out[rank] = [t.numpy() for t in (o, lse, dq, dk, dv)]
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_over_gloo_matches_oracle(world, causal):
    ctx = mp.get_context("spawn")
    port = 29600 + (os.getpid() % 300) + 10 * world + int(causal)
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, causal, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    B, H, n, d = 1, 2, 8, 8
    q, k, v, do = (t.numpy() for t in _inputs(B, H, n * world, d, seed=7))
    for h in range(H):
        o_ref, l_ref = OR.fwd(q[0, h], k[0, h], v[0, h], 0.4, causal, nthreads=1)
        dq_ref, dk_ref, dv_ref, _, _ = OR.bwd(q[0, h], k[0, h], v[0, h], do[0, h], 0.4, causal, nthreads=1)
        for r in range(world):
            sl = slice(r * n, (r + 1) * n)
            o, lse, dq, dk, dv = res[r]
            np.testing.assert_allclose(o[0, h], o_ref[sl], atol=1e-12)
            np.testing.assert_allclose(lse[0, h], l_ref[sl], atol=1e-12)
            np.testing.assert_allclose(dq[0, h], dq_ref[sl], atol=1e-11)
            np.testing.assert_allclose(dk[0, h], dk_ref[sl], atol=1e-11)
            np.testing.assert_allclose(dv[0, h], dv_ref[sl], atol=1e-11)


def test_emulated_ring_matches_oracle():
    # the single-process emulation runs the same per-rank steps
    from exact_attention_159_b200 import ring
    world, B, H, n, d = 4, 1, 2, 6, 8
    q, k, v, do = _inputs(B, H, n * world, d, seed=9)
    chunks = [[t[:, :, r * n:(r + 1) * n].contiguous() for r in range(world)] for t in (q, k, v, do)]
    be = Fp64Backend()
    for causal in (False, True):
        os_, lses = ring.ring_attention_fwd_emulated(chunks[0], chunks[1], chunks[2], 0.3, causal, backend=be)
        dqs, dks, dvs = ring.ring_attention_bwd_emulated(chunks[0], chunks[1], chunks[2], os_, chunks[3], lses, 0.3,
                                                         causal, backend=be)
        for h in range(H):
            o_ref, l_ref = OR.fwd(q[0, h].numpy(), k[0, h].numpy(), v[0, h].numpy(), 0.3, causal, nthreads=1)
            dq_ref, dk_ref, dv_ref, _, _ = OR.bwd(q[0, h].numpy(), k[0, h].numpy(), v[0, h].numpy(),
                                                  do[0, h].numpy(), 0.3, causal, nthreads=1)
            for r in range(world):
                sl = slice(r * n, (r + 1) * n)
                np.testing.assert_allclose(os_[r][0, h].numpy(), o_ref[sl], atol=1e-12)
                np.testing.assert_allclose(lses[r][0, h].numpy(), l_ref[sl], atol=1e-12)
                np.testing.assert_allclose(dqs[r][0, h].numpy(), dq_ref[sl], atol=1e-11)
                np.testing.assert_allclose(dks[r][0, h].numpy(), dk_ref[sl], atol=1e-11)
                np.testing.assert_allclose(dvs[r][0, h].numpy(), dv_ref[sl], atol=1e-11)


def test_block_schedule():
    from exact_attention_159_b200 import ring
    # every rank sees every chunk exactly once over the steps, its own first
    for world in (1, 2, 5):
        for r in range(world):
            srcs = [ring.source(r, s, world) for s in range(world)]
            assert srcs[0] == r and sorted(srcs) == list(range(world))
    assert ring.block_kind(2, 1, True) == "full" and ring.block_kind(2, 2, True) == "diag"
    assert ring.block_kind(2, 3, True) is None and ring.block_kind(2, 3, False) == "full"


def _group_worker(rank, world, port, out):
    import torch.distributed as dist
    from exact_attention_159_b200 import ring
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # two independent rings, ranks {0, 2} and {1, 3} (group ranks differ from global ranks)
        groups = [dist.new_group([0, 2]), dist.new_group([1, 3])]
        g = groups[rank % 2]
        gr = dist.get_rank(g)
        B, H, n, d = 1, 2, 8, 8
        q, k, v, do = _inputs(B, H, 2 * n, d, seed=11 + rank % 2)  # each ring its own sequence
        sl = slice(gr * n, (gr + 1) * n)
        qc, kc, vc, doc = (t[:, :, sl].contiguous() for t in (q, k, v, do))
        be = Fp64Backend()
        o, lse = ring.ring_attention_fwd(qc, kc, vc, 0.4, True, group=g, backend=be)
        dq, dk, dv = ring.ring_attention_bwd(qc, kc, vc, o, doc, lse, 0.4, True, group=g, backend=be)
        out[rank] = [t.numpy() for t in (o, lse, dq, dk, dv)]
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_ring_over_a_subgroup_of_ranks():
    ctx = mp.get_context("spawn")
    port = 29950 + (os.getpid() % 40)
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_group_worker, args=(4, port, out), nprocs=4, join=True, start_method="spawn")
        res = dict(out)
    B, H, n, d = 1, 2, 8, 8
    for parity in (0, 1):
        q, k, v, do = (t.numpy() for t in _inputs(B, H, 2 * n, d, seed=11 + parity))
        for h in range(H):
            o_ref, l_ref = OR.fwd(q[0, h], k[0, h], v[0, h], 0.4, True, nthreads=1)
            dq_ref, dk_ref, dv_ref, _, _ = OR.bwd(q[0, h], k[0, h], v[0, h], do[0, h], 0.4, True, nthreads=1)
            for gr, rank in enumerate((parity, parity + 2)):
                sl = slice(gr * n, (gr + 1) * n)
                o, lse, dq, dk, dv = res[rank]
                np.testing.assert_allclose(o[0, h], o_ref[sl], atol=1e-12)
                np.testing.assert_allclose(lse[0, h], l_ref[sl], atol=1e-12)
                np.testing.assert_allclose(dq[0, h], dq_ref[sl], atol=1e-11)
                np.testing.assert_allclose(dk[0, h], dk_ref[sl], atol=1e-11)
                np.testing.assert_allclose(dv[0, h], dv_ref[sl], atol=1e-11)
