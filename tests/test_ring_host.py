"""Ring (context-parallel) attention: the schedule and the exchanges over gloo ranks on CPU.

The ring driver (exact_attention_159_b200/ring.py) is run by 2, 3 and 4 gloo ranks with an
fp64 CPU stand-in for the per-block kernels (test infrastructure, below): the stand-in computes
each block's attention with the oracle and folds it in by the log-sum-exp, and each block's
backward from the definition with the rows' final LSE and D.  What is checked is the ring
itself -- the zig-zag layout, which chunk each rank holds at each step, which block pairs the
causal mask keeps, the fold of partial results and the return of the dK / dV accumulators to
their owners -- against the oracle on the whole sequence, to fp64 rounding.  The kernels are
checked on their own by the GPU tests.
"""
import os

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import oracle as OR


class Fp64Backend:
    """The per-block steps in fp64 on CPU (tensors B x H x n x d, float64)."""

    @staticmethod
    def _scores(q, k, scale, causal):
        s = scale * torch.einsum("bhid,bhjd->bhij", q, k)
        if causal:
            n = q.shape[2]
            s = s.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), -float("inf"))
        return s

    def fwd_acc(self, q, k, v, o_acc, lse_acc, scale, causal, first):
        B, H = q.shape[:2]
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:-1], dtype=torch.float64)
        for b in range(B):
            for h in range(H):
                ob, lb = OR.fwd(q[b, h].numpy(), k[b, h].numpy(), v[b, h].numpy(), scale, causal, nthreads=1)
                o[b, h] = torch.from_numpy(ob)
                lse[b, h] = torch.from_numpy(lb)
        if first:
            o_acc.copy_(o)
            lse_acc.copy_(lse)
            return
        l_new = torch.logaddexp(lse_acc, lse)
        o_acc.copy_(torch.exp(lse_acc - l_new)[..., None] * o_acc + torch.exp(lse - l_new)[..., None] * o)
        lse_acc.copy_(l_new)

    def bwd_prepare(self, o, do, lse):
        # the workspace: D from the rows' final O, their final LSE, and a zeroed dQ accumulator
        return {"D": (do * o).sum(-1, keepdim=True), "lse": lse.clone(), "dq": torch.zeros_like(o)}

    def bwd_acc(self, ws, q, k, v, do, dk_acc, dv_acc, scale, causal, first):
        p = torch.exp(self._scores(q, k, scale, causal) - ws["lse"][..., None])
        ds = p * (torch.einsum("bhid,bhjd->bhij", do, v) - ws["D"])
        ws["dq"] += scale * torch.einsum("bhij,bhjd->bhid", ds, k)
        dk = scale * torch.einsum("bhij,bhid->bhjd", ds, q)
        dv = torch.einsum("bhij,bhid->bhjd", p, do)
        if first:
            dk_acc.copy_(dk)
            dv_acc.copy_(dv)
        else:
            dk_acc.add_(dk)
            dv_acc.add_(dv)

    def bwd_finish(self, ws, q, scale):
        return ws["dq"].clone()

    def add(self, acc, x):
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
        qc, kc, vc, doc = (ring.zigzag_shard(t, rank, world) for t in (q, k, v, do))
        be = Fp64Backend()
        o, lse = ring.ring_attention_fwd(qc, kc, vc, 0.4, causal, backend=be)
        dq, dk, dv = ring.ring_attention_bwd(qc, kc, vc, o, doc, lse, 0.4, causal, backend=be)
        out[rank] = [t.numpy() for t in (o, lse, dq, dk, dv)]
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_over_gloo_matches_oracle(world, causal):
    ctx = mp.get_context("spawn")
    port = 29600 + (os.getpid() % 300) + 10 * world + int(causal)
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, causal, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    from exact_attention_159_b200 import ring
    B, H, n, d = 1, 2, 8, 8
    q, k, v, do = (t.numpy() for t in _inputs(B, H, n * world, d, seed=7))
    # the whole-sequence results, reassembled from the ranks' zig-zag chunks
    got = [ring.zigzag_unshard([torch.from_numpy(res[r][i]) for r in range(world)]).numpy() for i in range(5)]
    for h in range(H):
        o_ref, l_ref = OR.fwd(q[0, h], k[0, h], v[0, h], 0.4, causal, nthreads=1)
        dq_ref, dk_ref, dv_ref, _, _ = OR.bwd(q[0, h], k[0, h], v[0, h], do[0, h], 0.4, causal, nthreads=1)
        np.testing.assert_allclose(got[0][0, h], o_ref, atol=1e-12)
        np.testing.assert_allclose(got[1][0, h], l_ref, atol=1e-12)
        np.testing.assert_allclose(got[2][0, h], dq_ref, atol=1e-11)
        np.testing.assert_allclose(got[3][0, h], dk_ref, atol=1e-11)
        np.testing.assert_allclose(got[4][0, h], dv_ref, atol=1e-11)


def test_emulated_ring_matches_oracle():
    # the single-process emulation runs the same per-rank steps
    from exact_attention_159_b200 import ring
    world, B, H, n, d = 4, 1, 2, 6, 8
    q, k, v, do = _inputs(B, H, n * world, d, seed=9)
    chunks = [[ring.zigzag_shard(t, r, world) for r in range(world)] for t in (q, k, v, do)]
    be = Fp64Backend()
    for causal in (False, True):
        os_, lses = ring.ring_attention_fwd_emulated(chunks[0], chunks[1], chunks[2], 0.3, causal, backend=be)
        dqs, dks, dvs = ring.ring_attention_bwd_emulated(chunks[0], chunks[1], chunks[2], os_, chunks[3], lses, 0.3,
                                                         causal, backend=be)
        got = [ring.zigzag_unshard(x).numpy() for x in (os_, lses, dqs, dks, dvs)]
        for h in range(H):
            o_ref, l_ref = OR.fwd(q[0, h].numpy(), k[0, h].numpy(), v[0, h].numpy(), 0.3, causal, nthreads=1)
            dq_ref, dk_ref, dv_ref, _, _ = OR.bwd(q[0, h].numpy(), k[0, h].numpy(), v[0, h].numpy(),
                                                  do[0, h].numpy(), 0.3, causal, nthreads=1)
            np.testing.assert_allclose(got[0][0, h], o_ref, atol=1e-12)
            np.testing.assert_allclose(got[1][0, h], l_ref, atol=1e-12)
            np.testing.assert_allclose(got[2][0, h], dq_ref, atol=1e-11)
            np.testing.assert_allclose(got[3][0, h], dk_ref, atol=1e-11)
            np.testing.assert_allclose(got[4][0, h], dv_ref, atol=1e-11)


def test_block_schedule():
    from exact_attention_159_b200 import ring
    # every rank sees every chunk exactly once over the steps, its own first
    for world in (1, 2, 5):
        for r in range(world):
            srcs = [ring.source(r, s, world) for s in range(world)]
            assert srcs[0] == r and sorted(srcs) == list(range(world))


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_zigzag_pairs_cover_the_causal_mask_with_equal_work(world):
    # the block pairs each rank computes, over all steps, are exactly the (query block, key block)
    # pairs the causal mask keeps, each once, squares on the diagonal; and at every step every rank
    # computes the same number of h x h blocks (two, three on its own chunk)
    from exact_attention_159_b200 import ring
    seen = {}
    for s in range(world):
        work = []
        for r in range(world):
            src = ring.source(r, s, world)
            qb, kb = ring.zigzag_blocks(r, world), ring.zigzag_blocks(src, world)
            pairs = ring.block_pairs(r, src, True)
            work.append(len(pairs))
            for qi, kj, diag in pairs:
                key = (qb[qi], kb[kj])
                assert key not in seen
                seen[key] = diag
        assert all(w == work[0] for w in work), (s, work)
        assert work[0] == (3 if s == 0 else 2)
    want = {(i, j): i == j for i in range(2 * world) for j in range(2 * world) if j <= i}
    assert seen == want
    # without the mask every pair of halves is a full block
    assert ring.block_pairs(0, 1, False) == [(0, 0, False), (0, 1, False), (1, 0, False), (1, 1, False)]


def test_zigzag_shard_roundtrip():
    from exact_attention_159_b200 import ring
    x = torch.arange(2 * 3 * 24 * 4, dtype=torch.float64).reshape(2, 3, 24, 4)
    for world in (1, 2, 3, 4):
        chunks = [ring.zigzag_shard(x, r, world) for r in range(world)]
        assert all(c.shape == (2, 3, 24 // world, 4) for c in chunks)
        assert torch.equal(ring.zigzag_unshard(chunks), x)
    with pytest.raises(ValueError):
        ring.zigzag_shard(x, 0, 5)


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
        qc, kc, vc, doc = (ring.zigzag_shard(t, gr, 2) for t in (q, k, v, do))
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
    from exact_attention_159_b200 import ring
    B, H, n, d = 1, 2, 8, 8
    for parity in (0, 1):
        q, k, v, do = (t.numpy() for t in _inputs(B, H, 2 * n, d, seed=11 + parity))
        got = [ring.zigzag_unshard([torch.from_numpy(res[rank][i]) for rank in (parity, parity + 2)]).numpy()
               for i in range(5)]
        for h in range(H):
            o_ref, l_ref = OR.fwd(q[0, h], k[0, h], v[0, h], 0.4, True, nthreads=1)
            dq_ref, dk_ref, dv_ref, _, _ = OR.bwd(q[0, h], k[0, h], v[0, h], do[0, h], 0.4, True, nthreads=1)
            np.testing.assert_allclose(got[0][0, h], o_ref, atol=1e-12)
            np.testing.assert_allclose(got[1][0, h], l_ref, atol=1e-12)
            np.testing.assert_allclose(got[2][0, h], dq_ref, atol=1e-11)
            np.testing.assert_allclose(got[3][0, h], dk_ref, atol=1e-11)
            np.testing.assert_allclose(got[4][0, h], dv_ref, atol=1e-11)
