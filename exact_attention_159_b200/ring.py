"""Ring (context-parallel) exact attention across GPUs, over torch.distributed.

The sequence is split into R equal, contiguous chunks, one per rank: rank r holds query,
key and value rows r*n .. r*n + n - 1 of every head (B, H, n, d tensors).  The key/value
chunks travel around the ring of ranks (point-to-point sends over NCCL, each one overlapped
with the attention on the chunk already held); every rank attends its queries to each chunk
as it passes, and folds the partial results together through their log-sum-exp:
exact attention over the union of disjoint key sets is
    L = ln(exp(LSE_a) + exp(LSE_b)),   O = exp(LSE_a - L) O_a + exp(LSE_b - L) O_b
(``fa_lse_merge``).  Under the causal mask, chunk src is entirely visible to rank r's queries
when src < r, is the usual causal square when src == r, and is skipped when src > r.

The backward sends each key/value chunk around the ring once more, together with fp32
accumulators of its dK and dV: every rank adds the gradients of its queries' attention to
the chunk it holds (``fa_bwd`` with the global O and LSE of its rows, which make the
per-chunk pieces exact), keeps its own dQ in fp32, and after the last step hands each
chunk's accumulators back to the chunk's owner.  Both transfers overlap compute: the next
key/value chunk travels while a step computes, and a chunk's accumulators travel while the
receiving rank computes its gradients for that chunk, which it adds once they have arrived.

The pages name multi-card use of the kernels for long contexts ("NVIDIA Blackwell:
FlashAttention-4 Overcomes Memory Bottlenecks", body); the exchange itself is the
standard ring schedule.  Every arithmetic step runs in libfa's kernels (attention, merge,
fp32 accumulation, conversion); torch only holds device memory and moves the chunks.
``*_emulated`` run the same per-rank steps for R ranks inside one process (the chunks are
handed over in Python instead of sent), so the arithmetic can be checked on a single GPU.
"""
from __future__ import annotations

import math

import torch

from . import api


class LibBackend:
    """The kernels of libfa (the product path)."""

    def fwd(self, q, k, v, scale, causal):
        return api.fa_fwd(q, k, v, scale, causal)

    def bwd(self, q, k, v, o, do, lse, scale, causal):
        return api.fa_bwd(q, k, v, o, do, lse, scale, causal)

    def merge(self, o_part, lse_part, o_acc, lse_acc, first):
        api.fa_lse_merge(o_part, lse_part, o_acc, lse_acc, first)

    def accumulate(self, acc, x, first):
        api.fa_accumulate_bf16(acc, x, first)

    def to_bf16(self, x):
        return api.fa_convert_f32_bf16(x)

    def f32_like(self, t):
        return torch.empty(t.shape, dtype=torch.float32, device=t.device)

    def lse_like(self, q):
        return torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)


def block_kind(r: int, src: int, causal: bool):
    """How rank r's query chunk sees key chunk src: 'full', 'diag' (the causal square) or None."""
    if not causal or src < r:
        return "full"
    return "diag" if src == r else None


def source(r: int, s: int, world: int) -> int:
    """The key/value chunk rank r holds at step s (chunks move one rank forward per step)."""
    return (r - s) % world


# ---------------------------------------------------------------- per-rank steps
class _FwdState:
    def __init__(self, be, q):
        self.o_acc, self.lse_acc, self.first = be.f32_like(q), be.lse_like(q), True


def _fwd_step(be, st, r, s, world, q, k, v, scale, causal):
    kind = block_kind(r, source(r, s, world), causal)
    if kind is not None:
        o_p, lse_p = be.fwd(q, k, v, scale, kind == "diag")
        be.merge(o_p, lse_p, st.o_acc, st.lse_acc, st.first)
        st.first = False


class _BwdState:
    def __init__(self, be, q):
        self.dq_acc, self.first = be.f32_like(q), True


def _bwd_partial(be, r, s, world, q, k, v, o, do, lse, scale, causal):
    """Rank r's gradients for the chunk it holds at step s (None when the causal mask skips it)."""
    kind = block_kind(r, source(r, s, world), causal)
    return None if kind is None else be.bwd(q, k, v, o, do, lse, scale, kind == "diag")


def _bwd_accumulate(be, st, s, part, dk_acc, dv_acc):
    """Adds a step's partial gradients to dQ and to the held chunk's dK, dV accumulators."""
    if part is None:
        return
    dq_p, dk_p, dv_p = part
    be.accumulate(st.dq_acc, dq_p, st.first)
    st.first = False
    # the chunk's own rank starts its accumulators at step 0 (its diagonal block is never skipped)
    be.accumulate(dk_acc, dk_p, s == 0)
    be.accumulate(dv_acc, dv_p, s == 0)


# ------------------------------------------------------------- distributed drivers
def _ring_exchange(send, recv, rank, world, group):
    """Post the sends of `send` to the next rank and the receives into `recv` from the previous one."""
    import torch.distributed as dist
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    g_nxt = dist.get_global_rank(group, nxt) if group is not None else nxt
    g_prv = dist.get_global_rank(group, prv) if group is not None else prv
    ops = [dist.P2POp(dist.irecv, t, g_prv, group) for t in recv] + \
          [dist.P2POp(dist.isend, t, g_nxt, group) for t in send]
    return dist.batch_isend_irecv(ops)


def ring_attention_fwd(q, k, v, scale: float | None = None, causal: bool = False, group=None, backend=None):
    """O (bf16) and LSE (fp32) of this rank's query chunk over the whole sequence."""
    import torch.distributed as dist
    be = backend or LibBackend()
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)
    st = _FwdState(be, q)
    cur = [k.contiguous(), v.contiguous()]
    for s in range(world):
        reqs, nxt = [], None
        if s + 1 < world:
            nxt = [torch.empty_like(t) for t in cur]
            reqs = _ring_exchange(cur, nxt, rank, world, group)
        _fwd_step(be, st, rank, s, world, q, cur[0], cur[1], scale, causal)
        for req in reqs:
            req.wait()
        if nxt is not None:
            cur = nxt
    return be.to_bf16(st.o_acc), st.lse_acc


def ring_attention_bwd(q, k, v, o, do, lse, scale: float | None = None, causal: bool = False, group=None,
                       backend=None):
    """dQ of this rank's query chunk and dK, dV of its key/value chunk (bf16)."""
    import torch.distributed as dist
    be = backend or LibBackend()
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)
    st = _BwdState(be, q)
    kv = [k.contiguous(), v.contiguous()]
    acc = [be.f32_like(k), be.f32_like(v)]  # the held chunk's dK, dV accumulators
    acc_reqs, nxt_acc = [], None
    for s in range(world):
        reqs, nxt_kv = [], None
        if s + 1 < world:  # the chunk itself moves on while this step computes
            nxt_kv = [torch.empty_like(t) for t in kv]
            reqs = _ring_exchange(kv, nxt_kv, rank, world, group)
        # this step's gradients are computed while the held chunk's accumulators are still on their
        # way from the previous holder; they are added once those have arrived
        part = _bwd_partial(be, rank, s, world, q, kv[0], kv[1], o, do, lse, scale, causal)
        for req in acc_reqs:
            req.wait()
        if nxt_acc is not None:
            acc = nxt_acc
        _bwd_accumulate(be, st, s, part, acc[0], acc[1])
        if world > 1:  # the accumulators follow their chunk; after the last step they reach the owner
            nxt_acc = [torch.empty_like(t) for t in acc]
            acc_reqs = _ring_exchange(acc, nxt_acc, rank, world, group)
        for req in reqs:
            req.wait()
        if nxt_kv is not None:
            kv = nxt_kv
    for req in acc_reqs:
        req.wait()
    if nxt_acc is not None:
        acc = nxt_acc
    return be.to_bf16(st.dq_acc), be.to_bf16(acc[0]), be.to_bf16(acc[1])


# ------------------------------------------------------ single-process emulation
def ring_attention_fwd_emulated(qs, ks, vs, scale: float | None = None, causal: bool = False, backend=None):
    """The ring forward for len(qs) ranks in one process: lists of per-rank chunks in, out."""
    be = backend or LibBackend()
    world = len(qs)
    scale = 1.0 / math.sqrt(qs[0].shape[-1]) if scale is None else float(scale)
    states = [_FwdState(be, q) for q in qs]
    held = [(ks[r], vs[r]) for r in range(world)]
    for s in range(world):
        for r in range(world):
            _fwd_step(be, states[r], r, s, world, qs[r], held[r][0], held[r][1], scale, causal)
        held = [held[(r - 1) % world] for r in range(world)]
    return [be.to_bf16(st.o_acc) for st in states], [st.lse_acc for st in states]


def ring_attention_bwd_emulated(qs, ks, vs, os_, dos, lses, scale: float | None = None, causal: bool = False,
                                backend=None):
    """The ring backward for len(qs) ranks in one process."""
    be = backend or LibBackend()
    world = len(qs)
    scale = 1.0 / math.sqrt(qs[0].shape[-1]) if scale is None else float(scale)
    states = [_BwdState(be, q) for q in qs]
    held = [[ks[r], vs[r], be.f32_like(ks[r]), be.f32_like(vs[r])] for r in range(world)]
    for s in range(world):
        for r in range(world):
            c = held[r]
            part = _bwd_partial(be, r, s, world, qs[r], c[0], c[1], os_[r], dos[r], lses[r], scale, causal)
            _bwd_accumulate(be, states[r], s, part, c[2], c[3])
        held = [held[(r - 1) % world] for r in range(world)]
    # after `world` rotations every chunk, with its accumulated dK and dV, is back at its owner
    return ([be.to_bf16(st.dq_acc) for st in states], [be.to_bf16(held[r][2]) for r in range(world)],
            [be.to_bf16(held[r][3]) for r in range(world)])
