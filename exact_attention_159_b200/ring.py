"""Ring (context-parallel) exact attention across GPUs, over torch.distributed.

Layout.  The sequence (length L) is cut into 2R equal blocks of h = L / 2R rows; rank r holds
blocks r and 2R-1-r, concatenated along the sequence axis into its local chunk of n = 2h rows
(``zigzag_shard`` / ``zigzag_unshard``).  The key/value chunks travel around the ring of ranks
(point-to-point sends over NCCL, each overlapped with the attention on the chunk already held),
and every rank attends its queries to each chunk as it passes.  Under the causal mask the local
query half a (block r) and half b (block 2R-1-r) meet the halves a' (block src) and b'
(block 2R-1-src) of the chunk from rank src as follows:
    src == r:  (a, a') and (b, b') causal squares, (b, a') full
    src <  r:  (a, a') and (b, a') full   -- b' lies after both query halves
    src >  r:  (b, a') and (b, b') full   -- half a lies before both key halves
so every rank computes two h x h blocks per step (three on its own chunk): equal work on every
rank at every step, where contiguous chunks would leave rank r with r + 1 blocks of work.
Without the mask every pair of halves is a full block.

Forward.  Each block's attention is folded into the rank's fp32 accumulators (O, LSE per query
half) inside the kernel by the log-sum-exp (``fa_fwd_accumulate``): exact attention over the
union of disjoint key sets is L = ln(exp(LSE_a) + exp(LSE_b)), O = exp(LSE_a - L) O_a +
exp(LSE_b - L) O_b.  Nothing is rounded to bf16 until the final O.

Backward.  ``fa_bwd_prepare`` computes D = rowsum(dO * O) and LSE * log2(e) of each local query
half once, from the final O and LSE, and zeroes its fp32 dQ accumulator; every block then adds
its dQ there (``fa_bwd_accumulate``) and its dK, dV into step-local fp32 buffers.  The key/value
chunk travels around the ring once more, followed by fp32 accumulators of its dK and dV: a rank
adds its step buffers to the held chunk's accumulators once they have arrived (their transfer
overlaps the step's kernels) and sends them on; after the last step they are back at the
chunk's owner.  dQ, dK and dV are rounded to bf16 once, at the end.

The pages name multi-card use of the kernels for long contexts ("NVIDIA Blackwell:
FlashAttention-4 Overcomes Memory Bottlenecks", body); the exchange itself is the standard ring
schedule with a causal load-balanced ("zig-zag") block assignment.  Every arithmetic step runs in
libfa's kernels; torch only holds device memory and moves the chunks.  ``*_emulated`` run the
same per-rank steps for R ranks inside one process (the chunks are handed over in Python
instead of sent), so the arithmetic can be checked on a single GPU.
"""
from __future__ import annotations

import math

import torch

from . import api


class LibBackend:
    """The kernels of libfa (the product path)."""

    def fwd_acc(self, q, k, v, o_acc, lse_acc, scale, causal, first):
        api.fa_fwd_accumulate(q, k, v, o_acc, lse_acc, scale, causal, first)

    def bwd_prepare(self, o, do, lse):
        return api.fa_bwd_prepare(o, do, lse)

    def bwd_acc(self, ws, q, k, v, do, dk_acc, dv_acc, scale, causal, first):
        api.fa_bwd_accumulate(q, k, v, do, ws, dk_acc, dv_acc, scale, causal, first)

    def bwd_finish(self, ws, q, scale):
        B, H, N, d = q.shape
        return api.fa_bwd_finish(ws, B, H, N, d, scale)

    def add(self, acc, x):
        api.fa_accumulate_f32(acc, x)

    def to_bf16(self, x):
        return api.fa_convert_f32_bf16(x)

    def f32_like(self, t):
        return torch.empty(t.shape, dtype=torch.float32, device=t.device)

    def lse_like(self, q):
        return torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)


# ------------------------------------------------------------------- layout
def zigzag_blocks(rank: int, world: int) -> tuple[int, int]:
    """The two sequence blocks (of 2 * world) that rank holds, in local order."""
    return rank, 2 * world - 1 - rank


def zigzag_shard(x: torch.Tensor, rank: int, world: int, dim: int = 2) -> torch.Tensor:
    """Rank's local chunk of a whole-sequence tensor: blocks r and 2R-1-r, concatenated."""
    if x.shape[dim] % (2 * world):
        raise ValueError(f"sequence length {x.shape[dim]} is not a multiple of 2 * world = {2 * world}")
    blocks = x.chunk(2 * world, dim=dim)
    a, b = zigzag_blocks(rank, world)
    return torch.cat([blocks[a], blocks[b]], dim=dim).contiguous()


def zigzag_unshard(chunks, dim: int = 2) -> torch.Tensor:
    """The whole-sequence tensor from every rank's local chunk (inverse of zigzag_shard)."""
    world = len(chunks)
    blocks = [None] * (2 * world)
    for r, c in enumerate(chunks):
        a, b = zigzag_blocks(r, world)
        blocks[a], blocks[b] = c.chunk(2, dim=dim)
    return torch.cat(blocks, dim=dim)


def block_pairs(r: int, src: int, causal: bool):
    """(query half, key half, causal square?) pairs rank r computes against the chunk of rank src."""
    if not causal:
        return [(0, 0, False), (0, 1, False), (1, 0, False), (1, 1, False)]
    if src == r:
        return [(0, 0, True), (1, 0, False), (1, 1, True)]
    if src < r:
        return [(0, 0, False), (1, 0, False)]
    return [(1, 0, False), (1, 1, False)]


def source(r: int, s: int, world: int) -> int:
    """The key/value chunk rank r holds at step s (chunks move one rank forward per step)."""
    return (r - s) % world


def _halves(x: torch.Tensor, dim: int = 2):
    return [t.contiguous() for t in x.chunk(2, dim=dim)]


# ---------------------------------------------------------------- per-rank steps
class _FwdState:
    def __init__(self, be, qh):
        self.o = [be.f32_like(q) for q in qh]
        self.lse = [be.lse_like(q) for q in qh]
        self.first = [True, True]


def _fwd_step(be, st, r, src, qh, kv, scale, causal):
    """Folds rank r's attention to the held chunk (kv = [k_a, k_b, v_a, v_b]) into its accumulators."""
    for qi, kj, diag in block_pairs(r, src, causal):
        be.fwd_acc(qh[qi], kv[kj], kv[2 + kj], st.o[qi], st.lse[qi], scale, diag, st.first[qi])
        st.first[qi] = False


def _bwd_step(be, ws, r, src, qh, doh, kv, dkv, scale, causal):
    """Rank r's gradients against the held chunk: dQ into the workspaces, dK and dV of the chunk's
    halves into dkv = [dk_a, dk_b, dv_a, dv_b] (stored by the first block that touches a half).
    Returns which key halves were touched."""
    touched = [False, False]
    for qi, kj, diag in block_pairs(r, src, causal):
        be.bwd_acc(ws[qi], qh[qi], kv[kj], kv[2 + kj], doh[qi], dkv[kj], dkv[2 + kj], scale, diag,
                   not touched[kj])
        touched[kj] = True
    return touched


def _scale(q, scale):
    return 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)


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
    """O (bf16) and LSE (fp32) of this rank's local query chunk (zig-zag layout) over the whole
    sequence; q, k, v: the rank's local chunks [B, H, n, d], n even."""
    import torch.distributed as dist
    be = backend or LibBackend()
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    scale = _scale(q, scale)
    qh = _halves(q)
    st = _FwdState(be, qh)
    kv = _halves(k) + _halves(v)
    for s in range(world):
        reqs, nxt = [], None
        if s + 1 < world:
            nxt = [torch.empty_like(t) for t in kv]
            reqs = _ring_exchange(kv, nxt, rank, world, group)
        _fwd_step(be, st, rank, source(rank, s, world), qh, kv, scale, causal)
        for req in reqs:
            req.wait()
        if nxt is not None:
            kv = nxt
    return torch.cat([be.to_bf16(o) for o in st.o], dim=2), torch.cat(st.lse, dim=2)


def ring_attention_bwd(q, k, v, o, do, lse, scale: float | None = None, causal: bool = False, group=None,
                       backend=None):
    """dQ of this rank's local query chunk and dK, dV of its local key/value chunk (bf16), given the
    chunk's O and LSE from ring_attention_fwd and the upstream dO."""
    import torch.distributed as dist
    be = backend or LibBackend()
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    scale = _scale(q, scale)
    qh, doh = _halves(q), _halves(do)
    ws = [be.bwd_prepare(oh, dh, lh) for oh, dh, lh in zip(_halves(o), doh, _halves(lse))]
    kv = _halves(k) + _halves(v)
    acc = [be.f32_like(t) for t in kv]   # dK, dV accumulators of the held chunk's halves
    step = [be.f32_like(t) for t in kv]  # this step's dK, dV of the held chunk
    acc_reqs, nxt_acc = [], None
    for s in range(world):
        reqs, nxt_kv = [], None
        if s + 1 < world:  # the chunk itself moves on while this step computes
            nxt_kv = [torch.empty_like(t) for t in kv]
            reqs = _ring_exchange(kv, nxt_kv, rank, world, group)
        # the owner's step (s == 0) starts the accumulators; later steps fill the step buffers while
        # the held chunk's accumulators are still on their way, and add them once they are here
        touched = _bwd_step(be, ws, rank, source(rank, s, world), qh, doh, kv, acc if s == 0 else step, scale,
                            causal)
        if s == 0:
            for kj in (0, 1):
                if not touched[kj]:  # (never under this schedule: the owner touches both halves)
                    raise RuntimeError("ring schedule left a key half without gradients on its owner")
        else:
            for req in acc_reqs:
                req.wait()
            acc = nxt_acc
            for kj in (0, 1):
                if touched[kj]:
                    be.add(acc[kj], step[kj])
                    be.add(acc[2 + kj], step[2 + kj])
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
    dq = torch.cat([be.bwd_finish(w, qq, scale) for w, qq in zip(ws, qh)], dim=2)
    dk = torch.cat([be.to_bf16(a) for a in acc[:2]], dim=2)
    dv = torch.cat([be.to_bf16(a) for a in acc[2:]], dim=2)
    return dq, dk, dv


# ------------------------------------------------------ single-process emulation
def ring_attention_fwd_emulated(qs, ks, vs, scale: float | None = None, causal: bool = False, backend=None):
    """The ring forward for len(qs) ranks in one process: lists of per-rank local chunks in, out."""
    be = backend or LibBackend()
    world = len(qs)
    scale = _scale(qs[0], scale)
    qhs = [_halves(q) for q in qs]
    states = [_FwdState(be, qh) for qh in qhs]
    held = [_halves(ks[r]) + _halves(vs[r]) for r in range(world)]
    for s in range(world):
        for r in range(world):
            _fwd_step(be, states[r], r, source(r, s, world), qhs[r], held[r], scale, causal)
        held = [held[(r - 1) % world] for r in range(world)]
    return ([torch.cat([be.to_bf16(o) for o in st.o], dim=2) for st in states],
            [torch.cat(st.lse, dim=2) for st in states])


def ring_attention_bwd_emulated(qs, ks, vs, os_, dos, lses, scale: float | None = None, causal: bool = False,
                                backend=None):
    """The ring backward for len(qs) ranks in one process."""
    be = backend or LibBackend()
    world = len(qs)
    scale = _scale(qs[0], scale)
    qhs = [_halves(q) for q in qs]
    dohs = [_halves(d) for d in dos]
    wss = [[be.bwd_prepare(oh, dh, lh) for oh, dh, lh in zip(_halves(os_[r]), dohs[r], _halves(lses[r]))]
           for r in range(world)]
    # held[r]: (key/value halves, their dK/dV accumulators) of the chunk rank r holds
    held = [(_halves(ks[r]) + _halves(vs[r]), None) for r in range(world)]
    for s in range(world):
        nxt = []
        for r in range(world):
            kv, acc = held[r]
            src = source(r, s, world)
            if s == 0:
                acc = [be.f32_like(t) for t in kv]
                _bwd_step(be, wss[r], r, src, qhs[r], dohs[r], kv, acc, scale, causal)
            else:
                step = [be.f32_like(t) for t in kv]
                touched = _bwd_step(be, wss[r], r, src, qhs[r], dohs[r], kv, step, scale, causal)
                for kj in (0, 1):
                    if touched[kj]:
                        be.add(acc[kj], step[kj])
                        be.add(acc[2 + kj], step[2 + kj])
            nxt.append((kv, acc))
        held = [nxt[(r - 1) % world] for r in range(world)]
    # after `world` rotations every chunk, with its accumulated dK and dV, is back at its owner
    dqs = [torch.cat([be.bwd_finish(w, qq, scale) for w, qq in zip(wss[r], qhs[r])], dim=2) for r in range(world)]
    dks = [torch.cat([be.to_bf16(a) for a in held[r][1][:2]], dim=2) for r in range(world)]
    dvs = [torch.cat([be.to_bf16(a) for a in held[r][1][2:]], dim=2) for r in range(world)]
    return dqs, dks, dvs
