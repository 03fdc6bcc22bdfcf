"""Sequence-split (context-parallel) prefill: the segments of a long sequence run at once.

Over one segment the token recurrence is affine in the state that enters it (page
"混合注意力学习(1)", section "Gated DeltaNet": each token maps the key-row state by
S -> alpha (I - beta k k^T) S + beta k v^T; plain and gated linear attention drop the
erase term): S_out = M S_in + N, with M (d x d) the ordered product of the segment's token
maps and N the segment's state from a zero start. With dk = dv = d a prefill run from
S0 = lambda I ends in lambda M + N and a run from S0 = 0 ends in N, so the prefill kernels
themselves produce the pair. lambda = 256 (``START_SCALE``, a power of two: the division by
it is exact) keeps the rounding of N, which the composition cancels, 256 times smaller next
to M than lambda = 1 would, while lambda M + N stays far inside the kernels' fp16 operand
range (M is a product of contractions and reflections, its entries at most 1 in size). The
steps, for P segments in order:

1. segment 0 runs from the true initial state (its outputs are final, its end state is
   the state entering segment 1); segments 1 .. P-2 run from 0 and from lambda I (the pair);
2. the pairs are exchanged (an all-gather across ranks, one (2, B, H, d, d) fp32 tensor
   per rank) and every segment composes the state entering it,
   S_in(p + 1) = ((lambda M + N)_p - N_p) / lambda S_in(p) + N_p  (``gdn_state_compose``);
3. segments 1 .. P-1 run again from their incoming state: outputs and end states.

Each segment is processed twice (the last one once), so on P devices a sequence of L
tokens costs about two runs of L / P tokens instead of one run of L. The compute of every
step is the library's CUDA kernels (prefill, composition, identity states); this module only
orders the launches and the exchange. ``context_parallel_prefill`` is the multi-rank form
(one rank per device, ``torch.distributed``); ``segmented_prefill`` runs the same steps on
one device, the segments of a (1, H, L) batch being the sequences of packed launches.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import _lib

START_SCALE = 256.0


class CudaOps:
    """The library calls the sequence split is made of (dense layout (B, H, L, d))."""

    @staticmethod
    def prefill(q, k, v, beta, g, s0, o, s_final, chunk, scale, stream=None):
        if beta is None:
            return _lib.lin_attn_chunk_fwd(q, k, v, g, o=o, s0=s0, s_final=s_final, chunk=chunk, scale=scale,
                                           stream=stream)
        return _lib.gdn_chunk_fwd(q, k, v, beta, g, o=o, s0=s0, s_final=s_final, chunk=chunk, scale=scale,
                                  stream=stream)

    @staticmethod
    def identity(count: int, d: int, device, value: float = 1.0, stream=None) -> torch.Tensor:
        s = torch.empty(count, d, d, dtype=torch.float32, device=device)
        _lib.gdn_state_identity(s, value, stream=stream)
        return s

    @staticmethod
    def compose(mn, n, s_in, out, lam: float = 1.0, stream=None):
        _lib.gdn_state_compose(mn, n, s_in, out, lam, stream=stream)
        return out


def _square(q, v):
    dk, dv = q.shape[-1], v.shape[-1]
    if dk != dv:
        raise ValueError(f"the sequence split needs dk == dv (the segment map is a d x d state), got {dk}, {dv}")
    return dk


def context_parallel_prefill(q, k, v, beta=None, g=None, s0=None, *, group=None, chunk: int = 64,
                             scale: float = 1.0, ops=None):
    """This rank's part of a sequence-split prefill over the ranks of ``group``.

    Rank r holds segment r of every sequence: q, k (B, H, L_r, d), v (B, H, L_r, d), beta and
    g (B, H, L_r) (beta None: plain / gated linear attention), all ranks with the same B, H,
    d, dtypes and mode; s0 (B, H, d, d) fp32 on rank 0 (the state before the first segment),
    ignored elsewhere. Returns (o, s_end): o (B, H, L_r, d) fp32, this segment's outputs, and
    s_end (B, H, d, d) fp32, the state at the end of this segment (on the last rank: the
    final state of the whole sequence). Every rank takes the same collective steps.
    """
    import torch.distributed as dist

    ops = ops or CudaOps
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, H, Lr, _ = q.shape
    d = _square(q, v)
    dev = q.device
    o = torch.empty(B, H, Lr, d, dtype=torch.float32, device=dev)
    s_end = torch.empty(B, H, d, d, dtype=torch.float32, device=dev)
    pair = torch.zeros(2, B, H, d, d, dtype=torch.float32, device=dev)   # (lambda M + N, N) of this segment
    lam = START_SCALE
    if rank == 0:
        # the true start: outputs and end state are final; as a pair, M = 0 and N = the end state
        ops.prefill(q, k, v, beta, g, s0, o, s_end, chunk, scale)
        pair[0].copy_(s_end)
        pair[1].copy_(s_end)
    elif rank < world - 1:
        scratch = torch.empty_like(o)
        ops.prefill(q, k, v, beta, g, None, scratch, pair[1], chunk, scale)
        eye = ops.identity(B * H, d, dev, lam).view(B, H, d, d)
        ops.prefill(q, k, v, beta, g, eye, scratch, pair[0], chunk, scale)
    # the last rank's pair is never composed past; it sends zeros
    pairs = [torch.empty_like(pair) for _ in range(world)]
    dist.all_gather(pairs, pair, group=group)
    if rank == 0:
        return o, s_end
    s_in = pairs[0][1].clone()             # the state entering segment 1
    nxt = torch.empty_like(s_in)
    for p in range(1, rank):
        ops.compose(pairs[p][0], pairs[p][1], s_in, nxt, lam)
        s_in, nxt = nxt, s_in
    ops.prefill(q, k, v, beta, g, s_in, o, s_end, chunk, scale)
    return o, s_end


def segment_bounds(L: int, segments: int, chunk: int = 64) -> list:
    """Token offsets 0 = b_0 < b_1 < ... < b_P = L of P segments of near-equal length, each
    boundary a multiple of ``chunk`` (so the segments' chunks are those of the whole
    sequence)."""
    if segments < 1:
        raise ValueError("segments must be >= 1")
    nch = (L + chunk - 1) // chunk
    segments = max(1, min(segments, nch))
    return [min(L, (nch * i // segments) * chunk) for i in range(segments)] + [L]


def segmented_prefill(q, k, v, beta=None, g=None, s0=None, *, segments: int = 4, chunk: int = 64,
                      scale: float = 1.0, o: Optional[torch.Tensor] = None,
                      s_final: Optional[torch.Tensor] = None, bounds: Optional[Sequence[int]] = None):
    """The sequence split on one device for a (1, H, L, d) batch: the P segments of every
    head run as the sequences of packed prefill launches (segment 0 from s0 and segments
    1 .. P-2 from 0 in one launch, segments 1 .. P-2 from lambda I in a second launch on a
    side stream, then the compositions, then segments 1 .. P-1 from their incoming states).
    q, k, v (1, H, L, d); beta, g (1, H, L) or None; s0 (1, H, d, d) or None. Returns
    (o (1, H, L, d) fp32, s_final (1, H, d, d) fp32); equal, up to rounding, to one prefill
    of the whole sequence."""
    Bq, H, L, _ = q.shape
    if Bq != 1:
        raise ValueError("segmented_prefill takes one sequence per head (B == 1)")
    d = _square(q, v)
    dev = q.device
    b = list(bounds) if bounds is not None else segment_bounds(L, segments, chunk)
    P = len(b) - 1
    if o is None:
        o = torch.empty(1, H, L, d, dtype=torch.float32, device=dev)
    if s_final is None:
        s_final = torch.empty(1, H, d, d, dtype=torch.float32, device=dev)
    packed = [t[0] if t is not None else None for t in (q, k, v, beta, g)]
    bounds_dev = torch.tensor(b, dtype=torch.int32, device=dev)    # one copy; launches take slices

    def run(first, last, s_init, out, ends, stream=None):
        # segments first .. last - 1 as one packed launch
        cu = bounds_dev[first:last + 1]
        qq, kk, vv, bb, gg = packed
        if bb is None:
            _lib.lin_attn_chunk_fwd_varlen(qq, kk, vv, cu, gg, o=out, s0=s_init, s_final=ends, chunk=chunk,
                                           scale=scale, stream=stream)
        else:
            _lib.gdn_chunk_fwd_varlen(qq, kk, vv, bb, cu, gg, o=out, s0=s_init, s_final=ends, chunk=chunk,
                                      scale=scale, stream=stream)

    if P == 1:
        run(0, 1, s0, o[0], s_final)
        return o, s_final
    # every buffer is allocated on the main stream before the side stream forks, and the main
    # stream waits for the side stream before any later use, so no buffer is reused early
    s_init = torch.zeros(P - 1, H, d, d, dtype=torch.float32, device=dev)
    if s0 is not None:
        s_init[0].copy_(s0[0])
    ends = torch.empty(P - 1, H, d, d, dtype=torch.float32, device=dev)   # N_p (p >= 1); S_in(1) at 0
    s_in = torch.empty(P - 1, H, d, d, dtype=torch.float32, device=dev)
    seg_ends = torch.empty(P - 1, H, d, d, dtype=torch.float32, device=dev)
    main = torch.cuda.current_stream(dev)
    mn = None
    if P > 2:
        mn = torch.empty(P - 2, H, d, d, dtype=torch.float32, device=dev)
        eye = torch.empty(P - 2, H, d, d, dtype=torch.float32, device=dev)
        scratch = torch.empty(H, L, d, dtype=torch.float32, device=dev)
        # pass 1b, concurrently with 1a: segments 1 .. P-2 from lambda I (lambda M + N), outputs
        # to the scratch buffer
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(main)
        _lib.gdn_state_identity(eye, START_SCALE, stream=side)
        run(1, P - 1, eye, scratch, mn, stream=side)
    # pass 1a: segments 0 .. P-2 (segment 0 from s0, the rest from 0)
    run(0, P - 1, s_init, o[0], ends)
    if P > 2:
        main.wait_stream(side)
    # compositions: the state entering segments 1 .. P-1
    s_in[0].copy_(ends[0])
    for p in range(1, P - 1):
        CudaOps.compose(mn[p - 1], ends[p], s_in[p - 1], s_in[p], START_SCALE)
    # pass 2: segments 1 .. P-1 from their incoming states
    run(1, P, s_in, o[0], seg_ends)
    s_final[0].copy_(seg_ends[P - 2])
    return o, s_final
