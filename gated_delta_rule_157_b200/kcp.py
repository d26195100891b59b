"""Context-parallel KDA forward across ranks (KCP).

A sequence too long for one GPU is split into contiguous segments, one per
rank of a process group.  The state recurrence is affine in the state
(page "Implémenter KDA", the composition test: running a segment from S0 gives
M S0 plus its run from zero), so each rank

  1. runs its segment from the zero state, keeping the final state S_seg and
     the cumulative transition M_seg (kda_chunk_fwd with output_transition),
  2. all-gathers (M_seg, S_seg) from every rank (the only exchange: a
     Dk x (Dk + Dv) fp32 block per chain),
  3. combines them in segment order into the state entering each segment
     (kda_compose: S_in[s+1] = M_s S_in[s] + S_seg[s], S_in[0] = the initial
     state), and
  4. reruns its segment from S_in[rank] for its output rows.

Every rank returns its own segment's o and the final state of the whole
sequence.  The compute steps run in the library's kernels; the exchange is a
process-group all-gather (NCCL between GPUs; a gloo group exchanges host
copies of the blocks).
"""
import torch
import torch.distributed as dist

from . import _lib


class _KernelOps:
    """The library's kernels and the process group's all-gather."""

    @staticmethod
    def forward(q, k, v, g, beta, S0, want_M, **kw):
        # the pass with the transition only needs the states: no o
        o, S_T, M_T = _lib.kda_chunk_fwd(q, k, v, g, beta, S0=S0, output_final_state=True,
                                         output_transition=want_M, output_o=not want_M, **kw)
        return o, S_T, M_T

    @staticmethod
    def compose(M, S_seg, S_init):
        return _lib.kda_compose(M, S_seg, S_init)

    @staticmethod
    def compose_into(M, S_seg, S_init, S_in):
        _lib.kda_compose(M, S_seg, S_init, S_in=S_in)

    @staticmethod
    def all_gather(t, world, group):
        if world == 1:
            return t.unsqueeze(0)
        src = t.contiguous()
        # a gloo group exchanges host memory: device blocks travel through host copies
        via_host = src.is_cuda and dist.get_backend(group) == "gloo"
        if via_host:
            src = src.cpu()
        parts = [torch.empty_like(src) for _ in range(world)]
        dist.all_gather(parts, src, group=group)
        out = torch.stack(parts)
        return out.to(t.device) if via_host else out


def _group_shape(group):
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(group), dist.get_rank(group)
    return 1, 0


def kcp_chunk_fwd(q, k, v, g, beta, *, A_log=None, dt_bias=None, S0=None, chunk=64, group=None,
                  g_min=-5.0, scale=1.0, l2_eps=1e-6, qk_l2norm_in_kernel=True,
                  beta_sigmoid_in_kernel=True, gate_in_kernel=True, g_per_head=False, algo="auto", ops=None):
    """Forward of this rank's segment of a sequence split across `group`.

    q, k [B,L,H,Dk]; v [B,L,HV,Dv]; g [B,L,HV,Dk]; beta [B,L,HV]: segment
    `rank` of the sequence (segments in rank order, any lengths).  A_log,
    dt_bias and the initial state S0 [B,HV,Dk,Dv] (or None) are the same on
    every rank.  gate_in_kernel and g_per_head as kda_chunk_fwd (g [B,L,HV]
    with g_per_head).  Returns (o [B,L,HV,Dv] of this segment, S_T [B,HV,Dk,Dv] of
    the whole sequence).  Every rank must call this collectively.
    """
    ops = ops or _KernelOps
    world, rank = _group_shape(group)
    B, _, _, Dk = q.shape
    HV, Dv = v.shape[2], v.shape[3]
    kw = dict(A_log=A_log, dt_bias=dt_bias, chunk=chunk, g_min=g_min, scale=scale, l2_eps=l2_eps,
              qk_l2norm_in_kernel=qk_l2norm_in_kernel, beta_sigmoid_in_kernel=beta_sigmoid_in_kernel,
              gate_in_kernel=gate_in_kernel, g_per_head=g_per_head, algo=algo)
    # 1. this segment from the zero state
    _, S_seg, M_seg = ops.forward(q, k, v, g, beta, None, True, **kw)
    # 2. exchange: [world, B*HV, Dk, Dk] and [world, B*HV, Dk, Dv]
    M_all = ops.all_gather(M_seg.reshape(B * HV, Dk, Dk), world, group)
    S_all = ops.all_gather(S_seg.reshape(B * HV, Dk, Dv), world, group)
    # 3. state entering every segment, and the final state
    S_init = None if S0 is None else S0.reshape(B * HV, Dk, Dv)
    S_in = ops.compose(M_all, S_all, S_init)
    # 4. this segment's rows from its incoming state
    o, _, _ = ops.forward(q, k, v, g, beta, S_in[rank].reshape(B, HV, Dk, Dv).contiguous(), False, **kw)
    return o, S_in[world].reshape(B, HV, Dk, Dv)


def seq_segments(B, HV, T, chunk, sms):
    """Segments per sequence for kda_chunk_fwd_seqpar: the power of two n
    (T divisible by n, at least two chunks per segment) that minimises the
    modelled time, waves x (chunks per segment + 2 for a CTA's start-up and
    pipeline fill), over the states-only pass (two CTAs per segment and
    chain: state and transition) and the output pass (one).  1 when the
    chains alone fill the SMs."""
    nchunks = -(-T // chunk)
    best, best_cost = 1, -(-B * HV // sms) * (nchunks + 2)
    n = 2
    while n <= 64 and T % n == 0 and -(-(T // n) // chunk) >= 2:
        seg = -(-(T // n) // chunk)
        cost = (-(-2 * B * HV * n // sms) + -(-B * HV * n // sms)) * (seg + 2)
        if cost < best_cost:
            best, best_cost = n, cost
        n *= 2
    return best


def kda_chunk_fwd_seqpar(q, k, v, g, beta, *, A_log=None, dt_bias=None, S0=None, chunk=64, segments=None,
                         g_min=-5.0, scale=1.0, l2_eps=1e-6, qk_l2norm_in_kernel=True,
                         beta_sigmoid_in_kernel=True, gate_in_kernel=True, g_per_head=False, algo="auto",
                         ops=None):
    """Forward of whole sequences on one GPU with every sequence cut into
    `segments` equal parts that run in parallel (by default seq_segments():
    when B x HV chains leave SMs idle, as for a single prefill).  The same
    affine composition as the context-parallel forward (page "Implémenter
    KDA", the composition test): the segments run from the zero state keeping
    their final states and transitions, kda_compose chains them into the
    state entering each segment, and the segments run again from those states
    for their output rows.  Returns (o [B,T,HV,Dv], S_T [B,HV,Dk,Dv]); S_T is
    the last segment's final state of the second pass (a view).  T must be
    divisible by `segments`; no transition output (M_T) on this path.
    """
    ops = ops or _KernelOps
    B, T, H, Dk = q.shape
    HV, Dv = v.shape[2], v.shape[3]
    kw = dict(A_log=A_log, dt_bias=dt_bias, chunk=chunk, g_min=g_min, scale=scale, l2_eps=l2_eps,
              qk_l2norm_in_kernel=qk_l2norm_in_kernel, beta_sigmoid_in_kernel=beta_sigmoid_in_kernel,
              gate_in_kernel=gate_in_kernel, g_per_head=g_per_head, algo=algo)
    if segments is None:
        sms = torch.cuda.get_device_properties(q.device).multi_processor_count if q.is_cuda else 1
        segments = seq_segments(B, HV, T, chunk, sms)
    n = int(segments)
    if n <= 1:
        o, S_T, _ = ops.forward(q, k, v, g, beta, S0, False, **kw)
        return o, S_T
    if T % n:
        raise ValueError("T = %d is not divisible into %d segments" % (T, n))
    Ts = T // n

    def seg(x):              # [B, T, ...] -> [B*n, T/n, ...]: a view of the contiguous input
        return x.reshape((B * n, Ts) + tuple(x.shape[2:]))

    # 1. every segment from the zero state: its final state and transition
    _, S_seg, M = ops.forward(seg(q), seg(k), seg(v), seg(g), seg(beta), None, True, **kw)
    S_seg = S_seg.reshape(B, n, HV, Dk, Dv)
    M = M.reshape(B, n, HV, Dk, Dk)
    # 2. the state entering each segment, written straight into the second
    #    pass's initial states (the last segment's transition is not needed)
    S_in = torch.empty((B, n, HV, Dk, Dv), dtype=S_seg.dtype, device=S_seg.device)
    for b in range(B):
        ops.compose_into(M[b, :n - 1], S_seg[b, :n - 1], None if S0 is None else S0[b], S_in[b])
    # 3. every segment from its incoming state: the output rows, and the
    #    whole sequence's final state as the last segment's
    o, S_out, _ = ops.forward(seg(q), seg(k), seg(v), seg(g), seg(beta), S_in.reshape(B * n, HV, Dk, Dv),
                              False, **kw)
    return o.reshape(B, T, HV, Dv), S_out.reshape(B, n, HV, Dk, Dv)[:, -1]
