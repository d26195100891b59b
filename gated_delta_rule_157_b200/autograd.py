"""torch.autograd binding of the chunk forward and its gradient.

KDAChunkFunction runs kda_chunk_fwd keeping the per-chunk states, and
kda_chunk_bwd in its backward.  Marshalling only: both passes run
in the library's kernels.
"""
import torch

from . import _lib


class KDAChunkFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, g, beta, A_log, dt_bias, S0, opts):
        opts = dict(opts)
        fwd_algo = opts.pop("fwd_algo", "auto")
        B, T, H, Dk = q.shape
        HV, Dv = v.shape[2], v.shape[3]
        chunk = opts["chunk"]
        S_chunks = torch.empty((B, HV, -(-T // chunk), Dk, Dv), dtype=torch.float32, device=q.device)
        o, S_T, _ = _lib.kda_chunk_fwd(q, k, v, g, beta, A_log=A_log, dt_bias=dt_bias, S0=S0,
                                       S_chunks=S_chunks, algo=fwd_algo, **opts)
        ctx.save_for_backward(q, k, v, g, beta, A_log, dt_bias, S_chunks)
        ctx.opts = opts
        ctx.has_S0 = S0 is not None
        return o, S_T

    @staticmethod
    def backward(ctx, do, dS_T):
        q, k, v, g, beta, A_log, dt_bias, S_chunks = ctx.saved_tensors
        if do is None:
            do = torch.zeros(q.shape[:2] + v.shape[2:], dtype=q.dtype, device=q.device)
        gr = _lib.kda_chunk_bwd(q, k, v, g, beta, S_chunks, do.to(q.dtype).contiguous(),
                                None if dS_T is None else dS_T.float().contiguous(),
                                A_log=A_log, dt_bias=dt_bias, want_dS0=ctx.has_S0, **ctx.opts)
        cast = lambda t, ref: None if t is None else t.to(ref.dtype)   # noqa: E731
        return (cast(gr["dq"], q), cast(gr["dk"], k), cast(gr["dv"], v), cast(gr["dg"], g),
                cast(gr["dbeta"], beta), gr["dA_log"] if A_log is not None else None,
                gr["ddt_bias"] if dt_bias is not None else None,
                gr["dS0"] if ctx.has_S0 else None, None)


def kda_chunk(q, k, v, g, beta, *, A_log=None, dt_bias=None, S0=None, chunk=64, g_min=-5.0,
              scale=1.0, l2_eps=1e-6, qk_l2norm_in_kernel=True, beta_sigmoid_in_kernel=True,
              gate_in_kernel=True, g_per_head=False, algo="auto"):
    """Differentiable chunk forward: returns (o, S_T); gradients flow to q, k,
    v, g, beta, A_log, dt_bias and S0 through kda_chunk_bwd.  gate_in_kernel
    and g_per_head as kda_chunk_fwd; algo picks the forward kernel ("auto":
    the tensor-core kernel where it applies, whose chunk states carry the bf16
    path's accuracy into the gradient; "simt": FP32 throughout)."""
    opts = dict(chunk=int(chunk), g_min=g_min, scale=scale, l2_eps=l2_eps,
                qk_l2norm_in_kernel=qk_l2norm_in_kernel, beta_sigmoid_in_kernel=beta_sigmoid_in_kernel,
                gate_in_kernel=gate_in_kernel, g_per_head=bool(g_per_head))
    if algo not in ("auto", "simt", "tc"):
        raise ValueError("algo must be 'auto', 'simt' or 'tc'")
    return KDAChunkFunction.apply(q, k, v, g, beta, A_log, dt_bias, S0, dict(opts, fwd_algo=algo))
