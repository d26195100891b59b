// C ABI of the library (declared in include/kda.h): host-side validation,
// dispatch and launch.  Validation errors return before anything is enqueued.
#include <stdint.h>

#include "kda_internal.cuh"

namespace {

using kda::ChunkParams;
using kda::StepParams;

struct Range {
    uintptr_t lo, hi;   // [lo, hi)
};

Range range_of(const void *p, size_t bytes) {
    uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return Range{a, a + bytes};
}

bool overlaps(Range a, Range b) {
    if (a.lo == a.hi || b.lo == b.hi) return false;
    return a.lo < b.hi && b.lo < a.hi;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

kda_status cuda_status(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

}  // namespace

extern "C" {

static kda_status chunk_fwd(const kda_chunk_args *a, void *stream, bool withhold_ready) {
    if (!a) return KDA_ERR_INVALID_ARG;
    if (a->B < 0 || a->T < 0 || a->H < 1 || a->HV < 1 || a->HV % a->H != 0)
        return KDA_ERR_INVALID_ARG;
    if (a->Dk < 1 || a->Dv < 1 || a->chunk < 1) return KDA_ERR_INVALID_ARG;
    if (a->dtype != KDA_DT_F32 && a->dtype != KDA_DT_BF16) return KDA_ERR_INVALID_ARG;
    if (a->algo != KDA_ALGO_AUTO && a->algo != KDA_ALGO_SIMT && a->algo != KDA_ALGO_TC)
        return KDA_ERR_INVALID_ARG;
    if (a->Dk > 128 || a->Dv > 128 || a->chunk > 64) return KDA_ERR_UNSUPPORTED;
    if (!(a->g_min < 0.f) || !(a->l2_eps >= 0.f)) return KDA_ERR_INVALID_ARG;
    if (a->gate_in_kernel < 0 || a->gate_in_kernel > 2) return KDA_ERR_INVALID_ARG;
    const bool bf16 = a->dtype == KDA_DT_BF16;
    const size_t es = bf16 ? 2 : 4;
    const size_t ntok = (size_t)a->B * a->T;
    const size_t gk = a->g_per_head ? 1 : (size_t)a->Dk;   // gate values per (token, value head)
    if (a->B == 0) return KDA_OK;

    if (ntok > 0) {
        if (!a->q || !a->k || !a->v || !a->g || !a->beta) return KDA_ERR_INVALID_ARG;   // o may be NULL
        if (a->gate_in_kernel && !a->A_log) return KDA_ERR_INVALID_ARG;
        const void *acts[] = {a->q, a->k, a->v, a->g, a->beta, a->o};
        for (const void *p : acts)
            if (!aligned(p, es)) return KDA_ERR_ALIGNMENT;
    }
    const float *fl[] = {a->A_log, a->dt_bias, a->S0, a->S_T, a->M_T, a->S_chunks};
    for (const float *p : fl)
        if (p && !aligned(p, 4)) return KDA_ERR_ALIGNMENT;

    // Aliasing: o must not overlap inputs; S_T / M_T must not overlap o, inputs
    // (S_T == S0 exactly is allowed) or each other.
    const size_t nq = ntok * a->H * a->Dk * es, nv = ntok * a->HV * a->Dv * es;
    const size_t ng = ntok * a->HV * gk * es, nb = ntok * a->HV * es;
    const size_t ns = (size_t)a->B * a->HV * a->Dk * a->Dv * 4;
    const size_t nm = (size_t)a->B * a->HV * a->Dk * a->Dk * 4;
    Range r_in[] = {range_of(a->q, ntok ? nq : 0), range_of(a->k, ntok ? nq : 0),
                    range_of(a->v, ntok ? nv : 0), range_of(a->g, ntok ? ng : 0),
                    range_of(a->beta, ntok ? nb : 0),
                    range_of(a->A_log, a->A_log ? (size_t)a->HV * 4 : 0),
                    range_of(a->dt_bias, a->dt_bias ? (size_t)a->HV * gk * 4 : 0)};
    Range r_s0 = range_of(a->S0, a->S0 ? ns : 0);
    Range r_o = range_of(a->o, (ntok && a->o) ? nv : 0);
    Range r_st = range_of(a->S_T, a->S_T ? ns : 0);
    Range r_mt = range_of(a->M_T, a->M_T ? nm : 0);
    const size_t nchunks = a->T > 0 ? ((size_t)a->T + a->chunk - 1) / a->chunk : 0;
    Range r_sc = range_of(a->S_chunks, a->S_chunks ? ns * nchunks : 0);
    for (Range r : r_in) {
        if (overlaps(r_o, r) || overlaps(r_st, r) || overlaps(r_mt, r) || overlaps(r_sc, r))
            return KDA_ERR_ALIAS;
    }
    if (overlaps(r_o, r_s0) || overlaps(r_o, r_st) || overlaps(r_o, r_mt) || overlaps(r_st, r_mt) ||
        overlaps(r_mt, r_s0))
        return KDA_ERR_ALIAS;
    if (overlaps(r_sc, r_o) || overlaps(r_sc, r_s0) || overlaps(r_sc, r_st) || overlaps(r_sc, r_mt))
        return KDA_ERR_ALIAS;
    if (overlaps(r_st, r_s0) && a->S_T != a->S0) return KDA_ERR_ALIAS;

    ChunkParams p;
    p.B = a->B; p.T = a->T; p.H = a->H; p.HV = a->HV; p.Dk = a->Dk; p.Dv = a->Dv;
    p.C = a->chunk; p.group = a->HV / a->H;
    p.g_min = a->g_min; p.scale = a->scale; p.l2_eps = a->l2_eps;
    p.l2norm = a->qk_l2norm_in_kernel != 0;
    p.beta_sigmoid = a->beta_sigmoid_in_kernel != 0;
    p.gate_in = a->gate_in_kernel;
    p.g_per_head = a->g_per_head != 0;
    p.q = a->q; p.k = a->k; p.v = a->v; p.g = a->g; p.beta = a->beta;
    p.A_log = a->A_log; p.dt_bias = a->dt_bias; p.S0 = a->S0;
    p.o = a->o; p.S_T = a->S_T; p.M_T = a->M_T; p.S_chunks = a->S_chunks;
    p.withhold_ready = withhold_ready ? 1 : 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    if (a->T == 0) return cuda_status(kda::launch_chunk_empty(p, s));

    // The tensor-core kernel's exponent scheme needs g >= g_min: with a
    // caller-given decay or the (unbounded) softplus gate it clamps g there
    // and reports the clamp, so AUTO sends both to the exact SIMT kernel.
    const bool tc_ok = kda::chunk_tc_supported(p, bf16);
    if (withhold_ready && (a->algo != KDA_ALGO_TC || !tc_ok)) return KDA_ERR_UNSUPPORTED;
    if (a->algo == KDA_ALGO_TC) {
        if (!tc_ok) return KDA_ERR_UNSUPPORTED;
        const void *v16[] = {a->q, a->k, a->v, a->g, a->o};
        for (const void *ptr : v16)
            if (!aligned(ptr, 16)) return KDA_ERR_ALIGNMENT;
        return cuda_status(kda::launch_chunk_tc(p, s));
    }
    // A log-decay given directly (no in-kernel gate) may lie below g_min, where
    // the tensor-core kernel's exponent bound does not hold: AUTO takes the
    // SIMT kernel, which is exact for any g <= 0.
    if (a->algo == KDA_ALGO_AUTO && tc_ok && a->gate_in_kernel == 1) {
        bool al16 = true;
        const void *v16[] = {a->q, a->k, a->v, a->g, a->o};
        for (const void *ptr : v16) al16 = al16 && aligned(ptr, 16);
        if (al16) return cuda_status(kda::launch_chunk_tc(p, s));
    }
    return cuda_status(kda::launch_chunk_simt(p, bf16, s));
}

kda_status kda_chunk_fwd(const kda_chunk_args *a, void *stream) { return chunk_fwd(a, stream, false); }

kda_status kda_debug_chunk_stall(const kda_chunk_args *a, void *stream) { return chunk_fwd(a, stream, true); }

kda_status kda_chunk_bwd(const kda_chunk_bwd_args *a, void *stream) {
    if (!a) return KDA_ERR_INVALID_ARG;
    if (a->B < 0 || a->T < 0 || a->H < 1 || a->HV < 1 || a->HV % a->H != 0)
        return KDA_ERR_INVALID_ARG;
    if (a->Dk < 1 || a->Dv < 1 || a->chunk < 1) return KDA_ERR_INVALID_ARG;
    if (a->dtype != KDA_DT_F32 && a->dtype != KDA_DT_BF16) return KDA_ERR_INVALID_ARG;
    if (a->algo != KDA_ALGO_AUTO && a->algo != KDA_ALGO_SIMT && a->algo != KDA_ALGO_TC)
        return KDA_ERR_INVALID_ARG;
    if (a->algo == KDA_ALGO_TC) return KDA_ERR_UNSUPPORTED;
    if (a->Dk > 128 || a->Dv > 128 || a->chunk > 64) return KDA_ERR_UNSUPPORTED;
    if (!(a->g_min < 0.f) || !(a->l2_eps >= 0.f)) return KDA_ERR_INVALID_ARG;
    if (a->gate_in_kernel < 0 || a->gate_in_kernel > 2) return KDA_ERR_INVALID_ARG;
    if (a->B == 0) return KDA_OK;
    const bool bf16 = a->dtype == KDA_DT_BF16;
    const size_t es = bf16 ? 2 : 4;
    const size_t ntok = (size_t)a->B * a->T;
    const size_t gk = a->g_per_head ? 1 : (size_t)a->Dk;
    if (ntok > 0) {
        if (!a->q || !a->k || !a->v || !a->g || !a->beta || !a->S_chunks || !a->dout) return KDA_ERR_INVALID_ARG;
        if (!a->dq || !a->dk || !a->dv || !a->dg || !a->dbeta) return KDA_ERR_INVALID_ARG;
        if (a->gate_in_kernel && !a->A_log) return KDA_ERR_INVALID_ARG;
        const void *acts[] = {a->q, a->k, a->v, a->g, a->beta, a->dout};
        for (const void *p : acts)
            if (!aligned(p, es)) return KDA_ERR_ALIGNMENT;
    }
    const float *fl[] = {a->A_log, a->dt_bias, a->S_chunks, a->dS_T, a->dq, a->dk, a->dv,
                         a->dg, a->dbeta, a->dS0, a->dA_log, a->ddt_bias};
    for (const float *p : fl)
        if (p && !aligned(p, 4)) return KDA_ERR_ALIGNMENT;

    const size_t nq = ntok * a->H * a->Dk, nv = ntok * a->HV * a->Dv;
    const size_t ng = ntok * a->HV * gk, nb = ntok * a->HV;
    const size_t ns = (size_t)a->B * a->HV * a->Dk * a->Dv;
    const size_t nchunks = a->T > 0 ? ((size_t)a->T + a->chunk - 1) / a->chunk : 0;
    const bool gate = a->gate_in_kernel != 0;
    Range r_in[] = {range_of(a->q, ntok ? nq * es : 0), range_of(a->k, ntok ? nq * es : 0),
                    range_of(a->v, ntok ? nv * es : 0), range_of(a->g, ntok ? ng * es : 0),
                    range_of(a->beta, ntok ? nb * es : 0), range_of(a->dout, ntok ? nv * es : 0),
                    range_of(a->A_log, a->A_log ? (size_t)a->HV * 4 : 0),
                    range_of(a->dt_bias, a->dt_bias ? (size_t)a->HV * gk * 4 : 0),
                    range_of(a->S_chunks, a->S_chunks ? ns * nchunks * 4 : 0),
                    range_of(a->dS_T, a->dS_T ? ns * 4 : 0)};
    Range r_out[] = {range_of(a->dq, ntok ? nq * 4 : 0), range_of(a->dk, ntok ? nq * 4 : 0),
                     range_of(a->dv, ntok ? nv * 4 : 0), range_of(a->dg, ntok ? ng * 4 : 0),
                     range_of(a->dbeta, ntok ? nb * 4 : 0), range_of(a->dS0, a->dS0 ? ns * 4 : 0),
                     range_of(gate ? a->dA_log : nullptr, gate && a->dA_log ? (size_t)a->HV * 4 : 0),
                     range_of(gate ? a->ddt_bias : nullptr, gate && a->ddt_bias ? (size_t)a->HV * gk * 4 : 0)};
    const int n_out = sizeof(r_out) / sizeof(r_out[0]);
    for (int i = 0; i < n_out; ++i) {
        for (Range r : r_in)
            if (overlaps(r_out[i], r)) return KDA_ERR_ALIAS;
        for (int j = i + 1; j < n_out; ++j)
            if (overlaps(r_out[i], r_out[j])) return KDA_ERR_ALIAS;
    }

    kda::BwdParams p;
    p.B = a->B; p.T = a->T; p.H = a->H; p.HV = a->HV; p.Dk = a->Dk; p.Dv = a->Dv;
    p.C = a->chunk; p.group = a->HV / a->H;
    p.g_min = a->g_min; p.scale = a->scale; p.l2_eps = a->l2_eps;
    p.l2norm = a->qk_l2norm_in_kernel != 0;
    p.beta_sigmoid = a->beta_sigmoid_in_kernel != 0;
    p.gate_in = a->gate_in_kernel;
    p.g_per_head = a->g_per_head != 0;
    p.q = a->q; p.k = a->k; p.v = a->v; p.g = a->g; p.beta = a->beta;
    p.A_log = a->A_log; p.dt_bias = a->dt_bias; p.S_chunks = a->S_chunks;
    p.dout = a->dout; p.dS_T = a->dS_T;
    p.dq = a->dq; p.dk = a->dk; p.dv = a->dv; p.dg = a->dg; p.dbeta = a->dbeta; p.dS0 = a->dS0;
    p.dA_log = gate ? a->dA_log : nullptr;
    p.ddt_bias = gate ? a->ddt_bias : nullptr;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    // The q/k/g/beta (and parameter) gradients are accumulated with atomics.
    struct Zero { void *p; size_t bytes; } zeros[] = {
        {p.dq, ntok ? nq * 4 : 0}, {p.dk, ntok ? nq * 4 : 0}, {p.dg, ntok ? ng * 4 : 0},
        {p.dbeta, ntok ? nb * 4 : 0}, {p.dA_log, p.dA_log ? (size_t)a->HV * 4 : 0},
        {p.ddt_bias, p.ddt_bias ? (size_t)a->HV * gk * 4 : 0}};
    for (const Zero &z : zeros) {
        if (z.bytes && cudaMemsetAsync(z.p, 0, z.bytes, s) != cudaSuccess) return KDA_ERR_CUDA;
    }
    return cuda_status(kda::launch_chunk_bwd(p, bf16, s));
}

kda_status kda_step(const kda_step_args *a, void *stream) {
    if (!a) return KDA_ERR_INVALID_ARG;
    if (a->B < 0 || a->H < 1 || a->HV < 1 || a->HV % a->H != 0) return KDA_ERR_INVALID_ARG;
    if (a->Dk < 1 || a->Dv < 1) return KDA_ERR_INVALID_ARG;
    if (a->dtype != KDA_DT_F32 && a->dtype != KDA_DT_BF16) return KDA_ERR_INVALID_ARG;
    if (a->Dk > 128 || a->Dv > 128 || a->Dv % 4 != 0) return KDA_ERR_UNSUPPORTED;
    if (!(a->g_min < 0.f) || !(a->l2_eps >= 0.f)) return KDA_ERR_INVALID_ARG;
    if (a->gate_in_kernel < 0 || a->gate_in_kernel > 2) return KDA_ERR_INVALID_ARG;
    if (a->B == 0) return KDA_OK;
    const size_t gk = a->g_per_head ? 1 : (size_t)a->Dk;
    if (!a->q || !a->k || !a->v || !a->g || !a->beta || !a->S || !a->o) return KDA_ERR_INVALID_ARG;
    if (a->gate_in_kernel && !a->A_log) return KDA_ERR_INVALID_ARG;
    const bool bf16 = a->dtype == KDA_DT_BF16;
    const size_t es = bf16 ? 2 : 4;
    const void *acts[] = {a->q, a->k, a->v, a->g, a->beta, a->o};
    for (const void *p : acts)
        if (!aligned(p, es)) return KDA_ERR_ALIGNMENT;
    if (!aligned(a->S, 16)) return KDA_ERR_ALIGNMENT;
    if ((a->A_log && !aligned(a->A_log, 4)) || (a->dt_bias && !aligned(a->dt_bias, 4)))
        return KDA_ERR_ALIGNMENT;

    const size_t B = a->B;
    Range r_in[] = {range_of(a->q, B * a->H * a->Dk * es), range_of(a->k, B * a->H * a->Dk * es),
                    range_of(a->v, B * a->HV * a->Dv * es), range_of(a->g, B * a->HV * gk * es),
                    range_of(a->beta, B * a->HV * es),
                    range_of(a->A_log, a->A_log ? (size_t)a->HV * 4 : 0),
                    range_of(a->dt_bias, a->dt_bias ? (size_t)a->HV * gk * 4 : 0)};
    Range r_s = range_of(a->S, B * a->HV * a->Dk * a->Dv * 4);
    Range r_o = range_of(a->o, B * a->HV * a->Dv * es);
    for (Range r : r_in)
        if (overlaps(r_o, r) || overlaps(r_s, r)) return KDA_ERR_ALIAS;
    if (overlaps(r_o, r_s)) return KDA_ERR_ALIAS;

    StepParams p;
    p.B = a->B; p.H = a->H; p.HV = a->HV; p.Dk = a->Dk; p.Dv = a->Dv; p.group = a->HV / a->H;
    p.g_min = a->g_min; p.scale = a->scale; p.l2_eps = a->l2_eps;
    p.l2norm = a->qk_l2norm_in_kernel != 0;
    p.beta_sigmoid = a->beta_sigmoid_in_kernel != 0;
    p.gate_in = a->gate_in_kernel;
    p.g_per_head = a->g_per_head != 0;
    p.q = a->q; p.k = a->k; p.v = a->v; p.g = a->g; p.beta = a->beta;
    p.A_log = a->A_log; p.dt_bias = a->dt_bias; p.S = a->S; p.o = a->o;
    return cuda_status(kda::launch_step(p, bf16, static_cast<cudaStream_t>(stream)));
}

kda_status kda_compose(int n_seg, int BH, int Dk, int Dv, const float *M, const float *S_seg,
                       const float *S_init, float *S_in, void *stream) {
    if (n_seg < 0 || BH < 0 || Dk < 1 || Dv < 1) return KDA_ERR_INVALID_ARG;
    if (Dk > 128 || Dv > 128) return KDA_ERR_UNSUPPORTED;
    if (BH == 0) return KDA_OK;
    if (!S_in || (n_seg > 0 && (!M || !S_seg))) return KDA_ERR_INVALID_ARG;
    const float *ps[] = {M, S_seg, S_init, S_in};
    for (const float *p : ps)
        if (p && !aligned(p, 4)) return KDA_ERR_ALIGNMENT;
    const size_t st = (size_t)BH * Dk * Dv * 4, mt = (size_t)BH * Dk * Dk * 4;
    Range r_out = range_of(S_in, st * (n_seg + 1));
    if (overlaps(r_out, range_of(M, M ? mt * n_seg : 0)) ||
        overlaps(r_out, range_of(S_seg, S_seg ? st * n_seg : 0)) ||
        overlaps(r_out, range_of(S_init, S_init ? st : 0)))
        return KDA_ERR_ALIAS;
    return cuda_status(kda::launch_compose(n_seg, BH, Dk, Dv, M, S_seg, S_init, S_in,
                                           static_cast<cudaStream_t>(stream)));
}

kda_status kda_short_conv(const kda_conv_args *a, void *stream) {
    if (!a) return KDA_ERR_INVALID_ARG;
    if (a->B < 0 || a->T < 0 || a->C < 1 || a->K < 1 || a->K > 4 || !(a->l2_eps >= 0.f))
        return KDA_ERR_INVALID_ARG;
    if (a->head_dim != 0 && a->head_dim != 128) return KDA_ERR_UNSUPPORTED;
    if (a->C % 128 != 0) return KDA_ERR_UNSUPPORTED;
    if (a->B == 0) return KDA_OK;
    const size_t ntok = (size_t)a->B * a->T, es = 2;
    if (!a->w || (ntok > 0 && (!a->x || !a->y))) return KDA_ERR_INVALID_ARG;
    // the kernels move 8 channels (16 bytes) per lane
    const void *p16[] = {a->x, a->y, a->state_in, a->state_out};
    for (const void *p : p16)
        if (p && !aligned(p, 16)) return KDA_ERR_ALIGNMENT;
    if (!aligned(a->w, 4) || (a->bias && !aligned(a->bias, 4))) return KDA_ERR_ALIGNMENT;
    const size_t nx = ntok * a->C * es, ns = (size_t)a->B * (a->K - 1) * a->C * es;
    Range r_y = range_of(a->y, ntok ? nx : 0), r_so = range_of(a->state_out, a->state_out ? ns : 0);
    Range r_in[] = {range_of(a->x, ntok ? nx : 0), range_of(a->state_in, a->state_in ? ns : 0),
                    range_of(a->w, (size_t)a->C * a->K * 4), range_of(a->bias, a->bias ? (size_t)a->C * 4 : 0)};
    for (Range r : r_in)
        if (overlaps(r_y, r) || overlaps(r_so, r)) return KDA_ERR_ALIAS;
    if (overlaps(r_y, r_so)) return KDA_ERR_ALIAS;
    kda::ConvParams p;
    p.B = a->B; p.T = a->T; p.C = a->C; p.K = a->K; p.head_dim = a->head_dim; p.silu = a->silu != 0;
    p.l2_eps = a->l2_eps;
    p.x = a->x; p.w = a->w; p.bias = a->bias; p.state_in = a->state_in; p.y = a->y; p.state_out = a->state_out;
    return cuda_status(kda::launch_short_conv(p, static_cast<cudaStream_t>(stream)));
}

kda_status kda_output_gate(const kda_gate_args *a, void *stream) {
    if (!a) return KDA_ERR_INVALID_ARG;
    if (a->N < 0 || a->HV < 1 || a->D < 1 || !(a->eps >= 0.f)) return KDA_ERR_INVALID_ARG;
    if (a->D != 128) return KDA_ERR_UNSUPPORTED;
    if (a->N == 0) return KDA_OK;
    if (!a->o || !a->gate || !a->y) return KDA_ERR_INVALID_ARG;
    const void *p8[] = {a->o, a->gate, a->y};
    for (const void *p : p8)
        if (!aligned(p, 8)) return KDA_ERR_ALIGNMENT;
    if (a->weight && !aligned(a->weight, 4)) return KDA_ERR_ALIGNMENT;
    const size_t n = (size_t)a->N * a->HV * a->D * 2;
    Range r_y = range_of(a->y, n);
    if (overlaps(r_y, range_of(a->o, n)) || overlaps(r_y, range_of(a->gate, n)) ||
        overlaps(r_y, range_of(a->weight, a->weight ? (size_t)a->D * 4 : 0)))
        return KDA_ERR_ALIAS;
    kda::GateParams p;
    p.N = a->N; p.HV = a->HV; p.D = a->D; p.eps = a->eps;
    p.o = a->o; p.gate = a->gate; p.weight = a->weight; p.y = a->y;
    return cuda_status(kda::launch_output_gate(p, static_cast<cudaStream_t>(stream)));
}

kda_status kda_device_status(void *stream) {
    unsigned int word = 0, step_word = 0, conv_word = 0;
    cudaError_t e = kda::read_and_clear_device_error(static_cast<cudaStream_t>(stream), &word);
    if (e == cudaSuccess) e = kda::read_and_clear_step_error(&step_word);
    if (e == cudaSuccess) e = kda::read_and_clear_conv_error(&conv_word);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    word |= step_word | conv_word;
    if (word & 1u) return KDA_ERR_TIMEOUT;
    return (word & 2u) ? KDA_ERR_RANGE : KDA_OK;
}

const char *kda_status_string(kda_status s) {
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_ALIGNMENT: return "KDA_ERR_ALIGNMENT";
        case KDA_ERR_ALIAS: return "KDA_ERR_ALIAS";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
        case KDA_ERR_RANGE: return "KDA_ERR_RANGE";
    }
    return "KDA_ERR_UNKNOWN";
}

int kda_version(void) { return 200; }

}  // extern "C"
