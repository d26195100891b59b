/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention core.
 *
 * KDA keeps, per (batch b, value head hv), a state S in R^{Dk x Dv} (row c =
 * key channel, column j = value channel) and, for every token t, applies
 * (page "Implémenter KDA", sections "La forme récurrente de référence" and
 * "Trois pièges"; page "KDA 模块交互式演示", section 1.3 Eq. 1):
 *
 *     S <- Diag(alpha_t) S                      decay, alpha_t = exp(g_t) per key channel
 *     S <- S + beta_t k_t (v_t - S^T k_t)^T     delta-rule write of the retrieval error
 *     o_t = scale * S^T q_t                     read AFTER the update
 *
 * Three optional preprocessing steps run inside the kernels (page
 * "KDAAttention 层", section "chunk_kda 内部做了什么"; all three default on):
 *     qk_l2norm_in_kernel:    q <- q / sqrt(|q|^2 + l2_eps), same for k
 *     beta_sigmoid_in_kernel: beta <- 1 / (1 + exp(-beta))
 *     gate_in_kernel = 1:     g <- g_min * sigmoid(exp(A_log[hv]) * (g + dt_bias[hv,:]))
 *                             (bounded decay; page "KDA 模块交互式演示" section 1.4
 *                             Eq. 5, page "Implémenter KDA" "La décroissance bornée")
 *     gate_in_kernel = 2:     g <- -exp(A_log[hv]) * softplus(g + dt_bias[hv,:])
 *                             (the unbounded gate of the first KDA version, page
 *                             "Implémenter KDA" "La décroissance bornée"; the SIMT
 *                             kernels only)
 *     gate_in_kernel = 0:     g is the log-decay itself.
 * With g_per_head set, g holds one value per (token, value head), shared by
 * the Dk key channels (the Gated DeltaNet form, page "线性注意力交互式演示"
 * Eq. 6), and dt_bias one value per value head.
 *
 * Value head hv reads q/k head h = hv / (HV / H) (contiguous groups).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers (CUDA global memory on the
 *     current device), row-major and contiguous in the stated layout.  The
 *     caller owns every buffer; the library allocates nothing and keeps no
 *     state across calls except one device-resident error word per device.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns without synchronising.
 *   - Argument errors are detected on the host before anything is launched and
 *     are returned as a kda_status; nothing is written in that case.  A failed
 *     launch returns KDA_ERR_CUDA.  Device-side faults of the tensor-core
 *     kernel (a bounded wait that ran out, a caller-given log-decay below
 *     g_min) are recorded in the device error word and reported by
 *     kda_device_status().
 *   - No entry point falls back to the CPU.
 */
#ifndef KDA_B200_H
#define KDA_B200_H

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* NULL pointer, bad size, HV % H != 0, ... */
    KDA_ERR_UNSUPPORTED = 2,   /* valid request no kernel of this build handles */
    KDA_ERR_ALIGNMENT = 3,     /* a pointer is not aligned as the layout requires */
    KDA_ERR_ALIAS = 4,         /* an output overlaps an input or another output */
    KDA_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed */
    KDA_ERR_TIMEOUT = 6,       /* a bounded device-side wait gave up (see kda_device_status) */
    KDA_ERR_RANGE = 7          /* a log-decay given directly to the tensor-core kernel was
                                  below g_min and was clamped (see kda_device_status) */
} kda_status;

typedef enum {
    KDA_DT_F32 = 0,            /* IEEE binary32 */
    KDA_DT_BF16 = 1            /* bfloat16 (rounded to nearest even by the producer) */
} kda_dtype;

typedef enum {
    KDA_ALGO_AUTO = 0,         /* tensor-core kernel when the shape allows it, else SIMT */
    KDA_ALGO_SIMT = 1,         /* FP32 FMA chunk kernel (any supported shape, both dtypes) */
    KDA_ALGO_TC = 2            /* tcgen05 BF16 chunk kernel (bf16, Dk = Dv = 128, chunk = 64) */
} kda_algo;

/*
 * kda_chunk_fwd -- chunk-parallel forward over whole sequences.
 *
 * Computes, for every (b, hv), the outputs o_t of the recurrence above for
 * t = 0..T-1 from the initial state S0, the final state S_T and, optionally,
 * the cumulative transition M_T = prod_{t=T-1..0} (I - beta_t k_t k_t^T) Diag(alpha_t)
 * (page "Implémenter KDA", "Test 2 - l'identité de composition"), so that
 * S_T = M_T S0 + (state reached from S0 = 0).
 * The chunk form it uses is the one of page "KDA 模块交互式演示" section 1.5
 * (Eqs. 3-4) with the decay-weighted UT transform: per chunk of `chunk`
 * tokens, a cumulative sum of g, the triangular solve
 * (I + tril(Diag(beta)(K*Gamma)(K/Gamma)^T, -1))^-1, the intra-chunk
 * Tril[(Q*Gamma)(K/Gamma)^T] product and the serial state carry.
 *
 * Layouts (element type `dtype` unless stated):
 *   q, k    [B, T, H,  Dk]
 *   v       [B, T, HV, Dv]
 *   g       [B, T, HV, Dk]  ([B, T, HV] with g_per_head) log-decay g, or the raw
 *           gate input z when gate_in_kernel;
 *           a log-decay given directly should lie in [g_min, 0]: the SIMT
 *           kernel takes any value (KDA_ALGO_AUTO picks it for a log-decay
 *           given directly); the tensor-core kernel, asked for explicitly
 *           (whose exponent bound, 16 |g_min| per 16-token tile, rests on
 *           it), clamps values below g_min up to g_min and records
 *           KDA_ERR_RANGE for kda_device_status()
 *   beta    [B, T, HV]      write strength, or its logit when beta_sigmoid_in_kernel
 *   A_log   [HV]      fp32  read iff gate_in_kernel (must then be non-NULL)
 *   dt_bias [HV, Dk]  fp32  ([HV] with g_per_head) read iff gate_in_kernel; NULL means 0
 *   S0      [B, HV, Dk, Dv] fp32, or NULL for zeros
 *   o       [B, T, HV, Dv]  output, element type `dtype` (bf16 rounded to nearest even),
 *           or NULL when only the states are wanted (e.g. the first pass of a
 *           segmented run, which needs S_T and M_T): the output work is skipped
 *   S_T     [B, HV, Dk, Dv] fp32 output, or NULL; may be the same buffer as S0
 *           (exactly, not partially overlapping)
 *   M_T     [B, HV, Dk, Dk] fp32 output, or NULL
 *   S_chunks [B, HV, NC, Dk, Dv] fp32 output, or NULL: the state entering each
 *           of the NC = ceil(T / chunk) chunks (S_chunks[.., 0, ..] = S0); the
 *           input kda_chunk_bwd needs.  Both kernels write it: the SIMT kernel
 *           its fp32 state, the tensor-core kernel the fp32 state it carries
 *           between its bf16 MMAs (bf16-path accuracy).
 *
 * Limits: B, T >= 0; 1 <= H <= HV, HV % H == 0; 1 <= Dk, Dv <= 128;
 * 1 <= chunk <= 64.  q, k, v, g, beta, o must be aligned to their element size;
 * KDA_ALGO_TC additionally needs dtype = BF16, Dk = Dv = 128, chunk = 64 and
 * 16-byte aligned q, k, v, g, o.  Its exponent scheme rests on g >= g_min:
 * with gate_in_kernel = 0 (a caller-given log-decay) or 2 (the softplus gate,
 * unbounded below) it clamps every g below g_min to g_min and reports the
 * clamp as KDA_ERR_RANGE through kda_device_status (never silently).
 * KDA_ALGO_AUTO takes the tensor-core kernel only for the bounded gate
 * (gate_in_kernel = 1) and the SIMT kernel, exact for any g <= 0, otherwise.
 * gate_in_kernel must be 0, 1 or 2.  o must not overlap any input; S_T, M_T and
 * S_chunks must not overlap each other, o, or any input except S_T == S0.
 * T == 0 writes S_T = S0 (or 0) and M_T = I.
 */
typedef struct {
    int B, T, H, HV, Dk, Dv, chunk;
    int dtype;                 /* kda_dtype of q, k, v, g, beta and o */
    int algo;                  /* kda_algo */
    float g_min;               /* lower bound of the log-decay, -5 for Kimi K3 */
    float scale;               /* output scale (the pages apply none: 1) */
    float l2_eps;              /* epsilon inside the L2-norm square root */
    int qk_l2norm_in_kernel, beta_sigmoid_in_kernel, gate_in_kernel;
    const void *q, *k, *v, *g, *beta;
    const float *A_log, *dt_bias;
    const float *S0;
    void *o;
    float *S_T;
    float *M_T;
    float *S_chunks;
    int g_per_head;            /* g [B, T, HV] and dt_bias [HV]: one decay per head */
} kda_chunk_args;

kda_status kda_chunk_fwd(const kda_chunk_args *args, void *stream);

/*
 * kda_chunk_bwd -- gradient of the chunk forward.
 *
 * For the loss <dout, o> + <dS_T, S_T> of a kda_chunk_fwd call with the same
 * arguments, writes the gradients with respect to every input: q, k, v, g
 * (the raw gate input z when gate_in_kernel), beta (its logit when
 * beta_sigmoid_in_kernel), the initial state, and A_log, dt_bias when the gate
 * runs in the kernel.  The pages print no backward; this is the exact
 * derivative of the forward's chunk form (page "KDA 模块交互式演示" section 1.5
 * with the decay-weighted UT transform), chunk by chunk in reverse, through
 * the three in-kernel switches, computed in FP32 on the CUDA cores.
 *
 * Inputs: q, k, v, g, beta, A_log, dt_bias and the switches exactly as given
 * to the forward; S_chunks as the forward wrote it with the same `chunk`
 * (the forward's S0 is S_chunks[.., 0, ..]); dout [B, T, HV, Dv] dtype;
 * dS_T [B, HV, Dk, Dv] fp32 or NULL (zeros).
 * Outputs (fp32, every element written): dq, dk [B, T, H, Dk] (summed over
 * the value heads that share a q/k head); dv [B, T, HV, Dv]; dg [B, T, HV, Dk]
 * ([B, T, HV] with g_per_head); dbeta [B, T, HV]; dS0 [B, HV, Dk, Dv] or NULL;
 * dA_log [HV] and ddt_bias [HV, Dk] ([HV] with g_per_head) when gate_in_kernel
 * (else not touched; either may be NULL).
 *
 * Limits as kda_chunk_fwd (1 <= Dk, Dv <= 128, 1 <= chunk <= 64); algo must be
 * KDA_ALGO_AUTO or KDA_ALGO_SIMT.  Activation pointers aligned to their
 * element size, fp32 pointers to 4 bytes.  No output may overlap an input or
 * another output.  The q/k/g/beta gradients are sums of fp32 atomic adds, so
 * their last bits depend on the order the CTAs run in.
 */
typedef struct {
    int B, T, H, HV, Dk, Dv, chunk;
    int dtype;                 /* kda_dtype of q, k, v, g, beta and dout */
    int algo;                  /* KDA_ALGO_AUTO or KDA_ALGO_SIMT */
    float g_min, scale, l2_eps;
    int qk_l2norm_in_kernel, beta_sigmoid_in_kernel, gate_in_kernel;
    const void *q, *k, *v, *g, *beta;
    const float *A_log, *dt_bias;
    const float *S_chunks;     /* [B, HV, NC, Dk, Dv] fp32, NC = ceil(T / chunk) */
    const void *dout;          /* [B, T, HV, Dv] */
    const float *dS_T;         /* [B, HV, Dk, Dv] or NULL */
    float *dq, *dk;            /* [B, T, H, Dk] */
    float *dv;                 /* [B, T, HV, Dv] */
    float *dg;                 /* [B, T, HV, Dk] */
    float *dbeta;              /* [B, T, HV] */
    float *dS0;                /* [B, HV, Dk, Dv] or NULL */
    float *dA_log;             /* [HV] or NULL */
    float *ddt_bias;           /* [HV, Dk] ([HV] with g_per_head) or NULL */
    int g_per_head;            /* as kda_chunk_fwd; dg is then [B, T, HV] */
} kda_chunk_bwd_args;

kda_status kda_chunk_bwd(const kda_chunk_bwd_args *args, void *stream);

/*
 * kda_step -- one decode token for B*HV independent chains against a resident
 * state, updated in place (page "Implémenter KDA", "La forme récurrente de
 * référence"; page "KDA 模块交互式演示" section 1.1 single-step decode).
 *
 * Layouts:
 *   q, k    [B, H,  Dk]   dtype
 *   v       [B, HV, Dv]   dtype
 *   g       [B, HV, Dk]   dtype (log-decay, or raw z when gate_in_kernel);
 *           [B, HV] with g_per_head
 *   beta    [B, HV]       dtype
 *   A_log   [HV], dt_bias [HV, Dk] ([HV] with g_per_head) fp32, as in kda_chunk_fwd
 *   S       [B, HV, Dk, Dv] fp32, read and written in place, 16-byte aligned
 *   o       [B, HV, Dv]   dtype output
 *
 * Limits: 1 <= Dk <= 128, 4 <= Dv <= 128 with Dv % 4 == 0.  o must not overlap
 * S or any input.  One read and one write of S per call.
 */
typedef struct {
    int B, H, HV, Dk, Dv;
    int dtype;
    float g_min, scale, l2_eps;
    int qk_l2norm_in_kernel, beta_sigmoid_in_kernel, gate_in_kernel;
    const void *q, *k, *v, *g, *beta;
    const float *A_log, *dt_bias;
    float *S;
    void *o;
    int g_per_head;            /* g [B, HV] and dt_bias [HV] */
} kda_step_args;

kda_status kda_step(const kda_step_args *args, void *stream);

/*
 * kda_compose -- prefix combine of segment results (KCP; page "KDA 模块交互式演示"
 * section 1.6, page "Implémenter KDA" "Test 3 - le balayage préfixe"):
 *
 *     S_in[0] = S_init (or 0 when S_init is NULL)
 *     S_in[s+1] = M[s] S_in[s] + S_seg[s],   s = 0..n_seg-1
 *
 * S_in[s] is the state entering segment s; S_in[n_seg] is the final state.
 * Layouts (all fp32, device): M [n_seg, BH, Dk, Dk], S_seg [n_seg, BH, Dk, Dv],
 * S_init [BH, Dk, Dv] or NULL, S_in [n_seg + 1, BH, Dk, Dv] output.
 * Limits: n_seg >= 0, BH >= 0, 1 <= Dk, Dv <= 128.  S_in must not overlap the inputs.
 */
kda_status kda_compose(int n_seg, int BH, int Dk, int Dv, const float *M,
                       const float *S_seg, const float *S_init, float *S_in,
                       void *stream);

/* ---------------------------------------------------------------------------
 * Layer prologue and epilogue around the core (page "KDA 模块交互式演示",
 * sections 1.1 and 1.7; page "Implémenter KDA", "La paramétrisation" and
 * "La porte de sortie de rang plein"): the parts of the KDA layer that need no
 * projection weights.
 * ------------------------------------------------------------------------- */

/* Causal depthwise short convolution, then optional SiLU and per-head L2
 * norm (the q / k / v prologue: q = L2Norm(SiLU(ShortConv(x)))):
 *
 *     u[t, c] = bias[c] + sum_{j=0}^{K-1} w[c, j] * x[t - (K-1) + j, c]
 *     y[t, c] = silu ? u / (1 + exp(-u)) : u
 *     y[t, c] <- y[t, c] / sqrt(sum_{c' in head(c)} y[t, c']^2 + l2_eps)   if head_dim > 0
 *
 * Tap K-1 multiplies the current token, so w[:, K-1] = 1 (zero elsewhere,
 * bias 0) is the identity the pages initialise with.  Tokens before the first
 * one come from state_in (the K-1 previous tokens, oldest first) or are zero;
 * state_out receives the last K-1 tokens of state_in ++ x, so a sequence run
 * in pieces (or one token at a time for decode) matches one run over the
 * whole sequence. */
typedef struct {
    int B, T, C;               /* tokens [B, T]; C channels per token, C % 128 == 0 */
    int K;                     /* taps, 1..4 (4 on the pages) */
    int head_dim;              /* 0 (no norm) or 128: L2-normalise every 128 channels */
    int silu;                  /* apply SiLU after the convolution */
    float l2_eps;              /* 1e-6 */
    const void *x;             /* [B, T, C] bf16 */
    const float *w;            /* [C, K] fp32 */
    const float *bias;         /* [C] fp32, or NULL (= 0) */
    const void *state_in;      /* [B, K-1, C] bf16, or NULL (= zeros) */
    void *y;                   /* [B, T, C] bf16 */
    void *state_out;           /* [B, K-1, C] bf16, or NULL */
} kda_conv_args;

/* Runs the prologue above.  T may be 0 (only state_out is written).  x, y,
 * state_in and state_out must be 16-byte aligned (KDA_ERR_ALIGNMENT
 * otherwise); y and state_out must not overlap any input or each other.
 * Errors as for kda_chunk_fwd; rows of a multiple of 256 channels are
 * streamed through shared memory with clock-bounded waits, and a wait that
 * gives up is reported by kda_device_status as KDA_ERR_TIMEOUT. */
kda_status kda_short_conv(const kda_conv_args *args, void *stream);

/* Output gate of the layer (the epilogue before the output projection):
 *
 *     y[n, h, :] = sigmoid(gate[n, h, :]) * weight * o[n, h, :] / sqrt(mean(o[n, h, :]^2) + eps)
 *
 * per row n (token), head h: RMSNorm over the D channels of each head with a
 * per-channel scale shared by the heads, times the sigmoid gate. */
typedef struct {
    int N, HV, D;              /* rows (B * T), heads, channels per head (D == 128) */
    float eps;                 /* 1e-6 */
    const void *o;             /* [N, HV, D] bf16 (the core's output) */
    const void *gate;          /* [N, HV, D] bf16, before the sigmoid */
    const float *weight;       /* [D] fp32, or NULL (= 1) */
    void *y;                   /* [N, HV, D] bf16 */
} kda_gate_args;

/* Runs the epilogue above.  o, gate and y must be 8-byte aligned; y must not
 * overlap o or gate.  Errors as for kda_chunk_fwd. */
kda_status kda_output_gate(const kda_gate_args *args, void *stream);

/* Reads and clears the device error words of the current device (chunk
 * kernel, decode step, layer prologue) after synchronising `stream`.
 * Returns KDA_OK, KDA_ERR_TIMEOUT (a bounded wait gave up since the last
 * call; takes precedence), KDA_ERR_RANGE (a
 * tensor-core call clamped a caller-given log-decay below g_min) or
 * KDA_ERR_CUDA. */
kda_status kda_device_status(void *stream);

/* Test hook for the failure path of the tensor-core chunk kernel (no
 * counterpart in the method): validates and launches exactly like
 * kda_chunk_fwd with algo KDA_ALGO_TC, except that the kernel's prep warps
 * never hand a chunk over to its state warps.  The state warps' bounded wait
 * then gives up after about two seconds, every CTA records the device error
 * word, frees its tensor memory and returns; the outputs are unspecified.
 * kda_device_status() afterwards reports KDA_ERR_TIMEOUT and the context stays
 * usable.  Returns KDA_ERR_UNSUPPORTED unless the arguments select the
 * tensor-core kernel; otherwise as kda_chunk_fwd. */
kda_status kda_debug_chunk_stall(const kda_chunk_args *args, void *stream);

/* Human-readable name of a status code (static storage, never NULL). */
const char *kda_status_string(kda_status status);

/* Library version as 10000 * major + 100 * minor + patch. */
int kda_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KDA_B200_H */
