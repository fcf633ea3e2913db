/*
 * gdn.h -- C ABI of libgdn.so, the B200 (sm_100a) chunkwise gated delta-rule
 * forward pass and the backward pass of the gated delta rule.
 *
 * What it computes.  For every (batch b, head h) sequence, with the state S_t
 * a d_v x d_k matrix (keys to values):
 *
 *   gated delta rule (default):
 *     S_t = S_{t-1} alpha_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = S_t q_t.
 *   The pages read the delta rule as an online SGD step on the least-squares
 *   loss 1/2||S k_t - v_t||^2 ("Resumo Tecnico: Preconditioned DeltaNet",
 *   section 1), alpha is the decay axis and beta the gain axis ("Preconditioned
 *   DeltaNet: Curvature-aware Sequence Modeling for Linear Recurrences",
 *   Arabic summary, section 2c).
 *
 *   preconditioned two-gate rule (precond / erase / write / per-channel alpha):
 *     rho_t = rho_decay rho_{t-1} + k_t (.) k_t,  kw_t = k_t / sqrt(rho_t + rho_eps),
 *     S_t = S_{t-1}(diag(alpha_t) - (b_t (.) kw_t) kw_t^T) + (w_t (.) v_t) kw_t^T,
 *     o_t = S_t q_t  (q is the read key, kw the write key).
 *   Diagonal curvature preconditioner: same Arabic summary, section 2b; read
 *   and write keys: "Resumo Tecnico: Preconditioned DeltaNet", section 2;
 *   channel-wise erase gate b_t (key axis) and write gate w_t (value axis):
 *   "NVIDIA Apresenta Gated DeltaNet-2", section "Como DeltaNet-2 Redesenhou
 *   a Arquitetura".
 *
 * How.  Chunkwise-parallel (WY/UT) form over chunks of C tokens: per chunk the
 * strictly lower triangular A is built from the key Gram matrix, and
 * T = (I - A)^-1 ("Quando o 'Bom o Suficiente' e Otimo: Aproximacao de
 * Inversao de Matriz Baseada Apenas em Multiplicacao para Gated DeltaNet
 * Quantizado", section "Declaracao do Problema") is formed either exactly
 * (GDN_INV_EXACT) or as the truncated Neumann series sum_{n<=N} A^n with the
 * structural diagonal mask M_ij = [i - j <= N] (GDN_INV_NEUMANN; same page,
 * section "Metodologia", items 1 and 2).  The fp32 state is carried from
 * chunk to chunk inside one kernel.
 *
 * Layouts (all row-major, innermost last, no padding):
 *   q, k     [B, T, H, dk]   io_dtype          (q is the read key)
 *   v        [B, T, H, dv]   io_dtype
 *   alpha    [B, T, H] fp32, or [B, T, H, dk] fp32 when alpha_per_channel
 *   beta     [B, T, H] fp32
 *   erase    [B, T, H, dk]   io_dtype          (gate b_t)
 *   write    [B, T, H, dv]   io_dtype          (gate w_t)
 *   S0, S_T  [B, H, dk, dv]  fp32              (h = S^T: row = key channel)
 *   o        [B, T, H, dv]   o_dtype
 *
 * Ownership.  Every pointer is a DEVICE pointer owned by the caller, who
 * allocates inputs, outputs and the workspace.  The library allocates no
 * device memory and keeps no state between calls.  The fused tensor-core
 * kernel (GDN_KERNEL_TC) needs no workspace: its per-chunk inverses move
 * between the two CTAs of a cluster through shared memory.  The split
 * tensor-core kernels (GDN_KERNEL_TC_SPLIT) keep, per chunk and head,
 * T diag(beta), T diag(beta e^g) and the decayed causal scores P (fp16,
 * 24 KB) in the workspace between their two launches; at C = 128 also, per
 * second 64-token half, the band corner's two parts (16 (dk + dv) fp32); for
 * the two-gate rule instead the prep's operands as fp16 rows (TB, P, U as
 * hi + lo pairs, E, Q', K'', the decay; (640 + 2 dv + 4) x 128 B) and the
 * preconditioner's running averages.  The SIMT kernels
 * (GDN_KERNEL_SIMT) keep, per chunk and head, the state-independent fp32
 * matrices of the chunk (T diag(beta), the decayed scores, the decayed keys
 * and queries, 2 C^2 + 3 C dk + dk floats) and, for the preconditioned
 * two-gate rule, the running average at every chunk start (dk floats).
 * gdn_workspace_bytes() gives the size.
 *
 * Execution and errors.  gdn_chunk_fwd validates its arguments on the host
 * and returns an error before launching anything (nothing is written) when
 * they are invalid.  Otherwise it enqueues the work on `stream` (a
 * cudaStream_t passed as void*, NULL = legacy default stream) and returns
 * without synchronising; launch failures map to GDN_ERR_CUDA.  o must not
 * alias any input; S_T may alias S0 (each block reads its slice of S0 before
 * it writes the same slice of S_T).  gdn_last_error() returns a message for
 * the calling thread's most recent failure.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDN_ABI_VERSION 9

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,    /* NULL pointer, bad size, bad enum value */
    GDN_ERR_UNSUPPORTED = 2,    /* valid request this build cannot run */
    GDN_ERR_ALIGNMENT = 3,      /* a pointer or row stride is not 16-byte aligned */
    GDN_ERR_CUDA = 4,           /* the CUDA runtime reported an error */
    GDN_ERR_DEVICE_CHECK = 5,   /* a kernel's own bounds check recorded a failure */
    GDN_ERR_FAULT_INJECTED = 6  /* GDN_FAULT_INJECT=1 in the environment (tests) */
} gdn_status;

typedef enum { GDN_F32 = 0, GDN_BF16 = 1 } gdn_dtype;

typedef enum {
    GDN_INV_EXACT = 0,          /* T = (I - A)^-1 exactly (blocked inversion) */
    GDN_INV_NEUMANN = 1,        /* T = M^(N) (.) sum_{n=0}^{N} A^n */
    GDN_INV_NEUMANN_RESIDUAL = 2 /* T0 = M^(N) (.) sum_{n=0}^{N} A^n, E = I - (I - A) T0,
                                   T = T0 sum_{s=0}^{S} E^s ("Quando o 'Bom o Suficiente' e
                                   Otimo ...", section "Metodologia", item 3); tensor-core
                                   kernel only */
} gdn_inv_mode;

typedef enum {
    GDN_KERNEL_AUTO = 0,        /* the first of TC_SPLIT, TC, SIMT that supports the call
                                   (RECURRENT for T <= 8) */
    GDN_KERNEL_SIMT = 1,        /* fp32 CUDA-core kernels (all variants): the chunk matrices
                                   of every chunk at once into the workspace, then the
                                   state chain */
    GDN_KERNEL_TC = 2,          /* fused tcgen05/TMEM/TMA kernel, one launch of 2-CTA
                                   clusters per (batch, head): bf16 q/k/v, scalar decay,
                                   C = 64, dk = dv = 128, exact or Neumann mode (any N).
                                   Needs no workspace (gdn_workspace_bytes() is 0). */
    GDN_KERNEL_RECURRENT = 3,   /* token-by-token kernel for short sequences and decode steps
                                   (scalar decay, exact mode, dk a multiple of 8, dv of 32);
                                   AUTO picks it for T <= 8 */
    GDN_KERNEL_TC_SPLIT = 4     /* the tensor-core path as two launches (a key-side kernel
                                   per chunk, then the state chain) with the per-chunk
                                   inverses in a caller workspace: bf16 q/k/v, dk = 128,
                                   dv a multiple of 64, and
                                   - the scalar rule at C = 64, all three inverse modes
                                     (Neumann N <= 15);
                                   - the scalar rule at C = 128 with the masked series
                                     (N <= 15): each 128-token chunk as two 64-token
                                     halves plus the band's corner (a third launch);
                                   - the two-gate rule at C = 64, exact or Neumann, with
                                     preconditioner form 0 or 1: the SIMT kernels' prep
                                     writes fp16 operands for the tensor-core chain
                                     (the preconditioner's running-average kernels
                                     first, when it is on) */
} gdn_kernel;

typedef struct {
    int32_t B, T, H;            /* batch, tokens (>= 1), heads */
    int32_t dk, dv;             /* key / value head dims: 16, 32, 64 or 128 */
    int32_t chunk;              /* C: 16, 32, 64 or 128 */
    int32_t io_dtype;           /* gdn_dtype of q, k, v, erase, write */
    int32_t o_dtype;            /* gdn_dtype of o */
    const void *q, *k, *v;
    const float *alpha;         /* decay in (0, 1]; NULL => 1 */
    int32_t alpha_per_channel;  /* 0: [B,T,H]; 1: [B,T,H,dk] */
    const float *beta;          /* write strength; NULL => 1 */
    int32_t precond;            /* diagonal curvature preconditioner, a per-channel factor
                                   f of rho_t = rho_decay rho_{t-1} + k_t (.) k_t:
                                   0 none; 1 f = 1/sqrt(rho + eps), erase read with the
                                   preconditioned key; 2 f = 1/(rho + eps) (P_t =
                                   Diag(A_t)^-1); 3 form 2 squashed into [1/x, x] on a
                                   log scale, x = precond_x ("Preconditioned DeltaNet",
                                   Arabic summary 2b; "Resumo Tecnico" section 2).
                                   Forms 2, 3 read the state with the raw key. */
    float rho_decay, rho_eps;   /* preconditioner EMA constant and epsilon */
    const void *erase;          /* erase gate b_t or NULL (=> 1); needs beta == NULL */
    const void *write;          /* write gate w_t or NULL (=> 1); needs beta == NULL */
    const float *S0;            /* initial state or NULL (=> 0) */
    void *o;                    /* output, caller-allocated */
    float *S_T;                 /* final state, caller-allocated, or NULL */
    int32_t mode;               /* gdn_inv_mode */
    int32_t neumann_N;          /* N for GDN_INV_NEUMANN: 0 <= N <= chunk - 1 */
    int32_t kernel;             /* gdn_kernel selection */
    int32_t dv_split;           /* value-axis slices per head (0 = choose) */
    void *workspace;            /* device scratch of >= gdn_workspace_bytes(args) bytes,
                                   16-byte aligned, caller-owned; may be NULL when that is 0 */
    uint64_t workspace_bytes;   /* size of workspace */
    int32_t residual_S;         /* S for GDN_INV_NEUMANN_RESIDUAL: 0 <= S <= 64 */
    float precond_x;            /* squash bound x > 1 for precond 3 */
    int32_t precond_query;      /* 1: apply the factor to the query (ATQ) instead of the
                                   write key (ATK); the write key is then k_t itself */
    int32_t seq_segments;       /* split tensor-core path, scalar rule, chunk 64, B = 1:
                                   0 = the library chooses (3 from 256 chunks when three
                                   rows of chains, H * dv / 64 each, fit the 148 SMs),
                                   1 = one pass over the chunks, 3 = three sequence
                                   segments (see gdn_select_segments) */
} gdn_fwd_args;

/* Chunkwise forward: o and S_T from q, k, v, gates and S0 (see above). */
GDN_API gdn_status gdn_chunk_fwd(const gdn_fwd_args *args, void *stream);

/* Workspace bytes gdn_chunk_fwd needs for these arguments (0 for the fused
 * and the recurrent kernels), or 0 with gdn_last_error() set if the arguments
 * are invalid.  Host only. */
GDN_API uint64_t gdn_workspace_bytes(const gdn_fwd_args *args);

/* Which kernel gdn_chunk_fwd would launch for these arguments (gdn_kernel
 * value, never AUTO), or a negative gdn_status if they are invalid.  Host
 * only; launches nothing. */
GDN_API int32_t gdn_select_kernel(const gdn_fwd_args *args);

/* Sequence segments gdn_chunk_fwd would use for these arguments (1 or 3), or
 * a negative gdn_status if they are invalid.  Host only; launches nothing.
 *
 * The state update is affine in the state (S_t = S_{t-1} alpha_t (I - beta_t
 * k_t k_t^T) + beta_t v_t k_t^T, "Resumo Tecnico: Preconditioned DeltaNet",
 * section 1), so over any run of chunks h_end = M h_start + N, with M the
 * run's d_k x d_k product of transitions (the run from h = I with v = 0) and N
 * its end state from h = 0.  With 3 segments s0, s1, s2 (s0 and s1 of
 * floor(chunks / 3) chunks each) the call runs, on three library-owned
 * high-priority streams joined back into `stream`: s0 from S0, s1 from 0 and
 * s1 with v = 0 from the identity side by side (the key-side kernel of s2
 * beside them on a fourth, low-priority stream); then h(s2) = M h(s1) + N and
 * s1, s2 from their true starts.  Two chain passes of a third of the chunks
 * each replace one over all of them: the serial chain per (head, value slice)
 * is the cost when B * H * dv / 64 chains fill few of the SMs.  The schedule
 * is this library's, not the pages'.  The workspace grows by
 * H * dk * (2 dk + 3 dv) floats (identity, M, N, two start states).  The
 * streams and events are made on the first such call on each device (with
 * that device current) and kept until exit; concurrent calls from several
 * host threads take turns enqueueing. */
GDN_API int32_t gdn_select_segments(const gdn_fwd_args *args);

/* Synchronises `stream` (void* cudaStream_t), then reports and clears a
 * failure recorded on the device by the kernels' own checks: a bounded wait
 * inside a tensor-core kernel that gave up (after about two seconds) makes
 * the block skip its remaining work and record an error code; this call then
 * returns GDN_ERR_DEVICE_CHECK.  GDN_ERR_CUDA if synchronising failed, else
 * GDN_OK. */
GDN_API gdn_status gdn_device_check(void *stream);

/* Inspection entry for tests: gdn_chunk_fwd on the fused tensor-core kernel
 * (it writes o and S_T exactly as that call does) that also copies the
 * 64 x 64 fp32 matrix T the kernel formed for chunk n of sequence (b, h)
 * into T_out: T = (I - A)^-1 in GDN_INV_EXACT mode, the masked truncated
 * Neumann series M^(N) (.) sum_{n<=N} A^n in GDN_INV_NEUMANN mode ("Quando o
 * 'Bom o Suficiente' e Otimo ...", section "Declaracao do Problema" and
 * section "Metodologia", items 1 and 2), as it stood before its rounding to
 * fp16 for the WY products.  A = -L with L_ri = beta_r e^{g_r - g_i}
 * (k_r . k_i), i < r, g the in-chunk cumulative log decay.
 *
 * T_out: DEVICE pointer, 4096 floats, 16-byte aligned, row-major (row = token
 * row of the chunk), written on `stream`.  In a tail chunk of Cv < 64 tokens,
 * rows and columns past Cv hold the identity.  Errors: GDN_ERR_INVALID_ARG for
 * (b, h, n) outside the call or a NULL T_out; GDN_ERR_UNSUPPORTED unless the
 * arguments select the fused kernel (kernel AUTO or TC); otherwise as
 * gdn_chunk_fwd. */
GDN_API gdn_status gdn_debug_chunk_T(const gdn_fwd_args *args, int32_t b, int32_t h, int32_t n, float *T_out,
                                     void *stream);

/* Static string for a status code. */
GDN_API const char *gdn_status_string(gdn_status s);

/* Message for the calling thread's most recent non-OK return ("" if none). */
GDN_API const char *gdn_last_error(void);

/* GDN_ABI_VERSION of the loaded library. */
GDN_API int32_t gdn_abi_version(void);

/* Size of the fixed device scratch array of gdn_chunk_fwd_static_scratch:
 * 24 MiB = 1024 chunk-heads of three 64 x 64 fp16 matrices each. */
#define GDN_STATIC_SCRATCH_BYTES (24ull << 20)

/* ------------------------------------------------------------ backward pass
 *
 * Gradient of the gated delta rule (the default rule above: scalar decay
 * alpha, scalar beta; exact inverse, or the truncated series of the forward's
 * Neumann modes) with respect to q, k, v, alpha, beta and
 * S0, given dL/do and dL/dS_T.  The pages use chunkwise forms to make
 * training parallel ("Quando o 'Bom o Suficiente' e Otimo ...", sections
 * "Resumo" and "Declaracao do Problema") but print no backward pass; this is
 * the reverse-mode derivative of the chunked WY/UT form, fp32 on CUDA cores,
 * in four launches (five with the truncated series, below):
 *   1. per chunk-head: g, L, T = (I + L)^-1, the causal scores M, W, U, and the
 *      state-independent M^T dO and (diag(e^g) Q)^T dO;
 *   2. per 32-column value slice, chunks in order: the state at every chunk
 *      start and Delta = U - W h;
 *   3. per slice, chunks in reverse: dL/dh at every chunk end, Y = T^T dDelta,
 *      dv and dS0;
 *   4. per chunk-head: dq, dk, dbeta, dalpha.
 * The forward is recomputed inside the call (only S0 is taken from the
 * caller), so the call needs no saved activations.
 *
 * With mode GDN_INV_NEUMANN it is the gradient of the forward whose chunk
 * inverse is the masked truncated series T_N = M^(N) (.) sum_{n<=N} A^n (same
 * page, section "Metodologia", items 1 and 2): launch 1 forms T_N (on the band
 * it equals the exact inverse, off it the mask gives zero) and keeps the exact
 * inverse, and a launch between 3 and 4 forms, per chunk-head,
 * dA = T^T (M (.) dT_N) T^T with dT_N = T_N^-T (Y Delta^T) T_N^-T, the gradient
 * reaching A = -L through the series (the workspace grows by C x C floats per
 * chunk-head).  With GDN_INV_NEUMANN_RESIDUAL (same section, item 3) the
 * forward's inverse T0 sum_{s<=S} E^s equals T - T_out E^S (T_out the part of the
 * exact T below the band, E = T^-1 T_out); launch 1 forms it with 2 S products
 * per chunk-head and the extra launch applies the adjoint of that form
 * (3 S + 9 products).
 *
 * Layouts as gdn_fwd_args; every gradient is fp32 in the layout of its input
 * (grad_S0 and grad_S_T in the h = S^T layout [B, H, dk, dv]).
 *
 * Shapes: chunk 16, 32 or 64; dk 16, 32, 64 or 128; dv 32, 64, 96 or 128;
 * B, H <= 65535.  Other shapes return GDN_ERR_UNSUPPORTED.
 *
 * Ownership and errors as gdn_chunk_fwd: caller-allocated device buffers,
 * host-side validation before any launch, asynchronous on `stream`.  The
 * outputs must not alias the inputs or one another; every output pointer
 * given is written in full.  alpha must be in (0, 1] (its logarithm is taken).
 */
typedef struct {
    int32_t B, T, H, dk, dv, chunk;
    int32_t io_dtype;           /* gdn_dtype of q, k, v */
    int32_t do_dtype;           /* gdn_dtype of grad_o */
    const void *q, *k, *v;      /* [B,T,H,dk|dv] */
    const float *alpha;         /* [B,T,H] in (0, 1], or NULL (=> 1) */
    const float *beta;          /* [B,T,H], or NULL (=> 1) */
    const float *S0;            /* [B,H,dk,dv] fp32, or NULL (=> 0) */
    const void *grad_o;         /* [B,T,H,dv] dL/do, required */
    const float *grad_S_T;      /* [B,H,dk,dv] fp32 dL/dS_T, or NULL (=> 0) */
    float *grad_q, *grad_k;     /* [B,T,H,dk] fp32, required */
    float *grad_v;              /* [B,T,H,dv] fp32, required */
    float *grad_alpha;          /* [B,T,H] fp32 or NULL; NULL when alpha is NULL */
    float *grad_beta;           /* [B,T,H] fp32 or NULL; NULL when beta is NULL */
    float *grad_S0;             /* [B,H,dk,dv] fp32 or NULL */
    void *workspace;            /* >= gdn_bwd_workspace_bytes(args) bytes, 16-byte aligned */
    uint64_t workspace_bytes;
    int32_t mode;               /* the chunk inverse of the forward being differentiated:
                                   GDN_INV_EXACT, GDN_INV_NEUMANN (the masked truncated
                                   series of order neumann_N, 0 <= N <= chunk - 1), or
                                   GDN_INV_NEUMANN_RESIDUAL (that series corrected with
                                   residual_S terms) */
    int32_t neumann_N;
    int32_t residual_S;         /* GDN_INV_NEUMANN_RESIDUAL: the series of order neumann_N
                                   with residual_S (0..64) correction terms */
} gdn_bwd_args;

/* Backward pass (see above). */
GDN_API gdn_status gdn_chunk_bwd(const gdn_bwd_args *args, void *stream);

/* Workspace bytes gdn_chunk_bwd needs: per chunk-head, fp32 g (C), T, the
 * decayed Gram and the causal scores (C x C each), W (C x dk), U / Delta and
 * M^T dO / Y (C x dv each), (diag(e^g) Q)^T dO, the state and its gradient
 * (dk x dv each); 0 with gdn_last_error() set if the arguments are invalid.
 * Host only. */
GDN_API uint64_t gdn_bwd_workspace_bytes(const gdn_bwd_args *args);

/* gdn_chunk_fwd on the split tensor-core kernels (GDN_KERNEL_TC_SPLIT), with
 * a fixed scratch array inside the library in place of args->workspace.  The pages have no counterpart:
 * this is a calling convenience of this library, not a step of the method.
 *
 * For callers that cannot allocate device memory per call: a plain C host
 * program that links only this library and the CUDA runtime and holds no
 * allocator, or a serving loop that must not call cudaMalloc after start-up
 * (cudaMalloc and cudaFree may synchronise the device).  The call allocates
 * nothing (no cudaMalloc, cudaFree or allocating library routine).
 *
 * Arguments as gdn_chunk_fwd, except: args->workspace must be NULL and
 * args->workspace_bytes 0; the call runs one pass over the chunks (seq_segments
 * 3 returns GDN_ERR_UNSUPPORTED, 0 means one pass here); args->kernel must be
 * AUTO, TC or TC_SPLIT and the shape one the split tensor-core kernels support,
 * else GDN_ERR_UNSUPPORTED (whatever the kernel field, this entry point runs
 * the split kernels); and the workspace the call needs there
 * (gdn_workspace_bytes with kernel TC_SPLIT and seq_segments 1:
 * B * H * ceil(T / 64) * 24576 for the scalar rule at C = 64) must
 * be <= GDN_STATIC_SCRATCH_BYTES, else GDN_ERR_INVALID_ARG with the needed
 * size in gdn_last_error().  Nothing in the scratch has to start at zero: the
 * call's first kernels write every entry the chain kernel reads.
 *
 * Set-up: the first call on each device, with that device current, looks up
 * the array's address with cudaGetSymbolAddress (an error there returns
 * GDN_ERR_CUDA).  Make that first call before any stream capture.
 *
 * One scratch per device: calls that overlap in time on one device (from
 * different streams or threads) race on it and give wrong results.  Calls
 * ordered on one stream are safe. */
GDN_API gdn_status gdn_chunk_fwd_static_scratch(const gdn_fwd_args *args, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
