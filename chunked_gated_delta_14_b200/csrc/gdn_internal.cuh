// Internal declarations shared by the launchers of libgdn.so.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "gdn.h"

namespace gdn {

// Everything a kernel needs, resolved from gdn_fwd_args by the host layer.
struct FwdParams {
    int B, T, H, dk, dv, C;
    int dvs;            // value columns per block (dv / slices)
    int slices;
    int io_bf16, o_bf16;
    const void *q, *k, *v;
    const float *alpha;
    int alpha_pc;
    const float *beta;
    int precond;        // 0 none, 1 1/sqrt(rho+eps), 2 1/(rho+eps), 3 the latter squashed
    float rho_decay, rho_eps;
    float precond_x;    // squash bound x (precond 3)
    int precond_query;  // 1: factor on the query (ATQ) instead of the write key
    const void *erase, *write;
    const float *S0;
    void *o;
    float *S_T;
    int mode, N;
    int S;              // residual-correction terms (GDN_INV_NEUMANN_RESIDUAL)
    int general;        // two-gate rule (per-channel decay / gates / preconditioner)
    int segments;       // split tensor-core path: 1 one pass, 3 three sequence segments
};

// SIMT fp32 chunk kernel: shared-memory bytes for p, or 0 if p does not fit.
// Token-by-token kernel (decode steps): chosen automatically for T <= kRecurrentMaxT.
constexpr int kRecurrentMaxT = 8;
bool recurrent_supports(const FwdParams &p, const char **why);
cudaError_t launch_recurrent(const FwdParams &p, cudaStream_t stream);

size_t simt_smem_bytes(const FwdParams &p);
// Workspace of the SIMT path: per chunk-head the state-independent matrices
// (fp32), plus the preconditioner's running average at chunk starts.
size_t simt_workspace_bytes(const FwdParams &p);
cudaError_t launch_simt(const FwdParams &p, void *workspace, cudaStream_t stream);

// The two-gate rule on the tensor-core chain: the SIMT prep kernel's matrices as
// fp16 rows of 64 (128 B) per chunk-head, ready for the chain kernel's TMA loads.
// TB, P and U = w (.) v go as hi/lo fp16 pairs (x = hi + lo to about 2^-22): with
// the preconditioned write keys the first tokens' outputs are hundreds of times
// the sequence's RMS, and one fp16 rounding of those operands would leave the
// accuracy bar there.  E, Q', K'' are 64-column blocks (channels 0..63, 64..127),
// U one block per 64 value columns, d (the state's decay) fp32.  Chunk 64, d_k 128.
struct GenRows {
    int tb, tbl, pp, ppl, e, q, k, u, ul, d, rows;
};
__host__ __device__ inline GenRows gen_rows(int dv) {
    GenRows g;
    g.tb = 0; g.tbl = 64; g.pp = 128; g.ppl = 192; g.e = 256; g.q = 384; g.k = 512; g.u = 640;
    g.ul = 640 + dv; g.d = 640 + 2 * dv; g.rows = g.d + 4;
    return g;
}
// Workspace of that prep (rows for every chunk-head, then the preconditioner's
// running averages) and its launch: the running-average kernels and the prep.
size_t gen_prep_workspace_bytes(const FwdParams &p);
cudaError_t launch_gen_prep(const FwdParams &p, void *workspace, cudaStream_t stream);

// Tensor-core kernel (tcgen05 / TMEM / TMA).
bool tc_supports(const FwdParams &p, const char **why);
int tc_default_slices(const FwdParams &p);
size_t tc_workspace_bytes(const FwdParams &p);
// Sequence segments of the split path (B = 1, scalar rule, chunk 64): whether p
// allows them, and the count chosen when the caller leaves it to the library.
bool tc_segments_support(const FwdParams &p, const char **why);
int tc_auto_segments(const FwdParams &p);
cudaError_t launch_tc(const FwdParams &p, void *workspace, cudaStream_t stream, const char **why);
// Synchronise `stream`, return (and clear) the tensor-core kernel's error word.
unsigned int tc_read_and_clear_error(cudaStream_t stream, cudaError_t *err);

// Fused tensor-core kernel: one 2-CTA cluster per (batch, head), no workspace.
bool fused_supports(const FwdParams &p, const char **why);
// dbg_T (device, 64 x 64 fp32) receives the T of chunk dbg_n of (dbg_b, dbg_h) when non-NULL.
cudaError_t launch_fused(const FwdParams &p, cudaStream_t stream, const char **why, float *dbg_T = nullptr,
                         int dbg_b = 0, int dbg_h = 0, int dbg_n = 0);
// Return (and clear) the fused kernel's error word; the caller has synchronised.
unsigned int fused_read_and_clear_error(cudaError_t *err);

}  // namespace gdn
