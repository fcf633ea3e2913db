// Host side of libgdn.so: argument validation, kernel selection, launch.
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "gdn_bwd.cuh"
#include "gdn_internal.cuh"

// Fixed scratch of gdn_chunk_fwd_static_scratch: the per-chunk T matrices of
// the tensor-core path (24 KiB per chunk-head), GDN_STATIC_SCRATCH_BYTES in all.
static __device__ __align__(256) unsigned char gdn_static_scratch[GDN_STATIC_SCRATCH_BYTES];

namespace {

thread_local char g_msg[512] = "";

gdn_status fail(gdn_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    if (getenv("GDN_LOG")) fprintf(stderr, "[gdn] %s: %s\n", gdn_status_string(s), g_msg);
    return s;
}

bool pow2_in(int x, int lo, int hi) { return x >= lo && x <= hi && (x & (x - 1)) == 0; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validate and resolve; on success fills *out.  Never touches the GPU.
gdn_status resolve(const gdn_fwd_args *a, gdn::FwdParams *out, int *kernel) {
    if (!a) return fail(GDN_ERR_INVALID_ARG, "args is NULL");
    if (a->B < 1 || a->H < 1 || a->T < 1)
        return fail(GDN_ERR_INVALID_ARG, "B, T, H must be >= 1 (got %d, %d, %d)", a->B, a->T, a->H);
    if ((long long)a->B * a->T * a->H > (1ll << 40))
        return fail(GDN_ERR_INVALID_ARG, "B*T*H too large");
    if (!pow2_in(a->dk, 16, 128) || !pow2_in(a->dv, 16, 128))
        return fail(GDN_ERR_INVALID_ARG, "dk, dv must be 16, 32, 64 or 128 (got %d, %d)", a->dk, a->dv);
    if (!pow2_in(a->chunk, 16, 128))
        return fail(GDN_ERR_INVALID_ARG, "chunk must be 16, 32, 64 or 128 (got %d)", a->chunk);
    if (a->io_dtype != GDN_F32 && a->io_dtype != GDN_BF16)
        return fail(GDN_ERR_INVALID_ARG, "io_dtype %d unknown", a->io_dtype);
    if (a->o_dtype != GDN_F32 && a->o_dtype != GDN_BF16)
        return fail(GDN_ERR_INVALID_ARG, "o_dtype %d unknown", a->o_dtype);
    if (!a->q || !a->k || !a->v || !a->o)
        return fail(GDN_ERR_INVALID_ARG, "q, k, v and o are required");
    if (a->mode != GDN_INV_EXACT && a->mode != GDN_INV_NEUMANN && a->mode != GDN_INV_NEUMANN_RESIDUAL)
        return fail(GDN_ERR_INVALID_ARG, "mode %d unknown", a->mode);
    if (a->mode != GDN_INV_EXACT && (a->neumann_N < 0 || a->neumann_N > a->chunk - 1))
        return fail(GDN_ERR_INVALID_ARG, "neumann_N must be in [0, chunk-1] (got %d)", a->neumann_N);
    if (a->mode == GDN_INV_NEUMANN_RESIDUAL && (a->residual_S < 0 || a->residual_S > 64))
        return fail(GDN_ERR_INVALID_ARG, "residual_S must be in [0, 64] (got %d)", a->residual_S);
    if (a->mode != GDN_INV_EXACT && (a->neumann_N < 0 || a->neumann_N > a->chunk - 1))
        return fail(GDN_ERR_INVALID_ARG, "neumann_N must be in [0, chunk-1] (got %d)", a->neumann_N);
    if (a->alpha_per_channel && !a->alpha)
        return fail(GDN_ERR_INVALID_ARG, "alpha_per_channel needs alpha");
    if (a->alpha_per_channel != 0 && a->alpha_per_channel != 1)
        return fail(GDN_ERR_INVALID_ARG, "alpha_per_channel must be 0 or 1");
    if (a->precond < 0 || a->precond > 3)
        return fail(GDN_ERR_INVALID_ARG, "precond must be 0, 1, 2 or 3 (got %d)", a->precond);
    if (a->precond == 3 && !(a->precond_x > 1.f))
        return fail(GDN_ERR_INVALID_ARG, "precond 3 needs precond_x > 1 (got %g)", (double)a->precond_x);
    if (a->precond_query != 0 && a->precond_query != 1)
        return fail(GDN_ERR_INVALID_ARG, "precond_query must be 0 or 1");
    if (a->precond_query && !a->precond)
        return fail(GDN_ERR_INVALID_ARG, "precond_query needs a preconditioner (precond 1, 2 or 3)");
    const int general = a->alpha_per_channel || a->precond || a->erase || a->write;
    if (general && a->beta)
        return fail(GDN_ERR_INVALID_ARG,
                    "beta must be NULL with the two-gate rule (erase/write/precond/per-channel alpha)");
    if (a->precond && !(a->rho_eps > 0.f && a->rho_decay >= 0.f))
        return fail(GDN_ERR_INVALID_ARG, "precond needs rho_eps > 0 and rho_decay >= 0");
    const void *ins[] = {a->q, a->k, a->v, a->alpha, a->beta, a->erase, a->write, a->S0};
    for (const void *x : ins)
        if (x && x == a->o) return fail(GDN_ERR_INVALID_ARG, "o aliases an input");
    if (a->S_T && (const void *)a->S_T == a->o) return fail(GDN_ERR_INVALID_ARG, "o aliases S_T");
    const void *al[] = {a->q, a->k, a->v, a->o, a->erase, a->write, a->S0, a->S_T, a->alpha, a->beta,
                        a->workspace};
    for (const void *x : al)
        if (x && !aligned16(x)) return fail(GDN_ERR_ALIGNMENT, "pointers must be 16-byte aligned");
    if (a->kernel < GDN_KERNEL_AUTO || a->kernel > GDN_KERNEL_TC_SPLIT)
        return fail(GDN_ERR_INVALID_ARG, "kernel %d unknown", a->kernel);
    if (a->dv_split < 0 || (a->dv_split > 0 && (a->dv % a->dv_split != 0 || a->dv / a->dv_split < 16)))
        return fail(GDN_ERR_INVALID_ARG, "dv_split must divide dv into slices of >= 16 columns");
    if (a->seq_segments != 0 && a->seq_segments != 1 && a->seq_segments != 3)
        return fail(GDN_ERR_INVALID_ARG, "seq_segments must be 0, 1 or 3 (got %d)", a->seq_segments);

    gdn::FwdParams p{};
    p.B = a->B; p.T = a->T; p.H = a->H; p.dk = a->dk; p.dv = a->dv; p.C = a->chunk;
    p.io_bf16 = a->io_dtype == GDN_BF16;
    p.o_bf16 = a->o_dtype == GDN_BF16;
    p.q = a->q; p.k = a->k; p.v = a->v;
    p.alpha = a->alpha; p.alpha_pc = a->alpha_per_channel; p.beta = a->beta;
    p.precond = a->precond; p.precond_x = a->precond_x; p.precond_query = a->precond_query; p.rho_decay = a->rho_decay; p.rho_eps = a->rho_eps;
    p.erase = a->erase; p.write = a->write; p.S0 = a->S0; p.o = a->o; p.S_T = a->S_T;
    p.mode = a->mode; p.N = a->mode != GDN_INV_EXACT ? a->neumann_N : 0;
    p.S = a->mode == GDN_INV_NEUMANN_RESIDUAL ? a->residual_S : 0;
    p.general = general;

    const char *why = "";
    int kern = a->kernel;
    if (kern == GDN_KERNEL_AUTO && p.T <= gdn::kRecurrentMaxT && gdn::recurrent_supports(p, &why)) {
        // a few tokens (decode steps): the token recurrence beats any chunked form
        kern = GDN_KERNEL_RECURRENT;
    } else if (kern == GDN_KERNEL_AUTO) {
        // the split tensor-core kernels (the faster path on B200 at these shapes),
        // else the fused one, else the SIMT kernel
        gdn::FwdParams t = p;
        kern = GDN_KERNEL_SIMT;
        if (gdn::tc_supports(t, &why)) {
            t.slices = a->dv_split ? a->dv_split : gdn::tc_default_slices(t);
            t.dvs = t.dv / t.slices;
            if (t.dv % t.slices == 0 && gdn::tc_supports(t, &why)) kern = GDN_KERNEL_TC_SPLIT;
        }
        if (kern == GDN_KERNEL_SIMT && a->dv_split <= 1 && gdn::fused_supports(p, &why)) kern = GDN_KERNEL_TC;
    }
    p.segments = 1;
    if (a->seq_segments == 3 && kern != GDN_KERNEL_TC_SPLIT)
        return fail(GDN_ERR_UNSUPPORTED, "seq_segments 3 runs on the split tensor-core kernels only");
    if (kern == GDN_KERNEL_RECURRENT) {
        if (!gdn::recurrent_supports(p, &why))
            return fail(GDN_ERR_UNSUPPORTED, "recurrent kernel: %s", why);
        p.slices = p.dv / 32;
        p.dvs = 32;
    } else if (kern == GDN_KERNEL_TC) {
        if (a->dv_split > 1) return fail(GDN_ERR_UNSUPPORTED, "fused tensor-core kernel: dv_split must be 0 or 1");
        if (!gdn::fused_supports(p, &why))
            return fail(GDN_ERR_UNSUPPORTED, "fused tensor-core kernel: %s", why);
        p.slices = 1;
        p.dvs = p.dv;
    } else if (kern == GDN_KERNEL_TC_SPLIT) {
        if (!gdn::tc_supports(p, &why))
            return fail(GDN_ERR_UNSUPPORTED, "split tensor-core kernels: %s", why);
        p.slices = a->dv_split ? a->dv_split : gdn::tc_default_slices(p);
        if (p.dv % p.slices) return fail(GDN_ERR_UNSUPPORTED, "dv_split does not divide dv");
        p.dvs = p.dv / p.slices;
        if (!gdn::tc_supports(p, &why))
            return fail(GDN_ERR_UNSUPPORTED, "split tensor-core kernels: %s", why);
        // Exact inversion at chunk 128 as two 64-token chunks: T = (I - A)^-1 of a
        // 128-token chunk is block lower triangular with the two halves' inverses on
        // its diagonal, and its off-diagonal block is what the state carried from
        // the first half to the second applies, so o and S_T are those of chunk 64.
        if (p.C == 128 && p.mode == GDN_INV_EXACT && !p.general) p.C = 64;
        if (a->seq_segments == 3 && !gdn::tc_segments_support(p, &why))
            return fail(GDN_ERR_UNSUPPORTED, "split tensor-core kernels: %s", why);
        p.segments = a->seq_segments ? a->seq_segments : gdn::tc_auto_segments(p);
    } else {
        if (p.mode == GDN_INV_NEUMANN_RESIDUAL)
            return fail(GDN_ERR_UNSUPPORTED,
                        "residual correction runs on the split tensor-core kernels only (bf16 q/k/v, "
                        "scalar decay, chunk 64, dk 128)%s%s", why[0] ? ": " : "", why);
        // SIMT: widest value slice that fits shared memory, at least
        // ~one block per SM where the problem allows it.
        int slices = a->dv_split;
        if (!slices) {
            slices = 1;
            while (p.dv / (slices * 2) >= 16 && (long long)p.B * p.H * slices < 148) slices *= 2;
        }
        for (;;) {
            p.slices = slices;
            p.dvs = p.dv / slices;
            if (gdn::simt_smem_bytes(p) <= 227 * 1024) break;
            if (a->dv_split || p.dvs <= 16)
                return fail(GDN_ERR_UNSUPPORTED,
                            "SIMT kernel: chunk %d, dk %d, value slice %d needs %zu B of shared memory",
                            p.C, p.dk, p.dvs, gdn::simt_smem_bytes(p));
            slices *= 2;
        }
    }
    *out = p;
    *kernel = kern;
    return GDN_OK;
}

struct Span {
    const void *p;
    size_t bytes;
};

bool overlap(const Span &a, const Span &b) {
    if (!a.p || !b.p || !a.bytes || !b.bytes) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a.p), y = reinterpret_cast<uintptr_t>(b.p);
    return x < y + b.bytes && y < x + a.bytes;
}

// Validate the backward arguments; on success fills *out (workspace regions
// not yet carved).  Never touches the GPU.
gdn_status resolve_bwd(const gdn_bwd_args *a, gdn::BwdParams *out) {
    if (!a) return fail(GDN_ERR_INVALID_ARG, "args is NULL");
    if (a->B < 1 || a->H < 1 || a->T < 1)
        return fail(GDN_ERR_INVALID_ARG, "B, T, H must be >= 1 (got %d, %d, %d)", a->B, a->T, a->H);
    if (a->B > 65535 || a->H > 65535)
        return fail(GDN_ERR_INVALID_ARG, "B and H must be <= 65535 (got %d, %d)", a->B, a->H);
    if ((long long)a->B * a->T * a->H > (1ll << 40)) return fail(GDN_ERR_INVALID_ARG, "B*T*H too large");
    if (a->io_dtype != GDN_F32 && a->io_dtype != GDN_BF16)
        return fail(GDN_ERR_INVALID_ARG, "io_dtype %d unknown", a->io_dtype);
    if (a->do_dtype != GDN_F32 && a->do_dtype != GDN_BF16)
        return fail(GDN_ERR_INVALID_ARG, "do_dtype %d unknown", a->do_dtype);
    if (!a->q || !a->k || !a->v || !a->grad_o)
        return fail(GDN_ERR_INVALID_ARG, "q, k, v and grad_o are required");
    if (!a->grad_q || !a->grad_k || !a->grad_v)
        return fail(GDN_ERR_INVALID_ARG, "grad_q, grad_k and grad_v are required");
    if (a->grad_alpha && !a->alpha) return fail(GDN_ERR_INVALID_ARG, "grad_alpha needs alpha");
    if (a->grad_beta && !a->beta) return fail(GDN_ERR_INVALID_ARG, "grad_beta needs beta");
    if (a->mode != GDN_INV_EXACT && a->mode != GDN_INV_NEUMANN && a->mode != GDN_INV_NEUMANN_RESIDUAL)
        return fail(GDN_ERR_INVALID_ARG, "backward mode %d unknown", a->mode);
    if (a->mode == GDN_INV_NEUMANN_RESIDUAL && (a->residual_S < 0 || a->residual_S > 64))
        return fail(GDN_ERR_INVALID_ARG, "residual_S must be in [0, 64] (got %d)", a->residual_S);
    if (a->mode != GDN_INV_EXACT && (a->neumann_N < 0 || a->neumann_N > a->chunk - 1))
        return fail(GDN_ERR_INVALID_ARG, "neumann_N must be in [0, chunk-1] (got %d)", a->neumann_N);
    gdn::BwdParams p{};
    p.B = a->B; p.T = a->T; p.H = a->H; p.dk = a->dk; p.dv = a->dv; p.C = a->chunk;
    p.NC = (a->T + a->chunk - 1) / (a->chunk > 0 ? a->chunk : 1);
    p.neumann = a->mode == GDN_INV_NEUMANN || a->mode == GDN_INV_NEUMANN_RESIDUAL;
    p.N = p.neumann ? a->neumann_N : 0;
    // S = 0 terms of the correction leave the masked series itself
    p.residual = a->mode == GDN_INV_NEUMANN_RESIDUAL && a->residual_S > 0;
    p.S = p.residual ? a->residual_S : 0;
    const char *why = "";
    if (!gdn::bwd_supports(p, &why)) return fail(GDN_ERR_UNSUPPORTED, "backward: %s", why);

    const size_t tok = (size_t)a->B * a->T * a->H;
    const size_t io = a->io_dtype == GDN_BF16 ? 2 : 4, od = a->do_dtype == GDN_BF16 ? 2 : 4;
    const size_t st = (size_t)a->B * a->H * a->dk * a->dv * 4;
    const size_t ws = gdn::bwd_workspace_bytes(p);
    const Span ins[] = {{a->q, tok * a->dk * io}, {a->k, tok * a->dk * io}, {a->v, tok * a->dv * io},
                        {a->alpha, tok * 4}, {a->beta, tok * 4}, {a->S0, st},
                        {a->grad_o, tok * a->dv * od}, {a->grad_S_T, st}};
    const Span outs[] = {{a->grad_q, tok * a->dk * 4}, {a->grad_k, tok * a->dk * 4},
                         {a->grad_v, tok * a->dv * 4}, {a->grad_alpha, tok * 4},
                         {a->grad_beta, tok * 4}, {a->grad_S0, st},
                         {a->workspace, a->workspace ? ws : 0}};
    const int n_out = (int)(sizeof(outs) / sizeof(outs[0]));
    for (int i = 0; i < n_out; ++i) {
        for (const Span &x : ins)
            if (overlap(outs[i], x)) return fail(GDN_ERR_INVALID_ARG, "an output or the workspace overlaps an input");
        for (int j = i + 1; j < n_out; ++j)
            if (overlap(outs[i], outs[j]))
                return fail(GDN_ERR_INVALID_ARG, "outputs (or the workspace) overlap one another");
    }
    for (const Span &x : ins)
        if (x.p && !aligned16(x.p)) return fail(GDN_ERR_ALIGNMENT, "pointers must be 16-byte aligned");
    for (const Span &x : outs)
        if (x.p && !aligned16(x.p)) return fail(GDN_ERR_ALIGNMENT, "pointers must be 16-byte aligned");

    p.io_bf16 = a->io_dtype == GDN_BF16;
    p.do_bf16 = a->do_dtype == GDN_BF16;
    p.q = a->q; p.k = a->k; p.v = a->v; p.alpha = a->alpha; p.beta = a->beta; p.S0 = a->S0;
    p.grad_o = a->grad_o; p.grad_S_T = a->grad_S_T;
    p.grad_q = a->grad_q; p.grad_k = a->grad_k; p.grad_v = a->grad_v;
    p.grad_alpha = a->grad_alpha; p.grad_beta = a->grad_beta; p.grad_S0 = a->grad_S0;
    *out = p;
    return GDN_OK;
}

}  // namespace

extern "C" {

const char *gdn_status_string(gdn_status s) {
    switch (s) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
        case GDN_ERR_ALIGNMENT: return "GDN_ERR_ALIGNMENT";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_DEVICE_CHECK: return "GDN_ERR_DEVICE_CHECK";
        case GDN_ERR_FAULT_INJECTED: return "GDN_ERR_FAULT_INJECTED";
    }
    return "GDN_UNKNOWN_STATUS";
}

const char *gdn_last_error(void) { return g_msg; }

int32_t gdn_abi_version(void) { return GDN_ABI_VERSION; }

uint64_t gdn_workspace_bytes(const gdn_fwd_args *args) {
    gdn::FwdParams p;
    int kern = 0;
    if (resolve(args, &p, &kern) != GDN_OK) return 0;
    g_msg[0] = 0;
    if (kern == GDN_KERNEL_TC_SPLIT) return (uint64_t)gdn::tc_workspace_bytes(p);
    if (kern == GDN_KERNEL_SIMT) return (uint64_t)gdn::simt_workspace_bytes(p);
    return 0;
}

int32_t gdn_select_kernel(const gdn_fwd_args *args) {
    gdn::FwdParams p;
    int kern = 0;
    gdn_status s = resolve(args, &p, &kern);
    if (s != GDN_OK) return -(int32_t)s;
    g_msg[0] = 0;
    return kern;
}

int32_t gdn_select_segments(const gdn_fwd_args *args) {
    gdn::FwdParams p;
    int kern = 0;
    gdn_status s = resolve(args, &p, &kern);
    if (s != GDN_OK) return -(int32_t)s;
    g_msg[0] = 0;
    return p.segments;
}

gdn_status gdn_device_check(void *stream) {
    cudaError_t e = cudaSuccess;
    const unsigned int code = gdn::tc_read_and_clear_error(reinterpret_cast<cudaStream_t>(stream), &e);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "device check: %s", cudaGetErrorString(e));
    const unsigned int fcode = gdn::fused_read_and_clear_error(&e);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "device check: %s", cudaGetErrorString(e));
    if (code) return fail(GDN_ERR_DEVICE_CHECK, "split tensor-core kernel wait %u gave up", code);
    if (fcode) return fail(GDN_ERR_DEVICE_CHECK, "fused tensor-core kernel wait %u gave up", fcode);
    g_msg[0] = 0;
    return GDN_OK;
}

gdn_status gdn_chunk_fwd(const gdn_fwd_args *args, void *stream) {
    const char *inj = getenv("GDN_FAULT_INJECT");
    if (inj && inj[0] == '1') return fail(GDN_ERR_FAULT_INJECTED, "GDN_FAULT_INJECT=1");
    gdn::FwdParams p;
    int kern = 0;
    gdn_status s = resolve(args, &p, &kern);
    if (s != GDN_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    const char *why = "";
    if (kern == GDN_KERNEL_TC) {
        e = gdn::launch_fused(p, st, &why);
    } else if (kern == GDN_KERNEL_TC_SPLIT) {
        const size_t need = gdn::tc_workspace_bytes(p);
        if (!args->workspace || args->workspace_bytes < need)
            return fail(GDN_ERR_INVALID_ARG, "split tensor-core kernels need a workspace of %zu bytes (got %llu)",
                        need, (unsigned long long)args->workspace_bytes);
        e = gdn::launch_tc(p, args->workspace, st, &why);
    } else if (kern == GDN_KERNEL_RECURRENT) {
        e = gdn::launch_recurrent(p, st);
    } else {
        const size_t need = gdn::simt_workspace_bytes(p);
        if (!args->workspace || args->workspace_bytes < need)
            return fail(GDN_ERR_INVALID_ARG, "the SIMT kernels need a workspace of %zu bytes (got %llu)", need,
                        (unsigned long long)args->workspace_bytes);
        e = gdn::launch_simt(p, args->workspace, st);
    }
    if (e != cudaSuccess)
        return fail(GDN_ERR_CUDA, "%s launch: %s %s",
                    kern == GDN_KERNEL_TC ? "tc" : kern == GDN_KERNEL_TC_SPLIT ? "tc_split"
                    : (kern == GDN_KERNEL_RECURRENT ? "recurrent" : "simt"),
                    cudaGetErrorString(e), why);
    g_msg[0] = 0;
    return GDN_OK;
}

// Tensor-core path with the file's fixed scratch array in place of a caller
// workspace: nothing is allocated.  The array's device address is looked up
// once per device, with that device current, on the first call made there.
gdn_status gdn_chunk_fwd_static_scratch(const gdn_fwd_args *args, void *stream) {
    if (!args) return fail(GDN_ERR_INVALID_ARG, "args is NULL");
    if (args->kernel != GDN_KERNEL_AUTO && args->kernel != GDN_KERNEL_TC && args->kernel != GDN_KERNEL_TC_SPLIT)
        return fail(GDN_ERR_UNSUPPORTED, "the fixed-scratch entry point runs the split tensor-core kernels only");
    gdn_fwd_args a = *args;
    a.kernel = GDN_KERNEL_TC_SPLIT;
    gdn::FwdParams p;
    int kern = 0;
    gdn_status s = resolve(&a, &p, &kern);
    if (s != GDN_OK) return s;
    if (args->workspace || args->workspace_bytes)
        return fail(GDN_ERR_INVALID_ARG, "the fixed-scratch entry point takes no workspace (pass NULL, 0)");
    if (args->seq_segments == 3)
        return fail(GDN_ERR_UNSUPPORTED, "the fixed-scratch entry point runs one pass over the chunks (seq_segments 0 or 1)");
    p.segments = 1;     // one pass: the segment schedule's streams and states are not for this entry
    const size_t need = gdn::tc_workspace_bytes(p);
    if (need > (size_t)GDN_STATIC_SCRATCH_BYTES)
        return fail(GDN_ERR_INVALID_ARG,
                    "needs %zu bytes of scratch (gdn_workspace_bytes of the split tensor-core kernels); "
                    "the fixed array holds %llu bytes",
                    need, (unsigned long long)GDN_STATIC_SCRATCH_BYTES);
    constexpr int kMaxDevices = 64;
    static void *dev_ptr[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(GDN_ERR_UNSUPPORTED, "device index %d >= %d", dev, kMaxDevices);
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!dev_ptr[dev]) {
            void *ptr = nullptr;
            e = cudaGetSymbolAddress(&ptr, gdn_static_scratch);
            if (e != cudaSuccess)
                return fail(GDN_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
            dev_ptr[dev] = ptr;
        }
        scratch = dev_ptr[dev];
    }
    const char *why = "";
    e = gdn::launch_tc(p, scratch, reinterpret_cast<cudaStream_t>(stream), &why);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "tc launch: %s %s", cudaGetErrorString(e), why);
    g_msg[0] = 0;
    return GDN_OK;
}

gdn_status gdn_debug_chunk_T(const gdn_fwd_args *args, int32_t b, int32_t h, int32_t n, float *T_out,
                             void *stream) {
    if (!args) return fail(GDN_ERR_INVALID_ARG, "args is NULL");
    gdn_fwd_args a = *args;
    if (a.kernel == GDN_KERNEL_AUTO) a.kernel = GDN_KERNEL_TC;   // this entry inspects the fused kernel
    gdn::FwdParams p;
    int kern = 0;
    gdn_status s = resolve(&a, &p, &kern);
    if (s != GDN_OK) return s;
    if (kern != GDN_KERNEL_TC)
        return fail(GDN_ERR_UNSUPPORTED, "gdn_debug_chunk_T inspects the fused tensor-core kernel only "
                                         "(bf16 q/k/v, scalar decay, chunk 64, dk = dv = 128)");
    const int NC = (p.T + p.C - 1) / p.C;
    if (b < 0 || b >= p.B || h < 0 || h >= p.H || n < 0 || n >= NC)
        return fail(GDN_ERR_INVALID_ARG, "(b, h, n) = (%d, %d, %d) outside B = %d, H = %d, %d chunks", b, h, n,
                    p.B, p.H, NC);
    if (!T_out) return fail(GDN_ERR_INVALID_ARG, "T_out is NULL");
    if (!aligned16(T_out)) return fail(GDN_ERR_ALIGNMENT, "T_out must be 16-byte aligned");
    const char *why = "";
    const cudaError_t e = gdn::launch_fused(p, reinterpret_cast<cudaStream_t>(stream), &why, T_out, b, h, n);
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "tc launch: %s %s", cudaGetErrorString(e), why);
    g_msg[0] = 0;
    return GDN_OK;
}

uint64_t gdn_bwd_workspace_bytes(const gdn_bwd_args *args) {
    gdn::BwdParams p;
    if (resolve_bwd(args, &p) != GDN_OK) return 0;
    g_msg[0] = 0;
    return (uint64_t)gdn::bwd_workspace_bytes(p);
}

gdn_status gdn_chunk_bwd(const gdn_bwd_args *args, void *stream) {
    gdn::BwdParams p;
    gdn_status s = resolve_bwd(args, &p);
    if (s != GDN_OK) return s;
    const size_t need = gdn::bwd_workspace_bytes(p);
    if (!args->workspace || args->workspace_bytes < need)
        return fail(GDN_ERR_INVALID_ARG, "backward needs a workspace of %zu bytes (got %llu)", need,
                    (unsigned long long)args->workspace_bytes);
    gdn::bwd_carve_workspace(p, args->workspace);
    const cudaError_t e = gdn::launch_bwd(p, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(GDN_ERR_CUDA, "backward launch: %s", cudaGetErrorString(e));
    g_msg[0] = 0;
    return GDN_OK;
}

}  // extern "C"
