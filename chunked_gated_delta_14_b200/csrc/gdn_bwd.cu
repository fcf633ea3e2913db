// Launchers of the chunked backward pass (kernels in gdn_bwd_kernels.cuh).
#include "gdn_bwd.cuh"
#include "gdn_bwd_kernels.cuh"

namespace gdn {
namespace {

size_t region(size_t floats_per_chunk, size_t chunks) {
    return (floats_per_chunk * chunks * sizeof(float) + 255) & ~(size_t)255;
}

template <class K>
cudaError_t launch_one(K kernel, dim3 grid, size_t smem_floats, const BwdParams &p, cudaStream_t stream,
                       int threads = bwd::kThreads) {
    const size_t bytes = smem_floats * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    kernel<<<grid, threads, bytes, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

bool bwd_supports(const BwdParams &p, const char **why) {
    if (p.C != 16 && p.C != 32 && p.C != 64) { *why = "chunk must be 16, 32 or 64"; return false; }
    if (p.dk != 16 && p.dk != 32 && p.dk != 64 && p.dk != 128) { *why = "dk must be 16, 32, 64 or 128"; return false; }
    if (p.dv % bwd::kCols != 0 || p.dv > 128) { *why = "dv must be 32, 64, 96 or 128"; return false; }
    if (p.neumann && (p.N < 0 || p.N > p.C - 1)) { *why = "neumann_N must be in [0, chunk - 1]"; return false; }
    if (p.residual && (p.S < 1 || p.S > 64)) { *why = "residual_S must be in [0, 64]"; return false; }
    return true;
}

size_t bwd_workspace_bytes(const BwdParams &p) {
    const size_t nch = (size_t)p.B * p.H * p.NC;
    const size_t C = p.C, dk = p.dk, dv = p.dv;
    return region(C, nch) + 3 * region(C * C, nch) + region(C * dk, nch) + 2 * region(C * dv, nch) +
           3 * region(dk * dv, nch) + (p.neumann ? region(C * C, nch) : 0);
}

void bwd_carve_workspace(BwdParams &p, void *workspace) {
    const size_t nch = (size_t)p.B * p.H * p.NC;
    const size_t C = p.C, dk = p.dk, dv = p.dv;
    char *w = static_cast<char *>(workspace);
    p.ws_g = reinterpret_cast<float *>(w);  w += region(C, nch);
    p.ws_T = reinterpret_cast<float *>(w);  w += region(C * C, nch);
    p.ws_S = reinterpret_cast<float *>(w);  w += region(C * C, nch);
    p.ws_M = reinterpret_cast<float *>(w);  w += region(C * C, nch);
    p.ws_W = reinterpret_cast<float *>(w);  w += region(C * dk, nch);
    p.ws_D = reinterpret_cast<float *>(w);  w += region(C * dv, nch);
    p.ws_Y = reinterpret_cast<float *>(w);  w += region(C * dv, nch);
    p.ws_P = reinterpret_cast<float *>(w);  w += region(dk * dv, nch);
    p.ws_h = reinterpret_cast<float *>(w);  w += region(dk * dv, nch);
    p.ws_dh = reinterpret_cast<float *>(w);  w += region(dk * dv, nch);
    p.ws_dA = p.neumann ? reinterpret_cast<float *>(w) : nullptr;
}

cudaError_t launch_bwd(const BwdParams &p, cudaStream_t stream) {
    const dim3 per_chunk(p.NC, p.H, p.B);
    const dim3 per_slice(p.dv / bwd::kCols, p.H, p.B);
    cudaError_t e = launch_one(bwd::bwd_prep_kernel, per_chunk, bwd::prep_smem_floats(p.C, p.dk, p.dv, p.residual), p, stream,
                               bwd::kPrepThreads);
    if (e != cudaSuccess) return e;
    e = launch_one(bwd::bwd_state_fwd_kernel, per_slice, bwd::state_fwd_smem_floats(p.C, p.dk), p, stream);
    if (e != cudaSuccess) return e;
    e = launch_one(bwd::bwd_state_rev_kernel, per_slice, bwd::state_rev_smem_floats(p.C, p.dk), p, stream);
    if (e != cudaSuccess) return e;
    if (p.neumann) {
        e = launch_one(bwd::bwd_neumann_kernel, per_chunk, bwd::neumann_smem_floats(p.C, p.dv, p.residual), p, stream,
                       bwd::kPrepThreads);
        if (e != cudaSuccess) return e;
    }
    const size_t gs = bwd::grad_smem_floats(p.C, p.dk);
    switch (p.dk) {
        case 16: return launch_one(bwd::bwd_grad_kernel<16>, per_chunk, gs, p, stream, bwd::kGradThreads);
        case 32: return launch_one(bwd::bwd_grad_kernel<32>, per_chunk, gs, p, stream, bwd::kGradThreads);
        case 64: return launch_one(bwd::bwd_grad_kernel<64>, per_chunk, gs, p, stream, bwd::kGradThreads);
        case 128: return launch_one(bwd::bwd_grad_kernel<128>, per_chunk, gs, p, stream, bwd::kGradThreads);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace gdn
