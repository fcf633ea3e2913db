// Token-by-token kernel for short sequences (decode steps) of the gated delta
// rule  S_t = S_{t-1} alpha_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
// o_t = S_t q_t, written for the stored state h = S^T (d_k x d_v):
//
//   p   = h^T k_t                          (= S_{t-1} k_t)
//   h  <- alpha_t h + k_t (beta_t (v_t - alpha_t p))^T
//   o_t = h^T q_t
//
// One CTA per (batch, head, 32-column value slice) keeps its slice of h in
// registers for the whole call: 8 warps x (d_k / 8) rows, lane = value column.
// Per token two block reductions over d_k (p and o); h is read from S0 once
// and written to S_T once, so a decode step is bound by the state traffic.
#include <cuda_bf16.h>

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kRecThreads = 256;
constexpr int kRecCols = 32;

__device__ __forceinline__ float rec_load(const void *p, size_t i, int bf16) {
    if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
    return reinterpret_cast<const float *>(p)[i];
}

template <int R>   // state rows per warp: d_k / 8
__global__ void __launch_bounds__(kRecThreads) recurrent_kernel(const FwdParams p) {
    __shared__ float ks[128], qs[128];
    __shared__ float red[8][kRecCols + 1];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slice = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int dk = p.dk, dv = p.dv, T = p.T, H = p.H;
    const int j = slice * kRecCols + lane;          // value column of this thread
    const int r0 = warp * R;                        // first state row of this warp
    const size_t bh = (size_t)b * H + h;

    float hr[R];
#pragma unroll
    for (int r = 0; r < R; ++r) hr[r] = p.S0 ? p.S0[(bh * dk + r0 + r) * dv + j] : 0.f;

    for (int t = 0; t < T; ++t) {
        const size_t tok = ((size_t)b * T + t) * H + h;
        for (int i = tid; i < dk; i += kRecThreads) {
            ks[i] = rec_load(p.k, tok * dk + i, p.io_bf16);
            qs[i] = rec_load(p.q, tok * dk + i, p.io_bf16);
        }
        const float a = p.alpha ? p.alpha[tok] : 1.f;
        const float be = p.beta ? p.beta[tok] : 1.f;
        const float vj = rec_load(p.v, tok * dv + j, p.io_bf16);
        __syncthreads();
        // p_j = sum_i h_ij k_i
        float part = 0.f;
#pragma unroll
        for (int r = 0; r < R; ++r) part += hr[r] * ks[r0 + r];
        red[warp][lane] = part;
        __syncthreads();
        float pj = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) pj += red[w][lane];
        const float u = be * (vj - a * pj);
        // h <- alpha h + k u^T, then o_j = sum_i h_ij q_i
        float op = 0.f;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            hr[r] = a * hr[r] + ks[r0 + r] * u;
            op += hr[r] * qs[r0 + r];
        }
        __syncthreads();                            // every p_j read before red is reused
        red[warp][lane] = op;
        __syncthreads();
        if (warp == 0) {
            float o = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) o += red[w][lane];
            if (p.o_bf16) reinterpret_cast<__nv_bfloat16 *>(p.o)[tok * dv + j] = __float2bfloat16_rn(o);
            else reinterpret_cast<float *>(p.o)[tok * dv + j] = o;
        }
    }
    if (p.S_T) {
#pragma unroll
        for (int r = 0; r < R; ++r) p.S_T[(bh * dk + r0 + r) * dv + j] = hr[r];
    }
}

}  // namespace

bool recurrent_supports(const FwdParams &p, const char **why) {
    if (p.general) { *why = "two-gate rule runs on the SIMT kernel"; return false; }
    if (p.mode != GDN_INV_EXACT) { *why = "token recurrence has no truncated inverse"; return false; }
    if (p.dk % 8 != 0 || p.dk > 128) { *why = "needs dk a multiple of 8, at most 128"; return false; }
    if (p.dv % kRecCols != 0) { *why = "needs dv a multiple of 32"; return false; }
    return true;
}

cudaError_t launch_recurrent(const FwdParams &p, cudaStream_t stream) {
    const dim3 grid(p.dv / kRecCols, p.H, p.B);
    switch (p.dk / 8) {
        case 2: recurrent_kernel<2><<<grid, kRecThreads, 0, stream>>>(p); break;
        case 4: recurrent_kernel<4><<<grid, kRecThreads, 0, stream>>>(p); break;
        case 8: recurrent_kernel<8><<<grid, kRecThreads, 0, stream>>>(p); break;
        case 16: recurrent_kernel<16><<<grid, kRecThreads, 0, stream>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace gdn
