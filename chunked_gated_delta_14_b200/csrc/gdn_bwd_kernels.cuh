// Kernels of the chunked backward pass of the gated delta rule (fp32, CUDA
// cores).  Device code only; the launchers are in gdn_bwd.cu.
//
// The pages give the chunkwise WY/UT form as what makes training parallel
// ("Quando o 'Bom o Suficiente' e Otimo: Aproximacao de Inversao de Matriz
// Baseada Apenas em Multiplicacao para Gated DeltaNet Quantizado", sections
// "Resumo" and "Declaracao do Problema") but print no backward pass.  This is
// the reverse-mode derivative of that chunk form, derived here.  Per chunk of
// Cn tokens with h the state at its start (d_k x d_v, h = S^T), in-chunk
// cumulative log decay g, Gamma_ri = e^{g_r - g_i} (i <= r):
//
//   forward   L_ri = beta_r Gamma_ri k_r.k_i (i < r),  T = (I + L)^-1
//             U = T diag(beta) V,  W = T diag(beta e^g) K,  Delta = U - W h
//             O = diag(e^g) Q h + M Delta,  M_ri = Gamma_ri q_r.k_i (i <= r)
//             h' = e^{g_C} h + (diag(e^{g_C - g}) K)^T Delta
//   backward  given dO and dh' (the gradient reaching h'):
//             dDelta = M^T dO + diag(e^{g_C - g}) K dh'
//             Y      = T^T dDelta
//             dh     = e^{g_C} dh' + (diag(e^g) Q)^T dO - (diag(beta e^g) K)^T Y
//             dV     = diag(beta) Y
//             dM     = dO Delta^T (i <= r),   dL = -Y Delta^T (i < r)
//             dQ     = diag(e^g) dO h^T + (dM (.) Gamma) K
//             dK     = (dM (.) Gamma)^T Q + diag(e^{g_C - g}) Delta dh'^T
//                      - diag(beta e^g) Y h^T + (dG + dG^T) K,
//                      dG = diag(beta) (dL (.) Gamma)
//             dbeta_r = Y_r.V_r - e^{g_r} k_r.(Y h^T)_r + sum_i dL_ri Gamma_ri k_r.k_i
//             dg_r   = the partial derivatives of L, M, diag(e^g), W and h'
//                      in g_r (see bwd_grad_kernel),
//             dlog(alpha_t) = sum_{r >= t} dg_r (summed without the terms that
//                      cancel), dalpha_t = dlog(alpha_t) / alpha_t.
// (dT = dDelta (Vb - Kb h)^T and dL = -T^T dT T^T collapse to -Y Delta^T
// because T (Vb - Kb h) = Delta.)
//
// Four launches: prep (per chunk-head: g, L, T, M, W, U, the decayed Gram, and the
// state-independent M^T dO and (diag(e^g) Q)^T dO), the forward state chain
// (per 32-column value slice: h at every chunk start, Delta), the reverse chain
// (per slice: dh' at every chunk end, Y, dV, dS0) and the key-side gradients
// (per chunk-head: dQ, dK, dbeta, dalpha).
#pragma once

#include "gdn_bwd_params.cuh"

namespace gdn {
namespace bwd {

constexpr int kThreads = 256;
constexpr int kPrepThreads = 512;   // the prep kernel: one block per SM (shared memory), 16 warps
constexpr int kGradThreads = 512;   // the key-side gradient kernel, likewise
constexpr int kGradGroups = kGradThreads / 32;   // its key-column groups (32 row pairs)
constexpr int kCols = 32;     // value columns per block of the two chains and per tile
constexpr int kMaxC = 64;     // largest chunk

extern __shared__ float4 bwd_smem[];

__device__ __forceinline__ float ld_in(const void *ptr, size_t i, int bf16) {
    if (bf16) return __uint_as_float((unsigned int)reinterpret_cast<const uint16_t *>(ptr)[i] << 16);
    return reinterpret_cast<const float *>(ptr)[i];
}

// Four consecutive inputs from element i (i a multiple of 4; bf16 or fp32).
__device__ __forceinline__ float4 ld4_in(const void *ptr, size_t i, int bf16) {
    float4 v;
    if (bf16) {
        const uint32_t *u = reinterpret_cast<const uint32_t *>(ptr) + i / 2;
        const uint32_t a = u[0], b = u[1];
        v.x = __uint_as_float(a << 16); v.y = __uint_as_float(a & 0xffff0000u);
        v.z = __uint_as_float(b << 16); v.w = __uint_as_float(b & 0xffff0000u);
    } else {
        v = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(ptr) + i);
    }
    return v;
}

__device__ __forceinline__ size_t tok_index(const BwdParams &p, int b, int t, int h) {
    return ((size_t)b * p.T + t) * p.H + h;
}

// C rows of D values of [B, T, H, D] inputs (tokens t0.., head h; zero rows from
// Cn on) into shared memory with row stride Dp, from one source (src1 null) or two
// with the same shape.  Four consecutive values per item, and four items' loads
// in flight before the first store: the loads' latencies overlap.
template <int NT>
__device__ __forceinline__ void load_rows(const BwdParams &p, int b, int h, int t0, int C, int Cn, int D, int Dp,
                                          const void *src0, int bf0, float *dst0, const void *src1, int bf1,
                                          float *dst1, int tid) {
    constexpr int UNR = 4;
    const int n4 = C * D / 4;
    for (int base = tid; base < n4; base += NT * UNR) {
        float4 v0[UNR], v1[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int i4 = base + NT * u;
            v0[u] = v1[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i4 < n4) {
                const int r = (4 * i4) / D, c = (4 * i4) % D;
                if (r < Cn) {
                    const size_t gi = tok_index(p, b, t0 + r, h) * D + c;
                    v0[u] = ld4_in(src0, gi, bf0);
                    if (src1) v1[u] = ld4_in(src1, gi, bf1);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int i4 = base + NT * u;
            if (i4 < n4) {
                const int r = (4 * i4) / D, c = (4 * i4) % D;
                float *d0 = dst0 + r * Dp + c;
                d0[0] = v0[u].x; d0[1] = v0[u].y; d0[2] = v0[u].z; d0[3] = v0[u].w;
                if (src1) {
                    float *d1 = dst1 + r * Dp + c;
                    d1[0] = v1[u].x; d1[1] = v1[u].y; d1[2] = v1[u].z; d1[3] = v1[u].w;
                }
            }
        }
    }
}

// out[r][c] = sum_{i < nterm} A(r, i) scale[i] X[i][c] for r < nrow, c < n, with
// A(r, i) = A[r * ra + i * ia] in shared memory (so A or its transpose) and
// scale null meaning 1; written to global memory row-major.  With q = n / 4 and
// rstep = NT / q row groups, thread t < rstep q takes the four columns t % q + q j
// (j < 4) and the rows t / q + rstep m: each A load serves four columns and each
// X load all of the thread's rows, with a separate accumulator per output
// (threads past the last full group idle).  n a multiple of 4, 16 <= n <= 128,
// and ceil(nrow / rstep) <= MAXR.
template <int MAXR, int NT = kThreads>
__device__ __forceinline__ void block_product(const float *A, int ra, int ia, int nrow, int nterm,
                                              const float *scale, const float *X, int xp, int n,
                                              float *out, int tid) {
    const int q = n / 4;
    const int c = tid % q, rg = tid / q, rstep = NT / q;
    if (rg >= rstep || rg >= nrow) return;
    const int nr = (nrow - rg + rstep - 1) / rstep;   // rows rg + rstep m < nrow
    float acc[MAXR][4];
#pragma unroll
    for (int m = 0; m < MAXR; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;
    for (int i = 0; i < nterm; ++i) {
        const float sc = scale ? scale[i] : 1.f;
        const float *xr = X + i * xp + c;
        const float x0 = sc * xr[0], x1 = sc * xr[q], x2 = sc * xr[2 * q], x3 = sc * xr[3 * q];
#pragma unroll
        for (int m = 0; m < MAXR; ++m) {
            if (m < nr) {
                const float a = A[(rg + rstep * m) * ra + i * ia];
                acc[m][0] += a * x0;
                acc[m][1] += a * x1;
                acc[m][2] += a * x2;
                acc[m][3] += a * x3;
            }
        }
    }
#pragma unroll
    for (int m = 0; m < MAXR; ++m) {
        if (m < nr) {
            float *o = out + (size_t)(rg + rstep * m) * n + c;
            o[0] = acc[m][0];
            o[q] = acc[m][1];
            o[2 * q] = acc[m][2];
            o[3 * q] = acc[m][3];
        }
    }
}

// out(r, c) = sum_{k < K} A(r, k) B(k, c) for r, c < C (or out += that with
// `accumulate`), A(r, k) = A[r ra + k ia], B(k, c) = B[k rb + c ib],
// out(r, c) = out[r os + c].  4 x 4 register tiles, two lanes per tile on the even
// and odd k, summed with a shuffle.  out must not be A or B.  Ends with a barrier.
template <int NT>
__device__ __forceinline__ void tile_product(const float *A, int ra, int ia, const float *B, int rb, int ib, int K,
                                             float *out, int os, int C, int tid, bool accumulate = false) {
    const int nt = C / 4, items = 2 * nt * nt;
    for (int w = tid; w < items; w += NT) {
        const int part = w & 1, t = w >> 1;
        const int r0 = 4 * (t / nt), c0 = 4 * (t % nt);
        float acc[4][4] = {};
        for (int k = part; k < K; k += 2) {
            float a[4], bb[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                a[e] = A[(r0 + e) * ra + k * ia];
                bb[e] = B[k * rb + (c0 + e) * ib];
            }
#pragma unroll
            for (int e = 0; e < 4; ++e)
#pragma unroll
                for (int f = 0; f < 4; ++f) acc[e][f] += a[e] * bb[f];
        }
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
            for (int f = 0; f < 4; ++f) acc[e][f] += __shfl_xor_sync(0xffffffffu, acc[e][f], 1);
        if (part == 0) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
#pragma unroll
                for (int f = 0; f < 4; ++f) {
                    float *o = out + (r0 + e) * os + c0 + f;
                    *o = accumulate ? *o + acc[e][f] : acc[e][f];
                }
        }
    }
    __syncthreads();
}

// T = (I + L)^-1 for strictly lower L (C x C in shared memory, row stride Cp),
// blocked: the 16 x 16 diagonal blocks by forward substitution (one column per
// thread; each solved entry updates the rows below it), then the merges
// 16 -> 32 -> 64 of neighbouring blocks, T21 = -T22 L21 T11, with every thread.
// T must be zero on entry (the blocks above the diagonal stay zero); Ys holds
// C * C / 4 floats of scratch.  Ends with a barrier.
template <int NT>
__device__ __forceinline__ void block_inverse(const float *Ls, float *Ts, float *Ys, int C, int Cp, int tid) {
    if (tid < C) {
        const int c = tid, base = c & ~15, jc = c & 15;
        float acc[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) acc[r] = (r == jc) ? 1.f : 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float xi = acc[i];
#pragma unroll
            for (int r = i + 1; r < 16; ++r) acc[r] -= Ls[(base + r) * Cp + base + i] * xi;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Ts[(base + r) * Cp + c] = acc[r];
    }
    __syncthreads();
    for (int sz = 16; sz < C; sz *= 2) {
        const int work = (C / (2 * sz)) * sz * sz;      // outputs of one product, all pairs
        for (int o = tid; o < work; o += NT) {
            const int pr = o / (sz * sz), rr = (o / sz) % sz, cc = o % sz;
            const int b0 = 2 * sz * pr, b1 = b0 + sz;
            float y = 0.f;
            for (int k = 0; k < sz; ++k) y += Ls[(b1 + rr) * Cp + b0 + k] * Ts[(b0 + k) * Cp + b0 + cc];
            Ys[o] = y;
        }
        __syncthreads();
        for (int o = tid; o < work; o += NT) {
            const int pr = o / (sz * sz), rr = (o / sz) % sz, cc = o % sz;
            const int b0 = 2 * sz * pr, b1 = b0 + sz;
            float z = 0.f;
            for (int k = 0; k < sz; ++k) z += Ts[(b1 + rr) * Cp + b1 + k] * Ys[pr * sz * sz + k * sz + cc];
            Ts[(b1 + rr) * Cp + b0 + cc] = -z;
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------- prep
// One block per chunk-head.  Shared memory (floats): K, Q (C x (dk+1)),
// V and then dO (C x (dv+1)), L, T, M (C x (C+1)), g, beta, beta e^g, e^g (C each).
__host__ __device__ inline size_t prep_smem_floats(int C, int dk, int dv, int residual = 0) {
    return 2 * (size_t)C * (dk + 1) + (size_t)C * (dv + 1) + 3 * (size_t)C * (C + 1) + 4 * (size_t)C +
           (size_t)C * C / 4 +                        // the inverse's merge scratch
           (residual ? 3 * (size_t)C * (C + 1) : 0);  // the residual correction's products
}

__global__ void __launch_bounds__(kPrepThreads) bwd_prep_kernel(const BwdParams p) {
    float *sm = reinterpret_cast<float *>(bwd_smem);
    const int C = p.C, dk = p.dk, dv = p.dv;
    const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const int t0 = n * C;
    const int Cn = min(C, p.T - t0);
    const int dkp = dk + 1, dvp = dv + 1, Cp = C + 1;
    float *Ks = sm;
    float *Qs = Ks + C * dkp;
    float *Vs = Qs + C * dkp;
    float *Ls = Vs + C * dvp;
    float *Ts = Ls + C * Cp;
    float *Ms = Ts + C * Cp;
    float *g = Ms + C * Cp;
    float *bb = g + C;
    float *bg = bb + C;
    float *eg = bg + C;
    float *Ys = eg + C;        // C/2 x C/2: the inverse's merge scratch
    float *Rs = Ys + C * C / 4;   // residual correction: 3 x C x (C+1)
    const size_t ch = ((size_t)b * p.H + h) * p.NC + n;

    load_rows<kPrepThreads>(p, b, h, t0, C, Cn, dk, dkp, p.k, p.io_bf16, Ks, p.q, p.io_bf16, Qs, tid);
    load_rows<kPrepThreads>(p, b, h, t0, C, Cn, dv, dvp, p.v, p.io_bf16, Vs, nullptr, 0, nullptr, tid);
    for (int x = tid; x < C * C; x += kPrepThreads) Ts[(x / C) * Cp + x % C] = 0.f;
    // gates: every token's log alpha and beta in parallel, then the in-chunk scan
    if (tid < C) {
        float la = 0.f, be = 0.f;
        if (tid < Cn) {
            const size_t ti = tok_index(p, b, t0 + tid, h);
            la = p.alpha ? logf(p.alpha[ti]) : 0.f;
            be = p.beta ? p.beta[ti] : 1.f;
        }
        g[tid] = la;             // rows past the tail add 0, so g repeats g_{Cn-1}; their beta is 0
        bb[tid] = be;
    }
    __syncthreads();
    if (tid == 0) {
        float acc = 0.f;
        for (int r = 0; r < C; ++r) {
            acc += g[r];
            g[r] = acc;
        }
    }
    __syncthreads();
    if (tid < C) {
        eg[tid] = expf(g[tid]);
        bg[tid] = bb[tid] * eg[tid];
    }
    __syncthreads();

    // L (strictly lower) and M (lower with diagonal) in 4 x 4 register tiles of
    // (rows r0.., keys i0..): per channel the tile's four key rows, query rows and
    // column keys (12 loads per 32 products).  Two neighbouring lanes take the even
    // and odd channels of one tile and add their sums with a shuffle.  Tiles above
    // the diagonal only write zeros; the rows past the tail are the zero rows.
    {
        const int nt = C / 4, tiles = nt * nt;
        for (int w = tid; w < 2 * tiles; w += kPrepThreads) {
            const int part = w & 1, t = w >> 1;
            const int r0 = 4 * (t / nt), i0 = 4 * (t % nt);
            float gk[4][4] = {}, qk[4][4] = {};
            if (i0 <= r0 + 3) {
                for (int c = part; c < dk; c += 2) {
                    float kr[4], qr[4], ki[4];
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        kr[a] = Ks[(r0 + a) * dkp + c];
                        qr[a] = Qs[(r0 + a) * dkp + c];
                        ki[a] = Ks[(i0 + a) * dkp + c];
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            gk[a][e] += kr[a] * ki[e];
                            qk[a][e] += qr[a] * ki[e];
                        }
                }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    gk[a][e] += __shfl_xor_sync(0xffffffffu, gk[a][e], 1);
                    qk[a][e] += __shfl_xor_sync(0xffffffffu, qk[a][e], 1);
                }
            if (part == 0) {
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int r = r0 + a, i = i0 + e;
                        float gg = 0.f, m = 0.f;
                        if (r < Cn && i <= r) {
                            const float gam = expf(g[r] - g[i]);
                            m = gam * qk[a][e];
                            if (i < r) gg = gam * gk[a][e];
                        }
                        Ls[r * Cp + i] = bb[r] * gg;
                        Ms[r * Cp + i] = m;
                        p.ws_S[ch * C * C + r * C + i] = gg;
                        p.ws_M[ch * C * C + r * C + i] = m;
                    }
            }
        }
    }
    __syncthreads();

    block_inverse<kPrepThreads>(Ls, Ts, Ys, C, Cp, tid);
    // Rows past the tail have zero L rows; their diagonal is cleared, so that T is
    // zero outside the sequence as the chains expect.
    if (tid < C && tid >= Cn) Ts[tid * Cp + tid] = 0.f;
    __syncthreads();
    if (p.neumann) {
        // The masked truncated series M^(N) (.) sum_{n<=N} A^n: A is strictly lower,
        // so A^n vanishes within n - 1 of the diagonal and the series agrees with the
        // exact inverse on the band i - j <= N; outside it the mask gives zero.  The
        // exact inverse goes to the adjoint kernel, which needs it for the gradient.
        for (int x = tid; x < C * C; x += kPrepThreads) {
            const int r = x / C, c = x % C;
            p.ws_dA[ch * C * C + x] = Ts[r * Cp + c];
        }
        __syncthreads();
        if (!p.residual) {
            for (int x = tid; x < C * C; x += kPrepThreads) {
                const int r = x / C, c = x % C;
                if (r - c > p.N) Ts[r * Cp + c] = 0.f;
            }
            __syncthreads();
        } else {
            // The residual-corrected series T0 sum_{s<=S} E^s, E = I - (I - A) T0,
            // T0 the masked series ("Metodologia", item 3), is T - T_out E^S with
            // T_out = T - T0 (T's entries below the band) and E = T^-1 T_out =
            // (I + L) T_out: W_0 = T_out, W_{s+1} = (W_s + W_s L) T_out, T_res = T - W_S.
            float *Os = Rs, *Wt = Rs + C * Cp, *Xt = Rs + 2 * C * Cp;
            for (int x = tid; x < C * C; x += kPrepThreads) {
                const int r = x / C, c = x % C;
                const float t = r - c > p.N ? Ts[r * Cp + c] : 0.f;
                Os[r * Cp + c] = t;
                Wt[r * Cp + c] = t;
            }
            __syncthreads();
            for (int it = 0; it < p.S; ++it) {
                tile_product<kPrepThreads>(Wt, Cp, 1, Ls, Cp, 1, C, Xt, Cp, C, tid);     // W L
                for (int x = tid; x < C * C; x += kPrepThreads) Xt[(x / C) * Cp + x % C] += Wt[(x / C) * Cp + x % C];
                __syncthreads();
                tile_product<kPrepThreads>(Xt, Cp, 1, Os, Cp, 1, C, Wt, Cp, C, tid);     // (W + W L) T_out
            }
            for (int x = tid; x < C * C; x += kPrepThreads) Ts[(x / C) * Cp + x % C] -= Wt[(x / C) * Cp + x % C];
            __syncthreads();
        }
    }

    for (int x = tid; x < C * C; x += kPrepThreads) p.ws_T[ch * C * C + x] = Ts[(x / C) * Cp + x % C];
    if (tid < C) p.ws_g[ch * C + tid] = g[tid];
    // W = T diag(beta e^g) K and U = T diag(beta) V (zero rows past the tail)
    block_product<kMaxC / 16, kPrepThreads>(Ts, Cp, 1, C, Cn, bg, Ks, dkp, dk, p.ws_W + ch * C * dk,
                                                           tid);
    block_product<kMaxC / 16, kPrepThreads>(Ts, Cp, 1, C, Cn, bb, Vs, dvp, dv, p.ws_D + ch * C * dv,
                                                           tid);
    __syncthreads();   // V consumed: its buffer takes dO
    float *dOs = Vs;
    load_rows<kPrepThreads>(p, b, h, t0, C, Cn, dv, dvp, p.grad_o, p.do_bf16, dOs, nullptr, 0, nullptr, tid);
    __syncthreads();
    // the state-independent parts of the reverse chain: M^T dO (C x dv) and
    // (diag(e^g) Q)^T dO (dk x dv)
    block_product<kMaxC / 16, kPrepThreads>(Ms, 1, Cp, C, Cn, nullptr, dOs, dvp, dv,
                                                           p.ws_Y + ch * C * dv, tid);
    block_product<128 / 16, kPrepThreads>(Qs, 1, dkp, dk, Cn, eg, dOs, dvp, dv,
                                                         p.ws_P + ch * dk * dv, tid);
}

// ------------------------------------------------- masked-series adjoint
// With the masked truncated series T_N = M^(N) (.) sum_{n<=N} A^n as the chunk
// inverse ("Quando o 'Bom o Suficiente' e Otimo ...", section "Metodologia",
// items 1 and 2), the gradient reaching L differs from the exact inverse's
// -Y Delta^T.  Per chunk-head, from the reverse chain's Y = T_N^T dDelta and the
// forward chain's Delta = T_N R (R = diag(beta) V - diag(beta e^g) K h):
//   dT_N = dDelta R^T = T_N^-T (Y Delta^T) T_N^-T;
// T_N equals M (.) (I - A)^-1 for every strictly lower A (the series and the
// exact inverse agree on the band, the mask zeroes the rest), so
//   dA = T^T (M (.) dT_N) T^T,  T = (I - A)^-1 exact,  dL = -dA,
// written to ws_dA (over the exact inverse the prep left there) for the
// key-side gradient kernel.  With the residual correction (item 3) the forward's
// inverse is T_res = T - T_out E^S (T_out the part of T below the band,
// E = T^-1 T_out) and the gradient reaching T follows from that form (below).
// All products C x C (the first over d_v), fp32.
__host__ __device__ inline size_t neumann_smem_floats(int C, int dv, int residual = 0) {
    (void)dv;
    return 2 * (size_t)C * 33 + (residual ? 9 : 5) * (size_t)C * (C + 1) + (size_t)C * C / 4;
}

__global__ void __launch_bounds__(kPrepThreads) bwd_neumann_kernel(const BwdParams p) {
    constexpr int NT = kPrepThreads;
    float *sm = reinterpret_cast<float *>(bwd_smem);
    const int C = p.C, dv = p.dv, Cp = C + 1;
    const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const size_t ch = ((size_t)b * p.H + h) * p.NC + n;
    float *Yt = sm;                 // a 32-column tile of Y, C x 32
    float *Dt = Yt + C * 33;        // the same tile of Delta
    float *Ss = Dt + C * 33;        // Y Delta^T, then dT, then the gradient reaching T
    float *Bs = Ss + C * Cp;        // strictly lower parts to invert; later T_out, powers of E
    float *Ti = Bs + C * Cp;        // T_N^-1 (or T_res^-1), then T^-1
    float *Tx = Ti + C * Cp;        // the exact inverse
    float *Tm = Tx + C * Cp;        // products in between; E
    float *Ys = Tm + C * Cp;        // scratch of the inverse, C * C / 4
    float *R1 = Ys + C * C / 4;     // residual correction only: K, Q2
    float *R2 = R1 + C * Cp, *R3 = R2 + C * Cp, *R4 = R3 + C * Cp;

    for (int x = tid; x < C * C; x += NT) {
        const int r = x / C, c = x % C;
        const float tn = p.ws_T[ch * C * C + x];
        Bs[r * Cp + c] = c < r ? tn : 0.f;      // rows past the tail are zero: the inverse is 1 there
        Ti[r * Cp + c] = 0.f;
        Tx[r * Cp + c] = p.ws_dA[ch * C * C + x];
    }
    // S = Y Delta^T over d_v, 32 columns at a time
    for (int j0 = 0; j0 < dv; j0 += 32) {
        __syncthreads();
        for (int x = tid; x < C * 32; x += NT) {
            const int r = x / 32, c = x % 32;
            Yt[r * 33 + c] = p.ws_Y[(ch * C + r) * dv + j0 + c];
            Dt[r * 33 + c] = p.ws_D[(ch * C + r) * dv + j0 + c];
        }
        __syncthreads();
        tile_product<NT>(Yt, 33, 1, Dt, 1, 33, 32, Ss, Cp, C, tid, j0 > 0);
    }
    // dT = T_^-T S T_^-T for the truncated inverse T_ the forward used
    block_inverse<NT>(Bs, Ti, Ys, C, Cp, tid);
    tile_product<NT>(Ss, Cp, 1, Ti, 1, Cp, C, Tm, Cp, C, tid);     // S T_^-T
    tile_product<NT>(Ti, 1, Cp, Tm, Cp, 1, C, Ss, Cp, C, tid);     // T_^-T (S T_^-T) = G
    if (!p.residual) {
        // T_N = M (.) T: the gradient reaching T is M (.) G (entries above the
        // diagonal add nothing to the strictly lower dA)
        for (int x = tid; x < C * C; x += NT) {
            const int r = x / C, c = x % C;
            if (r - c > p.N) Ss[r * Cp + c] = 0.f;
        }
        __syncthreads();
    } else {
        // T_res = T - T_out E^S, T_out = (1 - M) (.) T, E = T^-1 T_out.  With
        // K = T_out^T G and H = sum_{j<S} (E^T)^j K (E^T)^{S-1-j}, the gradient
        // reaching T is G - (1 - M) (.) (G (E^S)^T + T^-T H) + T^-T H E^T.
        for (int x = tid; x < C * C; x += NT) {
            const int r = x / C, c = x % C;
            Bs[r * Cp + c] = c < r ? Tx[r * Cp + c] : 0.f;
            Ti[r * Cp + c] = 0.f;
        }
        __syncthreads();
        block_inverse<NT>(Bs, Ti, Ys, C, Cp, tid);                   // T^-1
        for (int x = tid; x < C * C; x += NT) {
            const int r = x / C, c = x % C;
            Bs[r * Cp + c] = r - c > p.N ? Tx[r * Cp + c] : 0.f;     // T_out
        }
        __syncthreads();
        tile_product<NT>(Ti, Cp, 1, Bs, Cp, 1, C, Tm, Cp, C, tid);     // E = T^-1 T_out
        tile_product<NT>(Bs, 1, Cp, Ss, Cp, 1, C, R1, Cp, C, tid);     // K = T_out^T G
        for (int x = tid; x < C * Cp; x += NT) {
            Bs[x] = Tm[x];                                              // P = E^1
            R2[x] = R1[x];                                              // X_0 = K
        }
        __syncthreads();
        float *P = Bs, *Pn = R4, *X = R2, *Xn = R3;
        for (int m = 1; m < p.S; ++m) {
            tile_product<NT>(Tm, 1, Cp, X, Cp, 1, C, Xn, Cp, C, tid);          // E^T X_{m-1}
            tile_product<NT>(R1, Cp, 1, P, 1, Cp, C, Xn, Cp, C, tid, true);    // + K (E^m)^T
            tile_product<NT>(P, Cp, 1, Tm, Cp, 1, C, Pn, Cp, C, tid);          // E^{m+1}
            float *t = X; X = Xn; Xn = t;
            t = P; P = Pn; Pn = t;
        }
        // X = H, P = E^S; Pn and Xn are free
        tile_product<NT>(Ss, Cp, 1, P, 1, Cp, C, Pn, Cp, C, tid);     // Q1 = G (E^S)^T
        tile_product<NT>(Ti, 1, Cp, X, Cp, 1, C, R1, Cp, C, tid);      // Q2 = T^-T H
        tile_product<NT>(R1, Cp, 1, Tm, 1, Cp, C, Xn, Cp, C, tid);     // Q3 = Q2 E^T
        for (int x = tid; x < C * C; x += NT) {
            const int r = x / C, c = x % C, i = r * Cp + c;
            const float out = r - c > p.N ? Pn[i] + R1[i] : 0.f;
            Ss[i] = Ss[i] - out + Xn[i];
        }
        __syncthreads();
    }
    // dA = T^T (gradient reaching T) T^T with the exact inverse, to the workspace
    tile_product<NT>(Ss, Cp, 1, Tx, 1, Cp, C, Tm, Cp, C, tid);
    tile_product<NT>(Tx, 1, Cp, Tm, Cp, 1, C, p.ws_dA + ch * C * C, C, C, tid);
}

// ------------------------------------------------------ forward state chain
// One block per (batch, head, 32 value columns); walks the chunks in order.
// Shared memory: h (dk x 33), W, K (C x (dk+1) each), Delta (C x 33), e^{g_C - g} (C).
__host__ __device__ inline size_t state_fwd_smem_floats(int C, int dk) {
    return (size_t)dk * 33 + 2 * (size_t)C * (dk + 1) + (size_t)C * 33 + (size_t)C;
}

__global__ void __launch_bounds__(kThreads) bwd_state_fwd_kernel(const BwdParams p) {
    float *sm = reinterpret_cast<float *>(bwd_smem);
    const int C = p.C, dk = p.dk, dv = p.dv;
    const int j0 = blockIdx.x * kCols, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const int jj = tid & 31, rr = tid >> 5;     // loads and stores: column jj, rows rr + 8m
    const int jp = tid & 15, rg = tid >> 4;     // products: columns jp, jp + 16, rows rg + 16m
    const int dkp = dk + 1;
    float *hs = sm;
    float *Ws = hs + dk * 33;
    float *Ks = Ws + C * dkp;
    float *Ds = Ks + C * dkp;
    float *es = Ds + C * 33;
    const size_t bh = (size_t)b * p.H + h;

    for (int c = rr; c < dk; c += 8) hs[c * 33 + jj] = p.S0 ? p.S0[(bh * dk + c) * dv + j0 + jj] : 0.f;
    for (int n = 0; n < p.NC; ++n) {
        const int t0 = n * C, Cn = min(C, p.T - t0);
        const size_t ch = bh * p.NC + n;
        __syncthreads();   // h complete; the previous chunk's reads of W, K, Delta done
        for (int c = rr; c < dk; c += 8) p.ws_h[(ch * dk + c) * dv + j0 + jj] = hs[c * 33 + jj];
        const float glast = p.ws_g[ch * C + Cn - 1];
        // W and the raw keys, four elements a load; the decay e^{g_C - g} goes on the
        // rows of Delta in the state update instead of on every key element
        for (int x = tid; x < C * dk / 4; x += kThreads) {
            const int r = 4 * x / dk, c = 4 * x % dk;
            const float4 w = *reinterpret_cast<const float4 *>(p.ws_W + ch * C * dk + 4 * x);
            float4 kv = {0.f, 0.f, 0.f, 0.f};
            if (r < Cn) kv = ld4_in(p.k, tok_index(p, b, t0 + r, h) * dk + c, p.io_bf16);
            float *wr = Ws + r * dkp + c, *kr = Ks + r * dkp + c;
            wr[0] = w.x; wr[1] = w.y; wr[2] = w.z; wr[3] = w.w;
            kr[0] = kv.x; kr[1] = kv.y; kr[2] = kv.z; kr[3] = kv.w;
        }
        if (tid < C) es[tid] = tid < Cn ? expf(glast - p.ws_g[ch * C + tid]) : 0.f;
        for (int r = rr; r < C; r += 8) Ds[r * 33 + jj] = p.ws_D[(ch * C + r) * dv + j0 + jj];
        __syncthreads();
        // Delta = U - W h: this thread's columns jp, jp + 16 and rows rg + 16m
        {
            float a0[kMaxC / 16], a1[kMaxC / 16];
#pragma unroll
            for (int m = 0; m < kMaxC / 16; ++m) {
                const int r = rg + 16 * m;
                a0[m] = r < Cn ? Ds[r * 33 + jp] : 0.f;
                a1[m] = r < Cn ? Ds[r * 33 + jp + 16] : 0.f;
            }
            for (int c = 0; c < dk; ++c) {
                const float h0 = hs[c * 33 + jp], h1 = hs[c * 33 + jp + 16];
#pragma unroll
                for (int m = 0; m < kMaxC / 16; ++m) {
                    if (rg + 16 * m < Cn) {
                        const float wv = Ws[(rg + 16 * m) * dkp + c];
                        a0[m] -= wv * h0;
                        a1[m] -= wv * h1;
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < kMaxC / 16; ++m) {
                const int r = rg + 16 * m;
                if (r < Cn) {
                    Ds[r * 33 + jp] = a0[m];
                    Ds[r * 33 + jp + 16] = a1[m];
                    p.ws_D[(ch * C + r) * dv + j0 + jp] = a0[m];
                    p.ws_D[(ch * C + r) * dv + j0 + jp + 16] = a1[m];
                }
            }
        }
        __syncthreads();
        // h <- e^{g_C} h + (diag(e^{g_C - g}) K)^T Delta: columns jp, jp + 16, key rows rg + 16m
        {
            const float eglast = expf(glast);
            float a0[128 / 16], a1[128 / 16];
#pragma unroll
            for (int m = 0; m < 128 / 16; ++m) {
                const int c = rg + 16 * m;
                a0[m] = c < dk ? eglast * hs[c * 33 + jp] : 0.f;
                a1[m] = c < dk ? eglast * hs[c * 33 + jp + 16] : 0.f;
            }
            for (int r = 0; r < Cn; ++r) {
                const float d0 = es[r] * Ds[r * 33 + jp], d1 = es[r] * Ds[r * 33 + jp + 16];
#pragma unroll
                for (int m = 0; m < 128 / 16; ++m) {
                    if (rg + 16 * m < dk) {
                        const float kv = Ks[r * dkp + rg + 16 * m];
                        a0[m] += kv * d0;
                        a1[m] += kv * d1;
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < 128 / 16; ++m) {
                const int c = rg + 16 * m;
                if (c < dk) {
                    hs[c * 33 + jp] = a0[m];
                    hs[c * 33 + jp + 16] = a1[m];
                }
            }
        }
    }
}

// ------------------------------------------------------ reverse state chain
// One block per (batch, head, 32 value columns); walks the chunks backwards.
// The state-independent terms M^T dO and (diag(e^g) Q)^T dO come from the prep
// kernel, so the serial step per chunk is K dh', T^T dDelta and K^T Y.
// Shared memory: dh (dk x 33), T (C x (C+1)), K (C x (dk+1)), X (C x 33),
// g, beta, e^g (C each).
__host__ __device__ inline size_t state_rev_smem_floats(int C, int dk) {
    return (size_t)dk * 33 + (size_t)C * (C + 1) + (size_t)C * (dk + 1) + (size_t)C * 33 + 3 * (size_t)C;
}

__global__ void __launch_bounds__(kThreads) bwd_state_rev_kernel(const BwdParams p) {
    float *sm = reinterpret_cast<float *>(bwd_smem);
    const int C = p.C, dk = p.dk, dv = p.dv;
    const int j0 = blockIdx.x * kCols, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const int jj = tid & 31, rr = tid >> 5;     // loads and stores: column jj, rows rr + 8m
    const int jp = tid & 15, rg = tid >> 4;     // products: columns jp, jp + 16, rows rg + 16m
    const int dkp = dk + 1, Cp = C + 1;
    float *dhs = sm;
    float *Ts = dhs + dk * 33;
    float *Ks = Ts + C * Cp;
    float *Xs = Ks + C * dkp;
    float *gs = Xs + C * 33;
    float *bs = gs + C;
    float *egs = bs + C;
    const size_t bh = (size_t)b * p.H + h;

    for (int c = rr; c < dk; c += 8)
        dhs[c * 33 + jj] = p.grad_S_T ? p.grad_S_T[(bh * dk + c) * dv + j0 + jj] : 0.f;
    for (int n = p.NC - 1; n >= 0; --n) {
        const int t0 = n * C, Cn = min(C, p.T - t0);
        const size_t ch = bh * p.NC + n;
        __syncthreads();   // dh complete; the previous chunk's reads done
        for (int c = rr; c < dk; c += 8) p.ws_dh[(ch * dk + c) * dv + j0 + jj] = dhs[c * 33 + jj];
        for (int x = tid; x < C * C / 4; x += kThreads) {
            const int r = 4 * x / C, c = 4 * x % C;
            const float4 t = *reinterpret_cast<const float4 *>(p.ws_T + ch * C * C + 4 * x);
            float *tr = Ts + r * Cp + c;
            tr[0] = t.x; tr[1] = t.y; tr[2] = t.z; tr[3] = t.w;
        }
        for (int x = tid; x < C * dk / 4; x += kThreads) {
            const int r = 4 * x / dk, c = 4 * x % dk;
            float4 kv = {0.f, 0.f, 0.f, 0.f};
            if (r < Cn) kv = ld4_in(p.k, tok_index(p, b, t0 + r, h) * dk + c, p.io_bf16);
            float *kr = Ks + r * dkp + c;
            kr[0] = kv.x; kr[1] = kv.y; kr[2] = kv.z; kr[3] = kv.w;
        }
        if (tid < C) {
            const float gv = p.ws_g[ch * C + tid];
            gs[tid] = gv;
            bs[tid] = tid < Cn ? (p.beta ? p.beta[tok_index(p, b, t0 + tid, h)] : 1.f) : 0.f;
            egs[tid] = expf(gv);
        }
        __syncthreads();
        const float glast = gs[Cn - 1];
        // dDelta = M^T dO + diag(e^{g_C - g}) K dh': columns jp, jp + 16, rows rg + 16m
        {
            float u0[kMaxC / 16], u1[kMaxC / 16];
#pragma unroll
            for (int m = 0; m < kMaxC / 16; ++m) u0[m] = u1[m] = 0.f;
            for (int c = 0; c < dk; ++c) {
                const float h0 = dhs[c * 33 + jp], h1 = dhs[c * 33 + jp + 16];
#pragma unroll
                for (int m = 0; m < kMaxC / 16; ++m) {
                    if (rg + 16 * m < Cn) {
                        const float kv = Ks[(rg + 16 * m) * dkp + c];
                        u0[m] += kv * h0;
                        u1[m] += kv * h1;
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < kMaxC / 16; ++m) {
                const int r = rg + 16 * m;
                if (r < Cn) {
                    const float e = expf(glast - gs[r]);
                    const size_t w = (ch * C + r) * dv + j0 + jp;
                    Xs[r * 33 + jp] = p.ws_Y[w] + e * u0[m];
                    Xs[r * 33 + jp + 16] = p.ws_Y[w + 16] + e * u1[m];
                }
            }
        }
        __syncthreads();
        // Y = T^T dDelta (T is lower triangular, zero above the diagonal)
        float y0[kMaxC / 16], y1[kMaxC / 16];
#pragma unroll
        for (int m = 0; m < kMaxC / 16; ++m) y0[m] = y1[m] = 0.f;
        for (int r2 = 0; r2 < Cn; ++r2) {
            const float x0 = Xs[r2 * 33 + jp], x1 = Xs[r2 * 33 + jp + 16];
#pragma unroll
            for (int m = 0; m < kMaxC / 16; ++m) {
                if (rg + 16 * m < Cn) {
                    const float tv = Ts[r2 * Cp + rg + 16 * m];
                    y0[m] += tv * x0;
                    y1[m] += tv * x1;
                }
            }
        }
        __syncthreads();   // every read of dDelta done
#pragma unroll
        for (int m = 0; m < kMaxC / 16; ++m) {
            const int r = rg + 16 * m;
            if (r < C) {
                Xs[r * 33 + jp] = y0[m];
                Xs[r * 33 + jp + 16] = y1[m];
            }
            if (r < Cn) {
                const size_t w = (ch * C + r) * dv + j0 + jp;     // over M^T dO, read above by this thread
                p.ws_Y[w] = y0[m];
                p.ws_Y[w + 16] = y1[m];
                const size_t o = tok_index(p, b, t0 + r, h) * dv + j0 + jp;
                p.grad_v[o] = bs[r] * y0[m];
                p.grad_v[o + 16] = bs[r] * y1[m];
            }
        }
        __syncthreads();
        // dh <- e^{g_C} dh' + (diag(e^g) Q)^T dO - (diag(beta e^g) K)^T Y:
        // columns jp, jp + 16, key rows rg + 16m
        {
            const float eglast = expf(glast);
            float a0[128 / 16], a1[128 / 16];
#pragma unroll
            for (int m = 0; m < 128 / 16; ++m) {
                const int c = rg + 16 * m;
                const size_t w = (ch * dk + c) * dv + j0 + jp;
                a0[m] = c < dk ? eglast * dhs[c * 33 + jp] + p.ws_P[w] : 0.f;
                a1[m] = c < dk ? eglast * dhs[c * 33 + jp + 16] + p.ws_P[w + 16] : 0.f;
            }
            for (int r = 0; r < Cn; ++r) {
                const float eb = egs[r] * bs[r];
                const float yb0 = eb * Xs[r * 33 + jp], yb1 = eb * Xs[r * 33 + jp + 16];
#pragma unroll
                for (int m = 0; m < 128 / 16; ++m) {
                    if (rg + 16 * m < dk) {
                        const float kv = Ks[r * dkp + rg + 16 * m];
                        a0[m] -= kv * yb0;
                        a1[m] -= kv * yb1;
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < 128 / 16; ++m) {
                const int c = rg + 16 * m;
                if (c < dk) {
                    dhs[c * 33 + jp] = a0[m];
                    dhs[c * 33 + jp + 16] = a1[m];
                }
            }
        }
    }
    __syncthreads();
    if (p.grad_S0)
        for (int c = rr; c < dk; c += 8) p.grad_S0[(bh * dk + c) * dv + j0 + jj] = dhs[c * 33 + jj];
}

// ------------------------------------------------------ key-side gradients
// One block per chunk-head of kGradThreads threads (16 warps: the block holds
// 170 KB of shared memory, so one block per SM; the warps hide each other's
// shared-memory latency).  With NG = kGradThreads / 32 column groups, thread
// (rp, cg) = (tid / NG, tid % NG) owns the two rows r0 = 2 rp, r1 = 2 rp + 1 and
// the key columns cg + NG m of the three
// C x dk products over the value axis (dO h^T, Y h^T, Delta dh'^T),
// accumulated in registers over 32-column value tiles, and the entries
// (r0 or r1, cg + NG m) of dO Delta^T and Y Delta^T in shared memory.  Each
// loaded h, dh' and K element serves both rows.
// Shared memory: K, Q (C x (DK+1)), two C x (C+1) score buffers, the value
// tiles (h, dh': DK x 33; dO, Y, Delta, V: C x 33; reused afterwards for two
// C x (C+1) buffers), g, beta, e^g (C), kGradThreads partials, 4 x NG x kMaxC
// row partials and 10 x kMaxC row values.
__host__ __device__ inline size_t grad_smem_floats(int C, int DK) {
    return 2 * (size_t)C * (DK + 1) + 2 * (size_t)C * (C + 1) + 2 * (size_t)DK * 33 + 4 * (size_t)C * 33 +
           3 * (size_t)C + kGradThreads + 4 * (size_t)kGradGroups * kMaxC + 10 * kMaxC;
}

enum { RV_A2K = 0, RV_QA1, RV_K3, RV_YV, RV_KAP, RV_DB, RV_DG, RV_HDH };

template <int DK>
__global__ void __launch_bounds__(kGradThreads) bwd_grad_kernel(const BwdParams p) {
    constexpr int NT = kGradThreads, NG = kGradGroups;
    constexpr int MK = DK / NG;        // key columns per thread
    constexpr int MC = kMaxC / NG;     // score columns per thread
    constexpr int dkp = DK + 1;
    float *sm = reinterpret_cast<float *>(bwd_smem);
    const int C = p.C, dv = p.dv;
    const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const int cg = tid % NG, r0 = 2 * (tid / NG), r1 = r0 + 1;
    const int t0 = n * C, Cn = min(C, p.T - t0);
    const bool v0 = r0 < Cn, v1 = r1 < Cn;     // r1 < C whenever v0 (C is even)
    const int Cp = C + 1;
    float *Ks = sm;
    float *Qs = Ks + C * dkp;
    float *dMs = Qs + C * dkp;
    float *dLs = dMs + C * Cp;
    float *tile = dLs + C * Cp;
    float *ht = tile;
    float *dht = ht + DK * 33;
    float *dOt = dht + DK * 33;
    float *Yt = dOt + C * 33;
    float *Dt = Yt + C * 33;
    float *Vt = Dt + C * 33;
    float *gs = Vt + C * 33;
    float *bs = gs + C;
    float *egs = bs + C;
    float *red = egs + C;
    float *part = red + NT;              // [4 quantities][NG cg][kMaxC]
    float *rowv = part + 4 * NG * kMaxC; // [10][kMaxC]
    const size_t ch = ((size_t)b * p.H + h) * p.NC + n;

    load_rows<NT>(p, b, h, t0, C, Cn, DK, dkp, p.k, p.io_bf16, Ks, p.q, p.io_bf16, Qs, tid);
    // dLs accumulates -dL: Y Delta^T over the value tiles, or (masked series) the
    // adjoint kernel's dA
    for (int x = tid; x < C * Cp; x += NT) {
        const int r = x / Cp, c = x % Cp;
        dMs[x] = 0.f;
        dLs[x] = (p.neumann && c < C) ? p.ws_dA[ch * C * C + r * C + c] : 0.f;
    }
    if (tid < C) {
        const float gv = p.ws_g[ch * C + tid];
        gs[tid] = gv;
        bs[tid] = tid < Cn ? (p.beta ? p.beta[tok_index(p, b, t0 + tid, h)] : 1.f) : 0.f;
        egs[tid] = expf(gv);
    }

    float A1[2][MK], A2[2][MK], A3[2][MK];
#pragma unroll
    for (int m = 0; m < MK; ++m) A1[0][m] = A2[0][m] = A3[0][m] = A1[1][m] = A2[1][m] = A3[1][m] = 0.f;
    float yv0 = 0.f, yv1 = 0.f, hdh = 0.f;

    for (int j0 = 0; j0 < dv; j0 += kCols) {
        __syncthreads();   // previous tile consumed (and, first time, the set-up above)
        // the tile's inputs four values at a time, every load of a pass issued
        // before its first store
        {
            constexpr int NH = DK * (kCols / 4);                      // float4 items (h, dh)
            constexpr int HQ = (NH + NT - 1) / NT;        // per thread
            float4 hv[HQ], dhv[HQ];
#pragma unroll
            for (int u = 0; u < HQ; ++u) {
                const int x = tid + NT * u, c = x / (kCols / 4), q4 = x % (kCols / 4);
                if (x < NH) {
                    const size_t o = (ch * DK + c) * dv + j0 + 4 * q4;
                    hv[u] = *reinterpret_cast<const float4 *>(p.ws_h + o);
                    dhv[u] = *reinterpret_cast<const float4 *>(p.ws_dh + o);
                }
            }
#pragma unroll
            for (int u = 0; u < HQ; ++u) {
                const int x = tid + NT * u, c = x / (kCols / 4), q4 = x % (kCols / 4);
                if (x < NH) {
                    float *hd = ht + c * 33 + 4 * q4, *dd = dht + c * 33 + 4 * q4;
                    hd[0] = hv[u].x; hd[1] = hv[u].y; hd[2] = hv[u].z; hd[3] = hv[u].w;
                    dd[0] = dhv[u].x; dd[1] = dhv[u].y; dd[2] = dhv[u].z; dd[3] = dhv[u].w;
                }
            }
        }
        for (int base = tid; base < C * (kCols / 4); base += 2 * NT) {
            float4 a4[2], v4[2], y4[2], d4[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int x = base + NT * u, r2 = x / (kCols / 4), q4 = x % (kCols / 4);
                a4[u] = v4[u] = y4[u] = d4[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (x < C * (kCols / 4) && r2 < Cn) {
                    const size_t ti = tok_index(p, b, t0 + r2, h) * dv + j0 + 4 * q4;
                    a4[u] = ld4_in(p.grad_o, ti, p.do_bf16);
                    v4[u] = ld4_in(p.v, ti, p.io_bf16);
                    y4[u] = *reinterpret_cast<const float4 *>(p.ws_Y + (ch * C + r2) * dv + j0 + 4 * q4);
                    d4[u] = *reinterpret_cast<const float4 *>(p.ws_D + (ch * C + r2) * dv + j0 + 4 * q4);
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int x = base + NT * u, r2 = x / (kCols / 4), q4 = x % (kCols / 4);
                if (x < C * (kCols / 4)) {
                    const int o = r2 * 33 + 4 * q4;
                    dOt[o] = a4[u].x; dOt[o + 1] = a4[u].y; dOt[o + 2] = a4[u].z; dOt[o + 3] = a4[u].w;
                    Vt[o] = v4[u].x; Vt[o + 1] = v4[u].y; Vt[o + 2] = v4[u].z; Vt[o + 3] = v4[u].w;
                    Yt[o] = y4[u].x; Yt[o + 1] = y4[u].y; Yt[o + 2] = y4[u].z; Yt[o + 3] = y4[u].w;
                    Dt[o] = d4[u].x; Dt[o + 1] = d4[u].y; Dt[o + 2] = d4[u].z; Dt[o + 3] = d4[u].w;
                }
            }
        }
        __syncthreads();
        if (v0) {   // tile rows at and past Cn are zero, so row r1 needs no test here
            for (int jj = 0; jj < kCols; ++jj) {
                const float a0 = dOt[r0 * 33 + jj], y0 = Yt[r0 * 33 + jj], d0 = Dt[r0 * 33 + jj];
                const float a1 = dOt[r1 * 33 + jj], y1 = Yt[r1 * 33 + jj], d1 = Dt[r1 * 33 + jj];
#pragma unroll
                for (int m = 0; m < MK; ++m) {
                    const int c = cg + NG * m;
                    const float hv = ht[c * 33 + jj], dhv = dht[c * 33 + jj];
                    A1[0][m] += a0 * hv;
                    A2[0][m] += y0 * hv;
                    A3[0][m] += d0 * dhv;
                    A1[1][m] += a1 * hv;
                    A2[1][m] += y1 * hv;
                    A3[1][m] += d1 * dhv;
                }
            }
            for (int jj = cg; jj < kCols; jj += NG) {
                yv0 += Yt[r0 * 33 + jj] * Vt[r0 * 33 + jj];
                yv1 += Yt[r1 * 33 + jj] * Vt[r1 * 33 + jj];
            }
            // this tile's part of dO Delta^T and Y Delta^T at (r0 or r1, cg + NG m)
            float s1[2][MC], s2[2][MC];
#pragma unroll
            for (int m = 0; m < MC; ++m) s1[0][m] = s2[0][m] = s1[1][m] = s2[1][m] = 0.f;
            for (int jj = 0; jj < kCols; ++jj) {
                const float a0 = dOt[r0 * 33 + jj], y0 = Yt[r0 * 33 + jj];
                const float a1 = dOt[r1 * 33 + jj], y1 = Yt[r1 * 33 + jj];
#pragma unroll
                for (int m = 0; m < MC; ++m) {
                    if (cg + NG * m < Cn) {
                        const float d = Dt[(cg + NG * m) * 33 + jj];
                        s1[0][m] += a0 * d;
                        s2[0][m] += y0 * d;
                        s1[1][m] += a1 * d;
                        s2[1][m] += y1 * d;
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < MC; ++m) {
                const int i = cg + NG * m;
                if (i < Cn) {
                    dMs[r0 * Cp + i] += s1[0][m];
                    if (!p.neumann) dLs[r0 * Cp + i] += s2[0][m];
                    if (v1) {
                        dMs[r1 * Cp + i] += s1[1][m];
                        if (!p.neumann) dLs[r1 * Cp + i] += s2[1][m];
                    }
                }
            }
        }
        for (int x = tid; x < DK * kCols; x += NT) {
            const int c = x / kCols, jj = x % kCols;
            hdh += ht[c * 33 + jj] * dht[c * 33 + jj];
        }
    }

    // row dot products k_r.(Y h^T)_r, q_r.(dO h^T)_r, k_r.(Delta dh'^T)_r
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int r = r0 + e;
        float a2k = 0.f, qa1 = 0.f, k3 = 0.f;
        if (r < Cn) {
#pragma unroll
            for (int m = 0; m < MK; ++m) {
                const int c = cg + NG * m;
                a2k += A2[e][m] * Ks[r * dkp + c];
                qa1 += A1[e][m] * Qs[r * dkp + c];
                k3 += A3[e][m] * Ks[r * dkp + c];
            }
        }
        part[(0 * NG + cg) * kMaxC + r] = a2k;
        part[(1 * NG + cg) * kMaxC + r] = qa1;
        part[(2 * NG + cg) * kMaxC + r] = k3;
        part[(3 * NG + cg) * kMaxC + r] = e ? yv1 : yv0;
    }
    red[tid] = hdh;
    __syncthreads();
    if (tid < kMaxC) {
        for (int qn = 0; qn < 4; ++qn) {
            float s = 0.f;
            for (int k = 0; k < NG; ++k) s += part[(qn * NG + k) * kMaxC + tid];
            rowv[qn * kMaxC + tid] = s;   // RV_A2K, RV_QA1, RV_K3, RV_YV
        }
    }
    if (tid == 0) {
        float s = 0.f;
        for (int x = 0; x < NT; ++x) s += red[x];
        rowv[RV_HDH * kMaxC] = s;
    }

    // per score entry, with the decayed Gram and scores of the prep kernel
    float *Fs = tile;             // dL (.) L + dM (.) M: F_ri enters dg_r with +, dg_i with -
    float *Es = tile + C * Cp;    // dL (.) Gamma (.) k_r.k_i, the beta-derivative of L
    for (int x = tid; x < C * C; x += NT) {
        const int r2 = x / C, i = x % C;
        float F = 0.f, E = 0.f, dmg = 0.f, dgv = 0.f;
        if (r2 < Cn && i <= r2) {
            const float gam = expf(gs[r2] - gs[i]);
            const float dm = dMs[r2 * Cp + i];
            F = dm * p.ws_M[ch * C * C + x];
            dmg = dm * gam;
            if (i < r2) {
                const float dl = -dLs[r2 * Cp + i];
                const float gg = p.ws_S[ch * C * C + x];   // Gamma_ri k_r.k_i
                F += dl * bs[r2] * gg;
                E = dl * gg;
                dgv = bs[r2] * dl * gam;
            }
        }
        Fs[(x / C) * Cp + x % C] = F;
        Es[(x / C) * Cp + x % C] = E;
        dMs[r2 * Cp + i] = dmg;   // dM (.) Gamma
        dLs[r2 * Cp + i] = dgv;   // dG
    }
    __syncthreads();

    if (tid < Cn) {
        const int rr = tid;
        float er = 0.f;
        for (int i = 0; i < Cn; ++i) er += Es[rr * Cp + i];
        const float kap = expf(gs[Cn - 1] - gs[rr]) * rowv[RV_K3 * kMaxC + rr];
        const float a2k = rowv[RV_A2K * kMaxC + rr];
        rowv[RV_KAP * kMaxC + rr] = kap;
        rowv[RV_DB * kMaxC + rr] = rowv[RV_YV * kMaxC + rr] - egs[rr] * a2k + er;
        // the derivative in g_r of diag(e^g) Q h and of W (F and kappa enter below)
        rowv[RV_DG * kMaxC + rr] = -bs[rr] * egs[rr] * a2k + egs[rr] * rowv[RV_QA1 * kMaxC + rr];
    }
    __syncthreads();
    if (tid < Cn) {
        const int rr = tid;
        // d log alpha_t = sum_{r >= t} dg_r, where dg_r collects the terms above,
        // +F_ri for every i <= r, -F_ir for every i >= r, -kappa_r, and at the
        // chunk end e^{g_C}<h, dh'> + sum_i kappa_i.  Summed over r >= t, the F terms
        // with both indices >= t and the kappa terms with index >= t cancel exactly;
        // only those crossing t are added, so no large terms cancel in fp32.
        float s = expf(gs[Cn - 1]) * rowv[RV_HDH * kMaxC];
        for (int i = 0; i < rr; ++i) s += rowv[RV_KAP * kMaxC + i];
        for (int r2 = rr; r2 < Cn; ++r2) s += rowv[RV_DG * kMaxC + r2];
        for (int r2 = rr; r2 < Cn; ++r2)
            for (int i = 0; i < rr; ++i) s += Fs[r2 * Cp + i];
        const size_t ti = tok_index(p, b, t0 + rr, h);
        if (p.grad_alpha) p.grad_alpha[ti] = s / p.alpha[ti];
        if (p.grad_beta) p.grad_beta[ti] = rowv[RV_DB * kMaxC + rr];
    }

    if (v0) {
        // dQ = diag(e^g) dO h^T + (dM (.) Gamma) K, accumulated into A1.  dM (.) Gamma
        // is zero above the diagonal, so both rows run over i <= r1.
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const float eg = egs[r0 + e];   // row r1 past the tail: beta 0, its outputs unused
#pragma unroll
            for (int m = 0; m < MK; ++m) A1[e][m] *= eg;
        }
        for (int i = 0; i <= r1 && i < Cn; ++i) {
            const float dm0 = dMs[r0 * Cp + i], dm1 = dMs[r1 * Cp + i];
#pragma unroll
            for (int m = 0; m < MK; ++m) {
                const float kv = Ks[i * dkp + cg + NG * m];
                A1[0][m] += dm0 * kv;
                A1[1][m] += dm1 * kv;
            }
        }
        // dK = (dM (.) Gamma)^T Q + diag(e^{g_C-g}) Delta dh'^T - diag(beta e^g) Y h^T
        //      + (dG + dG^T) K, accumulated into A3
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int r = r0 + e;
            const float ebr = bs[r] * egs[r], edec = expf(gs[Cn - 1] - gs[r]);
#pragma unroll
            for (int m = 0; m < MK; ++m) A3[e][m] = edec * A3[e][m] - ebr * A2[e][m];
        }
        for (int r2 = r0; r2 < Cn; ++r2) {
            const float dm0 = dMs[r2 * Cp + r0], dm1 = dMs[r2 * Cp + r1];   // dm1 = 0 at r2 = r0
#pragma unroll
            for (int m = 0; m < MK; ++m) {
                const float qv = Qs[r2 * dkp + cg + NG * m];
                A3[0][m] += dm0 * qv;
                A3[1][m] += dm1 * qv;
            }
        }
        for (int i = 0; i < Cn; ++i) {
            const float g0 = dLs[r0 * Cp + i] + dLs[i * Cp + r0];
            const float g1 = dLs[r1 * Cp + i] + dLs[i * Cp + r1];
#pragma unroll
            for (int m = 0; m < MK; ++m) {
                const float kv = Ks[i * dkp + cg + NG * m];
                A3[0][m] += g0 * kv;
                A3[1][m] += g1 * kv;
            }
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            if (e == 0 || v1) {
                const size_t out = tok_index(p, b, t0 + r0 + e, h) * DK;
#pragma unroll
                for (int m = 0; m < MK; ++m) {
                    p.grad_q[out + cg + NG * m] = A1[e][m];
                    p.grad_k[out + cg + NG * m] = A3[e][m];
                }
            }
        }
    }
}

}  // namespace bwd
}  // namespace gdn
