// fp32 CUDA-core chunk kernel for every variant of the chunkwise gated
// delta rule.  One block per (batch, head, value slice) walks the chunks of
// its sequence in order and carries the fp32 state h = S^T (dk x dvs) in
// shared memory.  Per chunk of C tokens (local rows r, keys i):
//
//   scalar decay (gated delta rule):
//     g_r = sum_{i<=r} log alpha_i
//     L_ri = beta_r exp(g_r - g_i) (k_r . k_i), i < r;   A = -L
//     T    = (I - A)^-1 = (I + L)^-1       exact, or M^(N) (.) sum_{n<=N} A^n
//     R_r  = beta_r (v_r - e^{g_r} h^T k_r)
//     Delta = T R
//     O_r  = e^{g_r} h^T q_r + sum_{i<=r} exp(g_r - g_i)(q_r . k_i) Delta_i
//     h   <- e^{g_last} h + sum_r e^{g_last - g_r} k_r Delta_r^T
//
//   two-gate rule (per-channel decay G, write key kw, erase key e = b (.) kw,
//   written value u = w (.) v):
//     L_ri = sum_c e_rc kw_ic exp(G_{r-1,c} - G_ic), i < r
//     R_r  = u_r - h^T (e_r (.) e^{G_{r-1}})
//     O_r  = h^T (q_r (.) e^{G_r}) + sum_{i<=r} [sum_c q_rc kw_ic exp(G_rc - G_ic)] Delta_i
//     h   <- diag(e^{G_last}) h + sum_r (kw_r (.) e^{G_last - G_r}) Delta_r^T
//
// The triangular inverse T = (I - A)^-1 with A strictly lower triangular and
// its truncated Neumann form with the structural mask follow "Quando o 'Bom o
// Suficiente' e Otimo: Aproximacao de Inversao de Matriz Baseada Apenas em
// Multiplicacao para Gated DeltaNet Quantizado" (sections "Declaracao do
// Problema" and "Metodologia", items 1-2).  Exact mode uses row-by-row forward
// substitution; Neumann mode evaluates the masked series by Horner's rule,
// T <- M (.) (I + A T), keeping only the band the mask leaves non-zero.
// Decay ratios are always exp(later - earlier) <= 1.

#include <cuda_bf16.h>

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float load_in(const void *p, size_t i, int bf16) {
    if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
    return reinterpret_cast<const float *>(p)[i];
}

template <typename S>
__device__ __forceinline__ float ld_s(const S *a, int i) {
    if constexpr (sizeof(S) == 2) return __bfloat162float(a[i]);
    else return a[i];
}

template <typename S>
__device__ __forceinline__ void st_s(S *a, int i, float x) {
    if constexpr (sizeof(S) == 2) a[i] = __float2bfloat16_rn(x);
    else a[i] = x;
}

// Shared-memory carve-up, identical on host and device.
struct SimtLayout {
    size_t kx, qx, ex, gx, tp, band, hs, ux, dx, rows, rho, total;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

__host__ __device__ inline SimtLayout simt_layout(int C, int dk, int dvs, int N, int neumann,
                                                  int general, int key_bytes) {
    SimtLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t at = off; off = align16(off + bytes); return at; };
    // general: kw, q, e, G all fp32; scalar: k, q stored in the io dtype
    const size_t kb = general ? 4 : (size_t)key_bytes;
    L.kx = take((size_t)C * dk * kb);
    L.qx = take((size_t)C * dk * kb);
    L.ex = general ? take((size_t)C * dk * 4) : off;
    L.gx = general ? take((size_t)C * dk * 4) : off;
    L.tp = take((size_t)C * C * 4);
    L.band = neumann ? take((size_t)2 * C * (N + 1) * 4) : off;
    L.hs = take((size_t)dk * dvs * 4);
    L.ux = take((size_t)C * dvs * 4);
    L.dx = take((size_t)C * dvs * 4);
    L.rows = take((size_t)4 * C * 4);        // g / log alpha, beta, lrow, spare
    L.rho = general ? take((size_t)dk * 4) : off;
    L.total = off;
    return L;
}

// Inclusive prefix sum of x[0..n) in place (n <= 128), by warp 0.
__device__ void warp0_inclusive_scan(float *x, int n) {
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    float carry = 0.f;
    for (int base = 0; base < n; base += 32) {
        float v = (base + lane < n) ? x[base + lane] : 0.f;
        for (int o = 1; o < 32; o <<= 1) {
            float y = __shfl_up_sync(0xffffffffu, v, o);
            if (lane >= o) v += y;
        }
        v += carry;
        if (base + lane < n) x[base + lane] = v;
        carry = __shfl_sync(0xffffffffu, v, 31);
    }
}

template <typename KS, bool GENERAL>
__global__ void __launch_bounds__(kThreads)
simt_chunk_kernel(const FwdParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int slice = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int C = p.C, dk = p.dk, dv = p.dv, dvs = p.dvs, H = p.H, T = p.T;
    const int v0 = slice * dvs;
    const int tid = threadIdx.x;
    const int neumann = (p.mode == GDN_INV_NEUMANN);
    const int N = p.N;
    const SimtLayout Ly = simt_layout(C, dk, dvs, N, neumann, GENERAL ? 1 : 0,
                                      (int)sizeof(KS));
    KS *kx = reinterpret_cast<KS *>(smem + Ly.kx);       // keys (write keys kw)
    KS *qx = reinterpret_cast<KS *>(smem + Ly.qx);       // read keys
    float *ex = reinterpret_cast<float *>(smem + Ly.ex); // erase keys (two-gate)
    float *gx = reinterpret_cast<float *>(smem + Ly.gx); // per-channel cumulative log decay
    float *tp = reinterpret_cast<float *>(smem + Ly.tp); // L -> T -> P, C x C
    float *band = reinterpret_cast<float *>(smem + Ly.band);
    float *hs = reinterpret_cast<float *>(smem + Ly.hs); // state h, dk x dvs
    float *ux = reinterpret_cast<float *>(smem + Ly.ux); // values -> R
    float *dx = reinterpret_cast<float *>(smem + Ly.dx); // Delta
    float *rows = reinterpret_cast<float *>(smem + Ly.rows);
    float *g = rows;                 // scalar: log alpha -> cumulative g
    float *bet = rows + C;           // scalar: beta
    float *lrow = rows + 2 * C;      // forward-substitution row copy
    float *rho = reinterpret_cast<float *>(smem + Ly.rho);

    const size_t bh = (size_t)b * H + h;
    // initial state
    for (int idx = tid; idx < dk * dvs; idx += kThreads) {
        const int c = idx / dvs, j = idx % dvs;
        hs[idx] = p.S0 ? p.S0[(bh * dk + c) * dv + v0 + j] : 0.f;
    }
    if (GENERAL)
        for (int c = tid; c < dk; c += kThreads) rho[c] = 0.f;

    for (int t0 = 0; t0 < T; t0 += C) {
        const int Cv = min(C, T - t0);
        __syncthreads();  // previous chunk fully consumed
        // ---------------------------------------------------------- load
        for (int idx = tid; idx < C * dk; idx += kThreads) {
            const int r = idx / dk, c = idx % dk;
            const size_t gi = (((size_t)b * T + t0 + r) * H + h) * dk + c;
            const bool ok = r < Cv;
            st_s(kx, idx, ok ? load_in(p.k, gi, p.io_bf16) : 0.f);
            st_s(qx, idx, ok ? load_in(p.q, gi, p.io_bf16) : 0.f);
            if (GENERAL) {
                ex[idx] = ok ? (p.erase ? load_in(p.erase, gi, p.io_bf16) : 1.f) : 0.f;
                gx[idx] = (ok && p.alpha) ? logf(p.alpha[p.alpha_pc ? gi : gi / dk]) : 0.f;
            }
        }
        for (int idx = tid; idx < C * dvs; idx += kThreads) {
            const int r = idx / dvs, j = idx % dvs;
            const size_t gi = (((size_t)b * T + t0 + r) * H + h) * dv + v0 + j;
            float u = 0.f;
            if (r < Cv) {
                u = load_in(p.v, gi, p.io_bf16);
                if (GENERAL && p.write) u *= load_in(p.write, gi, p.io_bf16);
            }
            ux[idx] = u;
        }
        if (!GENERAL) {
            for (int r = tid; r < C; r += kThreads) {
                const size_t ti = ((size_t)b * T + t0 + r) * H + h;
                g[r] = (r < Cv && p.alpha) ? logf(p.alpha[ti]) : 0.f;
                bet[r] = (r < Cv) ? (p.beta ? p.beta[ti] : 1.f) : 0.f;
            }
        }
        __syncthreads();
        // ------------------------------------------- gates and scans
        if (GENERAL) {
            // per channel: preconditioner EMA (carried across chunks), write
            // key, erase key, cumulative log decay
            // preconditioner factor f(rho): 1 1/sqrt(rho+eps), 2 1/(rho+eps) (Diag(A)^-1),
            // 3 the latter squashed into [1/x, x] on a log scale; applied to the
            // write key (forms 2, 3 read the state with the raw key) or to the query
            const float lnx = p.precond == 3 ? logf(p.precond_x) : 1.f;
            for (int c = tid; c < dk; c += kThreads) {
                float rh = rho[c], G = 0.f;
                for (int r = 0; r < C; ++r) {
                    const int idx = r * dk + c;
                    const float kv = ld_s(kx, idx);
                    float f = 1.f;
                    if (p.precond && r < Cv) {
                        rh = p.rho_decay * rh + kv * kv;
                        const float a = rh + p.rho_eps;
                        f = p.precond == 1 ? rsqrtf(a)
                          : p.precond == 2 ? 1.f / a
                          : expf(lnx * tanhf(-logf(a) / lnx));
                    }
                    if (p.precond_query) {
                        st_s(qx, idx, ld_s(qx, idx) * f);
                        ex[idx] *= kv;
                    } else {
                        const float kw = kv * f;
                        st_s(kx, idx, kw);
                        ex[idx] *= (p.precond == 1 ? kw : kv);
                    }
                    G += gx[idx];
                    gx[idx] = G;
                }
                rho[c] = rh;
            }
        } else {
            warp0_inclusive_scan(g, C);
        }
        __syncthreads();
        // ------------------------------------------------ L (strictly lower)
        for (int idx = tid; idx < C * C; idx += kThreads) {
            const int r = idx / C, i = idx % C;
            float val = 0.f;
            if (i < r) {
                float acc = 0.f;
                if (GENERAL) {
                    for (int c = 0; c < dk; ++c)
                        acc += ex[r * dk + c] * ld_s(kx, i * dk + c) *
                               expf(gx[(r - 1) * dk + c] - gx[i * dk + c]);
                    val = acc;
                } else {
                    for (int c = 0; c < dk; ++c) acc += ld_s(kx, r * dk + c) * ld_s(kx, i * dk + c);
                    val = bet[r] * expf(g[r] - g[i]) * acc;
                }
            }
            tp[idx] = val;
        }
        __syncthreads();
        // ------------------------------------------------ T = (I + L)^-1
        if (!neumann) {
            // forward substitution, one row at a time: T_rc = -sum_{c<=i<r} L_ri T_ic
            for (int r = 1; r < C; ++r) {
                if (tid < r) lrow[tid] = tp[r * C + tid];
                __syncthreads();
                if (tid < r) {
                    const int c = tid;
                    float s = lrow[c];
                    for (int i = c + 1; i < r; ++i) s += lrow[i] * tp[i * C + c];
                    tp[r * C + c] = -s;
                }
                __syncthreads();
            }
            for (int r = tid; r < C; r += kThreads) tp[r * C + r] = 1.f;
        } else {
            // Horner on the band: T <- M (.) (I + A T), A = -L, T^(0) = I.
            // band[i*(N+1)+d] holds T_{i,i-d}.
            const int W = N + 1;
            float *cur = band, *nxt = band + (size_t)C * W;
            for (int idx = tid; idx < C * W; idx += kThreads) cur[idx] = (idx % W == 0) ? 1.f : 0.f;
            __syncthreads();
            for (int step = 0; step < N; ++step) {
                for (int idx = tid; idx < C * W; idx += kThreads) {
                    const int i = idx / W, d = idx % W, j = i - d;
                    float val = 0.f;
                    if (j >= 0) {
                        val = (d == 0) ? 1.f : 0.f;
                        // sum_{k=j}^{i-1} A_ik T_kj with T_kj in band (k - j <= N)
                        const int kmax = min(i - 1, j + N);
                        for (int kk = j; kk <= kmax; ++kk) val -= tp[i * C + kk] * cur[kk * W + (kk - j)];
                    }
                    nxt[idx] = val;
                }
                __syncthreads();
                float *sw = cur; cur = nxt; nxt = sw;
            }
            for (int idx = tid; idx < C * C; idx += kThreads) {
                const int i = idx / C, j = idx % C, d = i - j;
                tp[idx] = (d >= 0 && d <= N) ? cur[i * W + d] : 0.f;
            }
        }
        __syncthreads();
        // ------------------------------------------------ R = u - h^T e'
        if (GENERAL) {
            // e'_rc = e_rc exp(G_{r-1,c})
            for (int idx = tid; idx < C * dk; idx += kThreads) {
                const int r = idx / dk;
                ex[idx] *= (r > 0) ? expf(gx[idx - dk]) : 1.f;
            }
            __syncthreads();
        }
        for (int idx = tid; idx < C * dvs; idx += kThreads) {
            const int r = idx / dvs, j = idx % dvs;
            float acc = 0.f;
            if (GENERAL) {
                for (int c = 0; c < dk; ++c) acc += ex[r * dk + c] * hs[c * dvs + j];
                ux[idx] = ux[idx] - acc;
            } else {
                for (int c = 0; c < dk; ++c) acc += ld_s(kx, r * dk + c) * hs[c * dvs + j];
                ux[idx] = bet[r] * (ux[idx] - expf(g[r]) * acc);
            }
        }
        __syncthreads();
        // ------------------------------------------------ Delta = T R
        for (int idx = tid; idx < C * dvs; idx += kThreads) {
            const int r = idx / dvs, j = idx % dvs;
            float acc = 0.f;
            for (int i = 0; i <= r; ++i) acc += tp[r * C + i] * ux[i * dvs + j];
            dx[idx] = acc;
        }
        __syncthreads();
        // ------------------------------------------------ P (causal, decayed)
        for (int idx = tid; idx < C * C; idx += kThreads) {
            const int r = idx / C, i = idx % C;
            float val = 0.f;
            if (i <= r) {
                float acc = 0.f;
                if (GENERAL) {
                    for (int c = 0; c < dk; ++c)
                        acc += ld_s(qx, r * dk + c) * ld_s(kx, i * dk + c) *
                               expf(gx[r * dk + c] - gx[i * dk + c]);
                    val = acc;
                } else {
                    for (int c = 0; c < dk; ++c) acc += ld_s(qx, r * dk + c) * ld_s(kx, i * dk + c);
                    val = expf(g[r] - g[i]) * acc;
                }
            }
            tp[idx] = val;
        }
        __syncthreads();
        if (GENERAL) {
            // q <- q (.) e^{G_r};  kw <- kw (.) e^{G_last - G_r}
            for (int idx = tid; idx < C * dk; idx += kThreads) {
                const int c = idx % dk;
                const float Gl = gx[(C - 1) * dk + c];
                st_s(qx, idx, ld_s(qx, idx) * expf(gx[idx]));
                st_s(kx, idx, ld_s(kx, idx) * expf(Gl - gx[idx]));
            }
            __syncthreads();
        }
        // ------------------------------------------------ O
        for (int idx = tid; idx < C * dvs; idx += kThreads) {
            const int r = idx / dvs, j = idx % dvs;
            if (r >= Cv) continue;
            float acc = 0.f;
            for (int c = 0; c < dk; ++c) acc += ld_s(qx, r * dk + c) * hs[c * dvs + j];
            if (!GENERAL) acc *= expf(g[r]);
            for (int i = 0; i <= r; ++i) acc += tp[r * C + i] * dx[i * dvs + j];
            const size_t go = (((size_t)b * T + t0 + r) * H + h) * dv + v0 + j;
            if (p.o_bf16) reinterpret_cast<__nv_bfloat16 *>(p.o)[go] = __float2bfloat16_rn(acc);
            else reinterpret_cast<float *>(p.o)[go] = acc;
        }
        __syncthreads();
        // ------------------------------------------------ state update
        for (int idx = tid; idx < dk * dvs; idx += kThreads) {
            const int c = idx / dvs, j = idx % dvs;
            float acc = 0.f;
            float decay;
            if (GENERAL) {
                for (int r = 0; r < C; ++r) acc += ld_s(kx, r * dk + c) * dx[r * dvs + j];
                decay = expf(gx[(C - 1) * dk + c]);
            } else {
                const float gl = g[C - 1];
                for (int r = 0; r < C; ++r)
                    acc += ld_s(kx, r * dk + c) * expf(gl - g[r]) * dx[r * dvs + j];
                decay = expf(gl);
            }
            hs[idx] = decay * hs[idx] + acc;
        }
    }
    __syncthreads();
    if (p.S_T) {
        for (int idx = tid; idx < dk * dvs; idx += kThreads) {
            const int c = idx / dvs, j = idx % dvs;
            p.S_T[(bh * dk + c) * dv + v0 + j] = hs[idx];
        }
    }
}

}  // namespace

size_t simt_smem_bytes(const FwdParams &p) {
    const int key_bytes = (p.io_bf16 && !p.general) ? 2 : 4;
    const SimtLayout L = simt_layout(p.C, p.dk, p.dvs, p.N, p.mode == GDN_INV_NEUMANN,
                                     p.general, key_bytes);
    return L.total;
}

cudaError_t launch_simt(const FwdParams &p, cudaStream_t stream) {
    const size_t smem = simt_smem_bytes(p);
    dim3 grid(p.slices, p.H, p.B);
    cudaError_t e;
    if (p.general) {
        auto kern = simt_chunk_kernel<float, true>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, kThreads, smem, stream>>>(p);
    } else if (p.io_bf16) {
        auto kern = simt_chunk_kernel<__nv_bfloat16, false>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, kThreads, smem, stream>>>(p);
    } else {
        auto kern = simt_chunk_kernel<float, false>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, kThreads, smem, stream>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace gdn
