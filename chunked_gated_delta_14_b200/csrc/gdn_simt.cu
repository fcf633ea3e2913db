// fp32 CUDA-core path of the chunkwise gated delta rule, for every variant
// (any chunk 16-128, d 16-128, fp32 io, the two-gate rule with per-channel
// decay, gates and the preconditioner).  Per chunk of C tokens (local rows r,
// keys i):
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
// Both are one form, Delta = TB (U - E h), O = Q' h + P Delta,
// h <- diag(d) h + K''^T Delta, whose matrices TB (T diag(beta), or T), P, E,
// Q', K'' and d depend on the keys and gates only.  So the path is two kernels:
//
// 1. simt_prep_kernel -- one block per (chunk, head, batch), all chunks at
//    once: gates, L, T, and the six matrices into the workspace (fp32).  The
//    preconditioner's running average is carried across chunks; two small
//    kernels (rho_local_kernel, rho_combine_kernel) give each chunk its value
//    at the chunk start first.
// 2. simt_chain_kernel -- one block per (batch, head, value slice) walks the
//    chunks in order with the fp32 state h = S^T (dk x dvs) in shared memory,
//    reading each matrix once per chunk.
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
#include <cuda_fp16.h>

#include "gdn_internal.cuh"
#include "gdn_tc_common.cuh"

namespace gdn {
namespace {

constexpr int kThreads = 256;
constexpr int kPrepThreads = 512;   // prep kernel: one block per SM by shared memory, so 16 warps

__device__ __forceinline__ float load_in(const void *p, size_t i, int bf16) {
    if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
    return reinterpret_cast<const float *>(p)[i];
}

// Four consecutive inputs from element i (i a multiple of 4; bf16 or fp32).
__device__ __forceinline__ float4 load4_in(const void *p, size_t i, int bf16) {
    if (bf16) {
        const uint2 u = *reinterpret_cast<const uint2 *>(reinterpret_cast<const __nv_bfloat16 *>(p) + i);
        return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                           __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
    }
    return *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(p) + i);
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

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

// 2^x on the special-function unit (PTX ex2.approx.ftz.f32, relative error
// about 2^-22): the per-channel decay ratios of the two-gate rule, kept in
// log2 form.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Workspace: per chunk-head, fp32 [TB C x C | P C x C | E C x dk | Q' C x dk |
// K'' C x dk | d dk], padded to 16 bytes; then, for the preconditioned two-gate
// rule, the running average at every chunk start, each chunk's own sum and the
// decay's power over the chunk, three times [B, H, chunks, dk].
struct SimtWs {
    size_t tb, pp, e, q, k, d, stride;   // floats
};

__host__ __device__ inline SimtWs simt_ws(int C, int dk) {
    SimtWs w;
    w.tb = 0;
    w.pp = (size_t)C * C;
    w.e = 2 * (size_t)C * C;
    w.q = w.e + (size_t)C * dk;
    w.k = w.q + (size_t)C * dk;
    w.d = w.k + (size_t)C * dk;
    w.stride = (w.d + dk + 3) & ~size_t(3);
    return w;
}

// Row stride (elements) of a C x dk key matrix in shared memory: one extra
// 32-bit word per row, so that a warp reading channel c of 32 consecutive rows
// touches 32 distinct banks.
__host__ __device__ inline int key_stride(int dk, int elem_bytes) { return dk + 4 / elem_bytes; }

// Shared-memory carve-up of the prep kernel, identical on host and device.
struct PrepLayout {
    size_t kx, qx, ex, gx, tp, band, rows, inv, total;
};

__host__ __device__ inline PrepLayout prep_layout(int C, int dk, int N, int neumann, int general,
                                                  int key_bytes) {
    PrepLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t at = off; off = align16(off + bytes); return at; };
    // general: kw, q, e, G all fp32; scalar: k, q stored in the io dtype
    const size_t kb = general ? 4 : (size_t)key_bytes;
    const size_t ks = key_stride(dk, (int)kb);
    L.kx = take((size_t)C * ks * kb);
    L.qx = take((size_t)C * ks * kb);
    L.ex = general ? take((size_t)C * ks * 4) : off;
    L.gx = general ? take((size_t)C * ks * 4) : off;
    L.tp = take((size_t)C * C * 4);
    L.band = neumann ? take((size_t)2 * C * (N + 1) * 4) : off;
    L.rows = take((size_t)4 * C * 4);        // g / log alpha, beta, lrow, spare
    // chunk 64, exact: the blocked inverse's L and T (row stride LSTR) and scratch
    L.inv = (C == 64 && !neumann) ? take((size_t)(2 * 64 * tc::LSTR + 1024) * 4) : off;
    L.total = off;
    return L;
}

// Shared-memory carve-up of the chain kernel.
struct ChainLayout {
    size_t hs, ux, dx, ox, mat, dl, total;
};

__host__ __device__ inline ChainLayout chain_layout(int C, int dk, int dvs) {
    ChainLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t at = off; off = align16(off + bytes); return at; };
    L.hs = take((size_t)dk * dvs * 4);
    L.ux = take((size_t)C * dvs * 4);
    L.dx = take((size_t)C * dvs * 4);
    L.ox = take((size_t)C * dvs * 4);
    L.mat = take((size_t)C * ((C > dk ? C : dk) + 4) * 4);   // rows padded by 4 floats
    L.dl = take((size_t)dk * 4);
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

// The preconditioner's running average rho_t = decay rho_{t-1} + k_t (.) k_t,
// per (batch, head, key channel), at every chunk start.  Over a chunk of Cv
// tokens rho_end = decay^Cv rho_start + sum_r decay^(Cv-1-r) k_r (.) k_r, so the
// chunks' own sums come first, in parallel (rho_local_kernel), and a short
// pass over the chunks chains them (rho_combine_kernel).
__global__ void rho_local_kernel(const FwdParams p, float *sums, float *pows) {
    const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z, c = threadIdx.x;
    if (c >= p.dk) return;
    const int NC = (p.T + p.C - 1) / p.C;
    const int t0 = n * p.C, t1 = min(p.T, t0 + p.C);
    float s = 0.f, a = 1.f;
#pragma unroll 4
    for (int t = t0; t < t1; ++t) {
        const float kv = load_in(p.k, (((size_t)b * p.T + t) * p.H + h) * p.dk + c, p.io_bf16);
        s = p.rho_decay * s + kv * kv;
        a *= p.rho_decay;
    }
    const size_t o = (((size_t)b * p.H + h) * NC + n) * p.dk + c;
    sums[o] = s;
    pows[o] = a;
}

__global__ void rho_combine_kernel(const FwdParams p, const float *sums, const float *pows, float *rho_start) {
    const int h = blockIdx.x, b = blockIdx.y, c = threadIdx.x;
    if (c >= p.dk) return;
    const int NC = (p.T + p.C - 1) / p.C;
    float rh = 0.f;
    for (int n = 0; n < NC; ++n) {
        const size_t o = (((size_t)b * p.H + h) * NC + n) * p.dk + c;
        rho_start[o] = rh;
        rh = pows[o] * rh + sums[o];
    }
}

// One block per (chunk, head, batch): the state-independent matrices of one chunk.
// TCOUT (two-gate rule, chunk 64, d_k 128): written as fp16 rows for the
// tensor-core chain (gen_rows), together with U = w (.) v, instead of fp32.
// rho0: the preconditioner's running average at every chunk start.
template <typename KS, bool GENERAL, bool TCOUT = false>
__global__ void __launch_bounds__(kPrepThreads)
simt_prep_kernel(const FwdParams p, float *ws, const float *rho0) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int C = p.C, dk = p.dk, H = p.H, T = p.T;
    const int NC = (T + C - 1) / C;
    const int t0 = n * C, Cv = min(C, T - t0);
    const int tid = threadIdx.x;
    const int neumann = (p.mode == GDN_INV_NEUMANN);
    const int N = p.N;
    const PrepLayout Ly = prep_layout(C, dk, N, neumann, GENERAL ? 1 : 0, (int)sizeof(KS));
    // key rows padded by one word: threads that read the same channel of
    // consecutive rows then hit distinct banks
    const int ks = key_stride(dk, GENERAL ? 4 : (int)sizeof(KS));
    KS *kx = reinterpret_cast<KS *>(smem + Ly.kx);       // keys (write keys kw)
    KS *qx = reinterpret_cast<KS *>(smem + Ly.qx);       // read keys
    float *ex = reinterpret_cast<float *>(smem + Ly.ex); // erase keys (two-gate)
    float *gx = reinterpret_cast<float *>(smem + Ly.gx); // per-channel cumulative log2 decay
    float *tp = reinterpret_cast<float *>(smem + Ly.tp); // L -> T, C x C
    float *band = reinterpret_cast<float *>(smem + Ly.band);
    float *rows = reinterpret_cast<float *>(smem + Ly.rows);
    float *g = rows;                 // scalar: log alpha -> cumulative g
    float *bet = rows + C;           // scalar: beta
    float *lrow = rows + 2 * C;      // forward-substitution row copy
    const size_t bh = (size_t)b * H + h;
    const SimtWs W = simt_ws(C, dk);
    float *out = ws + (bh * NC + n) * W.stride;
    const GenRows GR = gen_rows(p.dv);
    __half *ob = reinterpret_cast<__half *>(ws) + (bh * NC + n) * (size_t)GR.rows * 64;   // TCOUT rows

    // ---------------------------------------------------------- load
    // four consecutive channels per item, four items' loads issued before the
    // first store, so that their latencies overlap
    {
        constexpr int UNR = 4;
        const int n4 = C * dk / 4;
        const float4 zero4 = make_float4(0.f, 0.f, 0.f, 0.f), one4 = make_float4(1.f, 1.f, 1.f, 1.f);
        for (int base = tid; base < n4; base += kPrepThreads * UNR) {
            float4 kv[UNR], qv[UNR], ev[UNR], av[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int i4 = base + kPrepThreads * u;
                kv[u] = qv[u] = ev[u] = zero4;
                av[u] = one4;
                if (i4 < n4) {
                    const int r = (4 * i4) / dk, c = (4 * i4) % dk;
                    if (r < Cv) {
                        const size_t gi = (((size_t)b * T + t0 + r) * H + h) * dk + c;
                        kv[u] = load4_in(p.k, gi, p.io_bf16);
                        qv[u] = load4_in(p.q, gi, p.io_bf16);
                        if (GENERAL) {
                            ev[u] = p.erase ? load4_in(p.erase, gi, p.io_bf16) : one4;
                            if (p.alpha) {
                                if (p.alpha_pc) {
                                    av[u] = *reinterpret_cast<const float4 *>(p.alpha + gi);
                                } else {
                                    const float a = p.alpha[gi / dk];
                                    av[u] = make_float4(a, a, a, a);
                                }
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int i4 = base + kPrepThreads * u;
                if (i4 < n4) {
                    const int r = (4 * i4) / dk, c = (4 * i4) % dk, si = r * ks + c;
                    const float kk[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
                    const float qq[4] = {qv[u].x, qv[u].y, qv[u].z, qv[u].w};
                    const float ee[4] = {ev[u].x, ev[u].y, ev[u].z, ev[u].w};
                    const float aa[4] = {av[u].x, av[u].y, av[u].z, av[u].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        st_s(kx, si + e, kk[e]);
                        st_s(qx, si + e, qq[e]);
                        if (GENERAL) {
                            ex[si + e] = ee[e];
                            gx[si + e] = log2f(aa[e]);   // 0 past the end and without a decay
                        }
                    }
                }
            }
        }
    }
    if (!GENERAL) {
        for (int r = tid; r < C; r += kPrepThreads) {
            const size_t ti = ((size_t)b * T + t0 + r) * H + h;
            g[r] = (r < Cv && p.alpha) ? logf(p.alpha[ti]) : 0.f;
            bet[r] = (r < Cv) ? (p.beta ? p.beta[ti] : 1.f) : 0.f;
        }
    }
    __syncthreads();
    // ------------------------------------------- gates and scans
    if (GENERAL) {
        // per channel: preconditioner average (from the chunk start), write
        // key, erase key, cumulative log decay.  Preconditioner factor f(rho):
        // 1 1/sqrt(rho+eps), 2 1/(rho+eps) (Diag(A)^-1), 3 the latter squashed
        // into [1/x, x] on a log scale; applied to the write key (forms 2, 3
        // read the state with the raw key) or to the query
        const float lnx = p.precond == 3 ? logf(p.precond_x) : 1.f;
        for (int c = tid; c < dk; c += kPrepThreads) {
            float rh = p.precond ? rho0[(bh * NC + n) * dk + c] : 0.f, G = 0.f;
            for (int r = 0; r < C; ++r) {
                const int idx = r * ks + c;
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
        }
    } else {
        warp0_inclusive_scan(g, C);
    }
    __syncthreads();
    // The two-gate rule's decayed Gram sums_c X[r][c] kw[i][c] 2^{GX[r][c] - G[i][c]}
    // over the lower 4 x 4 tiles (r-block >= i-block), four lanes per tile on
    // interleaved channel quarters (c = 4 cc + part), reduced with shuffles: every
    // warp of the block has work and each chain is a quarter as long.  GX is G_r,
    // or G_{r-1} (shift 1, G_{-1} = 0).  store(r0, i0, acc) writes one tile.
    auto decayed_gram = [&](const float *X, int shift, auto &&store) {
        // tiles below the diagonal first (4 (nT (nT - 1) / 2) items, whole warps at
        // C = 64), then the diagonal ones, so that no warp mixes the two forms
        const int nT = C / 4, offd = nT * (nT - 1) / 2, tiles = offd + nT;
        const int items = ((4 * tiles + 31) / 32) * 32;
        for (int w = tid; w < items; w += kPrepThreads) {
            const int part = w & 3, tix = w >> 2;
            const bool need = tix < tiles, diag = tix >= offd;
            int R = tix - offd, I = R;
            if (!diag) {
                R = 1;
                while ((R + 1) * R / 2 <= tix) ++R;
                I = tix - R * (R - 1) / 2;
            }
            const int r0 = 4 * R, i0 = 4 * I;
            float acc[4][4] = {};
            if (need && !diag) {
                // every row's exponent point lies after the tile's last key m = i0 + 3:
                // 2^{GX_r - G_i} = 2^{GX_r - G_m} 2^{G_m - G_i}, both factors <= 1,
                // 8 exponentials per 16 products
                for (int cc = 0; cc < dk / 4; ++cc) {
                    const int c = 4 * cc + part;
                    const float gm = gx[(i0 + 3) * ks + c];
                    float xr[4], yi[4];
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        xr[a] = X[(r0 + a) * ks + c] * fast_exp2(gx[(r0 + a - shift) * ks + c] - gm);
                        yi[a] = ld_s(kx, (i0 + a) * ks + c) * fast_exp2(gm - gx[(i0 + a) * ks + c]);
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc[a][e] += xr[a] * yi[e];
                }
            } else if (need) {
                for (int cc = 0; cc < dk / 4; ++cc) {
                    const int c = 4 * cc + part;
                    float xr[4], gr[4], yi[4], gi[4];
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        xr[a] = X[(r0 + a) * ks + c];
                        gr[a] = (shift && r0 + a == 0) ? 0.f : gx[(r0 + a - shift) * ks + c];
                        yi[a] = ld_s(kx, (i0 + a) * ks + c);
                        gi[a] = gx[(i0 + a) * ks + c];
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc[a][e] += xr[a] * yi[e] * fast_exp2(gr[a] - gi[e]);
                }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc[a][e] += __shfl_xor_sync(0xffffffffu, acc[a][e], 1);
                    acc[a][e] += __shfl_xor_sync(0xffffffffu, acc[a][e], 2);
                }
            if (need && part == 0) store(r0, i0, acc);
        }
    };
    // ------------------------------------------------ L (strictly lower)
    if (GENERAL) {
        decayed_gram(reinterpret_cast<const float *>(ex), 1, [&](int r0, int i0, const float (&acc)[4][4]) {
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int e = 0; e < 4; ++e) tp[(r0 + a) * C + i0 + e] = (i0 + e < r0 + a) ? acc[a][e] : 0.f;
        });
        for (int idx = tid; idx < C * C; idx += kPrepThreads)
            if (((idx % C) >> 2) > ((idx / C) >> 2)) tp[idx] = 0.f;   // tiles above the diagonal
    } else {
        // 4 x 4 register tiles (rows r0.., keys i0..): 8 loads per 16 products
        for (int t = tid; t < (C / 4) * (C / 4); t += kPrepThreads) {
            const int r0 = 4 * (t / (C / 4)), i0 = 4 * (t % (C / 4));
            float acc[4][4] = {};
            if (i0 < r0 + 3) {
                for (int c = 0; c < dk; ++c) {
                    float kr[4], ki[4];
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        kr[a] = ld_s(kx, (r0 + a) * ks + c);
                        ki[a] = ld_s(kx, (i0 + a) * ks + c);
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc[a][e] += kr[a] * ki[e];
                }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = r0 + a, i = i0 + e;
                    tp[r * C + i] = (i < r) ? bet[r] * expf(g[r] - g[i]) * acc[a][e] : 0.f;
                }
        }
    }
    __syncthreads();
    // ------------------------------------------------ T = (I + L)^-1
    if (!neumann && C == 64) {
        // blocked: 16 x 16 diagonal blocks by forward substitution, merged
        // 16 -> 32 -> 64 by T21 = -T22 L21 T11, by the first 256 threads
        float *Lb = reinterpret_cast<float *>(smem + Ly.inv), *Tb = Lb + 64 * tc::LSTR, *Yb = Tb + 64 * tc::LSTR;
        for (int idx = tid; idx < 64 * 64; idx += kPrepThreads) {
            const int r = idx >> 6, c = idx & 63;
            Lb[r * tc::LSTR + c] = tp[idx];
            Tb[r * tc::LSTR + c] = 0.f;
        }
        __syncthreads();
        if (tid < 256) tc::invert_exact(Lb, Tb, Yb, tid, 1);
        __syncthreads();
        for (int idx = tid; idx < 64 * 64; idx += kPrepThreads) {
            const int r = idx >> 6, c = idx & 63;
            tp[idx] = (c <= r) ? Tb[r * tc::LSTR + c] : 0.f;
        }
    } else if (!neumann) {
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
        for (int r = tid; r < C; r += kPrepThreads) tp[r * C + r] = 1.f;
    } else {
        // Horner on the band: T <- M (.) (I + A T), A = -L, T^(0) = I.
        // band[i*(N+1)+d] holds T_{i,i-d}.
        const int Wd = N + 1;
        float *cur = band, *nxt = band + (size_t)C * Wd;
        for (int idx = tid; idx < C * Wd; idx += kPrepThreads) cur[idx] = (idx % Wd == 0) ? 1.f : 0.f;
        __syncthreads();
        for (int step = 0; step < N; ++step) {
            for (int idx = tid; idx < C * Wd; idx += kPrepThreads) {
                const int i = idx / Wd, d = idx % Wd, j = i - d;
                float val = 0.f;
                if (j >= 0) {
                    val = (d == 0) ? 1.f : 0.f;
                    // sum_{k=j}^{i-1} A_ik T_kj with T_kj in band (k - j <= N)
                    const int kmax = min(i - 1, j + N);
                    for (int kk = j; kk <= kmax; ++kk) val -= tp[i * C + kk] * cur[kk * Wd + (kk - j)];
                }
                nxt[idx] = val;
            }
            __syncthreads();
            float *sw = cur; cur = nxt; nxt = sw;
        }
        for (int idx = tid; idx < C * C; idx += kPrepThreads) {
            const int i = idx / C, j = idx % C, d = i - j;
            tp[idx] = (d >= 0 && d <= N) ? cur[i * Wd + d] : 0.f;
        }
    }
    __syncthreads();
    // ------------------------------------------------ the chunk's matrices
    // TB = T diag(beta) (scalar rule; the two-gate rule has no beta)
    for (int idx = tid; idx < C * C; idx += kPrepThreads) {
        const float tb = GENERAL ? tp[idx] : tp[idx] * bet[idx % C];
        if (TCOUT) {
            const __half hi = __float2half_rn(tb);
            ob[(size_t)GR.tb * 64 + idx] = hi;
            ob[(size_t)GR.tbl * 64 + idx] = __float2half_rn(tb - __half2float(hi));
        } else {
            out[W.tb + idx] = tb;
        }
    }
    // P: decayed causal scores
    auto store_p = [&](int r, int i, float val) {
        if (TCOUT) {
            const __half hi = __float2half_rn(val);
            ob[(size_t)(GR.pp + r) * 64 + i] = hi;
            ob[(size_t)(GR.ppl + r) * 64 + i] = __float2half_rn(val - __half2float(hi));
        } else {
            out[W.pp + r * C + i] = val;
        }
    };
    if (GENERAL) {
        decayed_gram(reinterpret_cast<const float *>(qx), 0, [&](int r0, int i0, const float (&acc)[4][4]) {
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int e = 0; e < 4; ++e) store_p(r0 + a, i0 + e, (i0 + e <= r0 + a) ? acc[a][e] : 0.f);
        });
        for (int idx = tid; idx < C * C; idx += kPrepThreads)
            if (((idx % C) >> 2) > ((idx / C) >> 2)) store_p(idx / C, idx % C, 0.f);   // above the diagonal
    } else {
        // 4 x 4 register tiles
        for (int t = tid; t < (C / 4) * (C / 4); t += kPrepThreads) {
            const int r0 = 4 * (t / (C / 4)), i0 = 4 * (t % (C / 4));
            float acc[4][4] = {};
            if (i0 <= r0 + 3) {
                for (int c = 0; c < dk; ++c) {
                    float qr[4], ki[4];
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        qr[a] = ld_s(qx, (r0 + a) * ks + c);
                        ki[a] = ld_s(kx, (i0 + a) * ks + c);
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc[a][e] += qr[a] * ki[e];
                }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = r0 + a, i = i0 + e;
                    store_p(r, i, (i <= r) ? expf(g[r] - g[i]) * acc[a][e] : 0.f);
                }
        }
    }
    // E (the state read), Q' (the output read), K'' (the state write)
    if (TCOUT) {
        // 64-column blocks: channel c of row r at row (block base + 64 (c / 64) + r);
        // two channels per item, stored as one fp16 pair
        for (int idx = tid; idx < C * dk / 2; idx += kPrepThreads) {
            const int r = (2 * idx) / dk, c = (2 * idx) % dk, si = r * ks + c;
            float e2[2], q2[2], k2[2];
#pragma unroll
            for (int z = 0; z < 2; ++z) {
                const float Gl = gx[(C - 1) * ks + c + z];
                e2[z] = ex[si + z] * ((r > 0) ? fast_exp2(gx[si + z - ks]) : 1.f);
                q2[z] = ld_s(qx, si + z) * fast_exp2(gx[si + z]);
                k2[z] = ld_s(kx, si + z) * fast_exp2(Gl - gx[si + z]);
            }
            const size_t o = (size_t)(64 * (c >> 6) + r) * 64 + (c & 63);
            *reinterpret_cast<__half2 *>(ob + (size_t)GR.e * 64 + o) = __floats2half2_rn(e2[0], e2[1]);
            *reinterpret_cast<__half2 *>(ob + (size_t)GR.q * 64 + o) = __floats2half2_rn(q2[0], q2[1]);
            *reinterpret_cast<__half2 *>(ob + (size_t)GR.k * 64 + o) = __floats2half2_rn(k2[0], k2[1]);
        }
    }
    for (int idx = tid; idx < (TCOUT ? 0 : C * dk); idx += kPrepThreads) {
        const int r = idx / dk, c = idx % dk, si = r * ks + c;
        if (GENERAL) {
            const float Gl = gx[(C - 1) * ks + c];
            out[W.e + idx] = ex[si] * ((r > 0) ? fast_exp2(gx[si - ks]) : 1.f);
            out[W.q + idx] = ld_s(qx, si) * fast_exp2(gx[si]);
            out[W.k + idx] = ld_s(kx, si) * fast_exp2(Gl - gx[si]);
        } else {
            const float gl = g[C - 1];
            out[W.e + idx] = ld_s(kx, si) * expf(g[r]);
            out[W.q + idx] = ld_s(qx, si) * expf(g[r]);
            out[W.k + idx] = ld_s(kx, si) * expf(gl - g[r]);
        }
    }
    // d: the state's decay over the chunk
    for (int c = tid; c < dk; c += kPrepThreads) {
        const float dc = GENERAL ? fast_exp2(gx[(C - 1) * ks + c]) : expf(g[C - 1]);
        if (TCOUT) reinterpret_cast<float *>(ob + (size_t)GR.d * 64)[c] = dc;
        else out[W.d + c] = dc;
    }
    if (TCOUT) {
        // U = w (.) v (hi, lo), one 64-column block per value slice; zero past the
        // end.  Four values per item, four items' loads in flight together.
        constexpr int UNR = 4;
        const int n4 = C * p.dv / 4;
        for (int base = tid; base < n4; base += kPrepThreads * UNR) {
            float4 vv[UNR], ww[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int i4 = base + kPrepThreads * u;
                vv[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                ww[u] = make_float4(1.f, 1.f, 1.f, 1.f);
                if (i4 < n4) {
                    const int r = (4 * i4) / p.dv, j = (4 * i4) % p.dv;
                    if (r < Cv) {
                        const size_t gi = (((size_t)b * T + t0 + r) * H + h) * p.dv + j;
                        vv[u] = load4_in(p.v, gi, p.io_bf16);
                        if (p.write) ww[u] = load4_in(p.write, gi, p.io_bf16);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int i4 = base + kPrepThreads * u;
                if (i4 < n4) {
                    const int r = (4 * i4) / p.dv, j = (4 * i4) % p.dv;
                    const float x[4] = {vv[u].x * ww[u].x, vv[u].y * ww[u].y, vv[u].z * ww[u].z, vv[u].w * ww[u].w};
                    __half hi[4], lo[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        hi[e] = __float2half_rn(x[e]);
                        lo[e] = __float2half_rn(x[e] - __half2float(hi[e]));
                    }
                    const size_t o = (size_t)(64 * (j >> 6) + r) * 64 + (j & 63);
                    *reinterpret_cast<__half2 *>(ob + (size_t)GR.u * 64 + o) = __halves2half2(hi[0], hi[1]);
                    *reinterpret_cast<__half2 *>(ob + (size_t)GR.u * 64 + o + 2) = __halves2half2(hi[2], hi[3]);
                    *reinterpret_cast<__half2 *>(ob + (size_t)GR.ul * 64 + o) = __halves2half2(lo[0], lo[1]);
                    *reinterpret_cast<__half2 *>(ob + (size_t)GR.ul * 64 + o + 2) = __halves2half2(lo[2], lo[3]);
                }
            }
        }
    }
}

// Copy a rows x cols matrix (cols a multiple of 4, 16-byte aligned) from the
// workspace into shared memory with rows cols + 4 floats apart, so that the
// row reads of one warp fall into different banks.
__device__ __forceinline__ void stage(float *dst, const float *src, int rows, int cols) {
    const int q = cols / 4;
    const float4 *s = reinterpret_cast<const float4 *>(src);
    for (int i = threadIdx.x; i < rows * q; i += kThreads) {
        const int r = i / q, c = i % q;
        *reinterpret_cast<float4 *>(dst + (size_t)r * (cols + 4) + 4 * c) = __ldg(s + i);
    }
}

// 2 x 2 output tiles of a rows x dvs product: rows r0, r0 + 1, columns j0, j0 + 1.
#define FOR_TILES(rows, dvs)                                                         \
    for (int t_ = threadIdx.x; t_ < ((rows) / 2) * ((dvs) / 2); t_ += kThreads)      \
        if (const int r0 = 2 * (t_ / ((dvs) / 2)), j0 = 2 * (t_ % ((dvs) / 2)); true)

// One block per (value slice, head, batch): the chunks of one sequence in order.
template <bool GENERAL>
__global__ void __launch_bounds__(kThreads)
simt_chain_kernel(const FwdParams p, const float *ws) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int slice = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int C = p.C, dk = p.dk, dv = p.dv, dvs = p.dvs, H = p.H, T = p.T;
    const int NC = (T + C - 1) / C;
    const int v0 = slice * dvs;
    const int tid = threadIdx.x;
    const ChainLayout Ly = chain_layout(C, dk, dvs);
    float *hs = reinterpret_cast<float *>(smem + Ly.hs);   // state h, dk x dvs
    float *ux = reinterpret_cast<float *>(smem + Ly.ux);   // values -> R
    float *dx = reinterpret_cast<float *>(smem + Ly.dx);   // Delta
    float *ox = reinterpret_cast<float *>(smem + Ly.ox);   // Q' h
    float *mat = reinterpret_cast<float *>(smem + Ly.mat); // the chunk matrix of each step
    float *dl = reinterpret_cast<float *>(smem + Ly.dl);   // the state's decay
    const int mk = dk + 4, mc = C + 4;                     // staged row strides
    const size_t bh = (size_t)b * H + h;
    const SimtWs W = simt_ws(C, dk);
    auto ld2 = [](const float *x) { return *reinterpret_cast<const float2 *>(x); };

    for (int idx = tid; idx < dk * dvs; idx += kThreads) {
        const int c = idx / dvs, j = idx % dvs;
        hs[idx] = p.S0 ? p.S0[(bh * dk + c) * dv + v0 + j] : 0.f;
    }
    for (int n = 0; n < NC; ++n) {
        const int t0 = n * C, Cv = min(C, T - t0);
        const float *src = ws + (bh * NC + n) * W.stride;
        __syncthreads();  // previous chunk fully consumed
        // ---------------------------------------------- U and E
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
        stage(mat, src + W.e, C, dk);
        for (int c = tid; c < dk; c += kThreads) dl[c] = src[W.d + c];
        __syncthreads();
        // ---------------------------------------------- R = U - E h
        FOR_TILES(C, dvs) {
            float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
            for (int c = 0; c < dk; ++c) {
                const float e0 = mat[r0 * mk + c], e1 = mat[(r0 + 1) * mk + c];
                const float2 hv = ld2(hs + c * dvs + j0);
                a00 += e0 * hv.x; a01 += e0 * hv.y; a10 += e1 * hv.x; a11 += e1 * hv.y;
            }
            ux[r0 * dvs + j0] -= a00; ux[r0 * dvs + j0 + 1] -= a01;
            ux[(r0 + 1) * dvs + j0] -= a10; ux[(r0 + 1) * dvs + j0 + 1] -= a11;
        }
        __syncthreads();
        stage(mat, src + W.tb, C, C);
        __syncthreads();
        // ---------------------------------------------- Delta = TB R (TB lower triangular)
        FOR_TILES(C, dvs) {
            float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
            for (int i = 0; i < r0 + 2; ++i) {
                const float t0v = mat[r0 * mc + i], t1v = mat[(r0 + 1) * mc + i];
                const float2 rv = ld2(ux + i * dvs + j0);
                a00 += t0v * rv.x; a01 += t0v * rv.y; a10 += t1v * rv.x; a11 += t1v * rv.y;
            }
            dx[r0 * dvs + j0] = a00; dx[r0 * dvs + j0 + 1] = a01;
            dx[(r0 + 1) * dvs + j0] = a10; dx[(r0 + 1) * dvs + j0 + 1] = a11;
        }
        __syncthreads();
        stage(mat, src + W.q, C, dk);
        __syncthreads();
        // ---------------------------------------------- O = Q' h + P Delta
        FOR_TILES(C, dvs) {
            float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
            for (int c = 0; c < dk; ++c) {
                const float q0 = mat[r0 * mk + c], q1 = mat[(r0 + 1) * mk + c];
                const float2 hv = ld2(hs + c * dvs + j0);
                a00 += q0 * hv.x; a01 += q0 * hv.y; a10 += q1 * hv.x; a11 += q1 * hv.y;
            }
            ox[r0 * dvs + j0] = a00; ox[r0 * dvs + j0 + 1] = a01;
            ox[(r0 + 1) * dvs + j0] = a10; ox[(r0 + 1) * dvs + j0 + 1] = a11;
        }
        __syncthreads();
        stage(mat, src + W.pp, C, C);
        __syncthreads();
        FOR_TILES(C, dvs) {
            float a[2][2] = {{ox[r0 * dvs + j0], ox[r0 * dvs + j0 + 1]},
                             {ox[(r0 + 1) * dvs + j0], ox[(r0 + 1) * dvs + j0 + 1]}};
            for (int i = 0; i < r0 + 2; ++i) {
                const float p0 = mat[r0 * mc + i], p1 = mat[(r0 + 1) * mc + i];
                const float2 dv2 = ld2(dx + i * dvs + j0);
                a[0][0] += p0 * dv2.x; a[0][1] += p0 * dv2.y; a[1][0] += p1 * dv2.x; a[1][1] += p1 * dv2.y;
            }
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int r = r0 + e;
                if (r >= Cv) continue;
                const size_t go = (((size_t)b * T + t0 + r) * H + h) * dv + v0 + j0;
                if (p.o_bf16) {
                    __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(p.o) + go;
                    o[0] = __float2bfloat16_rn(a[e][0]);
                    o[1] = __float2bfloat16_rn(a[e][1]);
                } else {
                    float *o = reinterpret_cast<float *>(p.o) + go;
                    o[0] = a[e][0];
                    o[1] = a[e][1];
                }
            }
        }
        __syncthreads();
        stage(mat, src + W.k, C, dk);
        __syncthreads();
        // ---------------------------------------------- h <- diag(d) h + K''^T Delta
        FOR_TILES(dk, dvs) {
            const int c0 = r0;
            float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
            for (int r = 0; r < C; ++r) {
                const float2 kv = ld2(mat + r * mk + c0);
                const float2 dv2 = ld2(dx + r * dvs + j0);
                a00 += kv.x * dv2.x; a01 += kv.x * dv2.y; a10 += kv.y * dv2.x; a11 += kv.y * dv2.y;
            }
            float *h0 = hs + c0 * dvs + j0, *h1 = hs + (c0 + 1) * dvs + j0;
            h0[0] = dl[c0] * h0[0] + a00; h0[1] = dl[c0] * h0[1] + a01;
            h1[0] = dl[c0 + 1] * h1[0] + a10; h1[1] = dl[c0 + 1] * h1[1] + a11;
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
#undef FOR_TILES

template <typename KS, bool GENERAL>
cudaError_t launch_pair(const FwdParams &p, float *ws, cudaStream_t stream) {
    const int NC = (p.T + p.C - 1) / p.C;
    const PrepLayout pl = prep_layout(p.C, p.dk, p.N, p.mode == GDN_INV_NEUMANN, GENERAL ? 1 : 0, (int)sizeof(KS));
    const ChainLayout cl = chain_layout(p.C, p.dk, p.dvs);
    auto prep = simt_prep_kernel<KS, GENERAL>;
    auto chain = simt_chain_kernel<GENERAL>;
    cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.total);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(chain, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cl.total);
    if (e != cudaSuccess) return e;
    const size_t chunks = (size_t)p.B * p.H * NC;
    float *rho0 = ws + chunks * simt_ws(p.C, p.dk).stride;
    if (GENERAL && p.precond) {
        float *sums = rho0 + chunks * p.dk, *pows = sums + chunks * p.dk;
        rho_local_kernel<<<dim3(NC, p.H, p.B), 128, 0, stream>>>(p, sums, pows);
        rho_combine_kernel<<<dim3(p.H, p.B), 128, 0, stream>>>(p, sums, pows, rho0);
    }
    prep<<<dim3(NC, p.H, p.B), kPrepThreads, pl.total, stream>>>(p, ws, rho0);
    chain<<<dim3(p.slices, p.H, p.B), kThreads, cl.total, stream>>>(p, ws);
    return cudaGetLastError();
}

}  // namespace

size_t simt_smem_bytes(const FwdParams &p) {
    const int key_bytes = (p.io_bf16 && !p.general) ? 2 : 4;
    const PrepLayout pl = prep_layout(p.C, p.dk, p.N, p.mode == GDN_INV_NEUMANN, p.general, key_bytes);
    const ChainLayout cl = chain_layout(p.C, p.dk, p.dvs);
    return pl.total > cl.total ? pl.total : cl.total;
}

size_t simt_workspace_bytes(const FwdParams &p) {
    const size_t NC = (size_t)(p.T + p.C - 1) / p.C;
    const size_t chunks = (size_t)p.B * p.H * NC;
    size_t floats = chunks * simt_ws(p.C, p.dk).stride;
    if (p.general && p.precond) floats += 3 * chunks * p.dk;   // start values, chunk sums, decay powers
    return floats * sizeof(float);
}

size_t gen_prep_workspace_bytes(const FwdParams &p) {
    const size_t NC = (size_t)(p.T + p.C - 1) / p.C;
    const size_t chunks = (size_t)p.B * p.H * NC;
    size_t bytes = chunks * (size_t)gen_rows(p.dv).rows * 128;
    if (p.precond) bytes += 3 * chunks * p.dk * sizeof(float);
    return bytes;
}

cudaError_t launch_gen_prep(const FwdParams &p, void *workspace, cudaStream_t stream) {
    const int NC = (p.T + p.C - 1) / p.C;
    const size_t chunks = (size_t)p.B * p.H * NC;
    float *ws = reinterpret_cast<float *>(workspace);
    float *rho0 = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) +
                                            chunks * (size_t)gen_rows(p.dv).rows * 128);
    const PrepLayout pl = prep_layout(p.C, p.dk, p.N, p.mode == GDN_INV_NEUMANN, 1, 4);
    auto prep = simt_prep_kernel<float, true, true>;
    cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.total);
    if (e != cudaSuccess) return e;
    if (p.precond) {
        float *sums = rho0 + chunks * p.dk, *pows = sums + chunks * p.dk;
        rho_local_kernel<<<dim3(NC, p.H, p.B), 128, 0, stream>>>(p, sums, pows);
        rho_combine_kernel<<<dim3(p.H, p.B), 128, 0, stream>>>(p, sums, pows, rho0);
    }
    prep<<<dim3(NC, p.H, p.B), kPrepThreads, pl.total, stream>>>(p, ws, rho0);
    return cudaGetLastError();
}

cudaError_t launch_simt(const FwdParams &p, void *workspace, cudaStream_t stream) {
    float *ws = reinterpret_cast<float *>(workspace);
    if (p.general) return launch_pair<float, true>(p, ws, stream);
    if (p.io_bf16) return launch_pair<__nv_bfloat16, false>(p, ws, stream);
    return launch_pair<float, false>(p, ws, stream);
}

}  // namespace gdn
