// Device pieces shared by the two tensor-core kernels (key side, state chain).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "sm100.cuh"

namespace gdn {
namespace tc {

using namespace sm100;

constexpr int C = 64;     // chunk
constexpr int DK = 128;   // key dim

// Per-chunk gate quantities, written by one warp's scan.
struct ChunkParams {
    float g2[C];    // cumulative log2 decay at each row
    float al[C];    // alpha_r (1 on padded rows)
    float dblk[C];  // 2^(g2 at the end of r's 16-row block - g2_r)
    float eg[C];    // e^{g_r}
    float bet[C];   // beta_r (0 on padded rows)
    float egc[C];   // e^{g_C - g_r}
    float egC;      // e^{g_C}
    int Cv;         // valid rows
    float pad[2];
};

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float2 unpack_h2(uint32_t u) {
    __half2 h = *reinterpret_cast<__half2 *>(&u);
    return __half22float2(h);
}

__device__ __forceinline__ float2 unpack_bf2(uint32_t u) {
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162 *>(&u);
    return __bfloat1622float2(h);
}

// Write 64 fp32 values as one fp16 row of a 128-byte swizzled tile.
__device__ __forceinline__ void st_row_f16(uint8_t *tile, int r, const float *x) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint4 u;
        u.x = pack_h2(x[8 * j + 0], x[8 * j + 1]);
        u.y = pack_h2(x[8 * j + 2], x[8 * j + 3]);
        u.z = pack_h2(x[8 * j + 4], x[8 * j + 5]);
        u.w = pack_h2(x[8 * j + 6], x[8 * j + 7]);
        *reinterpret_cast<uint4 *>(tile + sw128_off(r, j)) = u;
    }
}

__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float *x) {
    uint32_t a[32], b[32];
    tmem_ld32(taddr, a);
    tmem_ld32(taddr + 32, b);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        x[i] = __uint_as_float(a[i]);
        x[32 + i] = __uint_as_float(b[i]);
    }
}

// Gates of rows (lane, lane + 32) of one chunk: alpha (1 past the end), beta (0 past the end).
__device__ __forceinline__ void fetch_gates(const float *alpha, const float *beta, int b, int T, int H,
                                            int h, int t0, int lane, bool valid_chunk, float &a0, float &a1,
                                            float &b0, float &b1) {
    const int r0 = lane, r1 = lane + 32;
    const size_t i0 = ((size_t)b * T + t0 + r0) * H + h;
    const size_t i1 = ((size_t)b * T + t0 + r1) * H + h;
    const bool ok0 = valid_chunk && (t0 + r0 < T), ok1 = valid_chunk && (t0 + r1 < T);
    a0 = ok0 ? (alpha ? __ldg(alpha + i0) : 1.f) : 1.f;
    a1 = ok1 ? (alpha ? __ldg(alpha + i1) : 1.f) : 1.f;
    b0 = ok0 ? (beta ? __ldg(beta + i0) : 1.f) : 0.f;
    b1 = ok1 ? (beta ? __ldg(beta + i1) : 1.f) : 0.f;
}

// Cumulative log2 decay over one chunk by one warp (warp-shuffle scan, rows
// lane and lane + 32), and the derived per-row factors.
__device__ __forceinline__ void scan_gates(ChunkParams *par, float a0, float a1, float b0, float b1,
                                           int lane, int Cv) {
    float x0 = lg2_approx(a0), x1 = lg2_approx(a1);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y0 = __shfl_up_sync(0xffffffffu, x0, o);
        const float y1 = __shfl_up_sync(0xffffffffu, x1, o);
        if (lane >= o) { x0 += y0; x1 += y1; }
    }
    x1 += __shfl_sync(0xffffffffu, x0, 31);
    const float gC = __shfl_sync(0xffffffffu, x1, 31);
    // cumulative decay at the last row of each row's 16-row block
    const float e0 = __shfl_sync(0xffffffffu, x0, lane | 15);
    const float e1 = __shfl_sync(0xffffffffu, x1, lane | 15);
    par->g2[lane] = x0;
    par->g2[lane + 32] = x1;
    par->al[lane] = a0;
    par->al[lane + 32] = a1;
    par->dblk[lane] = ex2_approx(e0 - x0);
    par->dblk[lane + 32] = ex2_approx(e1 - x1);
    par->eg[lane] = ex2_approx(x0);
    par->eg[lane + 32] = ex2_approx(x1);
    par->egc[lane] = ex2_approx(gC - x0);
    par->egc[lane + 32] = ex2_approx(gC - x1);
    par->bet[lane] = b0;
    par->bet[lane + 32] = b1;
    if (lane == 0) {
        par->egC = ex2_approx(gC);
        par->Cv = Cv;
    }
}

// The gate factors the chain kernel reads: e^{g_r} (Q'), e^{g_C - g_r} (K') and
// e^{g_C} (the state decay), the same arithmetic as scan_gates.
struct ChainParams {
    float eg[C];
    float egc[C];
    float egC;
    float pad[3];
};

__device__ __forceinline__ void scan_gates_chain(ChainParams *par, float a0, float a1, int lane) {
    float x0 = lg2_approx(a0), x1 = lg2_approx(a1);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y0 = __shfl_up_sync(0xffffffffu, x0, o);
        const float y1 = __shfl_up_sync(0xffffffffu, x1, o);
        if (lane >= o) { x0 += y0; x1 += y1; }
    }
    x1 += __shfl_sync(0xffffffffu, x0, 31);
    const float gC = __shfl_sync(0xffffffffu, x1, 31);
    par->eg[lane] = ex2_approx(x0);
    par->eg[lane + 32] = ex2_approx(x1);
    par->egc[lane] = ex2_approx(gC - x0);
    par->egc[lane + 32] = ex2_approx(gC - x1);
    if (lane == 0) par->egC = ex2_approx(gC);
}

// Decay factors exp(g_r - g_i) of row r for the 32 columns [32 hf, 32 hf + 32),
// columns right of r zero.  No per-element exponential: 16-blocks left of r's
// block as 2^(g_r - g_blockend) * dblk[i], r's own block as a running product
// of alpha.  `tile` is warp-uniform: 0 below the diagonal tile, 1 on it.
__device__ __forceinline__ void decay_row(const ChunkParams *par, int r, int hf, bool on_diag,
                                          float (&gam)[32]) {
    const float gr = par->g2[r];
    if (!on_diag) {
        const float E0 = ex2_approx(gr - par->g2[32 * hf + 15]);
        const float E1 = ex2_approx(gr - par->g2[32 * hf + 31]);
#pragma unroll
        for (int j = 0; j < 32; ++j) gam[j] = (j < 16 ? E0 : E1) * par->dblk[32 * hf + j];
    } else {
        const int br = r >> 4;
#pragma unroll
        for (int bb = 0; bb < 2; ++bb) {
            const int blk = 2 * hf + bb;
            const float E = ex2_approx(gr - par->g2[16 * blk + 15]);
            float c = 1.f;
#pragma unroll
            for (int ii = 15; ii >= 0; --ii) {
                const int i = 16 * blk + ii;
                const float chain = (i <= r) ? c : 0.f;
                c = (i <= r) ? c * par->al[i] : c;
                gam[16 * bb + ii] = (blk < br) ? E * par->dblk[i] : ((blk == br) ? chain : 0.f);
            }
        }
    }
}

constexpr int LSTR = 68;   // fp32 row stride of the L and T work matrices

// T = (I + L)^-1 = (I - A)^-1 for strictly lower L (64 x 64 fp32, row stride
// LSTR) by 256 threads: 16 x 16 diagonal blocks by forward substitution, then
// T21 = -T22 L21 T11 merges 16 -> 32 -> 64.  Tb's entries above the diagonal
// blocks must be zero on entry.  Yb: 1024 floats.  Ends with a barrier.
// The first two levels of invert_exact: the 16 x 16 diagonal blocks and the
// 16 -> 32 merges (T00 and T11 of the two 32-blocks complete).  Yb: 512 floats.
// Ends with a barrier.
__device__ __forceinline__ void invert_exact_to32(const float *Lb, float *Tb, float *Yb, int kt, int bar_id) {
    if (kt < 64) {
        // one column per thread; each solved entry updates the rows below it at once
        const int c = kt, base = c & ~15, jc = c & 15;
        float acc[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) acc[r] = (r == jc) ? 1.f : 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float xi = acc[i];
#pragma unroll
            for (int r = i + 1; r < 16; ++r) acc[r] -= Lb[(base + r) * LSTR + base + i] * xi;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tb[(base + r) * LSTR + c] = acc[r];
    }
    named_bar(bar_id, 256);
    {
        // 16 -> 32 for both 32-blocks, two adjacent columns per thread
        const int pr = kt >> 7, rr = (kt >> 3) & 15, c0 = (kt & 7) * 2;
        const int b0 = 32 * pr, b1 = b0 + 16;
        float y0 = 0.f, y1 = 0.f;
        const float *Lr = Lb + (b1 + rr) * LSTR + b0;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float l = Lr[k];
            const float2 t = *reinterpret_cast<const float2 *>(Tb + (b0 + k) * LSTR + b0 + c0);
            y0 += l * t.x; y1 += l * t.y;
        }
        *reinterpret_cast<float2 *>(Yb + pr * 256 + rr * 16 + c0) = make_float2(y0, y1);
        named_bar(bar_id, 256);
        float z0 = 0.f, z1 = 0.f;
        const float *Tr = Tb + (b1 + rr) * LSTR + b1;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float t = Tr[k];
            const float2 yy = *reinterpret_cast<const float2 *>(Yb + pr * 256 + k * 16 + c0);
            z0 += t * yy.x; z1 += t * yy.y;
        }
        *reinterpret_cast<float2 *>(Tb + (b1 + rr) * LSTR + b0 + c0) = make_float2(-z0, -z1);
    }
    named_bar(bar_id, 256);
}

__device__ __forceinline__ void invert_exact(const float *Lb, float *Tb, float *Yb, int kt, int bar_id) {
    invert_exact_to32(Lb, Tb, Yb, kt, bar_id);
    {
        // 32 -> 64: Y = L10 T00, T10 = -T11 Y; thread (row, 4 columns), full unroll
        const int rr = kt >> 3, c0 = (kt & 7) * 4;
        float y[4] = {0.f, 0.f, 0.f, 0.f};
        const float *Lr = Lb + (32 + rr) * LSTR;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const float l = Lr[k];
            const float4 t = *reinterpret_cast<const float4 *>(Tb + k * LSTR + c0);
            y[0] += l * t.x; y[1] += l * t.y; y[2] += l * t.z; y[3] += l * t.w;
        }
        *reinterpret_cast<float4 *>(Yb + rr * 32 + c0) = make_float4(y[0], y[1], y[2], y[3]);
        named_bar(bar_id, 256);
        float z[4] = {0.f, 0.f, 0.f, 0.f};
        const float *Tr = Tb + (32 + rr) * LSTR + 32;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const float t = Tr[k];
            const float4 a = *reinterpret_cast<const float4 *>(Yb + k * 32 + c0);
            z[0] += t * a.x; z[1] += t * a.y; z[2] += t * a.z; z[3] += t * a.w;
        }
        *reinterpret_cast<float4 *>(Tb + (32 + rr) * LSTR + c0) = make_float4(-z[0], -z[1], -z[2], -z[3]);
    }
    named_bar(bar_id, 256);
}

// Masked truncated Neumann series M^(N) (.) sum_{n<=N} A^n with A = -L, by
// Horner's rule T <- M (.) (I + A T) on the band the mask leaves (N <= 15).
// Band rows are 16 wide in Yb (2 x 1024 floats): band[i*16 + d] = T_{i,i-d}.
// Writes the dense T (zeros outside the band) to Tb.  Ends with a barrier.
__device__ __forceinline__ void invert_neumann(const float *Lb, float *Tb, float *Yb, int kt, int N,
                                               int bar_id) {
    const int i = kt >> 2, dq = kt & 3;
    float *cur = Yb, *nxt = Yb + 1024;
#pragma unroll
    for (int u = 0; u < 4; ++u) cur[i * 16 + dq + 4 * u] = (dq + 4 * u == 0) ? 1.f : 0.f;
    named_bar(bar_id, 256);
    for (int step = 0; step < N; ++step) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int d = dq + 4 * u, j = i - d;
            float val = 0.f;
            if (j >= 0 && d <= N) {
                val = (d == 0) ? 1.f : 0.f;
                // k from j to i-1; T_kj lies in the band while k - j <= N
                for (int k = j; k < i; ++k) val -= Lb[i * LSTR + k] * cur[k * 16 + (k - j)];
            }
            nxt[i * 16 + d] = val;
        }
        named_bar(bar_id, 256);
        float *sw = cur; cur = nxt; nxt = sw;
    }
#pragma unroll 4
    for (int qq = 0; qq < 16; ++qq) {
        const int e = kt + 256 * qq, ii = e >> 6, j = e & 63, d = ii - j;
        Tb[ii * LSTR + j] = (d >= 0 && d <= N) ? cur[ii * 16 + d] : 0.f;
    }
    named_bar(bar_id, 256);
}

// ---------------------------------------------------- 128-thread inverses
// The fused kernel inverts with one group of four warps per chunk (two groups
// work on alternate chunks), so these take 128 threads.

// T = (I + L)^-1 = (I - A)^-1 for strictly lower L (64 x 64 fp32, row stride
// LSTR) by 128 threads t: the 16 x 16 diagonal blocks by forward substitution
// (one column per thread), then T21 = -T22 L21 T11 merges 16 -> 32 -> 64.
// Tb's entries above the diagonal blocks must be zero on entry (they are
// never written).  Yb: 1024 floats of scratch.  Ends with a barrier.
__device__ __forceinline__ void invert_exact128(const float *Lb, float *Tb, float *Yb, int t, int bar_id) {
    if (t < 64) {
        const int c = t, base = c & ~15, jc = c & 15;
        float acc[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) acc[r] = (r == jc) ? 1.f : 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float xi = acc[i];
#pragma unroll
            for (int r = i + 1; r < 16; ++r) acc[r] -= Lb[(base + r) * LSTR + base + i] * xi;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) Tb[(base + r) * LSTR + c] = acc[r];
    }
    named_bar(bar_id, 128);
    {
        // 16 -> 32 for both 32-blocks: Y = L21 T11, then T21 = -T22 Y; thread (row, 4 columns)
        const int pr = t >> 6, rr = (t >> 2) & 15, c0 = (t & 3) * 4;
        const int b0 = 32 * pr, b1 = b0 + 16;
        float y[4] = {0.f, 0.f, 0.f, 0.f};
        const float *Lr = Lb + (b1 + rr) * LSTR + b0;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float l = Lr[k];
            const float4 v = *reinterpret_cast<const float4 *>(Tb + (b0 + k) * LSTR + b0 + c0);
            y[0] += l * v.x; y[1] += l * v.y; y[2] += l * v.z; y[3] += l * v.w;
        }
        *reinterpret_cast<float4 *>(Yb + pr * 256 + rr * 16 + c0) = make_float4(y[0], y[1], y[2], y[3]);
        named_bar(bar_id, 128);
        float z[4] = {0.f, 0.f, 0.f, 0.f};
        const float *Tr = Tb + (b1 + rr) * LSTR + b1;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float a = Tr[k];
            const float4 v = *reinterpret_cast<const float4 *>(Yb + pr * 256 + k * 16 + c0);
            z[0] += a * v.x; z[1] += a * v.y; z[2] += a * v.z; z[3] += a * v.w;
        }
        *reinterpret_cast<float4 *>(Tb + (b1 + rr) * LSTR + b0 + c0) = make_float4(-z[0], -z[1], -z[2], -z[3]);
    }
    named_bar(bar_id, 128);
    {
        // 32 -> 64: Y = L10 T00, T10 = -T11 Y; thread (two rows, 4 columns)
        const int rr = 2 * (t >> 3), c0 = (t & 7) * 4;
        float y0[4] = {0.f, 0.f, 0.f, 0.f}, y1[4] = {0.f, 0.f, 0.f, 0.f};
        const float *L0 = Lb + (32 + rr) * LSTR, *L1 = L0 + LSTR;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const float4 v = *reinterpret_cast<const float4 *>(Tb + k * LSTR + c0);
            const float l0 = L0[k], l1 = L1[k];
            y0[0] += l0 * v.x; y0[1] += l0 * v.y; y0[2] += l0 * v.z; y0[3] += l0 * v.w;
            y1[0] += l1 * v.x; y1[1] += l1 * v.y; y1[2] += l1 * v.z; y1[3] += l1 * v.w;
        }
        *reinterpret_cast<float4 *>(Yb + rr * 32 + c0) = make_float4(y0[0], y0[1], y0[2], y0[3]);
        *reinterpret_cast<float4 *>(Yb + (rr + 1) * 32 + c0) = make_float4(y1[0], y1[1], y1[2], y1[3]);
        named_bar(bar_id, 128);
        float z0[4] = {0.f, 0.f, 0.f, 0.f}, z1[4] = {0.f, 0.f, 0.f, 0.f};
        const float *T0 = Tb + (32 + rr) * LSTR + 32, *T1 = T0 + LSTR;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const float4 v = *reinterpret_cast<const float4 *>(Yb + k * 32 + c0);
            const float a0 = T0[k], a1 = T1[k];
            z0[0] += a0 * v.x; z0[1] += a0 * v.y; z0[2] += a0 * v.z; z0[3] += a0 * v.w;
            z1[0] += a1 * v.x; z1[1] += a1 * v.y; z1[2] += a1 * v.z; z1[3] += a1 * v.w;
        }
        *reinterpret_cast<float4 *>(Tb + (32 + rr) * LSTR + c0) = make_float4(-z0[0], -z0[1], -z0[2], -z0[3]);
        *reinterpret_cast<float4 *>(Tb + (33 + rr) * LSTR + c0) = make_float4(-z1[0], -z1[1], -z1[2], -z1[3]);
    }
    named_bar(bar_id, 128);
}

// Masked truncated Neumann series M^(N) (.) sum_{n<=N} A^n with A = -L by 128
// threads, Horner's rule T <- M (.) (I + A T).  N <= 15: on the band the mask
// leaves, rows 16 wide in Yb (2 x 1024 floats).  N > 15: dense 64 x 64
// steps with Yb (4096 floats, row stride 64) as the second buffer.  Writes
// the dense T (zeros outside the band) to Tb (row stride LSTR).  Ends with a
// barrier.
__device__ __forceinline__ void invert_neumann128(const float *Lb, float *Tb, float *Yb, int t, int N,
                                                  int bar_id) {
    if (N <= 15) {
        const int i = t >> 1, dq = t & 1;
        float *cur = Yb, *nxt = Yb + 1024;
#pragma unroll
        for (int u = 0; u < 8; ++u) cur[i * 16 + dq + 2 * u] = (dq + 2 * u == 0) ? 1.f : 0.f;
        named_bar(bar_id, 128);
        for (int step = 0; step < N; ++step) {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int d = dq + 2 * u, j = i - d;
                float val = 0.f;
                if (j >= 0 && d <= N) {
                    val = (d == 0) ? 1.f : 0.f;
                    for (int k = j; k < i; ++k) val -= Lb[i * LSTR + k] * cur[k * 16 + (k - j)];
                }
                nxt[i * 16 + d] = val;
            }
            named_bar(bar_id, 128);
            float *sw = cur; cur = nxt; nxt = sw;
        }
#pragma unroll 4
        for (int qq = 0; qq < 32; ++qq) {
            const int e = t + 128 * qq, ii = e >> 6, j = e & 63, d = ii - j;
            Tb[ii * LSTR + j] = (d >= 0 && d <= N) ? cur[ii * 16 + d] : 0.f;
        }
        named_bar(bar_id, 128);
        return;
    }
    // dense: thread t owns row i = t >> 1, columns [32 (t & 1), + 32)
    const int i = t >> 1, j0 = 32 * (t & 1);
    for (int jj = 0; jj < 32; ++jj) Tb[i * LSTR + j0 + jj] = (i == j0 + jj) ? 1.f : 0.f;
    named_bar(bar_id, 128);
    for (int step = 0; step < N; ++step) {
        // Yb <- M (.) (I - L Tb), then copy back into Tb
        for (int jj = 0; jj < 32; ++jj) {
            const int j = j0 + jj, d = i - j;
            float val = 0.f;
            if (d >= 0 && d <= N) {
                val = (d == 0) ? 1.f : 0.f;
                for (int k = j; k < i; ++k) val -= Lb[i * LSTR + k] * Tb[k * LSTR + j];
            }
            Yb[i * 64 + j] = val;
        }
        named_bar(bar_id, 128);
        for (int jj = 0; jj < 32; ++jj) Tb[i * LSTR + j0 + jj] = Yb[i * 64 + j0 + jj];
        named_bar(bar_id, 128);
    }
}

// Z = A + sgn * (X Y) for lower-triangular 64 x 64 fp32 matrices (row stride
// LSTR, zeros above the diagonal stored).  A is the identity (a_kind 1),
// I - Y (a_kind 2) or zero (a_kind 0).  256 threads, one 4 x 4 tile each;
// tiles above the diagonal are written as zeros.  Z must not alias X or Y.
// Ends with a barrier.
__device__ __forceinline__ void tri_mm(const float *X, const float *Y, float *Z, int kt, int a_kind, float sgn,
                                       int bar_id) {
    const int ib = kt >> 4, jb = kt & 15, i0 = 4 * ib, j0 = 4 * jb;
    float acc[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
    if (jb <= ib) {
        // X_ik = 0 for k > i and Y_kj = 0 for k < j: k runs over [j0, i0 + 3]
        for (int k = j0; k <= i0 + 3; ++k) {
            const float4 y = *reinterpret_cast<const float4 *>(Y + k * LSTR + j0);
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float x = X[(i0 + r) * LSTR + k];
                acc[r][0] += x * y.x; acc[r][1] += x * y.y; acc[r][2] += x * y.z; acc[r][3] += x * y.w;
            }
        }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        float z[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int i = i0 + r, j = j0 + c;
            float a = 0.f;
            if (a_kind == 1) a = (i == j) ? 1.f : 0.f;
            else if (a_kind == 2) a = ((i == j) ? 1.f : 0.f) - Y[i * LSTR + j];
            z[c] = a + sgn * acc[r][c];
        }
        *reinterpret_cast<float4 *>(Z + (i0 + r) * LSTR + j0) = make_float4(z[0], z[1], z[2], z[3]);
    }
    named_bar(bar_id, 256);
}

// Parallel residual correction of a truncated series T0 (in Tb) of
// T = (I + L)^-1: E = I - (I + L) T0 = (I - T0) - L T0, T ~= T0 sum_{s=0}^{S} E^s
// by Horner's rule, R <- I + E R.  Eb, R0, R1: three 64 x LSTR scratch
// matrices.  Returns the buffer that holds the corrected T.  Ends with a barrier.
__device__ __forceinline__ const float *residual_correct(const float *Lb, const float *Tb, float *Eb, float *R0,
                                                         float *R1, int kt, int S, int bar_id) {
    tri_mm(Lb, Tb, Eb, kt, 2, -1.f, bar_id);                 // E = (I - T0) - L T0
    // R = I
    for (int e = kt; e < 64 * 64; e += 256) R0[(e >> 6) * LSTR + (e & 63)] = ((e >> 6) == (e & 63)) ? 1.f : 0.f;
    named_bar(bar_id, 256);
    float *cur = R0, *nxt = R1;
    for (int s = 0; s < S; ++s) {
        tri_mm(Eb, cur, nxt, kt, 1, 1.f, bar_id);             // R <- I + E R
        float *t = cur; cur = nxt; nxt = t;
    }
    tri_mm(Tb, cur, Eb, kt, 0, 1.f, bar_id);                 // T = T0 R (E no longer needed)
    return Eb;
}

}  // namespace tc
}  // namespace gdn
