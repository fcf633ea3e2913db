// Tensor-core path of the chunkwise gated delta rule on sm_100a: two kernels.
//
// 1. keyside_kernel -- the state-independent part of every chunk, one CTA per
//    (chunk, head, batch), all chunks in parallel.  TMA loads Q and K; one
//    tcgen05 MMA forms [Q ; K] K^T (bf16, exact products, fp32 in TMEM).  From
//    TMEM: the decayed causal scores P_ri = (q_r.k_i) exp(g_r - g_i), i <= r,
//    and L_ri = beta_r exp(g_r - g_i) (k_r.k_i), i < r (A = -L).  T = (I - A)^-1
//    exactly (16 x 16 diagonal blocks by forward substitution, merged
//    16 -> 32 -> 64 by T21 = -T22 L21 T11, the last merge on the tensor cores),
//    or the masked truncated Neumann series M^(N) (.) sum_{n<=N} A^n by Horner's
//    rule as N - 1 masked MMAs, or (with the residual correction T0 sum_{s<=S}
//    E^s) its band form on the CUDA cores.  Written to the workspace
//    as fp16: T diag(beta), T diag(beta e^g) and P, 24 KB per chunk-head.
// 2. chain_kernel -- one CTA per (batch, head, 64-column value slice) walks
//    the chunks in order with the fp32 state h = S^T (128 x 64) in TMEM.
//      warp 0      TMA producer: q, k and P into a ring of three stages; the
//                  v slice, T diag(beta), T diag(beta e^g) into one early slot
//      warp 1      TMEM allocation, then the output MMAs O += P Delta
//      warps 2-9   key side of chunk m (runs ahead of the chain): gate scan,
//                  fp16 operands Q' = diag(e^g) Q, K, V; U = T diag(beta) V and
//                  W = T diag(beta e^g) K (MMAs); -W to shared memory; K
//                  rescaled in place by e^{g_C - g} for the state update
//      warps 10-13 state chain:
//                  h16 <- h;  h <- e^{g_C} h               (TMEM)
//                  [-W h ; Q' h] = [-W ; Q'] h16            (MMA)
//                  Delta = U - W h                          (CUDA cores)
//                  h += (e^{g_C - g} K)^T Delta                (MMA)
//                  O = Q'h + P Delta is finished by warp 1 off the chain
//    Every MMA is tcgen05.mma kind::f16, M = 128: a 64-row operand is paired
//    with the 64 rows that follow it in the same stage; the TMEM lanes those
//    rows produce are never read.  Derived operands are fp16: with bf16 ones
//    this workload's outputs leave the 2e-2-of-RMS accuracy bar.
//
// The recurrence is S_t = S_{t-1} alpha_t (I - beta_t k_t k_t^T) +
// beta_t v_t k_t^T, o_t = S_t q_t; the chunk system (I - A) Delta =
// diag(beta)(V - diag(e^g) K h) with T = (I - A)^-1 is the step "Quando o 'Bom
// o Suficiente' e Otimo: Aproximacao de Inversao de Matriz Baseada Apenas em
// Multiplicacao para Gated DeltaNet Quantizado" (section "Declaracao do
// Problema") singles out; its Neumann, mask and residual items are
// "Metodologia" 1-3.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "gdn_internal.cuh"
#include "gdn_tc_common.cuh"

namespace gdn {

__device__ unsigned int g_tc_error = 0;

namespace {

using namespace sm100;
using tc::C;
using tc::ChunkParams;
using tc::DK;
using tc::LSTR;
using tc::pack_h2;
using tc::st_row_f16;
using tc::tmem_ld64;
using tc::unpack_bf2;
using tc::unpack_h2;

constexpr int DVS = 64;            // value columns per chain CTA
constexpr int kSMs = 148;          // B200
constexpr int kSegAutoMinChunks = 256;   // sequence segments by default from 16384 tokens
constexpr int kNeumannMaxN = 15;
constexpr unsigned long long kWaitLimit = 4000000000ull;   // ~2 s at the boost clock

// error codes recorded in g_tc_error (first one wins)
enum { E_FULL = 1, E_EMPTY, E_KSREADY, E_KSFREE, E_O, E_UW, E_X, E_H, E_K1_TMA, E_K1_MMA, E_XISS, E_DREADY };

constexpr uint32_t IDESC_BF_KK = idesc_f16(128, 64, 1, 1, 0, 0);    // bf16, K-major x K-major, N 64
constexpr uint32_t IDESC_KM64 = idesc_f16(128, 64, 0, 0, 0, 1);     // fp16, K-major x MN-major, N 64
constexpr uint32_t IDESC_KM128 = idesc_f16(128, 128, 0, 0, 0, 1);   // fp16, K-major x MN-major, N 128
constexpr uint32_t IDESC_MM64 = idesc_f16(128, 64, 0, 0, 1, 1);     // fp16, MN-major x MN-major, N 64

// =========================================================== key-side kernel

// Workspace per chunk-head: three 64 x 64 fp16 row-major matrices,
// T diag(beta), T diag(beta e^g) and the decayed causal scores P.
constexpr int WS_ROWS = 192;                           // rows of 128 bytes per chunk-head
constexpr size_t WS_CHUNK_BYTES = (size_t)WS_ROWS * 128;

constexpr int K1_THREADS = 256;
constexpr int K1_BLOCKS_PER_SM = 3;
constexpr uint32_t K1_MAT = 64 * LSTR * 4;
constexpr uint32_t K1_OFF_QK = 0;                      // per key block kb: [Q | K] at kb * 16 KB
constexpr uint32_t K1_OFF_LB = 0;                      // L fp32 and the inverse scratch reuse the
constexpr uint32_t K1_OFF_YB = K1_MAT;                 // tiles once the Gram MMA has read them
constexpr uint32_t K1_OFF_TB = 32768;
constexpr uint32_t K1_OFF_PAR = K1_OFF_TB + K1_MAT;
constexpr uint32_t K1_OFF_BAR = K1_OFF_PAR + ((sizeof(ChunkParams) + 15) & ~15u);
// fp16 staging of the 32 -> 64 inverse merge (exact mode): B2 over the 16 -> 32
// merge's scratch, A1 in the rest of the tile region (L occupies its start), A2
// and B1 in a region of their own; a 64-row A operand drags 96 more rows along
constexpr uint32_t K1_OFF_STG = (K1_OFF_BAR + 64 + 1023) & ~1023u;
constexpr uint32_t K1_OFF_B2 = K1_OFF_YB, K1_OFF_A1 = 22528, K1_OFF_A2 = K1_OFF_STG, K1_OFF_B1 = K1_OFF_STG + 4096;
constexpr uint32_t K1_SMEM = K1_OFF_STG + 16384 + 1024;  // + base alignment slack
// residual correction: three more 64 x LSTR fp32 matrices (E, R ping-pong)
constexpr uint32_t K1_OFF_RES = K1_OFF_BAR + 64;
constexpr uint32_t K1_SMEM_RES = K1_OFF_RES + 3 * K1_MAT + 1024;

struct K1Params {
    int B, T, H, NC;
    const float *alpha, *beta;
    uint8_t *ws;
    int neumann, N;     // neumann: 1 truncated series, 2 series + residual correction
    int S;              // residual-correction terms
};

// Chunk 128 of the masked series as two 64-token halves a, b.  The second half's
// Delta differs from that of a 64-token chunk only through the band's corner T_ba
// (rows 0..N-1 of b, columns 64-N..63 of a) and through the state at the start of
// the 128-token chunk: Delta_b = U_b - (W_b + C2') e^{g_aC} h_a + C1 V_a, with
// C1 = T_ba diag(beta_a) (N x N over a's last N rows) and
// C2' = T_ba diag(beta_a e^{g_a - g_aC}) K_a (N x DK).  Per second half and head,
// fp32: C2' (16 x DK), then C1 V_a as one 16 x 64 block per 64-column value slice;
// rows N..15 zero.
constexpr int PAIR_MAXN = 16;
constexpr size_t pair_stride(int dv) { return (size_t)PAIR_MAXN * (DK + dv); }

struct PairParams {
    int B, T, H, dv, NC, N;
    const void *k, *v;          // bf16 [B, T, H, DK], [B, T, H, dv]
    const float *alpha, *beta;  // [B, T, H] (nullptr: 1)
    float *pair_ws;
};

constexpr int PAIR_THREADS = 128;

// One CTA per (second half, head, batch): the band corner of a 128-token chunk.  The
// entries of the masked series within the band equal those of the exact inverse
// (A is strictly lower triangular, so A^n vanishes more than n - 1 below the
// diagonal), and an entry (r, c) depends only on the tokens between c and r: T_ba
// is the exact inverse of the 2N-token window around the halves' boundary, read
// in the band.  Window row w < N is the first half's row 64 - N + w, row N + i
// the second half's row i.  Small and latency-bound: many CTAs per SM, the band N
// a template argument so that every loop has its exact trip count.
template <int N>
__global__ void __launch_bounds__(PAIR_THREADS)
pair_corner_kernel(const PairParams p) {
    constexpr int NW = 2 * N, NWP = NW > 0 ? NW : 1, NP = N > 0 ? N : 1;
    __shared__ float kw[NWP][DK + 1];            // window keys, fp32
    __shared__ float aw[NWP][NWP + 1];           // A of the window (band)
    __shared__ float gw[NWP], bw[NWP], ew[NP];
    __shared__ float cw[NP][NP];                 // C1 = T_ba diag(beta_a)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = 2 * blockIdx.x + 1, h = blockIdx.y, b = blockIdx.z;
    const int t0 = n * C - N;                    // window start token
    const int rs = p.H * DK;
    const uint16_t *kg = reinterpret_cast<const uint16_t *>(p.k) + (((size_t)b * p.T + t0) * p.H + h) * DK;
    const uint16_t *vg = reinterpret_cast<const uint16_t *>(p.v) + (((size_t)b * p.T + t0) * p.H + h) * p.dv;
    float *dst = p.pair_ws + (((size_t)b * p.H + h) * p.NC + n) * pair_stride(p.dv);

    // every global load of the window first, so that their latencies overlap:
    // keys as 16-byte pieces (16 per row), the first value column of this thread,
    // the gates (warp 0)
    constexpr int KQ = (NW * 16 + PAIR_THREADS - 1) / PAIR_THREADS;
    uint4 kr[KQ > 0 ? KQ : 1];
#pragma unroll
    for (int q = 0; q < KQ; ++q) {
        const int x = tid + PAIR_THREADS * q, w = x >> 4;
        kr[q] = make_uint4(0u, 0u, 0u, 0u);
        if (w < NW && t0 + w < p.T) kr[q] = *reinterpret_cast<const uint4 *>(kg + (size_t)w * rs + 8 * (x & 15));
    }
    float vj[NP];
#pragma unroll
    for (int j = 0; j < N; ++j)
        vj[j] = tid < p.dv ? __uint_as_float((uint32_t)vg[(size_t)j * p.H * p.dv + tid] << 16) : 0.f;
    float la = 0.f, be = 0.f;
    if (warp == 0 && lane < NW && t0 + lane < p.T) {
        const size_t ti = ((size_t)b * p.T + t0 + lane) * p.H + h;
        la = p.alpha ? logf(p.alpha[ti]) : 0.f;
        be = p.beta ? p.beta[ti] : 1.f;
    }
#pragma unroll
    for (int q = 0; q < KQ; ++q) {
        const int x = tid + PAIR_THREADS * q, w = x >> 4;
        if (w < NW) {
            float *d = &kw[w][8 * (x & 15)];
            const uint32_t u[4] = {kr[q].x, kr[q].y, kr[q].z, kr[q].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                d[2 * e] = __uint_as_float(u[e] << 16);
                d[2 * e + 1] = __uint_as_float(u[e] & 0xffff0000u);
            }
        }
    }
    if (warp == 0) {
        // cumulative log decay over the window (only differences are used)
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, la, o);
            if (lane >= o) la += y;
        }
        if (lane < NW) { gw[lane] = la; bw[lane] = be; }
    }
    __syncthreads();
    // A_ij = -beta_i e^{g_i - g_j} k_i.k_j for 0 < i - j <= N: four lanes per entry,
    // 32 channels each (rotated by 8 per lane so that the four do not share banks)
    constexpr int TOTAL = NW * NW * 4;
    for (int q0 = warp * 32; q0 < TOTAL; q0 += PAIR_THREADS) {
        const int q = q0 + lane, e = q >> 2, part = q & 3;
        const int i = e / NWP, j = e - i * NWP;
        const bool need = q < TOTAL && j < i && i - j <= N;
        float d = 0.f;
        if (need) {
#pragma unroll 8
            for (int cc = 0; cc < 32; ++cc) {
                const int c = 32 * part + ((cc + 8 * part) & 31);
                d += kw[i][c] * kw[j][c];
            }
        }
        d += __shfl_xor_sync(0xffffffffu, d, 1);
        d += __shfl_xor_sync(0xffffffffu, d, 2);
        if (need && part == 0) aw[i][j] = -bw[i] * expf(gw[i] - gw[j]) * d;
    }
    __syncthreads();
    if (tid < N) {
        // column j = tid of the window's inverse by forward substitution, rows j..N+j
        // (every A entry it reads lies in the band); C1 = T_ba diag(beta_a) in the
        // band (i <= j), zero below it
        const int j = tid;
        float t[NWP];
#pragma unroll
        for (int k = 0; k < NW; ++k) {
            float acc = (k == j) ? 1.f : 0.f;
            if (k > j && k <= N + j) {
#pragma unroll
                for (int m = 0; m < k; ++m)
                    if (m >= j) acc += aw[k][m] * t[m];
            }
            t[k] = acc;
        }
#pragma unroll
        for (int i = 0; i < N; ++i) cw[i][j] = i <= j ? t[N + i] * bw[j] : 0.f;
        ew[j] = expf(gw[j] - gw[N - 1]);
    }
    __syncthreads();
    {
        // C2'[i][c] = sum_j C1[i][j] e^{g_j - g_{N-1}} k_j[c], column c = tid; rows >= N zero
        const int c = tid;
        float kc[NP];
#pragma unroll
        for (int j = 0; j < N; ++j) kc[j] = ew[j] * kw[j][c];
#pragma unroll 4
        for (int i = 0; i < PAIR_MAXN; ++i) {
            float acc = 0.f;
            if (i < N) {
#pragma unroll
                for (int j = 0; j < N; ++j) acc += cw[i < N ? i : 0][j] * kc[j];
            }
            dst[i * DK + c] = acc;
        }
    }
    // C1 V_a, column c of the value rows t0 .. t0 + N - 1, one 16 x 64 block per
    // 64-column value slice
    for (int c = tid; c < p.dv; c += PAIR_THREADS) {
        if (c != tid) {
#pragma unroll
            for (int j = 0; j < N; ++j) vj[j] = __uint_as_float((uint32_t)vg[(size_t)j * p.H * p.dv + c] << 16);
        }
        float *dc = dst + PAIR_MAXN * DK + (c >> 6) * (PAIR_MAXN * 64) + (c & 63);
#pragma unroll 4
        for (int i = 0; i < PAIR_MAXN; ++i) {
            float acc = 0.f;
            if (i < N) {
#pragma unroll
                for (int j = 0; j < N; ++j) acc += cw[i < N ? i : 0][j] * vj[j];
            }
            dc[i * 64] = acc;
        }
    }
}

// One CTA per (chunk, head, batch).  [Q ; K] K^T in one MMA: TMEM lanes 0..63
// hold Q K^T (-> P), lanes 64..127 hold K K^T (-> L -> T).
__global__ void __launch_bounds__(K1_THREADS, K1_BLOCKS_PER_SM)
keyside_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const K1Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    float *Lb = reinterpret_cast<float *>(sm + K1_OFF_LB);
    float *Tb = reinterpret_cast<float *>(sm + K1_OFF_TB);
    float *Yb = reinterpret_cast<float *>(sm + K1_OFF_YB);
    ChunkParams *par = reinterpret_cast<ChunkParams *>(sm + K1_OFF_PAR);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + K1_OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + K1_OFF_BAR + 24);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + K1_OFF_BAR + 28);
    volatile int *okflag = reinterpret_cast<volatile int *>(sm + K1_OFF_BAR + 32);
    uint8_t *ws = p.ws + ((((size_t)b * p.H + h) * p.NC + n) * WS_CHUNK_BYTES);

    const int t0 = n * C;
    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_init(&bars[2], 1);
        *abort_flag = 0;
        fence_mbar_init();
        // the tiles first: their latency overlaps the set-up below
        mbar_arrive_expect_tx(&bars[0], 32768);
        tma_load_4d(sm + K1_OFF_QK, &tm_q, &bars[0], 0, h, t0, b);
        tma_load_4d(sm + K1_OFF_QK + 8192, &tm_k, &bars[0], 0, h, t0, b);
        tma_load_4d(sm + K1_OFF_QK + 16384, &tm_q, &bars[0], 64, h, t0, b);
        tma_load_4d(sm + K1_OFF_QK + 24576, &tm_k, &bars[0], 64, h, t0, b);
    }
    __syncwarp();
    // set-up in parallel: warp 0 has issued the tile loads, warp 1 fetches and scans
    // the gates (their global loads are the longest wait before the Gram), warp 2
    // allocates TMEM, everyone clears the two upper 16 x 16 blocks of the inverse's
    // 32-blocks (the 32 -> 64 merge reads them as zeros; the rest of T above the
    // diagonal is never read as anything but zero: the final writes mask it)
    if (warp == 1) {
        float a0, a1, b0, b1;
        tc::fetch_gates(p.alpha, p.beta, b, p.T, p.H, h, t0, lane, true, a0, a1, b0, b1);
        tc::scan_gates(par, a0, a1, b0, b1, lane, min(C, p.T - t0));
    }
    if (warp == 2) {
        tmem_alloc(tmem_slot, 128);      // Gram (64 columns), inverse merge (64)
        tmem_relinquish();
    }
    if (!p.neumann) {
        const int blk = tid >> 7, u = tid & 127;
        *reinterpret_cast<float2 *>(Tb + (32 * blk + (u >> 3)) * LSTR + 32 * blk + 16 + 2 * (u & 7)) =
            make_float2(0.f, 0.f);
    }
    tc_fence_before();
    block_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (tid == 0) {
        if (mbar_wait(&bars[0], 0, abort_flag, E_K1_TMA, kWaitLimit)) {
            tc_fence_after();
            const uint32_t a0 = smem_u32(sm + K1_OFF_QK);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                umma_f16_ss(tmem, sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(a0 + off + 8192, 16, 1024),
                            IDESC_BF_KK, kk > 0);
            }
            umma_commit(&bars[1]);
            if (!mbar_wait(&bars[1], 0, abort_flag, E_K1_MMA, kWaitLimit))
                mbar_wait_drain(&bars[1], 0, kWaitLimit);
        } else {
            mbar_wait_drain(&bars[0], 0, kWaitLimit);
        }
    }
    __syncwarp();
    block_sync();
    const bool go = (*abort_flag == 0);
    if (go) {
        mbar_try_wait(&bars[1], 0);
        tc_fence_after();
        // sub-partition sp holds rows 32 sp .. 32 sp + 31 of [Q K^T ; K K^T];
        // warp half hf takes columns [32 hf, 32 hf + 32).
        const int sp = warp & 3, hf = warp >> 2;
        const int r = 32 * (sp & 1) + lane;               // chunk row
        const bool diag = (hf == (sp & 1));
        uint32_t xr[32];
        float gam[32];
        if (hf <= (sp & 1)) {
            tmem_ld32(tmem + ((uint32_t)(32 * sp) << 16) + 32 * hf, xr);
            tc::decay_row(par, r, hf, diag, gam);
            tmem_wait_ld();
        }
        if (sp < 2) {
            // P_ri = (q_r . k_i) exp(g_r - g_i), i <= r: straight to the workspace
            uint4 *dst = reinterpret_cast<uint4 *>(ws + (size_t)(128 + r) * 128 + 64 * hf);
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                uint4 u = make_uint4(0u, 0u, 0u, 0u);
                if (hf <= sp) {
                    const int j = 8 * jj;
                    u.x = pack_h2(gam[j] * __uint_as_float(xr[j]), gam[j + 1] * __uint_as_float(xr[j + 1]));
                    u.y = pack_h2(gam[j + 2] * __uint_as_float(xr[j + 2]), gam[j + 3] * __uint_as_float(xr[j + 3]));
                    u.z = pack_h2(gam[j + 4] * __uint_as_float(xr[j + 4]), gam[j + 5] * __uint_as_float(xr[j + 5]));
                    u.w = pack_h2(gam[j + 6] * __uint_as_float(xr[j + 6]), gam[j + 7] * __uint_as_float(xr[j + 7]));
                }
                dst[jj] = u;
            }
        } else {
            // L_ri = beta_r exp(g_r - g_i) (k_r . k_i), i < r
            float *Lr = Lb + r * LSTR + 32 * hf;
            if (hf > (sp & 1)) {
#pragma unroll
                for (int j = 0; j < 32; j += 4) *reinterpret_cast<float4 *>(Lr + j) = make_float4(0.f, 0.f, 0.f, 0.f);
            } else {
                const float br = par->bet[r];
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const int i = 32 * hf + j;
                    float4 v;
                    v.x = (i + 0 < r) ? br * gam[j + 0] * __uint_as_float(xr[j + 0]) : 0.f;
                    v.y = (i + 1 < r) ? br * gam[j + 1] * __uint_as_float(xr[j + 1]) : 0.f;
                    v.z = (i + 2 < r) ? br * gam[j + 2] * __uint_as_float(xr[j + 2]) : 0.f;
                    v.w = (i + 3 < r) ? br * gam[j + 3] * __uint_as_float(xr[j + 3]) : 0.f;
                    *reinterpret_cast<float4 *>(Lr + j) = v;
                }
            }
        }
        tc_fence_before();
        named_bar(1, K1_THREADS);
        bool inv_ok = true;
        if (p.neumann == 1) {
            // The masked truncated Neumann series by Horner's rule, T <- M (.) (I + A T),
            // with the products on the tensor cores: T1 = M (.) (I + A) from L, then
            // N - 1 steps of one MMA (A and T fp16, fp32 accumulate) and the mask.
            // A = -L sits in the staging region (its 64 padding rows stay inside the
            // block), T in the inverse scratch.
            uint8_t *aS = sm + K1_OFF_STG, *bS = sm + K1_OFF_YB;
            const uint32_t tI = tmem + 64;
            const int N = p.N;
            {
                const int r = tid >> 2, j0 = (tid & 3) * 2;     // row r, 16-byte chunks j0, j0 + 1
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int j = j0 + q;
                    float a[8], t[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int c = 8 * j + e, d = r - c;
                        const float l = Lb[r * LSTR + c];
                        a[e] = -l;
                        t[e] = d == 0 ? 1.f : (d > 0 && d <= N ? -l : 0.f);
                    }
                    *reinterpret_cast<uint4 *>(aS + sw128_off(r, j)) =
                        make_uint4(pack_h2(a[0], a[1]), pack_h2(a[2], a[3]), pack_h2(a[4], a[5]), pack_h2(a[6], a[7]));
                    *reinterpret_cast<uint4 *>(bS + sw128_off(r, j)) =
                        make_uint4(pack_h2(t[0], t[1]), pack_h2(t[2], t[3]), pack_h2(t[4], t[5]), pack_h2(t[6], t[7]));
                    if (N <= 1) {
                        *reinterpret_cast<float4 *>(Tb + r * LSTR + 8 * j) = make_float4(t[0], t[1], t[2], t[3]);
                        *reinterpret_cast<float4 *>(Tb + r * LSTR + 8 * j + 4) = make_float4(t[4], t[5], t[6], t[7]);
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(1, K1_THREADS);
#pragma unroll 1
            for (int step = 1; step < N; ++step) {
                if (tid == 0) {
                    // D = [A ; any 64 rows] T (TMEM lanes 0..63 real), K = 64 in four MMAs
                    tc_fence_after();
                    const uint32_t aa = smem_u32(aS), bb = smem_u32(bS);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ss(tI, sdesc_sw128(aa + kk * 32, 16, 1024), sdesc_sw128(bb + kk * 2048, 16384, 1024),
                                    IDESC_KM64, kk > 0);
                    umma_commit(&bars[2]);
                    const bool w = mbar_wait(&bars[2], (step - 1) & 1, abort_flag, E_K1_MMA, kWaitLimit);
                    if (!w) mbar_wait_drain(&bars[2], (step - 1) & 1, kWaitLimit);
                    *okflag = w ? 1 : 0;
                }
                __syncwarp();
                named_bar(1, K1_THREADS);
                if (!*okflag) { inv_ok = false; break; }
                mbar_try_wait(&bars[2], (step - 1) & 1);
                tc_fence_after();
                if ((warp & 3) < 2) {
                    // warps 0, 1, 4, 5: rows 32 sp + lane, columns [32 hf, 32 hf + 32)
                    const int sp = warp & 3, hf = warp >> 2, r = 32 * sp + lane;
                    const bool last = (step == N - 1);
                    uint32_t x[32];
                    tmem_ld32(tI + ((uint32_t)(32 * sp) << 16) + 32 * hf, x);
                    tmem_wait_ld();
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        float t[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int c = 32 * hf + 8 * jj + e, d = r - c;
                            t[e] = d == 0 ? 1.f : (d > 0 && d <= N ? __uint_as_float(x[8 * jj + e]) : 0.f);
                        }
                        if (last) {
                            float *dst = Tb + r * LSTR + 32 * hf + 8 * jj;
                            *reinterpret_cast<float4 *>(dst) = make_float4(t[0], t[1], t[2], t[3]);
                            *reinterpret_cast<float4 *>(dst + 4) = make_float4(t[4], t[5], t[6], t[7]);
                        } else {
                            *reinterpret_cast<uint4 *>(bS + sw128_off(r, 4 * hf + jj)) =
                                make_uint4(pack_h2(t[0], t[1]), pack_h2(t[2], t[3]), pack_h2(t[4], t[5]),
                                           pack_h2(t[6], t[7]));
                        }
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar(1, K1_THREADS);
            }
        } else if (p.neumann) {
            // the residual-corrected series keeps the band form on the CUDA cores
            tc::invert_neumann(Lb, Tb, Yb, tid, p.N, 1);
        } else {
            // T = (I + L)^-1: the 16 x 16 diagonal blocks and the 16 -> 32 merges on
            // the CUDA cores, the 32 -> 64 merge T10 = -T11 L10 T00 as two MMAs (fp16
            // operands, fp32 accumulate).  Staging tiles in the free part of the q/k
            // tile region and the scratch of the 16 -> 32 merge; the 96 rows each
            // 64-row A operand drags along lie in tiles that stay unchanged while it runs.
            tc::invert_exact_to32(Lb, Tb, Yb, tid, 1);
            uint8_t *a1 = sm + K1_OFF_A1, *b1 = sm + K1_OFF_B1, *a2 = sm + K1_OFF_A2, *b2 = sm + K1_OFF_B2;
            const uint32_t tI = tmem + 64;
            {
                const int u = tid & 127, rw = u >> 2, j = u & 3;
                const float *src = tid < 128 ? Lb + (32 + rw) * LSTR + 8 * j : Tb + (32 + rw) * LSTR + 32 + 8 * j;
                const float sg = tid < 128 ? 1.f : -1.f;
                const float4 x0 = *reinterpret_cast<const float4 *>(src);
                const float4 x1 = *reinterpret_cast<const float4 *>(src + 4);
                *reinterpret_cast<uint4 *>((tid < 128 ? a1 : a2) + sw128_off(rw, j)) =
                    make_uint4(pack_h2(sg * x0.x, sg * x0.y), pack_h2(sg * x0.z, sg * x0.w),
                               pack_h2(sg * x1.x, sg * x1.y), pack_h2(sg * x1.z, sg * x1.w));
                const int k = tid >> 3, jb = tid & 7;
                const float *tr = Tb + k * LSTR + 8 * jb;
                const float4 y0 = *reinterpret_cast<const float4 *>(tr);
                const float4 y1 = *reinterpret_cast<const float4 *>(tr + 4);
                *reinterpret_cast<uint4 *>(b1 + sw128_off(k, jb)) =
                    make_uint4(pack_h2(y0.x, y0.y), pack_h2(y0.z, y0.w), pack_h2(y1.x, y1.y), pack_h2(y1.z, y1.w));
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(1, K1_THREADS);
#pragma unroll 1
            for (int step = 0; step < 2; ++step) {
                if (tid == 0) {
                    // step 0: Y = [L10 ; any 96 rows] T[0..31, 0..63] (columns 32..63 of T are 0)
                    // step 1: T10 = [-T11 ; any 96 rows] Y (columns 32..63 of B2 are not used)
                    tc_fence_after();
                    const uint32_t aa = smem_u32(step ? a2 : a1), bb = smem_u32(step ? b2 : b1);
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        umma_f16_ss(tI, sdesc_sw128(aa + kk * 32, 16, 1024), sdesc_sw128(bb + kk * 2048, 16384, 1024),
                                    IDESC_KM64, kk > 0);
                    umma_commit(&bars[2]);
                    const bool w = mbar_wait(&bars[2], step, abort_flag, E_K1_MMA, kWaitLimit);
                    if (!w) mbar_wait_drain(&bars[2], step, kWaitLimit);
                    *okflag = w ? 1 : 0;
                }
                __syncwarp();
                named_bar(1, K1_THREADS);
                if (!*okflag) { inv_ok = false; break; }
                mbar_try_wait(&bars[2], step);
                tc_fence_after();
                if (warp == 0) {
                    uint32_t y[32];
                    tmem_ld32(tI, y);
                    tmem_wait_ld();
                    if (step == 0) {
                        // Y rows (TMEM lanes 0..31, columns 0..31) -> fp16 rows of B2
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            *reinterpret_cast<uint4 *>(b2 + sw128_off(lane, j)) = make_uint4(
                                pack_h2(__uint_as_float(y[8 * j]), __uint_as_float(y[8 * j + 1])),
                                pack_h2(__uint_as_float(y[8 * j + 2]), __uint_as_float(y[8 * j + 3])),
                                pack_h2(__uint_as_float(y[8 * j + 4]), __uint_as_float(y[8 * j + 5])),
                                pack_h2(__uint_as_float(y[8 * j + 6]), __uint_as_float(y[8 * j + 7])));
                        fence_proxy_async_smem();
                    } else {
                        float *dst = Tb + (32 + lane) * LSTR;
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4 *>(dst + j) = make_float4(
                                __uint_as_float(y[j]), __uint_as_float(y[j + 1]), __uint_as_float(y[j + 2]),
                                __uint_as_float(y[j + 3]));
                    }
                }
                tc_fence_before();
                named_bar(1, K1_THREADS);
            }
        }
        const float *Tsrc = Tb;
        if (p.neumann == 2) {
            float *res = reinterpret_cast<float *>(sm + K1_OFF_RES);
            Tsrc = tc::residual_correct(Lb, Tb, res, res + 64 * LSTR, res + 2 * 64 * LSTR, tid, p.S, 1);
        }
        // T diag(beta) and T diag(beta e^g) -> fp16, row-major
        if (inv_ok) {
            const int rr = tid >> 2, j0 = (tid & 3) * 2;
            uint4 *d1 = reinterpret_cast<uint4 *>(ws + (size_t)rr * 128);
            uint4 *d2 = reinterpret_cast<uint4 *>(ws + (size_t)(64 + rr) * 128);
            const float *Tr = Tsrc + rr * LSTR;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int j = j0 + q;
                float t[8], sb[8], sg[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    t[e] = 8 * j + e <= rr ? Tr[8 * j + e] : 0.f;    // T is lower triangular
                    sb[e] = t[e] * par->bet[8 * j + e];
                    sg[e] = sb[e] * par->eg[8 * j + e];
                }
                d1[j] = make_uint4(pack_h2(sb[0], sb[1]), pack_h2(sb[2], sb[3]), pack_h2(sb[4], sb[5]),
                                   pack_h2(sb[6], sb[7]));
                d2[j] = make_uint4(pack_h2(sg[0], sg[1]), pack_h2(sg[2], sg[3]), pack_h2(sg[4], sg[5]),
                                   pack_h2(sg[6], sg[7]));
            }
        }
    }
    tc_fence_before();
    block_sync();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
    if (tid == 0 && *abort_flag) atomicCAS(&g_tc_error, 0u, (unsigned)*abort_flag);
}

// ============================================================ chain kernel

constexpr int K2_THREADS = 448;    // 14 warps
constexpr int KS_THREADS = 256, CH_THREADS = 128;
// Main stage (x3): per 64-column key block kb: [W | Q | K] at kb * 24 KB, then
// P.  It holds a chunk from its load until the chain's MMAs of the chunk are
// complete; three of them let the load of chunk m + 2 start while the key side
// works on m + 1 and the chain on m.  A 128-token chunk of the masked series,
// run as two 64-token halves, keeps two stages: its extra tiles take the third.
constexpr uint32_t MSTG = 57344;
constexpr uint32_t S_W = 0, S_Q = 8192, S_K = 16384, S_KB = 24576, S_P = 49152;
constexpr uint32_t MAIN_TX = 40960;                    // bytes loaded per main stage: Q, K, P
// Early slot (x1): T diag(beta), T diag(beta e^g) and the V slice, read only by
// the U and W MMAs and reloaded as soon as those are complete.
constexpr uint32_t ES_TB = 0, ES_TBG = 8192, ES_V = 16384;
constexpr uint32_t EARLY_TX = 24576;
// Every M = 128 MMA whose A operand has only 64 real rows also reads the 8 KB
// next to them; the lanes those rows produce are never read.  The neighbours
// are not rewritten while the MMA runs: U reads T diag(beta) + T diag(beta e^g),
// W reads T diag(beta e^g) + V, the output MMA the second K block + P.
constexpr uint32_t PAR_BYTES = (sizeof(tc::ChainParams) + 15) & ~15u;
enum { B_FULL = 0, B_EMPTY = 3, B_EFULL = 6, B_EEMPTY = 7, B_KSREADY = 8, B_KSFREE = 10, B_UW = 12, B_X = 13,
       B_H = 14, B_O = 15, B_XISS = 17, B_DREADY = 18, N_BARS = 20 };
// Modes of the chain kernel: the gated delta rule at chunk 64, chunk 128 as two
// halves (the masked series), the two-gate rule (every operand from the prep's
// fp16 rows: Q', K'' in the Q and K slots, P as hi, lo; early slot TB hi, lo,
// U hi, lo, E; Delta kept as hi, lo).
enum { K2_PLAIN = 0, K2_PAIR = 1, K2_GEN = 2 };
constexpr uint32_t S_PL = S_P + 8192;                  // K2_GEN: P lo after P hi
constexpr uint32_t ES_VL = 24576, ES_E = 32768;        // K2_GEN: U lo, E (two 64-column blocks)
constexpr uint32_t GEN_MAIN_TX = 6 * 8192;             // Q', K'' (two blocks each), P hi, lo
constexpr uint32_t GEN_EARLY_TX = 6 * 8192;            // TB hi, lo, U hi, lo, E
// Shared-memory layout of the chain kernel.
template <int MODE> struct K2Layout {
    static constexpr bool PAIR = MODE == K2_PAIR, GEN = MODE == K2_GEN;
    static constexpr int NSTAGE = (PAIR || GEN) ? 2 : 3;
    static constexpr uint32_t STG = GEN ? MSTG + 8192 : MSTG;
    static constexpr uint32_t EARLY = NSTAGE * STG;
    static constexpr uint32_t HS = EARLY + (GEN ? GEN_EARLY_TX : EARLY_TX);   // h fp16, 128 rows
    static constexpr uint32_t HH = HS + 16384;                  // PAIR: e^{g_C} h of a first half, fp16
    static constexpr uint32_t DS = HH + (PAIR ? 16384 : 0);     // Delta fp16 x 2 (GEN: hi x 2, lo x 2)
    static constexpr uint32_t CORNER = DS + (GEN ? 4 : 2) * 8192; // PAIR: C1 V_a, 16 x 64 fp32, x 2
    static constexpr uint32_t C2S = CORNER + (PAIR ? 8192 : 0); // PAIR: C2', 16 x 128 fp32
    static constexpr uint32_t PAR = C2S + (PAIR ? 8192 : 0);
    static constexpr uint32_t BAR = PAR + 3 * PAR_BYTES;        // gate ring of 3
    static constexpr uint32_t MISC = BAR + N_BARS * 8;          // tmem slot, abort flag, group slots
    static constexpr uint32_t SMEM = MISC + 32 + 1024;
    static_assert((STG & 1023) == 0 && (EARLY & 1023) == 0 && (HS & 1023) == 0 && (HH & 1023) == 0 &&
                      (DS & 1023) == 0,
                  "swizzled tiles on 1024-byte boundaries");
    static_assert(SMEM <= 232448, "shared memory budget of one sm_100 block");
};
static_assert((MSTG & 1023) == 0, "swizzled tiles on 1024-byte boundaries");
static_assert(K1_SMEM * K1_BLOCKS_PER_SM <= 233472, "key-side blocks per SM");
static_assert(K1_SMEM_RES <= 232448, "residual-correction key-side block fits one SM");
static_assert(K1_OFF_YB + 8192 <= K1_OFF_TB, "L and the inverse scratch fit in the tile region");
static_assert(K1_OFF_LB + K1_MAT <= K1_OFF_B2 && K1_OFF_B2 + 4096 <= K1_OFF_A1 && K1_OFF_A1 + 4096 <= K1_OFF_TB &&
              K1_OFF_A1 + 16384 <= K1_OFF_TB + K1_MAT && (K1_OFF_B2 & 1023) == 0 && (K1_OFF_A1 & 1023) == 0 &&
              K1_OFF_A2 + 16384 + 1024 <= K1_SMEM,
              "inverse merge staging: tiles apart, 64-row operands' padding rows inside the block");

// TMEM columns
constexpr uint32_t TM_U0 = 0, TM_U1 = 64, TM_W = 128, TM_X0 = 256, TM_X1 = 320, TM_H = 384;
constexpr uint32_t TM_XB = 448;     // PAIR, second halves: [-(W + C2') ; Q'] e^{g_C} h of the first half
constexpr uint32_t TM_COLS = 512;

struct K2Params {
    int B, T, H, dv, NC;
    const float *alpha, *beta, *S0;
    const float *pair_ws;   // PAIR: C2' and C1 V_a of every second half
    const uint8_t *gen_ws;  // GEN: the prep's rows (gen_rows), ws_rows per chunk-head
    int ws_rows;            // rows of 128 B per chunk-head in the workspace map
    void *o;                // nullptr: the outputs are not stored (a state-only run)
    float *S_T;
    int o_bf16;
    int v_zero;             // PLAIN: V = 0 (no V loads), the state map's linear part
};

template <int MODE>
__global__ void __launch_bounds__(K2_THREADS, 1)
chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_t,
             const K2Params p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned base for the 128-byte swizzled tiles.  The offset is
    // applied to the __shared__ array itself so that every access below stays
    // a shared-memory access (an integer round trip would turn them generic).
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slice = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int T = p.T, H = p.H, dv = p.dv, NC = p.NC;
    const int v0 = slice * DVS;
    using L = K2Layout<MODE>;
    constexpr bool PAIR = L::PAIR, GEN = L::GEN;
    constexpr int NSTAGE = L::NSTAGE;
    constexpr uint32_t MSTG = L::STG;   // main stage stride of this mode
    constexpr uint32_t OFF_EARLY = L::EARLY, OFF_HS = L::HS, OFF_DS = L::DS, OFF_PAR = L::PAR, OFF_BAR = L::BAR,
                       OFF_MISC = L::MISC;

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    tc::ChainParams *params = reinterpret_cast<tc::ChainParams *>(sm + OFF_PAR);
    const unsigned long long lim = kWaitLimit;

    // One warp of a group polls the phase (all its lanes, so the warp stays
    // converged), the other warps wait at the group's named barrier and then
    // take the acquire with one test.
    auto group_wait = [&](uint64_t *bar, uint32_t parity, int code, int id, int nthreads, bool leader_warp,
                          bool sleep) {
        if (leader_warp) {
            if (sleep) mbar_wait(bar, parity, abort_flag, code, lim);
            else mbar_wait_spin(bar, parity, abort_flag, code, lim);
            __syncwarp();
        }
        named_bar(id, nthreads);
        if (!leader_warp) mbar_try_wait(bar, parity);
    };
    // Named barrier that also broadcasts the abort state, so that every thread
    // of a group leaves its loop at the same barrier.  Two slots per barrier id.
    auto sync_ok = [&](int id, int nthreads, bool leader, int &cnt) -> bool {
        volatile int *slots = reinterpret_cast<volatile int *>(sm + OFF_MISC + 8 + 8 * (id - 1));
        const int k = cnt++ & 1;
        if (leader) slots[k] = *abort_flag;
        __syncwarp();
        named_bar(id, nthreads);
        return slots[k] == 0;
    };

    // ------------------------------------------------------------- setup
    if (tid == 0) {
        for (int i = 0; i < NSTAGE; ++i) {
            mbar_init(&bars[B_FULL + i], 1);
            // a stage is free once the chain's MMAs (X, state update) and warp 1's
            // output MMAs that read it are complete: one commit from each issuer
            mbar_init(&bars[B_EMPTY + i], 2);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars[B_KSREADY + i], 1);
            mbar_init(&bars[B_KSFREE + i], 1);
            mbar_init(&bars[B_DREADY + i], 1);
        }
        mbar_init(&bars[B_EFULL], 1);
        mbar_init(&bars[B_EEMPTY], 1);
        mbar_init(&bars[B_UW], 1);
        mbar_init(&bars[B_X], 1);
        mbar_init(&bars[B_H], 1);
        mbar_init(&bars[B_O], 1);
        mbar_init(&bars[B_O + 1], 1);
        mbar_init(&bars[B_XISS], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncwarp();
    if (warp == 1) {
        tmem_alloc(tmem_slot, TM_COLS);
        tmem_relinquish();
    }
    if (!PAIR && !GEN && p.v_zero) {
        // V = 0: the V tile is never loaded; its in-place conversion keeps zeros
        uint4 *z = reinterpret_cast<uint4 *>(sm + OFF_EARLY + ES_V);
        for (int i = tid; i < 8192 / 16; i += K2_THREADS) z[i] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    block_sync();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ========================================================= producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_q);
            tma_prefetch_desc(&tm_k);
            tma_prefetch_desc(&tm_v);
            tma_prefetch_desc(&tm_t);
            int issued = 0, issued_early = 0;
            for (int m = 0; m < NC; ++m) {
                const int ms = m % NSTAGE;
                const int wrow = (((b * H) + h) * NC + m) * p.ws_rows;
                const int t0 = m * C;
                // main stage: free once the chain's MMAs of chunk m - 3 are complete
                if (m >= NSTAGE &&
                    !mbar_wait(&bars[B_EMPTY + ms], ((m / NSTAGE) - 1) & 1, abort_flag, E_EMPTY, lim))
                    break;
                uint64_t *fb = &bars[B_FULL + ms];
                uint8_t *st = sm + ms * MSTG;
                if (GEN) {
                    // the prep's fp16 rows: Q', K'' (two key blocks each), P hi, lo
                    const GenRows G = gen_rows(dv);
                    mbar_arrive_expect_tx(fb, GEN_MAIN_TX);
                    tma_load_4d(st + S_Q, &tm_t, fb, 0, 0, wrow + G.q, 0);
                    tma_load_4d(st + S_KB + S_Q, &tm_t, fb, 0, 0, wrow + G.q + 64, 0);
                    tma_load_4d(st + S_K, &tm_t, fb, 0, 0, wrow + G.k, 0);
                    tma_load_4d(st + S_KB + S_K, &tm_t, fb, 0, 0, wrow + G.k + 64, 0);
                    tma_load_4d(st + S_P, &tm_t, fb, 0, 0, wrow + G.pp, 0);
                    tma_load_4d(st + S_PL, &tm_t, fb, 0, 0, wrow + G.ppl, 0);
                } else {
                    mbar_arrive_expect_tx(fb, MAIN_TX);
                    tma_load_4d(st + S_Q, &tm_q, fb, 0, h, t0, b);
                    tma_load_4d(st + S_KB + S_Q, &tm_q, fb, 64, h, t0, b);
                    tma_load_4d(st + S_K, &tm_k, fb, 0, h, t0, b);
                    tma_load_4d(st + S_KB + S_K, &tm_k, fb, 64, h, t0, b);
                    tma_load_4d(st + S_P, &tm_t, fb, 0, 0, wrow + 128, 0);
                }
                issued = m + 1;
                // early slot: free once the U and W MMAs of chunk m - 1 are complete
                if (m >= 1 && !mbar_wait(&bars[B_EEMPTY], (m - 1) & 1, abort_flag, E_EMPTY, lim)) break;
                uint64_t *eb = &bars[B_EFULL];
                const bool second = PAIR && (m & 1);
                uint8_t *es = sm + OFF_EARLY;
                if (GEN) {
                    // TB hi, lo, this slice's U = w (.) v hi, lo, and E (read only by the
                    // U and W products, like the rest of the early slot)
                    const GenRows G = gen_rows(dv);
                    mbar_arrive_expect_tx(eb, GEN_EARLY_TX);
                    tma_load_4d(es + ES_TB, &tm_t, eb, 0, 0, wrow + G.tb, 0);
                    tma_load_4d(es + ES_TBG, &tm_t, eb, 0, 0, wrow + G.tbl, 0);
                    tma_load_4d(es + ES_V, &tm_t, eb, 0, 0, wrow + G.u + 64 * slice, 0);
                    tma_load_4d(es + ES_VL, &tm_t, eb, 0, 0, wrow + G.ul + 64 * slice, 0);
                    tma_load_4d(es + ES_E, &tm_t, eb, 0, 0, wrow + G.e, 0);
                    tma_load_4d(es + ES_E + 8192, &tm_t, eb, 0, 0, wrow + G.e + 64, 0);
                } else {
                    mbar_arrive_expect_tx(eb, EARLY_TX - (p.v_zero ? 8192u : 0u) + (second ? 8192u + 4096u : 0u));
                    if (!p.v_zero) tma_load_4d(es + ES_V, &tm_v, eb, v0, h, t0, b);
                    tma_load_4d(es + ES_TB, &tm_t, eb, 0, 0, wrow, 0);
                    tma_load_4d(es + ES_TBG, &tm_t, eb, 0, 0, wrow + 64, 0);
                }
                if (second) {
                    // second half of a 128-token chunk: C2' for the key side and this
                    // slice's C1 V_a for the chain (two buffers: the chain may still be
                    // reading the previous pair's while this one lands)
                    const float *src = p.pair_ws + (((size_t)b * H + h) * NC + m) * pair_stride(dv);
                    bulk_load_g2s(sm + L::C2S, src, 8192u, eb);
                    bulk_load_g2s(sm + L::CORNER + ((m >> 1) & 1) * 4096u, src + PAIR_MAXN * DK + slice * (PAIR_MAXN * 64),
                                  4096u, eb);
                }
                issued_early = m + 1;
            }
            // no copy may still be in flight when the block exits: the last load of
            // each stage, and of the early slot
            for (int m = issued - NSTAGE < 0 ? 0 : issued - NSTAGE; m < issued; ++m)
                mbar_wait_drain(&bars[B_FULL + m % NSTAGE], (m / NSTAGE) & 1, lim);
            if (issued_early > 0) mbar_wait_drain(&bars[B_EFULL], (issued_early - 1) & 1, lim);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ========================================================= output MMAs
        // O(n) += [preceding rows ; P] Delta(n) into lanes 64..127 of X(n)'s
        // buffer, once the chain has stored Delta(n) and issued its state update.
        // Off the chain: its issue no longer holds up the chain's own warps.
        if (lane == 0) {
            int opend = -1, opar = 0;
            for (int n = 0; n < NC; ++n) {
                const int s = n & 1;
                if (!mbar_wait_spin(&bars[B_DREADY + s], (n >> 1) & 1, abort_flag, E_DREADY, lim)) break;
                tc_fence_after();
                uint8_t *st = sm + (n % NSTAGE) * MSTG;
                const uint32_t ap = smem_u32(st + S_P) - 8192, bd = smem_u32(sm + OFF_DS + s * 8192);
                const uint32_t xcol = s ? TM_X1 : TM_X0;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16_ss(tmem + xcol, sdesc_sw128(ap + kk * 32, 16, 1024),
                                sdesc_sw128(bd + kk * 2048, 8192, 1024), IDESC_KM64, 1);
                if (GEN) {
                    // P and Delta as hi + lo: + P_hi Delta_lo, + P_lo Delta_hi ([P_hi ; P_lo]:
                    // its top half lands in lanes 0..63, whose -W h the chain has read)
                    const uint32_t bdl = bd + 16384;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ss(tmem + xcol, sdesc_sw128(ap + kk * 32, 16, 1024),
                                    sdesc_sw128(bdl + kk * 2048, 8192, 1024), IDESC_KM64, 1);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ss(tmem + xcol, sdesc_sw128(ap + 8192 + kk * 32, 16, 1024),
                                    sdesc_sw128(bd + kk * 2048, 8192, 1024), IDESC_KM64, 1);
                }
                umma_commit(&bars[B_O + s]);
                umma_commit(&bars[B_EMPTY + n % NSTAGE]);
                opend = B_O + s;
                opar = (n >> 1) & 1;
            }
            // error path: no MMA of this role may still be running when TMEM is released
            if (opend >= 0 && *abort_flag) mbar_wait_drain(&bars[opend], opar, lim);
        }
        __syncwarp();
    } else if (warp >= 2 && warp < 10) {
        // ========================================================= key side
        // 8 warps, two per TMEM sub-partition; warp half hf takes columns
        // [32 hf, 32 hf + 32) of the rows its sub-partition holds.
        const int kt = tid - 64;                  // 0..255
        const int sp = warp & 3;
        const int hf = (warp - 2) >> 2;
        const bool leader = (kt == 0);           // MMA issue and flag writes
        const bool lwarp = (kt >> 5) == 0;        // polls the group's waits
        const bool scan_warp = (kt >> 5) == 2;
        float ga0 = 1.f, ga1 = 1.f, gb0 = 0.f, gb1 = 0.f;
        // GEN: the state's per-channel decay d of chunk mm (128 floats) into the
        // gate record (channels 0..63 in eg, 64..127 in egc), by the scan warp
        auto load_d = [&](int mm, tc::ChainParams *dst) {
            const GenRows G = gen_rows(dv);
            const float4 v = *reinterpret_cast<const float4 *>(
                p.gen_ws + ((((size_t)b * H + h) * NC + mm) * p.ws_rows + G.d) * 128 + 16 * lane);
            float *dd = lane < 16 ? dst->eg + 4 * lane : dst->egc + 4 * (lane - 16);
            dd[0] = v.x; dd[1] = v.y; dd[2] = v.z; dd[3] = v.w;
        };
        if (scan_warp) {
            if (GEN) {
                load_d(0, &params[0]);
            } else {
                tc::fetch_gates(p.alpha, p.beta, b, T, H, h, 0, lane, true, ga0, ga1, gb0, gb1);
                tc::scan_gates_chain(&params[0], ga0, ga1, lane);
                tc::fetch_gates(p.alpha, p.beta, b, T, H, h, C, lane, NC > 1, ga0, ga1, gb0, gb1);
            }
        }
        int kcnt = 0;
        int pend = -1;   // leader: barrier of the last commit not yet known complete
        int pend_par = 0;
        for (int m = 0; m < NC; ++m) {
            const int s = m & 1, ms = m % NSTAGE;
            const tc::ChainParams *par = &params[m % 3];
            uint8_t *st = sm + ms * MSTG;
            uint8_t *es = sm + OFF_EARLY;
            // chain finished chunk m-2: the U buffer s is free (the stage's W slots
            // came free with the stage itself)
            // one warp polls both phases, one barrier releases the group; the other
            // warps then take the acquire of the loaded tiles with one test
            if (lwarp) {
                if (m >= 2) mbar_wait(&bars[B_KSFREE + s], ((m - 2) >> 1) & 1, abort_flag, E_KSFREE, lim);
                mbar_wait(&bars[B_FULL + ms], (m / NSTAGE) & 1, abort_flag, E_FULL, lim);
                __syncwarp();
            }
            if (!sync_ok(1, KS_THREADS, leader, kcnt)) break;
            if (!lwarp) mbar_try_wait(&bars[B_FULL + ms], (m / NSTAGE) & 1);
            // in-place fp16 operands: Q -> e^{g_r} Q, K -> K in the main stage, then
            // V in the early slot once it has landed.  Every load of a pass is
            // issued before the first store, so they overlap instead of waiting on
            // one another.
            auto convert = [&](uint8_t *const (&addr)[8], const float (&sc)[8], int cnt) {
                uint4 w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (i < cnt) w[i] = *reinterpret_cast<const uint4 *>(addr[i]);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    if (i < cnt) {
                        const float2 f0 = unpack_bf2(w[i].x), f1 = unpack_bf2(w[i].y);
                        const float2 f2 = unpack_bf2(w[i].z), f3 = unpack_bf2(w[i].w);
                        uint4 o;
                        o.x = pack_h2(f0.x * sc[i], f0.y * sc[i]);
                        o.y = pack_h2(f1.x * sc[i], f1.y * sc[i]);
                        o.z = pack_h2(f2.x * sc[i], f2.y * sc[i]);
                        o.w = pack_h2(f3.x * sc[i], f3.y * sc[i]);
                        *reinterpret_cast<uint4 *>(addr[i]) = o;
                    }
                }
            };
            if (!GEN) {
                uint8_t *addr[8];
                float sc[8];
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const int u = kt + 256 * (it & 1);      // 16-byte chunk within one 8 KB tile
                    const int tile = it >> 1;               // Q0, Q1, K0, K1
                    const uint32_t off = tile == 0 ? S_Q : tile == 1 ? S_KB + S_Q : tile == 2 ? S_K : S_KB + S_K;
                    addr[it] = st + off + (u << 4);
                    sc[it] = tile < 2 ? par->eg[u >> 3] : 1.f;
                }
                convert(addr, sc, 8);
            }
            group_wait(&bars[B_EFULL], m & 1, E_FULL, 1, KS_THREADS, lwarp, true);
            if (!GEN) {
                uint8_t *addr[8];
                float sc[8];
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    addr[it] = es + ES_V + ((kt + 256 * (it & 1)) << 4);
                    sc[it] = 1.f;
                }
                convert(addr, sc, 2);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            if (!sync_ok(1, KS_THREADS, leader, kcnt)) break;
            // the U and W MMAs of chunk m go into the tensor pipe right after the
            // chain has issued X(m - 1): they run while its Delta epilogue does,
            // instead of landing ahead of the state update it waits for
            if (leader && m >= 1 && !mbar_wait(&bars[B_XISS], (m - 1) & 1, abort_flag, E_XISS, lim)) {
                // abort: the group leaves at the next wait
            } else if (leader) {
                tc_fence_after();
                const uint32_t at = smem_u32(es + ES_TB), av = smem_u32(es + ES_V);
                const uint32_t du = tmem + (s ? TM_U1 : TM_U0);
                if (GEN) {
                    // U = TB U_in and W = TB E with TB, U_in as hi + lo (the lo x lo
                    // product, about 2^-22 relative, dropped).  A = TB hi or lo with the
                    // 8 KiB after it as padding rows; E two 64-column blocks 8 KiB apart.
                    const uint32_t atl = smem_u32(es + ES_TBG), avl = smem_u32(es + ES_VL);
                    const uint32_t ae = smem_u32(es + ES_E);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ss(du, sdesc_sw128(at + kk * 32, 16, 1024),
                                    sdesc_sw128(av + kk * 2048, 8192, 1024), IDESC_KM64, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ss(du, sdesc_sw128(at + kk * 32, 16, 1024),
                                    sdesc_sw128(avl + kk * 2048, 8192, 1024), IDESC_KM64, 1);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ss(du, sdesc_sw128(atl + kk * 32, 16, 1024),
                                    sdesc_sw128(av + kk * 2048, 8192, 1024), IDESC_KM64, 1);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ss(tmem + TM_W, sdesc_sw128(at + kk * 32, 16, 1024),
                                    sdesc_sw128(ae + kk * 2048, 8192, 1024), IDESC_KM128, kk > 0);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ss(tmem + TM_W, sdesc_sw128(atl + kk * 32, 16, 1024),
                                    sdesc_sw128(ae + kk * 2048, 8192, 1024), IDESC_KM128, 1);
                } else {
                    const uint32_t ag = smem_u32(es + ES_TBG), ak = smem_u32(st + S_K);
                    // U = T diag(beta) V: [T diag(beta) ; next rows] x V (MN-major), K = 64 tokens
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ss(du, sdesc_sw128(at + kk * 32, 16, 1024),
                                    sdesc_sw128(av + kk * 2048, 8192, 1024), IDESC_KM64, kk > 0);
                    // W = T diag(beta e^g) K: K as MN-major B with N = 128 (two key blocks)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ss(tmem + TM_W, sdesc_sw128(ag + kk * 32, 16, 1024),
                                    sdesc_sw128(ak + kk * 2048, S_KB, 1024), IDESC_KM128, kk > 0);
                }
                umma_commit(&bars[B_UW]);
                umma_commit(&bars[B_EEMPTY]);       // the early slot reloads once U and W are formed
                pend = B_UW; pend_par = m & 1;
            }
            __syncwarp();
            // gates of the next chunk meanwhile
            if (scan_warp && m + 1 < NC) {
                if (GEN) {
                    load_d(m + 1, &params[(m + 1) % 3]);
                } else {
                    tc::scan_gates_chain(&params[(m + 1) % 3], ga0, ga1, lane);
                    tc::fetch_gates(p.alpha, p.beta, b, T, H, h, (m + 2) * C, lane, m + 2 < NC, ga0, ga1, gb0, gb1);
                }
            }
            group_wait(&bars[B_UW], m & 1, E_UW, 1, KS_THREADS, lwarp, false);
            if (!sync_ok(1, KS_THREADS, leader, kcnt)) break;
            tc_fence_after();
            if (sp < 2) {
                // -W rows (TMEM lanes 0..63) -> fp16 into the W slot of key block hf
                const int r = 32 * sp + lane;
                float x[64];
                tmem_ld64(tmem + ((uint32_t)(32 * sp) << 16) + TM_W + 64 * hf, x);
                if (PAIR && (m & 1) && r < PAIR_MAXN) {
                    // -(W + C2'): the band corner's key part of a second half
                    const float *c2 = reinterpret_cast<const float *>(sm + L::C2S) + r * 128 + 64 * hf;
#pragma unroll
                    for (int j = 0; j < 64; ++j) x[j] = -x[j] - c2[j];
                } else {
#pragma unroll
                    for (int j = 0; j < 64; ++j) x[j] = -x[j];
                }
                st_row_f16(st + hf * S_KB + S_W, r, x);
            } else if (!GEN) {
                // W has read K: K -> diag(e^{g_C - g}) K in place for the state update
                // (GEN: K'' comes scaled from the prep)
                const int t2 = 64 * hf + 32 * (sp - 2) + lane;
                uint8_t *addr[8];
                uint4 w[8];
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const int idx = t2 + 128 * it;               // 16-byte chunk of the two K blocks
                    addr[it] = st + (idx >> 9) * S_KB + S_K + ((idx & 511) << 4);
                    w[it] = *reinterpret_cast<const uint4 *>(addr[it]);
                }
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const float sc = par->egc[((t2 + 128 * it) & 511) >> 3];
                    const float2 f0 = unpack_h2(w[it].x), f1 = unpack_h2(w[it].y);
                    const float2 f2 = unpack_h2(w[it].z), f3 = unpack_h2(w[it].w);
                    uint4 o;
                    o.x = pack_h2(f0.x * sc, f0.y * sc);
                    o.y = pack_h2(f1.x * sc, f1.y * sc);
                    o.z = pack_h2(f2.x * sc, f2.y * sc);
                    o.w = pack_h2(f3.x * sc, f3.y * sc);
                    *reinterpret_cast<uint4 *>(addr[it]) = o;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar(1, KS_THREADS);
            if (leader) {
                pend = -1;
                mbar_arrive(&bars[B_KSREADY + s]);
            }
            __syncwarp();
        }
        if (leader && pend >= 0 && *abort_flag) mbar_wait_drain(&bars[pend], pend_par, lim);
        __syncwarp();
    } else if (warp >= 10) {
        // ========================================================= state chain
        const int ct = tid - 320;          // 0..127
        const int sp = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * sp) << 16;
        const int hrow = 32 * sp + lane;   // key row of h held by this thread
        const bool rowpart = (sp < 2);     // Delta rows live in TMEM lanes 0..63
        const bool issuer = (ct == 64);    // warp 12 lane 0, sub-partition 0: MMA issue
        const bool iwarp = (ct >> 5) == 2; // warp 12 polls the chain's waits
        uint8_t *hs = sm + OFF_HS;
        const size_t bh = (size_t)b * H + h;
        {
            float x[64];
#pragma unroll
            for (int j = 0; j < 64; j += 4) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (p.S0) v = *reinterpret_cast<const float4 *>(p.S0 + (bh * DK + hrow) * dv + v0 + j);
                x[j] = v.x; x[j + 1] = v.y; x[j + 2] = v.z; x[j + 3] = v.w;
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t y[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) y[j] = __float_as_uint(x[32 * hh + j]);
                tmem_st32(tmem + lane_base + TM_H + 32 * hh, y);
            }
            tmem_wait_st();
        }
        auto store_o = [&](int n) {
            // O rows of chunk n: TMEM lanes 64..127 of its X buffer
            const int r = 32 * (sp - 2) + lane;
            float x[64];
            tmem_ld64(tmem + lane_base + ((n & 1) ? TM_X1 : TM_X0), x);
            const int t = n * C + r;
            if (t < T && p.o) {
                const size_t go = (((size_t)b * T + t) * H + h) * dv + v0;
                if (p.o_bf16) {
                    __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(p.o) + go;
#pragma unroll
                    for (int j = 0; j < 64; j += 8) {
                        uint4 u;
                        __nv_bfloat162 q0 = __floats2bfloat162_rn(x[j], x[j + 1]);
                        __nv_bfloat162 q1 = __floats2bfloat162_rn(x[j + 2], x[j + 3]);
                        __nv_bfloat162 q2 = __floats2bfloat162_rn(x[j + 4], x[j + 5]);
                        __nv_bfloat162 q3 = __floats2bfloat162_rn(x[j + 6], x[j + 7]);
                        u.x = *reinterpret_cast<uint32_t *>(&q0);
                        u.y = *reinterpret_cast<uint32_t *>(&q1);
                        u.z = *reinterpret_cast<uint32_t *>(&q2);
                        u.w = *reinterpret_cast<uint32_t *>(&q3);
                        *reinterpret_cast<uint4 *>(dst + j) = u;
                    }
                } else {
                    float *dst = reinterpret_cast<float *>(p.o) + go;
#pragma unroll
                    for (int j = 0; j < 64; j += 4)
                        *reinterpret_cast<float4 *>(dst + j) = make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
                }
            }
        };
        // Warps 10, 11: the output rows of chunk j once its P Delta MMA is complete.
        auto out_rows = [&](int j) {
            if (mbar_wait(&bars[B_O + (j & 1)], (j >> 1) & 1, abort_flag, E_O, lim)) {
                __syncwarp();
                tc_fence_after();
                store_o(j);
            }
            __syncwarp();
        };
        // every chain warp polls a phase itself (all lanes, so the warp stays converged)
        auto warp_wait = [&](uint64_t *bar, uint32_t parity, int code) {
            const bool ok = mbar_wait_spin(bar, parity, abort_flag, code, lim);
            __syncwarp();
            return ok;
        };
        int ccnt = 0, dcnt = 0;
        int pend = -1, pend_par = 0;       // issuer: last commit not yet known complete
        bool done = true;
        for (int n = 0; n < NC; ++n) {
            const int s = n & 1;
            const tc::ChainParams *par = &params[n % 3];
            uint8_t *st = sm + (n % NSTAGE) * MSTG;
            const uint32_t xcol = s ? TM_X1 : TM_X0;
            // state update of the previous chunk complete (its output rows may still be running)
            if (n > 0) warp_wait(&bars[B_H], (n - 1) & 1, E_H);
            // the gates of chunk 0 are scanned by the key side at start-up: wait for it
            else warp_wait(&bars[B_KSREADY], 0, E_KSREADY);
            tc_fence_after();
            // ---- h <- e^{g_C} h in TMEM (issued first), h -> fp16 operand.  The
            // gates of chunk n > 0 were scanned before the key side released chunk n-1.
            {
                float x[64];
                tmem_ld64(tmem + lane_base + TM_H, x);
                // the state's decay over the chunk: e^{g_C}, or per key channel (GEN)
                const float egC = GEN ? (hrow < 64 ? par->eg[hrow] : par->egc[hrow - 64]) : par->egC;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t y[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) y[j] = __float_as_uint(x[32 * hh + j] * egC);
                    tmem_st32(tmem + lane_base + TM_H + 32 * hh, y);
                }
                st_row_f16(hs, hrow, x);
                if (PAIR && !(n & 1) && n + 1 < NC) {
                    // first half of a 128-token chunk: e^{g_C} h, the state the second
                    // half's Delta is formed from
#pragma unroll
                    for (int j = 0; j < 64; ++j) x[j] *= egC;
                    st_row_f16(sm + L::HH, hrow, x);
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            // Only the MMAs read the key side's operands of chunk n: the issuing warp
            // waits for them, and the barrier then orders every chain warp after that
            // acquire (the gates of chunk n + 1, which the next c1 reads, were scanned
            // before the key side released chunk n).
            if (iwarp) warp_wait(&bars[B_KSREADY + s], (n >> 1) & 1, E_KSREADY);
            if (!sync_ok(2, CH_THREADS, issuer, ccnt)) { done = false; break; }
            if (issuer) {
                // [-W ; Q'] h16: lanes 0..63 -W h, lanes 64..127 Q'h
                tc_fence_after();
                const uint32_t a0 = smem_u32(st), b0 = smem_u32(hs);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t aoff = (kk >> 2) * S_KB + (kk & 3) * 32;
                    umma_f16_ss(tmem + xcol, sdesc_sw128(a0 + S_W + aoff, 16, 1024),
                                sdesc_sw128(b0 + kk * 2048, 8192, 1024), IDESC_KM64, kk > 0);
                }
                if (PAIR && (n & 1)) {
                    // second half: [-(W + C2') ; Q'] (e^{g_C} h of the first half); only
                    // its lanes 0..63 are read
                    const uint32_t b1 = smem_u32(sm + L::HH);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t aoff = (kk >> 2) * S_KB + (kk & 3) * 32;
                        umma_f16_ss(tmem + TM_XB, sdesc_sw128(a0 + S_W + aoff, 16, 1024),
                                    sdesc_sw128(b1 + kk * 2048, 8192, 1024), IDESC_KM64, kk > 0);
                    }
                }
                umma_commit(&bars[B_X]);
                mbar_arrive(&bars[B_XISS]);
                pend = B_X; pend_par = n & 1;
            }
            __syncwarp();
            if (!rowpart) {
                // sub-partitions 2, 3: output rows of the previous chunk, off the chain
                if (n > 0) out_rows(n - 1);
                continue;
            }
            warp_wait(&bars[B_X], n & 1, E_X);
            tc_fence_after();
            // ---- Delta = U - W h (rows in lanes 0..63) -> fp16 operands
            {
                const int r = 32 * sp + lane;
                float x[64], u[64];
                tmem_ld64(tmem + lane_base + ((PAIR && s) ? TM_XB : xcol), x);
                tmem_ld64(tmem + lane_base + (s ? TM_U1 : TM_U0), u);
#pragma unroll
                for (int j = 0; j < 64; ++j) x[j] += u[j];
                if (PAIR && s && r < PAIR_MAXN) {
                    // second half: + C1 V_a, the corner's value part
                    const float *cr = reinterpret_cast<const float *>(sm + L::CORNER + ((n >> 1) & 1) * 4096u) + r * 64;
#pragma unroll
                    for (int j = 0; j < 64; ++j) x[j] += cr[j];
                }
                if (GEN) {
                    // Delta as hi + lo fp16 (u reused for the low parts)
#pragma unroll
                    for (int j = 0; j < 64; ++j) u[j] = x[j] - __half2float(__float2half_rn(x[j]));
                    st_row_f16(sm + OFF_DS + 16384 + s * 8192, r, u);
                }
                st_row_f16(sm + OFF_DS + s * 8192, r, x);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            // 64-thread barrier of sub-partitions 0, 1; an abort here only stops the
            // MMAs, the loop exits at the next 128-thread barrier
            if (sync_ok(3, 64, issuer, dcnt) && issuer) {
                tc_fence_after();
                const uint32_t ak = smem_u32(st + S_K), bd = smem_u32(sm + OFF_DS + s * 8192);
                // h += (diag(e^{g_C - g}) K)^T Delta: the next chunk waits on it alone.
                // The key side rescaled K in place; K^T as MN-major A over the two key
                // blocks.  The output MMAs of this chunk are warp 1's.
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16_ss(tmem + TM_H, sdesc_sw128(ak + kk * 2048, S_KB, 1024),
                                sdesc_sw128(bd + kk * 2048, 8192, 1024), IDESC_MM64, 1);
                if (GEN) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ss(tmem + TM_H, sdesc_sw128(ak + kk * 2048, S_KB, 1024),
                                    sdesc_sw128(bd + 16384 + kk * 2048, 8192, 1024), IDESC_MM64, 1);
                }
                umma_commit(&bars[B_H]);
                umma_commit(&bars[B_EMPTY + n % NSTAGE]);   // X and the state update have read the stage
                umma_commit(&bars[B_KSFREE + s]);            // and Delta has read U
                tc_fence_before();
                mbar_arrive(&bars[B_DREADY + s]);
                pend = B_H; pend_par = n & 1;
            }
            __syncwarp();
        }
        if (done && NC > 0) {
            warp_wait(&bars[B_H], (NC - 1) & 1, E_H);
            if (sync_ok(2, CH_THREADS, issuer, ccnt)) {
                tc_fence_after();
                if (!rowpart) out_rows(NC - 1);
                if (p.S_T) {
                    float x[64];
                    tmem_ld64(tmem + lane_base + TM_H, x);
                    float *dst = p.S_T + (bh * DK + hrow) * dv + v0;
#pragma unroll
                    for (int j = 0; j < 64; j += 4)
                        *reinterpret_cast<float4 *>(dst + j) = make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
                }
            }
        }
        // error path: no MMA of this role may still be running when TMEM is released
        if (issuer && pend >= 0 && *abort_flag) mbar_wait_drain(&bars[pend], pend_par, lim);
        __syncwarp();
    }
    // ---------------------------------------------------------- teardown
    tc_fence_before();
    block_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
    if (tid == 0 && *abort_flag) atomicCAS(&g_tc_error, 0u, (unsigned)*abort_flag);
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// [B, T, H, D] bf16 viewed as 4-D (D, H, T, B); box 64 x 1 x 64 x 1, 128-byte swizzle.
bool make_map_bthd(CUtensorMap *m, const void *ptr, int B, int T, int H, int D) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)C, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Workspace [rows, 64] fp16 viewed as 4-D (64, 1, rows, 1); box 64 x 1 x 64 x 1
// (one of the three matrices of a chunk-head).
bool make_map_t(CUtensorMap *m, const void *ptr, size_t rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {64, 1, (cuuint64_t)rows, 1};
    cuuint64_t strides[3] = {128, 128, (cuuint64_t)rows * 128};
    cuuint32_t box[4] = {64, 1, 64, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}


// ------------------------------------------------- sequence segments (B = 1)
//
// The recurrence is affine in the state: over any run of tokens the final h is
// M h_start + N, M (d_k x d_k) the run's product of transitions and N its final
// state from h_start = 0.  A long sequence is cut into three segments s0, s1,
// s2.  Pass 1 runs s0 from S0, s1 from 0 (-> N) and s1 with V = 0 from the
// identity (-> M) side by side; then h(s2 start) = M h(s1 start) + N; pass 2
// runs s1 and s2 from their true starts.  Two chain passes of a third of the
// chunks each, instead of one pass over all of them, when the per-head chains
// alone cannot fill the SMs.

// h = S^T of every head set to the identity (d_k x d_k): the start of M's run.
__global__ void seg_identity_kernel(float *I, int dk) {
    const int h = blockIdx.y, r = blockIdx.x;
    for (int c = threadIdx.x; c < dk; c += blockDim.x) I[((size_t)h * dk + r) * dk + c] = r == c ? 1.f : 0.f;
}

// out = M h1 + N per head: M [H, dk, dk], h1, N, out [H, dk, dv]; one block per
// (row, head), one thread per value column.
__global__ void seg_compose_kernel(const float *M, const float *h1, const float *N, float *out, int dk, int dv) {
    __shared__ float mr[DK];
    const int h = blockIdx.y, r = blockIdx.x;
    for (int i = threadIdx.x; i < dk; i += blockDim.x) mr[i] = M[((size_t)h * dk + r) * dk + i];
    __syncthreads();
    const float *hh = h1 + (size_t)h * dk * dv;
    for (int c = threadIdx.x; c < dv; c += blockDim.x) {
        float acc = N[((size_t)h * dk + r) * dv + c];
        for (int i = 0; i < dk; ++i) acc = fmaf(mr[i], hh[(size_t)i * dv + c], acc);
        out[((size_t)h * dk + r) * dv + c] = acc;
    }
}

// The key-side kernel over p's tokens, T matrices into ws.
cudaError_t launch_k1_plain(const FwdParams &p, void *ws, cudaStream_t stream) {
    CUtensorMap mq, mk;
    if (!make_map_bthd(&mq, p.q, p.B, p.T, p.H, p.dk) || !make_map_bthd(&mk, p.k, p.B, p.T, p.H, p.dk))
        return cudaErrorInvalidValue;
    const int NC = (p.T + C - 1) / C;
    K1Params k1;
    k1.B = p.B; k1.T = p.T; k1.H = p.H; k1.NC = NC;
    k1.alpha = p.alpha; k1.beta = p.beta;
    k1.ws = reinterpret_cast<uint8_t *>(ws);
    k1.neumann = p.mode == GDN_INV_NEUMANN ? 1 : (p.mode == GDN_INV_NEUMANN_RESIDUAL ? 2 : 0);
    k1.N = p.N; k1.S = p.S;
    keyside_kernel<<<dim3(NC, p.H, p.B), K1_THREADS, k1.neumann == 2 ? K1_SMEM_RES : K1_SMEM, stream>>>(mq, mk, k1);
    return cudaGetLastError();
}

// The chain kernel (chunk 64) over p's tokens, reading the T matrices from ws;
// p.v == nullptr runs it with V = 0.
cudaError_t launch_k2_plain(const FwdParams &p, const void *ws, cudaStream_t stream) {
    CUtensorMap mq, mk, mv, mt;
    const int NC = (p.T + C - 1) / C;
    if (!make_map_bthd(&mq, p.q, p.B, p.T, p.H, p.dk) || !make_map_bthd(&mk, p.k, p.B, p.T, p.H, p.dk) ||
        !make_map_t(&mt, ws, (size_t)p.B * p.H * NC * WS_ROWS))
        return cudaErrorInvalidValue;
    if (p.v) {
        if (!make_map_bthd(&mv, p.v, p.B, p.T, p.H, p.dv)) return cudaErrorInvalidValue;
    } else {
        mv = mq;    // never read: the kernel loads no V
    }
    K2Params k2{};
    k2.ws_rows = WS_ROWS;
    k2.B = p.B; k2.T = p.T; k2.H = p.H; k2.dv = p.dv; k2.NC = NC;
    k2.alpha = p.alpha; k2.beta = p.beta; k2.S0 = p.S0; k2.o = p.o; k2.S_T = p.S_T;
    k2.o_bf16 = p.o_bf16;
    k2.v_zero = p.v ? 0 : 1;
    chain_kernel<K2_PLAIN><<<dim3(p.dv / DVS, p.H, p.B), K2_THREADS, K2Layout<K2_PLAIN>::SMEM, stream>>>(mq, mk, mv, mt,
                                                                                                  k2);
    return cudaGetLastError();
}

// Streams and events of the segment schedule, one set per device, made on first
// use with that device current.  The chain runs go to high-priority streams so
// that their blocks are placed ahead of the key-side blocks running beside them.
struct SegStreams {
    bool ready = false;
    cudaStream_t run[3] = {};
    cudaStream_t side = nullptr;
    cudaEvent_t ev[8] = {};
};
constexpr int kSegMaxDevices = 64;
SegStreams g_seg[kSegMaxDevices];
std::mutex g_seg_mu;

cudaError_t seg_streams(int dev, SegStreams **out) {
    SegStreams &S = g_seg[dev];
    if (!S.ready) {
        int lo = 0, hi = 0;
        cudaError_t e = cudaDeviceGetStreamPriorityRange(&lo, &hi);
        if (e != cudaSuccess) return e;
        for (auto &r : S.run)
            if ((e = cudaStreamCreateWithPriority(&r, cudaStreamNonBlocking, hi)) != cudaSuccess) return e;
        if ((e = cudaStreamCreateWithPriority(&S.side, cudaStreamNonBlocking, lo)) != cudaSuccess) return e;
        for (auto &v : S.ev)
            if ((e = cudaEventCreateWithFlags(&v, cudaEventDisableTiming)) != cudaSuccess) return e;
        S.ready = true;
    }
    *out = &S;
    return cudaSuccess;
}

// p with its token range cut to [t0, t0 + T) (B = 1: every [B, T, H, *] tensor
// is contiguous in t).
FwdParams seg_view(const FwdParams &p, int t0, int T) {
    FwdParams s = p;
    const size_t r = (size_t)t0 * p.H;
    s.T = T;
    s.q = reinterpret_cast<const uint8_t *>(p.q) + r * p.dk * 2;
    s.k = reinterpret_cast<const uint8_t *>(p.k) + r * p.dk * 2;
    s.v = reinterpret_cast<const uint8_t *>(p.v) + r * p.dv * 2;
    s.alpha = p.alpha ? p.alpha + r : nullptr;
    s.beta = p.beta ? p.beta + r : nullptr;
    s.o = reinterpret_cast<uint8_t *>(p.o) + r * p.dv * (p.o_bf16 ? 2 : 4);
    return s;
}

// Workspace of the segment schedule: the T matrices of every chunk-head (as one
// pass), then the identity, M, N, h(s1 start) and h(s2 start) per head.
size_t seg_state_floats(const FwdParams &p) { return (size_t)p.H * p.dk * (2 * (size_t)p.dk + 3 * (size_t)p.dv); }

cudaError_t launch_tc_segments(const FwdParams &p, void *workspace, cudaStream_t stream) {
    const int NC = (p.T + C - 1) / C;
    const int L = NC / 3;                   // chunks of s0 and of s1; s2 takes the rest
    const int T0 = L * C;
    const int t0[3] = {0, T0, 2 * T0}, Ts[3] = {T0, T0, p.T - 2 * T0};
    const size_t per_seg = (size_t)p.H * L * WS_CHUNK_BYTES;
    uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
    uint8_t *wsg[3] = {ws, ws + per_seg, ws + 2 * per_seg};
    float *sI = reinterpret_cast<float *>(ws + (size_t)p.H * NC * WS_CHUNK_BYTES);
    const size_t kk = (size_t)p.H * p.dk * p.dk, kv = (size_t)p.H * p.dk * p.dv;
    float *sM = sI + kk, *sN = sM + kk, *sH1 = sN + kv, *sH2 = sH1 + kv;

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kSegMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_seg_mu);   // one schedule at a time uses the set
    SegStreams *S = nullptr;
    if ((e = seg_streams(dev, &S)) != cudaSuccess) return e;
    cudaEvent_t ev_k1 = S->ev[0], ev_n = S->ev[1], ev_m = S->ev[2], ev_h1 = S->ev[3], ev_k1b = S->ev[4],
                ev_s1 = S->ev[5], ev_s2 = S->ev[6];
    cudaStream_t r0 = S->run[0], r1 = S->run[1], r2 = S->run[2], side = S->side;
#define GDN_SEG_TRY(x) \
    do { if ((e = (x)) != cudaSuccess) return e; } while (0)

    // key side of s0 and s1, and the identity, on the caller's stream
    const FwdParams v0 = seg_view(p, t0[0], Ts[0]), v1 = seg_view(p, t0[1], Ts[1]), v2 = seg_view(p, t0[2], Ts[2]);
    GDN_SEG_TRY(launch_k1_plain(v0, wsg[0], stream));
    GDN_SEG_TRY(launch_k1_plain(v1, wsg[1], stream));
    seg_identity_kernel<<<dim3(p.dk, p.H), 128, 0, stream>>>(sI, p.dk);
    GDN_SEG_TRY(cudaGetLastError());
    GDN_SEG_TRY(cudaEventRecord(ev_k1, stream));

    // pass 1: s0 from S0 (its outputs; h at s1's start), s1 from 0 (N), s1 with
    // V = 0 from the identity (M, a d_k-column state); the key side of s2 beside them
    FwdParams a0 = v0;
    a0.S_T = sH1;
    FwdParams an = v1;
    an.S0 = nullptr; an.o = nullptr; an.S_T = sN;
    FwdParams am = v1;
    am.v = nullptr; am.dv = p.dk; am.S0 = sI; am.o = nullptr; am.S_T = sM;
    GDN_SEG_TRY(cudaStreamWaitEvent(r0, ev_k1, 0));
    GDN_SEG_TRY(cudaStreamWaitEvent(r1, ev_k1, 0));
    GDN_SEG_TRY(cudaStreamWaitEvent(r2, ev_k1, 0));
    GDN_SEG_TRY(cudaStreamWaitEvent(side, ev_k1, 0));
    GDN_SEG_TRY(launch_k2_plain(a0, wsg[0], r0));
    GDN_SEG_TRY(launch_k2_plain(an, wsg[1], r1));
    GDN_SEG_TRY(launch_k2_plain(am, wsg[1], r2));
    GDN_SEG_TRY(launch_k1_plain(v2, wsg[2], side));
    GDN_SEG_TRY(cudaEventRecord(ev_h1, r0));
    GDN_SEG_TRY(cudaEventRecord(ev_n, r1));
    GDN_SEG_TRY(cudaEventRecord(ev_m, r2));
    GDN_SEG_TRY(cudaEventRecord(ev_k1b, side));

    // pass 2: s1 from h(s1 start); h(s2 start) = M h(s1 start) + N, then s2 from it
    FwdParams a1 = v1;
    a1.S0 = sH1; a1.S_T = nullptr;
    GDN_SEG_TRY(cudaStreamWaitEvent(r1, ev_h1, 0));
    GDN_SEG_TRY(launch_k2_plain(a1, wsg[1], r1));
    GDN_SEG_TRY(cudaEventRecord(ev_s1, r1));
    GDN_SEG_TRY(cudaStreamWaitEvent(r0, ev_n, 0));
    GDN_SEG_TRY(cudaStreamWaitEvent(r0, ev_m, 0));
    seg_compose_kernel<<<dim3(p.dk, p.H), 128, 0, r0>>>(sM, sH1, sN, sH2, p.dk, p.dv);
    GDN_SEG_TRY(cudaGetLastError());
    FwdParams a2 = v2;
    a2.S0 = sH2;    // S_T: the caller's (it may alias S0, which pass 1 has read)
    GDN_SEG_TRY(cudaStreamWaitEvent(r0, ev_k1b, 0));
    GDN_SEG_TRY(launch_k2_plain(a2, wsg[2], r0));
    GDN_SEG_TRY(cudaEventRecord(ev_s2, r0));

    // join: the caller's stream continues after both pass-2 runs
    GDN_SEG_TRY(cudaStreamWaitEvent(stream, ev_s1, 0));
    GDN_SEG_TRY(cudaStreamWaitEvent(stream, ev_s2, 0));
#undef GDN_SEG_TRY
    return cudaSuccess;
}

}  // namespace

bool tc_supports(const FwdParams &p, const char **why) {
    if (!p.io_bf16) { *why = "needs bf16 q/k/v"; return false; }
    if (p.general) {
        // the two-gate rule: the SIMT prep's matrices in fp16 for the chain kernel
        if (p.C != C) { *why = "two-gate rule: needs chunk 64"; return false; }
        if (p.mode == GDN_INV_NEUMANN_RESIDUAL) { *why = "two-gate rule: no residual correction"; return false; }
        if (p.precond > 1) {
            *why = "two-gate rule: preconditioner forms 2 and 3 (unbounded write keys) run on the SIMT kernel";
            return false;
        }
        if (p.dk != DK) { *why = "needs dk 128"; return false; }
        if (p.dv % DVS != 0) { *why = "needs dv a multiple of 64"; return false; }
        if (p.slices && p.dvs != DVS) { *why = "value slices must be 64 columns"; return false; }
        return true;
    }
    if (p.C != C && !(p.C == 2 * C && (p.mode == GDN_INV_NEUMANN || p.mode == GDN_INV_EXACT))) {
        *why = "needs chunk 64 (or 128, exact or with the masked series)";
        return false;
    }
    if (p.dk != DK) { *why = "needs dk 128"; return false; }
    if (p.dv % DVS != 0) { *why = "needs dv a multiple of 64"; return false; }
    if (p.mode != GDN_INV_EXACT && p.N > kNeumannMaxN) { *why = "Neumann N > 15"; return false; }
    if (p.slices && p.dvs != DVS) { *why = "value slices must be 64 columns"; return false; }
    return true;
}

int tc_default_slices(const FwdParams &p) { return p.dv / DVS; }

size_t tc_workspace_bytes(const FwdParams &p) {
    if (p.general) return gen_prep_workspace_bytes(p);
    const size_t nc = (size_t)(p.T + C - 1) / C;
    const size_t per = WS_CHUNK_BYTES + (p.C == 2 * C ? pair_stride(p.dv) * 4 : 0);
    return (size_t)p.B * p.H * nc * per + (p.segments == 3 ? seg_state_floats(p) * 4 : 0);
}

bool tc_segments_support(const FwdParams &p, const char **why) {
    if (p.B != 1) { *why = "sequence segments need B = 1"; return false; }
    if (p.general || p.C != C) { *why = "sequence segments: the scalar rule at chunk 64 only"; return false; }
    if ((p.T + C - 1) / C < 3) { *why = "sequence segments need at least 3 chunks"; return false; }
    return true;
}

int tc_auto_segments(const FwdParams &p) {
    const char *why = "";
    if (!tc_segments_support(p, &why)) return 1;
    // a long sequence whose chains fill under a third of the SMs: three chain runs
    // side by side in the first pass still fit in one wave
    const int NC = (p.T + C - 1) / C;
    return (NC >= kSegAutoMinChunks && 3 * p.H * (p.dv / DVS) <= kSMs) ? 3 : 1;
}

cudaError_t launch_tc(const FwdParams &p, void *workspace, cudaStream_t stream, const char **why) {
    const int NC = (p.T + C - 1) / C;
    if (p.segments == 3) {
        cudaError_t e = cudaFuncSetAttribute(keyside_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)K1_SMEM_RES);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(chain_kernel<K2_PLAIN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)K2Layout<K2_PLAIN>::SMEM);
        if (e == cudaSuccess) e = launch_tc_segments(p, workspace, stream);
        if (e != cudaSuccess) *why = "(sequence segments)";
        return e;
    }
    CUtensorMap mq, mk, mv, mt;
    if (p.general) {
        // the two-gate rule: the prep's fp16 rows, then the chain kernel (every
        // operand from the workspace through one map)
        const GenRows G = gen_rows(p.dv);
        if (!make_map_t(&mt, workspace, (size_t)p.B * p.H * NC * G.rows)) {
            *why = "(tensor map encoding failed)";
            return cudaErrorInvalidValue;
        }
        cudaError_t e = launch_gen_prep(p, workspace, stream);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(chain_kernel<K2_GEN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)K2Layout<K2_GEN>::SMEM);
        if (e != cudaSuccess) return e;
        K2Params k2{};
        k2.B = p.B; k2.T = p.T; k2.H = p.H; k2.dv = p.dv; k2.NC = NC;
        k2.S0 = p.S0; k2.o = p.o; k2.S_T = p.S_T; k2.o_bf16 = p.o_bf16;
        k2.gen_ws = reinterpret_cast<const uint8_t *>(workspace);
        k2.ws_rows = G.rows;
        chain_kernel<K2_GEN><<<dim3(p.slices, p.H, p.B), K2_THREADS, K2Layout<K2_GEN>::SMEM, stream>>>(mt, mt, mt,
                                                                                                      mt, k2);
        return cudaGetLastError();
    }
    if (!make_map_bthd(&mq, p.q, p.B, p.T, p.H, p.dk) || !make_map_bthd(&mk, p.k, p.B, p.T, p.H, p.dk) ||
        !make_map_bthd(&mv, p.v, p.B, p.T, p.H, p.dv) ||
        !make_map_t(&mt, workspace, (size_t)p.B * p.H * NC * WS_ROWS)) {
        *why = "(tensor map encoding failed)";
        return cudaErrorInvalidValue;
    }
    // The attribute belongs to the current device: set it on every launch (cheap)
    // rather than behind a process-wide flag that a second device would not share.
    // A 128-token chunk of the masked series runs as two 64-token halves ("pair"):
    // the second halves' band corners (a third kernel) go to the workspace after the
    // T matrices.
    const bool pair = p.C == 2 * C;
    float *pair_ws = pair ? reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) +
                                                      (size_t)p.B * p.H * NC * WS_CHUNK_BYTES)
                          : nullptr;
    {
        cudaError_t e = cudaFuncSetAttribute(keyside_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)K1_SMEM_RES);
        if (e != cudaSuccess) return e;
        e = pair ? cudaFuncSetAttribute(chain_kernel<K2_PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)K2Layout<K2_PAIR>::SMEM)
                 : cudaFuncSetAttribute(chain_kernel<K2_PLAIN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)K2Layout<K2_PLAIN>::SMEM);
        if (e != cudaSuccess) return e;
    }
    if (pair && NC / 2 > 0) {
        PairParams pp;
        pp.B = p.B; pp.T = p.T; pp.H = p.H; pp.dv = p.dv; pp.NC = NC; pp.N = p.N;
        pp.k = p.k; pp.v = p.v; pp.alpha = p.alpha; pp.beta = p.beta; pp.pair_ws = pair_ws;
        const dim3 grid(NC / 2, p.H, p.B);
        switch (p.N) {
#define GDN_PAIR_CASE(n) \
    case n: pair_corner_kernel<n><<<grid, PAIR_THREADS, 0, stream>>>(pp); break;
            GDN_PAIR_CASE(0) GDN_PAIR_CASE(1) GDN_PAIR_CASE(2) GDN_PAIR_CASE(3) GDN_PAIR_CASE(4)
            GDN_PAIR_CASE(5) GDN_PAIR_CASE(6) GDN_PAIR_CASE(7) GDN_PAIR_CASE(8) GDN_PAIR_CASE(9)
            GDN_PAIR_CASE(10) GDN_PAIR_CASE(11) GDN_PAIR_CASE(12) GDN_PAIR_CASE(13) GDN_PAIR_CASE(14)
            GDN_PAIR_CASE(15)
#undef GDN_PAIR_CASE
            default: *why = "(band N > 15 with chunk 128)"; return cudaErrorInvalidValue;
        }
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    K1Params k1;
    k1.B = p.B; k1.T = p.T; k1.H = p.H; k1.NC = NC;
    k1.alpha = p.alpha; k1.beta = p.beta;
    k1.ws = reinterpret_cast<uint8_t *>(workspace);
    k1.neumann = p.mode == GDN_INV_NEUMANN ? 1 : (p.mode == GDN_INV_NEUMANN_RESIDUAL ? 2 : 0);
    k1.N = p.N; k1.S = p.S;
    keyside_kernel<<<dim3(NC, p.H, p.B), K1_THREADS, k1.neumann == 2 ? K1_SMEM_RES : K1_SMEM, stream>>>(mq, mk, k1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    K2Params k2{};
    k2.ws_rows = WS_ROWS;
    k2.B = p.B; k2.T = p.T; k2.H = p.H; k2.dv = p.dv; k2.NC = NC;
    k2.alpha = p.alpha; k2.beta = p.beta; k2.S0 = p.S0; k2.o = p.o; k2.S_T = p.S_T;
    k2.pair_ws = pair_ws;
    k2.o_bf16 = p.o_bf16;
    if (pair)
        chain_kernel<K2_PAIR><<<dim3(p.slices, p.H, p.B), K2_THREADS, K2Layout<K2_PAIR>::SMEM, stream>>>(mq, mk, mv, mt,
                                                                                                  k2);
    else
        chain_kernel<K2_PLAIN><<<dim3(p.slices, p.H, p.B), K2_THREADS, K2Layout<K2_PLAIN>::SMEM, stream>>>(mq, mk, mv,
                                                                                                    mt, k2);
    return cudaGetLastError();
}

unsigned int tc_read_and_clear_error(cudaStream_t stream, cudaError_t *err) {
    unsigned int v = 0, zero = 0;
    *err = cudaStreamSynchronize(stream);
    if (*err != cudaSuccess) return 0;
    *err = cudaMemcpyFromSymbol(&v, g_tc_error, sizeof(v));
    if (*err == cudaSuccess && v) *err = cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(zero));
    return v;
}

}  // namespace gdn
