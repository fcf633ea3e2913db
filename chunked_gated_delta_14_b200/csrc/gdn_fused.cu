// Fused tensor-core forward of the chunkwise gated delta rule on sm_100a:
// one launch, one 2-CTA thread-block cluster per (batch, head), no scratch
// memory in HBM.
//
// The recurrence is S_t = S_{t-1} alpha_t (I - beta_t k_t k_t^T) +
// beta_t v_t k_t^T, o_t = S_t q_t.  Per chunk of C = 64 tokens, with h = S^T
// (d_k x d_v) the state at the chunk start, g_r = sum_{i<=r} log alpha_i:
//   L_ri = beta_r e^{g_r - g_i} (k_r . k_i) (i < r),  A = -L,  T = (I - A)^-1
//   U = T diag(beta) V,  W = T diag(beta e^g) K,  Delta = U - W h
//   O = diag(e^g) Q h + P Delta,  P_ri = (q_r . k_i) e^{g_r - g_i} (i <= r)
//   h <- e^{g_C} h + (diag(e^{g_C - g}) K)^T Delta
// The inverse T = (I - A)^-1 with A strictly lower is the step "Quando o 'Bom
// o Suficiente' e Otimo: Aproximacao de Inversao de Matriz Baseada Apenas em
// Multiplicacao para Gated DeltaNet Quantizado" (section "Declaracao do
// Problema") singles out; it is formed exactly (blocked inversion) or as the
// masked truncated Neumann series M^(N) (.) sum_{n<=N} A^n (section
// "Metodologia", items 1 and 2).
//
// CTA 0 of the cluster, the key side, walks the chunks of its head and does
// everything that does not depend on the state: one tcgen05 MMA forms
// [Q ; K] K^T (bf16, fp32 in TMEM); its epilogue gives the decayed causal
// scores P and L; T is inverted on the CUDA cores; T diag(beta) and
// T diag(beta e^g) go to fp16; a second MMA gives W = T diag(beta e^g) K.
// Two groups of four warps take alternate chunks.  Per chunk it ships
// [-W | T diag(beta) | P] (32 KB fp16) into the other CTA's shared memory
// with the bulk-copy engine (DSMEM, no multicast).
//
// CTA 1, the chain, holds the fp32 state h (128 x 128) in TMEM for the whole
// sequence.  Its TMA producer stages q, k, v; six warps convert them to the
// fp16 operands diag(e^g) Q, diag(e^{g_C - g}) K and V; one thread issues
// every MMA:
//   U:  X_n  = [T diag(beta) ; 0] V                    (lanes 0..63 U, 64..127 zero)
//   X:  X_n += [-W ; diag(e^g) Q] h16                  (lanes 0..63 Delta, 64..127 Q'h)
//   Z:  h   += (diag(e^{g_C - g}) K)^T Delta16
//   O:  X_n += [0 ; P] Delta16                        (lanes 64..127: O)
// Eight warps hold the state chain: h16 <- h and h <- e^{g_C} h (TMEM), Delta
// to fp16, and the output rows to HBM.  X_n rotates over three TMEM buffers
// so that the next chunk's U can run while this chunk's output is read.
//
// Every wait is bounded (about two seconds); a wait that gives up sets the
// CTA's abort flag, every role leaves its loop, in-flight copies and MMAs
// are drained, TMEM is freed and the error code is kept for
// gdn_device_check.  Both CTAs always meet at the two closing cluster
// barriers, so neither leaves while the other may still touch its shared
// memory.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "gdn_internal.cuh"
#include "gdn_tc_common.cuh"

namespace gdn {

__device__ unsigned int g_fused_error = 0;

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

constexpr int DV = 128;
constexpr int NTHREADS = 512;
constexpr unsigned long long kWait = 4000000000ull;   // ~2 s at the boost clock

// error codes (first one wins): key side 21.., chain side 41..
enum {
    E_K_Q = 21, E_K_GRAM, E_K_KFREE, E_K_KRECV, E_K_INV, E_K_LFULL, E_K_LFREE, E_K_TFULL, E_K_TFREE,
    E_C_SFREE = 41, E_C_SFULL, E_C_KFULL, E_C_CVT, E_C_HREADY, E_C_HSTORED, E_C_DDONE, E_C_XDONE,
    E_C_ZDONE, E_C_ODONE, E_C_XFREE, E_C_WDONE, E_C_WREADY
};

constexpr uint32_t IDESC_BF_KK = idesc_f16(128, 64, 1, 1, 0, 0);    // bf16 K-major x K-major, N 64
constexpr uint32_t IDESC_KM128 = idesc_f16(128, 128, 0, 0, 0, 1);   // fp16 K-major x MN-major, N 128
constexpr uint32_t IDESC_KM64 = idesc_f16(128, 64, 0, 0, 0, 1);     // fp16 K-major x MN-major, N 64
constexpr uint32_t IDESC_MM64 = idesc_f16(128, 64, 0, 0, 1, 1);     // fp16 MN-major x MN-major, N 64

constexpr uint32_t PARB = (sizeof(ChunkParams) + 15) & ~15u;
constexpr uint32_t MAT = 64 * LSTR * 4;                 // one 64 x LSTR fp32 matrix

// ------------------------------------------------ key CTA shared memory
// stage st (chunks of parity st): [Q0 | K0 | Q1 | K1], 8 KB each (64 rows of one
// 64-column box, 128-byte swizzle).  Send buffer sb (chunk m: sb = m % 3):
// [T diag(beta e^g) | T diag(beta) | P], fp16.  L and T: fp32, two each.
constexpr uint32_t K_QK = 0;
constexpr uint32_t K_SND = 65536;
constexpr uint32_t SNDB = 24576;
constexpr uint32_t SND_TBG = 0, SND_TB = 8192, SND_P = 16384;
constexpr uint32_t K_L = K_SND + 3 * SNDB;
constexpr uint32_t K_T = K_L + 2 * MAT;
constexpr uint32_t K_PAR = K_T + 2 * MAT;
constexpr uint32_t K_BAR = K_PAR + 3 * PARB;
enum {
    KB_QFULL = 0, KB_GRAM = 2, KB_LFULL = 4, KB_LFREE = 6, KB_TFULL = 8, KB_TFREE = 10, KB_INV = 12,
    KB_KFREE = 13, KB_KRECV = 15, KB_N = 18
};
constexpr uint32_t K_MISC = K_BAR + KB_N * 8;          // tmem slot, abort flag, stage sync slots
constexpr uint32_t K_END = K_MISC + 64;

// ---------------------------------------------- chain CTA shared memory
// slot s (chunks of parity s), 88 KB:
//   -W0 | Q0 | -W1 | Q1 | K0 | K1 | V0 | V1 | T diag(beta) | zero | P
// -W box kb sits right before Q box kb so that [-W ; Q'] is one 128-row MMA
// operand; T diag(beta) before the zero tile and the zero tile before P make
// [T diag(beta) ; 0] and [0 ; P].  Delta16 overwrites V once U has read it.
constexpr uint32_t SLOT = 90112;
constexpr uint32_t S_MW0 = 0, S_Q0 = 8192, S_MW1 = 16384, S_Q1 = 24576, S_K0 = 32768, S_K1 = 40960;
constexpr uint32_t S_V0 = 49152, S_V1 = 57344, S_TB = 65536, S_ZERO = 73728, S_P = 81920;
constexpr uint32_t C_SLOT = 0;
constexpr uint32_t C_HS = 2 * SLOT;                    // h16: two 64-column boxes of 128 rows
constexpr uint32_t C_PAR = C_HS + 32768;               // gate ring of 4
constexpr uint32_t C_BAR = C_PAR + 4 * PARB;
// per value half j (columns 64 j .. 64 j + 63): XDONE / ODONE [buffer][half],
// HREADY / HSTORED / DDONE / ZDONE [half]
enum {
    CB_SFULL = 0, CB_SFREE = 2, CB_KFULL = 4, CB_CVT = 6, CB_XDONE = 8, CB_ODONE = 12, CB_XFREE = 16,
    CB_HREADY = 18, CB_HSTORED = 20, CB_DDONE = 22, CB_ZDONE = 24, CB_WDONE = 26, CB_WREADY = 27, CB_UDONE = 28,
    CB_N = 29
};
constexpr uint32_t C_MISC = C_BAR + CB_N * 8;          // tmem slot, abort, sent counts, sync slots
constexpr uint32_t C_END = C_MISC + 64;

constexpr uint32_t SMEM_USED = (K_END > C_END ? K_END : C_END);
constexpr uint32_t FUSED_SMEM = SMEM_USED + 1024;      // + base alignment slack
static_assert(FUSED_SMEM <= 232448, "shared memory budget of one sm_100 block");
static_assert(K_SND + 3 * SNDB <= K_L && (K_L & 15) == 0 && (K_BAR & 7) == 0, "key layout");
static_assert((C_HS & 1023) == 0 && (K_L & 15) == 0, "alignment");

// chain TMEM: h (128 columns), two X buffers, W; key TMEM: Gram x 2, inverse merge
constexpr uint32_t TM_H = 0, TM_X = 128, TM_WC = 384;
constexpr uint32_t TM_G = 0, TM_INV = 128;

struct FusedParams {
    int B, T, H, NC;
    const float *alpha, *beta, *S0;
    void *o;
    float *S_T;
    int o_bf16;
    int neumann, N;
    float *dbg_T;       // inspection: the fp32 T of chunk dbg_n of (dbg_b, dbg_h), or NULL
    int dbg_b, dbg_h, dbg_n;
};

// Group wait: lane 0 of the polling warp waits, the group meets at a named
// barrier, and the abort state read once by that lane decides for everyone
// (two alternating slots, see sync note below).
struct GroupSync {
    volatile int *slots;
    int cnt;
    int id, n;
    bool poller;      // lane 0 of the polling warp
    bool pwarp;       // the polling warp
};

__device__ __forceinline__ bool group_wait(GroupSync &gs, uint64_t *bar, uint32_t parity, volatile int *abort,
                                           int code, bool cluster_scope) {
    const int k = gs.cnt++ & 1;
    if (gs.pwarp) {
        if (gs.poller) {
            if (cluster_scope) mbar_wait_cluster(bar, parity, abort, code, kWait);
            else mbar_wait(bar, parity, abort, code, kWait);
            gs.slots[k] = *abort;
        }
        __syncwarp();
    }
    named_bar(gs.id, gs.n);
    const bool ok = gs.slots[k] == 0;
    if (ok && !gs.poller) {
        if (cluster_scope) mbar_try_wait_cluster(bar, parity);
        else mbar_try_wait(bar, parity);
    }
    return ok;
}
// Slot k written before barrier j is read right after it; it is written again
// only at barrier j + 2, after every thread has passed barrier j + 1.

// One warp waits on its own: lane 0 polls, the result is broadcast.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort, int code,
                                          bool spin) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0)
        ok = spin ? mbar_wait_spin(bar, parity, abort, code, kWait) : mbar_wait(bar, parity, abort, code, kWait);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) mbar_try_wait(bar, parity);
    return ok != 0;
}

// =================================================================== key CTA
// A pipeline of three warp groups, one chunk in each stage:
//   A (warps 0..3):   q, k tiles (TMA), gate scan, [Q ; K] K^T (MMA), and from
//                     it the decayed scores P (fp16, send buffer) and L (fp32)
//   B (warps 4..11):  T = (I + L)^-1, or the masked truncated Neumann series
//   C (warps 12..15): T diag(beta), T diag(beta e^g) (fp16), then the copy of
//                     [T diag(beta e^g) | T diag(beta) | P] into the chain CTA
// Stages hand over through mbarriers: A -> B (L full / free), B -> C (T full /
// free); a send buffer is reused once the chain CTA has received its copy.

__device__ __forceinline__ void key_cta(uint8_t *sm, const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                        const FusedParams &p, int b, int h, uint32_t tmem, volatile int *abort) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NC = p.NC;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + K_BAR);
    auto Lbuf = [&](int m) { return reinterpret_cast<float *>(sm + K_L + (m & 1) * MAT); };
    auto Tbuf = [&](int m) { return reinterpret_cast<float *>(sm + K_T + (m & 1) * MAT); };
    auto par_of = [&](int m) { return reinterpret_cast<ChunkParams *>(sm + K_PAR + (m % 3) * PARB); };
    auto snd_of = [&](int m) { return sm + K_SND + (m % 3) * SNDB; };

    if (warp < 4) {
        // ------------------------------------------------------------ stage A
        const int sp = warp;
        const uint32_t lane_base = (uint32_t)(32 * sp) << 16;
        GroupSync gs{reinterpret_cast<volatile int *>(sm + K_MISC + 16), 0, 1, 128, tid == 0, warp == 0};
        const bool leader = (tid == 0);
        auto load_qk = [&](int m) {
            uint64_t *fb = &bars[KB_QFULL + (m & 1)];
            uint8_t *st = sm + K_QK + (m & 1) * 32768;
            mbar_arrive_expect_tx(fb, 32768);
            tma_load_4d(st, tm_q, fb, 0, h, m * C, b);
            tma_load_4d(st + 8192, tm_k, fb, 0, h, m * C, b);
            tma_load_4d(st + 16384, tm_q, fb, 64, h, m * C, b);
            tma_load_4d(st + 24576, tm_k, fb, 64, h, m * C, b);
        };
        int q_out[2] = {-1, -1};                   // leader: phases of loads not yet consumed
        if (leader) {
            tma_prefetch_desc(tm_q);
            tma_prefetch_desc(tm_k);
            for (int m = 0; m < 2 && m < NC; ++m) { load_qk(m); q_out[m] = 0; }
        }
        int pend = -1, pend_par = 0;
        for (int m = 0; m < NC; ++m) {
            const int st = m & 1;
            uint8_t *qk = sm + K_QK + st * 32768;
            const uint32_t tG = tmem + TM_G + 64 * st;
            ChunkParams *par = par_of(m);
            uint8_t *snd = snd_of(m);
            float *Lb = Lbuf(m);
            // the send buffer (and the gate slot) of chunk m - 3 are free once the
            // chain CTA has received that chunk
            if (m >= 3 && !group_wait(gs, &bars[KB_KRECV + m % 3], ((m - 3) / 3) & 1, abort, E_K_KRECV, true))
                break;
            if (warp == 1) {
                float a0, a1, b0, b1;
                tc::fetch_gates(p.alpha, p.beta, b, p.T, p.H, h, m * C, lane, true, a0, a1, b0, b1);
                tc::scan_gates(par, a0, a1, b0, b1, lane, min(C, p.T - m * C));
            }
            if (!group_wait(gs, &bars[KB_QFULL + st], (m >> 1) & 1, abort, E_K_Q, false)) break;
            if (leader) {
                q_out[st] = -1;
                tc_fence_after();
                const uint32_t a0 = smem_u32(qk);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    umma_f16_ss(tG, sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(a0 + off + 8192, 16, 1024),
                                IDESC_BF_KK, kk > 0);
                }
                umma_commit(&bars[KB_GRAM + st]);
                pend = KB_GRAM + st; pend_par = (m >> 1) & 1;
            }
            __syncwarp();
            // stage B has read L of chunk m - 2
            if (m >= 2 && !group_wait(gs, &bars[KB_LFREE + st], ((m - 2) >> 1) & 1, abort, E_K_LFREE, false))
                break;
            if (!group_wait(gs, &bars[KB_GRAM + st], (m >> 1) & 1, abort, E_K_GRAM, false)) break;
            pend = -1;
            if (leader && m + 2 < NC) { load_qk(m + 2); q_out[st] = ((m + 2) >> 1) & 1; }   // q, k are read
            tc_fence_after();
            // sub-partitions 0, 1: rows of Q K^T -> P; sub-partitions 2, 3: rows of K K^T -> L
            const int rb = sp & 1, r = 32 * rb + lane;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t xr[32];
                float gam[32];
                const bool live = hf <= rb;
                if (live) {
                    tmem_ld32(tG + lane_base + 32 * hf, xr);
                    tc::decay_row(par, r, hf, hf == rb, gam);
                    tmem_wait_ld();
                }
                if (sp < 2) {
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        uint4 u = make_uint4(0u, 0u, 0u, 0u);
                        if (live) {
                            const int j = 8 * jj;
                            u.x = pack_h2(gam[j] * __uint_as_float(xr[j]), gam[j + 1] * __uint_as_float(xr[j + 1]));
                            u.y = pack_h2(gam[j + 2] * __uint_as_float(xr[j + 2]), gam[j + 3] * __uint_as_float(xr[j + 3]));
                            u.z = pack_h2(gam[j + 4] * __uint_as_float(xr[j + 4]), gam[j + 5] * __uint_as_float(xr[j + 5]));
                            u.w = pack_h2(gam[j + 6] * __uint_as_float(xr[j + 6]), gam[j + 7] * __uint_as_float(xr[j + 7]));
                        }
                        *reinterpret_cast<uint4 *>(snd + SND_P + sw128_off(r, 4 * hf + jj)) = u;
                    }
                } else {
                    float *Lr = Lb + r * LSTR + 32 * hf;
                    const float br = par->bet[r];
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const int i = 32 * hf + j;
                        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (live) {
                            v.x = (i + 0 < r) ? br * gam[j + 0] * __uint_as_float(xr[j + 0]) : 0.f;
                            v.y = (i + 1 < r) ? br * gam[j + 1] * __uint_as_float(xr[j + 1]) : 0.f;
                            v.z = (i + 2 < r) ? br * gam[j + 2] * __uint_as_float(xr[j + 2]) : 0.f;
                            v.w = (i + 3 < r) ? br * gam[j + 3] * __uint_as_float(xr[j + 3]) : 0.f;
                        }
                        *reinterpret_cast<float4 *>(Lr + j) = v;
                    }
                }
            }
            fence_proxy_async_smem();     // P is read by the bulk copy
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[KB_LFULL + st]);
        }
        if (leader) {
            // error path: nothing of this stage may still run when the block exits
            if (pend >= 0) mbar_wait_drain(&bars[pend], pend_par, kWait);
            for (int i = 0; i < 2; ++i)
                if (q_out[i] >= 0) mbar_wait_drain(&bars[KB_QFULL + i], q_out[i], kWait);
        }
        __syncwarp();
        return;
    }

    if (warp < 12) {
        // ------------------------------------------------------------ stage B
        const int bt = tid - 128;                 // 0..255
        const int wl = warp - 4;
        GroupSync gs{reinterpret_cast<volatile int *>(sm + K_MISC + 24), 0, 2, 256, bt == 0, wl == 0};
        const bool leader = (bt == 0);
        const uint32_t tI = tmem + TM_INV;
        // T's blocks above the diagonal stay zero for the whole sequence
        for (int i = bt; i < 2 * 64 * LSTR; i += 256) reinterpret_cast<float *>(sm + K_T)[i] = 0.f;
        named_bar(gs.id, 256);
        int pend = -1, pend_par = 0;
        for (int m = 0; m < NC; ++m) {
            const int lb = m & 1;
            float *Lb = Lbuf(m), *Tb = Tbuf(m);
            uint8_t *snd = snd_of(m);
            float *Yb = reinterpret_cast<float *>(snd + SND_TBG);   // scratch until stage C writes there
            if (!group_wait(gs, &bars[KB_LFULL + lb], (m >> 1) & 1, abort, E_K_LFULL, false)) break;
            if (m >= 2 && !group_wait(gs, &bars[KB_TFREE + lb], ((m - 2) >> 1) & 1, abort, E_K_TFREE, false))
                break;
            bool fail = false;
            if (!p.neumann) {
                // the 16 x 16 diagonal blocks and the 16 -> 32 merges on the CUDA
                // cores, the 32 -> 64 merge T10 = -T11 L10 T00 as two MMAs (fp16
                // operands, fp32 accumulate; the rounding stays below that of the
                // fp16 copies of T that the WY products use)
                tc::invert_exact_to32(Lb, Tb, Yb, bt, gs.id);
                uint8_t *a1 = snd + SND_TBG, *b1 = snd + SND_TBG + 4096;   // rows: L10 | T rows 0..31
                uint8_t *a2 = snd + SND_TB, *b2 = snd + SND_TB + 4096;     // rows: -T11 | Y
                {
                    const int u = bt & 127, r = u >> 2, j = u & 3;
                    const float *src = bt < 128 ? Lb + (32 + r) * LSTR + 8 * j : Tb + (32 + r) * LSTR + 32 + 8 * j;
                    const float sg = bt < 128 ? 1.f : -1.f;
                    const float4 x0 = *reinterpret_cast<const float4 *>(src);
                    const float4 x1 = *reinterpret_cast<const float4 *>(src + 4);
                    *reinterpret_cast<uint4 *>((bt < 128 ? a1 : a2) + sw128_off(r, j)) =
                        make_uint4(pack_h2(sg * x0.x, sg * x0.y), pack_h2(sg * x0.z, sg * x0.w),
                                   pack_h2(sg * x1.x, sg * x1.y), pack_h2(sg * x1.z, sg * x1.w));
                    const int k = bt >> 3, jb = bt & 7;
                    const float *tr = Tb + k * LSTR + 8 * jb;
                    const float4 y0 = *reinterpret_cast<const float4 *>(tr);
                    const float4 y1 = *reinterpret_cast<const float4 *>(tr + 4);
                    *reinterpret_cast<uint4 *>(b1 + sw128_off(k, jb)) =
                        make_uint4(pack_h2(y0.x, y0.y), pack_h2(y0.z, y0.w), pack_h2(y1.x, y1.y), pack_h2(y1.z, y1.w));
                }
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar(gs.id, 256);
#pragma unroll 1
                for (int step = 0; step < 2 && !fail; ++step) {
                    if (leader) {
                        // step 0: Y = [L10 ; any 96 rows] T[0..31, 0..63] (columns 32..63 of T are 0)
                        // step 1: T10 = [-T11 ; any 96 rows] Y (B2 columns 32..63 are not used)
                        tc_fence_after();
                        const uint32_t aa = smem_u32(step ? a2 : a1), bb = smem_u32(step ? b2 : b1);
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk)
                            umma_f16_ss(tI, sdesc_sw128(aa + kk * 32, 16, 1024), sdesc_sw128(bb + kk * 2048, 16384, 1024),
                                        IDESC_KM64, kk > 0);
                        umma_commit(&bars[KB_INV]);
                        pend = KB_INV; pend_par = step;
                    }
                    __syncwarp();
                    if (!group_wait(gs, &bars[KB_INV], step, abort, E_K_INV, false)) { fail = true; break; }
                    pend = -1;
                    tc_fence_after();
                    if (wl == 0) {
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
                    named_bar(gs.id, 256);
                }
            } else if (p.N <= 15) {
                tc::invert_neumann(Lb, Tb, Yb, bt, p.N, gs.id);
            } else {
                // a long series (test sizes): dense steps by the first 128 threads
                if (bt < 128) tc::invert_neumann128(Lb, Tb, Yb, bt, p.N, 4);
                named_bar(gs.id, 256);
            }
            if (fail) break;
            if (p.dbg_T && m == p.dbg_n && b == p.dbg_b && h == p.dbg_h)
                for (int i = bt; i < 64 * 64; i += 256) p.dbg_T[i] = Tb[(i >> 6) * LSTR + (i & 63)];
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[KB_LFREE + lb]);
                mbar_arrive(&bars[KB_TFULL + lb]);
            }
        }
        if (leader && pend >= 0) mbar_wait_drain(&bars[pend], pend_par, kWait);
        __syncwarp();
        return;
    }

    // ---------------------------------------------------------------- stage C
    const int ct = tid - 384;                     // 0..127
    GroupSync gs{reinterpret_cast<volatile int *>(sm + K_MISC + 32), 0, 3, 128, ct == 0, warp == 12};
    const bool leader = (ct == 0);
    int sent[2] = {0, 0};
    for (int m = 0; m < NC; ++m) {
        const int s = m & 1;
        const float *Tb = Tbuf(m);
        const ChunkParams *par = par_of(m);
        uint8_t *snd = snd_of(m);
        if (!group_wait(gs, &bars[KB_TFULL + s], (m >> 1) & 1, abort, E_K_TFULL, false)) break;
        {
            // T diag(beta), T diag(beta e^g) -> fp16; thread: row rr, 32 columns
            const int rr = ct >> 1, half = ct & 1;
            const float *Tr = Tb + rr * LSTR + 32 * half;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c8 = 4 * half + j;
                float sb[8], sg[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int col = 8 * c8 + e;
                    sb[e] = Tr[8 * j + e] * par->bet[col];
                    sg[e] = sb[e] * par->eg[col];
                }
                *reinterpret_cast<uint4 *>(snd + SND_TB + sw128_off(rr, c8)) =
                    make_uint4(pack_h2(sb[0], sb[1]), pack_h2(sb[2], sb[3]), pack_h2(sb[4], sb[5]), pack_h2(sb[6], sb[7]));
                *reinterpret_cast<uint4 *>(snd + SND_TBG + sw128_off(rr, c8)) =
                    make_uint4(pack_h2(sg[0], sg[1]), pack_h2(sg[2], sg[3]), pack_h2(sg[4], sg[5]), pack_h2(sg[6], sg[7]));
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[KB_TFREE + s]);
        // the chain has finished chunk m - 2: its slot s may be overwritten
        if (m >= 2) {
            if (!group_wait(gs, &bars[KB_KFREE + s], ((m - 2) >> 1) & 1, abort, E_K_KFREE, true)) break;
        } else {
            named_bar(gs.id, 128);
        }
        if (leader) {
            const uint32_t kf = mapa_shared(smem_u32(sm + C_BAR + 8 * (CB_KFULL + s)), 1);
            const uint32_t sl = mapa_shared(smem_u32(sm + C_SLOT + s * SLOT), 1);
            mbar_arrive_expect_tx_remote(kf, 24576);
            bulk_copy_to_peer(sl + S_MW0, snd + SND_TBG, 8192, kf);
            bulk_copy_to_peer(sl + S_TB, snd + SND_TB, 8192, kf);
            bulk_copy_to_peer(sl + S_P, snd + SND_P, 8192, kf);
        }
        __syncwarp();
        ++sent[s];
    }
    // tell the chain CTA how many chunks were shipped into each slot
    if (leader) {
        st_peer_u32(mapa_shared(smem_u32(sm + C_MISC + 8), 1), (uint32_t)sent[0]);
        st_peer_u32(mapa_shared(smem_u32(sm + C_MISC + 12), 1), (uint32_t)sent[1]);
    }
    __syncwarp();
}

// ================================================================= chain CTA

__device__ __forceinline__ void chain_cta(uint8_t *sm, const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                          const CUtensorMap *tm_v, const FusedParams &p, int b, int h,
                                          uint32_t tmem, volatile int *abort) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NC = p.NC, T = p.T, H = p.H;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + C_BAR);
    ChunkParams *cpar = reinterpret_cast<ChunkParams *>(sm + C_PAR);
    auto slot = [&](int s) { return sm + C_SLOT + s * SLOT; };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer: q, k, v
        if (lane == 0) {
            tma_prefetch_desc(tm_q);
            tma_prefetch_desc(tm_k);
            tma_prefetch_desc(tm_v);
            const uint32_t peer_kfree = mapa_shared(smem_u32(sm + K_BAR + 8 * KB_KFREE), 0);
            int issued = 0;
            for (int n = 0; n < NC; ++n) {
                const int s = n & 1;
                if (n >= 2) {
                    if (!mbar_wait(&bars[CB_SFREE + s], ((n - 2) >> 1) & 1, abort, E_C_SFREE, kWait)) break;
                    // every MMA of chunk n - 2 is complete: its key-side tiles are free
                    mbar_arrive_remote(peer_kfree + 8 * s);
                }
                uint64_t *fb = &bars[CB_SFULL + s];
                uint8_t *st = slot(s);
                mbar_arrive_expect_tx(fb, 49152);
                const int t0 = n * C;
                tma_load_4d(st + S_Q0, tm_q, fb, 0, h, t0, b);
                tma_load_4d(st + S_Q1, tm_q, fb, 64, h, t0, b);
                tma_load_4d(st + S_K0, tm_k, fb, 0, h, t0, b);
                tma_load_4d(st + S_K1, tm_k, fb, 64, h, t0, b);
                tma_load_4d(st + S_V0, tm_v, fb, 0, h, t0, b);
                tma_load_4d(st + S_V1, tm_v, fb, 64, h, t0, b);
                issued = n + 1;
            }
            for (int n = issued - 2 < 0 ? 0 : issued - 2; n < issued; ++n)
                mbar_wait_drain(&bars[CB_SFULL + (n & 1)], (n >> 1) & 1, kWait);
        }
        __syncwarp();
        return;
    }

    if (warp == 1) {
        // ------------------------------------------------ MMA issue (one thread)
        if (lane == 0) {
            const uint32_t hs = smem_u32(sm + C_HS);
            auto xbuf = [&](int n) { return tmem + TM_X + 128u * (uint32_t)(n & 1); };
            const uint32_t peer_krecv = mapa_shared(smem_u32(sm + K_BAR + 8 * KB_KRECV), 0);
            // W(n) = [T diag(beta e^g) ; Q'0] K16 once the key side's tiles and the
            // conversion of chunk n are in (lanes 64..127 of W are not used)
            auto w_ready = [&](int n) {
                return mbar_try_wait_cluster(&bars[CB_KFULL + (n & 1)], (n >> 1) & 1) &&
                       mbar_try_wait(&bars[CB_CVT + (n & 1)], (n >> 1) & 1);
            };
            auto w_wait = [&](int n) {
                return mbar_wait_cluster(&bars[CB_KFULL + (n & 1)], (n >> 1) & 1, abort, E_C_KFULL, kWait) &&
                       mbar_wait(&bars[CB_CVT + (n & 1)], (n >> 1) & 1, abort, E_C_CVT, kWait);
            };
            auto w_issue = [&](int n) {
                // the key side's copy of chunk n has landed: its send buffer is free
                mbar_arrive_remote(peer_krecv + 8 * (n % 3));
                tc_fence_after();
                const uint32_t st = smem_u32(slot(n & 1));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16_ss(tmem + TM_WC, sdesc_sw128(st + S_MW0 + kk * 32, 16, 1024),
                                sdesc_sw128(st + S_K0 + kk * 2048, 8192, 1024), IDESC_KM128, kk > 0);
                umma_commit(&bars[CB_WDONE]);
            };
            // U(n): X_n = [T diag(beta) ; 0] V
            auto u_issue = [&](int n) {
                tc_fence_after();
                const uint32_t st = smem_u32(slot(n & 1));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16_ss(xbuf(n), sdesc_sw128(st + S_TB + kk * 32, 16, 1024),
                                sdesc_sw128(st + S_V0 + kk * 2048, 8192, 1024), IDESC_KM128, kk > 0);
            };
            int pend = -1, pend_par = 0;
            int cons[2] = {0, 0};                 // key-side shipments consumed, per slot
            int nu = 0;                           // U commits (on a barrier only the error path waits for)
            bool ok = NC > 0 && w_wait(0);
            if (ok) {
                w_issue(0);
                u_issue(0);
                umma_commit(&bars[CB_UDONE]);
                cons[0] = 1; pend = CB_UDONE; pend_par = nu++ & 1;
            }
            for (int n = 0; ok && n < NC; ++n) {
                const int s = n & 1, xb = n & 1;
                const uint32_t par2 = (n >> 1) & 1;
                const uint32_t st = smem_u32(slot(s));
                // -W and K' of chunk n are in shared memory
                if (!mbar_wait(&bars[CB_WREADY], n & 1, abort, E_C_WREADY, kWait)) break;
                // X(n), one value half at a time: [-W ; Q'] h16_j onto U
                bool fail = false;
#pragma unroll 1
                for (int j = 0; j < 2; ++j) {
                    if (!mbar_wait_spin(&bars[CB_HREADY + j], n & 1, abort, E_C_HREADY, kWait)) { fail = true; break; }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_f16_ss(xbuf(n) + 64 * j, sdesc_sw128(st + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                                    sdesc_sw128(hs + 16384 * j + kk * 2048, 16384, 1024), IDESC_KM64, 1);
                    umma_commit(&bars[CB_XDONE + 2 * xb + j]);
                    pend = CB_XDONE + 2 * xb + j; pend_par = par2;
                }
                if (fail) break;
                // W(n+1) while the Delta epilogue runs (the tensor pipe is idle then);
                // U(n+1) only after Z(n), O(n): an MMA issue blocks while earlier MMAs
                // drain, so anything ahead of Z would delay the state chain
                bool w_next = n + 1 >= NC;
                if (!w_next && w_ready(n + 1)) { w_issue(n + 1); w_next = true; ++cons[(n + 1) & 1]; }
                // per half: Z(n) h_j += K'^T Delta16_j;  O(n) X_n,j += [0 ; P] Delta16_j
#pragma unroll 1
                for (int j = 0; j < 2; ++j) {
                    if (!mbar_wait_spin(&bars[CB_DDONE + j], n & 1, abort, E_C_DDONE, kWait)) { fail = true; break; }
                    if (!mbar_wait_spin(&bars[CB_HSTORED + j], n & 1, abort, E_C_HSTORED, kWait)) { fail = true; break; }
                    tc_fence_after();
                    const uint32_t dj = st + S_V0 + 8192 * j;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ss(tmem + TM_H + 64 * j, sdesc_sw128(st + S_K0 + kk * 2048, 8192, 1024),
                                    sdesc_sw128(dj + kk * 2048, 8192, 1024), IDESC_MM64, 1);
                    umma_commit(&bars[CB_ZDONE + j]);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16_ss(xbuf(n) + 64 * j, sdesc_sw128(st + S_ZERO + kk * 32, 16, 1024),
                                    sdesc_sw128(dj + kk * 2048, 8192, 1024), IDESC_KM64, 1);
                    umma_commit(&bars[CB_ODONE + 2 * xb + j]);
                    pend = CB_ODONE + 2 * xb + j; pend_par = par2;
                }
                if (fail) break;
                umma_commit(&bars[CB_SFREE + s]);
                pend = CB_SFREE + s; pend_par = par2;
                if (n + 1 < NC) {
                    if (!w_next) {
                        if (!w_wait(n + 1)) break;
                        w_issue(n + 1);
                        ++cons[(n + 1) & 1];
                    }
                    // X buffer (n+1) & 1 is free once the output rows of chunk n - 1 are read
                    if (n >= 1 && !mbar_wait(&bars[CB_XFREE + ((n + 1) & 1)], ((n - 1) >> 1) & 1, abort, E_C_XFREE, kWait))
                        break;
                    u_issue(n + 1);
                    umma_commit(&bars[CB_UDONE]);
                    pend = CB_UDONE; pend_par = nu++ & 1;
                }
            }
            // error path: no MMA may still run when TMEM is released
            if (pend >= 0 && *abort) mbar_wait_drain(&bars[pend], pend_par, kWait);
            reinterpret_cast<volatile uint32_t *>(sm + C_MISC)[6] = (uint32_t)cons[0];
            reinterpret_cast<volatile uint32_t *>(sm + C_MISC)[7] = (uint32_t)cons[1];
        }
        __syncwarp();
        return;
    }

    if (warp == 2 || warp == 3 || warp >= 12) {
        // ---------------------------------------- operand conversion (6 warps)
        // (a) q -> Q' = diag(e^g) Q, k -> K16, v -> V16 (fp16, in place);
        // (b) once W(n) is in TMEM: -W -> fp16 over T diag(beta e^g) (warps 12, 13:
        //     TMEM lanes 0..63) and K16 -> K' = diag(e^{g_C - g}) K in place
        const int cvi = (warp < 4 ? warp - 2 : warp - 10) * 32 + lane;   // 0..191
        const int sp = warp & 3;
        GroupSync gs{reinterpret_cast<volatile int *>(sm + C_MISC + 16), 0, 3, 192, warp == 2 && lane == 0,
                     warp == 2};
        float ga0 = 1.f, ga1 = 1.f, gb0 = 0.f, gb1 = 0.f;
        if (warp == 2) tc::fetch_gates(p.alpha, p.beta, b, T, H, h, 0, lane, true, ga0, ga1, gb0, gb1);
        for (int n = 0; n < NC; ++n) {
            const int s = n & 1;
            ChunkParams *par = &cpar[n & 3];
            if (warp == 2) {
                tc::scan_gates(par, ga0, ga1, gb0, gb1, lane, min(C, T - n * C));
                tc::fetch_gates(p.alpha, p.beta, b, T, H, h, (n + 1) * C, lane, n + 1 < NC, ga0, ga1, gb0, gb1);
            }
            if (!group_wait(gs, &bars[CB_SFULL + s], (n >> 1) & 1, abort, E_C_SFULL, false)) break;
            uint8_t *st = slot(s);
#pragma unroll 4
            for (int j = 0; j < 16; ++j) {
                const int idx = cvi + 192 * j;               // 16-byte chunk of Q0 Q1 K0 K1 V0 V1
                const int tile = idx >> 9, u = idx & 511, row = u >> 3;
                const uint32_t off = tile == 0 ? S_Q0 : tile == 1 ? S_Q1 : tile == 2 ? S_K0
                                   : tile == 3 ? S_K1 : tile == 4 ? S_V0 : S_V1;
                const float sc = tile < 2 ? par->eg[row] : 1.f;
                uint8_t *addr = st + off + (u << 4);
                uint4 w = *reinterpret_cast<uint4 *>(addr);
                const float2 f0 = unpack_bf2(w.x), f1 = unpack_bf2(w.y), f2 = unpack_bf2(w.z), f3 = unpack_bf2(w.w);
                w.x = pack_h2(f0.x * sc, f0.y * sc);
                w.y = pack_h2(f1.x * sc, f1.y * sc);
                w.z = pack_h2(f2.x * sc, f2.y * sc);
                w.w = pack_h2(f3.x * sc, f3.y * sc);
                *reinterpret_cast<uint4 *>(addr) = w;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[CB_CVT + s]);
            // (b)
            if (!group_wait(gs, &bars[CB_WDONE], n & 1, abort, E_C_WDONE, false)) break;
            tc_fence_after();
            if (warp >= 12 && sp < 2) {
                const uint32_t lb = (uint32_t)(32 * sp) << 16;
                const int r = 32 * sp + lane;
                float x[64];
                tmem_ld64(tmem + TM_WC + lb, x);
#pragma unroll
                for (int j = 0; j < 64; ++j) x[j] = -x[j];
                st_row_f16(st + S_MW0, r, x);
                tmem_ld64(tmem + TM_WC + lb + 64, x);
#pragma unroll
                for (int j = 0; j < 64; ++j) x[j] = -x[j];
                st_row_f16(st + S_MW1, r, x);
            }
#pragma unroll 2
            for (int j = 0; j < 6; ++j) {
                const int idx = cvi + 192 * j;               // 16-byte chunk of K0 K1 (1024 of them)
                if (idx < 1024) {
                    const int u = idx & 511;
                    uint8_t *addr = st + ((idx >> 9) ? S_K1 : S_K0) + (u << 4);
                    const float sc = par->egc[u >> 3];
                    uint4 w = *reinterpret_cast<uint4 *>(addr);
                    const float2 f0 = tc::unpack_h2(w.x), f1 = tc::unpack_h2(w.y), f2 = tc::unpack_h2(w.z),
                                 f3 = tc::unpack_h2(w.w);
                    w.x = pack_h2(f0.x * sc, f0.y * sc);
                    w.y = pack_h2(f1.x * sc, f1.y * sc);
                    w.z = pack_h2(f2.x * sc, f2.y * sc);
                    w.w = pack_h2(f3.x * sc, f3.y * sc);
                    *reinterpret_cast<uint4 *>(addr) = w;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[CB_WREADY]);
        }
        return;
    }

    // -------------------------------------------- state chain (warps 4..11)
    const int sp = warp & 3, hf = (warp - 4) >> 2;
    const uint32_t lb = (uint32_t)(32 * sp) << 16;
    const int r = 32 * sp + lane;                  // TMEM lane = key row of h = row of X
    const size_t bh = (size_t)b * H + h;
    uint8_t *hs = sm + C_HS + hf * 16384;
    {
        float x[64];
#pragma unroll
        for (int j = 0; j < 64; j += 4) {
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (p.S0) v = *reinterpret_cast<const float4 *>(p.S0 + (bh * DK + r) * DV + 64 * hf + j);
            x[j] = v.x; x[j + 1] = v.y; x[j + 2] = v.z; x[j + 3] = v.w;
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t y[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) y[j] = __float_as_uint(x[32 * hh + j]);
            tmem_st32(tmem + TM_H + lb + 64 * hf + 32 * hh, y);
        }
        tmem_wait_st();
    }
    auto xbuf = [&](int n) { return tmem + TM_X + 128u * (uint32_t)(n & 1); };
    // output rows of chunk j (this warp's value half): X_j lanes 64..127 once O(j) is complete
    auto out_rows = [&](int j) -> bool {
        if (!warp_wait(&bars[CB_ODONE + 2 * (j & 1) + hf], (j >> 1) & 1, abort, E_C_ODONE, false)) return false;
        tc_fence_after();
        float x[64];
        tmem_ld64(xbuf(j) + lb + 64 * hf, x);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[CB_XFREE + (j & 1)]);
        const int t = j * C + (r - 64);
        if (t < T) {
            const size_t go = (((size_t)b * T + t) * H + h) * DV + 64 * hf;
            if (p.o_bf16) {
                __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(p.o) + go;
#pragma unroll
                for (int c = 0; c < 64; c += 8) {
                    __nv_bfloat162 q0 = __floats2bfloat162_rn(x[c], x[c + 1]);
                    __nv_bfloat162 q1 = __floats2bfloat162_rn(x[c + 2], x[c + 3]);
                    __nv_bfloat162 q2 = __floats2bfloat162_rn(x[c + 4], x[c + 5]);
                    __nv_bfloat162 q3 = __floats2bfloat162_rn(x[c + 6], x[c + 7]);
                    uint4 u;
                    u.x = *reinterpret_cast<uint32_t *>(&q0);
                    u.y = *reinterpret_cast<uint32_t *>(&q1);
                    u.z = *reinterpret_cast<uint32_t *>(&q2);
                    u.w = *reinterpret_cast<uint32_t *>(&q3);
                    *reinterpret_cast<uint4 *>(dst + c) = u;
                }
            } else {
                float *dst = reinterpret_cast<float *>(p.o) + go;
#pragma unroll
                for (int c = 0; c < 64; c += 4)
                    *reinterpret_cast<float4 *>(dst + c) = make_float4(x[c], x[c + 1], x[c + 2], x[c + 3]);
            }
        }
        return true;
    };
    // the two value halves are independent chains (each column of h, Delta and O
    // depends only on the same column of U and h): warps of half hf wait only on
    // their own half's barriers
    bool ok = true;
    for (int n = 0; n < NC; ++n) {
        const int s = n & 1;
        // the gates of chunk n are scanned before its conversion completes
        if (!warp_wait(&bars[CB_CVT + s], (n >> 1) & 1, abort, E_C_CVT, false)) { ok = false; break; }
        if (n > 0 && !warp_wait(&bars[CB_ZDONE + hf], (n - 1) & 1, abort, E_C_ZDONE, true)) { ok = false; break; }
        tc_fence_after();
        {
            // h16 <- h (operand of X(n));  h <- e^{g_C} h for Z(n) to accumulate onto
            float x[64];
            tmem_ld64(tmem + TM_H + lb + 64 * hf, x);
            const float egC = cpar[n & 3].egC;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t y[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) y[j] = __float_as_uint(x[32 * hh + j] * egC);
                tmem_st32(tmem + TM_H + lb + 64 * hf + 32 * hh, y);
            }
            st_row_f16(hs, r, x);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[CB_HREADY + hf]);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[CB_HSTORED + hf]);
        if (sp < 2) {
            // Delta = U - W h (X_n lanes 0..63) -> fp16 over V in slot s
            if (!warp_wait(&bars[CB_XDONE + 2 * (n & 1) + hf], (n >> 1) & 1, abort, E_C_XDONE, true)) {
                ok = false;
                break;
            }
            tc_fence_after();
            float x[64];
            tmem_ld64(xbuf(n) + lb + 64 * hf, x);
            st_row_f16(slot(s) + S_V0 + hf * 8192, r, x);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[CB_DDONE + hf]);
        } else if (n > 0) {
            if (!out_rows(n - 1)) { ok = false; break; }
        }
    }
    if (ok && NC > 0) {
        if (sp >= 2) ok = out_rows(NC - 1);
        if (ok && warp_wait(&bars[CB_ZDONE + hf], (NC - 1) & 1, abort, E_C_ZDONE, false)) {
            tc_fence_after();
            float x[64];
            tmem_ld64(tmem + TM_H + lb + 64 * hf, x);
            if (p.S_T) {
                float *dst = p.S_T + (bh * DK + r) * DV + 64 * hf;
#pragma unroll
                for (int j = 0; j < 64; j += 4)
                    *reinterpret_cast<float4 *>(dst + j) = make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
            }
        }
    }
}

__global__ void __launch_bounds__(NTHREADS, 1)
fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const FusedParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5;
    const uint32_t rank = cluster_ctarank();
    const int h = blockIdx.y, b = blockIdx.z;
    const bool key = (rank == 0);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + (key ? K_BAR : C_BAR));
    uint8_t *misc = sm + (key ? K_MISC : C_MISC);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 4);

    if (tid == 0) {
        if (key) {
            for (int i = 0; i < KB_N; ++i) mbar_init(&bars[i], 1);
            for (int i = 0; i < 2; ++i) {
                mbar_init(&bars[KB_LFULL + i], 4);    // stage A warps
                mbar_init(&bars[KB_LFREE + i], 8);    // stage B warps
                mbar_init(&bars[KB_TFULL + i], 8);    // stage B warps
                mbar_init(&bars[KB_TFREE + i], 4);    // stage C warps
            }
        } else {
            for (int i = 0; i < 2; ++i) {
                mbar_init(&bars[CB_SFULL + i], 1);
                mbar_init(&bars[CB_SFREE + i], 1);
                mbar_init(&bars[CB_KFULL + i], 1);
                mbar_init(&bars[CB_CVT + i], 6);
            }
            for (int i = 0; i < 4; ++i) {
                mbar_init(&bars[CB_XDONE + i], 1);
                mbar_init(&bars[CB_ODONE + i], 1);
            }
            for (int i = 0; i < 2; ++i) mbar_init(&bars[CB_XFREE + i], 4);
            for (int j = 0; j < 2; ++j) {
                mbar_init(&bars[CB_HREADY + j], 4);
                mbar_init(&bars[CB_HSTORED + j], 4);
                mbar_init(&bars[CB_DDONE + j], 2);
                mbar_init(&bars[CB_ZDONE + j], 1);
            }
            mbar_init(&bars[CB_WDONE], 1);
            mbar_init(&bars[CB_WREADY], 6);
            mbar_init(&bars[CB_UDONE], 1);
            // [2], [3]: chunks the key side shipped per slot; [6], [7]: chunks consumed
            for (int i = 2; i < 8; ++i) reinterpret_cast<volatile uint32_t *>(misc)[i] = 0;
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (!key) {
        // the zero tiles of both slots ([T diag(beta) ; 0] and [0 ; P])
        for (int i = tid; i < 2 * 512; i += NTHREADS)
            *reinterpret_cast<uint4 *>(sm + C_SLOT + (i >> 9) * SLOT + S_ZERO + ((i & 511) << 4)) =
                make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
    }
    __syncwarp();
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    block_sync();
    tc_fence_after();
    // both CTAs' barriers are initialised before either touches the other's
    cluster_sync_all();
    const uint32_t tmem = *tmem_slot;

    if (key) key_cta(sm, &tm_q, &tm_k, p, b, h, tmem, abort_flag);
    else chain_cta(sm, &tm_q, &tm_k, &tm_v, p, b, h, tmem, abort_flag);

    // ------------------------------------------------------------ teardown
    tc_fence_before();
    block_sync();
    cluster_sync_all();          // the key side has stopped shipping and written its counts
    if (!key && tid == 0) {
        // shipments the chain never consumed (error path only): wait for them,
        // bounded, so that no copy still writes into this CTA when it exits
        volatile uint32_t *cnt = reinterpret_cast<volatile uint32_t *>(misc);
        for (int s = 0; s < 2; ++s)
            for (uint32_t i = cnt[6 + s]; i < cnt[2 + s]; ++i)
                mbar_wait_drain(&bars[CB_KFULL + s], i & 1, kWait);
    }
    __syncwarp();
    block_sync();
    cluster_sync_all();          // no copy into the chain CTA is in flight any more
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (tid == 0 && *abort_flag) atomicCAS(&g_fused_error, 0u, (unsigned)*abort_flag);
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
bool make_map(CUtensorMap *m, const void *ptr, int B, int T, int H, int D) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)C, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

bool fused_supports(const FwdParams &p, const char **why) {
    if (!p.io_bf16) { *why = "needs bf16 q/k/v"; return false; }
    if (p.general) { *why = "two-gate rule runs on the SIMT kernel"; return false; }
    if (p.C != C) { *why = "needs chunk 64"; return false; }
    if (p.dk != DK || p.dv != DV) { *why = "needs dk = dv = 128"; return false; }
    if (p.mode == GDN_INV_NEUMANN_RESIDUAL) { *why = "residual correction runs on the split kernels"; return false; }
    if (p.B > 65535 || p.H > 65535) { *why = "B, H <= 65535"; return false; }
    return true;
}

cudaError_t launch_fused(const FwdParams &p, cudaStream_t stream, const char **why, float *dbg_T, int dbg_b,
                         int dbg_h, int dbg_n) {
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, p.q, p.B, p.T, p.H, p.dk) || !make_map(&mk, p.k, p.B, p.T, p.H, p.dk) ||
        !make_map(&mv, p.v, p.B, p.T, p.H, p.dv)) {
        *why = "(tensor map encoding failed)";
        return cudaErrorInvalidValue;
    }
    // The attribute is per device: set it on every launch (cheap) rather than
    // remembering a process-wide flag that another device would not share.
    cudaError_t e = cudaFuncSetAttribute(fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FUSED_SMEM);
    if (e != cudaSuccess) return e;
    FusedParams k;
    k.B = p.B; k.T = p.T; k.H = p.H; k.NC = (p.T + C - 1) / C;
    k.alpha = p.alpha; k.beta = p.beta; k.S0 = p.S0; k.o = p.o; k.S_T = p.S_T; k.o_bf16 = p.o_bf16;
    k.neumann = p.mode == GDN_INV_NEUMANN ? 1 : 0;
    k.N = p.N;
    k.dbg_T = dbg_T; k.dbg_b = dbg_b; k.dbg_h = dbg_h; k.dbg_n = dbg_n;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, p.H, p.B);
    cfg.blockDim = dim3(NTHREADS, 1, 1);
    cfg.dynamicSmemBytes = FUSED_SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fused_kernel, mq, mk, mv, k);
}

unsigned int fused_read_and_clear_error(cudaError_t *err) {
    unsigned int v = 0, zero = 0;
    *err = cudaMemcpyFromSymbol(&v, g_fused_error, sizeof(v));
    if (*err == cudaSuccess && v) *err = cudaMemcpyToSymbol(g_fused_error, &zero, sizeof(zero));
    return v;
}

}  // namespace gdn
