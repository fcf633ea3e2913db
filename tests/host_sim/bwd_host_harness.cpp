// Test infrastructure: runs the four backward kernels of gdn_bwd_kernels.cuh on
// the host (see cuda_host_shim.h), grid block by grid block, with each kernel's
// block size (512 threads for the prep kernel, 256 for the others).  Before each block the shared-memory array is filled with NaN; after
// it, every word past the kernel's requested size must still be NaN (nothing
// wrote past its allocation).  The workspace starts NaN-filled too, so a read
// of an entry no kernel wrote shows up in the outputs.  Exposes one C entry:
//   host_bwd(...) -> 0, or 100 + the number of blocks that wrote past their
//   shared memory.
#include "cuda_host_shim.h"
#include "gdn_bwd_kernels.cuh"

using namespace gdn;
namespace gdn { namespace bwd { float4 bwd_smem[60000]; } }

static void fill_nan(void *p, size_t bytes) {
    const uint32_t nan = 0x7fc00000u;
    for (size_t i = 0; i + 4 <= bytes; i += 4) std::memcpy(static_cast<char *>(p) + i, &nan, 4);
}

static int g_overrun = 0;

template <class F>
static void run_grid(F kernel, dim3h grid, const BwdParams &p, size_t smem_floats, int nthreads = bwd::kThreads) {
    for (unsigned z = 0; z < grid.z; ++z)
        for (unsigned y = 0; y < grid.y; ++y)
            for (unsigned x = 0; x < grid.x; ++x) {
                blockIdx = {x, y, z};
                fill_nan(bwd::bwd_smem, sizeof(bwd::bwd_smem));
                std::barrier<> bar(nthreads);
                g_block_barrier = &bar;
                std::vector<std::barrier<> *> warps;
                for (int w = 0; w < (nthreads + 31) / 32; ++w) warps.push_back(new std::barrier<>(32));
                g_warp_barriers = warps.data();
                std::vector<std::thread> th;
                for (int t = 0; t < nthreads; ++t)
                    th.emplace_back([&, t] { threadIdx = {(unsigned)t, 0, 0}; kernel(p); });
                for (auto &t : th) t.join();
                for (auto *w : warps) delete w;
                const uint32_t *u = reinterpret_cast<const uint32_t *>(bwd::bwd_smem);
                for (size_t i = smem_floats; i < sizeof(bwd::bwd_smem) / 4; ++i)
                    if (u[i] != 0x7fc00000u) { ++g_overrun; break; }
            }
}

static size_t region(size_t floats, size_t n) { return (floats * n * sizeof(float) + 255) & ~(size_t)255; }

extern "C" int host_bwd(int B, int T, int H, int dk, int dv, int C, int io_bf16, int do_bf16,
                        const void *q, const void *k, const void *v, const float *alpha,
                        const float *beta, const float *S0, const void *grad_o, const float *grad_S_T,
                        float *gq, float *gk, float *gv, float *ga, float *gb, float *gS0, int neumann, int N,
                        int S) {
    BwdParams p{};
    p.neumann = neumann; p.N = N; p.residual = S > 0; p.S = S;
    p.B = B; p.T = T; p.H = H; p.dk = dk; p.dv = dv; p.C = C; p.NC = (T + C - 1) / C;
    p.io_bf16 = io_bf16; p.do_bf16 = do_bf16;
    p.q = q; p.k = k; p.v = v; p.alpha = alpha; p.beta = beta; p.S0 = S0;
    p.grad_o = grad_o; p.grad_S_T = grad_S_T;
    p.grad_q = gq; p.grad_k = gk; p.grad_v = gv; p.grad_alpha = ga; p.grad_beta = gb; p.grad_S0 = gS0;
    // the same regions, in the same order, as gdn::bwd_carve_workspace
    const size_t n = (size_t)B * H * p.NC, Cs = C, dks = dk, dvs = dv;
    const size_t bytes = region(Cs, n) + 3 * region(Cs * Cs, n) + region(Cs * dks, n) +
                         2 * region(Cs * dvs, n) + 3 * region(dks * dvs, n) + (neumann ? region(Cs * Cs, n) : 0);
    std::vector<char> ws(bytes);
    fill_nan(ws.data(), bytes);
    char *w = ws.data();
    p.ws_g = reinterpret_cast<float *>(w);  w += region(Cs, n);
    p.ws_T = reinterpret_cast<float *>(w);  w += region(Cs * Cs, n);
    p.ws_S = reinterpret_cast<float *>(w);  w += region(Cs * Cs, n);
    p.ws_M = reinterpret_cast<float *>(w);  w += region(Cs * Cs, n);
    p.ws_W = reinterpret_cast<float *>(w);  w += region(Cs * dks, n);
    p.ws_D = reinterpret_cast<float *>(w);  w += region(Cs * dvs, n);
    p.ws_Y = reinterpret_cast<float *>(w);  w += region(Cs * dvs, n);
    p.ws_P = reinterpret_cast<float *>(w);  w += region(dks * dvs, n);
    p.ws_h = reinterpret_cast<float *>(w);  w += region(dks * dvs, n);
    p.ws_dh = reinterpret_cast<float *>(w);  w += region(dks * dvs, n);
    p.ws_dA = neumann ? reinterpret_cast<float *>(w) : nullptr;
    g_overrun = 0;
    const dim3h per_chunk{(unsigned)p.NC, (unsigned)H, (unsigned)B};
    const dim3h per_slice{(unsigned)(dv / bwd::kCols), (unsigned)H, (unsigned)B};
    run_grid(bwd::bwd_prep_kernel, per_chunk, p, bwd::prep_smem_floats(C, dk, dv, p.residual), bwd::kPrepThreads);
    run_grid(bwd::bwd_state_fwd_kernel, per_slice, p, bwd::state_fwd_smem_floats(C, dk));
    run_grid(bwd::bwd_state_rev_kernel, per_slice, p, bwd::state_rev_smem_floats(C, dk));
    if (neumann) run_grid(bwd::bwd_neumann_kernel, per_chunk, p, bwd::neumann_smem_floats(C, dv, p.residual), bwd::kPrepThreads);
    const size_t gs = bwd::grad_smem_floats(C, dk);
    switch (dk) {
        case 16: run_grid(bwd::bwd_grad_kernel<16>, per_chunk, p, gs, bwd::kGradThreads); break;
        case 32: run_grid(bwd::bwd_grad_kernel<32>, per_chunk, p, gs, bwd::kGradThreads); break;
        case 64: run_grid(bwd::bwd_grad_kernel<64>, per_chunk, p, gs, bwd::kGradThreads); break;
        case 128: run_grid(bwd::bwd_grad_kernel<128>, per_chunk, p, gs, bwd::kGradThreads); break;
        default: return 1;
    }
    return g_overrun ? 100 + g_overrun : 0;
}
