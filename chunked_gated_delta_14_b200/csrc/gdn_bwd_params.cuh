// Resolved arguments of the backward kernels (gradient of the gated delta
// rule), filled by the host layer from gdn_bwd_args.  Plain data only.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace gdn {

struct BwdParams {
    int B, T, H, dk, dv, C;
    int NC;                       // chunks per sequence, ceil(T / C)
    int io_bf16, do_bf16;         // q/k/v and grad_o element types (1 = bf16, 0 = fp32)
    const void *q, *k, *v;        // [B, T, H, dk|dv]
    const float *alpha, *beta;    // [B, T, H] or null (=> 1)
    const float *S0;              // [B, H, dk, dv] or null (=> 0)
    const void *grad_o;           // [B, T, H, dv]
    const float *grad_S_T;        // [B, H, dk, dv] or null (=> 0)
    float *grad_q, *grad_k, *grad_v;
    float *grad_alpha, *grad_beta, *grad_S0;   // each may be null
    int neumann, N;               // chunk inverse: 0 exact; 1 the masked truncated series of order N
    int residual, S;              // with neumann: the series with S residual-correction terms
    // Workspace regions, fp32, each indexed by chunk-head (b*H + h)*NC + n:
    float *ws_g;    // C        in-chunk cumulative log decay g
    float *ws_T;    // C x C    T = (I + L)^-1
    float *ws_S;    // C x C    decayed Gram Gamma (.) K K^T, strictly lower
    float *ws_M;    // C x C    causal decayed scores M = Gamma (.) Q K^T, lower with diagonal
    float *ws_W;    // C x dk   W = T diag(beta e^g) K
    float *ws_D;    // C x dv   U = T diag(beta) V, overwritten with Delta = U - W h
    float *ws_Y;    // C x dv   M^T dO (M the causal decayed scores), overwritten with
                    //          Y = T^T dDelta
    float *ws_P;    // dk x dv  (diag(e^g) Q)^T dO
    float *ws_h;    // dk x dv  state h = S^T at the chunk's start
    float *ws_dh;   // dk x dv  dL/dh at the chunk's end
    float *ws_dA;   // C x C    masked series only: the exact inverse (prep), then dA = -dL
};

// fp32 words of workspace per chunk-head.
inline size_t bwd_ws_floats_per_chunk(int C, int dk, int dv) {
    return (size_t)C + 3 * (size_t)C * C + (size_t)C * dk + 2 * (size_t)C * dv + 3 * (size_t)dk * dv;
}

}  // namespace gdn
