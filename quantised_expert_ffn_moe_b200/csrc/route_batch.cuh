// route_batch.cuh -- the router for many tokens at once: logits as a tiled
// GEMM with fp64 accumulation, then one top-k CTA per token.
//
// Pages: "Qwen3.5-397B MoE fonctionne avec 14 Go de RAM via un chargement
// d'expert paginé sur M1 Ultra", opening paragraph (512 experts, top-10
// routing); "Flash-MoE - Exécuter un modèle de 397 milliards de paramètres sur
// un ordinateur portable", "Architecture du modèle".  The pages route one
// token at a time; the batched form is this library's.
#pragma once

#include "route.cuh"

namespace moeq {

// For a batch of tokens the router is a small GEMM, logits[T][rows] =
// x[T][H] * W[rows][H]^T (rows: the E router rows, then the shared-expert gate
// vector).  Each product of two bf16 values (or bf16 x fp32) is exact in
// fp64, so an fp64 fused multiply-add adds the exact product with one
// rounding: the same arithmetic as the one-token kernel, only summed in
// another order.  A CTA computes a 32-token x 64-row tile over K chunks of
// 64 staged in shared memory as fp64; each thread owns 4 tokens x 4 rows.

constexpr int kRgTok = 32;
constexpr int kRgRows = 64;
constexpr int kRgK = 64;
constexpr int kRgThreads = 128;
constexpr int kRouteGemmMinTokens = 64;  // from this many tokens on, the GEMM form

// grid (ceil(rows / 64), ceil(T / 32)), block 128.  Thread (tx, ty) =
// (tid % 16, tid / 16) owns rows tx + 16 j and tokens ty + 8 i (i, j < 4):
// per k step 8 shared-memory loads feed 16 fp64 FMAs.
template <bool kF32Router>
__global__ void __launch_bounds__(kRgThreads) k_route_gemm(RouteArgs a) {
    __shared__ double xs[kRgK][kRgTok];    // x chunk, k-major
    __shared__ double wsm[kRgK][kRgRows];  // router chunk, k-major
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.H;
    const int nrows = a.E + (a.shared_gate ? 1 : 0);
    const int row0 = blockIdx.x * kRgRows, t0 = blockIdx.y * kRgTok;
    // staging map: x: token `lane`, k blocks 8 warp + 32 q (q < 2);
    // W: row tid % 64, k blocks 8 (tid / 64) + 16 q (q < 4)
    constexpr int XQ = 2, WQ = 4;
    const int xt = t0 + lane;
    const int wr = row0 + (tid & 63), wk = 8 * (tid >> 6);
    const bool x_in = xt < a.T;
    const bool w_in = wr < nrows;
    const bool w_f32 = kF32Router && wr < a.E;
    const uint16_t *wrow16 = nullptr;
    const float *wrow32 = nullptr;
    if (w_in) {
        if (w_f32)
            wrow32 = reinterpret_cast<const float *>(a.w_router) + (size_t)wr * H;
        else
            wrow16 = wr < a.E ? reinterpret_cast<const uint16_t *>(a.w_router) + (size_t)wr * H : a.shared_gate;
    }
    uint4 xv[XQ];
    uint4 wv[WQ][2];  // bf16: [q][0] holds 8 values; fp32: [q][0..1] hold 8 values
    auto load_w = [&](int k0) {
#pragma unroll
        for (int q = 0; q < WQ; ++q) {
            const int k = k0 + wk + 16 * q;
            if (w_f32) {
                wv[q][0] = *reinterpret_cast<const uint4 *>(wrow32 + k);
                wv[q][1] = *reinterpret_cast<const uint4 *>(wrow32 + k + 4);
            } else {
                wv[q][0] = w_in ? ldg_stream(reinterpret_cast<const uint32_t *>(wrow16 + k)) : make_uint4(0u, 0u, 0u, 0u);
                wv[q][1] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
    };
    auto load_x = [&](int k0) {
#pragma unroll
        for (int q = 0; q < XQ; ++q)
            xv[q] = x_in ? *reinterpret_cast<const uint4 *>(a.x + (size_t)xt * H + k0 + 8 * warp + 32 * q)
                         : make_uint4(0u, 0u, 0u, 0u);
    };
    auto stage = [&]() {
#pragma unroll
        for (int q = 0; q < XQ; ++q) {
            const int kk = 8 * warp + 32 * q;
            const uint32_t xw[4] = {xv[q].x, xv[q].y, xv[q].z, xv[q].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xs[kk + 2 * i][lane] = (double)bf16_bits_to_float(xw[i] & 0xffffu);
                xs[kk + 2 * i + 1][lane] = (double)bf16_bits_to_float(xw[i] >> 16);
            }
        }
#pragma unroll
        for (int q = 0; q < WQ; ++q) {
            const int kk = wk + 16 * q;
            if (w_f32) {
                const float f[8] = {__uint_as_float(wv[q][0].x), __uint_as_float(wv[q][0].y),
                                    __uint_as_float(wv[q][0].z), __uint_as_float(wv[q][0].w),
                                    __uint_as_float(wv[q][1].x), __uint_as_float(wv[q][1].y),
                                    __uint_as_float(wv[q][1].z), __uint_as_float(wv[q][1].w)};
#pragma unroll
                for (int i = 0; i < 8; ++i) wsm[kk + i][tid & 63] = (double)f[i];
            } else {
                const uint32_t ww[4] = {wv[q][0].x, wv[q][0].y, wv[q][0].z, wv[q][0].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    wsm[kk + 2 * i][tid & 63] = (double)bf16_bits_to_float(ww[i] & 0xffffu);
                    wsm[kk + 2 * i + 1][tid & 63] = (double)bf16_bits_to_float(ww[i] >> 16);
                }
            }
        }
    };
    // the router rows do not depend on the previous kernel: the first chunk
    // is loaded before the dependency wait (x after it)
    load_w(0);
    griddep_wait();
    load_x(0);
    const int tx = tid & 15, ty = tid >> 4;
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
    for (int k0 = 0; k0 < H; k0 += kRgK) {
        stage();
        __syncthreads();
        if (k0 + kRgK < H) {
            load_w(k0 + kRgK);
            load_x(k0 + kRgK);
        }
#pragma unroll 4
        for (int k = 0; k < kRgK; ++k) {
            double xr[4], wrr[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) xr[i] = xs[k][ty + 8 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) wrr[j] = wsm[k][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fma(xr[i], wrr[j], acc[i][j]);
        }
        __syncthreads();
    }
    griddep_launch_dependents();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + ty + 8 * i;
        if (t >= a.T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = row0 + tx + 16 * j;
            if (r >= nrows) continue;
            double l = acc[i][j];
            if (r < a.E && a.logit_bias) l += (double)a.logit_bias[(size_t)t * a.E + r];
            if (!isfinite(l)) flag_status(a.ws.status, MOE_DEV_NONFINITE);
            a.ws.logits(t)[r] = l;
        }
    }
}

// grid T, block 256: top-k, weights and shared-expert gate of token t from
// its logits in the workspace.
__global__ void __launch_bounds__(kRouteThreads) k_route_topk(RouteArgs a) {
    __shared__ TopkSmem<kRouteThreads> sm;
    griddep_wait();
    const int t = blockIdx.x;
    topk_block<kRouteThreads>(a.ws.logits(t), a.E, a.k, sm);
    griddep_launch_dependents();
    topk_store<kRouteThreads>(a, t, sm);
}

}  // namespace moeq
