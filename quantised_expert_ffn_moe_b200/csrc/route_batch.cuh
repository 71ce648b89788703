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
// another order (the fp64 tensor-core MMA adds exact fp64 products).  A CTA
// computes a 32-token x 64-row tile.

constexpr int kRgTok = 32;
constexpr int kRgRows = 64;
constexpr int kRgThreads = 128;
constexpr int kRouteGemmMinTokens = 64;  // from this many tokens on, the GEMM form

// fp64 tensor-core product of a warp: D (8 x 8) += A (8 x 4) * B (4 x 8).
// Lane l holds A[l / 4][l % 4], B[l % 4][l / 4] and D[l / 4][2 (l % 4) + i].
__device__ __forceinline__ void dmma_8x8x4(double (&d)[2], double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                 : "+d"(d[0]), "+d"(d[1])
                 : "d"(a), "d"(b));
}

// grid (ceil(rows / 64), ceil(T / 32)), block 128.  K chunks of 32 are
// staged in shared memory as fp64 (rows of the k-major arrays padded so the
// fragment loads of a warp take two wavefronts); warp w computes all 32
// tokens x rows 16 w .. 16 w + 15 with the fp64 tensor-core MMA (8 x 8 x 4):
// 4 token blocks x 2 row blocks, 8 MMAs per 4 k values.
template <bool kF32Router>
__global__ void __launch_bounds__(kRgThreads) k_route_gemm(RouteArgs a) {
    constexpr int KC = 32;                   // k values per chunk
    constexpr int XS = kRgTok + 8, WS = kRgRows + 8;  // padded row strides (doubles)
    __shared__ double xs[KC][XS];   // x chunk, k-major
    __shared__ double wsm[KC][WS];  // router chunk, k-major
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = a.H;
    const int nrows = a.E + (a.shared_gate ? 1 : 0);
    const int row0 = blockIdx.x * kRgRows, t0 = blockIdx.y * kRgTok;
    // staging map: x: token `lane`, k block 8 warp; W: row tid % 64, k blocks
    // 8 (tid / 64) + 16 q (q < 2)
    constexpr int WQ = 2;
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
    uint4 xv;
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
        xv = x_in ? *reinterpret_cast<const uint4 *>(a.x + (size_t)xt * H + k0 + 8 * warp) : make_uint4(0u, 0u, 0u, 0u);
    };
    auto stage = [&]() {
        {
            const int kk = 8 * warp;
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
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
    const int g = lane >> 2, c = lane & 3;  // fragment row / column of this lane
    double acc[4][2][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;
    for (int k0 = 0; k0 < H; k0 += KC) {
        stage();
        __syncthreads();
        if (k0 + KC < H) {
            load_w(k0 + KC);
            load_x(k0 + KC);
        }
#pragma unroll
        for (int k4 = 0; k4 < KC; k4 += 4) {
            double af[4], bf[2];
#pragma unroll
            for (int i = 0; i < 4; ++i) af[i] = xs[k4 + c][8 * i + g];
#pragma unroll
            for (int j = 0; j < 2; ++j) bf[j] = wsm[k4 + c][16 * warp + 8 * j + g];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 2; ++j) dmma_8x8x4(acc[i][j], af[i], bf[j]);
        }
        __syncthreads();
    }
    griddep_launch_dependents();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + 8 * i + g;
        if (t >= a.T) continue;
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int r = row0 + 16 * warp + 8 * j + 2 * c + e;
                if (r >= nrows) continue;
                double l = acc[i][j][e];
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
