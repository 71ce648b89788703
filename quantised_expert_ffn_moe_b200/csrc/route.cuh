// route.cuh -- router kernel: logits (fp64 from exact products), softmax,
// warp-level top-k over up to 1024 logits, weights renormalised over the
// selected experts, and the shared-expert gate.
//
// Pages: "Qwen3.5-397B MoE fonctionne avec 14 Go de RAM via un chargement
// d'expert paginé sur M1 Ultra", opening paragraph (512 experts, top-10
// routing); "Flash-MoE - Exécuter un modèle de 397 milliards de paramètres sur
// un ordinateur portable", "Architecture du modèle" (K active experts per
// token, one shared) and "Shaders de calcul Metal" (MoE combine + gate).
#pragma once

#include "common.cuh"

namespace moeq {

struct RouteArgs {
    const uint16_t *x;         // bf16 [T][H]
    int T, H, E, k;
    const void *w_router;      // [E][H] bf16 or fp32
    const float *logit_bias;   // fp32 [T][E] or null
    const uint16_t *shared_gate;  // bf16 [H] or null
    int *topk_idx_out;         // optional user copies [T][k]
    float *topk_w_out;
    WsPtrs ws;
};

// Order-preserving map of a double onto uint64 (larger double -> larger key);
// -0 is folded onto +0 so equal values get equal keys.
__device__ __forceinline__ unsigned long long f64_key(double d) {
    if (d == 0.0) d = 0.0;
    unsigned long long u = (unsigned long long)__double_as_longlong(d);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}
__device__ __forceinline__ double key_f64(unsigned long long k) {
    unsigned long long u = (k >> 63) ? (k & 0x7fffffffffffffffull) : ~k;
    return __longlong_as_double((long long)u);
}

// Top-k of logits[0..E) by one warp.  Lane l holds logits l, l+32, ...; each
// of k rounds takes the lane-local best still available, then the warp-wide
// best by three redux steps (high word, low word, lowest expert id), so equal
// logits go to the lower id.  Lane r ends holding the r-th pick.
__device__ __forceinline__ void topk_warp(const RouteArgs &a, int t, int lane) {
    constexpr int PL = kMaxExperts / 32;
    const double *lg = a.ws.logits(t);
    const int E = a.E, k = a.k;
    unsigned long long key[PL];
#pragma unroll
    for (int j = 0; j < PL; ++j) {
        const int e = lane + 32 * j;
        key[j] = (e < E) ? f64_key(__ldcg(lg + e)) : 0ull;
    }
    unsigned taken = 0;
    int my_e = -1;
    double my_l = 0.0;
    for (int r = 0; r < k; ++r) {
        unsigned long long best = 0ull;
        int bj = -1;
#pragma unroll
        for (int j = 0; j < PL; ++j) {
            const bool avail = (lane + 32 * j < E) && !((taken >> j) & 1u);
            if (avail && (bj < 0 || key[j] > best)) {
                best = key[j];
                bj = j;
            }
        }
        const unsigned hi = bj >= 0 ? (unsigned)(best >> 32) : 0u;
        const unsigned mhi = __reduce_max_sync(0xffffffffu, hi);
        const bool c1 = bj >= 0 && hi == mhi;
        const unsigned lo = c1 ? (unsigned)best : 0u;
        const unsigned mlo = __reduce_max_sync(0xffffffffu, lo);
        const bool c2 = c1 && (unsigned)best == mlo;
        const unsigned eb = __reduce_min_sync(0xffffffffu, c2 ? (unsigned)(lane + 32 * bj) : 0xffffffffu);
        if ((int)(eb & 31u) == lane) taken |= 1u << (eb >> 5);
        if (lane == r) {
            my_e = (int)eb;
            my_l = key_f64(((unsigned long long)mhi << 32) | mlo);
        }
    }
    // weights: softmax restricted to the k selected logits (= renormalised softmax)
    const double l0 = __shfl_sync(0xffffffffu, my_l, 0);
    const double ex = (lane < k) ? exp(my_l - l0) : 0.0;
    const double z = warp_sum_f64(ex);
    if (lane < k) {
        const float w = (float)(ex / z);
        a.ws.topk_idx(t)[lane] = my_e;
        a.ws.topk_w(t)[lane] = w;
        if (a.topk_idx_out) a.topk_idx_out[(size_t)t * k + lane] = my_e;
        if (a.topk_w_out) a.topk_w_out[(size_t)t * k + lane] = w;
    }
    if (lane == 0) {
        float g = 1.0f;
        if (a.shared_gate) g = (float)(1.0 / (1.0 + exp(-__ldcg(lg + E))));
        *a.ws.gamma(t) = g;
    }
}

// grid (ceil((E + gate)/4), T), block 128: one warp per router row.  The last
// CTA of a token to finish (atomic arrival count) runs the top-k and resets
// the count to zero.
template <bool kF32Router>
__global__ void __launch_bounds__(kRouteWarps * 32) k_route(RouteArgs a) {
    extern __shared__ float xs[];  // x[t] as fp32, H values
    __shared__ int s_last;
    const int t = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int H = a.H;
    // x may come from the previous kernel on the stream; dependents are
    // released only after that wait, so they may read x in their prologue
    griddep_wait();
    griddep_launch_dependents();
    const uint16_t *xt = a.x + (size_t)t * H;
    for (int j = threadIdx.x * 8; j < H; j += blockDim.x * 8) {
        const uint4 v = *reinterpret_cast<const uint4 *>(xt + j);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            xs[j + 2 * i] = bf16_bits_to_float(w[i] & 0xffffu);
            xs[j + 2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
        }
    }
    __syncthreads();
    const int nrows = a.E + (a.shared_gate ? 1 : 0);
    const int row = blockIdx.x * kRouteWarps + warp;
    if (row < nrows) {
        double acc = 0.0;
        if (kF32Router && row < a.E) {
            // fp32 weight x bf16 input: the product is exact in fp64
            const float *wr = reinterpret_cast<const float *>(a.w_router) + (size_t)row * H;
            for (int j = lane * 4; j < H; j += 128) {
                const float4 w = *reinterpret_cast<const float4 *>(wr + j);
                acc += (double)w.x * (double)xs[j];
                acc += (double)w.y * (double)xs[j + 1];
                acc += (double)w.z * (double)xs[j + 2];
                acc += (double)w.w * (double)xs[j + 3];
            }
        } else {
            // bf16 x bf16: the product is exact in fp32, the sum runs in fp64
            const uint16_t *wr = row < a.E
                ? reinterpret_cast<const uint16_t *>(a.w_router) + (size_t)row * H
                : a.shared_gate;
#pragma unroll 4
            for (int j = lane * 8; j < H; j += 256) {
                const uint4 v = ldg_stream(reinterpret_cast<const uint32_t *>(wr + j));
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc += (double)(bf16_bits_to_float(w[i] & 0xffffu) * xs[j + 2 * i]);
                    acc += (double)(bf16_bits_to_float(w[i] >> 16) * xs[j + 2 * i + 1]);
                }
            }
        }
        acc = warp_sum_f64(acc);
        if (lane == 0) {
            if (row < a.E && a.logit_bias) acc += (double)a.logit_bias[(size_t)t * a.E + row];
            if (!isfinite(acc)) flag_status(a.ws.status, MOE_DEV_NONFINITE);
            a.ws.logits(t)[row] = acc;
            __threadfence();
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned old = atomicAdd(a.ws.route_cnt(t), 1u);
        s_last = (old == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (warp == 0) topk_warp(a, t, lane);
    if (threadIdx.x == 0) *a.ws.route_cnt(t) = 0u;
}

}  // namespace moeq
