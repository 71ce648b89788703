// route.cuh -- router kernel: logits (fp64 from exact products), softmax,
// top-k over up to 1024 logits, weights renormalised over the selected
// experts, and the shared-expert gate.
//
// Pages: "Qwen3.5-397B MoE fonctionne avec 14 Go de RAM via un chargement
// d'expert paginé sur M1 Ultra", opening paragraph (512 experts, top-10
// routing); "Flash-MoE - Exécuter un modèle de 397 milliards de paramètres sur
// un ordinateur portable", "Architecture du modèle" (K active experts per
// token, one shared) and "Shaders de calcul Metal" (MoE combine + gate).
#pragma once

#include "common.cuh"
#include "image.cuh"

namespace moeq {

constexpr int kRouteThreads = 256;     // 8 warps
constexpr int kRouteRowsPerCta = 4;    // 2 warps per router row
constexpr int kTopkBins = 256;

struct RouteArgs {
    const uint16_t *x;         // bf16 [T][H]
    int T, H, E, k;
    const void *w_router;      // [E][H] bf16 or fp32
    const float *logit_bias;   // fp32 [T][E] or null
    const uint16_t *shared_gate;  // bf16 [H] or null
    int *topk_idx_out;         // optional user copies [T][k]
    float *topk_w_out;
    WsPtrs ws;
    // 1: the last CTA of a token takes the top-k (the routing call on its
    // own); 0: only the logits are written (the layer call routes in its
    // gate/up kernel).
    int do_topk;
    // 1: one extra CTA per token (the last) builds the operand image of x
    // (bits-wide code layout) into the workspace for the gate/up kernel.
    int build_image;
    int bits;
    // 1: x is the un-normalised hidden state; every CTA normalises its copy
    // (RMS, unit weight, eps) and the last CTA writes x-hat to xhat_out
    // when that is not null
    int norm;
    float eps;
    uint16_t *xhat_out;
};

// Order-preserving map of a double onto uint64 (larger double -> larger key);
// -0 is folded onto +0 so equal values get equal keys.
__device__ __forceinline__ unsigned long long f64_key(double d) {
    if (d == 0.0) d = 0.0;
    unsigned long long u = (unsigned long long)__double_as_longlong(d);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// Inverse of f64_key.
__device__ __forceinline__ double f64_of_key(unsigned long long k) {
    return __longlong_as_double((long long)((k >> 63) ? (k & 0x7fffffffffffffffull) : ~k));
}

__device__ __forceinline__ double warp_max_f64(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ double warp_min_f64(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmin(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Top-k of logits[0..E) by one CTA of NT threads (every thread calls it):
//  1. every logit is loaded at once (kept in shared memory as fp64 for the
//     exact ranking, in registers as fp32 for the binning);
//  2. each logit gets a bin, a monotone function of its fp32 rounding over
//     [min, max] in 256 steps (rounding to fp32 is monotone, so a logit in a
//     lower bin is strictly below every logit in a higher bin); the
//     histogram gives the highest bin b* such that at least k logits lie in
//     bins >= b*;
//  3. the candidates (bins >= b*, normally just over k of them) are ranked
//     exactly on their fp64 values: rank = number of candidates with a larger
//     logit, or an equal logit and a lower expert id.  Rank r < k is the r-th
//     pick.
// Weights (sel_w) are the softmax restricted to the picks (= the softmax
// renormalised over them).  Results in shared memory after a final barrier.
template <int NT>
struct TopkSmem {
    double val[kMaxExperts];
    unsigned hist[kTopkBins];
    unsigned long long ckey[kMaxExperts];
    int cidx[kMaxExperts];
    int sel_idx[kMaxTopK];
    double sel_l[kMaxTopK];
    float sel_w[kMaxTopK];
    float red[2][NT / 32];
    int ncand, bstar;
};

template <int NT>
__device__ void topk_block(const double *lg, int E, int k, TopkSmem<NT> &sm) {
    constexpr int EPT = (kMaxExperts + NT - 1) / NT;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float f[EPT];
    float mx = -INFINITY, mn = INFINITY;
    {
        double v[EPT];
#pragma unroll
        for (int j = 0; j < EPT; ++j) {
            const int e = tid + j * NT;
            v[j] = e < E ? __ldcg(lg + e) : 0.0;
        }
#pragma unroll
        for (int j = 0; j < EPT; ++j) {
            const int e = tid + j * NT;
            f[j] = (float)v[j];
            if (e < E) {
                sm.val[e] = v[j];
                mx = fmaxf(mx, f[j]);
                mn = fminf(mn, f[j]);
            }
        }
    }
    for (int i = tid; i < kTopkBins; i += NT) sm.hist[i] = 0u;
    if (tid == 0) sm.ncand = 0;
    mx = warp_max_f32(mx);
    mn = -warp_max_f32(-mn);
    if (lane == 0) {
        sm.red[0][warp] = mx;
        sm.red[1][warp] = mn;
    }
    __syncthreads();
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        mx = fmaxf(mx, sm.red[0][w]);
        mn = fminf(mn, sm.red[1][w]);
    }
    const float scale = mx > mn ? (float)kTopkBins / (mx - mn) : 0.f;
    // clamped: a NaN or infinite logit (flagged when written) still lands in a bin
    auto bin_of = [&](float v) { return max(0, min(kTopkBins - 1, __float2int_rz((v - mn) * scale))); };
#pragma unroll
    for (int j = 0; j < EPT; ++j)
        if (tid + j * NT < E) atomicAdd(&sm.hist[bin_of(f[j])], 1u);
    __syncthreads();
    if (warp == 0) {
        // lane L owns bins [256 - 8(L+1), 256 - 8L); counts summed from the top
        constexpr int BPL = kTopkBins / 32;
        unsigned c[BPL], sum = 0;
#pragma unroll
        for (int i = 0; i < BPL; ++i) {
            c[i] = sm.hist[kTopkBins - 1 - (lane * BPL + i)];
            sum += c[i];
        }
        unsigned incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const unsigned ballot = __ballot_sync(0xffffffffu, incl >= (unsigned)k);
        const int first = __ffs(ballot) - 1;  // lane whose bins reach k (exists: total = E >= k)
        if (lane == first) {
            unsigned cum = incl - sum;
            int b = kTopkBins - 1 - lane * BPL;
#pragma unroll
            for (int i = 0; i < BPL; ++i) {
                cum += c[i];
                if (cum >= (unsigned)k) {
                    b = kTopkBins - 1 - (lane * BPL + i);
                    break;
                }
            }
            sm.bstar = b;
        }
    }
    __syncthreads();
    const int bstar = sm.bstar;
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
        const int e = tid + j * NT;
        if (e < E && bin_of(f[j]) >= bstar) {
            const int pos = atomicAdd(&sm.ncand, 1);
            sm.ckey[pos] = f64_key(sm.val[e]);
            sm.cidx[pos] = e;
        }
    }
    __syncthreads();
    const int C = sm.ncand;
    if (C <= 32) {
        if (warp == 0) {
            // one warp ranks the candidates through shuffles, then the softmax
            const unsigned long long kc = lane < C ? sm.ckey[lane] : 0ull;
            const int ic = lane < C ? sm.cidx[lane] : 0x7fffffff;
            int rank = 0;
            for (int d = 0; d < C; ++d) {
                const unsigned long long kd = __shfl_sync(0xffffffffu, kc, d);
                const int id = __shfl_sync(0xffffffffu, ic, d);
                rank += (kd > kc) || (kd == kc && id < ic);
            }
            if (lane < C && rank < k) {
                sm.sel_idx[rank] = ic;
                sm.sel_l[rank] = f64_of_key(kc);
            }
            __syncwarp();
        }
    } else {
        for (int ci = tid; ci < C; ci += NT) {
            const unsigned long long kc = sm.ckey[ci];
            const int ic = sm.cidx[ci];
            int rank = 0;
            for (int d = 0; d < C; ++d) {
                const unsigned long long kd = sm.ckey[d];
                rank += (kd > kc) || (kd == kc && sm.cidx[d] < ic);
            }
            if (rank < k) {
                sm.sel_idx[rank] = ic;
                sm.sel_l[rank] = f64_of_key(kc);
            }
        }
        __syncthreads();
    }
    if (warp == 0) {
        // exp of differences to the largest logit in fp32 (each within 2 ulp),
        // their sum in fp64, one fp32 reciprocal: relative error of a weight
        // about 3e-7
        const double my_l = lane < k ? sm.sel_l[lane] : 0.0;
        const double l0 = sm.sel_l[0];
        const float ex = lane < k ? expf((float)(my_l - l0)) : 0.f;
        const double z = warp_sum_f64((double)ex);
        const float rz = 1.0f / (float)z;
        if (lane < k) sm.sel_w[lane] = ex * rz;
    }
    __syncthreads();
}

// Shared-expert gate sigmoid(z) of a gate logit.
__device__ __forceinline__ float gate_of_logit(double z) { return 1.0f / (1.0f + expf(-(float)z)); }

// Writes token t's routing results (and the shared-expert gate) to the
// workspace and the optional caller copies.
template <int NT>
__device__ void topk_store(const RouteArgs &a, int t, const TopkSmem<NT> &sm) {
    const int tid = threadIdx.x;
    if (tid < a.k) {
        const int e = sm.sel_idx[tid];
        const float w = sm.sel_w[tid];
        a.ws.topk_idx(t)[tid] = e;
        a.ws.topk_w(t)[tid] = w;
        if (a.topk_idx_out) a.topk_idx_out[(size_t)t * a.k + tid] = e;
        if (a.topk_w_out) a.topk_w_out[(size_t)t * a.k + tid] = w;
    }
    if (tid == 0) *a.ws.gamma(t) = a.shared_gate ? gate_of_logit(__ldcg(a.ws.logits(t) + a.E)) : 1.0f;
}

// grid (ceil((E + gate)/4) [+ 1 image CTA], T), block 256: two warps per
// router row (the shared-expert gate vector is row E).  With do_topk, the last CTA of a token
// to finish (atomic arrival count) runs the top-k and resets the count.
template <bool kF32Router>
__global__ void __launch_bounds__(kRouteThreads) k_route(RouteArgs a) {
    extern __shared__ __align__(16) float xs[];  // x[t] as fp32, H values
    __shared__ TopkSmem<kRouteThreads> sm;
    __shared__ double s_part[kRouteThreads / 32];
    __shared__ int s_last;
    const int t = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H;
    const int nrows = a.E + (a.shared_gate ? 1 : 0);
    const int row = blockIdx.x * kRouteRowsPerCta + (warp >> 1);
    const int half = warp & 1;  // which half of the row this warp sums
    const int hh = H / 2;
    // bf16 rows: the first 8 loads of 16 bytes per lane (a whole half row
    // when H <= 4096) are issued before anything else; the router matrix does
    // not depend on the previous kernel
    constexpr int B = 8;
    const bool bf16_row = row < nrows && !(kF32Router && row < a.E);
    const uint16_t *wr16 = bf16_row ? (row < a.E ? reinterpret_cast<const uint16_t *>(a.w_router) + (size_t)row * H
                                                 : a.shared_gate) + half * hh
                                    : nullptr;
    uint4 wv[B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
        const int j = lane * 8 + 256 * b;
        wv[b] = bf16_row && j < hh ? ldg_stream(reinterpret_cast<const uint32_t *>(wr16 + j)) : make_uint4(0u, 0u, 0u, 0u);
    }
    // x may come from the previous kernel on the stream
    griddep_wait();
    MOEQ_STAMP(0, 0);
    const uint16_t *xt = a.x + (size_t)t * H;
    {
        constexpr int U = 4;  // all of a thread's loads in flight (H <= 8192)
        uint4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int j = (tid + u * kRouteThreads) * 8;
            if (j < H) v[u] = *reinterpret_cast<const uint4 *>(xt + j);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int j = (tid + u * kRouteThreads) * 8;
            if (j < H) {
                const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    xs[j + 2 * i] = bf16_bits_to_float(w[i] & 0xffffu);
                    xs[j + 2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
                }
            }
        }
    }
    __syncthreads();
    if (a.norm) {
        // RMS normalisation of the row in place (unit weight): the same
        // summation order and rounding as k_rmsnorm, so x-hat is bit-equal
        double ss = 0.0;
        for (int j = tid; j < H; j += kRouteThreads) {
            const double v = xs[j];
            ss += v * v;
        }
        ss = warp_sum_f64(ss);
        if (lane == 0) s_part[warp] = ss;
        __syncthreads();
        double z = 0.0;
        for (int i = 0; i < kRouteThreads / 32; ++i) z += s_part[i];
        const double inv = 1.0 / sqrt(z / (double)H + (double)a.eps);
        for (int j = tid; j < H; j += kRouteThreads) {
            const __nv_bfloat16 b = __double2bfloat16((double)xs[j] * inv);
            xs[j] = __bfloat162float(b);
            if (a.xhat_out && blockIdx.x == gridDim.x - 1) a.xhat_out[(size_t)t * H + j] = __bfloat16_as_ushort(b);
        }
        __syncthreads();
    }
    MOEQ_STAMP(0, 1);
    if (a.build_image && blockIdx.x == gridDim.x - 1) {
        // the operand image of x, its group sums and steps, for the gate/up
        // kernel
        const int nwin = (H + kWinK - 1) / kWinK;
        auto load8 = [&](int c, float(&f)[8]) {
#pragma unroll
            for (int u = 0; u < 8; ++u) f[u] = xs[8 * c + u];
        };
        if (a.bits == 4)
            build_images<4>(a.ws.ximg(t), a.ws.xsg(t), a.ws.xdg(t), 1, H, nwin, load8);
        else
            build_images<2>(a.ws.ximg(t), a.ws.xsg(t), a.ws.xdg(t), 1, H, nwin, load8);
        MOEQ_STAMP(0, 5);
        return;
    }
    double acc = 0.0;
    if (row < nrows) {
        double acc4[4] = {0.0, 0.0, 0.0, 0.0};  // independent fp64 add chains
        if (!bf16_row) {
            // fp32 weight x bf16 input: the product is exact in fp64
            const float *wr = reinterpret_cast<const float *>(a.w_router) + (size_t)row * H + half * hh;
            const float *xh = xs + half * hh;
            for (int j = lane * 4; j < hh; j += 128) {
                const float4 w = *reinterpret_cast<const float4 *>(wr + j);
                acc4[0] += (double)w.x * (double)xh[j];
                acc4[1] += (double)w.y * (double)xh[j + 1];
                acc4[2] += (double)w.z * (double)xh[j + 2];
                acc4[3] += (double)w.w * (double)xh[j + 3];
            }
        } else {
            // bf16 x bf16: the product is exact in fp32, the sum runs in fp64
            const float *xh = xs + half * hh;
            for (int j0 = lane * 8; j0 < hh; j0 += 256 * B) {
                if (j0 != lane * 8) {
#pragma unroll
                    for (int b = 0; b < B; ++b) {
                        const int j = j0 + 256 * b;
                        wv[b] = j < hh ? ldg_stream(reinterpret_cast<const uint32_t *>(wr16 + j)) : make_uint4(0u, 0u, 0u, 0u);
                    }
                }
#pragma unroll
                for (int b = 0; b < B; ++b) {
                    const int j = j0 + 256 * b;
                    if (j < hh) {
                        const uint32_t w[4] = {wv[b].x, wv[b].y, wv[b].z, wv[b].w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            acc4[i] += (double)(bf16_bits_to_float(w[i] & 0xffffu) * xh[j + 2 * i]);
                            acc4[i] += (double)(bf16_bits_to_float(w[i] >> 16) * xh[j + 2 * i + 1]);
                        }
                    }
                }
            }
        }
        acc = warp_sum_f64((acc4[0] + acc4[1]) + (acc4[2] + acc4[3]));
    }
    if (lane == 0) s_part[warp] = acc;
    __syncthreads();
    MOEQ_STAMP(0, 2);
    if (tid == 0) {
        // one writer per CTA: store this CTA's logits (then, with the top-k
        // here, one fence and the arrival)
        for (int r = 0; r < kRouteRowsPerCta; ++r) {
            const int rr = blockIdx.x * kRouteRowsPerCta + r;
            if (rr < nrows) {
                double l = s_part[2 * r] + s_part[2 * r + 1];
                if (rr < a.E && a.logit_bias) l += (double)a.logit_bias[(size_t)t * a.E + rr];
                if (!isfinite(l)) flag_status(a.ws.status, MOE_DEV_NONFINITE);
                a.ws.logits(t)[rr] = l;
            }
        }
        if (a.do_topk) {
            __threadfence();
            const unsigned old = atomicAdd(a.ws.route_cnt(t), 1u);
            s_last = (old == gridDim.x - 1u - (unsigned)a.build_image);
        } else {
            s_last = 0;
        }
    }
    __syncthreads();
    // Dependents (the gate/up kernel) are released once this CTA's loads are
    // done: launched any earlier, their CTAs slow this kernel's streaming.
    // x is complete by now, so they may read it before their own wait.
    griddep_launch_dependents();
    MOEQ_STAMP(0, 3);
    if (!s_last) return;
    __threadfence();
    topk_block<kRouteThreads>(a.ws.logits(t), a.E, a.k, sm);
    topk_store<kRouteThreads>(a, t, sm);
    if (tid == 0) *a.ws.route_cnt(t) = 0u;
    MOEQ_STAMP(0, 4);
}

}  // namespace moeq
