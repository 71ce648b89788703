// image.cuh -- the activation operand image of the decode mat-vecs: an
// activation vector in 16-bit fixed point, split into int8 high and low
// planes and laid out as the B fragments of mma.m16n8k32 (8 columns = high
// and low plane of the 4 groups of a 256-code window).
//
// Pages: "Flash-MoE - Exécuter un modèle de 397 milliards de paramètres sur un
// ordinateur portable", "Noyau de déquantification optimisé FMA": the
// regrouped dot product s * sum(q x) + b * sum(x) per group, whose code sums
// this image makes exact integer sums.
#pragma once

#include "common.cuh"

namespace moeq {

// ------------------------------------------------------------ operand image

// k index and in-window group of operand byte (window w, MMA step t, lane's
// quad column c, register r, byte jj).  The same mapping decides which code
// each A-fragment byte holds (see the extraction in compute_item), so the
// k-permutation inside each step is applied to both operands alike.
template <int BITS>
__device__ __forceinline__ void image_slot(int w, int t, int c, int &kbase, int &gl) {
    if (BITS == 4) {
        const int i = t >> 2, u = t & 3, wi = 16 * i + 4 * c + u;  // word of the window
        kbase = w * kWinK + 8 * wi;  // byte jj of register r holds code kbase + 2*jj + r
        gl = wi >> 3;
    } else {
        const int u = t >> 1, mm = t & 1, wi = 4 * c + u;
        kbase = w * kWinK + 16 * wi + 2 * mm;  // byte jj of register r holds code kbase + r + 4*jj
        gl = wi >> 2;
    }
}

// Operand image of a length-K activation vector, CTA-wide, in two passes.
// load8(i, f) gives elements 8i..8i+7 as fp32.
//  pass 1: max|v| and the group sums sg[g] (eight lanes per group, fixed
//          order: deterministic);
//  pass 2: fixed-point planes xh, xl (xq = rint(v / delta) = 256*hi + lo,
//          lo in [-128, 127]; zero past K up to nwin*256);
//  pass 3: the image itself.  Lane (gq, c) of step t holds, for B column
//          gq = 2*group + plane, the hi (plane 0) or lo (plane 1) bytes at its
//          k slots when that slot's group is `group`, else 0.
// Returns delta = max|v| / 32000.
template <int BITS, typename Load8>
__device__ float prep_image(uint2 *img, int8_t *xh, int8_t *xl, float *sg, float *red, int K, int nwin,
                            Load8 load8) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n8 = K / 8;
    const int rounds = (n8 + (int)blockDim.x - 1) / (int)blockDim.x;
    float m = 0.f;
    for (int r = 0; r < rounds; ++r) {
        const int i = tid + r * blockDim.x;
        float f[8];
        float s = 0.f;
        if (i < n8) {
            load8(i, f);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                m = fmaxf(m, fabsf(f[u]));
                s += f[u];
            }
        }
        // group i/8 = lanes 8q..8q+7 of this warp (blockDim is a multiple of 8)
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s += __shfl_xor_sync(0xffffffffu, s, 4);
        if (i < n8 && (i & 7) == 0) sg[i >> 3] = s;
    }
    m = warp_max_f32(m);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    float mx = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) mx = fmaxf(mx, red[w]);
    const float inv = mx > 0.f ? (float)kQuantMax / mx : 0.f;
    const int n8pad = nwin * kWinK / 8;
    for (int i = tid; i < n8pad; i += blockDim.x) {
        uint32_t h[2] = {0u, 0u}, l[2] = {0u, 0u};
        if (i < n8) {
            float f[8];
            load8(i, f);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int q = __float2int_rn(f[u] * inv);
                const int hi = (q + 128) >> 8;
                h[u >> 2] |= (uint32_t)(hi & 0xff) << (8 * (u & 3));
                l[u >> 2] |= (uint32_t)((q - 256 * hi) & 0xff) << (8 * (u & 3));
            }
        }
        *reinterpret_cast<uint2 *>(xh + 8 * i) = make_uint2(h[0], h[1]);
        *reinterpret_cast<uint2 *>(xl + 8 * i) = make_uint2(l[0], l[1]);
    }
    __syncthreads();
    const int total = nwin * kImgWinEntries;
    for (int e = tid; e < total; e += blockDim.x) {
        const int ln = e & 31, t = (e >> 5) & 7, w = e >> 8;
        const int gq = ln >> 2, c = ln & 3;
        int kb, gl;
        image_slot<BITS>(w, t, c, kb, gl);
        uint2 out = make_uint2(0u, 0u);
        if (gl == (gq >> 1)) {
            const int8_t *P = (gq & 1) ? xl : xh;
            if (BITS == 4) {
                const uint2 v8 = *reinterpret_cast<const uint2 *>(P + kb);  // codes kb..kb+7
                out.x = __byte_perm(v8.x, v8.y, 0x6420);  // even k: kb + 2jj
                out.y = __byte_perm(v8.x, v8.y, 0x7531);  // odd k:  kb + 2jj + 1
            } else {
                const int base = kb & ~15, mm2 = kb & 15;  // the word's 16 codes; step offset 2*mm
                const uint4 v16 = *reinterpret_cast<const uint4 *>(P + base);
                const unsigned s0 = (unsigned)mm2 | ((unsigned)(mm2 + 4) << 4);
                const unsigned s1 = (unsigned)(mm2 + 1) | ((unsigned)(mm2 + 5) << 4);
                out.x = __byte_perm(__byte_perm(v16.x, v16.y, s0), __byte_perm(v16.z, v16.w, s0), 0x5410);
                out.y = __byte_perm(__byte_perm(v16.x, v16.y, s1), __byte_perm(v16.z, v16.w, s1), 0x5410);
            }
        }
        img[e] = out;
    }
    __syncthreads();
    return mx / (float)kQuantMax;
}

}  // namespace moeq
