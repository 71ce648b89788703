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
// quad column c, register r, byte jj): the layout of the image.  The same
// mapping decides which code each A-fragment byte holds (see the extraction
// in compute_item), so the k-permutation inside each step is applied to both
// operands alike; build_images writes exactly these positions.
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

// Operand images of n activation vectors of length K (a multiple of 64),
// built by the whole CTA.  load8(c, f) gives chunk c = 8 consecutive values
// (chunks of all vectors numbered together: vector c / (K/8)) as fp32.
// Each group of 64 values gets its own fixed-point step, dg = max|v| / 32000
// over the group (an outlier only coarsens its own group).
//  pass 0: the n images are zeroed (entries of other groups stay zero) while
//          each thread's loads are in flight (up to KEEP rounds of chunks
//          kept in registers; longer inputs are read twice);
//  pass 1: group sums sg[j][g] and steps dg[j][g] (eight lanes per group,
//          fixed order: deterministic);
//  pass 2: each chunk is put in 16-bit fixed point, xq = rint(v / dg) =
//          256*hi + lo, and its high and low bytes go straight to the image
//          entries that hold them (image_slot: for 4-bit codes a chunk fills
//          one entry per plane; for 2-bit codes a chunk pair fills two).
// img: n images of nwin*kImgWinEntries entries; sg, dg: [n][K/64].
template <int BITS, typename Load8>
__device__ __forceinline__ void build_images(uint2 *img, float *sg, float *dg, int n, int K, int nwin, Load8 load8) {
    constexpr int KEEP = 2;
    const int tid = threadIdx.x, NT = blockDim.x, lane = tid & 31;
    const int c8 = K / 8, nch = n * c8;  // a group = 8 chunks, never across vectors
    const int rounds = (nch + NT - 1) / NT;
    const int per = nwin * kImgWinEntries;
    float f[KEEP][8], gmx[KEEP];
#pragma unroll
    for (int u = 0; u < KEEP; ++u) {
        const int c = tid + u * NT;
        if (u < rounds && c < nch)
            load8(c, f[u]);
        else
#pragma unroll
            for (int e = 0; e < 8; ++e) f[u][e] = 0.f;
    }
    uint4 *img4 = reinterpret_cast<uint4 *>(img);
    for (int i = tid; i < n * per / 2; i += NT) img4[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int r0 = 0; r0 < rounds; r0 += KEEP) {
        if (r0 > 0) {
#pragma unroll
            for (int u = 0; u < KEEP; ++u) {
                const int c = tid + (r0 + u) * NT;
                if (r0 + u < rounds && c < nch)
                    load8(c, f[u]);
                else
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[u][e] = 0.f;
            }
        }
#pragma unroll
        for (int u = 0; u < KEEP; ++u) {
            const int c = tid + (r0 + u) * NT;
            float m = 0.f, sum = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                m = fmaxf(m, fabsf(f[u][e]));
                sum += f[u][e];
            }
            // group c/8 = lanes 8q..8q+7 of this warp (NT and c8 multiples of 8)
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
                sum += __shfl_xor_sync(0xffffffffu, sum, o);
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            }
            gmx[u] = m;
            if (r0 + u < rounds && c < nch && (c & 7) == 0) {
                sg[c >> 3] = sum;
                dg[c >> 3] = m / (float)kQuantMax;
            }
        }
    }
    __syncthreads();  // images zeroed; steps of groups read back when values are reloaded
    for (int r = 0; r < rounds; ++r) {
        const int c = tid + r * NT;
        const bool in = c < nch;
        float g[8], mx = 0.f;
        if (rounds <= KEEP) {
#pragma unroll
            for (int u = 0; u < KEEP; ++u)
                if (u == r) {
                    mx = gmx[u];
#pragma unroll
                    for (int e = 0; e < 8; ++e) g[e] = f[u][e];
                }
        } else if (in) {
            load8(c, g);
            mx = dg[c >> 3] * (float)kQuantMax;
        }
        const int j = in ? c / c8 : 0, i = in ? c % c8 : 0;
        const float inv = mx > 0.f ? (float)kQuantMax / mx : 0.f;
        uint32_t hw[2] = {0u, 0u}, lw[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int q = in ? __float2int_rn(g[e] * inv) : 0;
            const int hi = (q + 128) >> 8;
            hw[e >> 2] |= (uint32_t)(hi & 0xff) << (8 * (e & 3));
            lw[e >> 2] |= (uint32_t)((q - 256 * hi) & 0xff) << (8 * (e & 3));
        }
        uint2 *im = img + (size_t)j * per;
        if (BITS == 4) {
            // chunk i = codes 8i..8i+7 = word wi of window w; step t, quad column cq
            const int w = i >> 5, wi = i & 31;
            const int t = 4 * (wi >> 4) + (wi & 3), cq = (wi >> 2) & 3, gl = wi >> 3;
            if (in) {
                im[w * kImgWinEntries + t * 32 + (2 * gl) * 4 + cq] =
                    make_uint2(__byte_perm(hw[0], hw[1], 0x6420), __byte_perm(hw[0], hw[1], 0x7531));
                im[w * kImgWinEntries + t * 32 + (2 * gl + 1) * 4 + cq] =
                    make_uint2(__byte_perm(lw[0], lw[1], 0x6420), __byte_perm(lw[0], lw[1], 0x7531));
            }
        } else {
            // chunk pair (2p, 2p+1) = codes 16p..16p+15 = word wi of window w,
            // quad column cq = group; steps 2u and 2u+1 take positions
            // {2mm + 4jj} and {2mm + 1 + 4jj}
            const uint32_t h2 = __shfl_down_sync(0xffffffffu, hw[0], 1), h3 = __shfl_down_sync(0xffffffffu, hw[1], 1);
            const uint32_t l2 = __shfl_down_sync(0xffffffffu, lw[0], 1), l3 = __shfl_down_sync(0xffffffffu, lw[1], 1);
            if (in && (lane & 1) == 0) {
                const int w = i >> 5, wi = (i >> 1) & 15;
                const int cq = wi >> 2, u = wi & 3;
#pragma unroll
                for (int mm = 0; mm < 2; ++mm) {
                    const unsigned s0 = (unsigned)(2 * mm) | ((unsigned)(2 * mm + 4) << 4);
                    const unsigned s1 = (unsigned)(2 * mm + 1) | ((unsigned)(2 * mm + 5) << 4);
                    const int t = 2 * u + mm;
                    im[w * kImgWinEntries + t * 32 + (2 * cq) * 4 + cq] =
                        make_uint2(__byte_perm(__byte_perm(hw[0], hw[1], s0), __byte_perm(h2, h3, s0), 0x5410),
                                   __byte_perm(__byte_perm(hw[0], hw[1], s1), __byte_perm(h2, h3, s1), 0x5410));
                    im[w * kImgWinEntries + t * 32 + (2 * cq + 1) * 4 + cq] =
                        make_uint2(__byte_perm(__byte_perm(lw[0], lw[1], s0), __byte_perm(l2, l3, s0), 0x5410),
                                   __byte_perm(__byte_perm(lw[0], lw[1], s1), __byte_perm(l2, l3, s1), 0x5410));
                }
            }
        }
    }
    __syncthreads();
}

}  // namespace moeq
