// ffn.cuh -- decode expert FFN kernels over 4-bit / 2-bit affine group-quantised
// weights: gate/up mat-vecs fused with SwiGLU, then down mat-vecs fused with
// the routing-weighted combine, the shared expert and the residual.
//
// Pages: "Flash-MoE - Exécuter un modèle de 397 milliards de paramètres sur un
// ordinateur portable": "Noyau de déquantification optimisé FMA" (weight =
// nibble*scale + bias, regrouped so scale and bias multiply per-group sums),
// "Shaders de calcul Metal" (4-bit/2-bit dequantising mat-vecs, SwiGLU, MoE
// combine + residual + gate), "SSD Expert Streaming" (only the active experts'
// weights are read).
//
// Arithmetic.  Per row r and group g of 64 codes, sum_j (q_j s + b) x_j =
// s * sum_j q_j x_j + b * S_g(x), S_g(x) = sum_{j in g} x_j.  The code sum is
// exact integer arithmetic: x is turned once into 16-bit fixed point
// xq = rint(x / delta), delta = max|x| / 32000, split as xq = 256*hi + lo with
// hi, lo in int8, and the tensor-core instruction mma.m16n8k32 (u8 codes x s8
// activations, s32 accumulate) sums 32 products per step.  Its 8 B-operand
// columns carry (hi, lo) for 4 groups, so one accumulator tile covers a
// "window" of 256 codes = 4 groups and each (row, group) partial stays
// separate for the per-group scale.  The only rounding on the code path is
// the fixed-point step (|error| <= delta/2 per element).
//
// Data movement.  One CTA per SM, 32 warps working independently.  A warp's
// work item is 16 rows x one window (4-bit; two for 2-bit) of one matrix; it
// loads the item's codes with 16-byte non-L1-allocating loads straight in
// the A-fragment layout (a quad of lanes reads 64 contiguous bytes of a row)
// one item ahead of the math.  (Measured on B200: 16-byte loads from 16+
// warps per SM stream ~7 TB/s, while 1-D TMA bulk copies of the 512-byte row
// pieces a row-major layout offers reach ~2 TB/s.)  A tile's item partials
// meet in a small shared-memory ring of tile slots; the warp that arrives
// last sums them in fixed order and writes the tile's result, so no
// CTA-wide barrier sits in the streaming loop and results are deterministic.
// Weight bytes are read from HBM exactly once.
#pragma once

#include "common.cuh"

namespace moeq {

enum CombineMode { kCombineFull = 0, kCombineSplit = 1 };

struct FfnArgs {
    int T, H, I, E, k, S;  // S = k + has_shared
    const uint16_t *x;     // bf16 [T][H]
    const QExpertDev *slots;
    int n_slots;
    QExpertDev shared;
    const int *idx_base;   // token t's ids at idx_base + t*idx_stride
    size_t idx_stride;
    const float *w_base;   // routing weights, same addressing
    size_t w_stride;
    const float *gamma_base;  // shared-expert gate per token, or null (gamma = 1)
    size_t gamma_stride;
    WsPtrs ws;
    const uint16_t *residual;  // bf16 [T][H] (full combine)
    uint16_t *out;             // bf16 [T][H] (full combine)
    float *ysplit;             // fp32 [T][2][H] (split combine)
    int mode;
    // 1 when the kernel before the gate/up kernel is this library's router
    // kernel, which releases its dependents only once x is complete; the
    // gate/up prologue may then read x before its own dependency wait.
    int x_ready_early;
    int ring_slots;            // tile slots of the shared-memory partial ring
};

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

// ------------------------------------------------------------ work items

// An item: 16 rows (a tile) x NWI windows of NMAT matrices (gate and up
// together, or down), loaded by one warp straight into A-fragment registers.
template <int BITS, int NMAT, int NWI>
struct Item {
    uint4 q[NWI][NMAT][2][BITS / 2];  // [window][matrix][row g / g+8][16-byte piece]
    uint32_t sb[NWI][NMAT][2];        // bf16 scale | bias << 16 for (row, group 4w+c)
};

// Loads one item: rows row0 + {g, g+8} of each matrix, windows w0...  With
// FULL (K a multiple of NWI windows) every access is in range and nothing is
// predicated; otherwise pieces past the row end read as zero.
template <int BITS, int NMAT, int NWI, bool FULL>
__device__ __forceinline__ void load_item(Item<BITS, NMAT, NWI> &R, const QMatDev (&M)[NMAT], int row0, int w0,
                                          int Kwords, int ngroups, int lane) {
    const int g = lane >> 2, c = lane & 3;
    constexpr int WPW = kWinK * BITS / 32;  // words per row per window
#pragma unroll
    for (int wi = 0; wi < NWI; ++wi)
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int row = row0 + g + 8 * rr;
                const int off0 = (w0 + wi) * WPW + 4 * c;
                const uint32_t *rp = M[m].codes + (size_t)row * Kwords + off0;
#pragma unroll
                for (int i = 0; i < BITS / 2; ++i)
                    R.q[wi][m][rr][i] = (FULL || off0 + 16 * i < Kwords) ? ldg_stream(rp + 16 * i)
                                                                         : make_uint4(0u, 0u, 0u, 0u);
                const int grp = 4 * (w0 + wi) + c;
                uint32_t sb = 0u;
                if (FULL || grp < ngroups) {
                    const size_t o = (size_t)row * ngroups + grp;
                    sb = ldg_u16(M[m].scale + o) | (ldg_u16(M[m].bias + o) << 16);
                }
                R.sb[wi][m][rr] = sb;
            }
}

template <int BITS, int NMAT, int NWI>
__device__ __forceinline__ void zero_item(Item<BITS, NMAT, NWI> &R) {
#pragma unroll
    for (int wi = 0; wi < NWI; ++wi)
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
#pragma unroll
                for (int i = 0; i < BITS / 2; ++i) R.q[wi][m][rr][i] = make_uint4(0u, 0u, 0u, 0u);
                R.sb[wi][m][rr] = 0u;
            }
}

// Activation-operand fragments of windows w0.. (8 MMA steps each), zero for
// windows past the end.
template <int NWI>
__device__ __forceinline__ void load_bfrag(uint2 (&bf)[NWI][kMmaPerWin], const uint2 *img, int w0, int nwin,
                                           int lane) {
#pragma unroll
    for (int wi = 0; wi < NWI; ++wi)
#pragma unroll
        for (int t = 0; t < kMmaPerWin; ++t)
            bf[wi][t] = (w0 + wi < nwin) ? img[(size_t)(w0 + wi) * kImgWinEntries + t * 32 + lane] : make_uint2(0u, 0u);
}

// Row partial sums of one item over its windows; after the quad reduction
// every lane of quad g holds rows g (v0[m]) and g+8 (v8[m]).
template <int BITS, int NMAT, int NWI>
__device__ __forceinline__ void compute_item(const Item<BITS, NMAT, NWI> &R, const uint2 (&bf)[NWI][kMmaPerWin],
                                             const float *sg, int w0, int ngroups, float delta, int lane,
                                             float (&v0)[NMAT], float (&v8)[NMAT]) {
    const int c = lane & 3;
#pragma unroll
    for (int m = 0; m < NMAT; ++m) v0[m] = v8[m] = 0.f;
#pragma unroll
    for (int wi = 0; wi < NWI; ++wi) {
        int acc[NMAT][4];
#pragma unroll
        for (int m = 0; m < NMAT; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0;
#pragma unroll
        for (int t = 0; t < kMmaPerWin; ++t) {
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
                uint32_t a0, a1, a2, a3;
                if (BITS == 4) {
                    // a0/a1: even nibbles of rows g/g+8, a2/a3: odd nibbles
                    const uint32_t x0 = u4_word(R.q[wi][m][0][t >> 2], t & 3);
                    const uint32_t x8 = u4_word(R.q[wi][m][1][t >> 2], t & 3);
                    a0 = x0 & 0x0F0F0F0Fu;
                    a1 = x8 & 0x0F0F0F0Fu;
                    a2 = (x0 >> 4) & 0x0F0F0F0Fu;
                    a3 = (x8 >> 4) & 0x0F0F0F0Fu;
                } else {
                    // word holds 16 codes; step t takes code positions
                    // {2mm + 4jj} (a0/a1) and {2mm + 1 + 4jj} (a2/a3)
                    const uint32_t x0 = u4_word(R.q[wi][m][0][0], t >> 1);
                    const uint32_t x8 = u4_word(R.q[wi][m][1][0], t >> 1);
                    const int sh = 4 * (t & 1);
                    a0 = (x0 >> sh) & 0x03030303u;
                    a1 = (x8 >> sh) & 0x03030303u;
                    a2 = (x0 >> (sh + 2)) & 0x03030303u;
                    a3 = (x8 >> (sh + 2)) & 0x03030303u;
                }
                mma_u8s8(acc[m], a0, a1, a2, a3, bf[wi][t].x, bf[wi][t].y);
            }
        }
        // accumulator columns (2c, 2c+1) = (hi, lo) sums of group 4w + c
        const int grp = 4 * (w0 + wi) + c;
        const float S = grp < ngroups ? sg[grp] : 0.f;
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
            const float d0 = (float)(acc[m][0] * 256 + acc[m][1]);
            const float d8 = (float)(acc[m][2] * 256 + acc[m][3]);
            const uint32_t s0 = R.sb[wi][m][0], s8 = R.sb[wi][m][1];
            v0[m] += fmaf(bf16_bits_to_float(s0 & 0xffffu) * d0, delta, bf16_bits_to_float(s0 >> 16) * S);
            v8[m] += fmaf(bf16_bits_to_float(s8 & 0xffffu) * d8, delta, bf16_bits_to_float(s8 >> 16) * S);
        }
    }
#pragma unroll
    for (int m = 0; m < NMAT; ++m) {
        v0[m] += __shfl_xor_sync(0xffffffffu, v0[m], 1);
        v0[m] += __shfl_xor_sync(0xffffffffu, v0[m], 2);
        v8[m] += __shfl_xor_sync(0xffffffffu, v8[m], 1);
        v8[m] += __shfl_xor_sync(0xffffffffu, v8[m], 2);
    }
}

// ------------------------------------------------------- expert resolution

// Fills sx[0..S) with token t's experts (routed slots then the shared one)
// and sok[] with their validity; flags problems in the status word.
__device__ void resolve_experts(const FfnArgs &a, int t, QExpertDev *sx, int *sok) {
    for (int s = threadIdx.x; s < a.S; s += blockDim.x) {
        QExpertDev ex = a.shared;
        bool ok = true;
        if (s < a.k) {
            const int id = a.idx_base[(size_t)t * a.idx_stride + s];
            if (id < 0 || id >= a.n_slots) {
                flag_status(a.ws.status, MOE_DEV_BAD_EXPERT_ID);
                ok = false;
            } else {
                ex = a.slots[id];
            }
        }
        if (ok && !(qmat_ok(ex.gate) && qmat_ok(ex.up) && qmat_ok(ex.down))) {
            flag_status(a.ws.status, MOE_DEV_BAD_SLOT);
            ok = false;
        }
        sx[s] = ex;
        sok[s] = ok;
    }
}

// ------------------------------------------------------ tile-slot ring

// Partial sums of tiles meet in R slots of shared memory: tile number j of
// this CTA's sequence uses slot j % R once the slot's epoch says tile j - R
// has finished.  Each of the tile's nwg items adds its partial; the warp that
// arrives last (shared-memory counter) sums them in item order, writes the
// tile's result and opens the slot for tile j + R.
struct TileRing {
    float *part;   // [R][nwg][vals]
    int *cnt;      // [R]
    int *epoch;    // [R]
    int R, lgR, nwg, vals;  // R = 1 << lgR
    __device__ __forceinline__ int slot(int j) const { return j & (R - 1); }
    __device__ __forceinline__ int round(int j) const { return j >> lgR; }
};

__device__ __forceinline__ void ring_init(const TileRing &r) {
    for (int i = threadIdx.x; i < r.R; i += blockDim.x) {
        r.cnt[i] = 0;
        r.epoch[i] = 0;
    }
}

// Waits (bounded) until tile j may use its slot; warp-uniform.
__device__ __forceinline__ void ring_acquire(const TileRing &r, int j, int *status) {
    volatile int *ep = r.epoch + r.slot(j);
    const int want = r.round(j);
    if (*ep == want) return;
    const unsigned long long t0 = globaltimer_ns();
    while (*ep != want) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            flag_status(status, MOE_DEV_TIMEOUT);
            return;
        }
    }
}

// Deposits this warp's partials (lanes of quad g hold rows g, g+8 of each
// matrix); returns true (to the whole warp) when this warp completed the
// tile, i.e. was the last of its `arrivals` items.
template <int NMAT>
__device__ __forceinline__ bool ring_deposit(const TileRing &r, int j, int wg, const float (&v0)[NMAT],
                                             const float (&v8)[NMAT], int lane, int arrivals) {
    const int slot = r.slot(j);
    float *pp = r.part + ((size_t)slot * r.nwg + wg) * r.vals;
    if ((lane & 3) == 0) {
        const int g = lane >> 2;
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
            pp[m * kTileRows + g] = v0[m];
            pp[m * kTileRows + g + 8] = v8[m];
        }
    }
    __threadfence_block();
    __syncwarp();
    int last = 0;
    if (lane == 0) last = (atomicAdd(r.cnt + slot, 1) == arrivals - 1);
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) __threadfence_block();
    return last != 0;
}

// Sum over the tile's items (fixed order) of value v (matrix m, row row).
__device__ __forceinline__ float ring_sum(const TileRing &r, int j, int m, int row) {
    const float *pp = r.part + (size_t)r.slot(j) * r.nwg * r.vals + m * kTileRows + row;
    float acc = 0.f;
    for (int wg = 0; wg < r.nwg; ++wg) acc += pp[(size_t)wg * r.vals];
    return acc;
}

__device__ __forceinline__ void ring_release(const TileRing &r, int j, int lane) {
    __syncwarp();
    if (lane == 0) {
        const int slot = r.slot(j);
        r.cnt[slot] = 0;
        __threadfence_block();
        *(volatile int *)(r.epoch + slot) = r.round(j) + 1;
    }
    __syncwarp();
}

// Streams the items of tiles [gt0, gt0 + n) of the flat (expert slot s,
// row tile rt) space, tps row tiles per slot; the tiles take ring numbers
// j0, j0 + 1, ...  A tile is nwg items of NWI windows each (all NMAT
// matrices of the window together); mat_of(s, M, ok) gives slot s's
// matrices.  Items go in tile-major order, warp w taking items w, w+16, ...;
// two register buffers alternate so each item's loads are issued one item
// ahead of its math; positions advance incrementally.  The activation
// fragments stay in registers while consecutive items of a warp use the same
// window and image.  finish(jl, s, rt) runs on the warp that completes tile
// jl (the ring slot still holds its sums).
template <int BITS, int NMAT, int NWI, bool FULL, typename MatOf, typename ImgOf, typename Finish>
__device__ void stream_items(const TileRing &ring, int j0, int gt0, int n, int tps, int K, MatOf mat_of,
                             ImgOf img_of, Finish finish, int *status) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwin = (K + kWinK - 1) / kWinK;
    const int nwg = (nwin + NWI - 1) / NWI;
    const int ngroups = K / kGroup;
    const int Kwords = K * BITS / 32;
    const int nitems = n * nwg;
    if (warp >= nitems) return;
    struct Pos {
        int it, jl, r, s, rt;  // item, ring tile number, window group, slot, row tile
    };
    auto advance = [&](Pos p) {
        p.it += kFfnWarps;
        p.r += kFfnWarps;
        while (p.r >= nwg) {
            p.r -= nwg;
            ++p.jl;
            if (++p.rt == tps) {
                p.rt = 0;
                ++p.s;
            }
        }
        return p;
    };
    using It = Item<BITS, NMAT, NWI>;
    auto issue = [&](It &R, const Pos &p) {
        if (p.it < nitems) {
            QMatDev M[NMAT];
            bool ok;
            mat_of(p.s, M, ok);
            if (ok)
                load_item<BITS, NMAT, NWI, FULL>(R, M, p.rt * kTileRows, p.r * NWI, Kwords, ngroups, lane);
            else
                zero_item(R);  // unusable expert (flagged): contributes zero
        }
    };
    uint2 bf[NWI][kMmaPerWin];
    const uint2 *bf_img = nullptr;
    int bf_w = -1;
    auto consume = [&](const It &R, const Pos &p) {
        const uint2 *img;
        const float *sg;
        float delta;
        img_of(p.s, img, sg, delta);
        const int w0 = p.r * NWI;
        if (img != bf_img || w0 != bf_w) {  // warp-uniform
            load_bfrag<NWI>(bf, img, w0, nwin, lane);
            bf_img = img;
            bf_w = w0;
        }
        float v0[NMAT], v8[NMAT];
        compute_item<BITS, NMAT, NWI>(R, bf, sg, w0, ngroups, delta, lane, v0, v8);
        ring_acquire(ring, p.jl, status);
        if (ring_deposit<NMAT>(ring, p.jl, p.r, v0, v8, lane, nwg)) {
            finish(p.jl, p.s, p.rt);
            ring_release(ring, p.jl, lane);
        }
    };
    const int t0 = gt0 + warp / nwg;
    Pos pa{warp, j0 + warp / nwg, warp % nwg, t0 / tps, t0 % tps};
    It A, B;
    issue(A, pa);
    while (true) {
        const Pos pb = advance(pa);
        issue(B, pb);
        consume(A, pa);
        if (pb.it >= nitems) break;
        pa = advance(pb);
        issue(A, pa);
        consume(B, pb);
        if (pa.it >= nitems) break;
    }
}

// ---------------------------------------------------------------- gate/up

// Gate/up mat-vecs and SwiGLU.  Work: tiles of 16 rows of (gate, up) of one
// selected expert; this CTA takes a contiguous slice of the token's
// S*I/16 tiles.  Shared memory: image | xh, xl | ring part | cnt | epoch.
template <int BITS, bool FULL>
__global__ void __launch_bounds__(kFfnThreads, 1) k_gateup(FfnArgs a) {
    constexpr int NWI = 1;
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ float red[kFfnWarps];
    __shared__ float sg[kMaxDim / kGroup];
    __shared__ QExpertDev sx[kMaxTopK + 1];
    __shared__ int sok[kMaxTopK + 1];
    const int H = a.H, I = a.I;
    const int nwin = (H + kWinK - 1) / kWinK;
    const int nwg = (nwin + NWI - 1) / NWI;
    uint2 *img = reinterpret_cast<uint2 *>(smem);
    int8_t *xh = reinterpret_cast<int8_t *>(img + (size_t)nwin * kImgWinEntries);
    int8_t *xl = xh + nwin * kWinK;
    TileRing ring;
    ring.part = reinterpret_cast<float *>(xl + nwin * kWinK);
    ring.R = a.ring_slots;
    ring.lgR = __ffs(ring.R) - 1;
    ring.nwg = nwg;
    ring.vals = 2 * kTileRows;  // gate rows then up rows
    ring.cnt = reinterpret_cast<int *>(ring.part + (size_t)ring.R * nwg * ring.vals);
    ring.epoch = ring.cnt + ring.R;
    const int tps = I / kTileRows;
    const int ntiles = a.S * tps;
    const int P = gridDim.x;
    const int tb = (int)((long long)ntiles * blockIdx.x / P);
    const int te = (int)((long long)ntiles * (blockIdx.x + 1) / P);
    const int lane = threadIdx.x & 31;
    MOEQ_STAMP(1, 0);
    ring_init(ring);
    if (!a.x_ready_early) griddep_wait();
    int jseq = 0;
    for (int t = 0; t < a.T; ++t) {
        // activation image of x[t]: independent of the routing, so (after the
        // router kernel) it is built before waiting on it
        const uint4 *xt = reinterpret_cast<const uint4 *>(a.x + (size_t)t * H);
        auto load8 = [&](int i, float(&f)[8]) {
            const uint4 v = __ldg(xt + i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                f[2 * u] = bf16_bits_to_float(w[u] & 0xffffu);
                f[2 * u + 1] = bf16_bits_to_float(w[u] >> 16);
            }
        };
        const float delta = prep_image<BITS>(img, xh, xl, sg, red, H, nwin, load8);
        MOEQ_STAMP(1, 1);
        if (t == 0 && a.x_ready_early) griddep_wait();  // routing results of the router kernel
        MOEQ_STAMP(1, 2);
        resolve_experts(a, t, sx, sok);
        __syncthreads();
        MOEQ_STAMP(1, 3);
        auto mat_of = [&](int s, QMatDev (&M)[2], bool &ok) {
            M[0] = sx[s].gate;
            M[1] = sx[s].up;
            ok = sok[s] != 0;
        };
        auto img_of = [&](int, const uint2 *&im, const float *&sgp, float &d) {
            im = img;
            sgp = sg;
            d = delta;
        };
        auto finish = [&](int jl, int s, int rt) {
            if (lane < kTileRows) {
                const float gs = ring_sum(ring, jl, 0, lane);
                const float us = ring_sum(ring, jl, 1, lane);
                a.ws.h(t)[(size_t)s * I + rt * kTileRows + lane] = gs / (1.f + expf(-gs)) * us;
            }
        };
        stream_items<BITS, 2, NWI, FULL>(ring, jseq, tb, te - tb, tps, H, mat_of, img_of, finish, a.ws.status);
        MOEQ_STAMP_MAX(1, 4);
        jseq += te - tb;
        __syncthreads();  // image and expert table are rebuilt for the next token
    }
    MOEQ_STAMP(1, 5);
    griddep_launch_dependents();  // after the streaming, so the next kernel does not compete with it
}

// ------------------------------------------------------------------- down

// Finish of a down tile (16 output rows of expert slot s): its partial
// output goes to the workspace; the last of the S contributions to the row
// band (global arrival count) sums them in fixed order with the routing
// weights w[], the gated shared expert and the residual.
__device__ __forceinline__ void down_finish(const FfnArgs &a, int t, const TileRing &ring, int jl, int s, int rt,
                                            int lane, const float *w, float gm) {
    const int H = a.H;
    const int col = rt * kTileRows + lane;
    float *yp = a.ws.ypart(t);
    if (lane < kTileRows) {
        yp[(size_t)s * H + col] = ring_sum(ring, jl, 0, lane);
        __threadfence();
    }
    __syncwarp();
    int done = 0;
    if (lane == 0) {
        unsigned *cnt = a.ws.band_cnt(t) + rt;
        done = (atomicAdd(cnt, 1u) == (unsigned)a.S - 1u);
        if (done) *cnt = 0u;  // every contribution to this band has arrived
    }
    done = __shfl_sync(0xffffffffu, done, 0);
    if (done && lane < kTileRows) {
        __threadfence();
        float yr = 0.f;
        for (int i = 0; i < a.k; ++i) yr += w[i] * __ldcg(yp + (size_t)i * H + col);
        const float ysh = (a.S > a.k) ? __ldcg(yp + (size_t)a.k * H + col) : 0.f;
        if (a.mode == kCombineFull) {
            const float r0 = bf16_bits_to_float(a.residual[(size_t)t * H + col]);
            a.out[(size_t)t * H + col] = __bfloat16_as_ushort(__float2bfloat16_rn(r0 + yr + gm * ysh));
        } else {
            a.ysplit[((size_t)t * 2) * H + col] = yr;
            a.ysplit[((size_t)t * 2 + 1) * H + col] = ysh;
        }
    }
}


// Down mat-vecs: tiles of 16 output rows of one selected expert; the tile's
// partial output goes to the workspace and the last of the S contributions to
// a row band (global arrival count) sums them in fixed order with the
// routing weights, the gated shared expert and the residual.  The per-expert
// activation images (of h) are built for at most kMaxImgSlots experts at a
// time.  Shared memory: images | xh, xl | ring part | cnt | epoch.
template <int BITS, bool FULL>
__global__ void __launch_bounds__(kFfnThreads, 1) k_down(FfnArgs a) {
    constexpr int NWI = BITS == 4 ? 1 : 2;
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ float red[kFfnWarps];
    __shared__ float sgs[kMaxImgSlots][kMaxDim / kGroup];
    __shared__ float sdelta[kMaxImgSlots];
    __shared__ QExpertDev sx[kMaxTopK + 1];
    __shared__ int sok[kMaxTopK + 1];
    const int H = a.H, I = a.I;
    const int nwin = (I + kWinK - 1) / kWinK;
    const int nwg = (nwin + NWI - 1) / NWI;
    const size_t img_slot = (size_t)nwin * kImgWinEntries;
    uint2 *img = reinterpret_cast<uint2 *>(smem);
    int8_t *xh = reinterpret_cast<int8_t *>(img + kMaxImgSlots * img_slot);
    int8_t *xl = xh + nwin * kWinK;
    TileRing ring;
    ring.part = reinterpret_cast<float *>(xl + nwin * kWinK);
    ring.R = a.ring_slots;
    ring.lgR = __ffs(ring.R) - 1;
    ring.nwg = nwg;
    ring.vals = kTileRows;
    ring.cnt = reinterpret_cast<int *>(ring.part + (size_t)ring.R * nwg * ring.vals);
    ring.epoch = ring.cnt + ring.R;
    const int tps = H / kTileRows;
    const int ntiles = a.S * tps;
    const int P = gridDim.x;
    const int tb = (int)((long long)ntiles * blockIdx.x / P);
    const int te = (int)((long long)ntiles * (blockIdx.x + 1) / P);
    const int lane = threadIdx.x & 31;
    MOEQ_STAMP(2, 0);
    ring_init(ring);
    griddep_wait();  // h from the gate/up kernel
    MOEQ_STAMP(2, 1);
    int jseq = 0;
    for (int t = 0; t < a.T; ++t) {
        if (tb >= te) break;
        resolve_experts(a, t, sx, sok);
        for (int pb = tb; pb < te;) {
            const int sb = pb / tps;
            const int pe = min(te, (sb + kMaxImgSlots) * tps);
            const int se = (pe - 1) / tps;
            for (int s = sb; s <= se; ++s) {
                __syncthreads();
                const float4 *hv = reinterpret_cast<const float4 *>(a.ws.h(t) + (size_t)s * I);
                auto load8 = [&](int i, float(&f)[8]) {
                    const float4 u = __ldcg(hv + 2 * i), v = __ldcg(hv + 2 * i + 1);
                    f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
                    f[4] = v.x; f[5] = v.y; f[6] = v.z; f[7] = v.w;
                };
                const float d = prep_image<BITS>(img + (s - sb) * img_slot, xh, xl, sgs[s - sb], red, I, nwin, load8);
                if (threadIdx.x == 0) sdelta[s - sb] = d;
            }
            __syncthreads();
            MOEQ_STAMP(2, 2);
            const int jp = jseq;
            auto mat_of = [&](int s, QMatDev (&M)[1], bool &ok) {
                M[0] = sx[s].down;
                ok = sok[s] != 0;
            };
            auto img_of = [&](int s, const uint2 *&im, const float *&sgp, float &d) {
                im = img + (s - sb) * img_slot;
                sgp = sgs[s - sb];
                d = sdelta[s - sb];
            };
            auto finish = [&](int jl, int s, int rt) {
                down_finish(a, t, ring, jl, s, rt, lane, a.w_base + (size_t)t * a.w_stride,
                            a.gamma_base ? a.gamma_base[(size_t)t * a.gamma_stride] : 1.f);
            };
            stream_items<BITS, 1, NWI, FULL>(ring, jp, pb, pe - pb, tps, I, mat_of, img_of, finish, a.ws.status);
            MOEQ_STAMP_MAX(2, 3);
            jseq += pe - pb;
            pb = pe;
        }
        __syncthreads();
    }
    MOEQ_STAMP(2, 4);
    griddep_launch_dependents();
}

// out = residual + y0 + gamma * y1 per token (gamma from the shared gate).
// grid T, block 256.
__global__ void __launch_bounds__(256) k_combine(const float *y, const uint16_t *residual,
                                                 const uint16_t *gate, const uint16_t *x, int H,
                                                 uint16_t *out) {
    __shared__ double red[8];
    const int t = blockIdx.x;
    griddep_wait();
    griddep_launch_dependents();
    float gm = 1.f;
    if (gate) {
        double acc = 0.0;
        for (int j = threadIdx.x; j < H; j += blockDim.x)
            acc += (double)(bf16_bits_to_float(gate[j]) * bf16_bits_to_float(x[(size_t)t * H + j]));
        acc = warp_sum_f64(acc);
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
        __syncthreads();
        double z = 0.0;
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i) z += red[i];
        gm = (float)(1.0 / (1.0 + exp(-z)));
    }
    for (int j = threadIdx.x; j < H; j += blockDim.x) {
        const float o = bf16_bits_to_float(residual[(size_t)t * H + j]) + y[(size_t)t * 2 * H + j] +
                        gm * y[((size_t)t * 2 + 1) * H + j];
        out[(size_t)t * H + j] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
    }
}

}  // namespace moeq
