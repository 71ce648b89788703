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
// Data movement.  Weights are read once, with 16-byte non-L1-allocating loads
// in the A-fragment layout directly from the row-major code arrays (one quad of
// lanes reads 64 contiguous bytes of a row), one work item ahead of the math,
// so 16 warps keep ~64 KB per SM in flight.  The activation operand ("image",
// 2 KB per window) is built once per CTA in shared memory.
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

// v: K fp32 values in shared memory.  Writes nwin windows of uint2 operand
// words: lane (gq, c) of step t holds, for B column gq = 2*group + plane, the
// hi (plane 0) or lo (plane 1) byte of the fixed-point activation at its k
// slots when that slot's group is `group`, else 0.
template <int BITS>
__device__ void build_image(uint2 *img, const float *v, int K, float inv, int nwin) {
    const int total = nwin * kImgWinEntries;
    for (int e = threadIdx.x; e < total; e += blockDim.x) {
        const int lane = e & 31, t = (e >> 5) & 7, w = e >> 8;
        const int gq = lane >> 2, c = lane & 3;
        int kb, gl;
        image_slot<BITS>(w, t, c, kb, gl);
        uint32_t b[2] = {0u, 0u};
        if (gl == (gq >> 1)) {
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int kk = (BITS == 4) ? kb + 2 * jj + r : kb + r + 4 * jj;
                    int val = 0;
                    if (kk < K) {
                        const int q = __float2int_rn(v[kk] * inv);
                        const int hi = (q + 128) >> 8;  // q = 256*hi + lo, lo in [-128, 127]
                        val = (gq & 1) ? (q - 256 * hi) : hi;
                    }
                    b[r] |= (uint32_t)(val & 0xff) << (8 * jj);
                }
        }
        img[e] = make_uint2(b[0], b[1]);
    }
}

// max|v| (returned to all threads through red[]) and per-group sums sg[].
// Uses red[0..kFfnWarps].  Fixed reduction order: deterministic.
__device__ float vec_stats(const float *v, int K, float *sg, float *red) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    float m = 0.f;
    for (int j = threadIdx.x; j < K; j += blockDim.x) m = fmaxf(m, fabsf(v[j]));
    m = warp_max_f32(m);
    if (lane == 0) red[warp] = m;
    for (int g = warp; g < K / kGroup; g += nw) {
        float s = v[g * kGroup + lane] + v[g * kGroup + 32 + lane];
        s = warp_sum_f32(s);
        if (lane == 0) sg[g] = s;
    }
    __syncthreads();
    if (warp == 0) {
        float mm = lane < nw ? red[lane] : 0.f;
        mm = warp_max_f32(mm);
        if (lane == 0) red[kFfnWarps] = mm;
    }
    __syncthreads();
    return red[kFfnWarps];
}

// ------------------------------------------------------------ work items

template <int BITS, int NMAT, int NWI>
struct ItemRegs {
    uint4 q[NWI][NMAT][2][BITS / 2];  // [window][matrix][row g / g+8][16-byte chunk]
    uint32_t sb[NWI][NMAT][2];        // bf16 scale | bias << 16 for (row, group 4w+c)
};

template <int NMAT>
struct Mats {
    QMatDev m[NMAT];
};

// Loads one item: rows row0 + {g, g+8} of each matrix, windows w0..w0+NWI-1.
template <int BITS, int NMAT, int NWI>
__device__ __forceinline__ void load_item(ItemRegs<BITS, NMAT, NWI> &R, const Mats<NMAT> &M,
                                          bool valid, int row0, int w0, int Kwords, int ngroups,
                                          int lane) {
    const int g = lane >> 2, c = lane & 3;
    constexpr int WPW = kWinK * BITS / 32;  // words per row per window
#pragma unroll
    for (int wi = 0; wi < NWI; ++wi)
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int row = row0 + g + 8 * rr;
                const uint32_t *rp = M.m[m].codes + (size_t)row * Kwords;
#pragma unroll
                for (int i = 0; i < BITS / 2; ++i) {
                    const int off = (w0 + wi) * WPW + 16 * i + 4 * c;
                    R.q[wi][m][rr][i] = (valid && off < Kwords) ? ldg_stream(rp + off)
                                                                : make_uint4(0u, 0u, 0u, 0u);
                }
                const int grp = 4 * (w0 + wi) + c;
                uint32_t sb = 0u;
                if (valid && grp < ngroups) {
                    const size_t o = (size_t)row * ngroups + grp;
                    sb = ldg_u16(M.m[m].scale + o) | (ldg_u16(M.m[m].bias + o) << 16);
                }
                R.sb[wi][m][rr] = sb;
            }
}

// Row partial sums of one item over its windows; after the quad reduction
// every lane of quad g holds rows g (v0) and g+8 (v8).
template <int BITS, int NMAT, int NWI>
__device__ __forceinline__ void compute_item(const ItemRegs<BITS, NMAT, NWI> &R, const uint2 *img,
                                             const float *sg, int w0, int nwin, int ngroups,
                                             float delta, int lane, float (&v0)[NMAT],
                                             float (&v8)[NMAT]) {
    const int c = lane & 3;
#pragma unroll
    for (int m = 0; m < NMAT; ++m) v0[m] = v8[m] = 0.f;
#pragma unroll
    for (int wi = 0; wi < NWI; ++wi) {
        const int w = w0 + wi;
        if (w < nwin) {
            int acc[NMAT][4];
#pragma unroll
            for (int m = 0; m < NMAT; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0;
            const uint2 *iw = img + (size_t)w * kImgWinEntries;
#pragma unroll
            for (int t = 0; t < kMmaPerWin; ++t) {
                const uint2 b = iw[t * 32 + lane];
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
                    mma_u8s8(acc[m], a0, a1, a2, a3, b.x, b.y);
                }
            }
            // accumulator columns (2c, 2c+1) = (hi, lo) sums of group 4w + c
            const int grp = 4 * w + c;
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

// ---------------------------------------------------------------- gate/up

// Gate/up mat-vecs and SwiGLU.  Work: tiles of 16 rows of (gate, up) of one
// selected expert; tile range of this CTA is a contiguous slice of
// [0, S*I/16); its 16 warps split each tile's windows, a round = TPR tiles.
template <int BITS>
__global__ void __launch_bounds__(kFfnThreads, 1) k_gateup(FfnArgs a) {
    constexpr int NWI = (BITS == 4) ? 1 : 2;
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ float red[kFfnWarps + 1];
    __shared__ QExpertDev sx[kMaxTopK + 1];
    __shared__ int sok[kMaxTopK + 1];
    const int H = a.H, I = a.I;
    const int nwin = (H + kWinK - 1) / kWinK;
    const int nwg = (nwin + NWI - 1) / NWI;
    const int ngroups = H / kGroup;
    const int Kwords = H * BITS / 32;
    const int tps = I / kTileRows;
    const int ntiles = a.S * tps;
    const int TPR = max(1, kFfnWarps / nwg);
    const int ipr = TPR * nwg;
    const int jpw = (ipr + kFfnWarps - 1) / kFfnWarps;
    uint2 *img = reinterpret_cast<uint2 *>(smem);
    float *xs = reinterpret_cast<float *>(smem + (size_t)nwin * kImgWinEntries * sizeof(uint2));
    float *sg = xs + H;
    float *part = sg + ngroups;  // [ipr][2][16]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = gridDim.x;
    const int tb = (int)((long long)ntiles * blockIdx.x / P);
    const int te = (int)((long long)ntiles * (blockIdx.x + 1) / P);

    if (!a.x_ready_early) {
        griddep_wait();
        griddep_launch_dependents();
    }
    for (int t = 0; t < a.T; ++t) {
        // activation image of x[t]; independent of the routing, so it runs
        // before waiting on the router kernel
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
        const float mx = vec_stats(xs, H, sg, red);
        const float inv = mx > 0.f ? (float)kQuantMax / mx : 0.f;
        const float delta = mx / (float)kQuantMax;
        build_image<BITS>(img, xs, H, inv, nwin);
        if (t == 0 && a.x_ready_early) {
            griddep_wait();  // routing results of the previous kernel
            griddep_launch_dependents();
        }
        resolve_experts(a, t, sx, sok);
        __syncthreads();
        if (tb >= te) continue;

        const int nmine = te - tb;
        const int nrounds = (nmine + TPR - 1) / TPR;
        const int npos = nrounds * jpw;
        ItemRegs<BITS, 2, NWI> cur, nxt;
        int n_tl = 0, n_wg = 0;
        bool n_in = false;
        auto prefetch = [&](int p) {
            const int r = p / jpw, j = warp + kFfnWarps * (p % jpw);
            n_tl = j / nwg;
            n_wg = j % nwg;
            n_in = (j < ipr) && (r * TPR + n_tl < nmine);
            Mats<2> M;
            int row0 = 0;
            bool ok = false;
            if (n_in) {
                const int tile = tb + r * TPR + n_tl;
                const int s = tile / tps;
                row0 = (tile % tps) * kTileRows;
                M.m[0] = sx[s].gate;
                M.m[1] = sx[s].up;
                ok = sok[s] != 0;
            } else {
                M.m[0] = M.m[1] = QMatDev{nullptr, nullptr, nullptr};
            }
            load_item<BITS, 2, NWI>(nxt, M, ok, row0, n_wg * NWI, Kwords, ngroups, lane);
        };
        prefetch(0);
        for (int p = 0; p < npos; ++p) {
            cur = nxt;
            const int c_tl = n_tl, c_wg = n_wg;
            const bool c_in = n_in;
            if (p + 1 < npos) prefetch(p + 1);
            if (c_in) {
                float v0[2], v8[2];
                compute_item<BITS, 2, NWI>(cur, img, sg, c_wg * NWI, nwin, ngroups, delta, lane, v0, v8);
                if ((lane & 3) == 0) {
                    float *pp = part + (size_t)(c_tl * nwg + c_wg) * 32;
                    const int g = lane >> 2;
                    pp[g] = v0[0];
                    pp[g + 8] = v8[0];
                    pp[16 + g] = v0[1];
                    pp[16 + g + 8] = v8[1];
                }
            }
            if ((p + 1) % jpw == 0) {
                __syncthreads();
                const int r = p / jpw;
                for (int e = threadIdx.x; e < TPR * kTileRows; e += blockDim.x) {
                    const int tl = e / kTileRows, row = e % kTileRows;
                    const int tile = tb + r * TPR + tl;
                    if (tile < te) {
                        float gs = 0.f, us = 0.f;
                        for (int wg = 0; wg < nwg; ++wg) {
                            gs += part[(size_t)(tl * nwg + wg) * 32 + row];
                            us += part[(size_t)(tl * nwg + wg) * 32 + 16 + row];
                        }
                        const int s = tile / tps, rt = tile % tps;
                        a.ws.h(t)[(size_t)s * I + rt * kTileRows + row] = gs / (1.f + expf(-gs)) * us;
                    }
                }
                __syncthreads();
            }
        }
    }
}

// ------------------------------------------------------------------- down

// Down mat-vecs: tiles of 16 output rows of one selected expert; per tile the
// partial output goes to the workspace and the last of the S contributions to
// a row band (atomic arrival count) sums them in fixed order with the
// routing weights, the gated shared expert and the residual.
template <int BITS>
__global__ void __launch_bounds__(kFfnThreads, 1) k_down(FfnArgs a) {
    constexpr int NWI = (BITS == 4) ? 2 : 4;
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ float red[kFfnWarps + 1];
    __shared__ float sdelta[kMaxImgSlots];
    __shared__ QExpertDev sx[kMaxTopK + 1];
    __shared__ int sok[kMaxTopK + 1];
    __shared__ int sdone[kFfnWarps];
    const int H = a.H, I = a.I;
    const int nwin = (I + kWinK - 1) / kWinK;
    const int nwg = (nwin + NWI - 1) / NWI;
    const int ngroups = I / kGroup;
    const int Kwords = I * BITS / 32;
    const int tps = H / kTileRows;
    const int ntiles = a.S * tps;
    const int TPR = max(1, kFfnWarps / nwg);
    const int ipr = TPR * nwg;
    const int jpw = (ipr + kFfnWarps - 1) / kFfnWarps;
    const size_t img_slot = (size_t)nwin * kImgWinEntries;
    uint2 *img = reinterpret_cast<uint2 *>(smem);  // [kMaxImgSlots][nwin][256]
    float *hs = reinterpret_cast<float *>(smem + kMaxImgSlots * img_slot * sizeof(uint2));
    float *sg = hs + I;                 // [kMaxImgSlots][ngroups]
    float *part = sg + kMaxImgSlots * ngroups;  // [ipr][16]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = gridDim.x;
    const int tb = (int)((long long)ntiles * blockIdx.x / P);
    const int te = (int)((long long)ntiles * (blockIdx.x + 1) / P);

    griddep_wait();  // h from the gate/up kernel
    griddep_launch_dependents();
    for (int t = 0; t < a.T; ++t) {
        if (tb >= te) break;
        resolve_experts(a, t, sx, sok);
        const int s_first = tb / tps, s_last = (te - 1) / tps;
        for (int sb = s_first; sb <= s_last; sb += kMaxImgSlots) {
            const int se = min(s_last, sb + kMaxImgSlots - 1);
            for (int s = sb; s <= se; ++s) {
                __syncthreads();
                const float *hsrc = a.ws.h(t) + (size_t)s * I;
                for (int j = threadIdx.x; j < I; j += blockDim.x) hs[j] = hsrc[j];
                __syncthreads();
                const float mx = vec_stats(hs, I, sg + (s - sb) * ngroups, red);
                if (threadIdx.x == 0) sdelta[s - sb] = mx / (float)kQuantMax;
                build_image<BITS>(img + (s - sb) * img_slot, hs, I, mx > 0.f ? (float)kQuantMax / mx : 0.f, nwin);
            }
            __syncthreads();
            const int pb = max(tb, sb * tps), pe = min(te, (se + 1) * tps);
            const int nmine = pe - pb;
            const int nrounds = (nmine + TPR - 1) / TPR;
            const int npos = nrounds * jpw;
            ItemRegs<BITS, 1, NWI> cur, nxt;
            int n_tl = 0, n_wg = 0, n_sl = 0;
            bool n_in = false;
            auto prefetch = [&](int p) {
                const int r = p / jpw, j = warp + kFfnWarps * (p % jpw);
                n_tl = j / nwg;
                n_wg = j % nwg;
                n_in = (j < ipr) && (r * TPR + n_tl < nmine);
                Mats<1> M;
                int row0 = 0;
                bool ok = false;
                if (n_in) {
                    const int tile = pb + r * TPR + n_tl;
                    const int s = tile / tps;
                    n_sl = s - sb;
                    row0 = (tile % tps) * kTileRows;
                    M.m[0] = sx[s].down;
                    ok = sok[s] != 0;
                } else {
                    M.m[0] = QMatDev{nullptr, nullptr, nullptr};
                }
                load_item<BITS, 1, NWI>(nxt, M, ok, row0, n_wg * NWI, Kwords, ngroups, lane);
            };
            if (npos > 0) prefetch(0);
            for (int p = 0; p < npos; ++p) {
                cur = nxt;
                const int c_tl = n_tl, c_wg = n_wg, c_sl = n_sl;
                const bool c_in = n_in;
                if (p + 1 < npos) prefetch(p + 1);
                if (c_in) {
                    float v0[1], v8[1];
                    compute_item<BITS, 1, NWI>(cur, img + c_sl * img_slot, sg + c_sl * ngroups,
                                               c_wg * NWI, nwin, ngroups, sdelta[c_sl], lane, v0, v8);
                    if ((lane & 3) == 0) {
                        float *pp = part + (size_t)(c_tl * nwg + c_wg) * 16;
                        pp[lane >> 2] = v0[0];
                        pp[(lane >> 2) + 8] = v8[0];
                    }
                }
                if ((p + 1) % jpw == 0) {
                    __syncthreads();
                    const int r = p / jpw;
                    for (int e = threadIdx.x; e < TPR * kTileRows; e += blockDim.x) {
                        const int tl = e / kTileRows, row = e % kTileRows;
                        const int tile = pb + r * TPR + tl;
                        if (tile < pe) {
                            float y = 0.f;
                            for (int wg = 0; wg < nwg; ++wg) y += part[(size_t)(tl * nwg + wg) * 16 + row];
                            const int s = tile / tps, rt = tile % tps;
                            a.ws.ypart(t)[(size_t)s * H + rt * kTileRows + row] = y;
                            __threadfence();
                        }
                    }
                    __syncthreads();
                    if (threadIdx.x < TPR) {
                        const int tile = pb + r * TPR + threadIdx.x;
                        int done = 0;
                        if (tile < pe) {
                            unsigned *cnt = a.ws.band_cnt(t) + (tile % tps);
                            const unsigned old = atomicAdd(cnt, 1u);
                            done = (old == (unsigned)a.S - 1u);
                            if (done) *cnt = 0u;  // every contribution has arrived
                        }
                        sdone[threadIdx.x] = done;
                    }
                    __syncthreads();
                    for (int e = threadIdx.x; e < TPR * kTileRows; e += blockDim.x) {
                        const int tl = e / kTileRows, row = e % kTileRows;
                        if (!sdone[tl]) continue;
                        __threadfence();
                        const int tile = pb + r * TPR + tl;
                        const int col = (tile % tps) * kTileRows + row;
                        const float *yp = a.ws.ypart(t);
                        float yr = 0.f;
                        for (int i = 0; i < a.k; ++i)
                            yr += a.w_base[(size_t)t * a.w_stride + i] * __ldcg(yp + (size_t)i * H + col);
                        const float ysh = (a.S > a.k) ? __ldcg(yp + (size_t)a.k * H + col) : 0.f;
                        if (a.mode == kCombineFull) {
                            const float gm = a.gamma_base ? a.gamma_base[(size_t)t * a.gamma_stride] : 1.f;
                            const float r0 = bf16_bits_to_float(a.residual[(size_t)t * H + col]);
                            const float o = r0 + yr + gm * ysh;
                            a.out[(size_t)t * H + col] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
                        } else {
                            a.ysplit[((size_t)t * 2) * H + col] = yr;
                            a.ysplit[((size_t)t * 2 + 1) * H + col] = ysh;
                        }
                    }
                    __syncthreads();
                }
            }
        }
    }
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
