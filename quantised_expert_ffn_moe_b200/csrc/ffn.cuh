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
// Data movement.  One CTA per SM, 16 warps working independently.  A warp's
// work item is one window of several 16-row blocks (4 KB of codes, see
// gu_sub / dn_sub); it loads the item's codes with 16-byte
// non-L1-allocating loads straight in the A-fragment layout (a quad of lanes
// reads 64 contiguous bytes of a row) one item ahead of the math.  (Measured on B200: 16-byte loads from 16+
// warps per SM stream ~7 TB/s, while 1-D TMA bulk copies of the 512-byte row
// pieces a row-major layout offers reach ~2 TB/s.)  A tile's item partials
// meet in a small shared-memory ring of tile slots; the warp that arrives
// last sums them in fixed order and writes the tile's result, so no
// CTA-wide barrier sits in the streaming loop and results are deterministic.
// The down kernel gives each CTA whole bands of output rows across all of
// the token's experts, so the routing-weighted combine, the gated shared
// expert and the residual are summed in shared memory by the CTA itself.
// Weight bytes are read from HBM exactly once.
#pragma once

#include "common.cuh"
#include "route.cuh"

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
    int ring_slots;            // tile slots of the shared-memory partial ring
    // Routing in the gate/up kernel: every CTA takes the token's top-k from
    // the workspace logits (E routed + the gate logit at E when has_gate);
    // CTA 0 publishes ids, weights and gamma to the workspace and to the
    // optional caller copies.  Otherwise ids come from idx_base.
    int route_in_gateup;
    // 1: the operand image of x is in the workspace (built by the router
    // kernel); the gate/up kernel copies it instead of building it
    int x_image_in_ws;
    int has_gate;
    int *topk_idx_out;         // [T][k] or null
    float *topk_w_out;
    int dn_slots;              // down kernel: expert images built per pass (<= S)
    int dn_bands_max;          // down kernel: most row bands a CTA owns
};

// ------------------------------------------------------------ work items

// Row sub-tiles per tile.  A work item is 4 KB of codes whatever the bit
// width: gate/up items hold one window of gate and up rows (4-bit: one
// 16-row sub-tile each; 2-bit: two), down items one window of 2 (4-bit) or
// 4 (2-bit) 16-row sub-tiles.  The sub-tiles of an item share the activation
// fragments; 4 KB per warp and two items in flight keep about 128 KB of loads
// in flight per SM, which is what streaming at HBM speed takes on B200.
__host__ __device__ constexpr int gu_sub(int bits) { return bits == 4 ? 1 : 2; }
__host__ __device__ constexpr int dn_sub(int bits) { return bits == 4 ? 2 : 4; }

// The same matrix, starting r rows further down.
__device__ __forceinline__ QMatDev qmat_rows(const QMatDev &m, int r, int Kwords, int ngroups) {
    return QMatDev{m.codes + (size_t)r * Kwords, m.scale + (size_t)r * ngroups, m.bias + (size_t)r * ngroups};
}

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
// every lane of quad g holds rows g (v0[m]) and g+8 (v8[m]).  Row blocks go
// in pairs whose two 8-step accumulator chains interleave (more blocks would
// cost the registers of the two item buffers).
template <int BITS, int NMAT, int NWI>
__device__ __forceinline__ void compute_item(const Item<BITS, NMAT, NWI> &R, const uint2 (&bf)[NWI][kMmaPerWin],
                                             const float *sg, const float *dg, int w0, int ngroups, int lane,
                                             float (&v0)[NMAT], float (&v8)[NMAT]) {
    constexpr int MG = NMAT < 2 ? NMAT : 2;
    static_assert(NMAT % MG == 0, "row blocks go in pairs");
    const int c = lane & 3;
#pragma unroll
    for (int m = 0; m < NMAT; ++m) v0[m] = v8[m] = 0.f;
#pragma unroll
    for (int wi = 0; wi < NWI; ++wi) {
        // accumulator columns (2c, 2c+1) = (hi, lo) sums of group 4w + c
        const int grp = 4 * (w0 + wi) + c;
        const float S = grp < ngroups ? sg[grp] : 0.f;
        const float delta = grp < ngroups ? dg[grp] : 0.f;  // the group's fixed-point step
#pragma unroll
        for (int m0 = 0; m0 < NMAT; m0 += MG) {
            int acc[MG][4];
#pragma unroll
            for (int mi = 0; mi < MG; ++mi) acc[mi][0] = acc[mi][1] = acc[mi][2] = acc[mi][3] = 0;
#pragma unroll
            for (int t = 0; t < kMmaPerWin; ++t) {
#pragma unroll
                for (int mi = 0; mi < MG; ++mi) {
                    const int m = m0 + mi;
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
                    mma_u8s8(acc[mi], a0, a1, a2, a3, bf[wi][t].x, bf[wi][t].y);
                }
            }
#pragma unroll
            for (int mi = 0; mi < MG; ++mi) {
                const int m = m0 + mi;
                const float d0 = (float)(acc[mi][0] * 256 + acc[mi][1]);
                const float d8 = (float)(acc[mi][2] * 256 + acc[mi][3]);
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
// and sok[] with their validity; ids from ids[] (routed ids in shared
// memory) or, when null, from idx_base; slot entries from table (a shared
// memory copy of the slot table) or, when null, from the slot table itself.
// Flags problems in the status word.  CTA 0 also publishes the table to the
// workspace for the down kernel.
__device__ void resolve_experts(const FfnArgs &a, int t, const int *ids, const QExpertDev *table, QExpertDev *sx,
                                int *sok) {
    for (int s = threadIdx.x; s < a.S; s += blockDim.x) {
        QExpertDev ex = a.shared;
        bool ok = true;
        if (s < a.k) {
            const int id = ids ? ids[s] : a.idx_base[(size_t)t * a.idx_stride + s];
            if (id < 0 || id >= a.n_slots) {
                flag_status(a.ws.status, MOE_DEV_BAD_EXPERT_ID);
                ok = false;
            } else {
                ex = table ? table[id] : a.slots[id];
            }
        }
        if (ok && !(qmat_ok(ex.gate) && qmat_ok(ex.up) && qmat_ok(ex.down))) {
            flag_status(a.ws.status, MOE_DEV_BAD_SLOT);
            ok = false;
        }
        sx[s] = ex;
        sok[s] = ok;
        if (blockIdx.x == 0) {
            a.ws.rx(t)[s] = ex;
            a.ws.rok(t)[s] = ok;
        }
    }
}

// CTA 0 publishes token t's routing (the top-k in tk) to the workspace and
// to the optional caller copies.
__device__ void publish_route(const FfnArgs &a, int t, const TopkSmem<kFfnThreads> &tk) {
    const int tid = threadIdx.x;
    if (tid < a.k) {
        const int e = tk.sel_idx[tid];
        const float w = tk.sel_w[tid];
        a.ws.topk_idx(t)[tid] = e;
        a.ws.topk_w(t)[tid] = w;
        if (a.topk_idx_out) a.topk_idx_out[(size_t)t * a.k + tid] = e;
        if (a.topk_w_out) a.topk_w_out[(size_t)t * a.k + tid] = w;
    }
    if (tid == 0) *a.ws.gamma(t) = a.has_gate ? gate_of_logit(__ldcg(a.ws.logits(t) + a.E)) : 1.0f;
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
    if (*(volatile int *)status & MOE_DEV_TIMEOUT) return;  // already broken: do not wait again
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

// L2 prefetch of one item: its code segments (one line each) and the lines of
// its scales and biases, spread over the warp's lanes.
template <int BITS, int NMAT>
__device__ __forceinline__ void prefetch_item(const QMatDev (&M)[NMAT], int row0, int w0, int Kwords, int ngroups,
                                              int lane) {
    constexpr int WPW = kWinK * BITS / 32;
#pragma unroll
    for (int i = lane; i < NMAT * kTileRows; i += 32) {
        const int m = i / kTileRows, row = row0 + i % kTileRows;
        const size_t o = (size_t)row * ngroups + 4 * w0;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(M[m].codes + (size_t)row * Kwords + w0 * WPW));
        asm volatile("prefetch.global.L2 [%0];" ::"l"(M[m].scale + o));
        asm volatile("prefetch.global.L2 [%0];" ::"l"(M[m].bias + o));
    }
}

// Streams the items of tiles g0, g0 + 1, ..., g0 + n - 1; tile_of(g, s, rt)
// names tile g's expert slot and row tile (RPT rows), next_tile(s, rt) steps
// to the following tile.  The tiles take ring numbers j0, j0 + 1, ...  A
// tile is nwg items of NWI windows each (all NMAT 16-row blocks of the window
// together); mat_of(s, M, ok) gives slot s's NMAT row blocks as matrices whose
// row 0 is the block's row 0 in row tile 0.  Items go in tile-major order,
// warp w taking items w, w+16, ...; two register buffers alternate so each
// item's loads are issued one item ahead of its math.  The activation
// fragments stay in registers while consecutive items of a warp use the same
// window and image.  finish(jl, s, rt) runs on the warp that completes tile
// jl (the ring slot still holds its sums).  pre() runs once on every warp
// before the first item's loads (it may hold CTA barriers); with PF each warp
// first sends its first two items to L2, so their HBM latency overlaps pre().
template <int BITS, int NMAT, int NWI, int RPT, bool FULL, bool PF, typename TileOf, typename NextTile,
          typename MatOf, typename ImgOf, typename Finish, typename Pre>
__device__ void stream_items(const TileRing &ring, int j0, int g0, int n, int K, TileOf tile_of, NextTile next_tile,
                             MatOf mat_of, ImgOf img_of, Finish finish, Pre pre, int *status) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwin = (K + kWinK - 1) / kWinK;
    const int nwg = (nwin + NWI - 1) / NWI;
    const int ngroups = K / kGroup;
    const int Kwords = K * BITS / 32;
    const int nitems = n * nwg;
    if (warp >= nitems) {
        pre();
        return;
    }
    struct Pos {
        int it, jl, r, s, rt;  // item, ring tile number, window group, slot, row tile
    };
    auto advance = [&](Pos p) {
        p.it += kFfnWarps;
        p.r += kFfnWarps;
        while (p.r >= nwg) {
            p.r -= nwg;
            ++p.jl;
            next_tile(p.s, p.rt);
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
                load_item<BITS, NMAT, NWI, FULL>(R, M, p.rt * RPT, p.r * NWI, Kwords, ngroups, lane);
            else
                zero_item(R);  // unusable expert (flagged): contributes zero
        }
    };
    auto prefetch = [&](const Pos &p) {
        if (p.it < nitems) {
            QMatDev M[NMAT];
            bool ok;
            mat_of(p.s, M, ok);
            if (ok) prefetch_item<BITS, NMAT>(M, p.rt * RPT, p.r * NWI, Kwords, ngroups, lane);
        }
    };
    uint2 bf[NWI][kMmaPerWin];
    const uint2 *bf_img = nullptr;
    int bf_w = -1;
    auto consume = [&](const It &R, const Pos &p) {
        const uint2 *img;
        const float *sg;
        const float *dg;
        img_of(p.s, img, sg, dg);
        const int w0 = p.r * NWI;
        if (img != bf_img || w0 != bf_w) {  // warp-uniform
            load_bfrag<NWI>(bf, img, w0, nwin, lane);
            bf_img = img;
            bf_w = w0;
        }
        float v0[NMAT], v8[NMAT];
        compute_item<BITS, NMAT, NWI>(R, bf, sg, dg, w0, ngroups, lane, v0, v8);
        ring_acquire(ring, p.jl, status);
        if (ring_deposit<NMAT>(ring, p.jl, p.r, v0, v8, lane, nwg)) {
            finish(p.jl, p.s, p.rt);
            ring_release(ring, p.jl, lane);
        }
    };
    Pos pa{warp, j0 + warp / nwg, warp % nwg, 0, 0};
    tile_of(g0 + warp / nwg, pa.s, pa.rt);
    if (PF) {
        prefetch(pa);
        prefetch(advance(pa));
    }
    pre();
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

// Gate/up mat-vecs and SwiGLU.  Work: tiles of RPT rows of (gate, up) of one
// selected expert; this CTA takes a contiguous slice of the token's
// S*I/RPT tiles.  With route_in_gateup, warp 0 takes the token's top-k while
// the operand image of x and (first token) the slot table land in shared
// memory by asynchronous copies.  Shared memory: image | ring part | cnt |
// epoch | slot table (routing in this kernel).
template <int BITS, bool FULL>
__global__ void __launch_bounds__(kFfnThreads, 1) k_gateup(FfnArgs a) {
    constexpr int NWI = 1;
    constexpr int SUB = gu_sub(BITS), NMAT = 2 * SUB, RPT = kTileRows * SUB;
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ float sg[kMaxDim / kGroup];
    __shared__ float dg[kMaxDim / kGroup];
    __shared__ QExpertDev sx[kMaxTopK + 1];
    __shared__ int sok[kMaxTopK + 1];
    __shared__ TopkSmem<kFfnThreads> tk;
    const int H = a.H, I = a.I;
    const int nwin = (H + kWinK - 1) / kWinK;
    const int nwg = (nwin + NWI - 1) / NWI;
    uint2 *img = reinterpret_cast<uint2 *>(smem);
    TileRing ring;
    ring.part = reinterpret_cast<float *>(img + (size_t)nwin * kImgWinEntries);
    ring.R = a.ring_slots;
    ring.lgR = __ffs(ring.R) - 1;
    ring.nwg = nwg;
    ring.vals = NMAT * kTileRows;  // per sub-tile: gate rows then up rows
    ring.cnt = reinterpret_cast<int *>(ring.part + (size_t)ring.R * nwg * ring.vals);
    ring.epoch = ring.cnt + ring.R;
    QExpertDev *stab = reinterpret_cast<QExpertDev *>(
        reinterpret_cast<uintptr_t>(ring.epoch + ring.R + 3) & ~(uintptr_t)15);
    const int tps = I / RPT;
    const int Kw = H * BITS / 32, ng = H / kGroup;
    const int ntiles = a.S * tps;
    const int P = gridDim.x;
    const int tb = (int)((long long)ntiles * blockIdx.x / P);
    const int te = (int)((long long)ntiles * (blockIdx.x + 1) / P);
    const int lane = threadIdx.x & 31;
    MOEQ_STAMP(1, 0);
    ring_init(ring);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        // the down kernel starts once every CTA here has passed its first
        // prologue, and CTA 0 clears the flags before that
        for (int t = 0; t < a.T; ++t) *a.ws.ready(t) = 0u;
        __threadfence();
    }
    if (!a.x_image_in_ws) griddep_wait();  // x and the ids come from earlier kernels
    int jseq = 0;
    for (int t = 0; t < a.T; ++t) {
        if (a.x_image_in_ws) {
            if (t == 0) griddep_wait();  // the router kernel's logits and image of x
            // the image (and the slot table) land in shared memory while the
            // top-k runs
            const uint4 *src = reinterpret_cast<const uint4 *>(a.ws.ximg(t));
            const int n16 = nwin * kImgWinEntries * (int)sizeof(uint2) / 16;
            for (int i = threadIdx.x; i < n16; i += blockDim.x) cp_async16(reinterpret_cast<uint4 *>(img) + i, src + i);
            if (a.route_in_gateup && t == 0) {
                const unsigned long long *ts = reinterpret_cast<const unsigned long long *>(a.slots);
                unsigned long long *td = reinterpret_cast<unsigned long long *>(stab);
                const int n8 = a.E * (int)(sizeof(QExpertDev) / 8);
                for (int i = threadIdx.x; i < n8; i += blockDim.x) cp_async8(td + i, ts + i);
            }
            for (int i = threadIdx.x; i < H / kGroup; i += blockDim.x) {
                sg[i] = __ldcg(a.ws.xsg(t) + i);
                dg[i] = __ldcg(a.ws.xdg(t) + i);
            }
            MOEQ_STAMP(1, 1);
        } else {
            // activation image of x[t]
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
            build_images<BITS>(img, sg, dg, 1, H, nwin, load8);
            MOEQ_STAMP(1, 1);
        }
        MOEQ_STAMP(1, 2);
        if (a.route_in_gateup) topk_block<kFfnThreads>(a.ws.logits(t), a.E, a.k, tk);
        MOEQ_STAMP(1, 10);
        if (a.x_image_in_ws) cp_async_wait_all();
        __syncthreads();
        if (a.route_in_gateup && blockIdx.x == 0) publish_route(a, t, tk);
        resolve_experts(a, t, a.route_in_gateup ? tk.sel_idx : nullptr, a.route_in_gateup ? stab : nullptr, sx, sok);
        __syncthreads();
        if (blockIdx.x == 0 && threadIdx.x == 0) {
            __threadfence();  // routing and expert table (published above) before the flag
            st_release_u32(a.ws.ready(t), 1u);
        }
        // The down kernel may start as CTAs here finish (it cannot share an
        // SM with one): it prefetches its weights into L2 meanwhile and waits
        // for this grid before it reads h.
        if (t == 0) griddep_launch_dependents();
        MOEQ_STAMP(1, 3);
        auto tile_of = [&](int g, int &s, int &rt) {
            s = g / tps;
            rt = g % tps;
        };
        auto next_tile = [&](int &s, int &rt) {
            if (++rt == tps) {
                rt = 0;
                ++s;
            }
        };
        auto mat_of = [&](int s, QMatDev (&M)[NMAT], bool &ok) {
#pragma unroll
            for (int u = 0; u < SUB; ++u) {
                M[2 * u] = qmat_rows(sx[s].gate, kTileRows * u, Kw, ng);
                M[2 * u + 1] = qmat_rows(sx[s].up, kTileRows * u, Kw, ng);
            }
            ok = sok[s] != 0;
        };
        auto img_of = [&](int, const uint2 *&im, const float *&sgp, const float *&dgp) {
            im = img;
            sgp = sg;
            dgp = dg;
        };
        auto finish = [&](int jl, int s, int rt) {
            if (lane < RPT) {
                const int u = lane / kTileRows, r = lane % kTileRows;
                const float gs = ring_sum(ring, jl, 2 * u, r);
                const float us = ring_sum(ring, jl, 2 * u + 1, r);
                a.ws.h(t)[(size_t)s * I + rt * RPT + lane] = gs / (1.f + expf(-gs)) * us;
            }
        };
        stream_items<BITS, NMAT, NWI, RPT, FULL, false>(ring, jseq, tb, te - tb, H, tile_of, next_tile, mat_of,
                                                        img_of, finish, [] {}, a.ws.status);
        MOEQ_STAMP_MAX(1, 4);
        jseq += te - tb;
        __syncthreads();  // image and expert table are rebuilt for the next token
    }
    MOEQ_STAMP(1, 5);
}

// ------------------------------------------------------------------- down

// Down mat-vecs with the combine.  Each CTA owns whole bands of RPT output
// rows (32 for 4-bit, 64 for 2-bit codes; a contiguous range of the token's
// H/RPT bands) across all S experts of the token, so a band's S partial
// outputs meet in this CTA's shared memory; the last of them to finish sums
// them in fixed order with the routing weights, the gated shared expert and
// the residual.  The experts' activation images (of h) are built dn_slots at
// a time.  Shared memory: images | group sums | group steps | ring part | cnt | epoch |
// band partials [dn_bands_max][S][RPT] | band counts | residual rows.
template <int BITS, bool FULL>
__global__ void __launch_bounds__(kFfnThreads, 1) k_down(FfnArgs a) {
    constexpr int NWI = 1;
    constexpr int NMAT = dn_sub(BITS), RPT = kTileRows * NMAT;
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ float sw[kMaxTopK];
    __shared__ float s_gamma;
    __shared__ QExpertDev sx[kMaxTopK + 1];
    __shared__ int sok[kMaxTopK + 1];
    const int H = a.H, I = a.I, S = a.S, Mx = a.dn_slots, NB = a.dn_bands_max;
    const int nwin = (I + kWinK - 1) / kWinK;
    const int nwg = (nwin + NWI - 1) / NWI;
    const int ngr = I / kGroup;
    const size_t img_slot = (size_t)nwin * kImgWinEntries;
    uint2 *img = reinterpret_cast<uint2 *>(smem);
    float *sgs = reinterpret_cast<float *>(img + (size_t)Mx * img_slot);  // [Mx][ngr] group sums
    float *dgs = sgs + (size_t)Mx * ngr;                                   // [Mx][ngr] group steps
    TileRing ring;
    ring.part = dgs + (size_t)Mx * ngr;
    ring.R = a.ring_slots;
    ring.lgR = __ffs(ring.R) - 1;
    ring.nwg = nwg;
    ring.vals = NMAT * kTileRows;
    ring.cnt = reinterpret_cast<int *>(ring.part + (size_t)ring.R * nwg * ring.vals);
    ring.epoch = ring.cnt + ring.R;
    float *yb = reinterpret_cast<float *>(ring.epoch + ring.R);  // [NB][S][RPT]
    int *bcnt = reinterpret_cast<int *>(yb + (size_t)NB * S * RPT);
    uint16_t *sres = reinterpret_cast<uint16_t *>(bcnt + NB);   // [NB][RPT]
    const int Kw = I * BITS / 32;
    const int nbands = H / RPT;
    const int P = gridDim.x;
    const int b0 = (int)((long long)nbands * blockIdx.x / P);
    const int b1 = (int)((long long)nbands * (blockIdx.x + 1) / P);
    const int nb = b1 - b0;
    const int lane = threadIdx.x & 31;
    MOEQ_STAMP(2, 0);
    ring_init(ring);
    int jseq = 0;
    for (int t = 0; t < a.T && nb > 0; ++t) {
        // the token's experts and routing, published by the gate/up kernel
        // while it still runs (bounded wait on its flag)
        if (threadIdx.x == 0) {
            const unsigned *rf = a.ws.ready(t);
            if (ld_acquire_u32(rf) == 0u) {
                const unsigned long long t0 = globaltimer_ns();
                while (ld_acquire_u32(rf) == 0u)
                    if (globaltimer_ns() - t0 > kWaitLimitNs) {
                        flag_status(a.ws.status, MOE_DEV_TIMEOUT);
                        break;
                    }
            }
        }
        __syncthreads();
        for (int s = threadIdx.x; s < S; s += blockDim.x) {
            sx[s] = a.ws.rx(t)[s];
            sok[s] = a.ws.rok(t)[s];
        }
        __syncthreads();
        // this CTA's down weights into L2 while the gate/up kernel finishes:
        // per expert, rows [b0*RPT, b1*RPT) are one contiguous block of codes
        for (int s = threadIdx.x; s < S; s += blockDim.x)
            if (sok[s]) {
                const QMatDev &m = sx[s].down;
                const size_t rowb = (size_t)Kw * 4;  // bytes per code row (a multiple of 16)
                const char *base = reinterpret_cast<const char *>(m.codes) + (size_t)b0 * RPT * rowb;
                size_t left = (size_t)nb * RPT * rowb;
                for (size_t o = 0; left > 0; o += 32768) {
                    const unsigned n = (unsigned)min(left, (size_t)32768);
                    prefetch_l2(base + o, n);
                    left -= n;
                }
            }
        for (int i = threadIdx.x; i < S * nb * RPT; i += blockDim.x) {  // one line per row of scales, biases
            const int s = i / (nb * RPT), r = b0 * RPT + i % (nb * RPT);
            if (sok[s] && (i % (nb * RPT)) % 4 == 0) {
                asm volatile("prefetch.global.L2 [%0];" ::"l"(sx[s].down.scale + (size_t)r * ngr));
                asm volatile("prefetch.global.L2 [%0];" ::"l"(sx[s].down.bias + (size_t)r * ngr));
            }
        }
        if (t == 0) griddep_wait();  // h from the gate/up kernel
        MOEQ_STAMP(2, 1);
        for (int i = threadIdx.x; i < a.k; i += blockDim.x) sw[i] = a.w_base[(size_t)t * a.w_stride + i];
        if (threadIdx.x == 0) s_gamma = a.gamma_base ? a.gamma_base[(size_t)t * a.gamma_stride] : 1.f;
        for (int i = threadIdx.x; i < nb; i += blockDim.x) bcnt[i] = 0;
        if (a.mode == kCombineFull)
            for (int i = threadIdx.x; i < nb * RPT; i += blockDim.x) sres[i] = a.residual[(size_t)t * H + b0 * RPT + i];
        __syncthreads();
        MOEQ_STAMP(2, 5);
        for (int s0 = 0; s0 < S; s0 += Mx) {
            const int s1 = min(S, s0 + Mx), ns = s1 - s0;
            auto tile_of = [&](int g, int &s, int &rt) {
                s = s0 + g % ns;
                rt = b0 + g / ns;
            };
            auto next_tile = [&](int &s, int &rt) {
                if (++s == s1) {
                    s = s0;
                    ++rt;
                }
            };
            auto mat_of = [&](int s, QMatDev (&M)[NMAT], bool &ok) {
#pragma unroll
                for (int u = 0; u < NMAT; ++u) M[u] = qmat_rows(sx[s].down, kTileRows * u, Kw, ngr);
                ok = sok[s] != 0;
            };
            auto img_of = [&](int s, const uint2 *&im, const float *&sgp, const float *&dgp) {
                im = img + (s - s0) * img_slot;
                sgp = sgs + (s - s0) * ngr;
                dgp = dgs + (s - s0) * ngr;
            };
            auto finish = [&](int jl, int s, int rt) {
                const int bl = rt - b0;
                float *yp = yb + ((size_t)bl * S + s) * RPT;
#pragma unroll
                for (int r = lane; r < RPT; r += 32) yp[r] = ring_sum(ring, jl, r / kTileRows, r % kTileRows);
                __threadfence_block();
                __syncwarp();
                int last = 0;
                if (lane == 0) last = atomicAdd(bcnt + bl, 1) == S - 1;
                if (!__shfl_sync(0xffffffffu, last, 0)) return;
                __threadfence_block();
                // all S partials of this band are in: combine in slot order
                const float *yl = yb + (size_t)bl * S * RPT;
#pragma unroll
                for (int r = lane; r < RPT; r += 32) {
                    float yr = 0.f;
                    for (int i = 0; i < a.k; ++i) yr += sw[i] * yl[(size_t)i * RPT + r];
                    const float ysh = S > a.k ? yl[(size_t)a.k * RPT + r] : 0.f;
                    const int col = rt * RPT + r;
                    if (a.mode == kCombineFull) {
                        const float r0 = bf16_bits_to_float(sres[bl * RPT + r]);
                        a.out[(size_t)t * H + col] = __bfloat16_as_ushort(__float2bfloat16_rn(r0 + yr + s_gamma * ysh));
                    } else {
                        a.ysplit[((size_t)t * 2) * H + col] = yr;
                        a.ysplit[((size_t)t * 2 + 1) * H + col] = ysh;
                    }
                }
            };
            auto pre = [&] {
                __syncthreads();  // the previous pass's items are done with the images
                const float4 *hv = reinterpret_cast<const float4 *>(a.ws.h(t) + (size_t)s0 * I);
                build_images<BITS>(img, sgs, dgs, ns, I, nwin, [&](int c, float(&f)[8]) {
                    const float4 u = __ldcg(hv + 2 * c), v = __ldcg(hv + 2 * c + 1);
                    f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
                    f[4] = v.x; f[5] = v.y; f[6] = v.z; f[7] = v.w;
                });
                MOEQ_STAMP(2, 2);
            };
            stream_items<BITS, NMAT, NWI, RPT, FULL, false>(ring, jseq, 0, nb * ns, I, tile_of, next_tile, mat_of,
                                                            img_of, finish, pre, a.ws.status);
            MOEQ_STAMP_MAX(2, 3);
            jseq += nb * ns;
        }
        __syncthreads();  // experts, weights and band counts are rebuilt for the next token
    }
    MOEQ_STAMP(2, 4);
    griddep_launch_dependents();
}

// RMS normalisation (unit weight) of one token per CTA; fp64 sum of squares.
__global__ void __launch_bounds__(256) k_rmsnorm(const uint16_t *x, int H, float eps, uint16_t *out) {
    __shared__ double red[8];
    const int t = blockIdx.x;
    griddep_wait();
    const uint16_t *xt = x + (size_t)t * H;
    double ss = 0.0;
    for (int j = threadIdx.x; j < H; j += blockDim.x) {
        const double v = bf16_bits_to_float(xt[j]);
        ss += v * v;
    }
    ss = warp_sum_f64(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    double z = 0.0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) z += red[i];
    const double inv = 1.0 / sqrt(z / (double)H + (double)eps);
    griddep_launch_dependents();
    for (int j = threadIdx.x; j < H; j += blockDim.x)
        out[(size_t)t * H + j] = __bfloat16_as_ushort(__double2bfloat16((double)bf16_bits_to_float(xt[j]) * inv));
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
