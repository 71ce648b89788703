// prefill.cuh -- the MoE layer for many tokens at once: the (token, expert)
// pairs are sorted by expert, and each expert's tokens go through its gate/up
// and down matrices as dense GEMMs on the fifth-generation tensor cores, with
// the 4-bit weights dequantised into tensor memory on the way.
//
// Pages: "Flash-MoE - Exécuter un modèle de 397 milliards de paramètres sur un
// ordinateur portable": "Noyau de déquantification optimisé FMA" (weight =
// nibble*scale + bias), "Shaders de calcul Metal" (dequantising products,
// SwiGLU, MoE combine + residual + gate); "Qwen3.5-397B MoE fonctionne avec
// 14 Go de RAM via un chargement d'expert paginé sur M1 Ultra" (512 experts,
// top-10).  The pages run one token at a time; sorting the pairs so that an
// expert's weights are read once for all of its tokens is this library's.
//
// Flow (one launch each): count pairs per expert, scan (row offsets padded to
// 16) and tile list, scatter (rows of the sorted activation matrix Xs in
// fp16), gate/up GEMM + SwiGLU (Hs, fp16), down GEMM (Ys, fp32 rows), combine.
//
// GEMM orientation.  D[weight rows x tokens] = W[rows x K] * X[tokens x K]^T:
// the dequantised weights are the MMA's A operand (M = 128 rows, read from
// tensor memory), an expert's tokens are B (N = up to 64, a multiple of 16,
// in shared memory), so experts with few tokens waste little.  fp16 operands
// (weights rounded once from the exact nibble*scale + bias; |rel err| <=
// 2^-11), fp32 accumulation in TMEM.
//
// K order.  A 4-bit word holds codes 0..7; the dequantiser makes fp16 pairs
// (0,4), (1,5), (2,6), (3,7) with one mask each, so the four 32-bit columns
// it writes hold the codes in the order 0,4,1,5,2,6,3,7.  Xs and Hs are
// stored with the same order inside every 8 values, so A and B agree without
// any shuffling.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "tc.cuh"

namespace moeq {

constexpr int kPfTok = 64;          // tokens per GEMM tile (MMA N, padded to 16)
constexpr int kPfRows = 128;        // weight rows per GEMM unit (MMA M)
constexpr int kPfK = 64;            // K per chunk (one quantisation group)
constexpr int kPfStages = 3;        // dequantised weight-tile stages
constexpr int kPfRaw = 8;           // raw-code ring depth
constexpr int kPfAhead = kPfRaw - 1;  // chunks of code copies in flight ahead of the one dequantised
constexpr int kPfBSlots = 4;        // token-tile slots (TMA; loaded as soon as a slot is free)
constexpr int kPfPad = 16;          // expert row blocks are padded to 16 rows

// Position of value j (0..7) of a group of 8 in the stored K order.
__host__ __device__ constexpr int pf_kpos(int j) { return (j & 3) * 2 + (j >> 2); }

struct PfWs {
    unsigned *cnt;    // [E+1] pairs per expert (index E: the shared expert)
    unsigned *fill;   // [E+1] scatter cursors
    int *off;         // [E+2] first row of each expert in the sorted matrices
    int *ntiles;      // [1]
    int *tile_e, *tile_r0, *tile_n;  // [tcap] expert, first row, token count
    int *pos;         // [T][S] sorted row of (token, slot)
    __half *xs;       // [pcap][H]
    __half *hs;       // [pcap][I]: h rounded to fp16
    __half *hl;       // [pcap][I]: h - hs rounded to fp16 (h = hs + hl to ~2^-22)
    float *ys;        // [pcap][H]
    int pcap, tcap;
    // TMA maps of xs, hs, hl: boxes of 64 values x 16 rows, 128-byte swizzle
    CUtensorMap tm_xs, tm_hs, tm_hl;
};

struct PfArgs {
    int T, H, I, E, k, S, has_shared;
    const uint16_t *x;         // bf16 [T][H]
    const uint16_t *residual;  // bf16 [T][H]
    uint16_t *out;             // bf16 [T][H]
    const QExpertDev *slots;
    QExpertDev shared;
    WsPtrs ws;                 // per-token routing results (ids, weights, gamma)
    PfWs p;
};

// -------------------------------------------------------------- sorting

// One thread per (token, slot) pair: count it under its expert.
__global__ void __launch_bounds__(256) k_pf_count(PfArgs a) {
    griddep_wait();
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= a.T * a.S) return;
    const int t = i / a.S, s = i % a.S;
    const int e = s < a.k ? a.ws.topk_idx(t)[s] : a.E;
    if (e >= 0 && e <= a.E) atomicAdd(a.p.cnt + e, 1u);
}

// One CTA: row offsets (each expert's block padded to 16 rows), the tile
// list (blocks of up to kPfTok rows per expert), scatter cursors reset.
__global__ void __launch_bounds__(1024) k_pf_scan(PfArgs a) {
    griddep_wait();
    __shared__ int wsum[2][32];
    const int n = a.E + 1, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int base_rows = 0, base_tiles = 0;
    for (int e0 = 0; e0 < n; e0 += 1024) {
        const int e = e0 + tid;
        const int c = e < n ? (int)a.p.cnt[e] : 0;
        const int rows = (c + kPfPad - 1) / kPfPad * kPfPad;
        const int tiles = (c + kPfTok - 1) / kPfTok;
        int ir = rows, it = tiles;  // inclusive scans in the warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int vr = __shfl_up_sync(0xffffffffu, ir, o), vt = __shfl_up_sync(0xffffffffu, it, o);
            if (lane >= o) {
                ir += vr;
                it += vt;
            }
        }
        if (lane == 31) {
            wsum[0][warp] = ir;
            wsum[1][warp] = it;
        }
        __syncthreads();
        int pr = 0, pt = 0, tr = 0, tt = 0;
        for (int w = 0; w < 32; ++w) {
            if (w < warp) {
                pr += wsum[0][w];
                pt += wsum[1][w];
            }
            tr += wsum[0][w];
            tt += wsum[1][w];
        }
        if (e < n) {
            const int r0 = base_rows + pr + ir - rows, t0 = base_tiles + pt + it - tiles;
            a.p.off[e] = r0;
            a.p.fill[e] = 0u;
            for (int j = 0; j < tiles; ++j) {
                a.p.tile_e[t0 + j] = e;
                a.p.tile_r0[t0 + j] = r0 + j * kPfTok;
                a.p.tile_n[t0 + j] = min(kPfTok, c - j * kPfTok);
            }
        }
        base_rows += tr;
        base_tiles += tt;
        __syncthreads();
    }
    if (tid == 0) {
        a.p.off[n] = base_rows;
        *a.p.ntiles = base_tiles;
    }
}

// One warp per (token, slot) pair: a row of Xs (x in fp16, stored K order)
// and the pair's row in pos.
__global__ void __launch_bounds__(256) k_pf_scatter(PfArgs a) {
    griddep_wait();
    const int lane = threadIdx.x & 31;
    const int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (i >= a.T * a.S) return;
    const int t = i / a.S, s = i % a.S;
    const int e = s < a.k ? a.ws.topk_idx(t)[s] : a.E;
    int row = -1;
    if (lane == 0 && e >= 0 && e <= a.E) row = a.p.off[e] + (int)atomicAdd(a.p.fill + e, 1u);
    row = __shfl_sync(0xffffffffu, row, 0);
    if (lane == 0) a.p.pos[i] = row;
    if (row < 0) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(a.x + (size_t)t * a.H);
    uint4 *dst = reinterpret_cast<uint4 *>(a.p.xs + (size_t)row * a.H);
    for (int c = lane; c < a.H / 8; c += 32) {
        const uint4 v = src[c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        __half h[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) h[pf_kpos(j)] = __float2half_rn(bf16_bits_to_float((w[j >> 1] >> (16 * (j & 1))) & 0xffffu));
        dst[c] = *reinterpret_cast<const uint4 *>(h);
    }
}

// -------------------------------------------------------------- GEMMs

// Four fp16 pairs (codes (0,4), (1,5), (2,6), (3,7) of a 4-bit word) as
// q*s + b, rounded once (exact code via the 1024 + q bit pattern).
__device__ __forceinline__ uint4 pf_dequant_word(uint32_t x, __half2 s2, __half2 b2) {
    const __half2 k1024 = __half2half2(__ushort_as_half((unsigned short)0x6400));
    uint32_t p[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t v = ((x >> (4 * j)) & 0x000F000Fu) | 0x64006400u;
        const __half2 q = __hsub2(*reinterpret_cast<const __half2 *>(&v), k1024);
        const __half2 w = __hfma2(q, s2, b2);
        p[j] = *reinterpret_cast<const uint32_t *>(&w);
    }
    return make_uint4(p[0], p[1], p[2], p[3]);
}

__device__ __forceinline__ __half2 pf_bf16_to_half2(uint16_t v) {
    return __half2half2(__float2half_rn(bf16_bits_to_float(v)));
}

// Shared memory of a GEMM kernel (1024-byte aligned pieces):
//   b[kPfBSlots][NB][kPfTok][128 B]      token tiles (TMA; NB = 2: the high
//                                        and low fp16 parts of the operand)
//   raw[kPfRaw][NMAT * 128][32 B]        raw code chunks (cp.async ring)
//   sb[8][producers]                     packed scale | bias of 8 chunks
// The dequantised weight tiles live in tensor memory (see pf_gemm).
template <int NMAT, int NB>
struct PfSmem {
    static constexpr size_t a_bytes = 0;
    static constexpr size_t b_bytes = (size_t)kPfBSlots * NB * kPfTok * 128;
    static constexpr size_t raw_bytes = (size_t)kPfRaw * NMAT * kPfRows * 32;
    static constexpr size_t sb_bytes = (size_t)NMAT * kPfRows * 2 * 8 * 4;
    static constexpr size_t total = a_bytes + b_bytes + raw_bytes + sb_bytes + 1024;  // + alignment slack
};

// Pipeline wait of the GEMM engine: bounded like every wait (1 s, then
// MOE_DEV_TIMEOUT), and once one of this thread's waits has timed out
// (`broken`, a register) its later ones give up at once, so a broken
// pipeline ends in about a second instead of a second per chunk.  Nothing
// is read from global memory on the way.
__device__ __forceinline__ void pf_wait(uint64_t *bar, unsigned parity, int *status, bool &broken) {
    if (mbar_try_wait(bar, parity) || broken) return;
    if (!mbar_wait(bar, parity, status)) broken = true;
}

// 2-D TMA load of one box (64 fp16 values x 16 rows) at (x, y) into shared
// memory, completing its bytes on bar.  x is a multiple of 64 (128 bytes).
__device__ __forceinline__ void pf_tma_box(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Build with -DMOEQ_PF_PROFILE to accumulate clock64 cycles per pipeline
// phase of the GEMM engine (summed over threads and CTAs) in g_pfprof;
// otherwise this compiles to nothing.
#ifdef MOEQ_PF_PROFILE
__device__ unsigned long long g_pfprof[2][16];
struct PfProf {
    long long last = 0;
    unsigned long long acc[8] = {};
    __device__ __forceinline__ void start() { last = clock64(); }
    __device__ __forceinline__ void tick(int i) {
        const long long n = clock64();
        acc[i] += (unsigned long long)(n - last);
        last = n;
    }
    __device__ __forceinline__ void flush(int k, int base) {
        for (int i = 0; i < 8; ++i) atomicAdd(&g_pfprof[k][base + i], acc[i]);
    }
};
#define PF_PROF(x) x
#else
#define PF_PROF(x)
#endif

// Index and phase of a ring position, advanced one step at a time.
struct PfPos {
    int i = 0, ph = 0;
    __device__ __forceinline__ void next(int n) {
        if (++i == n) {
            i = 0;
            ph ^= 1;
        }
    }
};

// One GEMM unit: the weight matrices (gate and up, or down), the first
// weight row of the 128-row block, the first sorted row and the token count
// of the tile.
template <int NMAT>
struct PfUnit {
    QMatDev m[NMAT];
    int wrow0, r0, nb;
};

// Producer threads of a GEMM: pf_split per weight row of each matrix, each
// 8 / pf_split code words (64 / pf_split codes) of the row's chunk (measured
// best: one per row for gate/up, two for down).
template <int NMAT>
__host__ __device__ constexpr int pf_split() { return NMAT == 2 ? 1 : 2; }
template <int NMAT>
__host__ __device__ constexpr int pf_producers() { return NMAT * kPfRows * pf_split<NMAT>(); }
template <int NMAT>
__host__ __device__ constexpr int pf_threads() { return pf_producers<NMAT>() + 96; }  // + 2 MMA warps, loader

// Accumulators per set: gate and up (NMAT = 2), or the products with the
// high and low fp16 parts of h (NB = 2).  Each has its own MMA-issuing
// thread: one thread's MMAs issue about 55 cycles apart (measured on B200,
// M = 128, K = 16, any N up to 64), and the tensor cores accept the MMAs of
// several threads at once.
constexpr int kPfIssuers = 2;

// The GEMM engine shared by gate/up (NMAT = 2: gate and up rows of the same
// index) and down (NMAT = 1).  Units (tile, row block) are dealt to the
// persistent CTAs in a strided order; a CTA's K chunks form one continuous
// stream.
//   Producer threads each own part of a weight row (pf_split threads per
//   row): they copy its codes of a chunk kPfAhead chunks ahead through their
//   own cp.async ring, dequantise them
//   into one of kPfStages weight-tile stages in tensor memory, and each warp
//   arrives once on the stage's `full` barrier; before reusing a stage a
//   warp waits (one lane) on its `empty` barrier (the MMAs of the chunk
//   kPfStages earlier).
//   Two MMA warps (one thread each, one accumulator each) wait for a chunk's
//   `full` and `bfull`, issue their MMAs and commit them to the stage's
//   `empty` and the token slot's `bempty` barriers (two arrivals each).  The loader warp (one thread) loads each chunk's token
//   tiles by TMA into one of kPfBSlots slots (`bfull`, transaction bytes) as
//   soon as the slot's `bempty` says the MMAs that read it are done.
// So dequantising overlaps the MMAs of the chunks before it and neither waits
// on the HBM latency of the codes.  A unit's accumulators (TMEM, two sets)
// are read out by `epilogue` in the producers once its last MMAs are done,
// while later units stream.  Ring positions advance incrementally (no
// divisions per chunk); producers keep only their own matrix of a unit.
template <int NMAT, int NB, typename UnitOf, typename Epilogue>
__device__ void pf_gemm(int nunits, int K, const CUtensorMap *bmap0, const CUtensorMap *bmap1, UnitOf unit_of,
                        Epilogue epilogue, int *status) {
    constexpr int NP = pf_producers<NMAT>();
    extern __shared__ __align__(1024) unsigned char pf_smem_raw[];
    __shared__ uint64_t full[kPfStages], empty[kPfStages], bfull[kPfBSlots], bempty[kPfBSlots];
    __shared__ uint32_t tbase;
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(pf_smem_raw) + 1023) &
                                                          ~(uintptr_t)1023);
    unsigned char *sa = sm;
    unsigned char *sb = sa + PfSmem<NMAT, NB>::a_bytes;
    unsigned char *sraw = sb + PfSmem<NMAT, NB>::b_bytes;
    uint32_t *ssb = reinterpret_cast<uint32_t *>(sraw + PfSmem<NMAT, NB>::raw_bytes);  // [8][NP]
    // tensor memory: two accumulator sets of NMAT x kPfTok fp32 columns, then
    // kPfStages weight-tile stages of NMAT x 32 columns (128 rows x 64 fp16)
    static_assert(NMAT * NB == kPfIssuers, "one issuing thread per accumulator");
    constexpr int kAccCols = kPfIssuers * kPfTok;
    constexpr int kABase = 2 * kAccCols;
    constexpr int kStageCols = NMAT * (kPfK / 2);
    constexpr int kTmemCols = 512;
    static_assert(kABase + kPfStages * kStageCols <= kTmemCols, "tensor memory budget");
    const int tid = threadIdx.x, warp = tid >> 5;
    if (warp == 0) {
        tmem_alloc(&tbase, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < kPfStages; ++i) {
            mbar_init(&full[i], NP / 32);  // one arrival per producer warp
            mbar_init(&empty[i], kPfIssuers);
        }
        for (int i = 0; i < kPfBSlots; ++i) {
            mbar_init(&bfull[i], 1);
            mbar_init(&bempty[i], kPfIssuers);
        }
        mbar_init_fence();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = tbase;
    const int nk = K / kPfK;
    // units in a strided order: the CTAs working on one tile's row blocks at
    // the same time share its token rows through L2 (a contiguous range per
    // CTA re-reads them from HBM)
    const int my_units = nunits > (int)blockIdx.x ? (nunits - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int nchunks = my_units * nk;
    const int u_first = (int)blockIdx.x, u_step = (int)gridDim.x;
    auto nb_pad = [](int nb) { return (nb + kPfPad - 1) / kPfPad * kPfPad; };
    bool broken = false;

    if (warp >= NP / 32 && warp < NP / 32 + kPfIssuers) {
        // ---- MMAs: one thread per accumulator: issuer q takes matrix q
        // (gate / up) or token part q (high / low part of h)
        const int q = warp - NP / 32;
        const int qm = NMAT == 2 ? q : 0, qb = NB == 2 ? q : 0;
        if ((tid & 31) == 0) {
            PF_PROF(PfProf pr; pr.start();)
            int kc = 0, ul = 0;
            uint32_t idesc = 0;
            // descriptor of token slot 0, part 0; slots and parts are whole
            // 1024-byte multiples apart, added in 16-byte units
            const uint64_t db0 = desc_k_sw128(sb);
            constexpr uint32_t kBPart = kPfTok * 128 / 16, kBSlot = NB * kBPart;
            PfPos apos, bcur;  // stage and token slot of chunk g
            for (int g = 0; g < nchunks; ++g) {
                if (kc == 0) {
                    PfUnit<NMAT> U;
                    unit_of(u_first + ul * u_step, U);
                    idesc = idesc_f16_f32(kPfRows, nb_pad(U.nb));
                }
                PF_PROF(pr.tick(0);)
                pf_wait(&bfull[bcur.i], (unsigned)bcur.ph, status, broken);
                PF_PROF(pr.tick(2);)
                pf_wait(&full[apos.i], (unsigned)apos.ph, status, broken);
                PF_PROF(pr.tick(3);)
                tc_fence_after();
                const uint32_t d = tm + (uint32_t)((ul & 1) * kAccCols + q * kPfTok);
                const uint32_t ta = tm + (uint32_t)(kABase + apos.i * kStageCols + qm * (kPfK / 2));
                const uint64_t db = db0 + (uint64_t)(bcur.i * kBSlot + qb * kBPart);
                const bool acc0 = kc > 0;
                tc_mma_f16_ta(d, ta, db, idesc, acc0);
                tc_mma_f16_ta(d, ta + 8, db + 2, idesc, true);
                tc_mma_f16_ta(d, ta + 16, db + 4, idesc, true);
                tc_mma_f16_ta(d, ta + 24, db + 6, idesc, true);
                tc_commit(&empty[apos.i]);
                tc_commit(&bempty[bcur.i]);
                PF_PROF(pr.tick(4);)
                apos.next(kPfStages);
                bcur.next(kPfBSlots);
                if (++kc == nk) {
                    kc = 0;
                    ++ul;
                }
            }
            // all MMAs done before the TMEM is released, whatever happened
            // to the other waits: the last phase completes with both
            // issuers' last commits, which cover every earlier MMA
            if (nchunks > 0) {
                PfPos last;
                for (int g = 0; g < nchunks - 1; ++g) last.next(kPfStages);
                mbar_wait(&empty[last.i], (unsigned)last.ph, status);
            }
            PF_PROF(if (q == 0) {
                pr.flush(NMAT - 1, 8);
                atomicAdd(&g_pfprof[NMAT - 1][15], (unsigned long long)nchunks);
            })
        }
        __syncwarp();
    } else if (warp == NP / 32 + kPfIssuers) {
        // ---- token tiles by TMA: one thread, each chunk's tiles as soon as
        // its slot is free
        if ((tid & 31) == 0) {
            int bkc = 0, bul = 0, b_r0 = 0, b_nbp = 0;
            PfPos bpos, bfree;  // slot of chunk g, slot (and phase) of chunk g - kPfBSlots
            for (int g = 0; g < nchunks; ++g) {
                if (bkc == 0) {
                    PfUnit<NMAT> U;
                    unit_of(u_first + bul * u_step, U);
                    b_r0 = U.r0;
                    b_nbp = nb_pad(U.nb);
                }
                if (g >= kPfBSlots) {
                    pf_wait(&bempty[bfree.i], (unsigned)bfree.ph, status, broken);
                    bfree.next(kPfBSlots);
                }
                uint64_t *bar = &bfull[bpos.i];
                mbar_arrive_expect_tx(bar, (unsigned)(b_nbp * 128 * NB));
#pragma unroll
                for (int bi = 0; bi < NB; ++bi) {
                    unsigned char *bt = sb + ((size_t)bpos.i * NB + bi) * kPfTok * 128;
                    for (int r = 0; r < b_nbp; r += 16)
                        pf_tma_box(bt + r * 128, bi == 0 ? bmap0 : bmap1, bkc * kPfK, b_r0 + r, bar);
                }
                bpos.next(kPfBSlots);
                if (++bkc == nk) {
                    bkc = 0;
                    ++bul;
                }
            }
            // the last tiles' MMAs are done before the CTA exits (the MMA
            // warp waits for them)
        }
        __syncwarp();
    } else {
        // ---- producers: warp w owns weight rows 32 (w % 4) .. + 31 (its
        // TMEM lanes) of matrix (w / 4) / split, part (w / 4) % split of
        // each chunk; lane = row within the group
        constexpr int SPLIT = pf_split<NMAT>();
        constexpr int WPT = 8 / SPLIT;  // code words per thread and chunk
        const int lane = tid & 31;
        const int m_idx = NMAT == 2 ? (warp >> 2) / SPLIT : 0;
        const int part = (warp >> 2) % SPLIT;
        const int r_idx = 32 * (warp & 3) + lane;
        const int row = m_idx * kPfRows + r_idx;
        const uint32_t t_lane = (uint32_t)(32 * (warp & 3)) << 16;
        auto raw_at = [&](int st) {
            return sraw + ((size_t)st * NMAT * kPfRows + (size_t)row) * 32 + part * WPT * 4;
        };
        struct Mine {  // this thread's matrix of a unit and the unit's weight rows
            QMatDev m;
            int wrow0;
        };
        auto fetch = [&](int ul, Mine &p) {
            PfUnit<NMAT> U;
            unit_of(u_first + ul * u_step, U);
            p.m = (NMAT == 2 && m_idx) ? U.m[NMAT - 1] : U.m[0];
            p.wrow0 = U.wrow0;
        };
        // code copies of the next chunk to issue, one commit group per chunk
        // either way
        Mine iu;
        int ig = 0, ikc = 0, iul = 0, islot = 0;
        auto issue_next = [&]() {
            if (ig < nchunks) {
                if (ikc == 0) fetch(iul, iu);
                const uint32_t *src =
                    iu.m.codes + (size_t)(iu.wrow0 + r_idx) * (K / 8) + (size_t)ikc * 8 + part * WPT;
                if (qmat_ok(iu.m)) {  // an unusable expert (flagged by the router path) leaves stale codes: no access
#pragma unroll
                    for (int q = 0; q < WPT / 4; ++q) cp_async16(raw_at(islot) + 16 * q, src + 4 * q);
                }
                ++ig;
                islot = islot + 1 == kPfRaw ? 0 : islot + 1;
                if (++ikc == nk) {
                    ikc = 0;
                    ++iul;
                }
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        };
        for (int g = 0; g < kPfAhead; ++g) issue_next();
        // scales and biases of this row for 8 chunks at a time (8 bf16 each,
        // in sv / bv), loaded one block ahead: two 16-byte loads when the
        // block is whole and aligned, else value by value
        uint4 sv, bv;
        auto load_sb = [&](const Mine &U, int kc0) {
            const size_t o = (size_t)(U.wrow0 + r_idx) * (K / kPfK) + kc0;
            const uint16_t *sp = U.m.scale + o, *bp = U.m.bias + o;
            const bool ok = qmat_ok(U.m);
            if (ok && kc0 + 8 <= nk && (((reinterpret_cast<uintptr_t>(sp) | reinterpret_cast<uintptr_t>(bp)) & 15u) == 0)) {
                sv = __ldg(reinterpret_cast<const uint4 *>(sp));
                bv = __ldg(reinterpret_cast<const uint4 *>(bp));
            } else {
                uint32_t s2[4], b2[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const bool in0 = ok && kc0 + 2 * j < nk, in1 = ok && kc0 + 2 * j + 1 < nk;
                    s2[j] = (in0 ? ldg_u16(sp + 2 * j) : 0u) | ((in1 ? ldg_u16(sp + 2 * j + 1) : 0u) << 16);
                    b2[j] = (in0 ? ldg_u16(bp + 2 * j) : 0u) | ((in1 ? ldg_u16(bp + 2 * j + 1) : 0u) << 16);
                }
                sv = make_uint4(s2[0], s2[1], s2[2], s2[3]);
                bv = make_uint4(b2[0], b2[1], b2[2], b2[3]);
            }
        };
        Mine cu, nu;  // current and next unit
        if (my_units > 0) {
            fetch(0, cu);
            load_sb(cu, 0);
        }
        // units whose accumulators are read out next: unit ep_ul, whose last
        // chunk is ep_last
        int ep_ul = 0, ep_last = nk - 1;
        auto run_epilogue = [&]() {
            PfUnit<NMAT> U;
            unit_of(u_first + ep_ul * u_step, U);
            epilogue(U.r0, U.nb, U.wrow0, tm + (uint32_t)(ep_ul & 1) * kAccCols);
            ++ep_ul;
            ep_last += nk;
        };
        int kc = 0, ul = 0, slot = 0;
        PfPos apos, epos;  // stage of chunk g, stage of chunk g - kPfStages
        PF_PROF(PfProf pr; pr.start();)
        for (int g = 0; g < nchunks; ++g) {
            if (kc == 0 && ul > 0) cu = nu;
            // the MMAs of chunk g - kPfStages are done: stage apos is free,
            // and a unit whose last chunk that was can be read out
            if (g >= kPfStages) {
                // one lane waits, the warp follows it
                if (lane == 0) pf_wait(&empty[epos.i], (unsigned)epos.ph, status, broken);
                __syncwarp();
                tc_fence_after();
                epos.next(kPfStages);
                PF_PROF(pr.tick(0);)
                if (g - kPfStages == ep_last) run_epilogue();
                PF_PROF(pr.tick(1);)
            }
            issue_next();
            PF_PROF(pr.tick(2);)
            if ((kc & 7) == 0) {
                // this block's values (loaded a block ago) to this thread's
                // own column of shared memory
                {
                    const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w}, bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        ssb[(2 * j) * NP + tid] = (sw[j] & 0xffffu) | (bw[j] << 16);
                        ssb[(2 * j + 1) * NP + tid] = (sw[j] >> 16) | (bw[j] & 0xffff0000u);
                    }
                }
                if (kc + 8 < nk) {
                    load_sb(cu, kc + 8);
                } else if (ul + 1 < my_units) {
                    fetch(ul + 1, nu);
                    load_sb(nu, 0);
                }
            }
            PF_PROF(pr.tick(3);)
            // this thread's copies of chunk g have landed
            asm volatile("cp.async.wait_group %0;" ::"n"(kPfAhead) : "memory");
            PF_PROF(pr.tick(4);)
            {
                // dequantised to fp16 pairs: word c of the row's chunk gives
                // TMEM columns 4c .. 4c + 3 (K order 0,4,1,5,2,6,3,7 per 8)
                const uint32_t sbv = ssb[(kc & 7) * NP + tid];
                const __half2 s2 = pf_bf16_to_half2((uint16_t)(sbv & 0xffffu));
                const __half2 b2 = pf_bf16_to_half2((uint16_t)(sbv >> 16));
                uint32_t ws[WPT];
#pragma unroll
                for (int q = 0; q < WPT / 4; ++q) {
                    const uint4 w4 = *reinterpret_cast<const uint4 *>(raw_at(slot) + 16 * q);
                    ws[4 * q] = w4.x;
                    ws[4 * q + 1] = w4.y;
                    ws[4 * q + 2] = w4.z;
                    ws[4 * q + 3] = w4.w;
                }
                uint32_t v[4 * WPT];
#pragma unroll
                for (int j = 0; j < WPT; ++j) {
                    const uint4 q = pf_dequant_word(ws[j], s2, b2);
                    v[4 * j] = q.x;
                    v[4 * j + 1] = q.y;
                    v[4 * j + 2] = q.z;
                    v[4 * j + 3] = q.w;
                }
                const uint32_t ta = tm + t_lane + (uint32_t)(kABase + apos.i * kStageCols + m_idx * (kPfK / 2) + part * 4 * WPT);
                if constexpr (WPT == 8)
                    tmem_st32(ta, *reinterpret_cast<const uint32_t(*)[32]>(&v[0]));
                else
                    tmem_st16(ta, *reinterpret_cast<const uint32_t(*)[16]>(&v[0]));
                tmem_st_wait();
            }
            PF_PROF(pr.tick(5);)
            // the warp's tensor-memory stores ordered before its one arrival
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[apos.i]);
            PF_PROF(pr.tick(6);)
            apos.next(kPfStages);
            slot = slot + 1 == kPfRaw ? 0 : slot + 1;
            if (++kc == nk) {
                kc = 0;
                ++ul;
            }
        }
        // the last MMAs (their commit covers all earlier ones), then the
        // units not yet read out
        if (nchunks > 0) {
            PfPos last;
            for (int g = 0; g < nchunks - 1; ++g) last.next(kPfStages);
            if (lane == 0) pf_wait(&empty[last.i], (unsigned)last.ph, status, broken);
            __syncwarp();
            tc_fence_after();
            while (ep_ul < my_units) run_epilogue();
        }
        PF_PROF(pr.flush(NMAT - 1, 0);)
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, kTmemCols);
    }
}

// Unit of the gate/up GEMM: tile t (expert e, rows r0.., nb tokens) x row
// block ib of I.
__device__ __forceinline__ void pf_unit_gu(const PfArgs &a, int u, PfUnit<2> &U) {
    const int nib = a.I / kPfRows;
    const int t = u / nib, ib = u % nib;
    const int e = a.p.tile_e[t];
    const QExpertDev &ex = e < a.E ? a.slots[e] : a.shared;
    U.m[0] = ex.gate;
    U.m[1] = ex.up;
    U.wrow0 = ib * kPfRows;
    U.r0 = a.p.tile_r0[t];
    U.nb = a.p.tile_n[t];
}

__global__ void __launch_bounds__(pf_threads<2>(), 1) k_pf_gateup(const __grid_constant__ PfArgs a) {
    griddep_wait();
    const int nunits = *a.p.ntiles * (a.I / kPfRows);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto unit_of = [&](int u, PfUnit<2> &U) { pf_unit_gu(a, u, U); };
    // producer warp w reads TMEM lanes 32(w%4).. (weight rows) and token
    // columns 8(w/4).. in steps of 8 x (producer warps / 4): h = silu(g) * u
    // to Hs (stored K order)
    auto epilogue = [&](int r0, int nb, int wrow0, uint32_t d) {
        const int row = 32 * (warp & 3) + lane;
        const int i = wrow0 + row;
        const int ipos = (i & ~7) | pf_kpos(i & 7);
        for (int c0 = 8 * (warp >> 2); c0 < nb; c0 += 8 * (pf_producers<2>() / 128)) {
            uint32_t g[8], u[8];
            tmem_ld8(d + ((uint32_t)(32 * (warp & 3)) << 16) + c0, g);
            tmem_ld8(d + ((uint32_t)(32 * (warp & 3)) << 16) + kPfTok + c0, u);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (c0 + j < nb) {
                    const float gs = __uint_as_float(g[j]), us = __uint_as_float(u[j]);
                    const float h = gs / (1.f + expf(-gs)) * us;
                    const __half hh = __float2half_rn(h);
                    a.p.hs[(size_t)(r0 + c0 + j) * a.I + ipos] = hh;
                    a.p.hl[(size_t)(r0 + c0 + j) * a.I + ipos] = __float2half_rn(h - __half2float(hh));
                }
        }
        tc_fence_before();
    };
    pf_gemm<2, 1>(nunits, a.H, &a.p.tm_xs, &a.p.tm_xs, unit_of, epilogue, a.ws.status);
}

// Unit of the down GEMM: tile t x row block hb of H.  h enters as its fp16
// high and low parts (two MMA passes into the same accumulator), so only the
// weights are rounded to fp16 here.
__global__ void __launch_bounds__(pf_threads<1>(), 1) k_pf_down(const __grid_constant__ PfArgs a) {
    griddep_wait();
    const int nhb = a.H / kPfRows;
    const int nunits = *a.p.ntiles * nhb;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto unit_of = [&](int u, PfUnit<1> &U) {
        const int t = u / nhb, hb = u % nhb;
        const int e = a.p.tile_e[t];
        U.m[0] = (e < a.E ? a.slots[e] : a.shared).down;
        U.wrow0 = hb * kPfRows;
        U.r0 = a.p.tile_r0[t];
        U.nb = a.p.tile_n[t];
    };
    auto epilogue = [&](int r0, int nb, int wrow0, uint32_t d) {
        const int row = 32 * (warp & 3) + lane;
        for (int c0 = 8 * (warp >> 2); c0 < nb; c0 += 8 * (pf_producers<1>() / 128)) {
            // y = W h_hi + W h_lo: the two accumulators of the set
            uint32_t y[8], yl[8];
            tmem_ld8(d + ((uint32_t)(32 * (warp & 3)) << 16) + c0, y);
            tmem_ld8(d + ((uint32_t)(32 * (warp & 3)) << 16) + kPfTok + c0, yl);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (c0 + j < nb)
                    a.p.ys[(size_t)(r0 + c0 + j) * a.H + wrow0 + row] = __uint_as_float(y[j]) + __uint_as_float(yl[j]);
        }
        tc_fence_before();
    };
    pf_gemm<1, 2>(nunits, a.I, &a.p.tm_hs, &a.p.tm_hl, unit_of, epilogue, a.ws.status);
}

// out[t] = residual[t] + sum_i w_i y_i + gamma y_shared, slot order; one CTA
// per token.
__global__ void __launch_bounds__(256) k_pf_combine(PfArgs a) {
    griddep_wait();
    const int t = blockIdx.x;
    const int *pos = a.p.pos + (size_t)t * a.S;
    const float *w = a.ws.topk_w(t);
    const float gm = *a.ws.gamma(t);
    for (int h = threadIdx.x; h < a.H; h += blockDim.x) {
        float yr = 0.f;
        for (int i = 0; i < a.k; ++i) {
            const int r = pos[i];
            if (r >= 0) yr += w[i] * a.p.ys[(size_t)r * a.H + h];
        }
        float ysh = 0.f;
        if (a.has_shared && pos[a.k] >= 0) ysh = a.p.ys[(size_t)pos[a.k] * a.H + h];
        const float o = bf16_bits_to_float(a.residual[(size_t)t * a.H + h]) + yr + gm * ysh;
        a.out[(size_t)t * a.H + h] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
    }
}

}  // namespace moeq
