// moeq.cu -- C ABI entry points of libmoeq (declared in include/moeq.h):
// host-side validation, workspace layout and kernel launches.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>

#include "cache.hpp"
#include "common.cuh"
#include "ffn.cuh"
#include "prefill.cuh"
#include "route.cuh"
#include "route_batch.cuh"

namespace moeq {
namespace {

thread_local std::string g_err;

moe_status fail(moe_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return st;
}

moe_status cuda_fail(cudaError_t e, const char *what) {
    return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Per-device cached attributes and one-time kernel attribute setup.
// FFN kernel variants: (gate/up | down) x (4 | 2 bits) x (K a multiple of
// the item's windows | ragged K).
enum FfnKernel { kGU4F, kGU4R, kGU2F, kGU2R, kD4F, kD4R, kD2F, kD2R, kRouteF32, kRouteBF16, kPfGU, kPfDown,
                 kNumKernels };

const void *kernel_ptr(int i) {
    switch (i) {
    case kGU4F: return reinterpret_cast<const void *>(&k_gateup<4, true>);
    case kGU4R: return reinterpret_cast<const void *>(&k_gateup<4, false>);
    case kGU2F: return reinterpret_cast<const void *>(&k_gateup<2, true>);
    case kGU2R: return reinterpret_cast<const void *>(&k_gateup<2, false>);
    case kD4F: return reinterpret_cast<const void *>(&k_down<4, true>);
    case kD4R: return reinterpret_cast<const void *>(&k_down<4, false>);
    case kD2F: return reinterpret_cast<const void *>(&k_down<2, true>);
    case kD2R: return reinterpret_cast<const void *>(&k_down<2, false>);
    case kRouteF32: return reinterpret_cast<const void *>(&k_route<true>);
    case kRouteBF16: return reinterpret_cast<const void *>(&k_route<false>);
    case kPfGU: return reinterpret_cast<const void *>(&k_pf_gateup);
    default: return reinterpret_cast<const void *>(&k_pf_down);
    }
}

struct DevInfo {
    int sms = 0;
    int smem_optin = 0;
    int static_smem[kNumKernels] = {};
    bool attrs_set = false;
};
constexpr int kMaxDevices = 64;
DevInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

moe_status dev_info(DevInfo **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device index %d", dev);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DevInfo &d = g_dev[dev];
    if (!d.attrs_set) {
        e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        int optin = 0;
        e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        d.smem_optin = optin;
        for (int i = 0; i < kNumKernels; ++i) {
            // the dynamic allowance is the opt-in limit minus the kernel's static shared memory
            cudaFuncAttributes fa{};
            e = cudaFuncGetAttributes(&fa, kernel_ptr(i));
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
            d.static_smem[i] = (int)fa.sharedSizeBytes;
            e = cudaFuncSetAttribute(kernel_ptr(i), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     optin - (int)fa.sharedSizeBytes);
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        }
        d.attrs_set = true;
    }
    *out = &d;
    return MOE_OK;
}

moe_status check_desc(const moe_layer_desc *d) {
    if (!d) return fail(MOE_ERR_INVALID_ARG, "desc is NULL");
    if (d->group_size != kGroup) return fail(MOE_ERR_UNSUPPORTED, "group_size %d (only 64)", d->group_size);
    if (d->bits != 4 && d->bits != 2) return fail(MOE_ERR_UNSUPPORTED, "bits %d (only 4 or 2)", d->bits);
    if (d->hidden <= 0 || d->hidden % kGroup || d->hidden > kMaxDim)
        return fail(MOE_ERR_INVALID_ARG, "hidden %d: need a multiple of 64 in [64, %d]", d->hidden, kMaxDim);
    if (d->inter <= 0 || d->inter % kGroup || d->inter > kMaxDim)
        return fail(MOE_ERR_INVALID_ARG, "inter %d: need a multiple of 64 in [64, %d]", d->inter, kMaxDim);
    if (d->n_experts <= 0 || d->n_experts > kMaxExperts)
        return fail(MOE_ERR_INVALID_ARG, "n_experts %d: need 1..%d", d->n_experts, kMaxExperts);
    if (d->top_k <= 0 || d->top_k > d->n_experts || d->top_k > kMaxTopK)
        return fail(MOE_ERR_INVALID_ARG, "top_k %d: need 1..min(n_experts, %d)", d->top_k, kMaxTopK);
    if (d->has_shared != 0 && d->has_shared != 1) return fail(MOE_ERR_INVALID_ARG, "has_shared must be 0 or 1");
    return MOE_OK;
}

int n_windows(int K) { return (K + kWinK - 1) / kWinK; }

WsLayout ws_layout(const moe_layer_desc &d) {
    WsLayout L{};
    const size_t S = (size_t)d.top_k + (size_t)d.has_shared;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    L.route_cnt = take(4);
    L.ready = take(4);
    L.logits = take(8 * ((size_t)d.n_experts + 1));
    L.topk_idx = take(4 * (size_t)d.top_k);
    L.topk_w = take(4 * (size_t)d.top_k);
    L.gamma = take(4);
    L.ximg = take(sizeof(uint2) * kImgWinEntries * (size_t)n_windows(d.hidden));
    L.xsg = take(4 * (size_t)(d.hidden / kGroup));
    L.xdg = take(4 * (size_t)(d.hidden / kGroup));
    L.rx = take(sizeof(QExpertDev) * S);
    L.rok = take(4 * S);
    L.h = take(4 * S * (size_t)d.inter);
    L.tok_stride = off;
    return L;
}

// ------------------------------------------------------------ prefill

// The layer takes the sorted grouped-GEMM path for this many tokens or more
// (4-bit experts, hidden and inter multiples of 128); fewer tokens take the
// decode kernels.
constexpr int kPrefillMinTokens = 64;

bool prefill_shape(const moe_layer_desc &d) {
    return d.bits == 4 && d.hidden % kPfRows == 0 && d.inter % kPfRows == 0;
}

struct PfLayout {
    size_t cnt, fill, off, ntiles, tile_e, tile_r0, tile_n, pos, xh, xs, hs, hl, ys, bytes;
    int pcap, tcap;
};

PfLayout pf_layout(const moe_layer_desc &d, int T) {
    PfLayout L{};
    const int S = d.top_k + d.has_shared, n = d.n_experts + 1;
    L.pcap = T * S + kPfPad * n;
    L.tcap = (T * S + kPfTok - 1) / kPfTok + n;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    L.cnt = take(4 * (size_t)n);
    L.fill = take(4 * (size_t)n);
    L.off = take(4 * ((size_t)n + 1));
    L.ntiles = take(4);
    L.tile_e = take(4 * (size_t)L.tcap);
    L.tile_r0 = take(4 * (size_t)L.tcap);
    L.tile_n = take(4 * (size_t)L.tcap);
    L.pos = take(4 * (size_t)T * S);
    L.xh = take(2 * (size_t)T * d.hidden);
    L.xs = take(2 * (size_t)L.pcap * d.hidden);
    L.hs = take(2 * (size_t)L.pcap * d.inter);
    L.hl = take(2 * (size_t)L.pcap * d.inter);
    L.ys = take(4 * (size_t)L.pcap * d.hidden);
    L.bytes = off;
    return L;
}

WsPtrs ws_ptrs(const moe_layer_desc &d, void *ws) {
    WsPtrs p;
    p.L = ws_layout(d);
    p.status = reinterpret_cast<int *>(ws);
    p.sync = reinterpret_cast<unsigned *>(reinterpret_cast<unsigned char *>(ws) + kWsSyncOffset);
    p.base = reinterpret_cast<unsigned char *>(ws) + kWsHeader;
    return p;
}

moe_status check_ws(void *ws) {
    if (!ws) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
    if (!aligned(ws, 256)) return fail(MOE_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    return MOE_OK;
}

moe_status check_tokens(int32_t T) {
    if (T < 0 || T > 65535) return fail(MOE_ERR_INVALID_ARG, "T %d: need 0..65535", T);
    return MOE_OK;
}

moe_status check_qmat_host(const moe_qmat &m, const char *what) {
    if (!m.codes || !m.scale || !m.bias) return fail(MOE_ERR_INVALID_ARG, "shared expert %s: NULL pointer", what);
    if (!aligned(m.codes, 16)) return fail(MOE_ERR_INVALID_ARG, "shared expert %s codes not 16-byte aligned", what);
    if (!aligned(m.scale, 2) || !aligned(m.bias, 2))
        return fail(MOE_ERR_INVALID_ARG, "shared expert %s scale/bias not 2-byte aligned", what);
    return MOE_OK;
}

moe_status check_experts(const moe_layer_desc &d, const moe_slot_table *slots, const moe_qexpert *shared) {
    if (!slots || !slots->slots) return fail(MOE_ERR_INVALID_ARG, "slot table is NULL");
    if (slots->n_slots < d.n_experts)
        return fail(MOE_ERR_INVALID_ARG, "slot table has %d slots < n_experts %d", slots->n_slots, d.n_experts);
    if (!aligned(slots->slots, 8)) return fail(MOE_ERR_INVALID_ARG, "slot table not 8-byte aligned");
    if (d.has_shared) {
        if (!shared) return fail(MOE_ERR_INVALID_ARG, "has_shared=1 but shared expert is NULL");
        moe_status st;
        if ((st = check_qmat_host(shared->gate, "gate")) || (st = check_qmat_host(shared->up, "up")) ||
            (st = check_qmat_host(shared->down, "down")))
            return st;
    } else if (shared) {
        return fail(MOE_ERR_INVALID_ARG, "shared expert given but has_shared=0");
    }
    return MOE_OK;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
    return pa < pb + nb && pb < pa + na;
}

QExpertDev to_dev(const moe_qexpert *e) {
    QExpertDev x{};
    if (e) std::memcpy(&x, e, sizeof x);
    return x;
}

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                   Args &&...args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

size_t route_smem(const moe_layer_desc &d) { return (size_t)d.hidden * sizeof(float); }


// Tile-slot ring of the FFN kernels: slots of nwg * vals floats, about 16 KB
// in all, between 4 and 128 slots.
int ring_slots(int nwg, int vals) {
    const int slot = nwg * vals * (int)sizeof(float);
    int r = 4;  // a power of two
    while (r < 128 && 2 * r * slot <= 16384) r *= 2;
    return r;
}
size_t ring_bytes(int nwg, int vals) {
    const int R = ring_slots(nwg, vals);
    return (size_t)R * nwg * vals * sizeof(float) + 2 * (size_t)R * sizeof(int);
}
// Work items hold one window of NMAT 16-row blocks: gate/up 2 * gu_sub,
// down dn_sub; a tile has one item per window.
int gateup_nwg(const moe_layer_desc &d) { return n_windows(d.hidden); }
int down_nwg(const moe_layer_desc &d) { return n_windows(d.inter); }
int gateup_vals(const moe_layer_desc &d) { return 2 * gu_sub(d.bits) * kTileRows; }
int down_vals(const moe_layer_desc &d) { return dn_sub(d.bits) * kTileRows; }
// Item loads need no bounds checks when K covers whole windows.
bool gateup_full(const moe_layer_desc &d) { return d.hidden % kWinK == 0; }
bool down_full(const moe_layer_desc &d) { return d.inter % kWinK == 0; }

// Gate/up kernel: image | tile ring | slot table (routing in the kernel;
// placed at the next 16-byte boundary).
size_t gateup_smem(const moe_layer_desc &d, bool with_table) {
    const int nw = n_windows(d.hidden);
    size_t b = (size_t)nw * kImgWinEntries * sizeof(uint2) + ring_bytes(gateup_nwg(d), gateup_vals(d));
    if (with_table) b += 16 + sizeof(QExpertDev) * (size_t)d.n_experts;
    return b;
}

// Down kernel with M expert images per pass and at most NB row bands per CTA:
// images | group sums | group steps | tile ring | band partials | band counts | residual
// rows.
size_t down_smem(const moe_layer_desc &d, int M, int NB) {
    const int nw = n_windows(d.inter), ngr = d.inter / kGroup;
    const int S = d.top_k + d.has_shared, rpt = dn_sub(d.bits) * kTileRows;
    return (size_t)M * ((size_t)nw * kImgWinEntries * sizeof(uint2) + 8 * (size_t)ngr) +
           ring_bytes(down_nwg(d), down_vals(d)) + (size_t)NB * S * rpt * 4 + (size_t)NB * 4 +
           (size_t)NB * rpt * 2;
}

moe_status launch_route(const moe_layer_desc &d, const void *x, int32_t T, const void *w_router,
                        moe_dtype rdt, const float *logit_bias, const void *shared_gate, int32_t *idx_out,
                        float *w_out, const WsPtrs &wp, cudaStream_t st, int do_topk, int build_image,
                        int norm = 0, float eps = 0.f, void *xhat_out = nullptr) {
    RouteArgs a{};
    a.norm = norm;
    a.eps = eps;
    a.xhat_out = static_cast<uint16_t *>(xhat_out);
    a.x = static_cast<const uint16_t *>(x);
    a.T = T;
    a.H = d.hidden;
    a.E = d.n_experts;
    a.k = d.top_k;
    a.w_router = w_router;
    a.logit_bias = logit_bias;
    a.shared_gate = static_cast<const uint16_t *>(shared_gate);
    a.topk_idx_out = idx_out;
    a.topk_w_out = w_out;
    a.ws = wp;
    a.do_topk = do_topk;
    a.build_image = build_image;
    a.bits = d.bits;
    const int rows = d.n_experts + (shared_gate ? 1 : 0);
    if (do_topk && !build_image && T >= kRouteGemmMinTokens) {
        // many tokens: the router as a tiled GEMM, then one top-k CTA per token
        const dim3 gg((rows + kRgRows - 1) / kRgRows, (T + kRgTok - 1) / kRgTok);
        cudaError_t e = rdt == MOE_DT_F32 ? launch(k_route_gemm<true>, gg, dim3(kRgThreads), 0, st, a)
                                          : launch(k_route_gemm<false>, gg, dim3(kRgThreads), 0, st, a);
        if (e != cudaSuccess) return cuda_fail(e, "launch k_route_gemm");
        if ((e = launch(k_route_topk, dim3(T), dim3(kRouteThreads), 0, st, a)) != cudaSuccess)
            return cuda_fail(e, "launch k_route_topk");
        return MOE_OK;
    }
    const dim3 grid((rows + kRouteRowsPerCta - 1) / kRouteRowsPerCta + build_image, T);
    const size_t smem = route_smem(d);
    cudaError_t e = rdt == MOE_DT_F32 ? launch(k_route<true>, grid, dim3(kRouteThreads), smem, st, a)
                                      : launch(k_route<false>, grid, dim3(kRouteThreads), smem, st, a);
    if (e != cudaSuccess) return cuda_fail(e, "launch k_route");
    return MOE_OK;
}

// Kernel boundary events of moe_set_kernel_events (per host thread).
thread_local cudaEvent_t g_kernel_events[4];
thread_local bool g_kernel_events_on = false;

moe_status record_event(int i, cudaStream_t st) {
    if (!g_kernel_events_on) return MOE_OK;
    cudaError_t e = cudaEventRecord(g_kernel_events[i], st);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "cudaEventRecord (kernel events)");
}

moe_status launch_ffn(const moe_layer_desc &d, const DevInfo &di, FfnArgs &a, cudaStream_t st) {
    const int b4 = d.bits == 4;
    const int kg = b4 ? (gateup_full(d) ? kGU4F : kGU4R) : (gateup_full(d) ? kGU2F : kGU2R);
    const int kd = b4 ? (down_full(d) ? kD4F : kD4R) : (down_full(d) ? kD2F : kD2R);
    const size_t sg = gateup_smem(d, a.route_in_gateup != 0);
    if ((long)sg > (long)di.smem_optin - di.static_smem[kg])
        return fail(MOE_ERR_UNSUPPORTED, "shared memory too small for this layer shape (gate/up)");
    // down: every CTA owns at most NB row bands; as many expert images per
    // pass as the shared memory holds
    const int S = d.top_k + d.has_shared;
    const int nbands = d.hidden / (dn_sub(d.bits) * kTileRows);
    const int NB = (nbands + di.sms - 1) / di.sms;
    int M = S;
    while (M > 0 && (long)down_smem(d, M, NB) > (long)di.smem_optin - di.static_smem[kd]) --M;
    if (M == 0) return fail(MOE_ERR_UNSUPPORTED, "shared memory too small for this layer shape (down)");
    const size_t sd = down_smem(d, M, NB);
    a.dn_slots = M;
    a.dn_bands_max = NB;
    cudaError_t e = cudaSuccess;
    a.ring_slots = ring_slots(gateup_nwg(d), gateup_vals(d));
    switch (kg) {
    case kGU4F: e = launch(k_gateup<4, true>, dim3(di.sms), dim3(kFfnThreads), sg, st, a); break;
    case kGU4R: e = launch(k_gateup<4, false>, dim3(di.sms), dim3(kFfnThreads), sg, st, a); break;
    case kGU2F: e = launch(k_gateup<2, true>, dim3(di.sms), dim3(kFfnThreads), sg, st, a); break;
    default: e = launch(k_gateup<2, false>, dim3(di.sms), dim3(kFfnThreads), sg, st, a); break;
    }
    if (e != cudaSuccess) return cuda_fail(e, "launch k_gateup");
    moe_status rs;
    if ((rs = record_event(2, st))) return rs;
    a.ring_slots = ring_slots(down_nwg(d), down_vals(d));
    switch (kd) {
    case kD4F: e = launch(k_down<4, true>, dim3(di.sms), dim3(kFfnThreads), sd, st, a); break;
    case kD4R: e = launch(k_down<4, false>, dim3(di.sms), dim3(kFfnThreads), sd, st, a); break;
    case kD2F: e = launch(k_down<2, true>, dim3(di.sms), dim3(kFfnThreads), sd, st, a); break;
    default: e = launch(k_down<2, false>, dim3(di.sms), dim3(kFfnThreads), sd, st, a); break;
    }
    if (e != cudaSuccess) return cuda_fail(e, "launch k_down");
    return MOE_OK;
}

// cuTensorMapEncodeTiled from the driver (looked up once per process).
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

moe_status encode_fn(EncodeTiledFn *fn) {
    static std::once_flag once;
    static EncodeTiledFn f = nullptr;
    static cudaError_t err = cudaSuccess;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) f = reinterpret_cast<EncodeTiledFn>(p);
    });
    if (!f) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled not available (%s)", cudaGetErrorString(err));
    *fn = f;
    return MOE_OK;
}

// TMA map of a row-major fp16 matrix [rows][cols] read in boxes of 64 values
// x 16 rows with the 128-byte swizzle (the layout the MMA descriptors use).
moe_status tma_map_rows(CUtensorMap *m, const void *base, int cols, int rows) {
    EncodeTiledFn fn;
    moe_status st;
    if ((st = encode_fn(&fn))) return st;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kPfK, 16};
    const cuuint32_t es[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return MOE_OK;
}

// The prefill chain after the router kernel: count, scan, scatter, gate/up
// GEMM, down GEMM, combine.
moe_status launch_prefill(const moe_layer_desc &d, const DevInfo &di, PfArgs &a, cudaStream_t st) {
    const size_t sg = PfSmem<2, 1>::total, sd = PfSmem<1, 2>::total;
    if ((long)sg > (long)di.smem_optin - di.static_smem[kPfGU] || (long)sd > (long)di.smem_optin - di.static_smem[kPfDown])
        return fail(MOE_ERR_UNSUPPORTED, "shared memory too small for the prefill kernels");
    moe_status ms;
    if ((ms = tma_map_rows(&a.p.tm_xs, a.p.xs, d.hidden, a.p.pcap)) ||
        (ms = tma_map_rows(&a.p.tm_hs, a.p.hs, d.inter, a.p.pcap)) ||
        (ms = tma_map_rows(&a.p.tm_hl, a.p.hl, d.inter, a.p.pcap)))
        return ms;
    const int pairs = a.T * a.S;
    cudaError_t e = cudaMemsetAsync(a.p.cnt, 0, 4 * ((size_t)d.n_experts + 1), st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync (prefill counts)");
    if ((e = launch(k_pf_count, dim3((pairs + 255) / 256), dim3(256), 0, st, a)) != cudaSuccess)
        return cuda_fail(e, "launch k_pf_count");
    if ((e = launch(k_pf_scan, dim3(1), dim3(1024), 0, st, a)) != cudaSuccess) return cuda_fail(e, "launch k_pf_scan");
    if ((e = launch(k_pf_scatter, dim3((pairs + 7) / 8), dim3(256), 0, st, a)) != cudaSuccess)
        return cuda_fail(e, "launch k_pf_scatter");
    if ((e = launch(k_pf_gateup, dim3(di.sms), dim3(pf_threads<2>()), sg, st, a)) != cudaSuccess)
        return cuda_fail(e, "launch k_pf_gateup");
    moe_status rs;
    if ((rs = record_event(2, st))) return rs;
    if ((e = launch(k_pf_down, dim3(di.sms), dim3(pf_threads<1>()), sd, st, a)) != cudaSuccess)
        return cuda_fail(e, "launch k_pf_down");
    if ((e = launch(k_pf_combine, dim3(a.T), dim3(256), 0, st, a)) != cudaSuccess)
        return cuda_fail(e, "launch k_pf_combine");
    return MOE_OK;
}

moe_status expert_ffn(int bits, const moe_layer_desc *desc, const void *x, int32_t T,
                      const moe_slot_table *slots, const moe_qexpert *shared, const int32_t *topk_idx,
                      const float *topk_w, float *y, void *ws, moe_stream_t stream) {
    g_err.clear();
    moe_status st;
    if ((st = check_desc(desc)) || (st = check_tokens(T)) || (st = check_ws(ws))) return st;
    if (desc->bits != bits)
        return fail(MOE_ERR_INVALID_ARG, "desc->bits is %d but this entry point is for %d-bit experts", desc->bits, bits);
    if ((st = check_experts(*desc, slots, shared))) return st;
    if (T == 0) return MOE_OK;
    if (!x || !aligned(x, 16)) return fail(MOE_ERR_INVALID_ARG, "x NULL or not 16-byte aligned");
    if (!topk_idx || !topk_w || !aligned(topk_idx, 4) || !aligned(topk_w, 4))
        return fail(MOE_ERR_INVALID_ARG, "topk_idx/topk_w NULL or misaligned");
    if (!y || !aligned(y, 4)) return fail(MOE_ERR_INVALID_ARG, "y NULL or misaligned");
    DevInfo *di;
    if ((st = dev_info(&di))) return st;
    FfnArgs a{};
    a.T = T;
    a.H = desc->hidden;
    a.I = desc->inter;
    a.E = desc->n_experts;
    a.k = desc->top_k;
    a.S = desc->top_k + desc->has_shared;
    a.x = static_cast<const uint16_t *>(x);
    a.slots = reinterpret_cast<const QExpertDev *>(slots->slots);
    a.n_slots = slots->n_slots;
    a.shared = to_dev(shared);
    a.idx_base = topk_idx;
    a.idx_stride = (size_t)desc->top_k;
    a.w_base = topk_w;
    a.w_stride = (size_t)desc->top_k;
    a.gamma_base = nullptr;
    a.ws = ws_ptrs(*desc, ws);
    a.ysplit = y;
    a.mode = kCombineSplit;
    return launch_ffn(*desc, *di, a, reinterpret_cast<cudaStream_t>(stream));
}

// Scratch of moe_layer_forward_noalloc: a fixed array in the device image
// (one copy per GPU that loads the library, held until exit).  Host code
// must not use the name g_noalloc_scratch as a device address: it is a host
// stand-in; the real address comes from cudaGetSymbolAddress, looked up once
// per device below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];
void *g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;

moe_status noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device index %d", dev);
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return MOE_OK;
}

}  // namespace
}  // namespace moeq

using namespace moeq;

extern "C" {

const char *moe_version(void) { return "moeq 0.1 (sm_100a)"; }

struct moe_expert_cache {
    moeq::ExpertCache c;
};

moe_status moe_cache_create(int32_t n_experts, int32_t n_slots, moe_expert_cache **out) {
    g_err.clear();
    if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (n_experts < 1 || n_slots < 1 || n_slots > n_experts)
        return fail(MOE_ERR_INVALID_ARG, "n_experts %d, n_slots %d: need 1 <= n_slots <= n_experts", n_experts,
                    n_slots);
    *out = new moe_expert_cache{moeq::ExpertCache(n_experts, n_slots)};
    return MOE_OK;
}

void moe_cache_destroy(moe_expert_cache *cache) { delete cache; }

moe_status moe_cache_plan(moe_expert_cache *cache, const int32_t *ids, int32_t k, int32_t *slot_of,
                          int32_t *fill_ids, int32_t *fill_slots, int32_t *n_fill) {
    g_err.clear();
    if (!cache || !ids || !slot_of || !fill_ids || !fill_slots || !n_fill)
        return fail(MOE_ERR_INVALID_ARG, "NULL argument");
    if (k < 1 || k > cache->c.n_slots())
        return fail(MOE_ERR_INVALID_ARG, "k %d: need 1 <= k <= n_slots (%d)", k, cache->c.n_slots());
    if (cache->c.plan(ids, k, slot_of, fill_ids, fill_slots, n_fill))
        return fail(MOE_ERR_INVALID_ARG, "expert id out of range or repeated");
    return MOE_OK;
}

moe_status moe_cache_stats(const moe_expert_cache *cache, int64_t *hits, int64_t *misses) {
    g_err.clear();
    if (!cache) return fail(MOE_ERR_INVALID_ARG, "cache is NULL");
    if (hits) *hits = cache->c.hits();
    if (misses) *misses = cache->c.misses();
    return MOE_OK;
}

const char *moe_last_error(void) { return g_err.c_str(); }

size_t moe_workspace_size(const moe_layer_desc *desc, int32_t max_tokens) {
    if (check_desc(desc) != MOE_OK || max_tokens < 0) return 0;
    size_t b = kWsHeader + (size_t)max_tokens * ws_layout(*desc).tok_stride;
    if (max_tokens >= kPrefillMinTokens && prefill_shape(*desc)) b += pf_layout(*desc, max_tokens).bytes;
    return b;
}

moe_status moe_workspace_init(void *ws, size_t bytes, moe_stream_t stream) {
    g_err.clear();
    moe_status st;
    if ((st = check_ws(ws))) return st;
    cudaError_t e = cudaMemsetAsync(ws, 0, bytes, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    return MOE_OK;
}

moe_status moe_route(const moe_layer_desc *desc, const void *x, int32_t T, const void *w_router,
                     moe_dtype router_dtype, const float *logit_bias, int32_t *topk_idx, float *topk_w,
                     void *ws, moe_stream_t stream) {
    g_err.clear();
    moe_status st;
    if ((st = check_desc(desc)) || (st = check_tokens(T)) || (st = check_ws(ws))) return st;
    if (router_dtype != MOE_DT_BF16 && router_dtype != MOE_DT_F32)
        return fail(MOE_ERR_INVALID_ARG, "router_dtype %d", (int)router_dtype);
    if (T == 0) return MOE_OK;
    if (!x || !aligned(x, 16)) return fail(MOE_ERR_INVALID_ARG, "x NULL or not 16-byte aligned");
    if (!w_router || !aligned(w_router, 16)) return fail(MOE_ERR_INVALID_ARG, "w_router NULL or not 16-byte aligned");
    if (logit_bias && !aligned(logit_bias, 4)) return fail(MOE_ERR_INVALID_ARG, "logit_bias misaligned");
    if (!topk_idx || !topk_w) return fail(MOE_ERR_INVALID_ARG, "topk_idx/topk_w NULL");
    DevInfo *di;
    if ((st = dev_info(&di))) return st;
    return launch_route(*desc, x, T, w_router, router_dtype, logit_bias, nullptr, topk_idx, topk_w,
                        ws_ptrs(*desc, ws), reinterpret_cast<cudaStream_t>(stream), 1, 0);
}

moe_status moe_expert_ffn_q4(const moe_layer_desc *desc, const void *x, int32_t T, const moe_slot_table *slots,
                             const moe_qexpert *shared, const int32_t *topk_idx, const float *topk_w, float *y,
                             void *ws, moe_stream_t stream) {
    return expert_ffn(4, desc, x, T, slots, shared, topk_idx, topk_w, y, ws, stream);
}

moe_status moe_expert_ffn_q2(const moe_layer_desc *desc, const void *x, int32_t T, const moe_slot_table *slots,
                             const moe_qexpert *shared, const int32_t *topk_idx, const float *topk_w, float *y,
                             void *ws, moe_stream_t stream) {
    return expert_ffn(2, desc, x, T, slots, shared, topk_idx, topk_w, y, ws, stream);
}

moe_status moe_combine_residual(const moe_layer_desc *desc, const float *y, const void *residual,
                                const void *shared_gate, const void *x, int32_t T, void *out,
                                moe_stream_t stream) {
    g_err.clear();
    moe_status st;
    if ((st = check_desc(desc)) || (st = check_tokens(T))) return st;
    if (T == 0) return MOE_OK;
    if (!y || !residual || !out) return fail(MOE_ERR_INVALID_ARG, "y/residual/out NULL");
    if (shared_gate && !x) return fail(MOE_ERR_INVALID_ARG, "shared_gate needs x");
    cudaError_t e = launch(k_combine, dim3(T), dim3(256), 0, reinterpret_cast<cudaStream_t>(stream), y,
                           static_cast<const uint16_t *>(residual), static_cast<const uint16_t *>(shared_gate),
                           static_cast<const uint16_t *>(x), (int)desc->hidden, static_cast<uint16_t *>(out));
    if (e != cudaSuccess) return cuda_fail(e, "launch k_combine");
    return MOE_OK;
}

// The layer, with x either the normalised input (norm = 0) or the hidden
// state h itself (norm = 1: x-hat = rmsnorm(h) inside, residual = h).
static moe_status layer_forward_impl(const moe_layer_desc *desc, const void *x, const void *residual, int32_t T,
                                     int norm, float eps, void *xhat_out, const void *w_router,
                                     moe_dtype router_dtype, const float *logit_bias, const moe_slot_table *slots,
                                     const moe_qexpert *shared, const void *shared_gate, void *out,
                                     int32_t *topk_idx_out, float *topk_w_out, void *ws, moe_stream_t stream) {
    moe_status st;
    if ((st = check_desc(desc)) || (st = check_tokens(T)) || (st = check_ws(ws))) return st;
    if ((st = check_experts(*desc, slots, shared))) return st;
    if (router_dtype != MOE_DT_BF16 && router_dtype != MOE_DT_F32)
        return fail(MOE_ERR_INVALID_ARG, "router_dtype %d", (int)router_dtype);
    if (shared_gate && !desc->has_shared) return fail(MOE_ERR_INVALID_ARG, "shared_gate given but has_shared=0");
    if (shared_gate && !aligned(shared_gate, 16))
        return fail(MOE_ERR_INVALID_ARG, "shared_gate not 16-byte aligned");
    if (T == 0) return MOE_OK;
    if (!x || !aligned(x, 16)) return fail(MOE_ERR_INVALID_ARG, "x NULL or not 16-byte aligned");
    if (!residual || !aligned(residual, 2)) return fail(MOE_ERR_INVALID_ARG, "residual NULL or misaligned");
    if (!out || !aligned(out, 2)) return fail(MOE_ERR_INVALID_ARG, "out NULL or misaligned");
    if (!w_router || !aligned(w_router, 16)) return fail(MOE_ERR_INVALID_ARG, "w_router NULL or not 16-byte aligned");
    if (logit_bias && !aligned(logit_bias, 4)) return fail(MOE_ERR_INVALID_ARG, "logit_bias misaligned");
    const size_t xb = (size_t)T * desc->hidden * 2;
    if (!norm && overlaps(out, xb, x, xb)) return fail(MOE_ERR_INVALID_ARG, "out overlaps x");
    if (residual != out && overlaps(out, xb, residual, xb))
        return fail(MOE_ERR_INVALID_ARG, "out partially overlaps residual");
    if (xhat_out && !aligned(xhat_out, 16)) return fail(MOE_ERR_INVALID_ARG, "xhat_out not 16-byte aligned");
    if (xhat_out && (overlaps(xhat_out, xb, x, xb) || overlaps(xhat_out, xb, out, xb)))
        return fail(MOE_ERR_INVALID_ARG, "xhat_out overlaps h or out");
    DevInfo *di;
    if ((st = dev_info(&di))) return st;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const WsPtrs wp = ws_ptrs(*desc, ws);
    if ((st = record_event(0, s))) return st;
    if (T >= kPrefillMinTokens && prefill_shape(*desc)) {
        // many tokens: (the normalisation into x-hat,) the router as a
        // batched GEMM with a top-k CTA per token, then the expert-sorted
        // GEMM path
        const PfLayout PL = pf_layout(*desc, T);
        unsigned char *pb = static_cast<unsigned char *>(ws) + kWsHeader + (size_t)T * wp.L.tok_stride;
        if (norm) {
            void *xh = xhat_out ? xhat_out : static_cast<void *>(pb + PL.xh);
            cudaError_t e = launch(k_rmsnorm, dim3(T), dim3(256), 0, s, static_cast<const uint16_t *>(x),
                                   (int)desc->hidden, eps, static_cast<uint16_t *>(xh));
            if (e != cudaSuccess) return cuda_fail(e, "launch k_rmsnorm");
            x = xh;
        }
        if ((st = launch_route(*desc, x, T, w_router, router_dtype, logit_bias, shared_gate, topk_idx_out,
                               topk_w_out, wp, s, 1, 0)))
            return st;
        if ((st = record_event(1, s))) return st;
        PfArgs pa{};
        pa.T = T;
        pa.H = desc->hidden;
        pa.I = desc->inter;
        pa.E = desc->n_experts;
        pa.k = desc->top_k;
        pa.S = desc->top_k + desc->has_shared;
        pa.has_shared = desc->has_shared;
        pa.x = static_cast<const uint16_t *>(x);
        pa.residual = static_cast<const uint16_t *>(residual);
        pa.out = static_cast<uint16_t *>(out);
        pa.slots = reinterpret_cast<const QExpertDev *>(slots->slots);
        pa.shared = to_dev(shared);
        pa.ws = wp;
        pa.p.cnt = reinterpret_cast<unsigned *>(pb + PL.cnt);
        pa.p.fill = reinterpret_cast<unsigned *>(pb + PL.fill);
        pa.p.off = reinterpret_cast<int *>(pb + PL.off);
        pa.p.ntiles = reinterpret_cast<int *>(pb + PL.ntiles);
        pa.p.tile_e = reinterpret_cast<int *>(pb + PL.tile_e);
        pa.p.tile_r0 = reinterpret_cast<int *>(pb + PL.tile_r0);
        pa.p.tile_n = reinterpret_cast<int *>(pb + PL.tile_n);
        pa.p.pos = reinterpret_cast<int *>(pb + PL.pos);
        pa.p.xs = reinterpret_cast<__half *>(pb + PL.xs);
        pa.p.hs = reinterpret_cast<__half *>(pb + PL.hs);
        pa.p.hl = reinterpret_cast<__half *>(pb + PL.hl);
        pa.p.ys = reinterpret_cast<float *>(pb + PL.ys);
        pa.p.pcap = PL.pcap;
        pa.p.tcap = PL.tcap;
        if ((st = launch_prefill(*desc, *di, pa, s))) return st;
        return record_event(3, s);
    }
    if ((st = launch_route(*desc, x, T, w_router, router_dtype, logit_bias, shared_gate, nullptr, nullptr, wp, s,
                           0, 1, norm, eps, xhat_out)))
        return st;
    if ((st = record_event(1, s))) return st;
    FfnArgs a{};
    a.T = T;
    a.H = desc->hidden;
    a.I = desc->inter;
    a.E = desc->n_experts;
    a.k = desc->top_k;
    a.S = desc->top_k + desc->has_shared;
    a.x = static_cast<const uint16_t *>(x);
    a.slots = reinterpret_cast<const QExpertDev *>(slots->slots);
    a.n_slots = slots->n_slots;
    a.shared = to_dev(shared);
    a.route_in_gateup = 1;
    a.x_image_in_ws = 1;
    a.has_gate = shared_gate != nullptr;
    a.topk_idx_out = topk_idx_out;
    a.topk_w_out = topk_w_out;
    a.w_base = wp.topk_w(0);
    a.w_stride = wp.L.tok_stride / sizeof(float);
    a.gamma_base = shared_gate ? wp.gamma(0) : nullptr;
    a.gamma_stride = wp.L.tok_stride / sizeof(float);
    a.ws = wp;
    a.residual = static_cast<const uint16_t *>(residual);
    a.out = static_cast<uint16_t *>(out);
    a.mode = kCombineFull;
    if ((st = launch_ffn(*desc, *di, a, s))) return st;
    return record_event(3, s);
}

moe_status moe_layer_forward(const moe_layer_desc *desc, const void *x, const void *residual, int32_t T,
                             const void *w_router, moe_dtype router_dtype, const float *logit_bias,
                             const moe_slot_table *slots, const moe_qexpert *shared, const void *shared_gate,
                             void *out, int32_t *topk_idx_out, float *topk_w_out, void *ws, moe_stream_t stream) {
    g_err.clear();
    return layer_forward_impl(desc, x, residual, T, 0, 0.f, nullptr, w_router, router_dtype, logit_bias, slots,
                              shared, shared_gate, out, topk_idx_out, topk_w_out, ws, stream);
}

moe_status moe_layer_forward_normed(const moe_layer_desc *desc, const void *h, int32_t T, float eps,
                                    const void *w_router, moe_dtype router_dtype, const float *logit_bias,
                                    const moe_slot_table *slots, const moe_qexpert *shared,
                                    const void *shared_gate, void *out, void *xhat_out, int32_t *topk_idx_out,
                                    float *topk_w_out, void *ws, moe_stream_t stream) {
    g_err.clear();
    if (!(eps >= 0.f)) return fail(MOE_ERR_INVALID_ARG, "eps must be >= 0");
    return layer_forward_impl(desc, h, h, T, 1, eps, xhat_out, w_router, router_dtype, logit_bias, slots, shared,
                              shared_gate, out, topk_idx_out, topk_w_out, ws, stream);
}

moe_status moe_layer_forward_noalloc(const moe_layer_desc *desc, const void *x, const void *residual, int32_t T,
                                     const void *w_router, moe_dtype router_dtype, const float *logit_bias,
                                     const moe_slot_table *slots, const moe_qexpert *shared,
                                     const void *shared_gate, void *out, int32_t *topk_idx_out,
                                     float *topk_w_out, moe_stream_t stream) {
    g_err.clear();
    moe_status st;
    if ((st = check_desc(desc)) || (st = check_tokens(T))) return st;
    const size_t need = moe_workspace_size(desc, T);
    if (need > MOE_NOALLOC_SCRATCH_BYTES)
        return fail(MOE_ERR_INVALID_ARG,
                    "no-alloc call needs %zu bytes of scratch for T=%d, more than the %zu-byte static "
                    "scratch; use fewer tokens per call or moe_layer_forward with a workspace",
                    need, T, (size_t)MOE_NOALLOC_SCRATCH_BYTES);
    if (T == 0) return MOE_OK;
    void *ws = nullptr;
    if ((st = noalloc_scratch(&ws))) return st;
    // clear what must start at zero: the status word and each token's
    // arrival counters (route count, row-band counts)
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const WsLayout L = ws_layout(*desc);
    cudaError_t e = cudaMemsetAsync(ws, 0, kWsHeader, s);
    if (e == cudaSuccess)
        e = cudaMemset2DAsync(static_cast<unsigned char *>(ws) + kWsHeader, L.tok_stride, 0, L.route_cnt + 4,
                              (size_t)T, s);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the no-alloc scratch counters");
    return moe_layer_forward(desc, x, residual, T, w_router, router_dtype, logit_bias, slots, shared,
                             shared_gate, out, topk_idx_out, topk_w_out, ws, stream);
}

moe_status moe_rmsnorm(const void *x, int32_t T, int32_t H, float eps, void *out, moe_stream_t stream) {
    g_err.clear();
    moe_status st;
    if ((st = check_tokens(T))) return st;
    if (H < 8 || H % 8 || H > kMaxDim) return fail(MOE_ERR_INVALID_ARG, "H %d: need a multiple of 8 in [8, %d]", H, kMaxDim);
    if (!(eps >= 0.f)) return fail(MOE_ERR_INVALID_ARG, "eps must be >= 0");
    if (T == 0) return MOE_OK;
    if (!x || !out || !aligned(x, 16) || !aligned(out, 16))
        return fail(MOE_ERR_INVALID_ARG, "x/out NULL or not 16-byte aligned");
    cudaError_t e = launch(k_rmsnorm, dim3(T), dim3(256), 0, reinterpret_cast<cudaStream_t>(stream),
                           static_cast<const uint16_t *>(x), (int)H, eps, static_cast<uint16_t *>(out));
    if (e != cudaSuccess) return cuda_fail(e, "launch k_rmsnorm");
    return MOE_OK;
}

#ifdef MOEQ_PF_PROFILE
// Profiling builds only: copies (and with reset, clears) the prefill GEMM
// phase counters, 2 x 16 values.
extern "C" moe_status moe_debug_pf_profile(unsigned long long *out, int32_t reset) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_pfprof, sizeof(g_pfprof));
    if (e == cudaSuccess && reset) {
        static const unsigned long long zero[2][16] = {};
        e = cudaMemcpyToSymbol(g_pfprof, zero, sizeof(zero));
    }
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "profile counters");
}
#endif

moe_status moe_set_kernel_events(void *const *events, int32_t n) {
    g_err.clear();
    if (!events && n == 0) {
        g_kernel_events_on = false;
        return MOE_OK;
    }
    if (!events || n != 4) return fail(MOE_ERR_INVALID_ARG, "kernel events: need 4 handles (or NULL, 0)");
    for (int i = 0; i < 4; ++i)
        if (!events[i]) return fail(MOE_ERR_INVALID_ARG, "kernel events: handle %d is NULL", i);
    for (int i = 0; i < 4; ++i) g_kernel_events[i] = static_cast<cudaEvent_t>(events[i]);
    g_kernel_events_on = true;
    return MOE_OK;
}

moe_status moe_get_device_status(void *ws, moe_stream_t stream, int32_t *st_out) {
    g_err.clear();
    moe_status st;
    if ((st = check_ws(ws))) return st;
    if (!st_out) return fail(MOE_ERR_INVALID_ARG, "st is NULL");
    int32_t v = 0;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof v, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "reading device status");
    *st_out = v;
    if (v == 0) return MOE_OK;
    if (v == MOE_DEV_TIMEOUT) return fail(MOE_ERR_TIMEOUT, "device wait timed out");
    return fail(MOE_ERR_DEVICE_FAULT, "device status 0x%x", (unsigned)v);
}

}  // extern "C"
