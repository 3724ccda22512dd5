// api.cu -- the C ABI (include/moe.h): handle lifetime, workspace, tensor maps and the launch
// sequence of one forward call.  Host code only; every step of the layer runs in the kernels.
//
// Prefill path (T > decode_max_tokens), all stream-ordered, no host synchronisation:
//   tensor-core router logits -> top-k/gates/histogram (+ fp16 activation rows, zeroed
//   accumulator) -> bucket scan + tile list -> scatter (bucket row -> token, gate) -> gather of
//   the token rows into bucket order -> tcgen05 gate/up GEMM + SwiGLU -> tcgen05 down GEMM +
//   combine -> bf16 finalize.
// Decode path (T <= decode_max_tokens): split-K router -> top-k/gates -> sparse GEMV gate/up +
//   SwiGLU -> sparse GEMV down + gated combine (bf16 out).
#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/moe.h"
#include "common.cuh"
#include "kernels.h"

using namespace moe;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

#define CUDA_TRY(expr)                                                                              \
    do {                                                                                            \
        cudaError_t _e = (expr);                                                                    \
        if (_e != cudaSuccess) return fail(MOE_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(_e)); \
    } while (0)

// NVTX range around one launch (or one entry-point call) so a timeline tool attributes device
// time to the library's phases; header-only NVTX, a no-op when no tool is attached.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};
#define MOE_LAUNCH(name, expr)    \
    do {                          \
        NvtxRange _nvtx(name);    \
        CUDA_TRY(expr);           \
    } while (0)

struct DeviceGuard {
    int prev = -1;
    bool changed = false;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) {
            changed = cudaSetDevice(dev) == cudaSuccess;
        }
    }
    ~DeviceGuard() {
        if (changed) cudaSetDevice(prev);
    }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Sizes derived from a configuration.
struct Layout {
    int H, I, E, k, G, Tm, Tdec, ks_dec, nblk_max, max_tiles, rows_cap, Epad;
    size_t w_gu_bytes, w_dn_bytes, router_bytes, wsplit_bytes, weights_bytes;
    size_t o_wrt, o_rbias, o_sgw, o_router32;   // offsets inside the router region
    // workspace offsets
    size_t o_part, o_idx, o_gates, o_sg, o_hist, o_sdone, o_counts, o_offsets, o_tiles, o_ntiles, o_perm, o_rtok,
        o_rgate, o_x16, o_xp, o_act, o_acc, o_dact, o_dscale, o_status, o_stage_x, o_stage_out, o_dfz_ticket,
        o_dfz_slots, o_dfz_outacc, o_dfz_cnt, o_dfz_dirty, ws_bytes;
};

struct Layout;
int router_n_exp(const Layout& L);

Layout make_layout(const moe_config& c) {
    Layout L{};
    L.H = c.hidden;
    L.I = c.inter;
    L.E = c.num_experts;
    L.k = c.top_k;
    L.G = c.num_experts + (c.has_shared ? 1 : 0);
    L.Tm = c.max_tokens;
    L.Tdec = c.decode_max_tokens < c.max_tokens ? (c.decode_max_tokens > 0 ? c.decode_max_tokens : 0)
                                                 : c.max_tokens;
    L.ks_dec = c.hidden / kRouterKSlice;
    L.nblk_max = (L.Tm + kTokPerBucketBlk - 1) / kTokPerBucketBlk;
    L.rows_cap = L.Tm * L.k + (c.has_shared ? L.Tm : 0);
    L.max_tiles = (L.rows_cap + 127) / 128 + L.G;   // tiles of >= 128 rows (gemm_tile_rows)
    const size_t per_mat_gu = (size_t)(L.I / 64) * (L.H / 64) * kBlockBytes;   // gate+up rows 2I
    const size_t per_mat_dn = (size_t)(L.H / 128) * (L.I / 64) * kBlockBytes;
    const bool experts = !(c.flags & MOE_FLAG_NO_EXPERTS);
    L.w_gu_bytes = experts ? per_mat_gu * L.G : 0;
    L.w_dn_bytes = experts ? per_mat_dn * L.G : 0;
    // router region: transposed fp32 [H][E], bias [E], shared-gate vector [H], public-layout fp32
    // copy [E][H]; every sub-buffer starts on a 256-byte boundary (vector loads need 16 B)
    L.o_wrt = 0;
    L.o_rbias = align_up(L.o_wrt + sizeof(float) * (size_t)L.H * L.E, 256);
    L.o_sgw = align_up(L.o_rbias + sizeof(float) * (size_t)L.E, 256);
    L.o_router32 = align_up(L.o_sgw + sizeof(float) * (size_t)L.H, 256);
    L.router_bytes = L.o_router32 + sizeof(float) * (size_t)L.H * L.E;
    L.Epad = (L.E + 127) / 128 * 128;
    L.wsplit_bytes = sizeof(uint16_t) * (size_t)L.Epad * 2 * L.H;
    L.weights_bytes = align_up(L.w_gu_bytes, 256) + align_up(L.w_dn_bytes, 256) + align_up(L.router_bytes, 256) +
                      align_up(L.wsplit_bytes, 256);

    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align_up(o + bytes, 256);
        return at;
    };
    size_t part_rows = (size_t)L.ks_dec * (size_t)L.Tdec;
    for (int T = 1; T <= L.Tm; ++T) part_rows = std::max(part_rows, (size_t)router_tc_splits(T, L.H) * T);
    L.o_part = take(sizeof(float) * part_rows * L.E);
    L.o_idx = take(sizeof(int) * (size_t)L.Tm * L.k);
    L.o_gates = take(sizeof(float) * (size_t)L.Tm * L.k);
    L.o_sg = take(sizeof(float) * (size_t)L.Tm);
    L.o_hist = take(sizeof(int) * (size_t)L.nblk_max * L.E);
    L.o_sdone = take(sizeof(unsigned));
    L.o_counts = take(sizeof(int) * (size_t)(L.G + 1));
    L.o_offsets = take(sizeof(int) * (size_t)(L.G + 2));
    L.o_tiles = take(sizeof(int4) * (size_t)L.max_tiles);
    L.o_ntiles = take(sizeof(int) * 4);
    L.o_perm = take(sizeof(int) * (size_t)L.Tm * L.k);
    L.o_rtok = take(sizeof(int) * (size_t)L.rows_cap);
    L.o_rgate = take(sizeof(float) * (size_t)L.rows_cap);
    L.o_x16 = take(sizeof(__half) * (size_t)L.Tm * L.H);
    L.o_xp = take(sizeof(__half) * (size_t)L.Tm * L.k * L.H);
    L.o_act = take(sizeof(__half) * (size_t)L.rows_cap * L.I);
    L.o_acc = take(sizeof(float) * (size_t)L.Tm * L.H);
    L.o_dact = take(sizeof(float) * (size_t)std::max(L.Tdec, 1) * (L.k + 1) * L.I);
    L.o_dscale = take(sizeof(float) * 2 * (size_t)std::max(L.Tdec, 1) * (L.k + 1) * (L.I / 64));
    L.o_status = take(sizeof(uint32_t) * 4);
    L.o_stage_x = take(sizeof(uint16_t) * (size_t)L.Tm * L.H);
    L.o_stage_out = take(sizeof(uint16_t) * (size_t)L.Tm * L.H);
    L.o_dfz_ticket = take(sizeof(unsigned long long));
    L.o_dfz_slots = take(sizeof(unsigned long long) * kDecodeFusedMaxT * (size_t)L.E);
    L.o_dfz_outacc = take(sizeof(float) * kDecodeFusedMaxT * (size_t)L.H);
    L.o_dfz_cnt = take(sizeof(unsigned) * kDecodeFusedMaxT * (size_t)(L.H / 128));
    L.o_dfz_dirty = take(sizeof(unsigned));
    L.ws_bytes = o;
    return L;
}

// experts as the router GEMM's N: E rounded up to a multiple of 16
int router_n_exp(const Layout& L) { return (L.E + 15) / 16 * 16; }

int validate_config(const moe_config* c) {
    if (!c) return fail(MOE_ERR_INVALID_ARG, "config is NULL");
    if (c->group != 64) return fail(MOE_ERR_INVALID_ARG, "group must be 64 (got %d)", c->group);
    if (c->hidden <= 0 || c->hidden % 128 != 0) return fail(MOE_ERR_INVALID_ARG, "hidden must be a positive multiple of 128");
    if (c->inter <= 0 || c->inter % 64 != 0) return fail(MOE_ERR_INVALID_ARG, "inter must be a positive multiple of 64");
    if (c->num_experts < 1 || c->num_experts > 256) return fail(MOE_ERR_INVALID_ARG, "num_experts must be in [1, 256]");
    if (c->top_k < 1 || c->top_k > c->num_experts || c->top_k > 32)
        return fail(MOE_ERR_INVALID_ARG, "top_k must be in [1, min(num_experts, 32)]");
    if (c->has_shared != 0 && c->has_shared != 1) return fail(MOE_ERR_INVALID_ARG, "has_shared must be 0 or 1");
    if (c->max_tokens < 1 || c->max_tokens > 65536) return fail(MOE_ERR_INVALID_ARG, "max_tokens must be in [1, 65536]");
    if (c->decode_max_tokens < 0 || c->decode_max_tokens > 65535)
        return fail(MOE_ERR_INVALID_ARG,
                    "decode_max_tokens must be in [0, 65535] (the GEMV path launches one grid slice per token)");
    if ((c->decode_max_tokens >= 2 || (c->flags & MOE_FLAG_DECODE_UNFUSED)) && c->top_k + c->has_shared > 16)
        return fail(MOE_ERR_INVALID_ARG, "the multi-kernel decode path supports top_k + has_shared <= 16");
    if (c->flags & ~(uint32_t)(MOE_FLAG_ROUTER_SIMT | MOE_FLAG_DECODE_UNFUSED | MOE_FLAG_POISON_WORKSPACE |
                               MOE_FLAG_HOST_SYNC_ROUTING | MOE_FLAG_DEQUANT_TO_HBM | MOE_FLAG_NO_ROUTER |
                               MOE_FLAG_NO_EXPERTS | MOE_FLAG_TEST_STALL))
        return fail(MOE_ERR_INVALID_ARG, "unknown flag bits 0x%x", c->flags);
    if ((c->flags & MOE_FLAG_NO_ROUTER) && (c->flags & MOE_FLAG_NO_EXPERTS))
        return fail(MOE_ERR_INVALID_ARG, "MOE_FLAG_NO_ROUTER and MOE_FLAG_NO_EXPERTS leave nothing to run");
    if ((c->flags & MOE_FLAG_NO_EXPERTS) && (c->flags & MOE_FLAG_DEQUANT_TO_HBM))
        return fail(MOE_ERR_INVALID_ARG, "MOE_FLAG_DEQUANT_TO_HBM needs expert weights");
    return MOE_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D 16-bit row-major [rows, cols] tensor, box {64 columns, box_rows rows}, 128-byte swizzle.
int encode_rows_map(CUtensorMap* m, const void* base, int rows, int cols, int box_rows,
                    CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT16) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return MOE_OK;
}

}  // namespace

void moe::set_last_error(const char* msg) { g_last_error = msg; }

constexpr int kProfCalls = 1024;
constexpr int kProfEvents = 9;  // at most 8 kernels per call + the leading event

struct moe_handle {
    int device = 0;
    // per-kernel profiling (moe_profile_enable)
    bool prof = false;
    cudaEvent_t* prof_ev = nullptr;        // [kProfCalls][kProfEvents]
    int prof_slot[kProfCalls][kProfEvents] = {};
    int prof_nev[kProfCalls] = {};
    int prof_calls = 0;
    moe_config cfg{};
    Layout L{};
    int num_sms = 0;
    uint8_t* wbuf = nullptr;
    uint8_t* ws = nullptr;
    Ctx base{};
    TokenMaps maps_gu{}, maps_dn{};
    CUtensorMap tm_wsplit{};
    uint16_t* wsplit = nullptr;
    cudaStream_t last_stream = nullptr;
    bool inexact_scales = false;
    // MOE_FLAG_DEQUANT_TO_HBM: the layer's weights dequantised once to fp16 rows in HBM, and
    // their tensor maps (box 64 columns x 128 rows), for the grouped-GEMM ablation variant
    __half* w16 = nullptr;
    CUtensorMap amap_gu{}, amap_dn{};
    // batch-1 decode: the fused kernel's geometry, when the shape and the device allow it
    bool fused_ok = false;
    DecodeGeom dgeom{};     // one token per launch
    DecodeGeom dgeom_m{};   // 1 .. kDecodeFusedMaxT tokens per launch
};

namespace {

Ctx make_ctx(const moe_handle* h, int T, const uint16_t* x, uint16_t* out, bool decode) {
    Ctx c = h->base;
    c.T = T;
    c.tile_rows = gemm_tile_rows(T, c.k, c.E);
    c.x = x;
    c.out = out;
    c.nblk = (T + kTokPerBucketBlk - 1) / kTokPerBucketBlk;
    c.ks = decode ? h->L.ks_dec : ((h->cfg.flags & MOE_FLAG_ROUTER_SIMT) ? 1 : router_tc_splits(T, h->L.H));
    return c;
}

int check_call(moe_handle* h, const void* x, int32_t T, const void* out, bool need_out) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T must be >= 0");
    if (T > h->cfg.max_tokens) return fail(MOE_ERR_TOO_LARGE, "T = %d exceeds max_tokens = %d", T, h->cfg.max_tokens);
    if (T > 0 && (!x || !aligned16(x))) return fail(MOE_ERR_INVALID_ARG, "x must be a 16-byte aligned device pointer");
    if (T > 0 && need_out && (!out || !aligned16(out)))
        return fail(MOE_ERR_INVALID_ARG, "out must be a 16-byte aligned device pointer");
    return MOE_OK;
}

bool use_decode(const moe_handle* h, int T) { return T <= h->cfg.decode_max_tokens; }

// Decode calls run the fused kernel, one launch per kDecodeFusedMaxT tokens (measured on one
// B200 at T = 16, per layer: 2 x 8 tokens 125 us, the grouped-GEMM path 143 us, the multi-kernel
// GEMV chain 155 us); the chain serves shapes the fused kernel does not fit.

// The fused kernel serves T <= kDecodeFusedMaxT when the shape fits its geometry and all of its
// clusters can be resident at once (decided at create); otherwise the multi-kernel GEMV chain does.
bool fused_decode_ok(const moe_handle* h) { return h->fused_ok && !(h->cfg.flags & MOE_FLAG_DECODE_UNFUSED); }

// Profiling: one event before the first kernel of a call and one after each kernel.
struct Prof {
    moe_handle* h;
    cudaStream_t st;
    int call = -1;
    Prof(moe_handle* hh, cudaStream_t s) : h(hh), st(s) {
        if (h->prof && h->prof_calls < kProfCalls) {
            call = h->prof_calls++;
            h->prof_nev[call] = 0;
            mark(-1);
        }
    }
    void mark(int slot) {
        if (call < 0) return;
        const int n = h->prof_nev[call];
        if (n >= kProfEvents) return;
        cudaEventRecord(h->prof_ev[call * kProfEvents + n], st);
        h->prof_slot[call][n] = slot;
        h->prof_nev[call] = n + 1;
    }
};

int enqueue_routing(moe_handle* h, Prof& pf, const Ctx& c, bool decode, cudaStream_t st) {
    if (decode || (h->cfg.flags & MOE_FLAG_ROUTER_SIMT)) {
        MOE_LAUNCH("moe.router_simt", launch_router_simt(c, st));
    } else {
        CUtensorMap tm_x;
        const int rc = encode_rows_map(&tm_x, c.x, c.T, c.H, 128, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
        if (rc != MOE_OK) return rc;
        MOE_LAUNCH("moe.router_tc", launch_router_tc(c, h->tm_wsplit, tm_x, router_n_exp(h->L), st));
    }
    pf.mark(0);
    MOE_LAUNCH("moe.topk", launch_topk(c, !decode, st));
    pf.mark(1);
    if (!decode) {
        MOE_LAUNCH("moe.scatter", launch_scatter(c, st));
        pf.mark(3);
    }
    return MOE_OK;
}

// The expert steps of a call after routing: the GEMV chain (decode) or the gather, the two grouped
// GEMMs and the finalisation (prefill).
int enqueue_experts(moe_handle* h, Prof& pf, const Ctx& c, bool decode, cudaStream_t st) {
    if (decode) {
        MOE_LAUNCH("moe.gemv_gateup", launch_gemv_gateup(c, st));
        pf.mark(7);
        MOE_LAUNCH("moe.gemv_down", launch_gemv_down(c, st));
        pf.mark(8);
    } else {
        MOE_LAUNCH("moe.gather_rows", launch_gather_rows(c, h->num_sms, st));
        pf.mark(10);
        int sms_gu = h->num_sms, sms_dn = h->num_sms;
        if (h->cfg.flags & MOE_FLAG_HOST_SYNC_ROUTING) {
            // ablation of GPU-resident routing: the host waits for the routing kernels, reads the
            // tile count back and sizes the grouped GEMMs' grids from it (same results)
            int nt = 0;
            {
                NvtxRange r("moe.host_sync_routing");
                CUDA_TRY(cudaMemcpyAsync(&nt, c.ntiles, sizeof(int), cudaMemcpyDeviceToHost, st));
                CUDA_TRY(cudaStreamSynchronize(st));
            }
            const int per_cta = c.tile_rows == 128 ? 2 : 1;   // CTAs per SM of the launch shape
            auto sms_for = [&](int tasks) { return std::max(1, std::min(h->num_sms, (tasks + per_cta - 1) / per_cta)); };
            sms_gu = sms_for(nt * (h->L.I / 64));
            sms_dn = sms_for(nt * (h->L.H / 128));
        }
        const bool a16 = h->w16 != nullptr;
        MOE_LAUNCH("moe.gemm_gateup", launch_gemm_gateup(c, h->maps_gu, a16 ? &h->amap_gu : nullptr, sms_gu, st));
        pf.mark(4);
        MOE_LAUNCH("moe.gemm_down", launch_gemm_down(c, h->maps_dn, a16 ? &h->amap_dn : nullptr, sms_dn, st));
        pf.mark(5);
        MOE_LAUNCH("moe.finalize", launch_finalize(c, st));
        pf.mark(6);
    }
    return MOE_OK;
}

}  // namespace

extern "C" {

int moe_version(void) { return 10000; }

const char* moe_last_error(void) { return g_last_error.c_str(); }

size_t moe_device_bytes(const moe_config* cfg) {
    if (validate_config(cfg) != MOE_OK) return 0;
    const Layout L = make_layout(*cfg);
    size_t extra = 0;
    if (cfg->flags & MOE_FLAG_DEQUANT_TO_HBM)
        extra = sizeof(__half) * ((size_t)L.G * 2 * L.I * L.H + (size_t)L.G * L.H * L.I);
    return L.weights_bytes + L.ws_bytes + extra;
}

int moe_create(const moe_config* cfg, const moe_weights* w, int device, void* stream, moe_handle** out) {
    g_last_error.clear();
    if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    int rc = validate_config(cfg);
    if (rc != MOE_OK) return rc;
    if (!w) return fail(MOE_ERR_INVALID_ARG, "weights is NULL");
    const bool experts = !(cfg->flags & MOE_FLAG_NO_EXPERTS), router = !(cfg->flags & MOE_FLAG_NO_ROUTER);
    if (experts) {
        const void* req[] = {w->q_gate, w->q_up, w->q_down, w->s_gate, w->b_gate, w->s_up, w->b_up, w->s_down, w->b_down};
        for (const void* p : req)
            if (!p || !aligned16(p)) return fail(MOE_ERR_INVALID_ARG, "a required weight pointer is NULL or misaligned");
        if (cfg->has_shared) {
            const void* sh[] = {w->qs_gate, w->qs_up, w->qs_down, w->ss_gate, w->bs_gate, w->ss_up, w->bs_up,
                                w->ss_down, w->bs_down};
            for (const void* p : sh)
                if (!p || !aligned16(p)) return fail(MOE_ERR_INVALID_ARG, "a shared-expert pointer is NULL or misaligned");
        }
    }
    if (router) {
        if (!w->router || !aligned16(w->router)) return fail(MOE_ERR_INVALID_ARG, "router is NULL or misaligned");
        if (cfg->has_shared && (!w->shared_gate || !aligned16(w->shared_gate)))
            return fail(MOE_ERR_INVALID_ARG, "shared_gate is NULL or misaligned");
        if (w->router_bias && !aligned16(w->router_bias)) return fail(MOE_ERR_INVALID_ARG, "router_bias misaligned");
    }

    int ndev = 0;
    CUDA_TRY(cudaGetDeviceCount(&ndev));
    if (device < 0 || device >= ndev) return fail(MOE_ERR_INVALID_ARG, "device %d out of range", device);
    cudaDeviceProp prop;
    CUDA_TRY(cudaGetDeviceProperties(&prop, device));
    if (prop.major != 10 || prop.minor != 0)
        return fail(MOE_ERR_UNSUPPORTED_DEVICE, "device %d is sm_%d%d; libmoe needs sm_100 (B200)", device, prop.major,
                    prop.minor);
    DeviceGuard guard(device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    moe_handle* h = new moe_handle();
    h->device = device;
    h->cfg = *cfg;
    h->L = make_layout(*cfg);
    h->num_sms = prop.multiProcessorCount;
    const Layout& L = h->L;
    auto cleanup = [&](int code) {
        if (h->w16) cudaFree(h->w16);
        if (h->wbuf) cudaFree(h->wbuf);
        if (h->ws) cudaFree(h->ws);
        delete h;
        return code;
    };
    cudaError_t e = cudaMalloc(&h->wbuf, L.weights_bytes);
    if (e != cudaSuccess) return cleanup(fail(MOE_ERR_CUDA, "cudaMalloc(weights %zu B): %s", L.weights_bytes, cudaGetErrorString(e)));
    e = cudaMalloc(&h->ws, L.ws_bytes);
    if (e != cudaSuccess) return cleanup(fail(MOE_ERR_CUDA, "cudaMalloc(workspace %zu B): %s", L.ws_bytes, cudaGetErrorString(e)));
    if (cfg->flags & MOE_FLAG_POISON_WORKSPACE) {
        // 0xFF bytes everywhere (NaN floats, -1 indices), then zero only the words the kernels
        // count on starting at zero: the bucketing histograms and the scatter's finish counter,
        // the status words and the fused
        // decode's call ticket and router words; its dirty word is raised, so the first decode
        // call resets its accumulator and counters on the device
        e = cudaMemsetAsync(h->ws, 0xFF, L.ws_bytes, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(h->ws + L.o_hist, 0, sizeof(int) * (size_t)L.nblk_max * L.E, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(h->ws + L.o_sdone, 0, sizeof(unsigned), st);
        if (e == cudaSuccess) e = cudaMemsetAsync(h->ws + L.o_status, 0, sizeof(uint32_t) * 4, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(h->ws + L.o_dfz_ticket, 0, sizeof(unsigned long long), st);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(h->ws + L.o_dfz_slots, 0, sizeof(unsigned long long) * kDecodeFusedMaxT * (size_t)L.E, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(h->ws + L.o_dfz_dirty, 0x01, sizeof(unsigned), st);
    } else {
        e = cudaMemsetAsync(h->ws, 0, L.ws_bytes, st);
    }
    if (e != cudaSuccess) return cleanup(fail(MOE_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e)));

    uint8_t* w_gu = h->wbuf;
    uint8_t* w_dn = w_gu + align_up(L.w_gu_bytes, 256);
    uint8_t* rregion = w_dn + align_up(L.w_dn_bytes, 256);
    float* wrt = reinterpret_cast<float*>(rregion + L.o_wrt);
    float* rbias = reinterpret_cast<float*>(rregion + L.o_rbias);
    float* sgw = reinterpret_cast<float*>(rregion + L.o_sgw);
    float* router32 = reinterpret_cast<float*>(rregion + L.o_router32);
    uint16_t* wsplit = reinterpret_cast<uint16_t*>(rregion + align_up(L.router_bytes, 256));
    h->wsplit = wsplit;
    uint32_t* status = reinterpret_cast<uint32_t*>(h->ws + L.o_status);

    RepackArgs a{};
    a.E = L.E;
    a.inexact = status + 1;
    a.gateup = 1;
    a.rows_per_mat = L.I;
    a.cols = L.H;
    a.q[0] = w->q_gate; a.s[0] = w->s_gate; a.b[0] = w->b_gate;
    a.q[1] = w->q_up;   a.s[1] = w->s_up;   a.b[1] = w->b_up;
    a.qs[0] = w->qs_gate; a.ss[0] = w->ss_gate; a.bs[0] = w->bs_gate;
    a.qs[1] = w->qs_up;   a.ss[1] = w->ss_up;   a.bs[1] = w->bs_up;
    a.dst = w_gu;
    e = experts ? launch_repack(a, L.G, L.I / 64, L.H / 64, st) : cudaSuccess;
    if (e != cudaSuccess) return cleanup(fail(MOE_ERR_CUDA, "repack gate/up: %s", cudaGetErrorString(e)));
    RepackArgs d{};
    d.E = L.E;
    d.inexact = status + 1;
    d.gateup = 0;
    d.rows_per_mat = L.H;
    d.cols = L.I;
    d.q[0] = w->q_down; d.s[0] = w->s_down; d.b[0] = w->b_down;
    d.q[1] = w->q_down; d.s[1] = w->s_down; d.b[1] = w->b_down;
    d.qs[0] = w->qs_down; d.ss[0] = w->ss_down; d.bs[0] = w->bs_down;
    d.qs[1] = w->qs_down; d.ss[1] = w->ss_down; d.bs[1] = w->bs_down;
    d.dst = w_dn;
    e = experts ? launch_repack(d, L.G, L.H / 128, L.I / 64, st) : cudaSuccess;
    if (e != cudaSuccess) return cleanup(fail(MOE_ERR_CUDA, "repack down: %s", cudaGetErrorString(e)));
    if (router) {
        e = launch_router_prep(w->router, w->router_bias, cfg->has_shared ? w->shared_gate : nullptr, L.H, L.E, wrt,
                               rbias, sgw, st);
        if (e != cudaSuccess) return cleanup(fail(MOE_ERR_CUDA, "router prep: %s", cudaGetErrorString(e)));
        e = cudaMemcpyAsync(router32, w->router, sizeof(float) * (size_t)L.E * L.H, cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return cleanup(fail(MOE_ERR_CUDA, "router copy: %s", cudaGetErrorString(e)));
        e = launch_router_split(w->router, L.H, L.E, L.Epad, wsplit, st);
        if (e != cudaSuccess) return cleanup(fail(MOE_ERR_CUDA, "router split: %s", cudaGetErrorString(e)));
    } else {
        e = cudaMemsetAsync(rregion, 0, align_up(L.router_bytes, 256) + L.wsplit_bytes, st);
        if (e != cudaSuccess) return cleanup(fail(MOE_ERR_CUDA, "router region: %s", cudaGetErrorString(e)));
    }
    uint32_t flags_host[2] = {0, 0};
    e = cudaMemcpyAsync(flags_host, status, sizeof flags_host, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cleanup(fail(MOE_ERR_CUDA, "create: %s", cudaGetErrorString(e)));
    h->inexact_scales = flags_host[1] != 0;
    e = cudaMemsetAsync(status, 0, 2 * sizeof(uint32_t), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cleanup(fail(MOE_ERR_CUDA, "create: %s", cudaGetErrorString(e)));

    Ctx& c = h->base;
    c.H = L.H; c.I = L.I; c.E = L.E; c.k = L.k; c.G = L.G; c.has_shared = cfg->has_shared;
    c.max_tiles = L.max_tiles;
    c.rows_cap = L.rows_cap;
    c.flags = cfg->flags;
    c.w_gu = w_gu; c.w_dn = w_dn; c.wrt = wrt; c.rbias = rbias; c.sgw = sgw; c.router32 = router32;
    uint8_t* ws = h->ws;
    c.part = reinterpret_cast<float*>(ws + L.o_part);
    c.idx = reinterpret_cast<int*>(ws + L.o_idx);
    c.gates = reinterpret_cast<float*>(ws + L.o_gates);
    c.sg = reinterpret_cast<float*>(ws + L.o_sg);
    c.hist = reinterpret_cast<int*>(ws + L.o_hist);
    c.scatter_done = reinterpret_cast<unsigned*>(ws + L.o_sdone);
    c.counts = reinterpret_cast<int*>(ws + L.o_counts);
    c.offsets = reinterpret_cast<int*>(ws + L.o_offsets);
    c.tiles1 = reinterpret_cast<int4*>(ws + L.o_tiles);
    c.tiles2 = c.tiles1;
    c.ntiles = reinterpret_cast<int*>(ws + L.o_ntiles);
    c.perm = reinterpret_cast<int*>(ws + L.o_perm);
    c.row_token = reinterpret_cast<int*>(ws + L.o_rtok);
    c.row_gate = reinterpret_cast<float*>(ws + L.o_rgate);
    c.x16 = reinterpret_cast<__half*>(ws + L.o_x16);
    c.xp = reinterpret_cast<__half*>(ws + L.o_xp);
    c.act = reinterpret_cast<__half*>(ws + L.o_act);
    c.acc = reinterpret_cast<float*>(ws + L.o_acc);
    c.dact = reinterpret_cast<float*>(ws + L.o_dact);
    c.dscale = reinterpret_cast<float*>(ws + L.o_dscale);
    c.status = status;
    c.dfz.ticket = reinterpret_cast<unsigned long long*>(ws + L.o_dfz_ticket);
    c.dfz.slots = reinterpret_cast<unsigned long long*>(ws + L.o_dfz_slots);
    c.dfz.outacc = reinterpret_cast<float*>(ws + L.o_dfz_outacc);
    c.dfz.cnt = reinterpret_cast<unsigned*>(ws + L.o_dfz_cnt);
    c.dfz.dirty = reinterpret_cast<unsigned*>(ws + L.o_dfz_dirty);

    if (experts && router && decode_fused_geometry(L.H, L.I, L.E, L.k, cfg->has_shared, 1, &h->dgeom) &&
        decode_fused_geometry(L.H, L.I, L.E, L.k, cfg->has_shared, kDecodeFusedMaxT, &h->dgeom_m)) {
        int n1 = 0, nm = 0;
        e = decode_fused_prepare(h->dgeom);
        if (e == cudaSuccess) e = decode_fused_prepare(h->dgeom_m);
        if (e == cudaSuccess) e = decode_fused_max_clusters(h->dgeom, &n1);
        if (e == cudaSuccess) e = decode_fused_max_clusters(h->dgeom_m, &nm);
        if (e != cudaSuccess) return cleanup(fail(MOE_ERR_CUDA, "decode kernel set-up: %s", cudaGetErrorString(e)));
        h->fused_ok = n1 >= h->dgeom.units && nm >= h->dgeom_m.units;
    }

    for (int hs = 0; hs < 3 && rc == MOE_OK; ++hs) {
        const int box = token_box_rows(hs);   // token tile box: 64, 128 or 256 rows
        rc = encode_rows_map(&h->maps_gu.m[0][hs], c.xp, L.Tm * L.k, L.H, box);
        if (rc == MOE_OK) rc = encode_rows_map(&h->maps_gu.m[1][hs], c.x16, L.Tm, L.H, box);
        if (rc == MOE_OK) rc = encode_rows_map(&h->maps_dn.m[0][hs], c.act, L.rows_cap, L.I, box);
        if (rc == MOE_OK) h->maps_dn.m[1][hs] = h->maps_dn.m[0][hs];
    }
    if (rc == MOE_OK)
        rc = encode_rows_map(&h->tm_wsplit, wsplit, L.Epad, 2 * L.H, router_n_exp(L), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
    if (rc != MOE_OK) return cleanup(rc);
    if (cfg->flags & MOE_FLAG_DEQUANT_TO_HBM) {
        const size_t rows_gu = (size_t)L.G * (L.I / 64) * 128, rows_dn = (size_t)L.G * (L.H / 128) * 128;
        e = cudaMalloc(&h->w16, sizeof(__half) * (rows_gu * L.H + rows_dn * L.I));
        if (e != cudaSuccess) return cleanup(fail(MOE_ERR_CUDA, "cudaMalloc(fp16 weights): %s", cudaGetErrorString(e)));
        __half* w16_dn = h->w16 + rows_gu * L.H;
        e = launch_dequant_rows(w_gu, L.G, L.I / 64, L.H / 64, h->w16, st);
        if (e == cudaSuccess) e = launch_dequant_rows(w_dn, L.G, L.H / 128, L.I / 64, w16_dn, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cleanup(fail(MOE_ERR_CUDA, "fp16 weights: %s", cudaGetErrorString(e)));
        rc = encode_rows_map(&h->amap_gu, h->w16, (int)rows_gu, L.H, 128);
        if (rc == MOE_OK) rc = encode_rows_map(&h->amap_dn, w16_dn, (int)rows_dn, L.I, 128);
        if (rc != MOE_OK) return cleanup(rc);
    }
    h->last_stream = st;
    *out = h;
    return MOE_OK;
}

int moe_forward(moe_handle* h, const uint16_t* x, int32_t T, uint16_t* out, void* stream) {
    int rc = check_call(h, x, T, out, true);
    if (rc != MOE_OK) return rc;
    if (h->cfg.flags & (MOE_FLAG_NO_ROUTER | MOE_FLAG_NO_EXPERTS))
        return fail(MOE_ERR_INVALID_ARG, "moe_forward needs a handle with router and experts (see MOE_FLAG_NO_*)");
    if (T == 0) return rc;
    NvtxRange range("moe_forward");
    DeviceGuard guard(h->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    h->last_stream = st;
    const bool decode = use_decode(h, T);
    const Ctx c = make_ctx(h, T, x, out, decode);
    Prof pf(h, st);
    if (decode && fused_decode_ok(h)) {
        // the fused kernel, one launch per kDecodeFusedMaxT tokens (each a programmatic dependent of
        // the last)
        for (int t0 = 0; t0 < T; t0 += kDecodeFusedMaxT) {
            Ctx ct = c;
            ct.T = std::min(kDecodeFusedMaxT, T - t0);
            ct.x = x + (size_t)t0 * h->L.H;
            ct.out = out + (size_t)t0 * h->L.H;
            ct.idx = c.idx + (size_t)t0 * h->L.k;
            ct.gates = c.gates + (size_t)t0 * h->L.k;
            ct.sg = c.sg + t0;
            MOE_LAUNCH("moe.decode_fused", launch_decode_fused(ct, ct.T == 1 ? h->dgeom : h->dgeom_m, st));
            pf.mark(9);
        }
        return MOE_OK;
    }
    rc = enqueue_routing(h, pf, c, decode, st);
    if (rc != MOE_OK) return rc;
    return enqueue_experts(h, pf, c, decode, st);
}

int moe_forward_host_async(moe_handle* h, const uint16_t* x_host, int32_t T, uint16_t* out_host, void* stream) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T must be >= 0");
    if (T > h->cfg.max_tokens) return fail(MOE_ERR_TOO_LARGE, "T = %d exceeds max_tokens = %d", T, h->cfg.max_tokens);
    if (h->cfg.flags & (MOE_FLAG_NO_ROUTER | MOE_FLAG_NO_EXPERTS))
        return fail(MOE_ERR_INVALID_ARG, "moe_forward needs a handle with router and experts (see MOE_FLAG_NO_*)");
    if (T == 0) return MOE_OK;
    if (!x_host || !out_host) return fail(MOE_ERR_INVALID_ARG, "host buffers must not be NULL");
    DeviceGuard guard(h->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint16_t* dx = reinterpret_cast<uint16_t*>(h->ws + h->L.o_stage_x);
    uint16_t* dout = reinterpret_cast<uint16_t*>(h->ws + h->L.o_stage_out);
    const size_t bytes = sizeof(uint16_t) * (size_t)T * h->L.H;
    CUDA_TRY(cudaMemcpyAsync(dx, x_host, bytes, cudaMemcpyHostToDevice, st));
    int rc = moe_forward(h, dx, T, dout, stream);
    if (rc != MOE_OK) return rc;
    CUDA_TRY(cudaMemcpyAsync(out_host, dout, bytes, cudaMemcpyDeviceToHost, st));
    return MOE_OK;
}

int moe_forward_routed(moe_handle* h, const uint16_t* x, int32_t T, const int32_t* idx, const float* gates,
                       const float* shared_gate, uint16_t* out, void* stream) {
    int rc = check_call(h, x, T, out, true);
    if (rc != MOE_OK) return rc;
    if (h->cfg.flags & MOE_FLAG_NO_EXPERTS)
        return fail(MOE_ERR_INVALID_ARG, "moe_forward_routed: handle created without expert weights");
    if (T == 0) return MOE_OK;
    if (!idx || !gates || !aligned16(idx) || !aligned16(gates))
        return fail(MOE_ERR_INVALID_ARG, "idx and gates must be 16-byte aligned device pointers");
    if (h->cfg.has_shared && (!shared_gate || !aligned16(shared_gate)))
        return fail(MOE_ERR_INVALID_ARG, "shared_gate must be a 16-byte aligned device pointer (has_shared = 1)");
    NvtxRange range("moe_forward_routed");
    DeviceGuard guard(h->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    h->last_stream = st;
    const bool decode = use_decode(h, T);
    const Ctx c = make_ctx(h, T, x, out, decode);
    Prof pf(h, st);
    MOE_LAUNCH("moe.routing_supplied", launch_routing_supplied(c, idx, gates, shared_gate, !decode, st));
    pf.mark(1);
    if (!decode) {
        MOE_LAUNCH("moe.scatter", launch_scatter(c, st));
        pf.mark(3);
    }
    return enqueue_experts(h, pf, c, decode, st);
}

int moe_combine_rows(moe_handle* h, const uint16_t* rows, int32_t n_rows, const int32_t* pos, int32_t T, int32_t k,
                     const uint16_t* base, uint16_t* out, void* stream) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
    if (T < 0 || n_rows < 0) return fail(MOE_ERR_INVALID_ARG, "T and n_rows must be >= 0");
    if (k < 1 || k > 32) return fail(MOE_ERR_INVALID_ARG, "k must be in [1, 32]");
    if (T == 0) return MOE_OK;
    if (!pos || !aligned16(pos) || !out || !aligned16(out) || (base && !aligned16(base)) ||
        (n_rows > 0 && (!rows || !aligned16(rows))))
        return fail(MOE_ERR_INVALID_ARG, "pointers must be 16-byte aligned device pointers");
    NvtxRange range("moe_combine_rows");
    DeviceGuard guard(h->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    h->last_stream = st;
    MOE_LAUNCH("moe.combine_rows", launch_combine_rows(rows, n_rows, pos, T, k, h->L.H, base, out, h->base.status,
                                                       h->num_sms, st));
    return MOE_OK;
}

int moe_forward_host(moe_handle* h, const uint16_t* x_host, int32_t T, uint16_t* out_host, void* stream) {
    const int rc = moe_forward_host_async(h, x_host, T, out_host, stream);
    if (rc != MOE_OK || T == 0) return rc;
    DeviceGuard guard(h->device);
    CUDA_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    return MOE_OK;
}

int moe_route(moe_handle* h, const uint16_t* x, int32_t T, int32_t* idx, float* gates, float* shared_gate,
              int32_t* offsets, int32_t* perm, void* stream) {
    int rc = check_call(h, x, T, nullptr, false);
    if (rc != MOE_OK) return rc;
    if (h->cfg.flags & MOE_FLAG_NO_ROUTER) return fail(MOE_ERR_INVALID_ARG, "moe_route: handle created without a router");
    if (T == 0) return rc;
    DeviceGuard guard(h->device);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    h->last_stream = st;
    const bool decode = use_decode(h, T);
    Ctx c = make_ctx(h, T, x, nullptr, decode);
    // the router the forward call would use for this T, then the prefill bucketing (so offsets
    // and perm exist for any T)
    Prof pf(h, st);
    pf.call = -1;
    rc = enqueue_routing(h, pf, c, decode, st);
    if (rc != MOE_OK) return rc;
    if (decode) {
        MOE_LAUNCH("moe.topk", launch_topk(c, true, st));
        MOE_LAUNCH("moe.scatter", launch_scatter(c, st));
    }
    const Layout& L = h->L;
    if (idx) CUDA_TRY(cudaMemcpyAsync(idx, c.idx, sizeof(int) * (size_t)T * L.k, cudaMemcpyDeviceToDevice, st));
    if (gates) CUDA_TRY(cudaMemcpyAsync(gates, c.gates, sizeof(float) * (size_t)T * L.k, cudaMemcpyDeviceToDevice, st));
    if (shared_gate) CUDA_TRY(cudaMemcpyAsync(shared_gate, c.sg, sizeof(float) * (size_t)T, cudaMemcpyDeviceToDevice, st));
    if (offsets) CUDA_TRY(cudaMemcpyAsync(offsets, c.offsets, sizeof(int) * (size_t)(L.E + 1), cudaMemcpyDeviceToDevice, st));
    if (perm) CUDA_TRY(cudaMemcpyAsync(perm, c.perm, sizeof(int) * (size_t)T * L.k, cudaMemcpyDeviceToDevice, st));
    return MOE_OK;
}

int moe_status(moe_handle* h) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
    DeviceGuard guard(h->device);
    CUDA_TRY(cudaStreamSynchronize(h->last_stream));
    uint32_t s = 0;
    CUDA_TRY(cudaMemcpy(&s, h->base.status, sizeof s, cudaMemcpyDeviceToHost));
    CUDA_TRY(cudaMemset(h->base.status, 0, sizeof s));
    // (a fused decode call that gave up part-way has raised the workspace's dirty word; the next
    // such call resets its state on the device, so nothing needs resetting here)
    if (s & MOE_STATUS_TIMEOUT) return fail(MOE_ERR_DEVICE_TIMEOUT, "a device-side wait timed out");
    if (s & MOE_STATUS_BOUNDS) return fail(MOE_ERR_DEVICE_BOUNDS, "a device-side index check failed");
    if (s & MOE_STATUS_RANGE) return fail(MOE_ERR_RANGE, "a value exceeded the fp16 operand range");
    return MOE_OK;
}

int moe_debug_copy(moe_handle* h, int which, void* dst, size_t bytes, void* stream) {
    if (!h || !dst) return fail(MOE_ERR_INVALID_ARG, "handle or dst is NULL");
    const Layout& L = h->L;
    const void* src = nullptr;
    size_t cap = 0;
    switch (which) {
        case 0: src = h->base.act; cap = sizeof(__half) * (size_t)L.rows_cap * L.I; break;
        case 1: src = h->base.x16; cap = sizeof(__half) * (size_t)L.Tm * L.H; break;
        case 2: src = h->base.part; cap = sizeof(float) * (size_t)L.Tm * L.E; break;
        case 3: src = h->base.acc; cap = sizeof(float) * (size_t)L.Tm * L.H; break;
        default: return fail(MOE_ERR_INVALID_ARG, "unknown buffer %d", which);
    }
    if (bytes > cap) return fail(MOE_ERR_INVALID_ARG, "%zu bytes exceed the buffer (%zu)", bytes, cap);
    DeviceGuard guard(h->device);
    CUDA_TRY(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)));
    return MOE_OK;
}

int moe_profile_enable(moe_handle* h, int enable) {
    if (!h) return fail(MOE_ERR_INVALID_ARG, "handle is NULL");
    DeviceGuard guard(h->device);
    if (enable && !h->prof_ev) {
        h->prof_ev = new cudaEvent_t[kProfCalls * kProfEvents]();
        for (int i = 0; i < kProfCalls * kProfEvents; ++i) CUDA_TRY(cudaEventCreate(&h->prof_ev[i]));
    }
    h->prof = enable != 0;
    h->prof_calls = 0;
    return MOE_OK;
}

int moe_profile_read(moe_handle* h, float* ms, int32_t* launches) {
    if (!h || !ms || !launches) return fail(MOE_ERR_INVALID_ARG, "NULL argument");
    for (int i = 0; i < MOE_PROF_SLOTS; ++i) {
        ms[i] = 0.f;
        launches[i] = 0;
    }
    if (!h->prof_ev) return MOE_OK;
    DeviceGuard guard(h->device);
    for (int cidx = 0; cidx < h->prof_calls; ++cidx) {
        for (int n = 1; n < h->prof_nev[cidx]; ++n) {
            cudaEvent_t a = h->prof_ev[cidx * kProfEvents + n - 1], b = h->prof_ev[cidx * kProfEvents + n];
            CUDA_TRY(cudaEventSynchronize(b));
            float t = 0.f;
            CUDA_TRY(cudaEventElapsedTime(&t, a, b));
            const int slot = h->prof_slot[cidx][n];
            if (slot >= 0 && slot < MOE_PROF_SLOTS) {
                ms[slot] += t;
                launches[slot] += 1;
            }
        }
    }
    h->prof_calls = 0;
    return MOE_OK;
}

void moe_destroy(moe_handle* h) {
    if (!h) return;
    {
        DeviceGuard guard(h->device);
        cudaDeviceSynchronize();
        if (h->prof_ev) {
            for (int i = 0; i < kProfCalls * kProfEvents; ++i) cudaEventDestroy(h->prof_ev[i]);
            delete[] h->prof_ev;
        }
        if (h->w16) cudaFree(h->w16);
        if (h->wbuf) cudaFree(h->wbuf);
        if (h->ws) cudaFree(h->ws);
    }
    delete h;
}

}  // extern "C"
