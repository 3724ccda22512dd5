// route_static.cu -- routing (router logits, top-k, renormalised gates) that allocates nothing.
//
// Who needs this: code that must not call cudaMalloc -- a thread that is recording a CUDA graph
// (allocation is not a stream operation and breaks capture), a latency-critical serving loop that
// is not allowed to enter the allocator, or a plug-in living inside a host framework that owns
// every device allocation.  Such callers cannot create a moe_handle (moe_create allocates the
// repacked weights and the workspace), yet they may still want the router's decision for a few
// tokens.  moe_route_static takes the router in its public layout straight from the caller and
// keeps its only scratch buffer -- the split-K partial logits -- in a fixed-size array that lives
// in the library's own device image (a file-scope __device__ array), so the call itself allocates
// nothing.  Every GPU that loads the library holds that array (1 MiB) until the process exits.
//
// The scratch array is shared by every call on a device and keeps the last call's contents.  Each
// call writes every partial it later reads, so nothing needs clearing; but two calls that overlap
// on the GPU (different streams, or different host threads without ordering) race on the array and
// may return wrong results: serialise them.
//
// Set-up: the device address of the array is looked up (cudaGetSymbolAddress) the first time the
// entry point runs in a CUDA context, with that context current.  That first call therefore makes
// a runtime query that is not a stream operation; make it before starting any stream capture.
// The address is cached per context (keyed on the driver's unique context id, not on the device
// ordinal): after cudaDeviceReset, or after the primary context is released and created again,
// the module is loaded anew and the array may sit at another address, so the first call in the
// new context looks it up again -- that call, too, belongs outside any capture.
#include <cudaTypedefs.h>

#include <mutex>
#include <unordered_map>

#include "../../include/moe.h"
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kKSlice = 32;                            // input columns per partial
constexpr int kStaticTT = 8;                           // tokens per CTA
static __device__ __align__(256) float g_route_scratch[MOE_ROUTE_STATIC_SCRATCH_FLOATS];

// part[s][t][e] = sum_{h in slice s} x[t][h] * router[e][h]   (router in the public [E][H] layout)
__global__ void __launch_bounds__(256) route_static_logits(const uint16_t* __restrict__ x, int T, int H,
                                                           const float* __restrict__ router, int E,
                                                           float* __restrict__ part) {
    const int s = blockIdx.x, t0 = blockIdx.y * kStaticTT, e = threadIdx.x;
    __shared__ float xs[kStaticTT][kKSlice];
    for (int i = threadIdx.x; i < kStaticTT * kKSlice; i += blockDim.x) {
        const int tt = i / kKSlice, hh = i % kKSlice, t = t0 + tt;
        xs[tt][hh] = t < T ? __uint_as_float((uint32_t)x[(size_t)t * H + s * kKSlice + hh] << 16) : 0.f;
    }
    __syncthreads();
    if (e >= E) return;
    float acc[kStaticTT];
#pragma unroll
    for (int tt = 0; tt < kStaticTT; ++tt) acc[tt] = 0.f;
    const float* w = router + (size_t)e * H + (size_t)s * kKSlice;
#pragma unroll 8
    for (int hh = 0; hh < kKSlice; ++hh) {
        const float wv = __ldg(w + hh);
#pragma unroll
        for (int tt = 0; tt < kStaticTT; ++tt) acc[tt] = fmaf(xs[tt][hh], wv, acc[tt]);
    }
#pragma unroll
    for (int tt = 0; tt < kStaticTT; ++tt)
        if (t0 + tt < T) part[((size_t)s * T + t0 + tt) * E + e] = acc[tt];
}

// One warp per token: sum the partials in slice order, add the bias, pick the top k (ties to the
// lower index, NaN as -inf), softmax over the selection.
__global__ void __launch_bounds__(256) route_static_topk(const float* __restrict__ part, int T, int E, int ks,
                                                         int k, const float* __restrict__ bias,
                                                         int32_t* __restrict__ idx, float* __restrict__ gates) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    float l[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        float v = -INFINITY;
        if (e < E) {
            float sum = 0.f;
            for (int q = 0; q < ks; ++q) sum += part[((size_t)q * T + t) * E + e];
            sum += bias ? bias[e] : 0.f;
            v = (sum != sum) ? -INFINITY : sum;
        }
        l[i] = v;
    }
    unsigned taken = 0;
    int my_e = 0;
    float my_v = 0.f;
    for (int j = 0; j < k; ++j) {
        float bv = 0.f;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((taken >> i) & 1u) && (be == 0x7fffffff || l[i] > bv)) { bv = l[i]; be = e; }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (oe != 0x7fffffff && (be == 0x7fffffff || ov > bv || (ov == bv && oe < be))) { bv = ov; be = oe; }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == j) { my_e = be; my_v = bv; }
    }
    const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
    const float p = lane < k ? expf(my_v - vmax) : 0.f;
    float z = p;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    if (lane < k) {
        idx[(size_t)t * k + lane] = my_e;
        gates[(size_t)t * k + lane] = p / z;
    }
}

std::mutex g_static_mu;
std::unordered_map<unsigned long long, void*> g_static_ptr;   // context id -> array address

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current CUDA context (0 if none is current yet).
bool current_context_id(unsigned long long* id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS) return false;
    *id = 0;
    return ctx == nullptr || get_id(ctx, id) == CUDA_SUCCESS;
}

int static_fail(int code, const char* msg) {
    set_last_error(msg);  // reported by moe_last_error() on this thread
    return code;
}

}  // namespace
}  // namespace moe

extern "C" int moe_route_static(const uint16_t* x, int32_t T, int32_t H, const float* router,
                                const float* router_bias, int32_t E, int32_t k, int32_t* idx, float* gates,
                                void* stream) {
    using namespace moe;
    if (T < 0 || H <= 0 || H % kKSlice != 0 || E < 1 || E > 256 || k < 1 || k > E || k > 32)
        return static_fail(MOE_ERR_INVALID_ARG, "moe_route_static: need T >= 0, H % 32 == 0, 1 <= k <= min(E, 32), E <= 256");
    if (T == 0) return MOE_OK;
    if (!x || !router || !idx || !gates) return static_fail(MOE_ERR_INVALID_ARG, "moe_route_static: NULL pointer");
    const int ks = H / kKSlice;
    if ((long long)T * ks * E > (long long)MOE_ROUTE_STATIC_SCRATCH_FLOATS)
        return static_fail(MOE_ERR_TOO_LARGE,
                           "moe_route_static: T * (H/32) * E exceeds the static scratch (MOE_ROUTE_STATIC_SCRATCH_FLOATS)");
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return static_fail(MOE_ERR_CUDA, "moe_route_static: no current CUDA device");
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_static_mu);
        unsigned long long ctx = 0;
        if (!current_context_id(&ctx)) return static_fail(MOE_ERR_CUDA, "moe_route_static: cannot identify the CUDA context");
        auto it = ctx ? g_static_ptr.find(ctx) : g_static_ptr.end();
        if (it != g_static_ptr.end()) {
            scratch = it->second;
        } else {
            // first call in this context (cudaGetSymbolAddress also makes the device's primary
            // context current when none is): look the array up, then key it on the context id
            void* p = nullptr;
            const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
            if (e != cudaSuccess || !p) return static_fail(MOE_ERR_CUDA, "moe_route_static: cudaGetSymbolAddress failed");
            if (!current_context_id(&ctx) || ctx == 0)
                return static_fail(MOE_ERR_CUDA, "moe_route_static: no CUDA context after set-up");
            g_static_ptr[ctx] = p;
            scratch = p;
        }
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    float* part = static_cast<float*>(scratch);
    dim3 g1(ks, (T + kStaticTT - 1) / kStaticTT);
    route_static_logits<<<g1, 256, 0, st>>>(x, T, H, router, E, part);
    route_static_topk<<<(T + 7) / 8, 256, 0, st>>>(part, T, E, ks, k, router_bias, idx, gates);
    if (cudaGetLastError() != cudaSuccess) return static_fail(MOE_ERR_CUDA, "moe_route_static: launch failed");
    return MOE_OK;
}
