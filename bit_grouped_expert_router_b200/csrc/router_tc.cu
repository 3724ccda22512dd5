// router_tc.cu -- prefill router logits on the tensor core.
//
// logits[t][e] = sum_h x[t][h] * W[e][h] with W the fp32 router.  W is split once (at create) into
// two bf16 terms, W1 = bf16(W) and W2 = bf16(W - W1), which carry 16 significant bits of every
// weight (relative residual <= 2^-17); x is bf16 already, so every product x*Wi is exact.  The
// tensor core's fp32 accumulation does not round to nearest on every add, so long accumulation
// chains drift: the K = 2H products of one logit are split into 4 or more separate partial sums
// (each its own short chain on the tensor core) that the top-k kernel adds in fp32, in split order.
// Short calls take more splits (up to 16), so that their few token tiles still spread over the
// SMs: 512 tokens are 4 tiles, 16 CTAs with four splits.  Measured
// against the fp64 oracle the logits agree to a few 1e-6 -- far inside the 1e-3 top-(k+1) gap
// the routing is checked with.  (The split-K SIMT router in route.cu serves decode-sized T.)
//
// CTA (token tile of 128, K quarter): TMA brings the 128x64 bf16 tile of x (A, M = 128 tokens) and
// the Epad16x64 tile of [W1 | W2] (B, N = all experts, <= 256) into a 4-stage ring with the
// 128-byte swizzle; one thread issues tcgen05.mma (both operands in shared memory, fp32
// accumulator in TMEM, lane = token, column = expert); four epilogue warps write the partial
// logits part[quarter][t][e] with 16-byte stores (a thread owns one token's row).
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kRM = 128;        // tokens per CTA (UMMA M)
constexpr int kRSplit = 4;      // K splits (partial sums) of calls with enough token tiles
constexpr int kRStages = 4;
constexpr int kRThreads = 192;  // warp 0 TMA, warp 1 MMA + TMEM, warps 2-5 epilogue
constexpr int kRAT = kRM * 128;  // bytes of the x tile
constexpr int kRBTMax = 256 * 128;
constexpr int kRStageBytes = kRAT + kRBTMax;
constexpr int kROffBar = kRStages * kRStageBytes;
constexpr int kRSmem = kROffBar + (2 * kRStages + 2) * 8 + 16 + 1024;

__global__ void __launch_bounds__(kRThreads, 1)
    router_tc_kernel(Ctx c, int n_exp, const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX) {
    griddep_wait();
    griddep_launch_dependents();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kROffBar);
    uint64_t* empty = full + kRStages;
    uint64_t* accfull = empty + kRStages;
    uint64_t* drainbar = accfull + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drainbar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int t0 = blockIdx.x * kRM;
    const int split = blockIdx.y, nsplit = gridDim.y;
    const int KH = c.H / 64;                 // k-steps per term (the x tile repeats for each term)
    const int KS = 2 * KH;
    const int k_begin = split * KS / nsplit, k_end = (split + 1) * KS / nsplit;
    const int tmem_cols = n_exp <= 32 ? 32 : (n_exp <= 64 ? 64 : (n_exp <= 128 ? 128 : 256));
    const uint32_t b_bytes = (uint32_t)n_exp * 128;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accfull, 1);
        mbar_init(drainbar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmW);
        prefetch_tmap(&tmX);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            uint32_t it = 0;
            for (int kc = k_begin; kc < k_end; ++kc, ++it) {
                const int s = it % kRStages;
                const uint32_t ph = (it / kRStages) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, c.status)) break;
                uint8_t* st = smem + s * kRStageBytes;
                mbar_arrive_expect_tx(&full[s], kRAT + b_bytes);
                tma_load_2d(st, &tmX, (kc % KH) * 64, t0, &full[s]);
                tma_load_2d(st + kRAT, &tmW, kc * 64, 0, &full[s]);
            }
            const uint32_t first = it > (uint32_t)kRStages ? it - kRStages : 0u;
            for (uint32_t i = first; i < it; ++i) mbar_drain(&full[i % kRStages], (i / kRStages) & 1u);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_f16(kRM, n_exp, true);
            bool ok = true, issued = false;
            uint32_t it = 0;
            for (int kc = k_begin; kc < k_end; ++kc, ++it) {
                const int s = it % kRStages;
                const uint32_t ph = (it / kRStages) & 1u;
                if (!mbar_wait(&full[s], ph, abort_flag, c.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t st = smem_u32(smem + s * kRStageBytes);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tmem, sdesc_sw128(st + 32 * kk), sdesc_sw128(st + kRAT + 32 * kk), idesc,
                           (kc != k_begin || kk) ? 1u : 0u);
                issued = true;
                tc_commit(&empty[s]);
            }
            if (ok) tc_commit(accfull);
            else if (issued) {
                tc_commit(drainbar);
                mbar_drain(drainbar, 0);
            }
        }
    } else {
        const int q = warp & 3;
        const int t = t0 + 32 * q + lane;
        if (mbar_wait(accfull, 0, abort_flag, c.status)) {
            tc_fence_after();
            float* dst = c.part + ((size_t)split * c.T + t) * c.E;
            for (int c0 = 0; c0 < n_exp; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + c0, v);
                if (k_end <= k_begin) {   // a split without k-steps (never chosen): its sum is 0
#pragma unroll
                    for (int r = 0; r < 32; ++r) v[r] = 0u;
                }
                if (t < c.T) {
                    if (c0 + 32 <= c.E && (c.E & 3) == 0) {
#pragma unroll
                        for (int r = 0; r < 32; r += 4)
                            *reinterpret_cast<float4*>(dst + c0 + r) =
                                make_float4(__uint_as_float(v[r]), __uint_as_float(v[r + 1]),
                                            __uint_as_float(v[r + 2]), __uint_as_float(v[r + 3]));
                    } else {
#pragma unroll
                        for (int r = 0; r < 32; ++r)
                            if (c0 + r < c.E) dst[c0 + r] = __uint_as_float(v[r]);
                    }
                }
            }
        }
    }
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, tmem_cols);
    }
}

// Wsplit[e][t*H + h] = term t of W[e][h] (t = 0, 1; the second is the bf16 rounding of what the
// first left); rows e >= E are zero.
__global__ void router_split_kernel(const float* __restrict__ router, int H, int E, int Epad,
                                    uint16_t* __restrict__ wsplit) {
    const size_t n = (size_t)Epad * H;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const size_t e = i / H, h = i % H;
        const float w = e < (size_t)E ? router[e * H + h] : 0.f;
        const __nv_bfloat16 hi = __float2bfloat16_rn(w);
        const __nv_bfloat16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
        wsplit[e * 2 * H + h] = __bfloat16_as_ushort(hi);
        wsplit[e * 2 * H + H + h] = __bfloat16_as_ushort(lo);
    }
}

}  // namespace

int router_tc_smem_bytes() { return kRSmem; }
int router_tc_splits(int T, int H) {
    const int tiles = (T + kRM - 1) / kRM;
    int s = kRSplit;
    // at least two k-steps per split (2H / 64 k-steps in all); 148: the SMs of a B200
    while (s < 16 && tiles * 2 * s <= 148 && 2 * s * 2 <= 2 * H / 64) s *= 2;
    return s;
}

cudaError_t launch_router_split(const float* router, int H, int E, int Epad, uint16_t* wsplit, cudaStream_t st) {
    router_split_kernel<<<256, 256, 0, st>>>(router, H, E, Epad, wsplit);
    return cudaGetLastError();
}

// tmW: [W1 | W2] bf16 [Epad][2H], box {64, n_exp}; tmX: x bf16 [T][H], box {64, 128}.
cudaError_t launch_router_tc(const Ctx& c, const CUtensorMap& tmW, const CUtensorMap& tmX, int n_exp,
                             cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRSmem);
    if (e != cudaSuccess) return e;
    dim3 grid((c.T + kRM - 1) / kRM, c.ks);
    return launch_pdl(router_tc_kernel, grid, dim3(kRThreads), kRSmem, st, c, n_exp, tmW, tmX);
}

}  // namespace moe
