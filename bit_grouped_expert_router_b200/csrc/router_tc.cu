// router_tc.cu -- prefill router logits on the tensor core.
//
// logits[t][e] = sum_h x[t][h] * W[e][h] with W the fp32 router.  W is split once (at create) into
// two bf16 terms, Wh = bf16(W) and Wl = bf16(W - Wh), which together carry 16 significant bits of
// each weight (relative residual <= 2^-16); x is bf16 already, so every product x*Wh and x*Wl is
// exact in the fp32 accumulator and the GEMM over K = 2H of [Wh | Wl] against [x | x] reproduces
// the fp32 dot product to a few 1e-6 -- far inside the 1e-3 top-(k+1) logit gap the routing is
// checked with.  (The split-K SIMT router in route.cu stays in use for decode-sized T.)
//
// One CTA per 64 tokens computes all experts (two 128-row m-tiles for E = 256): TMA brings the
// 128x64 bf16 tiles of [Wh | Wl] and the 64x64 tile of x (128-byte swizzle) into a 4-stage ring,
// one thread issues tcgen05.mma (both operands in shared memory, fp32 accumulators in TMEM), and
// four epilogue warps write the raw logits [T][E] (fp32) for the top-k kernel.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kRN = 64;        // tokens per CTA (UMMA N)
constexpr int kRStages = 4;
constexpr int kRThreads = 192;  // warp 0 TMA, warp 1 MMA + TMEM, warps 2-5 epilogue
constexpr int kRAT = 128 * 128;  // bytes of one 128-row x 64-col bf16 A tile
constexpr int kRBT = kRN * 128;  // bytes of the B tile
constexpr int kRStageBytes = 2 * kRAT + kRBT;
constexpr int kROffBar = kRStages * kRStageBytes;
constexpr int kRSmem = kROffBar + (2 * kRStages + 2) * 8 + 16 + 1024;

__global__ void __launch_bounds__(kRThreads, 1)
    router_tc_kernel(Ctx c, int mtiles, const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kROffBar);
    uint64_t* empty = full + kRStages;
    uint64_t* accfull = empty + kRStages;
    uint64_t* drainbar = accfull + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drainbar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int t0 = blockIdx.x * kRN;
    const int nvalid = min(kRN, c.T - t0);
    const int KH = c.H / 64;     // k-steps per half (x tile repeats in the second half)
    const int KS = 2 * KH;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accfull, 1);
        mbar_init(drainbar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 2 * kRN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            uint32_t it = 0;
            for (int kc = 0; kc < KS; ++kc, ++it) {
                const int s = it % kRStages;
                const uint32_t ph = (it / kRStages) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, c.status)) break;
                uint8_t* st = smem + s * kRStageBytes;
                mbar_arrive_expect_tx(&full[s], mtiles * kRAT + kRBT);
                for (int mt = 0; mt < mtiles; ++mt) tma_load_2d(st + mt * kRAT, &tmA, kc * 64, mt * 128, &full[s]);
                tma_load_2d(st + 2 * kRAT, &tmB, (kc % KH) * 64, t0, &full[s]);
            }
            const uint32_t first = it > (uint32_t)kRStages ? it - kRStages : 0u;
            for (uint32_t i = first; i < it; ++i) mbar_drain(&full[i % kRStages], (i / kRStages) & 1u);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const int n_inst = max(16, ((nvalid + 15) / 16) * 16);
            const uint32_t idesc = idesc_f16(128, n_inst, true);
            bool ok = true, issued = false;
            uint32_t it = 0;
            for (int kc = 0; kc < KS; ++kc, ++it) {
                const int s = it % kRStages;
                const uint32_t ph = (it / kRStages) & 1u;
                if (!mbar_wait(&full[s], ph, abort_flag, c.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t st = smem_u32(smem + s * kRStageBytes);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t bdesc = sdesc_sw128(st + 2 * kRAT + 32 * kk);
                    for (int mt = 0; mt < mtiles; ++mt)
                        mma_ss(tmem + mt * kRN, sdesc_sw128(st + mt * kRAT + 32 * kk), bdesc, idesc,
                               (kc | kk) != 0 ? 1u : 0u);
                }
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
        if (mbar_wait(accfull, 0, abort_flag, c.status)) {
            tc_fence_after();
            for (int mt = 0; mt < mtiles; ++mt) {
                const int e = mt * 128 + 32 * q + lane;
                for (int c0 = 0; c0 < nvalid; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + mt * kRN + c0, v);
                    if (e < c.E) {
#pragma unroll
                        for (int r = 0; r < 32; ++r) {
                            const int j = c0 + r;
                            if (j < nvalid) c.part[(size_t)(t0 + j) * c.E + e] = __uint_as_float(v[r]);
                        }
                    }
                }
            }
        }
    }
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 2 * kRN);
    }
}

// Wsplit[e][h] = bf16(W[e][h]), Wsplit[e][H + h] = bf16(W[e][h] - that); rows e >= E are zero.
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

cudaError_t launch_router_split(const float* router, int H, int E, int Epad, uint16_t* wsplit, cudaStream_t st) {
    router_split_kernel<<<256, 256, 0, st>>>(router, H, E, Epad, wsplit);
    return cudaGetLastError();
}

cudaError_t launch_router_tc(const Ctx& c, const CUtensorMap& tmA, const CUtensorMap& tmB, int mtiles,
                             cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRSmem);
    if (e != cudaSuccess) return e;
    const int blocks = (c.T + kRN - 1) / kRN;
    router_tc_kernel<<<blocks, kRThreads, kRSmem, st>>>(c, mtiles, tmA, tmB);
    return cudaGetLastError();
}

}  // namespace moe
