// decode_fused.cu -- batch-1 decode of one MoE layer in a single cooperative kernel.
//
// A decode token moves ~18 MB (router 2 MiB + 9 experts x 1.69 MiB), about 2.8 us of HBM time, so
// launch gaps and the first-byte latency of each dependent step dominate a multi-kernel chain.
// Following the pages' decode levers -- fuse the kernel chain and run independent work
// concurrently ("A Rust + Metal Inference Engine..." body; "Perplexity Open-Sources Lily..."
// section "Generation has a different bottleneck") -- one persistent grid (one 512-thread CTA
// per SM, co-resident by cooperative launch) runs three phases separated by two grid barriers:
//
//   phase 0  router logits (E x 4 quarter-row dot products, fp32) and, concurrently, the shared
//            expert's gate/up GEMV (it needs no routing); every CTA also stages the token.
//   phase 1  every CTA reduces the logits and picks the top k (identical result everywhere), then
//            the k routed experts' gate/up GEMVs.
//   phase 2  down GEMVs: a CTA owns one expert slot, builds act = silu(G) * U for it, streams the
//            down blocks, and adds gate * y into an fp32 row accumulator; the last task to finish
//            a 32-row chunk (atomic counter) rounds it to bf16, writes the output and re-zeroes the
//            accumulator and counter for the next call (self-cleaning, no memset launch).
//
// Each phase is a flat list of warp tasks (one weight-block slice each); task t runs on CTA
// t % grid, so every SM carries a share and all of a phase's weight loads are in flight at once.
// The down blocks of phase 2 are requested into L2 early (bulk L2 prefetch: the shared expert's
// at kernel start, the routed experts' right after top-k), and each phase-2 warp issues its
// weight loads before it builds act, so phase 2 mostly waits on L2, not HBM.  GEMV arithmetic as
// in decode.cu.
// Grid barrier: ever-growing arrival counters in the workspace; waits are bounded (1 s), on a
// timeout the status word records it and moe_status resets the barrier state.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kFThreads = 512;
constexpr int kFWarps = kFThreads / 32;
constexpr int kGuKR = 4;   // k-ranges of the gate/up GEMV tasks
constexpr int kDnKR = 4;   // k-ranges of the down GEMV tasks

__device__ __forceinline__ float pow2f(int n) { return __int_as_float((127 + n) << 23); }
__device__ __forceinline__ int group_exponent(float m) {
    int e = (int)((__float_as_uint(m) >> 23) & 0xFFu) - 127;
    return max(-126, min(100, e));
}
__device__ __forceinline__ int slot_of(int e8) { return (e8 >> 2) | ((e8 & 3) << 1); }

__device__ __forceinline__ float dot_group(const uint4& c0, const uint4& c1, const float* vp) {
    const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t m0 = w[i] & 0x0F0F0F0Fu;
        const uint32_t m1 = (w[i] >> 4) & 0x0F0F0F0Fu;
        const float4 x0 = *reinterpret_cast<const float4*>(vp + 8 * i);
        const float4 x1 = *reinterpret_cast<const float4*>(vp + 8 * i + 4);
        a0 = fma_keep_subnormal(__uint_as_float(__byte_perm(m0, 0u, 0x4440)), x0.x, a0);
        a1 = fma_keep_subnormal(__uint_as_float(__byte_perm(m0, 0u, 0x4441)), x0.y, a1);
        a0 = fma_keep_subnormal(__uint_as_float(__byte_perm(m0, 0u, 0x4442)), x0.z, a0);
        a1 = fma_keep_subnormal(__uint_as_float(__byte_perm(m0, 0u, 0x4443)), x0.w, a1);
        a0 = fma_keep_subnormal(__uint_as_float(__byte_perm(m1, 0u, 0x4440)), x1.x, a0);
        a1 = fma_keep_subnormal(__uint_as_float(__byte_perm(m1, 0u, 0x4441)), x1.y, a1);
        a0 = fma_keep_subnormal(__uint_as_float(__byte_perm(m1, 0u, 0x4442)), x1.z, a0);
        a1 = fma_keep_subnormal(__uint_as_float(__byte_perm(m1, 0u, 0x4443)), x1.w, a1);
    }
    return a0 + a1;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Grid barrier on kBarCounters counters that only grow, 256 bytes apart: CTA b adds 1 (release,
// GPU scope) to counter b mod kBarCounters, so few same-address atomics queue behind each other;
// the barrier index follows from the value it found, and warp 0 then polls every counter (acquire)
// until each has received one arrival per CTA mapped to it for this barrier.  No reset: between
// barriers every counter holds a multiple of its CTA count (the handle zeroes them after a
// timeout).  Bounded.
constexpr int kBarCounters = 16;
constexpr int kBarStride = 32;   // u64 words between counters

__device__ bool grid_barrier(unsigned long long* ctr, unsigned nblocks, uint32_t* status, volatile int* abort_flag) {
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const unsigned nc = nblocks < (unsigned)kBarCounters ? nblocks : (unsigned)kBarCounters;
        auto members = [&](unsigned j) { return nblocks / nc + (j < nblocks % nc ? 1u : 0u); };
        unsigned long long b = 0;
        if (lane == 0) {
            const unsigned j = blockIdx.x % nc;
            unsigned long long old;
            asm volatile("atom.add.release.gpu.u64 %0, [%1], 1;" : "=l"(old) : "l"(ctr + (size_t)j * kBarStride) : "memory");
            b = old / members(j);
        }
        b = __shfl_sync(0xffffffffu, b, 0);
        bool ok = true;
        if ((unsigned)lane < nc) {
            const unsigned long long target = (b + 1) * members((unsigned)lane);
            const unsigned long long* p = ctr + (size_t)lane * kBarStride;
            const unsigned long long t0 = globaltimer_ns();
            while (true) {
                unsigned long long v;
                asm volatile("ld.acquire.gpu.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
                if (v >= target) break;
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    set_status(status, MOE_STATUS_TIMEOUT);
                    ok = false;
                    break;
                }
            }
        }
        ok = __all_sync(0xffffffffu, ok);
        if (lane == 0) *abort_flag = ok ? 0 : 1;
    }
    __syncthreads();
    return *abort_flag == 0;
}

// Order-preserving map of a float to an unsigned key (-0 first made +0, so equal floats give
// equal keys).
__device__ __forceinline__ uint32_t ord_key(float v) {
    const uint32_t u = __float_as_uint(v + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct GemvTask {  // one warp: 32 rows (lane = row) of one m-tile, k-steps [k0, k1)
    const uint8_t* blocks;  // first block of the m-tile
    int row;                // block row of this lane
    int k0, k1;
};

// A task's codes and scale/bias words, loaded ahead of the arithmetic (up to 8 k-steps).
struct GemvRegs {
    uint4 a[8], b[8];
    uint32_t sb[8];
};

__device__ __forceinline__ void gemv_load(const GemvTask& t, GemvRegs& r) {
    const int n = t.k1 - t.k0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (i < n) {
            const uint8_t* blk = t.blocks + (size_t)(t.k0 + i) * kBlockBytes;
            r.a[i] = __ldg(reinterpret_cast<const uint4*>(blk + t.row * 16));
            r.b[i] = __ldg(reinterpret_cast<const uint4*>(blk + 2048 + t.row * 16));
            r.sb[i] = __ldg(reinterpret_cast<const uint32_t*>(blk + kBlockCodeBytes + t.row * 4));
        }
    }
}

__device__ __forceinline__ float gemv_dot(const GemvTask& t, const GemvRegs& r, const float* vperm,
                                          const float* vsum, const float* vsc) {
    const int n = t.k1 - t.k0;
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (i < n) {
            const int cc = t.k0 + i;
            const float s = __half2float(__ushort_as_half((unsigned short)(r.sb[i] & 0xFFFFu)));
            const float bb = __half2float(__ushort_as_half((unsigned short)(r.sb[i] >> 16)));
            const float P = dot_group(r.a[i], r.b[i], vperm + 64 * cc);
            acc += s * (P * vsc[cc]) + bb * vsum[cc];
        }
    }
    return acc;
}

__device__ __forceinline__ float run_gemv(const GemvTask& t, const float* vperm, const float* vsum, const float* vsc) {
    GemvRegs r;
    gemv_load(t, r);   // every load of the task in flight before the arithmetic
    return gemv_dot(t, r, vperm, vsum, vsc);
}

// One thread asks L2 to fetch the down blocks of (expert list entry, m-tile) chunks
// blockIdx.x, blockIdx.x + gridDim.x, ...: one m-tile's whole k range is one contiguous run.
// experts == nullptr stands for the shared expert (group E).  Not thread 0: its grid-barrier
// release would wait for the prefetches to finish.
__device__ __forceinline__ void prefetch_down(const Ctx& c, const int* experts, int nexp) {
    if (threadIdx.x != 32) return;
    const int MTd = c.H / 128, KSd = c.I / 64;
    for (int ch = blockIdx.x; ch < nexp * MTd; ch += gridDim.x) {
        const int e = experts ? experts[ch / MTd] : c.E, mt = ch % MTd;
        prefetch_l2(c.w_dn + ((size_t)e * MTd + mt) * KSd * kBlockBytes, (uint32_t)(KSd * kBlockBytes));
    }
}

// Per-64-element group power-of-two scaling (see decode.cu): vperm in slot order, group sums, 2^(149-K).
// One warp per group, 2 elements per lane; `src(i)` yields element i.
template <typename F>
__device__ __forceinline__ void stage_groups(int n, F src, float* vperm, float* vsum, float* vsc) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int grp = warp; grp < n / 64; grp += kFWarps) {
        const float a0 = src(64 * grp + 2 * lane), a1 = src(64 * grp + 2 * lane + 1);
        const float m = warp_max(fmaxf(fabsf(a0), fabsf(a1)));
        const float s = warp_sum(a0 + a1);
        const int K = 125 - group_exponent(m);
        const float f1 = pow2f(K / 2), f2 = pow2f(K - K / 2);
        const int e0 = 2 * lane, e1 = 2 * lane + 1;
        vperm[64 * grp + (e0 & ~7) + slot_of(e0 & 7)] = a0 * f1 * f2;
        vperm[64 * grp + (e1 & ~7) + slot_of(e1 & 7)] = a1 * f1 * f2;
        if (lane == 0) {
            vsum[grp] = s;
            vsc[grp] = pow2f(149 - K);
        }
    }
}

__global__ void __launch_bounds__(kFThreads, 1) decode_fused_kernel(Ctx c) {
    extern __shared__ __align__(16) float sm[];
    const int H = c.H, I = c.I, E = c.E, k = c.k;
    const int KSg = H / 64, MTg = I / 64;   // gate/up: k-steps, m-tiles
    const int KSd = I / 64, MTd = H / 128;  // down
    const int nslot = k + c.has_shared;
    float* x32 = sm;                 // [H]
    float* xperm = x32 + H;          // [H]
    float* xsum = xperm + H;         // [H/64]
    float* xsc = xsum + KSg;         // [H/64]
    float* aperm = xsc + KSg;        // [I]
    float* asum = aperm + I;         // [I/64]
    float* asc = asum + KSd;         // [I/64]
    float* logits = asc + KSd;       // [256]
    float* red = logits + 256;       // [32]
    int* sel = reinterpret_cast<int*>(red + 32);   // [32]
    float* selg = reinterpret_cast<float*>(sel + 32);  // [33]: gates, then the shared gate
    volatile int* abort_flag = reinterpret_cast<volatile int*>(selg + 33);

    float* rpart = c.dfz.rpart;      // [4][E]
    float* gu = c.dfz.gu;            // [slots][kGuKR][2I]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gw = warp * gridDim.x + blockIdx.x;   // task t -> SM t % grid: a phase spreads over every SM
    const int NW = gridDim.x * kFWarps;
    const uint16_t* xr = c.x;        // T == 1

    // ------------------------------------------------------------------ phase 0
    if (c.has_shared) prefetch_down(c, nullptr, 1);   // the shared expert's down blocks, needed in phase 2
    const int n_router = E * 4;
    const int n_shared = c.has_shared ? MTg * 4 * kGuKR : 0;
    const int hq = H / 4;   // router quarter row
    // A warp's first task reads weights that do not depend on x: they are requested into L2 before
    // x is staged, so the two memory latencies overlap (bulk L2 prefetch, lane 0 of the warp).
    if (lane == 0) {
        if (gw < n_router) {
            prefetch_l2(c.router32 + (size_t)(gw >> 2) * H + (gw & 3) * hq, (uint32_t)(hq * sizeof(float)));
        } else if (gw < n_router + n_shared) {
            const int s0 = gw - n_router;
            const int mt = s0 / (4 * kGuKR), q = (s0 / kGuKR) & 3, kr = s0 % kGuKR;
            const int k0 = kr * KSg / kGuKR, k1 = (kr + 1) * KSg / kGuKR;
            if (q == 0 && k1 > k0)   // the four row quarters share these blocks
                prefetch_l2(c.w_gu + (((size_t)E * MTg + mt) * KSg + k0) * kBlockBytes, (uint32_t)((k1 - k0) * kBlockBytes));
        }
    }
    // Launched as a programmatic dependent of the previous kernel in the stream: everything above
    // reads only the handle's weights; x and the workspace are touched only after the previous
    // grid has completed and its memory is visible.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int i = threadIdx.x; i < H; i += kFThreads) x32[i] = __uint_as_float((uint32_t)xr[i] << 16);
    if (threadIdx.x == 0) *abort_flag = 0;
    __syncthreads();
    stage_groups(H, [&](int i) { return x32[i]; }, xperm, xsum, xsc);
    float sgd = 0.f;
    if (c.has_shared)
        for (int i = threadIdx.x; i < H; i += kFThreads) sgd = fmaf(x32[i], c.sgw[i], sgd);
    sgd = warp_sum(sgd);
    if (lane == 0) red[warp] = sgd;
    __syncthreads();
    if (threadIdx.x == 0) {
        float z = 0.f;
        for (int w = 0; w < kFWarps; ++w) z += red[w];
        selg[32] = c.has_shared ? 1.f / (1.f + expf(-z)) : 0.f;
    }
    for (int task = gw; task < n_router + n_shared; task += NW) {
        if (task < n_router) {
            const int e = task >> 2, kq = task & 3;
            const float* wrow = c.router32 + (size_t)e * H + kq * hq;
            float d = 0.f;
#pragma unroll 4
            for (int h = lane * 4; h < hq; h += 128) {
                const float4 wv = __ldg(reinterpret_cast<const float4*>(wrow + h));
                const float4 xv = *reinterpret_cast<const float4*>(x32 + kq * hq + h);
                d = fmaf(wv.x, xv.x, fmaf(wv.y, xv.y, fmaf(wv.z, xv.z, fmaf(wv.w, xv.w, d))));
            }
            d = warp_sum(d);
            if (lane == 0) rpart[kq * E + e] = d;
        } else {
            const int s = task - n_router;
            const int mt = s / (4 * kGuKR), q = (s / kGuKR) & 3, kr = s % kGuKR;
            GemvTask t;
            t.blocks = c.w_gu + ((size_t)E * MTg + mt) * KSg * kBlockBytes;   // shared expert = group E
            t.row = 32 * q + lane;
            t.k0 = kr * KSg / kGuKR;
            t.k1 = (kr + 1) * KSg / kGuKR;
            const float v = run_gemv(t, xperm, xsum, xsc);
            gu[((size_t)k * kGuKR + kr) * (2 * I) + mt * 128 + t.row] = v;
        }
    }
    if (!grid_barrier(c.dfz.bar, gridDim.x, c.status, abort_flag)) return;

    // ------------------------------------------------------------------ phase 1: top-k, routed gate/up
    for (int e = threadIdx.x; e < 256; e += kFThreads) {
        float v = -INFINITY;
        if (e < E) {
            const float s = rpart[e] + rpart[E + e] + rpart[2 * E + e] + rpart[3 * E + e] + c.rbias[e];
            v = (s != s) ? -INFINITY : s;
        }
        logits[e] = v;
    }
    __syncthreads();
    if (warp == 0) {
        // top-k by logit, ties to the lower expert index: per round one warp-wide max of the keys
        // and one min of the indices holding it (two redux instructions)
        uint32_t key[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) key[i] = ord_key(logits[lane + 32 * i]);
        unsigned taken = 0;
        int my_e = 0;
        float my_v = 0.f;
        for (int j = 0; j < k; ++j) {
            uint32_t best = 0;
            int bi = -1;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (lane + 32 * i < E && !((taken >> i) & 1u) && (bi < 0 || key[i] > best)) { best = key[i]; bi = i; }
            }
            const uint32_t m = __reduce_max_sync(0xffffffffu, best);
            const uint32_t cand = (bi >= 0 && best == m) ? (uint32_t)(lane + 32 * bi) : 0xFFFFFFFFu;
            const uint32_t be = __reduce_min_sync(0xffffffffu, cand);
            if ((int)(be & 31u) == lane) taken |= 1u << (be >> 5);
            if (lane == j) { my_e = (int)be; my_v = logits[be & 255u]; }
        }
        const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
        const float p = lane < k ? expf(my_v - vmax) : 0.f;
        const float z = warp_sum(p);
        if (lane < k) {
            if (my_e < 0 || my_e >= E) { set_status(c.status, MOE_STATUS_BOUNDS); my_e = 0; }
            sel[lane] = my_e;
            selg[lane] = p / z;
            if (blockIdx.x == 0) {
                c.idx[lane] = my_e;
                c.gates[lane] = p / z;
            }
        }
        if (blockIdx.x == 0 && lane == 0) c.sg[0] = selg[32];
    }
    __syncthreads();
    prefetch_down(c, sel, k);   // the routed experts' down blocks stream into L2 during gate/up
    {
        const int n_tasks = k * MTg * 4 * kGuKR;
        for (int task = gw; task < n_tasks; task += NW) {
            const int j = task / (MTg * 4 * kGuKR);
            const int r = task % (MTg * 4 * kGuKR);
            const int mt = r / (4 * kGuKR), q = (r / kGuKR) & 3, kr = r % kGuKR;
            GemvTask t;
            t.blocks = c.w_gu + ((size_t)sel[j] * MTg + mt) * KSg * kBlockBytes;
            t.row = 32 * q + lane;
            t.k0 = kr * KSg / kGuKR;
            t.k1 = (kr + 1) * KSg / kGuKR;
            const float v = run_gemv(t, xperm, xsum, xsc);
            gu[((size_t)j * kGuKR + kr) * (2 * I) + mt * 128 + t.row] = v;
        }
    }
    if (!grid_barrier(c.dfz.bar, gridDim.x, c.status, abort_flag)) return;
    // the next kernel in the stream may be scheduled from here on (its CTAs take an SM as this
    // grid's CTAs leave it, and wait for this grid's completion before reading anything it writes)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // ------------------------------------------------------------------ phase 2: down + combine
    const int tasks_per_slot = MTd * 4 * kDnKR;
    const int blocks_per_slot = (tasks_per_slot + kFWarps - 1) / kFWarps;
    const int expected = nslot * kDnKR;
    for (int vb = blockIdx.x; vb < nslot * blocks_per_slot; vb += gridDim.x) {
        const int j = vb % nslot, bi = vb / nslot;
        const int e = (j < k) ? sel[j] : E;
        const float gate = (j < k) ? selg[j] : selg[32];
        const int task = bi * kFWarps + warp;
        GemvTask t;
        GemvRegs wr;
        if (task < tasks_per_slot) {   // weight loads first: they overlap the act staging below
            const int mt = task / (4 * kDnKR), q = (task / kDnKR) & 3, kr = task % kDnKR;
            t.blocks = c.w_dn + ((size_t)e * MTd + mt) * KSd * kBlockBytes;
            t.row = 32 * q + lane;
            t.k0 = kr * KSd / kDnKR;
            t.k1 = (kr + 1) * KSd / kDnKR;
            gemv_load(t, wr);
        }
        __syncthreads();
        // act = silu(G) * U for this slot, from the k-range partials (gate row / up row of column i)
        stage_groups(I, [&](int i) {
            const int mt = i >> 6, il = i & 63, q = il >> 4, li = il & 15;
            const int rg = mt * 128 + 32 * q + li, ru = rg + 16;
            float G = 0.f, U = 0.f;
#pragma unroll
            for (int kr = 0; kr < kGuKR; ++kr) {
                G += gu[((size_t)j * kGuKR + kr) * (2 * I) + rg];
                U += gu[((size_t)j * kGuKR + kr) * (2 * I) + ru];
            }
            return G * U / (1.f + expf(-G));
        }, aperm, asum, asc);
        __syncthreads();
        if (task < tasks_per_slot) {
            const int mt = task / (4 * kDnKR), q = (task / kDnKR) & 3;
            const float y = gemv_dot(t, wr, aperm, asum, asc) * gate;
            const int h = mt * 128 + t.row;
            atomicAdd(&c.dfz.outacc[h], y);
            __syncwarp();
            unsigned last = 0;
            if (lane == 0) {
                // acq_rel: releases this warp's additions, and the last arriver acquires everyone's
                unsigned old;
                asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(old) : "l"(&c.dfz.cnt[mt * 4 + q]) : "memory");
                last = old == (unsigned)expected - 1 ? 1u : 0u;
            }
            last = __shfl_sync(0xffffffffu, last, 0);
            __syncwarp();
            if (last) {
                const float v = atomicExch(&c.dfz.outacc[h], 0.f);
                c.out[h] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
                if (lane == 0) atomicExch(&c.dfz.cnt[mt * 4 + q], 0u);
            }
        }
    }
}

}  // namespace

int decode_fused_smem_bytes(int H, int I) {
    return (int)sizeof(float) * (2 * H + 2 * (H / 64) + I + 2 * (I / 64) + 256 + 32 + 32 + 33 + 4);
}

cudaError_t launch_decode_fused(const Ctx& c, int num_sms, cudaStream_t st) {
    const int smem = decode_fused_smem_bytes(c.H, c.I);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms);
    cfg.blockDim = dim3(kFThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlaps the launch with the previous kernel's tail
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, decode_fused_kernel, c);
}

}  // namespace moe
