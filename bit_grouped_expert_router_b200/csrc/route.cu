// route.cu -- router logits, top-k + renormalised gates, and token-to-expert bucketing.
//
// Everything stays on the device and in stream order (no host synchronisation anywhere): the
// prefill grouped GEMMs read their tile list and row counts from memory these kernels write.
// This follows "Perplexity Open-Sources Lily..." section "The optimizations follow the
// workload" (routing kept on the GPU, no CPU synchronisation during the MoE work).
//
// Bucketing is a stable counting sort done in three passes:
//   topk      : per CTA of 64 tokens, a histogram of its expert choices;
//   bucket_scan (one CTA): per-expert exclusive scan over the CTAs -> each CTA's base inside the
//               bucket, bucket sizes, bucket offsets, and the tile list of the grouped GEMMs;
//   scatter   : per CTA, ranks within the CTA in token order (warp match_any), giving every
//               (token, slot) entry its row in the bucketed layout; copies the token's
//               activations (bf16 -> fp16) into that row and into its shared-expert row.
#include <float.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// ---- router logits on CUDA cores ---------------------------------------------------------------
// part[ks][t][e] = sum over the CTA's K slice of x[t][h] * router[e][h]; thread = expert.
// grid (ceil(T/TT), ks), 256 threads.  The transposed fp32 router [H][E] makes each step one
// coalesced row read shared by TT tokens held in shared memory.
template <int TT>
__global__ void __launch_bounds__(256) router_simt_kernel(Ctx c) {
    constexpr int KC = 256;  // columns staged per pass
    __shared__ __align__(16) float xs[KC * TT];
    const int e = threadIdx.x;
    const int t0 = blockIdx.x * TT;
    const int ksl = c.H / c.ks;
    const int k0 = blockIdx.y * ksl;
    float acc[TT];
#pragma unroll
    for (int i = 0; i < TT; ++i) acc[i] = 0.f;
    for (int kc = 0; kc < ksl; kc += KC) {
        const int kn = min(KC, ksl - kc);
        __syncthreads();
        for (int i = threadIdx.x; i < kn * TT; i += blockDim.x) {
            const int tt = i / kn, hh = i % kn;
            const int t = t0 + tt;
            const float v = (t < c.T) ? __uint_as_float((uint32_t)c.x[(size_t)t * c.H + k0 + kc + hh] << 16) : 0.f;
            xs[hh * TT + tt] = v;
        }
        __syncthreads();
        if (e < c.E) {
            const float* w = c.wrt + (size_t)(k0 + kc) * c.E + e;
            for (int hh = 0; hh < kn; ++hh) {
                const float wv = __ldg(w + (size_t)hh * c.E);
                const float4* xv = reinterpret_cast<const float4*>(xs + hh * TT);
#pragma unroll
                for (int q = 0; q < TT / 4; ++q) {
                    const float4 v = xv[q];
                    acc[4 * q + 0] = fmaf(v.x, wv, acc[4 * q + 0]);
                    acc[4 * q + 1] = fmaf(v.y, wv, acc[4 * q + 1]);
                    acc[4 * q + 2] = fmaf(v.z, wv, acc[4 * q + 2]);
                    acc[4 * q + 3] = fmaf(v.w, wv, acc[4 * q + 3]);
                }
            }
        }
    }
    if (e < c.E) {
#pragma unroll
        for (int tt = 0; tt < TT; ++tt)
            if (t0 + tt < c.T) c.part[((size_t)blockIdx.y * c.T + t0 + tt) * c.E + e] = acc[tt];
    }
}

cudaError_t launch_router_simt(const Ctx& c, cudaStream_t st) {
    if (c.ks > 1) {
        dim3 grid((c.T + kRouterTTSmall - 1) / kRouterTTSmall, c.ks);
        router_simt_kernel<kRouterTTSmall><<<grid, 256, 0, st>>>(c);
    } else {
        dim3 grid((c.T + kRouterTT - 1) / kRouterTT, 1);
        router_simt_kernel<kRouterTT><<<grid, 256, 0, st>>>(c);
    }
    return cudaGetLastError();
}

// ---- top-k, renormalised softmax gates, shared gate, per-CTA histogram ------------------------
// One warp per token; lane L holds experts L, L+32, ... (E <= 256).  Selection: k rounds of a
// warp arg-max (ties -> lower expert index); NaN logits are treated as -inf so every selected
// index is valid.  Gates: exp(l_j - l_max) / sum over the selected (softmax restricted to the
// selection and renormalised).  Shared gate: sigmoid(x . w_sg).
__global__ void __launch_bounds__(256) topk_kernel(Ctx c, int do_hist) {
    __shared__ int hist[256];
    __shared__ float lg[8][256];
    const int lane = lane_id(), warp = threadIdx.x >> 5;
    if (do_hist) {
        for (int e = threadIdx.x; e < c.E; e += blockDim.x) hist[e] = 0;
    }
    const int t_begin = blockIdx.x * kTokPerBucketBlk;
    const int t_end = min(c.T, t_begin + kTokPerBucketBlk);
    for (int tb = t_begin; tb < t_end; tb += 8) {
        // phase 1: the block reduces the split-K partial logits of 8 tokens in parallel
        __syncthreads();
        for (int i = threadIdx.x; i < 8 * c.E; i += blockDim.x) {
            const int tt = i / c.E, e = i % c.E;
            const int t = tb + tt;
            if (t < t_end) {
                float s = 0.f;
#pragma unroll 8
                for (int q = 0; q < c.ks; ++q) s += c.part[((size_t)q * c.T + t) * c.E + e];
                s += c.rbias[e];
                lg[tt][e] = (s != s) ? -INFINITY : s;
            }
        }
        __syncthreads();
        // phase 2: one warp per token selects the top k
        const int t = tb + warp;
        if (t >= t_end) continue;
        float l[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            l[i] = (e < c.E) ? lg[warp][e] : -INFINITY;
        }
        unsigned taken = 0;
        int my_e = 0;
        float my_v = 0.f;
        for (int j = 0; j < c.k; ++j) {
            float bv = 0.f;
            int be = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = lane + 32 * i;
                if (e < c.E && !((taken >> i) & 1u)) {
                    if (be == 0x7fffffff || l[i] > bv) { bv = l[i]; be = e; }
                }
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
        const float p = (lane < c.k) ? expf(my_v - vmax) : 0.f;
        float z = p;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
        if (lane < c.k) {
            if (my_e < 0 || my_e >= c.E) { set_status(c.status, MOE_STATUS_BOUNDS); my_e = 0; }
            c.idx[(size_t)t * c.k + lane] = my_e;
            c.gates[(size_t)t * c.k + lane] = p / z;
            if (do_hist) atomicAdd(&hist[my_e], 1);
        }
        float sgv = 0.f;
        if (c.has_shared) {
            float d = 0.f;
            const uint16_t* xr = c.x + (size_t)t * c.H;
            for (int h = lane * 8; h < c.H; h += 256) {
                const uint4 raw = *reinterpret_cast<const uint4*>(xr + h);
                const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    d = fmaf(__uint_as_float(w4[q] << 16), c.sgw[h + 2 * q], d);
                    d = fmaf(__uint_as_float(w4[q] & 0xFFFF0000u), c.sgw[h + 2 * q + 1], d);
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
            sgv = 1.f / (1.f + expf(-d));
        }
        if (lane == 0) c.sg[t] = sgv;
    }
    if (do_hist) {
        __syncthreads();
        for (int e = threadIdx.x; e < c.E; e += blockDim.x) c.hist[(size_t)blockIdx.x * c.E + e] = hist[e];
    }
}

cudaError_t launch_topk(const Ctx& c, bool histogram, cudaStream_t st) {
    topk_kernel<<<c.nblk, 256, 0, st>>>(c, histogram ? 1 : 0);
    return cudaGetLastError();
}

// ---- bucket scan + tile list (one CTA) ---------------------------------------------------------
__device__ __forceinline__ int warp_incl_scan(int v) {
    const int lane = lane_id();
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += o;
    }
    return v;
}

__global__ void __launch_bounds__(1024) bucket_scan_kernel(Ctx c) {
    __shared__ int cnt[264], off[264], toff[264];
    const int tid = threadIdx.x, lane = lane_id();
    for (int e = tid; e < c.E; e += blockDim.x) {
        int run = 0;
        for (int b = 0; b < c.nblk; ++b) {
            const int v = c.hist[(size_t)b * c.E + e];
            c.hist[(size_t)b * c.E + e] = run;  // becomes this CTA's base inside bucket e
            run += v;
        }
        cnt[e] = run;
    }
    if (tid == 0 && c.has_shared) cnt[c.E] = c.T;
    __syncthreads();
    if (tid < 32) {
        int run = 0, trun = 0;
        for (int base = 0; base < c.G; base += 32) {
            const int g = base + lane;
            const int v = (g < c.G) ? cnt[g] : 0;
            const int nt = (v + kBN - 1) / kBN;
            const int inc = warp_incl_scan(v);
            const int tinc = warp_incl_scan(nt);
            if (g < c.G) { off[g] = run + inc - v; toff[g] = trun + tinc - nt; }
            run += __shfl_sync(0xffffffffu, inc, 31);
            trun += __shfl_sync(0xffffffffu, tinc, 31);
        }
        if (lane == 0) {
            off[c.G] = run;
            toff[c.G] = trun;
            c.ntiles[0] = trun;
        }
    }
    __syncthreads();
    for (int g = tid; g <= c.G; g += blockDim.x) c.offsets[g] = off[g];
    for (int g = tid; g < c.G; g += blockDim.x) c.counts[g] = cnt[g];
    for (int g = tid; g < c.G; g += blockDim.x) {
        const int n = cnt[g];
        int tslot = toff[g];
        for (int n0 = 0; n0 < n; n0 += kBN, ++tslot) {
            if (tslot < c.max_tiles) c.tiles1[tslot] = make_int4(g, off[g] + n0, min(kBN, n - n0), 0);
            else set_status(c.status, MOE_STATUS_BOUNDS);
        }
    }
}

cudaError_t launch_bucket_scan(const Ctx& c, cudaStream_t st) {
    bucket_scan_kernel<<<1, 1024, 0, st>>>(c);
    return cudaGetLastError();
}

// ---- scatter: bucket positions, row metadata, gathered fp16 activations ------------------------
__device__ __forceinline__ uint32_t bf16x2_to_half2_bits(uint32_t w, bool* range_bad) {
    const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xFFFF0000u);
    if (!(fabsf(lo) <= 65504.f) || !(fabsf(hi) <= 65504.f)) *range_bad = true;
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

__global__ void __launch_bounds__(256) scatter_kernel(Ctx c) {
    extern __shared__ int sm[];
    int* cnt = sm;          // [E] next free row of each bucket for this CTA
    int* pos = sm + c.E;    // [64 * k] row of each (token, slot) of this CTA
    const int lane = lane_id(), warp = threadIdx.x >> 5;
    const int t0 = blockIdx.x * kTokPerBucketBlk;
    const int nt = min(kTokPerBucketBlk, c.T - t0);
    for (int e = threadIdx.x; e < c.E; e += blockDim.x)
        cnt[e] = c.offsets[e] + c.hist[(size_t)blockIdx.x * c.E + e];
    __syncthreads();
    if (warp == 0) {
        const int n_entries = nt * c.k;
        for (int base = 0; base < n_entries; base += 32) {
            const int i = base + lane;
            const bool active = i < n_entries;
            const int flat = t0 * c.k + i;
            int e = active ? c.idx[flat] : -1;
            if (active && (e < 0 || e >= c.E)) { set_status(c.status, MOE_STATUS_BOUNDS); e = 0; }
            const unsigned mask = __match_any_sync(0xffffffffu, e);
            const int rank = __popc(mask & ((1u << lane) - 1u));
            const int p = active ? cnt[e] + rank : 0;
            __syncwarp();
            if (active && lane == __ffs(mask) - 1) cnt[e] += __popc(mask);
            __syncwarp();
            if (active) {
                if (p < 0 || p >= c.rows_cap) {
                    set_status(c.status, MOE_STATUS_BOUNDS);
                    pos[i] = -1;
                } else {
                    pos[i] = p;
                    c.perm[p] = flat;
                    c.row_token[p] = flat / c.k;
                    c.row_gate[p] = c.gates[flat];
                }
            }
        }
    }
    __syncthreads();
    const int shared_base = c.offsets[c.E];
    bool range_bad = false;
    for (int tt = warp; tt < nt; tt += 8) {
        const int t = t0 + tt;
        const uint16_t* xr = c.x + (size_t)t * c.H;
        for (int h = lane * 8; h < c.H; h += 256) {
            const uint4 raw = *reinterpret_cast<const uint4*>(xr + h);
            uint4 o;
            o.x = bf16x2_to_half2_bits(raw.x, &range_bad);
            o.y = bf16x2_to_half2_bits(raw.y, &range_bad);
            o.z = bf16x2_to_half2_bits(raw.z, &range_bad);
            o.w = bf16x2_to_half2_bits(raw.w, &range_bad);
            for (int j = 0; j < c.k; ++j) {
                const int p = pos[tt * c.k + j];
                if (p >= 0) *reinterpret_cast<uint4*>(c.xp + (size_t)p * c.H + h) = o;
            }
            if (c.has_shared) *reinterpret_cast<uint4*>(c.xp + (size_t)(shared_base + t) * c.H + h) = o;
        }
        float4* ar = reinterpret_cast<float4*>(c.acc + (size_t)t * c.H);
        for (int h4 = lane; h4 < c.H / 4; h4 += 32) ar[h4] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (c.has_shared && lane == 0) {
            c.row_token[shared_base + t] = t;
            c.row_gate[shared_base + t] = c.sg[t];
        }
    }
    if (range_bad) set_status(c.status, MOE_STATUS_RANGE);
}

cudaError_t launch_scatter(const Ctx& c, cudaStream_t st) {
    const size_t smem = sizeof(int) * (size_t)(c.E + kTokPerBucketBlk * c.k);
    scatter_kernel<<<c.nblk, 256, smem, st>>>(c);
    return cudaGetLastError();
}

}  // namespace moe
