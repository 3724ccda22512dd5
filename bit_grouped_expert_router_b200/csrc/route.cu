// route.cu -- router logits, top-k + renormalised gates, and token-to-expert bucketing.
//
// Everything stays on the device and in stream order (no host synchronisation anywhere): the
// prefill grouped GEMMs read their tile list and row counts from memory these kernels write.
// This follows "Perplexity Open-Sources Lily..." section "The optimizations follow the
// workload" (routing kept on the GPU, no CPU synchronisation during the MoE work).
//
// Bucketing is a stable counting sort done in two passes:
//   topk      : per 64-token bucketing block, a histogram of its expert choices (global atomics);
//   scatter   : every CTA (one per bucketing block) reads the whole histogram for the bucket sizes,
//               the bucket offsets (exclusive scan over the experts) and its own base inside each
//               bucket (the rows of earlier blocks); CTA 0 writes the sizes, offsets and the
//               grouped GEMMs' tile list.  Then ranks within the CTA in token order (warp
//               match_any) give every (token, slot) entry its row in the bucketed layout with its
//               token and gate (the gather copies the token's activation row there), and the last
//               CTA to finish re-zeroes the histogram for the next call.  (A separate one-CTA scan
//               kernel between the two cost a kernel boundary on the critical path.)
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
    griddep_wait();
    griddep_launch_dependents();
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
        return launch_pdl(router_simt_kernel<kRouterTTSmall>, grid, dim3(256), 0, st, c);
    } else {
        dim3 grid((c.T + kRouterTT - 1) / kRouterTT, 1);
        return launch_pdl(router_simt_kernel<kRouterTT>, grid, dim3(256), 0, st, c);
    }
}

__device__ __forceinline__ uint32_t bf16x2_to_half2_bits(uint32_t w, bool* range_bad) {
    const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xFFFF0000u);
    if (!(fabsf(lo) <= 65504.f) || !(fabsf(hi) <= 65504.f)) *range_bad = true;
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// ---- top-k, renormalised softmax gates, shared gate, bucket histogram ------------------------
// One warp per token (8 per CTA); lane L holds experts L, L+32, ... (E <= 256), each the sum of the
// c.ks partial logits plus the bias.  Selection: k rounds of a warp arg-max (ties -> lower expert
// index); NaN logits are treated as -inf so every selected index is valid.  Gates:
// exp(l_j - l_max) / sum over the selected (softmax restricted to the selection, renormalised).
// Shared gate: sigmoid(x . w_sg).  Prefill path (do_hist): count the token's experts into the
// histogram row of its 64-token bucketing block (global atomics; the scatter kernel re-zeroes the
// row after use) and zero the token's fp32 accumulator row for the down-projection combine.
// Order-preserving map of a float to an unsigned key (-0 first made +0, so equal floats give
// equal keys).
__device__ __forceinline__ uint32_t ord_key(float v) {
    const uint32_t u = __float_as_uint(v + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The per-token row pass of the routing step, one warp per token: optionally the shared-expert
// gate sigmoid(x_t . shared_gate) (dot), and on the prefill path the fp16 copy of the row for the
// tensor cores (range-checked) and the zeroing of the token's fp32 combine row.  Returns the gate
// (0 without dot) in every lane.
__device__ float token_row_pass(const Ctx& c, int t, int lane, bool dot, bool prefill) {
    float sgv = 0.f;
    const uint16_t* xr = c.x + (size_t)t * c.H;
    float d = 0.f;
    bool range_bad = false;
    if (dot || prefill) {
        // the lane's row loads (up to 8 chunks of 8 elements) are all issued before the arithmetic
        constexpr int kXU = 8;
        for (int h0 = lane * 8; h0 < c.H; h0 += 256 * kXU) {
            uint4 rawv[kXU];
#pragma unroll
            for (int u = 0; u < kXU; ++u)
                if (h0 + 256 * u < c.H) rawv[u] = __ldg(reinterpret_cast<const uint4*>(xr + h0 + 256 * u));
#pragma unroll
            for (int u = 0; u < kXU; ++u) {
                const int h = h0 + 256 * u;
                if (h >= c.H) break;
                const uint4 raw = rawv[u];
                if (dot) {
                    const float4 w0 = *reinterpret_cast<const float4*>(c.sgw + h);
                    const float4 w1 = *reinterpret_cast<const float4*>(c.sgw + h + 4);
                    d = fmaf(__uint_as_float(raw.x << 16), w0.x, d);
                    d = fmaf(__uint_as_float(raw.x & 0xFFFF0000u), w0.y, d);
                    d = fmaf(__uint_as_float(raw.y << 16), w0.z, d);
                    d = fmaf(__uint_as_float(raw.y & 0xFFFF0000u), w0.w, d);
                    d = fmaf(__uint_as_float(raw.z << 16), w1.x, d);
                    d = fmaf(__uint_as_float(raw.z & 0xFFFF0000u), w1.y, d);
                    d = fmaf(__uint_as_float(raw.w << 16), w1.z, d);
                    d = fmaf(__uint_as_float(raw.w & 0xFFFF0000u), w1.w, d);
                }
                if (prefill) {   // fp16 copy of the row for the tensor-core path (exact for |x| < 65504)
                    uint4 o;
                    o.x = bf16x2_to_half2_bits(raw.x, &range_bad);
                    o.y = bf16x2_to_half2_bits(raw.y, &range_bad);
                    o.z = bf16x2_to_half2_bits(raw.z, &range_bad);
                    o.w = bf16x2_to_half2_bits(raw.w, &range_bad);
                    *reinterpret_cast<uint4*>(c.x16 + (size_t)t * c.H + h) = o;
                }
            }
        }
    }
    if (dot) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
        sgv = 1.f / (1.f + expf(-d));
    }
    if (range_bad) set_status(c.status, MOE_STATUS_RANGE);
    if (prefill) {
        float4* ar = reinterpret_cast<float4*>(c.acc + (size_t)t * c.H);
        for (int h4 = lane; h4 < c.H / 4; h4 += 32) ar[h4] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    return sgv;
}

__global__ void __launch_bounds__(256) topk_kernel(Ctx c, int do_hist) {
    griddep_wait();
    griddep_launch_dependents();
    const int lane = lane_id();
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= c.T) return;
    // logits: the partial sums of expert e = lane + 32 i, summed in split order, plus the bias
    float l[8];
    if (c.ks == 4) {   // the tensor-core router's four partial sums: every load issued first
        float pq[4][8];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = lane + 32 * i;
                pq[q][i] = e < c.E ? c.part[((size_t)q * c.T + t) * c.E + e] : 0.f;
            }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            const float s = (((pq[0][i] + pq[1][i]) + pq[2][i]) + pq[3][i]) + (e < c.E ? c.rbias[e] : 0.f);
            l[i] = (e < c.E && s == s) ? s : -INFINITY;
        }
    } else if (c.ks % 4 == 0) {   // 8 or 16 partial sums (short calls): four splits' loads at a time
        float sacc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) sacc[i] = 0.f;
        for (int q0 = 0; q0 < c.ks; q0 += 4) {
            float pq[4][8];
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int e = lane + 32 * i;
                    pq[q][i] = e < c.E ? c.part[((size_t)(q0 + q) * c.T + t) * c.E + e] : 0.f;
                }
#pragma unroll
            for (int i = 0; i < 8; ++i) sacc[i] = (((sacc[i] + pq[0][i]) + pq[1][i]) + pq[2][i]) + pq[3][i];
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            const float s = sacc[i] + (e < c.E ? c.rbias[e] : 0.f);
            l[i] = (e < c.E && s == s) ? s : -INFINITY;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            float v = -INFINITY;
            if (e < c.E) {
                float s = 0.f;
                for (int q = 0; q < c.ks; ++q) s += c.part[((size_t)q * c.T + t) * c.E + e];
                s += c.rbias[e];
                v = (s != s) ? -INFINITY : s;
            }
            l[i] = v;
        }
    }
    // top k by logit, ties to the lower expert index: per pick one warp-wide max of the keys and
    // one min of the indices holding it
    uint32_t key[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) key[i] = ord_key(l[i]);
    unsigned taken = 0;
    int my_e = 0;
    float my_v = 0.f;
    for (int j = 0; j < c.k; ++j) {
        uint32_t best = 0;
        int bi = -1;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (lane + 32 * i < c.E && !((taken >> i) & 1u) && (bi < 0 || key[i] > best)) { best = key[i]; bi = i; }
        }
        const uint32_t m = __reduce_max_sync(0xffffffffu, best);
        const uint32_t cand = (bi >= 0 && best == m) ? (uint32_t)(lane + 32 * bi) : 0xFFFFFFFFu;
        const uint32_t be = __reduce_min_sync(0xffffffffu, cand);
        if ((int)(be & 31u) == lane) taken |= 1u << (be >> 5);
        if (lane == j) my_e = (int)be;
    }
    // each lane j < k fetches the value of its pick from the lane that holds it
    {
        const int src = my_e & 31, slot = my_e >> 5;
        float v = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float cand = __shfl_sync(0xffffffffu, l[i], src);
            if (i == slot) v = cand;
        }
        my_v = v;
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
        if (do_hist) atomicAdd(&c.hist[(size_t)(t / kTokPerBucketBlk) * c.E + my_e], 1);
    }
    const float sgv = token_row_pass(c, t, lane, c.has_shared != 0, do_hist != 0);
    if (lane == 0) c.sg[t] = sgv;
}

cudaError_t launch_topk(const Ctx& c, bool histogram, cudaStream_t st) {
    return launch_pdl(topk_kernel, dim3((c.T + 7) / 8), dim3(256), 0, st, c, histogram ? 1 : 0);
}

// Routing supplied by the caller (moe_forward_routed): the same outputs as topk_kernel -- expert
// ids, gates and shared gate in the workspace, the bucketing histogram and the row pass on the
// prefill path -- with idx / gates / shared gate read instead of selected.  An id outside [0, E)
// is recorded (BOUNDS) and becomes expert 0 with gate 0, so it contributes nothing.
__global__ void __launch_bounds__(256) routing_supplied_kernel(Ctx c, const int* __restrict__ idx_in,
                                                               const float* __restrict__ gates_in,
                                                               const float* __restrict__ sg_in, int prefill) {
    griddep_wait();
    griddep_launch_dependents();
    const int lane = lane_id();
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= c.T) return;
    if (lane < c.k) {
        const size_t j = (size_t)t * c.k + lane;
        int e = idx_in[j];
        float g = gates_in[j];
        if (e < 0 || e >= c.E) {
            set_status(c.status, MOE_STATUS_BOUNDS);
            e = 0;
            g = 0.f;
        }
        c.idx[j] = e;
        c.gates[j] = g;
        if (prefill) atomicAdd(&c.hist[(size_t)(t / kTokPerBucketBlk) * c.E + e], 1);
    }
    token_row_pass(c, t, lane, false, prefill != 0);
    if (lane == 0) c.sg[t] = c.has_shared ? sg_in[t] : 0.f;
}

cudaError_t launch_routing_supplied(const Ctx& c, const int* idx, const float* gates, const float* sg, bool prefill,
                                    cudaStream_t st) {
    return launch_pdl(routing_supplied_kernel, dim3((c.T + 7) / 8), dim3(256), 0, st, c, idx, gates, sg,
                      prefill ? 1 : 0);
}

// ---- bucket offsets + tile list, and the scatter ----------------------------------------------
__device__ __forceinline__ int warp_incl_scan(int v) {
    const int lane = lane_id();
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += o;
    }
    return v;
}

// ---- scatter: bucket positions and row metadata ---------------------------------------------

__global__ void __launch_bounds__(1024) scatter_kernel(Ctx c) {
    griddep_wait();
    griddep_launch_dependents();
    __shared__ int part[4][256], partb[4][256];
    __shared__ int cnt[264], off[264], toff[264];   // bucket sizes, offsets, first tile slots
    __shared__ int wtot[2][32];                     // per-warp totals of the group scan
    __shared__ int wcnt[32 * 256];                  // [warp][expert] counts, then bases, of a round
    __shared__ int last;
    int* nxt = partb[0];    // [E] next free row of each bucket for this CTA (after the scan)
    const int tid = threadIdx.x, lane = lane_id(), warp = tid >> 5;
    const int b = blockIdx.x;
    // Every CTA reads the whole histogram (one row per bucketing block): per expert the bucket
    // size and this block's base inside the bucket (the rows of earlier blocks), four threads per
    // expert each over a quarter of the blocks, loads issued eight at a time.  The L2 reads grow
    // with the square of the blocks: 4 MB for 4096 tokens, 64 MB for 16384, 1 GB for 65536 (a
    // few percent of a call that size).
    {
        const int e = tid & 255, quarter = tid >> 8;
        const int b_lo = quarter * c.nblk / 4, b_hi = (quarter + 1) * c.nblk / 4;
        int sum = 0, before = 0;
        if (e < c.E) {
            for (int b0 = b_lo; b0 < b_hi; b0 += 8) {
                int v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = (b0 + u < b_hi) ? c.hist[(size_t)(b0 + u) * c.E + e] : 0;
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    if (b0 + u < b) before += v[u];
                    sum += v[u];
                }
            }
        }
        part[quarter][e] = sum;
        partb[quarter][e] = before;
    }
    __syncthreads();
    int mybase = 0;
    if (tid < c.E) {
        cnt[tid] = part[0][tid] + part[1][tid] + part[2][tid] + part[3][tid];
        mybase = partb[0][tid] + partb[1][tid] + partb[2][tid] + partb[3][tid];
    }
    if (tid == 0 && c.has_shared) cnt[c.E] = c.T;
    __syncthreads();
    // bucket offsets and the tile list's first slot of each group: exclusive scans in group order,
    // 32 groups per warp, then the warps' totals added in front
    {
        const int g = tid, nwg = (c.G + 31) / 32;
        int v = 0, ntl = 0, inc = 0, tinc = 0;
        if (warp < nwg) {
            v = (g < c.G) ? cnt[g] : 0;
            ntl = (v + c.tile_rows - 1) / c.tile_rows;
            inc = warp_incl_scan(v);
            tinc = warp_incl_scan(ntl);
            if (lane == 31) { wtot[0][warp] = inc; wtot[1][warp] = tinc; }
        }
        __syncthreads();
        if (warp < nwg && g < c.G) {
            int pre = 0, tpre = 0;
            for (int w = 0; w < warp; ++w) { pre += wtot[0][w]; tpre += wtot[1][w]; }
            off[g] = pre + inc - v;
            toff[g] = tpre + tinc - ntl;
            if (g == c.G - 1) {
                off[c.G] = pre + inc;
                toff[c.G] = tpre + tinc;
                if (b == 0) c.ntiles[0] = tpre + tinc;
            }
        }
    }
    __syncthreads();
    if (tid < c.E) nxt[tid] = off[tid] + mybase;
    if (b == 0) {   // the bucket sizes, offsets and tile list, once
        for (int g = tid; g <= c.G; g += blockDim.x) c.offsets[g] = off[g];
        for (int g = tid; g < c.G; g += blockDim.x) c.counts[g] = cnt[g];
        for (int g = tid; g < c.G; g += blockDim.x) {
            const int n = cnt[g];
            int tslot = toff[g];
            for (int n0 = 0; n0 < n; n0 += c.tile_rows, ++tslot) {
                if (tslot < c.max_tiles) c.tiles1[tslot] = make_int4(g, off[g] + n0, min(c.tile_rows, n - n0), 0);
                else set_status(c.status, MOE_STATUS_BOUNDS);
            }
        }
    }
    __syncthreads();
    const int t0 = b * kTokPerBucketBlk;
    const int nt = min(kTokPerBucketBlk, c.T - t0);
    // Stable ranking of the block's entries in (token, slot) order, up to 1024 per round: each warp
    // ranks its 32 consecutive entries among equal experts (match), writes its per-expert counts,
    // and one thread per expert turns the warps' counts into bases by an exclusive scan in warp
    // order, so an entry's row is its expert's next free row + the base + its rank.
    const int n_entries = nt * c.k;
    for (int base = 0; base < n_entries; base += 1024) {
        const int nw = min(32, (n_entries - base + 31) / 32);
        for (int i = tid; i < nw * c.E; i += blockDim.x) wcnt[i] = 0;
        __syncthreads();
        const int i = base + tid;
        const bool active = warp < nw && i < n_entries;
        int e = -1, rank = 0;
        float gv = 0.f;
        if (warp < nw) {
            if (active) {
                e = c.idx[t0 * c.k + i];
                gv = c.gates[t0 * c.k + i];
                if (e < 0 || e >= c.E) { set_status(c.status, MOE_STATUS_BOUNDS); e = 0; }
            }
            const unsigned mask = __match_any_sync(0xffffffffu, e);
            rank = __popc(mask & ((1u << lane) - 1u));
            if (active && lane == __ffs(mask) - 1) wcnt[warp * c.E + e] = __popc(mask);
        }
        __syncthreads();
        if (tid < c.E) {
            int run = nxt[tid];
            for (int w = 0; w < nw; ++w) {
                const int v = wcnt[w * c.E + tid];
                wcnt[w * c.E + tid] = run;
                run += v;
            }
            nxt[tid] = run;
        }
        __syncthreads();
        if (active) {
            const int p = wcnt[warp * c.E + e] + rank;
            const int flat = t0 * c.k + i;
            if (p < 0 || p >= c.rows_cap) {
                set_status(c.status, MOE_STATUS_BOUNDS);
            } else {
                c.perm[p] = flat;
                c.row_token[p] = flat / c.k;
                c.row_gate[p] = gv;
            }
        }
        __syncthreads();   // the counts are re-zeroed by the next round
    }
    const int shared_base = off[c.E];
    if (c.has_shared) {
        for (int tt = threadIdx.x; tt < nt; tt += blockDim.x) {
            const int t = t0 + tt;
            c.row_token[shared_base + t] = t;
            c.row_gate[shared_base + t] = c.sg[t];
        }
    }
    // the last CTA to finish re-zeroes the histogram for the next call's counting (every CTA has
    // read all of it by then) and resets the counter
    if (tid == 0) {
        __threadfence();
        last = atomicAdd(c.scatter_done, 1u) == gridDim.x - 1 ? 1 : 0;
    }
    __syncthreads();
    if (last) {
        __threadfence();
        for (int i = tid; i < c.nblk * c.E; i += blockDim.x) c.hist[i] = 0;
        if (tid == 0) *c.scatter_done = 0u;
    }
}

cudaError_t launch_scatter(const Ctx& c, cudaStream_t st) {
    return launch_pdl(scatter_kernel, dim3(c.nblk), dim3(1024), 0, st, c);
}

}  // namespace moe
