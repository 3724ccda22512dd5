// decode.cu -- the decode path: sparse GEMVs over only the selected experts' packed weights.
//
// "Perplexity Lily engine" note (leslieli.dev), limits paragraph: the decode GEMVs run near the
// weight-read wall, and removing their arithmetic barely changes their speed; "A Rust + Metal
// Inference Engine..." (body): decode minimises the bytes moved per token.  So these kernels are
// a plain stream of 128-bit loads over the k routed experts' and the shared expert's blocks
// (kernel layout, see common.cuh), on CUDA cores in fp32, with no tensor cores.
//
// Arithmetic per 64-column group c of a row:  sum_i W_i v_i = s * sum_i q_i v_i + b * sum_i v_i.
// The code q_i becomes an fp32 operand in one byte-permute: a binary32 whose exponent field is
// zero encodes mantissa * 2^-149, so a zero-extended nibble IS the value q * 2^-149 (an IEEE
// subnormal, handled at full rate by FFMA without flush-to-zero; the FMAs are explicit fma.rn.f32 so
// no compiler flag can flush them).  The activations of the group
// are pre-scaled by an exact power of two 2^K chosen from the group maximum so every product and
// partial sum stays a normal number; the group result is rescaled by 2^(149-K).  Each byte of
// (word & 0x0F0F0F0F) and ((word >> 4) & 0x0F0F0F0F) is one code, so the activations are stored
// in the matching order: slot p of each 8-element word holds element kSlot[p] = {0,4,1,5,2,6,3,7}.
//
//   gemv_gateup : grid (I/64 m-tiles, k+1 slots, T), 512 threads.  Lane = weight row of the
//                 m-tile (gate and up of one column i 16 lanes apart), 4 K-splits reduced in
//                 shared memory, then act = silu(G) * U written pre-scaled for the down GEMV.
//   gemv_down   : grid (H/32, T), 64*(k+1) threads.  Warp = (slot, K half), lane = output row;
//                 the k+1 expert outputs are weighted by their gates and summed in shared memory
//                 (deterministic, no atomics) and rounded to bf16.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

__device__ __forceinline__ float pow2f(int n) {  // exact 2^n for n in [-126, 127]
    return __int_as_float((127 + n) << 23);
}

// exponent of the largest |v| of a group, clamped so 2^(125-e) splits into two finite factors
__device__ __forceinline__ int group_exponent(float m) {
    int e = (int)((__float_as_uint(m) >> 23) & 0xFFu) - 127;
    return max(-126, min(100, e));
}

__device__ __forceinline__ int slot_of(int e8) {  // inverse of {0,4,1,5,2,6,3,7}
    return (e8 >> 2) | ((e8 & 3) << 1);
}

// sum over one 64-column group of code * v', v' in slot order (smem, 16-byte aligned)
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

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Dot of one weight row (lane = row of the blocks at wb) over k-steps [c0, c1) with activations in
// slot order: every load of a chunk of up to D k-steps is issued before its arithmetic, so a warp
// keeps D x 36 bytes per lane in flight instead of waiting out one memory latency per k-step.
template <int D>
__device__ __forceinline__ float row_dot(const uint8_t* wb, int row, int c0, int c1, const float* vperm,
                                         const float* vsc, const float* vsum) {
    float acc = 0.f;
    for (int base = c0; base < c1; base += D) {
        const int n = min(D, c1 - base);
        uint4 v0[D], v1[D];
        uint32_t sb[D];
#pragma unroll
        for (int i = 0; i < D; ++i) {
            if (i < n) {
                const uint8_t* blk = wb + (size_t)(base + i) * kBlockBytes;
                v0[i] = __ldg(reinterpret_cast<const uint4*>(blk + row * 16));
                v1[i] = __ldg(reinterpret_cast<const uint4*>(blk + 2048 + row * 16));
                sb[i] = __ldg(reinterpret_cast<const uint32_t*>(blk + kBlockCodeBytes + row * 4));
            }
        }
#pragma unroll
        for (int i = 0; i < D; ++i) {
            if (i < n) {
                const int cc = base + i;
                const float s = __half2float(__ushort_as_half((unsigned short)(sb[i] & 0xFFFFu)));
                const float b = __half2float(__ushort_as_half((unsigned short)(sb[i] >> 16)));
                const float P = dot_group(v0[i], v1[i], vperm + 64 * cc);
                acc += s * (P * vsc[cc]) + b * vsum[cc];
            }
        }
    }
    return acc;
}

constexpr int kGateupThreads = 512;

__global__ void __launch_bounds__(kGateupThreads) gemv_gateup_kernel(Ctx c) {
    griddep_wait();
    griddep_launch_dependents();
    extern __shared__ __align__(16) float sm[];
    const int mt = blockIdx.x, j = blockIdx.y, t = blockIdx.z;
    const int nslot = c.k + c.has_shared;
    if (j >= nslot) return;
    int g = (j < c.k) ? c.idx[(size_t)t * c.k + j] : c.E;
    if (g < 0 || g >= c.G) {
        if (threadIdx.x == 0) set_status(c.status, MOE_STATUS_BOUNDS);
        return;
    }
    const int KS = c.H / 64, MT = c.I / 64;
    float* xperm = sm;            // [H] pre-scaled activations, slot order
    float* xsum = sm + c.H;       // [KS] plain group sums
    float* xsc = xsum + KS;       // [KS] 2^(149-K) per group
    float* red = xsc + KS;        // [4][128] K-split partials
    float* amax = red + 512;      // [4]
    const int warp = threadIdx.x >> 5, lane = lane_id();

    // ---- stage the token's activations (bf16 -> fp32, per-group power-of-two scaling)
    const uint16_t* xr = c.x + (size_t)t * c.H;
    for (int grp = warp; grp < KS; grp += kGateupThreads / 32) {
        const uint32_t raw = *reinterpret_cast<const uint32_t*>(xr + 64 * grp + 2 * lane);
        const float a0 = __uint_as_float(raw << 16), a1 = __uint_as_float(raw & 0xFFFF0000u);
        const float m = warp_max(fmaxf(fabsf(a0), fabsf(a1)));
        const float s = warp_sum(a0 + a1);
        const int K = 125 - group_exponent(m);
        const float f1 = pow2f(K / 2), f2 = pow2f(K - K / 2);
        const int e0 = 2 * lane, e1 = 2 * lane + 1;
        xperm[64 * grp + (e0 & ~7) + slot_of(e0 & 7)] = a0 * f1 * f2;
        xperm[64 * grp + (e1 & ~7) + slot_of(e1 & 7)] = a1 * f1 * f2;
        if (lane == 0) {
            xsum[grp] = s;
            xsc[grp] = pow2f(149 - K);
        }
    }
    __syncthreads();

    // ---- stream the expert's gate/up blocks of this m-tile
    const int q = warp & 3, ksp = warp >> 2;
    const int row = 32 * q + lane;
    const int c0 = ksp * KS / 4, c1 = (ksp + 1) * KS / 4;
    const uint8_t* wb = c.w_gu + ((size_t)g * MT + mt) * KS * kBlockBytes;
    red[ksp * 128 + row] = row_dot<8>(wb, row, c0, c1, xperm, xsc, xsum);
    __syncthreads();

    // ---- SwiGLU on the 64 columns of this m-tile, scaled for the down GEMV
    float a = 0.f;
    if (warp < 4) {
        const float v = red[row] + red[128 + row] + red[256 + row] + red[384 + row];
        const float other = __shfl_xor_sync(0xffffffffu, v, 16);
        if (lane < 16) a = v * other / (1.f + expf(-v));   // silu(G) * U
        const float m = warp_max(lane < 16 ? fabsf(a) : 0.f);
        if (lane == 0) amax[warp] = m;
    }
    __syncthreads();
    if (warp < 4 && lane < 16) {
        const float m = fmaxf(fmaxf(amax[0], amax[1]), fmaxf(amax[2], amax[3]));
        const int K = 125 - group_exponent(m);
        const int i = 16 * q + lane;                    // column within the 64-column group
        const size_t base = ((size_t)t * (c.k + 1) + j) * c.I + 64 * mt;
        c.dact[base + (i & ~7) + slot_of(i & 7)] = a * pow2f(K / 2) * pow2f(K - K / 2);
        const float asum = [&] {
            float s = a;
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0x0000ffffu, s, o);
            return s;
        }();
        if (lane == 0) red[q] = asum;  // red[] is free again after the barrier above
        if (q == 0 && lane == 0) {
            c.dscale[((size_t)t * (c.k + 1) + j) * MT + mt] = pow2f(149 - K);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0)
        c.dscale[(size_t)c.T * (c.k + 1) * MT + ((size_t)t * (c.k + 1) + j) * MT + mt] = red[0] + red[1] + red[2] + red[3];
}

__global__ void __launch_bounds__(1024) gemv_down_kernel(Ctx c) {
    griddep_wait();
    griddep_launch_dependents();
    extern __shared__ __align__(16) float sm[];
    const int hc = blockIdx.x, t = blockIdx.y;
    const int nslot = c.k + c.has_shared;
    const int KS = c.I / 64, MT = c.H / 128;
    float* aperm = sm;                    // [nslot][I]
    float* red = aperm + nslot * c.I;     // [nwarps][32]
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int nwarps = blockDim.x >> 5;
    for (int i = threadIdx.x; i < nslot * c.I; i += blockDim.x) {
        const int jj = i / c.I, ii = i % c.I;
        aperm[i] = c.dact[((size_t)t * (c.k + 1) + jj) * c.I + ii];
    }
    __syncthreads();
    const int j = warp >> 1, ksp = warp & 1;
    float contrib = 0.f;
    if (j < nslot) {
        const int g = (j < c.k) ? c.idx[(size_t)t * c.k + j] : c.E;
        const float gate = (j < c.k) ? c.gates[(size_t)t * c.k + j] : c.sg[t];
        if (g >= 0 && g < c.G) {
            const int h = 32 * hc + lane;
            const int mt = h >> 7, row = h & 127;
            const float* sc = c.dscale + ((size_t)t * (c.k + 1) + j) * KS;
            const float* sums = c.dscale + (size_t)c.T * (c.k + 1) * KS + ((size_t)t * (c.k + 1) + j) * KS;
            const uint8_t* wb = c.w_dn + ((size_t)g * MT + mt) * KS * kBlockBytes;
            const int c0 = ksp * KS / 2, c1 = (ksp + 1) * KS / 2;
            contrib = row_dot<4>(wb, row, c0, c1, aperm + j * c.I, sc, sums) * gate;
        } else if (lane == 0) {
            set_status(c.status, MOE_STATUS_BOUNDS);
        }
    }
    red[warp * 32 + lane] = contrib;
    __syncthreads();
    if (warp == 0) {
        float y = 0.f;
        for (int w = 0; w < nwarps; ++w) y += red[w * 32 + lane];
        c.out[(size_t)t * c.H + 32 * hc + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
    }
}

}  // namespace

cudaError_t launch_gemv_gateup(const Ctx& c, cudaStream_t st) {
    const int KS = c.H / 64;
    const size_t smem = sizeof(float) * ((size_t)c.H + 2 * KS + 512 + 4);
    dim3 grid(c.I / 64, c.k + 1, c.T);
    return launch_pdl(gemv_gateup_kernel, grid, dim3(kGateupThreads), smem, st, c);
}

cudaError_t launch_gemv_down(const Ctx& c, cudaStream_t st) {
    const int nslot = c.k + c.has_shared;
    const int threads = 64 * nslot;
    if (threads > 1024) return cudaErrorInvalidConfiguration;   // k + shared > 16 slots
    const size_t smem = sizeof(float) * ((size_t)nslot * c.I + (size_t)threads);
    dim3 grid(c.H / 32, c.T);
    return launch_pdl(gemv_down_kernel, grid, dim3(threads), smem, st, c);
}

}  // namespace moe
