// repack.cu -- one-time conversion of a layer's weights from the public layout to the kernel layout.
//
// Kernel layout of one expert matrix set (see common.cuh for the 4608-byte block format):
//   gate/up : (I/64) m-tiles x (H/64) k-steps of blocks.  In m-tile mt, TMEM lane / block row l
//             holds gate row (or, for l % 32 >= 16, up row) i = 64*mt + 16*(l/32) + (l % 16), so a
//             warp that owns lanes 32q..32q+31 sees gate and up of the same 16 columns i and can
//             pair them with one shuffle (SwiGLU without a trip through shared memory).
//   down    : (H/128) m-tiles x (I/64) k-steps; block row l is output row 128*mt + l.
// Group g < E is routed expert g, group E the shared expert.  Scales and biases are converted
// from bf16 to fp16 (round to nearest even); any value that is not exactly representable in fp16,
// and any nonzero scale below 2^-13 in magnitude (the dequantisation also uses s / 16), raises a
// flag that moe_create reports in its message (the weights stay usable).
#include "common.cuh"
#include "kernels.h"

namespace moe {

__device__ __forceinline__ uint32_t interleave_nibbles(uint32_t w) {
    uint32_t r = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t n = (w >> (4 * j)) & 0xFu;
        const int pos = (j & 1) ? (16 + 4 * (j >> 1)) : (4 * (j >> 1));
        r |= n << pos;
    }
    return r;
}

__device__ __forceinline__ uint32_t bf16_to_fp16_bits(uint16_t v, uint32_t* inexact) {
    const float f = __uint_as_float((uint32_t)v << 16);
    const __half h = __float2half_rn(f);
    if (__half2float(h) != f && f == f) atomicOr(inexact, 1u);
    return (uint32_t)__half_as_ushort(h);
}

// grid (k-steps, m-tiles, groups), 256 threads: one 4608-byte block per CTA.
__global__ void __launch_bounds__(256) repack_kernel(RepackArgs a) {
    const int c = blockIdx.x, mt = blockIdx.y, g = blockIdx.z;
    const int KS = gridDim.x, MT = gridDim.y;
    const int t = threadIdx.x;
    const int l = t >> 1, half = t & 1;
    const int cols = a.cols;
    const bool shared = (g == a.E);

    // source row and matrix for block row l
    int src_mat = 0, src_row;
    if (a.gateup) {
        src_mat = ((l & 31) >= 16) ? 1 : 0;
        src_row = 64 * mt + 16 * (l >> 5) + (l & 15);
    } else {
        src_row = 128 * mt + l;
    }
    const size_t mat_words = (size_t)a.rows_per_mat * (cols / 8);
    const size_t mat_groups = (size_t)a.rows_per_mat * (cols / 64);
    const uint32_t* q = shared ? a.qs[src_mat] : a.q[src_mat] + (size_t)g * mat_words;

    uint8_t* blk = a.dst + (((size_t)g * MT + mt) * KS + c) * kBlockBytes;
    const uint32_t* src = q + (size_t)src_row * (cols / 8) + (size_t)c * 8 + half * 4;
    uint4 o;
    o.x = interleave_nibbles(src[0]);
    o.y = interleave_nibbles(src[1]);
    o.z = interleave_nibbles(src[2]);
    o.w = interleave_nibbles(src[3]);
    *reinterpret_cast<uint4*>(blk + half * 2048 + l * 16) = o;

    if (t < 128) {
        int r2 = t, m2 = 0, row2;
        if (a.gateup) {
            m2 = ((r2 & 31) >= 16) ? 1 : 0;
            row2 = 64 * mt + 16 * (r2 >> 5) + (r2 & 15);
        } else {
            row2 = 128 * mt + r2;
        }
        const uint16_t* s2 = shared ? a.ss[m2] : a.s[m2] + (size_t)g * mat_groups;
        const uint16_t* b2 = shared ? a.bs[m2] : a.b[m2] + (size_t)g * mat_groups;
        const size_t gi = (size_t)row2 * (cols / 64) + c;
        const uint32_t sh = bf16_to_fp16_bits(s2[gi], a.inexact);
        {   // the tensor-core dequantisation also uses s / 16, exact in fp16 only for |s| >= 2^-13
            const float sf = fabsf(__half2float(__ushort_as_half((unsigned short)sh)));
            if (sf != 0.f && sf < 0.0001220703125f) atomicOr(a.inexact, 1u);
        }
        const uint32_t bh = bf16_to_fp16_bits(b2[gi], a.inexact);
        *reinterpret_cast<uint32_t*>(blk + kBlockCodeBytes + 4 * r2) = sh | (bh << 16);
    }
}

// Router weights: transposed fp32 copy [H][E] (coalesced per-expert reads in the SIMT router),
// bias (zeros when absent) and the shared-gate vector (zeros when absent).
__global__ void router_prep_kernel(const float* __restrict__ router, const float* __restrict__ bias,
                                   const float* __restrict__ sgw, int H, int E, float* __restrict__ wrt,
                                   float* __restrict__ bias_out, float* __restrict__ sgw_out) {
    const size_t n = (size_t)H * E;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const size_t h = i / E, e = i % E;
        wrt[i] = router[e * H + h];
    }
    if (blockIdx.x == 0) {
        for (int e = threadIdx.x; e < E; e += blockDim.x) bias_out[e] = bias ? bias[e] : 0.f;
        for (int h = threadIdx.x; h < H; h += blockDim.x) sgw_out[h] = sgw ? sgw[h] : 0.f;
    }
}

cudaError_t launch_repack(const RepackArgs& a, int groups, int m_tiles, int k_steps, cudaStream_t st) {
    dim3 grid(k_steps, m_tiles, groups);
    repack_kernel<<<grid, 256, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_router_prep(const float* router, const float* bias, const float* sgw, int H, int E,
                               float* wrt, float* bias_out, float* sgw_out, cudaStream_t st) {
    router_prep_kernel<<<256, 256, 0, st>>>(router, bias, sgw, H, E, wrt, bias_out, sgw_out);
    return cudaGetLastError();
}

// One block (g, mt, kc) per CTA of 256 threads; thread = (row, column half).  The same fp16
// arithmetic as the grouped GEMM's transform (exact for this format).
__global__ void __launch_bounds__(256) dequant_rows_kernel(const uint8_t* __restrict__ blocks, int m_tiles,
                                                           int k_steps, __half* __restrict__ dst) {
    const int kc = blockIdx.x, mt = blockIdx.y, g = blockIdx.z;
    const int row = threadIdx.x & 127, half = threadIdx.x >> 7;
    const uint8_t* blk = blocks + (((size_t)g * m_tiles + mt) * k_steps + kc) * kBlockBytes;
    const uint4 cw = *reinterpret_cast<const uint4*>(blk + half * 2048 + row * 16);
    const uint32_t sb = *reinterpret_cast<const uint32_t*>(blk + kBlockCodeBytes + row * 4);
    const __half2 s2 = __half2(__ushort_as_half((unsigned short)(sb & 0xFFFFu)), __ushort_as_half((unsigned short)(sb & 0xFFFFu)));
    const __half2 b2 = __half2(__ushort_as_half((unsigned short)(sb >> 16)), __ushort_as_half((unsigned short)(sb >> 16)));
    const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
    uint32_t out[16];
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int sft = 0; sft < 4; ++sft) {   // columns 8w + 2 sft, +1 of this half
            const __half2 v = __hfma2(codes_to_half2(words[w], sft), s2, b2);
            out[4 * w + sft] = *reinterpret_cast<const uint32_t*>(&v);
        }
    uint4* d = reinterpret_cast<uint4*>(dst + (((size_t)g * m_tiles + mt) * 128 + row) * (size_t)(64 * k_steps) +
                                        64 * kc + 32 * half);
#pragma unroll
    for (int i = 0; i < 4; ++i) d[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
}

cudaError_t launch_dequant_rows(const uint8_t* blocks, int groups, int m_tiles, int k_steps, __half* dst,
                                cudaStream_t st) {
    dequant_rows_kernel<<<dim3(k_steps, m_tiles, groups), 256, 0, st>>>(blocks, m_tiles, k_steps, dst);
    return cudaGetLastError();
}

}  // namespace moe
