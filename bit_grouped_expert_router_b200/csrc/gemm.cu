// gemm.cu -- prefill grouped GEMMs on the 5th-generation tensor core (tcgen05 + TMEM + TMA).
//
// "Perplexity Open-Sources Lily..." section "The optimizations follow the workload": the 4-bit
// weights are reconstructed inside the grouped matrix multiplication rather than expanded into a
// full weight array in memory.  Here that reconstruction lands in tensor memory: per pipeline
// stage a bulk copy brings one 4608-byte block of packed codes + fp16 scale/bias (128 weight rows
// x 64 input columns) into shared memory, four "transform" warps turn it into fp16 weights (exact
// for this format, see common.cuh) and store them with tcgen05.st into a TMEM stage, and one
// thread issues tcgen05.mma with the weights as the TMEM A operand and the tokens' activations as
// the shared-memory B operand (TMA tile load, 128-byte swizzle).  Swap-AB: M = 128 weight rows,
// N = up to 128 tokens of one expert, so experts with few tokens still fill the M dimension.
//
//   gate/up kernel : per tile (expert, 128 interleaved gate/up rows, <=128 tokens), K = H.
//                    Epilogue: act = silu(G) * U (G and U of one column i sit 16 TMEM lanes apart
//                    in the same warp, paired with one shuffle), fp16, staged in shared memory and
//                    written to the expert's act rows (only the tile's valid tokens).
//   down kernel    : per tile (expert, 128 output rows, <=128 tokens), K = I.
//                    Epilogue: y * gate (routing gate, or sigmoid gate for the shared expert)
//                    reduced with fp32 atomics (red.global.add) into the token's accumulator row.
//
// Warp roles (320 threads, one persistent CTA per SM, tiles taken round-robin from the device-
// built tile list so no tile count ever travels to the host):
//   warp 0      TMA producer (one lane)
//   warp 1      TMEM allocator + MMA issuer (one lane)
//   warps 2-5   transform: dequantise a stage into TMEM (warp w owns TMEM lanes 32*(w%4)..+31)
//   warps 6-9   epilogue: drain a TMEM accumulator (double-buffered, so it overlaps the next tile)
// TMEM columns: [0,128) and [128,256) accumulators, [256, 256+32*kStages) fp16 A stages.
// Every wait is bounded (common.cuh); on a timeout the roles unwind, the producer waits for its
// copies in flight, the MMA thread waits for its MMAs, and warp 1 frees the TMEM.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kThreads = 320;
constexpr int kTmemCols = 512;
constexpr int kAccCols = kBN;
constexpr int kACol0 = 2 * kAccCols;
static_assert(kACol0 + 32 * kStages <= kTmemCols, "TMEM budget");
static_assert(kBN % 32 == 0 && kBN <= 256, "tile N");

constexpr int kBTileBytes = kBN * 128;  // kBN rows x 64 fp16
constexpr int kOffB = 0;
constexpr int kOffW = kOffB + kStages * kBTileBytes;
constexpr int kOffStage = kOffW + kStages * kBlockBytes;
constexpr int kStageBytes = kBN * 128;  // act staging: kBN rows x 64 fp16
constexpr int kOffMeta = kOffStage + kStageBytes;
constexpr int kMetaBytes = 2 * kBN * 8;  // [2 buffers][kBN] token + gate
constexpr int kOffBar = kOffMeta + kMetaBytes;
constexpr int kNumBars = 3 * kStages + 5;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
static_assert(kOffW % 16 == 0 && kOffStage % 16 == 0 && kOffMeta % 16 == 0 && kOffBar % 8 == 0, "align");

__device__ __forceinline__ float silu_mul(float g, float u) { return g * u / (1.f + __expf(-g)); }

template <bool GATEUP>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_kernel(Ctx c, const __grid_constant__ CUtensorMap tmB) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* bsm = smem + kOffB;
    uint8_t* wsm = smem + kOffW;
    __half* stage = reinterpret_cast<__half*>(smem + kOffStage);
    int* meta_tok = reinterpret_cast<int*>(smem + kOffMeta);
    float* meta_gate = reinterpret_cast<float*>(smem + kOffMeta + 2 * kBN * 4);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* full = bars;                  // TMA data landed           (1 arrive + tx)
    uint64_t* afull = bars + kStages;       // fp16 A stage in TMEM      (128 arrives)
    uint64_t* empty = bars + 2 * kStages;   // MMAs of the stage done    (commit)
    uint64_t* accfull = bars + 3 * kStages; // accumulator ready         (commit)
    uint64_t* accempty = accfull + 2;       // accumulator drained       (128 arrives)
    uint64_t* drainbar = accfull + 4;       // MMA drain on abort        (commit)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int MT = GATEUP ? c.I / 64 : c.H / 128;   // weight m-tiles (128 rows each)
    const int KS = GATEUP ? c.H / 64 : c.I / 64;    // k-steps (one 64-column group each)
    const uint8_t* wbase = GATEUP ? c.w_gu : c.w_dn;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&afull[s], 128);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accfull[b], 1);
            mbar_init(&accempty[b], 128);
        }
        mbar_init(drainbar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int total = c.ntiles[0] * MT;

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0 && !(c.flags & 0x100u)) {
            uint32_t it = 0;
            for (int tau = blockIdx.x; tau < total; tau += gridDim.x) {
                const int4 tile = c.tiles1[tau / MT];
                const int mt = tau % MT;
                if (tile.x < 0 || tile.x >= c.G || tile.y < 0 || tile.y + tile.z > c.rows_cap) continue;
                const uint8_t* wsrc = wbase + ((size_t)tile.x * MT + mt) * KS * kBlockBytes;
                for (int kc = 0; kc < KS; ++kc, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, c.status)) goto producer_done;
                    mbar_arrive_expect_tx(&full[s], kBlockBytes + kBTileBytes);
                    bulk_g2s(wsm + s * kBlockBytes, wsrc + (size_t)kc * kBlockBytes, kBlockBytes, &full[s]);
                    tma_load_2d(bsm + s * kBTileBytes, &tmB, kc * 64, tile.y, &full[s]);
                }
            }
        producer_done:
            // every copy issued must land before the CTA may exit
            const uint32_t first = it > (uint32_t)kStages ? it - kStages : 0u;
            for (uint32_t i = first; i < it; ++i) mbar_drain(&full[i % kStages], (i / kStages) & 1u);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t it = 0, tl = 0;
            bool issued = false;
            for (int tau = blockIdx.x; tau < total; tau += gridDim.x, ++tl) {
                const int4 tile = c.tiles1[tau / MT];
                if (tile.x < 0 || tile.x >= c.G || tile.y < 0 || tile.y + tile.z > c.rows_cap) {
                    if (tau % MT == 0) set_status(c.status, MOE_STATUS_BOUNDS);
                    --tl;
                    continue;
                }
                const int n_inst = max(16, ((tile.z + 15) / 16) * 16);
                const uint32_t idesc = idesc_f16(128, n_inst, false);
                const uint32_t ab = tl & 1u, aph = (tl >> 1) & 1u;
                if (!mbar_wait(&accempty[ab], aph ^ 1u, abort_flag, c.status)) goto mma_done;
                tc_fence_after();
                const uint32_t d_tmem = tmem + ab * kAccCols;
                for (int kc = 0; kc < KS; ++kc, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!mbar_wait(&afull[s], ph, abort_flag, c.status)) goto mma_done;
                    if (!mbar_wait(&full[s], ph, abort_flag, c.status)) goto mma_done;
                    tc_fence_after();
                    const uint32_t b_addr = smem_u32(bsm + s * kBTileBytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        mma_ts(d_tmem, tmem + kACol0 + 32 * s + 8 * kk, sdesc_sw128(b_addr + 32 * kk), idesc,
                               (kc | kk) != 0 ? 1u : 0u);
                    }
                    issued = true;
                    tc_commit(&empty[s]);
                }
                tc_commit(&accfull[ab]);
            }
        mma_done:
            if (*abort_flag && issued) {
                tc_commit(drainbar);
                mbar_drain(drainbar, 0);
            }
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------------ transform
        const int q = warp & 3;
        const int row = 32 * q + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        uint32_t it = 0;
        for (int tau = blockIdx.x; tau < total; tau += gridDim.x) {
            const int4 tile = c.tiles1[tau / MT];
            if (tile.x < 0 || tile.x >= c.G || tile.y < 0 || tile.y + tile.z > c.rows_cap) continue;
            for (int kc = 0; kc < KS; ++kc, ++it) {
                const int s = it % kStages;
                const uint32_t ph = (it / kStages) & 1u;
                if (!mbar_wait(&full[s], ph, abort_flag, c.status)) goto transform_done;
                const uint8_t* blk = wsm + s * kBlockBytes;
                const uint4 c0 = *reinterpret_cast<const uint4*>(blk + row * 16);
                const uint4 c1 = *reinterpret_cast<const uint4*>(blk + 2048 + row * 16);
                const uint32_t sb = *reinterpret_cast<const uint32_t*>(blk + kBlockCodeBytes + row * 4);
                const __half2 s2 = __half2(__ushort_as_half((unsigned short)(sb & 0xFFFFu)),
                                           __ushort_as_half((unsigned short)(sb & 0xFFFFu)));
                const __half2 b2 = __half2(__ushort_as_half((unsigned short)(sb >> 16)),
                                           __ushort_as_half((unsigned short)(sb >> 16)));
                const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
                uint32_t r[32];
#pragma unroll
                for (int w = 0; w < 8; ++w) {
#pragma unroll
                    for (int sft = 0; sft < 4; ++sft) {
                        const __half2 v = __hfma2(codes_to_half2(words[w], sft), s2, b2);
                        r[4 * w + sft] = *reinterpret_cast<const uint32_t*>(&v);
                    }
                }
                tmem_st32(tmem + lane_base + kACol0 + 32 * s, r);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&afull[s]);
            }
        }
    transform_done:;
    } else {
        // ------------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int etid = threadIdx.x - 192;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        uint32_t tl = 0;
        bool range_bad = false;
        for (int tau = blockIdx.x; tau < total; tau += gridDim.x, ++tl) {
            const int4 tile = c.tiles1[tau / MT];
            const int mt = tau % MT;
            if (tile.x < 0 || tile.x >= c.G || tile.y < 0 || tile.y + tile.z > c.rows_cap) {
                --tl;
                continue;
            }
            const int row0 = tile.y, nvalid = tile.z;
            const uint32_t ab = tl & 1u, aph = (tl >> 1) & 1u;
            if (!GATEUP) {
                if (etid < nvalid) {
                    meta_tok[ab * kBN + etid] = c.row_token[row0 + etid];
                    meta_gate[ab * kBN + etid] = c.row_gate[row0 + etid];
                }
                named_bar(1, 128);
            }
            if (!mbar_wait(&accfull[ab], aph, abort_flag, c.status)) goto epilogue_done;
            tc_fence_after();
            const uint32_t taddr = tmem + lane_base + ab * kAccCols;
            if (GATEUP) {
                const int ilocal = 16 * q + (lane & 15);
                const bool is_gate = lane < 16;
                for (int c0 = 0; c0 < nvalid; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(taddr + c0, v);
#pragma unroll
                    for (int r = 0; r < 16; ++r) {
                        const float mine_lo = __uint_as_float(v[r]);
                        const float mine_hi = __uint_as_float(v[16 + r]);
                        const float recv = __shfl_xor_sync(0xffffffffu, is_gate ? mine_hi : mine_lo, 16);
                        const float G = is_gate ? mine_lo : recv;
                        const float U = is_gate ? recv : mine_hi;
                        const int col = c0 + r + (is_gate ? 0 : 16);
                        const float a = silu_mul(G, U);
                        if (col < nvalid && !(fabsf(a) <= 65504.f)) range_bad = true;
                        stage[col * 64 + ilocal] = __float2half_rn(a);  // columns >= nvalid: not copied out
                    }
                }
                tc_fence_before();
                mbar_arrive(&accempty[ab]);
                named_bar(1, 128);
                const size_t I = (size_t)c.I;
                for (int idx = etid; idx < nvalid * 8; idx += 128) {
                    const int j = idx >> 3, ch = idx & 7;
                    *reinterpret_cast<uint4*>(c.act + (size_t)(row0 + j) * I + mt * 64 + ch * 8) =
                        *reinterpret_cast<const uint4*>(stage + j * 64 + ch * 8);
                }
                named_bar(1, 128);
            } else {
                const int h = mt * 128 + 32 * q + lane;
                float* accp = c.acc + h;
                for (int c0 = 0; c0 < nvalid; c0 += 32) {
                    uint32_t v[32];
                    tmem_ld32(taddr + c0, v);
#pragma unroll
                    for (int r = 0; r < 32; ++r) {
                        const int j = c0 + r;
                        if (j < nvalid) {
                            const float y = __uint_as_float(v[r]) * meta_gate[ab * kBN + j];
                            const int tok = meta_tok[ab * kBN + j];
                            asm volatile("red.global.add.f32 [%0], %1;" ::"l"(accp + (size_t)tok * c.H), "f"(y)
                                         : "memory");
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(&accempty[ab]);
            }
        }
    epilogue_done:
        if (range_bad) set_status(c.status, MOE_STATUS_RANGE);
    }

    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

int gemm_smem_bytes(bool) { return kSmemBytes; }

cudaError_t launch_gemm_gateup(const Ctx& c, const CUtensorMap& tm_xp, int num_sms, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes);
    if (e != cudaSuccess) return e;
    grouped_gemm_kernel<true><<<num_sms, kThreads, kSmemBytes, st>>>(c, tm_xp);
    return cudaGetLastError();
}

cudaError_t launch_gemm_down(const Ctx& c, const CUtensorMap& tm_act, int num_sms, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes);
    if (e != cudaSuccess) return e;
    grouped_gemm_kernel<false><<<num_sms, kThreads, kSmemBytes, st>>>(c, tm_act);
    return cudaGetLastError();
}

// out[t][h] = bf16(acc[t][h]), round to nearest even; 8 elements per thread per step.
__global__ void __launch_bounds__(256) finalize_kernel(Ctx c) {
    const size_t n8 = (size_t)c.T * c.H / 8;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
        const float4 a = reinterpret_cast<const float4*>(c.acc)[2 * i];
        const float4 b = reinterpret_cast<const float4*>(c.acc)[2 * i + 1];
        __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x, a.y), p1 = __floats2bfloat162_rn(a.z, a.w);
        __nv_bfloat162 p2 = __floats2bfloat162_rn(b.x, b.y), p3 = __floats2bfloat162_rn(b.z, b.w);
        uint4 o;
        o.x = *reinterpret_cast<uint32_t*>(&p0);
        o.y = *reinterpret_cast<uint32_t*>(&p1);
        o.z = *reinterpret_cast<uint32_t*>(&p2);
        o.w = *reinterpret_cast<uint32_t*>(&p3);
        reinterpret_cast<uint4*>(c.out)[i] = o;
    }
}

cudaError_t launch_finalize(const Ctx& c, cudaStream_t st) {
    const size_t n8 = (size_t)c.T * c.H / 8;
    const int blocks = (int)((n8 + 255) / 256 < 148 * 8 ? (n8 + 255) / 256 : 148 * 8);
    finalize_kernel<<<blocks > 0 ? blocks : 1, 256, 0, st>>>(c);
    return cudaGetLastError();
}

}  // namespace moe
