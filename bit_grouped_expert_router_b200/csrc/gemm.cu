// gemm.cu -- prefill grouped GEMMs on the 5th-generation tensor core (tcgen05 + TMEM + TMA).
//
// "Perplexity Open-Sources Lily..." section "The optimizations follow the workload": the 4-bit
// weights are reconstructed inside the grouped matrix multiplication rather than expanded into a
// full weight array in memory.  Here one bulk copy brings kWB 4608-byte blocks of packed codes +
// fp16 scale/bias (128 weight rows x kWB x 64 input columns) into shared memory, the "transform"
// warps turn each block into an fp16 tile (exact for this format, see common.cuh) written straight
// into the tensor core's 128-byte-swizzled K-major operand layout, and one thread issues
// tcgen05.mma with that tile as A and a TMA tile of the expert's token rows as B, accumulating in
// tensor memory.  Swap-AB: M = 128 weight rows, N = up to kBN (256 or 128) tokens of one expert, so
// experts with few tokens still fill the M dimension.  The dequantised weights exist only in
// shared memory.
//
// Shaped by measurement on this part: every TMA operation costs an SM at least ~360 cycles
// whatever its size, while big copies stream at ~90 B/clk.  So the weight blocks travel several
// k-steps per copy, the token tile is a single box per k-step whose height (64/128/256 rows)
// follows the tile's token count, and the weight ring is sized apart from the operand stages:
//   weight ring     kWS stages x kWB blocks               (weight producer -> transform)
//   operand stages  kBS x (kBN x 64 tokens + 128 x 64 A)  (producer + transform -> MMA)
// A stage's token tile and A tile share one full and one empty barrier, so the MMA-issuing thread
// takes one wait and one commit per k-step.  Barrier arrivals are one per warp.
//
//   gate/up kernel : per tile (expert, 128 interleaved gate/up rows, <= kBN tokens), K = H.
//                    B = the expert's bucketed fp16 token rows (the shared expert reads the fp16
//                    activations directly: its rows are all tokens in order).  Epilogue:
//                    act = silu(G) * U (G and U of one column i sit 16 TMEM lanes apart in the
//                    same warp, paired with one shuffle), fp16, staged in shared memory and written
//                    to the expert's act rows (only the tile's valid tokens).
//   down kernel    : per tile (expert, 128 output rows, <= kBN tokens), K = I.  B = act rows.
//                    Epilogue: y * gate (routing gate, or sigmoid gate for the shared expert) added
//                    into the token's fp32 accumulator row.  A warp's block (32 output rows = TMEM
//                    lanes x 16 or 32 tokens) is transposed through shared memory so that each
//                    lane adds 4 consecutive rows of one token with one red.global.add.v4.f32 (8
//                    lanes cover a token's 128 contiguous bytes): a quarter of the reduction
//                    instructions of one scalar red per element, which made the down GEMM ~30 %
//                    faster on this part (the scalar form was bound by the epilogue's issue).
//
// Warp roles (GemmCfg; tiles taken round-robin from the device-built tile list so no tile count
// ever travels to the host).  kE epilogue warps: 4 for gate/up and the two-CTA shape, 16 for the
// one-CTA down GEMM.
//   warp 0      token-tile TMA producer (lane 0)
//   warp 1      TMEM allocator + MMA issuer (one lane)
//   epilogue    warps 2 .. 2+kE-1: drain a TMEM accumulator (double-buffered, so it overlaps the
//               next tile; warp w reads TMEM lanes 32*(w%4)..+31, the warps of a lane quarter take
//               alternate column chunks)
//   transform   the next warps not on scheduler 1 (warp % 4 != 1), 8 (or 4 in the two-CTA shape),
//               in groups taking alternate k-steps: dequantise a block into the A ring
//   the first warp left on scheduler 1 issues the weight-block copies (lane 0); one more idles.
// One CTA per SM: 512 threads for gate/up, 896 for down, 256-token tiles; two per SM: 352
// threads, 128-token tiles.
// TMEM: two fp32 accumulators of kBN columns.  Every wait is bounded (common.cuh); on a timeout the
// roles unwind, the producer waits for its copies in flight, the MMA thread waits for its MMAs,
// and warp 1 frees the TMEM.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

// Two launch shapes of the same kernel.  CTAS = 1: one CTA per SM (512 threads for gate/up, 896
// for down), 256-token tiles, 3 operand stages and 4-block weight copies.  CTAS = 2: two 352-thread
// CTAs per SM (half the roles and half the TMEM each), 128-token tiles, 2 stages and 2-block
// copies.  A k-step costs about the same whatever the tile's token count (a ring of hand-offs
// between the producers, the transform groups and the MMA-issuing thread), so when experts get
// few tokens (tiles far from full) two independent rings per SM win; when tiles are full, the
// larger tile's fewer k-steps win (host picks per call).
template <int CTAS, bool GATEUP = true>
struct GemmCfg {
    static_assert(CTAS == 1 || CTAS == 2, "CTAs per SM");
    static constexpr int kBN = CTAS == 1 ? 256 : 128;   // token columns per tile (= UMMA N)
    // The one-CTA down GEMM takes 4 epilogue warps per TMEM lane quarter: its combine epilogue
    // (transpose + vector reductions) of a full 256-token tile outlasts a unit's MMAs with 2, and
    // the MMA thread then waits for the accumulator (measured: 2 -> 3 -> 4 per quarter, down
    // 139.3 -> 134.3 -> 130.8 us per 4096-token chunk; 5 would cap the registers at 64).  The
    // gate/up epilogue (SwiGLU, ~1/3 of a unit's time with one warp per quarter) needs one; fewer
    // warps beside the transform warps: gate/up 189.7 -> 188.6 us against two per quarter.
    static constexpr int kEpiWarps = CTAS == 1 && !GATEUP ? 16 : 4;
    static constexpr int kDnChunk = kEpiWarps > 8 ? 16 : 32;   // down epilogue: tokens per chunk
    static constexpr int kTransformWarps = 8 / CTAS;
    // Warp roles, placed by scheduler (warp % 4): the MMA-issuing warp 1 must not share its
    // scheduler with the busy transform warps (measured: a tcgen05.mma issue took ~110 cycles
    // when it did, against ~45 alone), so the epilogue warps (idle between tiles) take warps
    // 2 .. 2 + kEpiWarps - 1 and the transform warps the following warps whose index is not 1
    // mod 4; the first of those left over issues the weight copies (a thread that mostly sleeps
    // in mbarrier waits), the other stays idle.
    static constexpr int kEpiWarp0 = 2;
    static constexpr int kXWarp0 = 2 + kEpiWarps;   // first transform-candidate warp
    static constexpr int kXCand = kTransformWarps + (kTransformWarps - 1) / 3;   // skipping every 4th
    static constexpr int kThreads = 32 * (kXWarp0 + kXCand);
    static constexpr int kTmemCols = 512 / CTAS;
    static constexpr int kAccCols = kBN;
    static constexpr int kWB = CTAS == 1 ? 4 : 2;   // weight blocks per bulk copy
    static constexpr int kWS = 2;                   // weight ring stages
    static constexpr int kBS = CTAS == 1 ? 3 : 2;   // operand stages (one token tile + one A tile each)
    static constexpr int kAS = kBS;
    static constexpr int kATileBytes = 128 * 128;   // 128 weight rows x 64 fp16
    static constexpr int kBTileBytes = kBN * 128;   // up to kBN token rows x 64 fp16
    static constexpr int kWStageBytes = kWB * kBlockBytes;
    static constexpr int kOffA = 0;
    static constexpr int kOffB = kOffA + kAS * kATileBytes;
    static constexpr int kOffW = kOffB + kBS * kBTileBytes;
    static constexpr int kOffStage = kOffW + kWS * kWStageBytes;
    static constexpr int kStageBytes = kBN * 128;   // gate/up: kBN x 64 fp16 act; down: 32 x 32 fp32 per epilogue warp
    static constexpr int kOffMeta = kOffStage + kStageBytes;
    static constexpr int kMetaBytes = 2 * kBN * 16; // [2 buffers][kBN] row pointer + gate (+ pad)
    static constexpr int kOffBar = kOffMeta + kMetaBytes;
    static constexpr int kNumBars = 2 * (kWS + kBS) + 5;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
    static_assert(kBN <= moe::kBN, "tile lists are sized for at most kBN rows per tile");
    static_assert(2 * kAccCols <= kTmemCols, "TMEM budget");
    static_assert(kStageBytes >= kEpiWarps * kDnChunk * 32 * 4, "down epilogue: one chunk x 32 fp32 block per warp");
    static_assert(kOffB % 1024 == 0 && kOffW % 16 == 0 && kOffStage % 16 == 0 && kOffMeta % 16 == 0 &&
                      kOffBar % 8 == 0,
                  "align");
    static_assert(kSmemBytes * CTAS <= 227 * 1024, "shared memory budget");
};

// silu(g) * u with the fast divide (a reciprocal and a multiply, within 2 ulp; the result is
// rounded to fp16 next); a denominator past 2^126 (g < -87) gives 0, the limit of silu there
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g * u, 1.f + __expf(-g)); }

// tcgen05.ld, shape 32x32b, 16 columns: thread i of the warp reads TMEM lane (warp's quarter base +
// i), registers r[j] = columns col..col+15 (the wait names the registers so no use moves above it).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15])
                 :
                 : "memory");
}

__device__ __forceinline__ bool tile_ok(const int4& t, const Ctx& c, int bn) {
    return t.x >= 0 && t.x < c.G && t.y >= 0 && t.z > 0 && t.z <= bn && t.y + t.z <= c.rows_cap;
}

// AHBM: the ablation variant that reads A as fp16 weights dequantised once into HBM (one 2-D TMA
// tile per k-step, box 64 columns x 128 rows, the same 128-byte swizzle the transform writes)
// instead of rebuilding it from the 4-bit blocks in shared memory; the transform warps idle.
template <bool GATEUP, int CTAS, bool AHBM>
__global__ void __launch_bounds__(GemmCfg<CTAS, GATEUP>::kThreads, CTAS)
    grouped_gemm_kernel(Ctx c, const __grid_constant__ TokenMaps maps, const __grid_constant__ CUtensorMap amap) {
    griddep_wait();
    griddep_launch_dependents();
    using K = GemmCfg<CTAS, GATEUP>;
    constexpr int kBN = K::kBN, kEpiWarps = K::kEpiWarps, kTransformWarps = K::kTransformWarps;
    constexpr int kEpiWarp0 = K::kEpiWarp0, kTmemCols = K::kTmemCols, kAccCols = K::kAccCols;
    constexpr int kWB = K::kWB, kWS = K::kWS, kBS = K::kBS, kAS = K::kAS;
    constexpr int kATileBytes = K::kATileBytes, kBTileBytes = K::kBTileBytes, kWStageBytes = K::kWStageBytes;
    constexpr int kOffA = K::kOffA, kOffB = K::kOffB, kOffW = K::kOffW, kOffStage = K::kOffStage;
    constexpr int kOffMeta = K::kOffMeta, kOffBar = K::kOffBar, kOffMisc = K::kOffMisc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* asm_ = smem + kOffA;
    uint8_t* bsm = smem + kOffB;
    uint8_t* wsm = smem + kOffW;
    __half* stage = reinterpret_cast<__half*>(smem + kOffStage);
    float** meta_row = reinterpret_cast<float**>(smem + kOffMeta);
    float* meta_gate = reinterpret_cast<float*>(smem + kOffMeta + 2 * kBN * 8);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* wfull = bars;                 // weight blocks landed          (1 arrive + tx)
    uint64_t* wempty = wfull + kWS;         // weight blocks consumed        (1 arrive per transform warp)
    // One barrier pair per operand stage: the stage is full when its token tile has landed (the
    // producer's arrive + tx) and its A tile is written (one arrive per warp of the transform group
    // that took the k-step, or the A
    // tile's tx as well when A comes from HBM), and empty when its MMAs are done (one commit).
    // The MMA thread thus takes one wait and one commit per k-step.
    uint64_t* sfull = wempty + kWS;         // stage's token + A tiles ready (1 + 4 transform arrives, + tx)
    uint64_t* sempty = sfull + kBS;         // stage's MMAs done             (commit)
    uint64_t* accfull = sempty + kBS;       // accumulator ready             (commit)
    uint64_t* accempty = accfull + 2;       // accumulator drained           (1 arrive per epilogue warp)
    uint64_t* drainbar = accfull + 4;       // MMA drain on abort            (commit)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int MT = GATEUP ? c.I / 64 : c.H / 128;   // weight m-tiles (128 rows each)
    const int KS = GATEUP ? c.H / 64 : c.I / 64;    // k-steps (one 64-column group each)
    const uint8_t* wbase = GATEUP ? c.w_gu : c.w_dn;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kWS; ++s) {
            mbar_init(&wfull[s], 1);
            mbar_init(&wempty[s], kTransformWarps);
        }
        for (int s = 0; s < kBS; ++s) {
            mbar_init(&sfull[s], AHBM ? 1 : 1 + (CTAS == 1 ? 4 : 2));   // the producer, the k-step's transform group
            mbar_init(&sempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accfull[b], 1);
            mbar_init(&accempty[b], kEpiWarps);
        }
        mbar_init(drainbar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        for (int i = 0; i < 2; ++i)
            for (int j = 0; j < 3; ++j) prefetch_tmap(&maps.m[i][j]);
        if (AHBM) prefetch_tmap(&amap);
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
        // Lane 0 waits for ring slots and issues the copies (the rest of the warp follows along).
        if (!(c.flags & 0x100u)) {
            const int shared_base = (GATEUP && c.has_shared) ? c.offsets[c.E] : 0;
            uint32_t bit = 0;
            int bs = 0;
            uint32_t bph = 0;
            for (int tau = blockIdx.x; tau < total; tau += gridDim.x) {
                const int4 tile = c.tiles1[tau / MT];
                const int mt = tau % MT;
                if (!tile_ok(tile, c, kBN)) continue;
                const int n_inst = max(16, ((tile.z + 15) / 16) * 16);
                const int hsel = n_inst <= 64 ? 0 : (n_inst <= 128 ? 1 : 2);
                const bool from_x = GATEUP && c.has_shared && tile.x == c.E;   // shared expert: token order
                const CUtensorMap* map = &maps.m[from_x ? 1 : 0][hsel];
                const int y = from_x ? tile.y - shared_base : tile.y;
                const uint32_t b_bytes = (uint32_t)token_box_rows(hsel) * 128;
                for (int kc = 0; kc < KS; ++kc) {
                    int ok = 1;
                    if (lane == 0) {
                        ok = mbar_wait(&sempty[bs], bph ^ 1u, abort_flag, c.status) ? 1 : 0;
                        if (ok) {
                            mbar_arrive_expect_tx(&sfull[bs], b_bytes + (AHBM ? (uint32_t)kATileBytes : 0u));
                            if (AHBM)   // the fp16 A tile of this k-step from HBM
                                tma_load_2d(asm_ + bs * kATileBytes, &amap, kc * 64, (tile.x * MT + mt) * 128, &sfull[bs]);
                            tma_load_2d(bsm + bs * kBTileBytes, map, kc * 64, y, &sfull[bs]);
                            ++bit;
                            if (++bs == kBS) { bs = 0; bph ^= 1u; }
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) goto producer_done;
                }
            }
        producer_done:
            // every copy issued must land before the CTA may exit (after an abort the transform
            // warps may have left without their arrivals; the bounded drain then waits out its
            // limit, far longer than any copy takes to land)
            if (lane == 0) {
                for (uint32_t i = bit > (uint32_t)kBS ? bit - kBS : 0u; i < bit; ++i)
                    mbar_drain(&sfull[i % kBS], (i / kBS) & 1u);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t tl = 0;
            int bs = 0;
            uint32_t bph = 0;
            bool issued = false;
            const uint32_t a0 = smem_u32(asm_), b0 = smem_u32(bsm);
            for (int tau = blockIdx.x; tau < total; tau += gridDim.x) {
                const int4 tile = c.tiles1[tau / MT];
                if (!tile_ok(tile, c, kBN)) {
                    if (tau % MT == 0) set_status(c.status, MOE_STATUS_BOUNDS);
                    continue;
                }
                const int n_inst = max(16, ((tile.z + 15) / 16) * 16);
                const uint32_t idesc = idesc_f16(128, n_inst, false);
                const uint32_t ab = tl & 1u, acph = (tl >> 1) & 1u;
                if (!mbar_wait(&accempty[ab], acph ^ 1u, abort_flag, c.status)) goto mma_done;
                const uint32_t d_tmem = tmem + ab * kAccCols;
                for (int kc = 0; kc < KS; ++kc) {
                    if (!mbar_wait(&sfull[bs], bph, abort_flag, c.status)) goto mma_done;
                    tc_fence_after();
                    // descriptors of the stage once; the kk-th 16-column slice starts 32 bytes on,
                    // i.e. +2 in the start-address field (no carry: shared addresses < 256 KB)
                    const uint64_t ad = sdesc_sw128(a0 + bs * kATileBytes), bd = sdesc_sw128(b0 + bs * kBTileBytes);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kc | kk) != 0 ? 1u : 0u);
                    issued = true;
                    tc_commit(&sempty[bs]);
                    if (++bs == kBS) { bs = 0; bph ^= 1u; }
                }
                tc_commit(&accfull[ab]);
                ++tl;
            }
        mma_done:
            if (*abort_flag && issued) {
                tc_commit(drainbar);
                mbar_drain(drainbar, 0);
            }
        }
    } else if (warp == K::kXWarp0 + 3) {
        // ------------------------------------------------------------------ weight producer
        // Lane 0 refills each weight stage as soon as the transform warps release it, so the
        // 4-bit blocks run up to kWS * kWB k-steps ahead of the transform whatever the token
        // ring's state (sharing the token producer's thread tied their lead to the token ring's).
        if (!AHBM && !(c.flags & 0x100u) && lane == 0) {
            uint32_t wit = 0, wph = 0;
            int ws = 0;
            for (int tau = blockIdx.x; tau < total; tau += gridDim.x) {
                const int4 tile = c.tiles1[tau / MT];
                const int mt = tau % MT;
                if (!tile_ok(tile, c, kBN)) continue;
                const uint8_t* wsrc = wbase + ((size_t)tile.x * MT + mt) * KS * kBlockBytes;
                for (int kc = 0; kc < KS; kc += kWB) {
                    const int nb = min(kWB, KS - kc);
                    if (!mbar_wait(&wempty[ws], wph ^ 1u, abort_flag, c.status)) goto wproducer_done;
                    mbar_arrive_expect_tx(&wfull[ws], (uint32_t)nb * kBlockBytes);
                    bulk_g2s(wsm + ws * kWStageBytes, wsrc + (size_t)kc * kBlockBytes, (uint32_t)nb * kBlockBytes,
                             &wfull[ws]);
                    ++wit;
                    if (++ws == kWS) { ws = 0; wph ^= 1u; }
                }
            }
        wproducer_done:
            // every copy issued must land before the CTA may exit
            for (uint32_t i = wit > (uint32_t)kWS ? wit - kWS : 0u; i < wit; ++i)
                mbar_drain(&wfull[i % kWS], (i / kWS) & 1u);
        }
    } else if (warp >= K::kXWarp0) {
        // ------------------------------------------------------------------ transform
        // Groups of 4 warps, thread = weight row (both 64-column halves); with two groups (the
        // one-CTA shape) they take alternate k-steps, so each warp converts a whole A tile's rows
        // every second k-step and its waits, proxy fence and arrival serve twice the weights (the
        // same per-warp work as in the two-CTA shape, whose k-steps per SM ran ~1.5x faster).
        // The fp16 pairs of 16-byte chunk ch of row r go to r*128 + ((ch ^ (r & 7)) * 16), the
        // 128-byte swizzle the MMA descriptor expects.
        const int wx = warp - K::kXWarp0;      // candidates: every warp not on scheduler 1
        const int ti = wx - (wx >> 2);          // transform warp index (when wx % 4 != 3)
        const bool active = !AHBM && (wx & 3) != 3 && ti < kTransformWarps;
        constexpr int kGW = CTAS == 1 ? 4 : 2;       // warps per group
        constexpr int kRT = 4 / kGW;                 // weight rows per thread
        constexpr int kXG = kTransformWarps / kGW;   // groups (2); k-steps dealt round-robin (KS is even)
        // A group's wait at k-step n (stage n % kAS, the MMAs of n - kAS done) is told apart from
        // the stage's previous phase by parity only, so that phase (the MMAs of n - 2 kAS) must be
        // complete when the group gets there: its wait at n - kXG guaranteed the MMAs of
        // n - kXG - kAS, which covers it while kXG <= kAS.
        static_assert(kXG <= kAS, "a transform group would reach a stage two phases ahead");
        const int grp = ti / kGW;
        const int row0 = (ti % kGW) * 32 + lane;   // rows row0, row0 + 128 / kRT, ...
        // the group's k-steps only; ring positions from the k-steps of the CTA's earlier units (nb)
        // (KS is a multiple of kWB, so weight stages start at unit boundaries)
        uint32_t nb = 0;
        for (int tau = active ? (int)blockIdx.x : total; tau < total; tau += gridDim.x) {
            const int4 tile = c.tiles1[tau / MT];
            if (!tile_ok(tile, c, kBN)) continue;
            for (int kc = grp; kc < KS; kc += kXG) {
                const int kw = kc % kWB;   // block of the weight stage
                const uint32_t n = nb + (uint32_t)kc, wchunk = n / kWB;
                const int as = (int)(n % kAS), ws = (int)(wchunk % kWS);
                const uint32_t aph = (n / kAS) & 1u, wph = (wchunk / kWS) & 1u;
                {
                    // waits end the same way for the whole warp (the vote), so no lane is left
                    // behind; the group's first k-step of a weight stage waits for the stage
                    bool ok = kw >= kXG || mbar_wait(&wfull[ws], wph, abort_flag, c.status);
                    ok = ok && mbar_wait(&sempty[as], aph ^ 1u, abort_flag, c.status);
                    if (!__all_sync(0xffffffffu, ok)) goto transform_done;
                    const uint8_t* blk = wsm + ws * kWStageBytes + kw * kBlockBytes;
#pragma unroll
                    for (int rr = 0; rr < kRT; ++rr) {
                        const int row = row0 + rr * (128 / kRT);
                        const uint32_t sw = (uint32_t)(row & 7);
                        const uint32_t sb = *reinterpret_cast<const uint32_t*>(blk + kBlockCodeBytes + row * 4);
                        const uint4 cwh[2] = {*reinterpret_cast<const uint4*>(blk + row * 16),
                                              *reinterpret_cast<const uint4*>(blk + 2048 + row * 16)};
                        const __half2 s2 = __half2(__ushort_as_half((unsigned short)(sb & 0xFFFFu)),
                                                   __ushort_as_half((unsigned short)(sb & 0xFFFFu)));
                        const __half2 b2 = __half2(__ushort_as_half((unsigned short)(sb >> 16)),
                                                   __ushort_as_half((unsigned short)(sb >> 16)));
                        // codes of nibble position 1 (bits 4-7 of each 16-bit half) are read in
                        // place as 16 q, so their scale is s / 16 (exact in fp16 for |s| >= 2^-13)
                        const __half2 s2_16 = __hmul2(s2, __half2(__float2half(0.0625f), __float2half(0.0625f)));
                        uint8_t* arow = asm_ + as * kATileBytes + row * 128;
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            const uint32_t words[4] = {cwh[half].x, cwh[half].y, cwh[half].z, cwh[half].w};
#pragma unroll
                            for (int w = 0; w < 4; ++w) {
                                const uint32_t lo = words[w], hi = words[w] >> 8;   // positions 0,1 | 2,3 (one shift)
                                const __half2 v0 = __hfma2(nibble_pair_pos0(lo), s2, b2);
                                const __half2 v1 = __hfma2(nibble_pair_pos1(lo), s2_16, b2);
                                const __half2 v2 = __hfma2(nibble_pair_pos0(hi), s2, b2);
                                const __half2 v3 = __hfma2(nibble_pair_pos1(hi), s2_16, b2);
                                const uint32_t ch = (uint32_t)(4 * half + w);
                                *reinterpret_cast<uint4*>(arow + ((ch ^ sw) << 4)) = make_uint4(
                                    *reinterpret_cast<const uint32_t*>(&v0), *reinterpret_cast<const uint32_t*>(&v1),
                                    *reinterpret_cast<const uint32_t*>(&v2), *reinterpret_cast<const uint32_t*>(&v3));
                            }
                        }
                    }
                    fence_proxy_async_smem();   // generic-proxy stores -> visible to the tensor core
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sfull[as]);
                    // the group's last k-step of this weight stage releases it (one arrival per warp)
                    if ((kw + kXG >= kWB || kc + kXG >= KS) && lane == 0) mbar_arrive(&wempty[ws]);
                }
            }
            nb += (uint32_t)KS;
        }
    transform_done:;
    } else {
        // ------------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const int eh = (warp - kEpiWarp0) >> 2;           // which of this quarter's warps (0 or 0/1)
        const int etid = threadIdx.x - 32 * kEpiWarp0;   // 0..255
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        uint32_t tl = 0;
        bool range_bad = false;
        for (int tau = blockIdx.x; tau < total; tau += gridDim.x) {
            const int4 tile = c.tiles1[tau / MT];
            const int mt = tau % MT;
            if (!tile_ok(tile, c, kBN)) continue;
            const int row0 = tile.y, nvalid = tile.z;
            const uint32_t ab = tl & 1u, aph = (tl >> 1) & 1u;
            ++tl;
            if (!GATEUP) {
                for (int j = etid; j < nvalid; j += 32 * kEpiWarps) {
                    meta_row[ab * kBN + j] = c.acc + (size_t)c.row_token[row0 + j] * c.H + mt * 128;
                    meta_gate[ab * kBN + j] = c.row_gate[row0 + j];
                }
                named_bar(1, 32 * kEpiWarps);
            }
            {
                const bool ok = mbar_wait(&accfull[ab], aph, abort_flag, c.status);
                if (named_bar_or(2, 32 * kEpiWarps, !ok)) goto epilogue_done;   // the group leaves together
            }
            tc_fence_after();
            const uint32_t taddr = tmem + lane_base + ab * kAccCols;
            if (GATEUP) {
                const int ilocal = 16 * q + (lane & 15);
                const bool is_gate = lane < 16;
                float amax = 0.f;   // largest |act| of this lane's valid columns (fp16 range check)
                for (int c0 = 32 * eh; c0 < nvalid; c0 += 32 * (kEpiWarps / 4)) {
                    uint32_t v[32];
                    tmem_ld32(taddr + c0, v);
                    const int lim = nvalid - c0 - (is_gate ? 0 : 16);   // this lane's valid r: r < lim
#pragma unroll
                    for (int r = 0; r < 16; ++r) {
                        const float mine_lo = __uint_as_float(v[r]);
                        const float mine_hi = __uint_as_float(v[16 + r]);
                        const float recv = __shfl_xor_sync(0xffffffffu, is_gate ? mine_hi : mine_lo, 16);
                        const float G = is_gate ? mine_lo : recv;
                        const float U = is_gate ? recv : mine_hi;
                        const int col = c0 + r + (is_gate ? 0 : 16);
                        const float a = silu_mul(G, U);
                        if (lim >= 16 || r < lim) amax = fmaxf(amax, fabsf(a));
                        stage[col * 64 + ilocal] = __float2half_rn(a);  // columns >= nvalid: not copied out
                    }
                }
                // (a NaN activation can only come from a NaN x, which the fp16 copy of x reports)
                if (!(amax <= 65504.f)) range_bad = true;
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&accempty[ab]);
                named_bar(1, 32 * kEpiWarps);
                const size_t I = (size_t)c.I;
                for (int idx = etid; idx < nvalid * 8; idx += 32 * kEpiWarps) {
                    const int j = idx >> 3, ch = idx & 7;
                    *reinterpret_cast<uint4*>(c.act + (size_t)(row0 + j) * I + mt * 64 + ch * 8) =
                        *reinterpret_cast<const uint4*>(stage + j * 64 + ch * 8);
                }
                named_bar(1, 32 * kEpiWarps);
            } else {
                // tr[r][l] = accumulator (row 32q + l, token c0 + r), kC tokens per chunk; lane l
                // then reads rows 32q + 4(l % 8) .. +3 of token c0 + (kC / 4)(l / 8) + g as one
                // float4, the gates and row pointers of its kC / 4 consecutive tokens with 16-byte
                // loads
                constexpr int kC = K::kDnChunk, kG = kC / 4;
                float* tr = reinterpret_cast<float*>(stage) + (warp - kEpiWarp0) * (kC * 32);
                const int h4 = 32 * q + 4 * (lane & 7);   // first of this lane's 4 output rows
                const int jl0 = kG * (lane >> 3);         // first of this lane's kG tokens of a chunk
                for (int c0 = kC * eh; c0 < nvalid; c0 += kC * (kEpiWarps / 4)) {
                    uint32_t v[kC];
                    if constexpr (kC == 32) tmem_ld32(taddr + c0, v);
                    else tmem_ld16(taddr + c0, v);
#pragma unroll
                    for (int r = 0; r < kC; ++r) tr[r * 32 + lane] = __uint_as_float(v[r]);
                    __syncwarp();
                    float gts[kG];
                    float* rows[kG];
                    {
                        const float4* gp = reinterpret_cast<const float4*>(meta_gate + ab * kBN + c0 + jl0);
#pragma unroll
                        for (int u = 0; u < kG / 4; ++u) {
                            const float4 gq = gp[u];
                            gts[4 * u] = gq.x; gts[4 * u + 1] = gq.y; gts[4 * u + 2] = gq.z; gts[4 * u + 3] = gq.w;
                        }
                        const ulonglong2* rp = reinterpret_cast<const ulonglong2*>(meta_row + ab * kBN + c0 + jl0);
#pragma unroll
                        for (int u = 0; u < kG / 2; ++u) {
                            const ulonglong2 pr = rp[u];
                            rows[2 * u] = reinterpret_cast<float*>(pr.x);
                            rows[2 * u + 1] = reinterpret_cast<float*>(pr.y);
                        }
                    }
#pragma unroll
                    for (int g = 0; g < kG; ++g) {
                        const int jl = jl0 + g;
                        if (c0 + jl < nvalid) {
                            const float4 y = *reinterpret_cast<const float4*>(tr + jl * 32 + 4 * (lane & 7));
                            const float gt = gts[g];
                            red_add_v4(rows[g] + h4, y.x * gt, y.y * gt, y.z * gt, y.w * gt);
                        }
                    }
                    __syncwarp();   // tr is rewritten by the next chunk
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&accempty[ab]);
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

// xp[p] = x16[row_token[p]] for the T*k routed bucket rows: one warp per row, 16-byte copies.
__global__ void __launch_bounds__(256) gather_rows_kernel(Ctx c) {
    griddep_wait();
    griddep_launch_dependents();
    const int lane = lane_id();
    const int nrows = c.T * c.k;
    for (int p = blockIdx.x * 8 + (threadIdx.x >> 5); p < nrows; p += gridDim.x * 8) {
        const int t = c.row_token[p];
        if (t < 0 || t >= c.T) {
            if (lane == 0) set_status(c.status, MOE_STATUS_BOUNDS);
            continue;
        }
        const uint4* src = reinterpret_cast<const uint4*>(c.x16 + (size_t)t * c.H);
        uint4* dst = reinterpret_cast<uint4*>(c.xp + (size_t)p * c.H);
        const int n16 = c.H / 8;
        for (int i0 = 0; i0 < n16; i0 += 32 * 8) {   // 8 loads in flight per lane before the stores
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + 32 * u + lane;
                if (i < n16) v[u] = src[i];
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + 32 * u + lane;
                if (i < n16) dst[i] = v[u];
            }
        }
    }
}

}  // namespace

namespace {

template <bool GATEUP, int CTAS, bool AHBM>
cudaError_t launch_grouped(const Ctx& c, const TokenMaps& maps, const CUtensorMap& amap, int num_sms, cudaStream_t st) {
    using K = GemmCfg<CTAS, GATEUP>;
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<GATEUP, CTAS, AHBM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, K::kSmemBytes);
    if (e != cudaSuccess) return e;
    return launch_pdl(grouped_gemm_kernel<GATEUP, CTAS, AHBM>, dim3(num_sms * CTAS), dim3(K::kThreads), K::kSmemBytes,
                      st, c, maps, amap);
}

template <bool GATEUP>
cudaError_t launch_shape(const Ctx& c, const TokenMaps& maps, const CUtensorMap* amap, int num_sms, cudaStream_t st) {
    static const CUtensorMap kNoMap = {};
    if (c.tile_rows == GemmCfg<2>::kBN)
        return amap ? launch_grouped<GATEUP, 2, true>(c, maps, *amap, num_sms, st)
                    : launch_grouped<GATEUP, 2, false>(c, maps, kNoMap, num_sms, st);
    if (c.tile_rows == GemmCfg<1>::kBN)
        return amap ? launch_grouped<GATEUP, 1, true>(c, maps, *amap, num_sms, st)
                    : launch_grouped<GATEUP, 1, false>(c, maps, kNoMap, num_sms, st);
    return cudaErrorInvalidValue;
}

}  // namespace

int gemm_tile_rows(int T, int k, int E) { return T * k <= 64 * E ? GemmCfg<2>::kBN : GemmCfg<1>::kBN; }

cudaError_t launch_gather_rows(const Ctx& c, int num_sms, cudaStream_t st) {
    const int rows = c.T * c.k;
    const int blocks = max(1, min((rows + 7) / 8, num_sms * 8));
    return launch_pdl(gather_rows_kernel, dim3(blocks), dim3(256), 0, st, c);
}

// The tile list (built for c.tile_rows rows per tile) selects the launch shape; amap (non-NULL)
// selects the fp16-weights-in-HBM ablation variant.
cudaError_t launch_gemm_gateup(const Ctx& c, const TokenMaps& maps, const CUtensorMap* amap, int num_sms,
                               cudaStream_t st) {
    return launch_shape<true>(c, maps, amap, num_sms, st);
}

cudaError_t launch_gemm_down(const Ctx& c, const TokenMaps& maps, const CUtensorMap* amap, int num_sms,
                             cudaStream_t st) {
    return launch_shape<false>(c, maps, amap, num_sms, st);
}

// out[t][h] = bf16(acc[t][h]), round to nearest even; 8 elements per thread per step.
__global__ void __launch_bounds__(256) finalize_kernel(Ctx c) {
    griddep_wait();
    griddep_launch_dependents();
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

// out[t] = bf16(base[t] + sum over j of rows[pos[t][j]]), fp32 sums in j order, 8 elements per
// thread per step; pos < 0 is no row, pos >= n_rows is recorded (BOUNDS) and skipped.
__global__ void __launch_bounds__(256) combine_rows_kernel(const uint16_t* __restrict__ rows, int n_rows,
                                                           const int* __restrict__ pos, int T, int k, int H,
                                                           const uint16_t* __restrict__ base, uint16_t* __restrict__ out,
                                                           uint32_t* status) {
    griddep_wait();
    griddep_launch_dependents();
    const int n8 = H / 8;
    const size_t total = (size_t)T * n8;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const size_t t = i / n8;
        const int ch = (int)(i % n8);
        float a[8];
        uint4 b = make_uint4(0u, 0u, 0u, 0u);
        if (base) b = *reinterpret_cast<const uint4*>(base + t * H + ch * 8);
        const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            a[2 * u] = __uint_as_float(bw[u] << 16);
            a[2 * u + 1] = __uint_as_float(bw[u] & 0xFFFF0000u);
        }
        for (int j = 0; j < k; ++j) {
            const int p = pos[t * k + j];
            if (p < 0) continue;
            if (p >= n_rows) {
                set_status(status, MOE_STATUS_BOUNDS);
                continue;
            }
            const uint4 r = *reinterpret_cast<const uint4*>(rows + (size_t)p * H + ch * 8);
            const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                a[2 * u] += __uint_as_float(rw[u] << 16);
                a[2 * u + 1] += __uint_as_float(rw[u] & 0xFFFF0000u);
            }
        }
        uint32_t ow[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            __nv_bfloat162 v = __floats2bfloat162_rn(a[2 * u], a[2 * u + 1]);
            ow[u] = *reinterpret_cast<uint32_t*>(&v);
        }
        *reinterpret_cast<uint4*>(out + t * H + ch * 8) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
    }
}

cudaError_t launch_combine_rows(const uint16_t* rows, int n_rows, const int* pos, int T, int k, int H,
                                const uint16_t* base, uint16_t* out, uint32_t* status, int num_sms, cudaStream_t st) {
    const size_t total = (size_t)T * (H / 8);
    const size_t want = (total + 255) / 256;
    const int blocks = (int)std::min<size_t>(want > 0 ? want : 1, (size_t)num_sms * 16);
    return launch_pdl(combine_rows_kernel, dim3(blocks), dim3(256), 0, st, rows, n_rows, pos, T, k, H, base, out,
                      status);
}

cudaError_t launch_finalize(const Ctx& c, cudaStream_t st) {
    const size_t n8 = (size_t)c.T * c.H / 8;
    // one 8-element chunk per thread (the loop only covers grids past the launch limit)
    const size_t want = (n8 + 255) / 256;
    const int blocks = (int)(want < (size_t)(1u << 30) ? want : (size_t)(1u << 30));
    return launch_pdl(finalize_kernel, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, st, c);
}

}  // namespace moe
