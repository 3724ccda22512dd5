// decode_fused.cu -- decode of up to kDecodeFusedMaxT tokens through one MoE layer in a single
// kernel of CTA pairs.
//
// A decode token moves ~18 MB (router 2 MiB + 9 experts x 1.69 MiB): about 2.8 us of HBM time,
// so what decides the layer's time is how many dependent memory round trips lie on its critical
// path and how much of the weight stream is in flight at once.  The pages' decode levers are to
// fuse the kernel chain and to run independent work concurrently ("A Rust + Metal Inference
// Engine..." body; "Perplexity Open-Sources Lily..." section "Generation has a different
// bottleneck").  Here the whole layer is one grid of 2-CTA clusters, one cluster per work unit
// (expert slot j, 64-column slice mt of the intermediate dimension):
//
//   routed unit (j, mt)   gate/up rows of slice mt (one 128-row m-tile: 64 gate + 64 up rows,
//                         interleaved) of the j-th selected expert; CTA r of the pair holds the
//                         input-column half r (H/128 blocks), and down-projection k-step mt for
//                         output rows [H/2 * r, H/2 * (r + 1)) (H/256 blocks);
//   shared unit (mt)      the same for the always-on shared expert.
//
// Per CTA the flow is:
//   1. before the previous kernel in the stream has finished (programmatic dependent launch):
//      bulk-copy the weights that do not depend on x -- the CTA's router rows (routed units) or
//      its whole shared-expert share (shared units) -- into shared memory;
//   2. stage x (fp32, and per 64-column group scaled by a power of two for the GEMVs);
//   3. routed CTAs: compute their router logits and publish each as one 64-bit word
//      (call tag << 32 | fp32 bits); every routed CTA polls all E words until they carry this
//      call's tag -- data and synchronisation in one round trip, no grid barrier -- and picks the
//      top k (every CTA gets the same answer); the CTA then bulk-copies its expert's gate/up half
//      and down blocks (~110 KB) into shared memory in one wave;
//   4. gate/up GEMV from shared memory as the copies land, the pair's two column halves summed
//      through distributed shared memory, act = silu(G) * U for the 64 columns of the slice;
//   5. down GEMV of the slice into the CTA's H/2 output rows, times the gate, added into an fp32
//      row accumulator (vector reductions in L2); per 128-row chunk an arrival counter finds the
//      last of the units, which rounds the chunk to bf16, writes it and re-zeroes the chunk's
//      accumulator and counter (self-cleaning, no memset).
// The shared-expert pairs never wait for routing.  With T > 1 tokens every step keeps per-token
// state (x, router words, selection, accumulators, counters); a routed unit runs steps 4-5 once
// per token for the token's j-th expert, and its gate/up and down buffers take the next token's
// expert as soon as the current token has read them, so that stream overlaps the current token's
// exchange, act and down GEMV; the shared unit loads its weights once for all tokens.
//
// Call state lives in the workspace: a ticket counter every CTA increments at start (call number
// = ticket / CTAs per call, so the router words of an earlier or abandoned call never carry the
// current tag), the fp32 accumulator and the chunk counters (zero between calls), and a dirty
// word that a CTA raises when one of its bounded waits runs out: the next call then zeroes the
// accumulator and counters before anything is added, with no host intervention.
//
// GEMV arithmetic: fp32 FMAs with fp16 multiplicands (fma.rn.f32.f16).  Each pair of 4-bit codes
// is masked out of its packed word straight into the two halves of a 32-bit register, where it
// reads as two fp16 subnormals (q * 2^-24, or q * 2^-20 for the upper nibble of a byte); the
// activations are staged once per call as fp16, each 64-column group scaled by a power of two
// (stage_f16), so every product is exact in fp32 and the sums are fp32.  The scale is applied once
// per (row, half group) and the bias as b * (sum of the half group's staged activations).  x is
// bf16, so staging it is exact (down to 2^-27 of its group's largest value); act is rounded to
// fp16, as on the prefill path.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kDThreads = 512;
constexpr int kDWarps = kDThreads / 32;
constexpr int kMaxRouterRows = 4;
constexpr int kMaxDM = 12;           // down blocks per CTA (H / 256)
constexpr int kMaxChunkBlocks = 8;   // gate/up blocks per landing chunk
constexpr int kPollStaggerCycles = 500;

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
// sum over the 16 lanes of each half warp (lanes 0-15 and 16-31 separately)
__device__ __forceinline__ float half_warp_sum(float v) {
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ uint32_t ord_key(float v) {
    const uint32_t u = __float_as_uint(v + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// {acc.x + c.lo * x.lo, acc.y + c.hi * x.hi}: fp32 FMAs with fp16 multiplicands (the product of
// two fp16 values is exact in fp32, so each is rounded once, in the sum); the 4-bit codes enter as
// fp16 subnormals, kept as such (no .ftz)
__device__ __forceinline__ float2 fma_f16pair(uint32_t c2, uint32_t x2, float2 acc) {
    float2 d;
    asm("{\n\t.reg .b16 cl, ch, xl, xh;\n\tmov.b32 {cl, ch}, %2;\n\tmov.b32 {xl, xh}, %3;\n\t"
        "fma.rn.f32.f16 %0, cl, xl, %4;\n\tfma.rn.f32.f16 %1, ch, xh, %5;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "r"(c2), "r"(x2), "f"(acc.x), "f"(acc.y));
    return d;
}

// Sum over the 32 columns of one half group: codes c (4 words of 8 nibbles), activations xv (32
// fp16 in column order, 8 per uint4).  Nibbles of a word, low bit first, hold columns
// 0 2 4 6 1 3 5 7, so the 16-bit halves of (w & 0x000F000F) are columns (0, 1) as q * 2^-24,
// of (w & 0x00F000F0) columns (2, 3) as q * 2^-20, and the same masks of w >> 8 columns (4, 5)
// and (6, 7): four ANDs and one shift per 8 columns.  The activations of pairs (2, 3) and (6, 7)
// carry a further factor 2^-4 (stage_f16), so every product is q * x * 2^(A - 24) for the
// group's A.
__device__ __forceinline__ float dot32h(const uint4& c, const uint4* xv) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    float2 a = make_float2(0.f, 0.f), b = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 xx = xv[i];
        const uint32_t hi = w[i] >> 8;
        a = fma_f16pair(w[i] & 0x000F000Fu, xx.x, a);
        b = fma_f16pair(w[i] & 0x00F000F0u, xx.y, b);
        a = fma_f16pair(hi & 0x000F000Fu, xx.z, a);
        b = fma_f16pair(hi & 0x00F000F0u, xx.w, b);
    }
    return (a.x + a.y) + (b.x + b.y);
}

// Stages a lane's two consecutive columns (2 lane, 2 lane + 1) of a 64-column group for dot32h:
// the group is scaled by 2^A, A = 14 - (exponent of the group's largest |value| m), so that every
// value is below 2^15 in magnitude; columns 2-3 and 6-7 of each 8 take a further 2^-4; the values
// are rounded to fp16 (bf16 inputs stay exact down to 2^-27 of the group's largest).  Returns the
// two fp16 values; *rounded receives their sum as the GEMV sees them (unscaled, for the bias
// term) and *undo the factor 2^(24 - A) that turns a dot32h sum into the plain dot.
__device__ __forceinline__ uint32_t stage_f16(float a0, float a1, int lane, float m, float* rounded, float* undo) {
    const int e = max(-100, min(100, (int)((__float_as_uint(m) >> 23) & 0xFFu) - 127));
    const int A = 14 - e - ((lane & 1) ? 4 : 0);
    const __half2 h = __floats2half2_rn(a0 * __int_as_float((127 + A) << 23), a1 * __int_as_float((127 + A) << 23));
    *rounded = (__low2float(h) + __high2float(h)) * __int_as_float((127 - A) << 23);
    *undo = __int_as_float((127 + 10 + e) << 23);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// One comparator of the descending sort of a lane's (key, expert) pairs: the larger key first,
// equal keys with the lower expert index first.
__device__ __forceinline__ void cas_desc(uint32_t& ka, uint32_t& ia, uint32_t& kb, uint32_t& ib) {
    const bool sw = kb > ka || (kb == ka && ib < ia);
    const uint32_t k0 = sw ? kb : ka, i0 = sw ? ib : ia, k1 = sw ? ka : kb, i1 = sw ? ia : ib;
    ka = k0; ia = i0; kb = k1; ib = i1;
}

// ---- cluster, memory-model and wait helpers ----------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
// 16 bytes into the shared memory of the cluster CTA `rank`, at the offset of `local`, completing
// 16 bytes of transaction count on that CTA's mbarrier at the offset of `local_bar`
__device__ __forceinline__ void st_async_peer_v4(const float* local, const uint64_t* local_bar, uint32_t rank,
                                                 float4 v) {
    uint32_t ra, rb;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rb) : "r"(smem_u32(local_bar)), "r"(rank));
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(ra),
                 "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(rb)
                 : "memory");
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u32(unsigned* p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned atom_add_acq_rel(unsigned* p, unsigned v) {
    unsigned old;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// Bounded wait for phase `parity` of an mbarrier (false after kWaitLimitNs).
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
    return true;
}

// Shared-memory carve-up (byte offsets, computed on the host from DecodeGeom and checked there).
// Per-token arrays hold TM tokens.
struct Smem {
    uint8_t* wgu;      // [nslots][cblk][4608] gate/up chunk buffers (this unit's m-tile, column half r)
    uint8_t* wdn;      // [DM][4608]  down blocks: k-step mt of the CTA's DM output m-tiles
    float* rrow;       // [R][H]      router rows of this CTA (routed units)
    float* sgw;        // [H]         shared-expert gate vector (shared units and CTA 0)
    uint16_t* xraw;    // [T][H]      x as given (bf16)
    uint32_t* xh;      // [T][H/2]    x as fp16 pairs, scaled per 64-column group (stage_f16)
    float* xsum;       // [T][H/32]   sum of the staged x over each half group, unscaled
    float* xsc;        // [T][H/64]   2^(24-A) per group (stage_f16)
    float* part;       // [4][128]    gate/up partial row sums (block parity x column half)
    float* mine;       // [128]       this CTA's gate/up row sums over its input-column half
    float* peer;       // [2][128]    the partner's, written by the partner (by token parity)
    uint32_t* act;     // [32]        act of the slice as fp16 pairs (stage_f16)
    float* misc;       // [32]        asum[2], asc; gate of token t at 4 + t; shared gate at 4 + TM + t
    float* ydn;        // [2][DM*128] down partial sums by column half
    float* red;        // [kDWarps][T][kMaxRouterRows + 1] per-warp partial dots (+ shared gate)
    int* ints;         // [kNumInts]  flags, see below
    uint64_t* bars;    // bar_r, bar_d[2], bar_x[2], bar_g[nslots]
};

template <int TM>
__device__ __forceinline__ Smem carve(uint8_t* base, const DecodeGeom& g) {
    Smem s;
    s.wgu = base + g.off_wgu;
    s.wdn = base + g.off_wdn;
    s.rrow = reinterpret_cast<float*>(base + g.off_rrow);
    s.sgw = reinterpret_cast<float*>(base + g.off_sgw);
    s.xraw = reinterpret_cast<uint16_t*>(base + g.off_xraw);
    s.xh = reinterpret_cast<uint32_t*>(base + g.off_xs);
    s.xsum = reinterpret_cast<float*>(base + g.off_xsum);
    s.xsc = reinterpret_cast<float*>(base + g.off_xsc);
    s.part = reinterpret_cast<float*>(base + g.off_part);
    s.mine = s.part + 4 * 128;
    s.peer = s.mine + 128;
    s.act = reinterpret_cast<uint32_t*>(s.peer + 2 * 128);
    s.misc = s.peer + 2 * 128 + 64;   // [32]
    s.ydn = reinterpret_cast<float*>(base + g.off_ydn);
    s.red = reinterpret_cast<float*>(base + g.off_logit);
    s.ints = reinterpret_cast<int*>(s.red + kDWarps * TM * (kMaxRouterRows + 1));
    s.bars = reinterpret_cast<uint64_t*>(base + g.off_bars);
    return s;
}

// ints: abort, dirty word, call tag, the selected expert of token t, the poll winner of token t,
// copy waves issued into each gate/up chunk buffer and into each down buffer, and per (token,
// chunk) whether this CTA finalises it
constexpr int kMaxSlots = 8;
enum {
    kIntAbort = 0, kIntDirty = 1, kIntTag = 2, kIntSel = 3, kIntPolled = kIntSel + kDecodeFusedMaxT,
    kIntWavesG = kIntPolled + kDecodeFusedMaxT, kIntWavesD = kIntWavesG + kMaxSlots,
    kIntFlags = kIntWavesD + 2, kNumInts = kIntFlags + kDecodeFusedMaxT * kMaxDM
};
enum { kMiscAsum0 = 0, kMiscAsum1 = 1, kMiscAsc = 2, kMiscGate = 4, kMiscSg = 4 + kDecodeFusedMaxT };
static_assert(kMiscSg + kDecodeFusedMaxT <= 32, "misc area");
constexpr int kRedStride = kMaxRouterRows + 1;   // per (warp, token): router rows, then the shared-gate dot

// TM: the most tokens a launch serves (1: the single-token form, whose loops and per-token
// registers collapse; kDecodeFusedMaxT: 1..kDecodeFusedMaxT tokens)
template <int TM>
__global__ void __launch_bounds__(kDThreads, 1) decode_fused_kernel(Ctx c, DecodeGeom g) {
    // warps polling the router words (every kPollStride-th warp; by token, then staggered)
    constexpr int kPollWarps = TM == 1 ? 3 : kDecodeFusedMaxT;
    constexpr int kPollStride = TM == 1 ? 4 : kDWarps / kDecodeFusedMaxT;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const Smem s = carve<TM>(smem_raw, g);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = c.H, E = c.E, k = c.k, T = TM == 1 ? 1 : c.T;
    const int KSg = H / 64, MTd = H / 128, KSd = c.I / 64;
    const uint32_t r = cluster_ctarank();
    const int q = blockIdx.x >> 1;                      // work unit = cluster
    const bool routed = q < k * g.MTg;
    const int j = routed ? q / g.MTg : k;               // expert slot (k = the shared expert)
    const int mt = routed ? q % g.MTg : q - k * g.MTg;  // 64-column slice of I
    const int cr = blockIdx.x;                          // routed CTA index (routed units come first)
    uint64_t* bar_r = s.bars;       // router rows and the shared-gate vector landed
    constexpr int kDSlots = 1;
    uint64_t* bar_d = s.bars + 1;   // [kDSlots] down blocks landed (one phase per fill)
    uint64_t* bar_x = s.bars + 3;   // [2] the partner's gate/up sums landed, by token parity
    uint64_t* bar_g = s.bars + 5;   // [nslots] gate/up chunk buffers landed (one phase per fill)
    const bool need_sg = c.has_shared && (!routed || blockIdx.x == 0);
    int nrows = 0;   // router rows of this CTA
    if (routed)
        for (int i = 0; i < g.R; ++i) nrows += (cr + g.NR * i < E) ? 1 : 0;

    if (tid == 0) {
        for (int i = 0; i < 5 + g.nslots; ++i) mbar_init(&s.bars[i], 1);
        fence_mbar_init();
        // exchange rounds 0 and 1, armed before the partner can send (cluster barrier 1)
        mbar_arrive_expect_tx(&bar_x[0], 128 * sizeof(float));
        if (T > 1) mbar_arrive_expect_tx(&bar_x[1], 128 * sizeof(float));
        s.ints[kIntAbort] = 0;
        for (int t = 0; t < kDecodeFusedMaxT; ++t) s.ints[kIntPolled + t] = 0;
        for (int sl = 0; sl < kMaxSlots; ++sl) s.ints[kIntWavesG + sl] = (!routed && sl < g.nch) ? 1 : 0;
        s.ints[kIntWavesD] = routed ? 0 : 1;
        s.ints[kIntWavesD + 1] = 0;
    }
    cluster_arrive_relaxed();   // (1) this CTA has started; waited on before the first remote store
    __syncthreads();

    // ---- 1. weights that do not depend on x (nothing written by an earlier kernel is read yet)
    // this unit's copies for expert e: the gate/up half in nch chunks (one thread, or one lane
    // per chunk), and the DM down blocks (one per lane of a warp, after lane 0 has set the
    // barrier's byte count).  A copy costs its issuing thread ~290 cycles, so a wave on the
    // critical path is issued one copy per lane.
    auto issue_gateup_chunk = [&](int e, int ch, int slot) {   // chunk ch of expert e into buffer slot
        const uint8_t* gu = c.w_gu + ((size_t)(e * g.MTg + mt) * KSg + (size_t)g.KH * r + (size_t)ch * g.cblk) * kBlockBytes;
        mbar_arrive_expect_tx(&bar_g[slot], (uint32_t)(g.cblk * kBlockBytes));
        bulk_g2s(s.wgu + (size_t)slot * g.cblk * kBlockBytes, gu, (uint32_t)(g.cblk * kBlockBytes), &bar_g[slot]);
        if (routed) ++s.ints[kIntWavesG + slot];   // one issuing thread per buffer at a time
    };
    auto issue_down = [&](int e, int dslot) {   // called by a whole warp
        uint64_t* bd = &bar_d[dslot];
        uint8_t* dst = s.wdn + (size_t)dslot * g.DM * kBlockBytes;
        if (lane == 0) mbar_arrive_expect_tx(bd, (uint32_t)(g.DM * kBlockBytes));
        __syncwarp();
        for (int b = lane; b < g.DM; b += 32) {
            const int mtd = g.DM * (int)r + b;
            bulk_g2s(dst + (size_t)b * kBlockBytes, c.w_dn + ((size_t)(e * MTd + mtd) * KSd + mt) * kBlockBytes,
                     kBlockBytes, bd);
        }
        if (lane == 0 && routed) ++s.ints[kIntWavesD + dslot];
    };
    const bool need_r = nrows > 0 || need_sg;
    if (need_r && warp == 2 && lane == 0) {
        mbar_arrive_expect_tx(bar_r, (uint32_t)((nrows + (need_sg ? 1 : 0)) * H * sizeof(float)));
        for (int i = 0; i < nrows; ++i)
            bulk_g2s(s.rrow + (size_t)i * H, c.router32 + (size_t)(cr + g.NR * i) * H, (uint32_t)(H * sizeof(float)),
                     bar_r);
        if (need_sg) bulk_g2s(s.sgw, c.sgw, (uint32_t)(H * sizeof(float)), bar_r);
    }
    if (!routed) {   // the shared expert is group E, the same for every token: one wave
        if (warp == 0 && lane < g.nch) issue_gateup_chunk(E, lane, lane);
        if (warp == 1) issue_down(E, 0);
    }
    const float my_bias = (tid < nrows) ? c.rbias[cr + g.NR * tid] : 0.f;

    // ---- 2. from here on x and the workspace are read: wait for the previous grid
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // x of the T tokens: 16-byte loads; the call ticket and the dirty word are fetched by the last
    // two warps at the same time (the tag is only needed at the router publish)
    for (int i = tid; i < T * H / 8; i += kDThreads)
        reinterpret_cast<uint4*>(s.xraw)[i] = reinterpret_cast<const uint4*>(c.x)[i];
    if (tid == kDThreads - 64) {   // call tag: CTAs started before this one, over CTAs per call (+1)
        const unsigned long long ticket = atomicAdd(c.dfz.ticket, 1ull);
        s.ints[kIntTag] = (int)(uint32_t)(ticket / (unsigned long long)gridDim.x + 1ull);
    }
    if (tid == kDThreads - 32) s.ints[kIntDirty] = (int)ld_acquire_u32(c.dfz.dirty);
    __syncthreads();
    const uint32_t tag = (uint32_t)s.ints[kIntTag];
    const bool dirty = s.ints[kIntDirty] != 0;
    // a call after one that gave up part-way: the routed CTAs put the accumulators and the chunk
    // counters of every token back to zero (ordered before their router words by a fence)
    if (dirty && routed) {
        for (int i = cr * kDThreads + tid; i < kDecodeFusedMaxT * H; i += g.NR * kDThreads) c.dfz.outacc[i] = 0.f;
        for (int i = cr * kDThreads + tid; i < kDecodeFusedMaxT * MTd; i += g.NR * kDThreads) c.dfz.cnt[i] = 0u;
    }

    // ---- 3. router logits and the shared gate sigmoid(x . w_sg) of every token (the shared
    // units' combine weight; CTA 0 also reports it)
    bool ok = true;
    if (need_r) ok = wait_bar(bar_r, 0);
    // tokens in passes of up to four (the per-thread partial sums live in registers)
    constexpr int kTG = TM < 4 ? TM : 4;
    for (int t0 = 0; t0 < T; t0 += kTG) {
        float acc[kTG][kMaxRouterRows];
        float d[kTG];
#pragma unroll
        for (int u = 0; u < kTG; ++u) {
            d[u] = 0.f;
#pragma unroll
            for (int i = 0; i < kMaxRouterRows; ++i) acc[u][i] = 0.f;
        }
        if (ok) {
            for (int h = tid; h < H; h += kDThreads) {
                float rv[kMaxRouterRows];
#pragma unroll
                for (int i = 0; i < kMaxRouterRows; ++i) rv[i] = i < nrows ? s.rrow[(size_t)i * H + h] : 0.f;
                const float sv = need_sg ? s.sgw[h] : 0.f;
#pragma unroll
                for (int u = 0; u < kTG; ++u) {
                    if (t0 + u < T) {
                        const float xv = __uint_as_float((uint32_t)s.xraw[(size_t)(t0 + u) * H + h] << 16);
#pragma unroll
                        for (int i = 0; i < kMaxRouterRows; ++i)
                            if (i < nrows) acc[u][i] = fmaf(xv, rv[i], acc[u][i]);
                        if (need_sg) d[u] = fmaf(xv, sv, d[u]);
                    }
                }
            }
        }
        if (TM == 1) {
            // one token: the warp sums of every router row and of the shared-gate dot, their
            // shuffle rounds interleaved (rows past nrows are zeros)
            float v[kRedStride];
#pragma unroll
            for (int i = 0; i < kMaxRouterRows; ++i) v[i] = acc[0][i];
            v[kMaxRouterRows] = d[0];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
#pragma unroll
                for (int i = 0; i < kRedStride; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
            if (lane == 0)
#pragma unroll
                for (int i = 0; i < kRedStride; ++i) s.red[warp * kRedStride + i] = v[i];
        } else {
#pragma unroll
            for (int u = 0; u < kTG; ++u) {
                const int t = t0 + u;
                if (t < T) {   // uniform across the CTA
#pragma unroll
                    for (int i = 0; i < kMaxRouterRows; ++i) {
                        if (i < nrows) {
                            const float v = warp_sum(acc[u][i]);
                            if (lane == 0) s.red[(warp * TM + t) * kRedStride + i] = v;
                        }
                    }
                    if (need_sg) {
                        const float v = warp_sum(d[u]);
                        if (lane == 0) s.red[(warp * TM + t) * kRedStride + kMaxRouterRows] = v;
                    }
                }
            }
        }
    }
    if (__syncthreads_or(!ok)) {
        ok = false;
        if (tid == 0) {
            set_status(c.status, MOE_STATUS_TIMEOUT);
            atomicOr(c.dfz.dirty, 1u);
        }
    }
    if (routed && ok && warp == 0 && lane < T * nrows) {
        // lane (t, i) sums router row i's per-warp partial dots of token t (all loads first)
        const int t = lane / nrows, i = lane - t * nrows;
        float pv[kDWarps];
#pragma unroll
        for (int w = 0; w < kDWarps; ++w) pv[w] = s.red[(w * TM + t) * kRedStride + i];
        float z = 0.f;
#pragma unroll
        for (int w = 0; w < kDWarps; ++w) z += pv[w];
        z += __shfl_sync(T * nrows >= 32 ? 0xffffffffu : (1u << (T * nrows)) - 1u, my_bias, i);
        const int e = cr + g.NR * i;
        const bool stall = (c.flags & 0x100u) && cr == 0 && tag == 1u;   // test only: first call withholds
        // the word carries its own data; after a failed call it must also follow this CTA's zeroing
        if (dirty) fence_acq_rel_gpu();
        if (!stall) st_relaxed_u64(c.dfz.slots + (size_t)t * E + e, ((unsigned long long)tag << 32) | __float_as_uint(z));
    }
    if (need_sg && tid >= 32 && tid < 32 + T) {
        const int t = tid - 32;
        float zz = 0.f;
        for (int w = 0; w < kDWarps; ++w) zz += s.red[(w * TM + t) * kRedStride + kMaxRouterRows];
        s.misc[kMiscSg + t] = 1.f / (1.f + expf(-zz));
    }
    // per-group scaling of x over the input-column half this CTA's gate/up blocks cover, every
    // token (only the gate/up GEMV reads it, so it follows the router publish)
    for (int p = warp; p < T * g.KH; p += kDWarps) {
        const int t = p / g.KH, grp = g.KH * (int)r + (p - t * g.KH);
        const uint32_t xw = reinterpret_cast<const uint32_t*>(s.xraw + (size_t)t * H)[32 * grp + lane];
        const float a0 = __uint_as_float(xw << 16), a1 = __uint_as_float(xw & 0xFFFF0000u);
        const float m = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fmaxf(fabsf(a0), fabsf(a1)))));
        float rsum, undo;
        s.xh[(size_t)t * (H / 2) + 32 * grp + lane] = stage_f16(a0, a1, lane, m, &rsum, &undo);
        const float hs = half_warp_sum(rsum);
        if ((lane & 15) == 0) s.xsum[(size_t)t * (H / 32) + 2 * grp + (lane >> 4)] = hs;
        if (lane == 0) s.xsc[(size_t)t * (H / 64) + grp] = undo;
    }
    if (ok && (routed || dirty) && warp % kPollStride == 0 && warp < kPollStride * kPollWarps) {
        // every router word of this call: relaxed polls (each word carries its data; no load is
        // left in flight when the loop ends).  kPollWarps warps poll; warp pw takes token pw % T,
        // several warps on one token staggered by a fraction of a round trip so the last word is
        // seen sooner after it lands; the first to see a token's words wins it (shared-memory
        // flag) and goes on, the others stop.
        const int pw = warp / kPollStride;
        const int tk = pw % T;
        if (pw >= T) {
            const long long c0 = clock64();
            while (clock64() - c0 < (long long)(pw / T) * kPollStaggerCycles) {}
        }
        const unsigned long long* words = c.dfz.slots + (size_t)tk * E;
        uint32_t key[8], idx[8];
        float lg[8];
        bool lost = false;
        const unsigned long long t0 = globaltimer_ns();
        while (true) {
            unsigned long long cur[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) cur[i] = (lane + 32 * i < E) ? ld_relaxed_u64(words + lane + 32 * i) : 0ull;
            bool all = true;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = lane + 32 * i;
                const float f = __uint_as_float((uint32_t)cur[i]);
                lg[i] = (e < E && f == f) ? f : -INFINITY;
                if (e < E && (uint32_t)(cur[i] >> 32) != tag) all = false;
            }
            if (__all_sync(0xffffffffu, all)) {
                int won = 0;
                if (lane == 0) won = atomicCAS(&s.ints[kIntPolled + tk], 0, 1) == 0;
                lost = __shfl_sync(0xffffffffu, won, 0) == 0;
                break;
            }
            if (__shfl_sync(0xffffffffu, *reinterpret_cast<volatile int*>(&s.ints[kIntPolled + tk]), 0) != 0) {
                lost = true;   // another polling warp has this token's words
                break;
            }
            if (__any_sync(0xffffffffu, globaltimer_ns() - t0 > kWaitLimitNs)) {   // one decision for the warp
                ok = false;
                break;
            }
        }
        ok = __all_sync(0xffffffffu, ok);
        if (lost) goto polled;
        if (dirty) fence_acq_rel_gpu();   // every routed CTA's zeroing precedes what follows
        if (ok && routed) {
            // top k by logit, ties to the lower expert index: each lane sorts its 8 (key, expert)
            // pairs once (19-comparator network), then every pick is the lanes' heads' maximum
            // key, the lowest expert among the heads holding it, and a pop of the winner's head
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = lane + 32 * i;
                key[i] = e < E ? ord_key(lg[i]) : 0u;
                idx[i] = e < E ? (uint32_t)e : 0xFFFFFFFFu;
            }
            cas_desc(key[0], idx[0], key[2], idx[2]); cas_desc(key[1], idx[1], key[3], idx[3]);
            cas_desc(key[4], idx[4], key[6], idx[6]); cas_desc(key[5], idx[5], key[7], idx[7]);
            cas_desc(key[0], idx[0], key[4], idx[4]); cas_desc(key[1], idx[1], key[5], idx[5]);
            cas_desc(key[2], idx[2], key[6], idx[6]); cas_desc(key[3], idx[3], key[7], idx[7]);
            cas_desc(key[0], idx[0], key[1], idx[1]); cas_desc(key[2], idx[2], key[3], idx[3]);
            cas_desc(key[4], idx[4], key[5], idx[5]); cas_desc(key[6], idx[6], key[7], idx[7]);
            cas_desc(key[2], idx[2], key[4], idx[4]); cas_desc(key[3], idx[3], key[5], idx[5]);
            cas_desc(key[1], idx[1], key[4], idx[4]); cas_desc(key[3], idx[3], key[6], idx[6]);
            cas_desc(key[1], idx[1], key[2], idx[2]); cas_desc(key[3], idx[3], key[4], idx[4]);
            cas_desc(key[5], idx[5], key[6], idx[6]);
            int my_e = 0;
            for (int jj = 0; jj < k; ++jj) {
                const uint32_t mx = __reduce_max_sync(0xffffffffu, key[0]);
                const uint32_t be = __reduce_min_sync(0xffffffffu, key[0] == mx ? idx[0] : 0xFFFFFFFFu);
                if (idx[0] == be) {   // pop the winner's head
#pragma unroll
                    for (int i = 0; i < 7; ++i) { key[i] = key[i + 1]; idx[i] = idx[i + 1]; }
                    key[7] = 0u;
                    idx[7] = 0xFFFFFFFFu;
                }
                if (lane == jj) my_e = (int)be;
            }
            // lane jj < k fetches the logit of its pick from the lane that holds it
            float my_v = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float cv = __shfl_sync(0xffffffffu, lg[i], my_e & 31);
                if ((my_e >> 5) == i) my_v = cv;
            }
            const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
            const float p = lane < k ? expf(my_v - vmax) : 0.f;
            const float zsum = warp_sum(p);
            if (lane < k && (my_e < 0 || my_e >= E)) {
                set_status(c.status, MOE_STATUS_BOUNDS);
                my_e = 0;
            }
            const int sel = __shfl_sync(0xffffffffu, my_e, j);
            const float gsel = __shfl_sync(0xffffffffu, p, j) / zsum;
            if (lane == 0) {
                s.ints[kIntSel + tk] = sel;
                s.misc[kMiscGate + tk] = gsel;
            }
            if (tk == 0) {   // the first token's wave at once: lanes 0 .. nch-1 a gate/up chunk each,
                             // lanes 16 .. 16 + DM - 1 a down block each
                if (lane < g.nch) issue_gateup_chunk(sel, lane, lane);
                if (lane == 16) mbar_arrive_expect_tx(bar_d, (uint32_t)(g.DM * kBlockBytes));
                __syncwarp();
                if (lane >= 16 && lane - 16 < g.DM) {
                    const int b = lane - 16, mtd = g.DM * (int)r + b;
                    bulk_g2s(s.wdn + (size_t)b * kBlockBytes,
                             c.w_dn + ((size_t)(sel * MTd + mtd) * KSd + mt) * kBlockBytes, kBlockBytes, bar_d);
                }
                if (lane == 16) s.ints[kIntWavesD] = 1;
            }
            if (blockIdx.x == 0 && lane < k) {
                c.idx[(size_t)tk * k + lane] = my_e;
                c.gates[(size_t)tk * k + lane] = p / zsum;
            }
        }
        if (lane == 0 && !ok) {
            set_status(c.status, MOE_STATUS_TIMEOUT);
            atomicOr(c.dfz.dirty, 1u);
        }
        if (lane == 0 && !ok) s.ints[kIntAbort] = 1;
    }
polled:
    __syncthreads();
    ok = ok && s.ints[kIntAbort] == 0;
    if (!routed && tid < T) s.misc[kMiscGate + tid] = s.misc[kMiscSg + tid];
    if (blockIdx.x == 0 && tid >= 32 && tid < 32 + T) {
        c.sg[tid - 32] = c.has_shared ? s.misc[kMiscSg + tid - 32] : 0.f;
    }
    if (blockIdx.x == 0 && tid == 64 && ok && dirty) st_release_u32(c.dfz.dirty, 0u);   // every routed CTA has read it
    // the next kernel in the stream may be scheduled from here on (it waits for this grid's
    // completion before it reads anything this grid writes)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // ---- 4./5. per token: gate/up GEMV as the chunks land, the pair's exchange, act, down GEMV,
    // gated reductions into the token's fp32 row.  A routed unit's gate/up chunk buffers take the
    // next token's expert once this token's GEMV has read them (the stream overlaps this token's
    // exchange, act and down GEMV), and its down buffer the next token's expert once this
    // token's down GEMV has read it; the shared unit's weights serve every token.
    const int row = tid & 127, hh = (tid >> 7) & 1, par = tid >> 8;
    unsigned arrivals[TM];   // counter values before this CTA's arrival (tid < DM)
#pragma unroll
    for (int t = 0; t < TM; ++t) arrivals[t] = 0u;
    for (int t = 0; t < T; ++t) {
        // this token's fill of the down buffer (the shared unit's one fill serves every token)
        const int dslot = 0;
        const uint32_t ph = routed ? (uint32_t)(t & 1) : 0u;
        float acc = 0.f;
        bool wok = ok;
        if (ok) {
            const uint32_t* xt = s.xh + (size_t)t * (H / 2);
            for (int ch = 0; ch < g.nch; ++ch) {
                // chunk number cs of the unit's gate/up stream, in buffer cs % nslots (the shared
                // unit's chunks stay in buffers 0 .. nch-1 for every token)
                const int cs = routed ? t * g.nch + ch : ch;
                const int slot = cs % g.nslots;
                if (!wait_bar(&bar_g[slot], (uint32_t)((cs / g.nslots) & 1))) { wok = false; break; }
                const uint8_t* cbase = s.wgu + (size_t)slot * g.cblk * kBlockBytes + hh * 2048 + row * 16;
                const int kc0 = g.KH * (int)r + ch * g.cblk;   // first 64-column group of x in the chunk
                const uint4* xc = reinterpret_cast<const uint4*>(xt + 32 * kc0 + 16 * hh);
                const float* xscc = s.xsc + (size_t)t * (H / 64) + kc0;
                const float* xsumc = s.xsum + (size_t)t * (H / 32) + 2 * kc0 + hh;
#pragma unroll 2
                for (int b = par; b < g.cblk; b += 2) {
                    const uint8_t* blk = cbase + (size_t)b * kBlockBytes;
                    const uint4 cw = *reinterpret_cast<const uint4*>(blk);
                    const uint32_t sb =
                        *reinterpret_cast<const uint32_t*>(blk - hh * 2048 - row * 16 + kBlockCodeBytes + row * 4);
                    const float P = dot32h(cw, xc + 8 * b);
                    const float sc = __half2float(__ushort_as_half((unsigned short)(sb & 0xFFFFu)));
                    const float bi = __half2float(__ushort_as_half((unsigned short)(sb >> 16)));
                    acc += sc * (P * xscc[b]) + bi * xsumc[2 * b];
                }
            }
        }
        s.part[(par * 2 + hh) * 128 + row] = acc;
        if (__syncthreads_or(!wok)) ok = false;
        // the gate/up buffers are read: the next token's expert streams into them, one chunk per lane
        if (TM > 1 && routed && ok && t + 1 < T && warp == 0 && lane < g.nch)
            issue_gateup_chunk(s.ints[kIntSel + t + 1], lane, lane);
        if (ok && tid < 128) s.mine[tid] = (s.part[tid] + s.part[128 + tid]) + (s.part[256 + tid] + s.part[384 + tid]);
        if (t == 0) cluster_wait();   // (1) the partner has started (its exchange mbarriers are armed)
        __syncthreads();
        // the pair's exchange, round t: this CTA's 128 row sums go into the partner's shared memory
        // with asynchronous remote stores that complete the partner's mbarrier of this token
        // parity; each CTA waits on its own.  Both CTAs take every round whatever their state
        // (a CTA that gave up sends what it has), so neither exits while the other may still be
        // writing into it, and no round waits for a partner that has left.
        float* peer = s.peer + 128 * (t & 1);
        uint64_t* bx = &bar_x[t & 1];
        if (tid < 32) st_async_peer_v4(peer + 4 * tid, bx, r ^ 1u, reinterpret_cast<const float4*>(s.mine)[tid]);
        if (!wait_bar(bx, (uint32_t)((t >> 1) & 1))) ok = false;
        if (__syncthreads_or(!ok)) ok = false;
        if (tid == 0 && t + 2 < T) mbar_arrive_expect_tx(bx, 128 * sizeof(float));   // round t + 2

        // act = silu(G) * U for the slice's 64 columns: G and U of column i are rows 32(i/16) + i%16
        // and 16 rows further of the interleaved m-tile; staged in fp16 for the down GEMV
        if (ok && warp == 0) {
            float a[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int i = 2 * lane + u;
                const int rg = 32 * (i >> 4) + (i & 15), ru = rg + 16;
                const float G = s.mine[rg] + peer[rg], U = s.mine[ru] + peer[ru];
                a[u] = G * U / (1.f + expf(-G));
            }
            const float m = warp_max(fmaxf(fabsf(a[0]), fabsf(a[1])));
            float rsum, undo;
            s.act[lane] = stage_f16(a[0], a[1], lane, m, &rsum, &undo);
            const float hs = half_warp_sum(rsum);
            if ((lane & 15) == 0) s.misc[kMiscAsum0 + (lane >> 4)] = hs;
            if (lane == 0) s.misc[kMiscAsc] = undo;
        }
        bool dok = ok;
        if (ok) dok = wait_bar(&bar_d[dslot], ph);
        if (__syncthreads_or(!dok)) ok = false;

        // down GEMV: DM output m-tiles x 128 rows x this slice's 64 columns
        if (ok) {
            uint4 av[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) av[i] = reinterpret_cast<const uint4*>(s.act + 16 * hh)[i];
            const float asc = s.misc[kMiscAsc], asum = s.misc[kMiscAsum0 + hh];
            // this thread's blocks b = par, par + 2, ... of the DM
            const uint8_t* dbase = s.wdn + (size_t)dslot * g.DM * kBlockBytes;
            float* yd = s.ydn + hh * g.DM * 128 + row;
#pragma unroll 2
            for (int b = par; b < g.DM; b += 2) {
                const uint8_t* blk = dbase + (size_t)b * kBlockBytes;
                const uint4 cw = *reinterpret_cast<const uint4*>(blk + hh * 2048 + row * 16);
                const uint32_t sb = *reinterpret_cast<const uint32_t*>(blk + kBlockCodeBytes + row * 4);
                const float P = dot32h(cw, av);
                const float sc = __half2float(__ushort_as_half((unsigned short)(sb & 0xFFFFu)));
                const float bi = __half2float(__ushort_as_half((unsigned short)(sb >> 16)));
                yd[b * 128] = sc * (P * asc) + bi * asum;
            }
        }
        __syncthreads();
        // the down buffer is read: the next token's expert streams into it
        if (TM > 1 && routed && ok && t + 1 < T && warp == 1) issue_down(s.ints[kIntSel + t + 1], dslot);
        if (ok) {
            const float gate = s.misc[kMiscGate + t];
            const int nrow = g.DM * 128;
            float* dst = c.dfz.outacc + (size_t)t * H + (size_t)g.DM * r * 128;
            for (int i4 = tid; 4 * i4 < nrow; i4 += kDThreads) {
                const float4 y0 = reinterpret_cast<const float4*>(s.ydn)[i4];
                const float4 y1 = reinterpret_cast<const float4*>(s.ydn + nrow)[i4];
                red_add_v4(dst + 4 * i4, (y0.x + y1.x) * gate, (y0.y + y1.y) * gate, (y0.z + y1.z) * gate,
                           (y0.w + y1.w) * gate);
            }
        }
        __syncthreads();
        // one arrival per 128-row chunk of this token; the counter values are read after the
        // last token, so the round trip overlaps the next token's work
        if (ok && tid < g.DM) {
#pragma unroll
            for (int u = 0; u < TM; ++u)
                if (u == t) arrivals[u] = atom_add_acq_rel(c.dfz.cnt + (size_t)t * MTd + g.DM * (int)r + tid, 1u);
        }
    }
    // the last of the units to arrive at a (token, chunk) finalises it: bf16 out, accumulator and
    // counter back to zero
    if (ok && tid < g.DM) {
#pragma unroll
        for (int u = 0; u < TM; ++u)
            if (u < T) s.ints[kIntFlags + u * kMaxDM + tid] = (arrivals[u] == (unsigned)(g.units - 1)) ? 1 : 0;
    }
    __syncthreads();
    if (ok) {
        for (int t = 0; t < T; ++t) {
            // four rows per thread: 16-byte reads at L2 (after the counter's acquire, through the
            // barrier) and zeroing stores, 8-byte bf16 stores
            for (int i4 = tid; 4 * i4 < g.DM * 128; i4 += kDThreads) {
                if (!s.ints[kIntFlags + t * kMaxDM + ((4 * i4) >> 7)]) continue;
                const size_t hrow = (size_t)g.DM * r * 128 + 4 * (size_t)i4;
                float4* src = reinterpret_cast<float4*>(c.dfz.outacc + (size_t)t * H + hrow);
                const float4 v = __ldcg(src);
                __stcg(src, make_float4(0.f, 0.f, 0.f, 0.f));
                const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
                *reinterpret_cast<uint2*>(c.out + (size_t)t * H + hrow) =
                    make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
            }
            if (tid < g.DM && s.ints[kIntFlags + t * kMaxDM + tid])
                atomicExch(c.dfz.cnt + (size_t)t * MTd + g.DM * (int)r + tid, 0u);
        }
    }
    if (!ok && tid == 0) {
        set_status(c.status, MOE_STATUS_TIMEOUT);
        atomicOr(c.dfz.dirty, 1u);
    }
    // nothing may still be landing in this CTA's shared memory when it exits: the last wave
    // issued into each buffer has landed (earlier ones were waited for, or precede it)
    if (tid == 0) {
        if (need_r) mbar_drain(bar_r, 0);
        for (int sl = 0; sl < g.nslots; ++sl) {
            const int wg = s.ints[kIntWavesG + sl];
            if (wg > 0) mbar_drain(&bar_g[sl], (uint32_t)((wg - 1) & 1));
        }
        for (int ds = 0; ds < kDSlots; ++ds) {
            const int wd = s.ints[kIntWavesD + ds];
            if (wd > 0) mbar_drain(&bar_d[ds], (uint32_t)((wd - 1) & 1));
        }
    }
    __syncthreads();
}

}  // namespace

// Launch geometry of the fused kernel for a layer shape, or false when the shape does not fit it
// (the multi-kernel GEMV chain then serves batch-1 decode).
bool decode_fused_geometry(int H, int I, int E, int k, int has_shared, int tm, DecodeGeom* out) {
    DecodeGeom g{};
    if (H % 256 != 0 || I % 64 != 0) return false;
    if (tm != 1 && tm != kDecodeFusedMaxT) return false;
    g.tm = tm;
    g.MTg = I / 64;
    g.units = (k + has_shared) * g.MTg;
    g.NR = 2 * k * g.MTg;
    g.R = (E + g.NR - 1) / g.NR;
    if (g.R > kMaxRouterRows) return false;
    g.KH = H / 128;
    g.nch = g.KH < 4 ? g.KH : 4;
    if (g.KH % g.nch != 0) return false;
    g.cblk = g.KH / g.nch;
    if (g.cblk > kMaxChunkBlocks) return false;
    g.nslots = g.nch;
    if (g.nslots > kMaxSlots) return false;
    g.DM = H / 256;
    if (g.DM > kMaxDM) return false;   // also bounds the chunk flags in the ints area
    auto al = [](size_t v) { return (v + 127) / 128 * 128; };
    const size_t TM = (size_t)tm;
    size_t o = 0;
    g.off_wgu = o; o = al(o + (size_t)g.nslots * g.cblk * kBlockBytes);
    g.off_wdn = o; o = al(o + (size_t)g.DM * kBlockBytes);
    g.off_rrow = o; o = al(o + sizeof(float) * (size_t)g.R * H);
    g.off_sgw = o; o = al(o + sizeof(float) * (size_t)H);
    g.off_xraw = o; o = al(o + sizeof(uint16_t) * TM * H);
    g.off_xs = o; o = al(o + sizeof(uint32_t) * TM * (H / 2));
    g.off_xsum = o; o = al(o + sizeof(float) * TM * (H / 32));
    g.off_xsc = o; o = al(o + sizeof(float) * TM * (H / 64));
    g.off_part = o; o = al(o + sizeof(float) * (4 * 128 + 128 + 2 * 128 + 64 + 32));
    g.off_ydn = o; o = al(o + sizeof(float) * 2 * (size_t)g.DM * 128);
    g.off_logit = o; o = al(o + sizeof(float) * kDWarps * TM * kRedStride + sizeof(int) * kNumInts);
    g.off_bars = o; o = al(o + sizeof(uint64_t) * (5 + (size_t)g.nslots));
    g.smem = (int)o;
    if (g.smem > 227 * 1024) return false;
    *out = g;
    return true;
}

cudaError_t decode_fused_prepare(const DecodeGeom& g) {
    if (g.tm == 1) return cudaFuncSetAttribute(decode_fused_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, g.smem);
    return cudaFuncSetAttribute(decode_fused_kernel<kDecodeFusedMaxT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                g.smem);
}

// Clusters of the fused kernel that fit on the device at once (all must be resident together).
cudaError_t decode_fused_max_clusters(const DecodeGeom& g, int* n) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * g.units);
    cfg.blockDim = dim3(kDThreads);
    cfg.dynamicSmemBytes = g.smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (g.tm == 1) return cudaOccupancyMaxActiveClusters(n, decode_fused_kernel<1>, &cfg);
    return cudaOccupancyMaxActiveClusters(n, decode_fused_kernel<kDecodeFusedMaxT>, &cfg);
}

// One launch for c.T tokens (1 <= c.T <= g.tm) with geometry g (decode_fused_geometry of g.tm).
cudaError_t launch_decode_fused(const Ctx& c, const DecodeGeom& g, cudaStream_t st) {
    if (c.T < 1 || c.T > g.tm) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * g.units);
    cfg.blockDim = dim3(kDThreads);
    cfg.dynamicSmemBytes = g.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlaps the launch with the previous kernel's tail
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (g.tm == 1) return cudaLaunchKernelEx(&cfg, decode_fused_kernel<1>, c, g);
    return cudaLaunchKernelEx(&cfg, decode_fused_kernel<kDecodeFusedMaxT>, c, g);
}

}  // namespace moe
