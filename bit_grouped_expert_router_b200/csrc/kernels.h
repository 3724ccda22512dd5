// kernels.h -- internal interface between the C-ABI host code (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// Tile geometry of the prefill grouped GEMMs (tokens per tile = UMMA N).
constexpr int kBN = 256;          // largest token tile of the grouped GEMMs (= UMMA N); tile lists are sized by 128
constexpr int kStages = 3;        // pipeline depth (shared-memory stages)
constexpr int kTokPerBucketBlk = 64;  // tokens per routing/bucketing CTA
constexpr int kRouterTT = 32;     // tokens per CTA in the SIMT router (prefill sizes)
constexpr int kRouterTTSmall = 8; // tokens per CTA in the SIMT router (decode sizes)
constexpr int kRouterKSlice = 32; // input columns per CTA in the split-K SIMT router

struct RepackArgs {
    const uint32_t* q[2];
    const uint16_t* s[2];
    const uint16_t* b[2];
    const uint32_t* qs[2];
    const uint16_t* ss[2];
    const uint16_t* bs[2];
    int E;             // routed experts (group E = shared)
    int rows_per_mat;  // rows of one source matrix (I for gate/up, H for down)
    int cols;          // input columns (H for gate/up, I for down)
    int gateup;        // 1: interleave gate/up rows; 0: plain rows
    uint8_t* dst;
    uint32_t* inexact;
};

// Workspace of the fused batch-1 decode kernel (zero when the handle is created).
// Tokens one launch of the fused decode kernel serves (its per-token buffers are sized for this).
constexpr int kDecodeFusedMaxT = 8;

struct DecodeFusedWs {
    unsigned long long* ticket;   // [1] CTAs started, over all calls (call number = ticket / CTAs per call)
    unsigned long long* slots;    // [kDecodeFusedMaxT][E] router logit of (token, expert) as (call tag << 32) | fp32 bits
    float* outacc;                // [kDecodeFusedMaxT][H] fp32 output accumulators; zero between calls
    unsigned* cnt;                // [kDecodeFusedMaxT][H/128] unit arrivals per 128-row output chunk; zero between calls
    unsigned* dirty;              // [1] raised by a call that gave up part-way; the next call resets
};

// Launch geometry and shared-memory carve-up of the fused batch-1 decode kernel (host-computed).
struct DecodeGeom {
    int MTg;      // 64-column slices of I (gate/up m-tiles of 128 interleaved rows)
    int units;    // (k + has_shared) * MTg work units, one 2-CTA cluster each
    int NR;       // routed CTAs (2 * k * MTg): router rows are dealt to them
    int R;        // router rows per routed CTA (ceil(E / NR))
    int KH;       // gate/up blocks per CTA (H / 128: one input-column half)
    int nch;      // landing chunks of the gate/up copy
    int cblk;     // gate/up blocks per chunk (KH / nch)
    int nslots;   // gate/up chunk buffers (nch)
    int tm;       // the most tokens a launch with this geometry serves (1 or kDecodeFusedMaxT)
    int DM;       // down blocks per CTA (H / 256 output m-tiles)
    int smem;     // dynamic shared memory bytes
    size_t off_wgu, off_wdn, off_rrow, off_sgw, off_xraw, off_xs, off_xsum, off_xsc, off_part, off_ydn, off_logit, off_bars;
};

// Everything a forward-path kernel needs (passed by value).
struct Ctx {
    int T, H, I, E, k, G, has_shared;
    int nblk;          // routing/bucketing CTAs for T tokens
    int ks;            // K slices of the router partial logits
    int max_tiles;     // capacity of each tile list
    int tile_rows;     // token rows per grouped-GEMM tile (128 or 256), set per call
    int rows_cap;      // row capacity of xp / act
    uint32_t flags;
    // weights, kernel layout
    const uint8_t* w_gu;
    const uint8_t* w_dn;
    const float* wrt;
    const float* router32;   // router fp32 [E][H] (public layout copy)
    const float* rbias;
    const float* sgw;
    // call inputs / outputs
    const uint16_t* x;
    uint16_t* out;
    // workspace
    float* part;
    int* idx;
    float* gates;
    float* sg;
    int* hist;
    unsigned* scatter_done;   // [1] scatter CTAs finished in this call (the last resets it to 0)
    int* counts;
    int* offsets;
    int4* tiles1;      // grouped-GEMM tile list {group, first bucket row, rows, 0}, ntiles[0] entries
    int4* tiles2;      // the same list (both GEMMs walk one list; kept as a separate name)
    int* ntiles;
    int* perm;
    int* row_token;
    float* row_gate;
    __half* x16;      // [T][H] fp16 copy of the activations (prefill path)
    __half* xp;       // [T*k][H] fp16 token rows in bucket order (routed experts)
    __half* act;
    float* acc;
    float* dact;
    float* dscale;
    uint32_t* status;
    DecodeFusedWs dfz;
};

cudaError_t launch_repack(const RepackArgs& a, int groups, int m_tiles, int k_steps, cudaStream_t st);
cudaError_t launch_router_prep(const float* router, const float* bias, const float* sgw, int H, int E,
                               float* wrt, float* bias_out, float* sgw_out, cudaStream_t st);

// routing + bucketing
cudaError_t launch_router_simt(const Ctx& c, cudaStream_t st);
cudaError_t launch_router_split(const float* router, int H, int E, int Epad, uint16_t* wsplit, cudaStream_t st);
cudaError_t launch_router_tc(const Ctx& c, const CUtensorMap& tmW, const CUtensorMap& tmX, int n_exp,
                             cudaStream_t st);
int router_tc_smem_bytes();
int router_tc_splits(int T, int H);   // partial sums of the tensor-core router, T tokens of H
cudaError_t launch_topk(const Ctx& c, bool histogram, cudaStream_t st);
cudaError_t launch_routing_supplied(const Ctx& c, const int* idx, const float* gates, const float* sg,
                                    bool prefill, cudaStream_t st);
cudaError_t launch_scatter(const Ctx& c, cudaStream_t st);

// Rows of the token-tile TMA box with selector h: 64, 128 or 256 (a tile of n tokens loads the
// smallest box that holds n rows; the one-CTA GEMM shape has tiles of up to 256 tokens, the
// two-CTA shape 128).
__host__ __device__ constexpr int token_box_rows(int h) { return 64 << h; }

// Token-tile TMA maps of one grouped GEMM: m[source][h] with box {64 columns, token_box_rows(h) rows}.
// gate/up: source 0 = bucketed rows xp, source 1 = the activations x16 (shared expert);
// down: source 0 = act (source 1 unused).
struct TokenMaps {
    CUtensorMap m[2][3];
};

// prefill grouped GEMMs
cudaError_t launch_gather_rows(const Ctx& c, int num_sms, cudaStream_t st);
// amap: NULL for the in-GEMM 4-bit dequantisation; else the tensor map of the layer's weights
// dequantised once to fp16 in HBM (the ablation variant, box 64 columns x 128 rows)
cudaError_t launch_gemm_gateup(const Ctx& c, const TokenMaps& maps, const CUtensorMap* amap, int num_sms,
                               cudaStream_t st);
cudaError_t launch_gemm_down(const Ctx& c, const TokenMaps& maps, const CUtensorMap* amap, int num_sms,
                             cudaStream_t st);
// Writes the layer's repacked 4-bit blocks of one matrix kind as fp16 rows: dst[(g*MT + mt)*128 + l]
// [64*kc + j] = the weight the grouped GEMM's transform would put in row l, column j of block
// (g, mt, kc) (the ablation's weights in HBM).
cudaError_t launch_dequant_rows(const uint8_t* blocks, int groups, int m_tiles, int k_steps, __half* dst,
                                cudaStream_t st);
cudaError_t launch_finalize(const Ctx& c, cudaStream_t st);
cudaError_t launch_combine_rows(const uint16_t* rows, int n_rows, const int* pos, int T, int k, int H,
                                const uint16_t* base, uint16_t* out, uint32_t* status, int num_sms, cudaStream_t st);
// Token rows per grouped-GEMM tile for a call of T tokens: 128 (two CTAs per SM) when the
// routed experts average at most 64 tokens (T * k <= 64 * E), else 256 (one CTA per SM).
int gemm_tile_rows(int T, int k, int E);

// host-side error text for moe_last_error() (defined in api.cu)
void set_last_error(const char* msg);

// decode sparse GEMV
// tm: 1 (the single-token form) or kDecodeFusedMaxT (1..kDecodeFusedMaxT tokens per launch)
bool decode_fused_geometry(int H, int I, int E, int k, int has_shared, int tm, DecodeGeom* out);
cudaError_t decode_fused_prepare(const DecodeGeom& g);
cudaError_t decode_fused_max_clusters(const DecodeGeom& g, int* n);
cudaError_t launch_decode_fused(const Ctx& c, const DecodeGeom& g, cudaStream_t st);
cudaError_t launch_gemv_gateup(const Ctx& c, cudaStream_t st);
cudaError_t launch_gemv_down(const Ctx& c, cudaStream_t st);

}  // namespace moe
