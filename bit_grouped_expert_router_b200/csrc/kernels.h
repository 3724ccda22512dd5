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

// Workspace of the fused batch-1 decode kernel.  outacc and cnt are zero between calls (the
// kernel re-zeroes what it used); bar holds grid-barrier arrival counts (between calls each a
// multiple of the number of CTAs that arrive on it).
struct DecodeFusedWs {
    float* rpart;    // [4][E] quarter-row router partial logits
    float* gu;       // [k+1][4][2I] gate/up k-range partial sums
    float* outacc;   // [H] fp32 output accumulator
    unsigned* cnt;   // [H/32] arrivals per 32-row output chunk
    unsigned long long* bar;   // [16 x 32] grid-barrier arrival counters (256 B apart), only ever incremented
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
    unsigned int* counters;
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
int router_tc_splits();
cudaError_t launch_topk(const Ctx& c, bool histogram, cudaStream_t st);
cudaError_t launch_bucket_scan(const Ctx& c, cudaStream_t st);
cudaError_t launch_scatter(const Ctx& c, cudaStream_t st);

// Token-tile TMA maps of one grouped GEMM: m[source][h] with box {64 columns, 64 << h rows}.
// gate/up: source 0 = bucketed rows xp, source 1 = the activations x16 (shared expert);
// down: source 0 = act (source 1 unused).
struct TokenMaps {
    CUtensorMap m[2][3];
};

// prefill grouped GEMMs
cudaError_t launch_gather_rows(const Ctx& c, int num_sms, cudaStream_t st);
cudaError_t launch_gemm_gateup(const Ctx& c, const TokenMaps& maps, int num_sms, cudaStream_t st);
cudaError_t launch_gemm_down(const Ctx& c, const TokenMaps& maps, int num_sms, cudaStream_t st);
cudaError_t launch_finalize(const Ctx& c, cudaStream_t st);
// Token rows per grouped-GEMM tile for a call of T tokens: 128 (two CTAs per SM) when the
// routed experts average at most 64 tokens (T * k <= 64 * E), else 256 (one CTA per SM).
int gemm_tile_rows(int T, int k, int E);

// host-side error text for moe_last_error() (defined in api.cu)
void set_last_error(const char* msg);

// decode sparse GEMV
cudaError_t launch_decode_fused(const Ctx& c, int num_sms, cudaStream_t st);
int decode_fused_smem_bytes(int H, int I);
cudaError_t launch_gemv_gateup(const Ctx& c, cudaStream_t st);
cudaError_t launch_gemv_down(const Ctx& c, cudaStream_t st);

}  // namespace moe
