// Internal launch interfaces shared by the .cu files of the library.
#pragma once

#include <algorithm>
#include <cstddef>

#include "common.cuh"

namespace moe {

// Launches a kernel with cudaLaunchKernelEx; with `pdl` the launch may begin
// while the previous kernel on the stream is still running (programmatic
// dependent launch); every kernel calls griddepcontrol.wait before it reads
// what its predecessor wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     bool pdl, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- S1/S2
// Limits of the routing and permutation kernels (the scan's shared-memory tables are sized
// for these): experts E, experts plus redundant slots E + B, and top-k.
constexpr int kMaxExperts = 1024;
constexpr int kMaxRows = 2 * kMaxExperts;
constexpr int kMaxTopk = 32;

cudaError_t launch_route_topk(const float* logits, int T, int E, int topk, int32_t* ids, float* w,
                              cudaStream_t st, bool pdl);

struct PermuteWs {
    int nblk;
    size_t blkcnt, blkoff, total, nrep, rep_ptr, rep_rows, rowstart, bytes;
};
PermuteWs permute_ws_layout(int T, int topk, int E, int B);
cudaError_t launch_permute(const int32_t* ids, const float* topk_w, int T, int topk, int E, int B,
                           const int32_t* replica_src, int32_t* cu_seqlens, int32_t* perm_token,
                           float* perm_w, int32_t* inv_perm, DevError* err, char* scratch,
                           cudaStream_t st, bool pdl);
// Routing (softmax -> top-k -> renormalise) and the permutation of 1 <= T <= 256 tokens in one
// launch; the same outputs as launch_route_topk followed by launch_permute.
cudaError_t launch_route_permute_one_block(const float* logits, int T, int E, int topk, int32_t* ids, float* w,
                                          int B, const int32_t* replica_src, int32_t* cu_seqlens,
                                          int32_t* perm_token, float* perm_w, int32_t* inv_perm, DevError* err,
                                          char* ws, cudaStream_t st, bool pdl);
cudaError_t launch_gather(int mode, const void* src, int H, const int32_t* perm_token, int NvS,
                          void* dst, const float* src_scale, float* dst_scale, cudaStream_t st,
                          bool pdl);
cudaError_t launch_rows_to_f16(const void* src, bool in_f32, int R, int K, __half* dst, float* scale,
                               cudaStream_t st, bool pdl);

// ---------------------------------------------------------------- S4/S6/S2q
cudaError_t launch_act_and_mul(const __nv_bfloat16* gate, const __nv_bfloat16* up,
                               const float* perm_w, int M, int I, int act, float sa, float sb,
                               __nv_bfloat16* out, cudaStream_t st, bool pdl);
// The same for a grid of CTA pairs (clusters of two CTAs; grid.x even).
template <typename... KArgs, typename... Args>
cudaError_t launch_k_pairs(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                           bool pdl, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

cudaError_t launch_combine(const __nv_bfloat16* y, const int32_t* inv_perm, const float* topk_w,
                           int T, int topk, int H, __nv_bfloat16* out, cudaStream_t st, bool pdl);
cudaError_t launch_combine_f32(const float* y, const int32_t* inv_perm, const float* topk_w, int T,
                               int topk, int H, __nv_bfloat16* out, cudaStream_t st, bool pdl);
// Rows [R, K] (bf16 or fp32, K % 32 == 0) -> e4m3 codes with one e8m0 scale per 32 values,
// Kp = mx8_kpad(K) codes per row (zero past K). two: hi and lo terms, scale chosen so the
// block max stays <= 448 (lo != nullptr); else one term with the OCP MX MXFP8 scale.
// Codes rows are code_stride bytes apart, scale rows sc_stride.
// With row_idx, output row r is taken from input row row_idx[r] (of in_rows): the staging of
// gathered rows in one pass.
cudaError_t launch_quant_mx8(const void* in, bool in_f32, int R, int K, int Kp, bool two, uint8_t* hi, uint8_t* lo,
                             uint8_t* sc, int code_stride, int sc_stride, cudaStream_t st, bool pdl,
                             const int32_t* row_idx = nullptr, int in_rows = 0);
// codes / sb rows are codes_stride / sb_stride bytes apart (K/2 and K/16 when dense); row_idx
// as for launch_quant_mx8.
cudaError_t launch_quant_nvfp4(const void* in, bool in_f32, int R, int K, uint8_t* codes, int codes_stride,
                               uint8_t* sb, int sb_stride, float* s, __half* deq, cudaStream_t st, bool pdl,
                               const int32_t* row_idx = nullptr, int in_rows = 0);

// ---------------------------------------------------------------- grouped GEMM
// Output kinds of the GEMM epilogue.
// OUT_MX8: the activation rows as the MXFP4 GEMM's operand records (see kMx8StageK below):
// e4m3 codes (hi and lo, or one term) and one e8m0 scale per 32 values, straight from the
// gate/up epilogue.
enum OutKind { OUT_BF16 = 0, OUT_F16 = 1, OUT_F32 = 2, OUT_MX8 = 3 };

struct GemmProblem {
    // tokens: [M_alloc, K] bf16 (BF16 weights) or f16 (FP4 weights), row-major
    const void* x;
    int M_alloc;
    const int32_t* cu_seqlens;  // [G] inclusive ends, device
    int G, N, K;
    int wfmt;                   // moe_wfmt_t
    bool dual;                  // gate+up with the activation epilogue
    // weights: BF16 [G,N,K] (w0 = gate or plain, w1 = up)
    const void* w0;
    const void* w1;
    // FP4 kernel format (prepared)
    const void* kdata0;
    const void* kscale0;
    const void* kdata1;
    const void* kscale1;
    const float* alpha0;        // per-row global scale or NULL
    const float* alpha1;
    const float* perm_w;        // route weight per token row (dual only) or NULL
    const float* tscale;        // per token-row scale or NULL
    float out_scale;
    int act;
    float situ_a, situ_b;
    void* out;                  // [M_alloc, N]
    int out_kind;               // OutKind
    bool zero_pad;              // write zeros to rows [cu[G-1], M_alloc)
    int bt;                     // token tile (0 = choose)
    DevError* err;
    // Block-scaled NVFP4 path (nvf4): x = packed e2m1 token rows (x_stride bytes apart),
    // xsf = their e4m3 block scales (xsf_stride bytes apart), tscale = the row scales,
    // kscale0/1 = the weights' block-scaled tiles. Needs K % kNvf4StageK == 0.
    bool nvf4;
    int x_stride;
    const void* xsf;
    int xsf_stride;
    // MXFP4 weights (mx8 = number of e4m3 terms per activation: 2 = hi/lo staging of bf16,
    // 1 = MXFP8 activations): x = records of mx8 * Kp codes then the scales (x_stride bytes
    // apart), kdata0/1 = the padded codes, kscale0/1 = the scale blocks.
    int mx8;
    // Per-expert fp32 biases [G, N] or NULL (gemm1_bias / gemm2_bias): the dual GEMM adds
    // bias0 to gate and bias1 to up before the activation; a single GEMM adds
    // bias_rw[row] * bias0 to its (scaled) output, bias_rw NULL meaning 1.
    const float* bias0;
    const float* bias1;
    const float* bias_rw;
    float sw_alpha, sw_beta, sw_limit;  // SWIGLUOAI (act == MOE_ACT_SWIGLUOAI)
    // OUT_MX8: records of out_terms e4m3 terms (2: hi/lo, 1: MXFP8), out_stride bytes apart
    int out_terms, out_stride;
    // BF16 gate/up (128-token tiles, or CTA pairs): token row r is row gather_idx[r] of
    // x [gather_rows, K] (the permutation's perm_token), so no pre-gathered copy is needed
    const int32_t* gather_idx;
    int gather_rows;
};
cudaError_t launch_grouped_gemm(const GemmProblem& p, cudaStream_t st, bool pdl);
bool gemm_can_gather(const GemmProblem& p);
int choose_token_tile(long long NvS, int G, bool wide_ok);

// FP4 kernel layout: tiles of 128 weight rows x 64 K values.
constexpr int kTileN = 128;
constexpr int kTileK = 64;
inline int fp4_scale_bytes_per_row(int wfmt) { return wfmt == MOE_W_MXFP4 ? 2 : 4; }
// Prepared FP4 chunk (128 rows x 64 K): codes then scales, contiguous.
inline int fp4_chunk_bytes(int wfmt) { return kTileN * 32 + kTileN * fp4_scale_bytes_per_row(wfmt); }
constexpr int kFp4StageK = 128;  // K values per FP4 pipeline stage (two chunks)

// Block-scaled NVFP4 tiles (weights used with NVFP4 activations): 128 weight rows x
// 256 K values per tile, one pipeline stage. A tile is the 16384-byte image of the rows'
// packed codes as the 128-byte swizzle lays them out in shared memory (row m at 128*m,
// its 16-byte chunk c at chunk position c ^ (m % 8)), then four 512-byte scale blocks,
// one per 64 K values j: byte 16*(m % 32) + 4*(m / 32) + i holds the e4m3 scale of
// values [64j + 16i, 64j + 16i + 16) of row m (the order the scale-factor copy into
// tensor memory reads).
constexpr int kNvf4StageK = 256;
constexpr int kNvf4CodeBytes = kTileN * kNvf4StageK / 2;   // 16384
constexpr int kNvf4SfBytes = 4 * 512;
constexpr int kNvf4TileBytes = kNvf4CodeBytes + kNvf4SfBytes;  // 18432

// MXFP4 weights for the block-scaled MXFP4 x MXFP8 GEMM: kdata = packed e2m1 codes
// [G, N, Kp/2] with K zero-padded to Kp = a multiple of 128 (what the 4-bit tensor map
// needs), kscale = one 512-byte scale block per (g, 128-row block nt, 128-K block kb),
// byte 16*(m % 32) + 4*(m / 32) + i = the e8m0 scale of values [128kb + 32i, +32) of
// row m. Activations are records of Kp "hi" e4m3 codes, Kp "lo" e4m3 codes and Kp/32
// e8m0 block scales padded to 16 bytes: value = (hi + lo) * 2^(scale - 127).
constexpr int kMx8StageK = 128;
inline int mx8_kpad(int K) { return (K + kMx8StageK - 1) / kMx8StageK * kMx8StageK; }
inline int mx8_scale_bytes(int K) { return (mx8_kpad(K) / 32 + 15) / 16 * 16; }
inline int mx8_rec_bytes(int K, int terms = 2) { return terms * mx8_kpad(K) + mx8_scale_bytes(K); }
// W4A8 (dynamic MXFP8 activations): one e4m3 term per value instead of hi/lo, with the
// OCP MX scale 2^(floor(log2 amax) - 8); records of mx8_rec_bytes(K, 1) bytes.

// ---------------------------------------------------------------- device info
int num_sms();

}  // namespace moe
