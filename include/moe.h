/*
 * moe.h — C ABI of the B200 (sm_100a) fused MoE expert layer.
 *
 * The layer, as the pages state it (vLLM API pages for the MoonEP experts,
 * FlashInfer MoE-EP experts, DeepSeek-V4 FlashInfer MoE and TRTLLM MXFP4
 * experts):
 *
 *   top-k routing -> permute into expert-contiguous segments (cu_seqlens over
 *   E experts plus B redundant slots) -> gate and up grouped GEMMs -> gated
 *   activation times the route weight -> down grouped GEMM -> top-k combine.
 *
 * Conventions for every entry point:
 *   - Pointers named in a signature are DEVICE pointers unless stated otherwise,
 *     owned by the caller, 16-byte aligned (TMA operands: 128-byte aligned is
 *     not needed, 16 is). The library never allocates on these paths.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Launches are
 *     asynchronous; nothing synchronises except moe_get_device_error and
 *     moe_prepare_weights.
 *   - Host-side validation returns a status with nothing launched. Nothing
 *     throws across the ABI. Errors a kernel detects (an out-of-range expert id,
 *     a pipeline wait that timed out) are written to an error word at the start
 *     of the caller's workspace and read back with moe_get_device_error.
 *   - bf16 is IEEE-style bfloat16 stored as uint16; rounding to it is RNE.
 *   - T = 0 (no tokens) is a no-op that returns MOE_OK.
 */
#ifndef MOE_B200_MOE_H
#define MOE_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* moe_stream_t; /* a cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,         /* a size, pointer or scalar argument is out of range */
    MOE_ERR_UNSUPPORTED = 2,         /* valid, but this format/activation/shape is not implemented */
    MOE_ERR_ALIGNMENT = 3,           /* K not a multiple of the block size, or a misaligned pointer */
    MOE_ERR_WORKSPACE_TOO_SMALL = 4,
    MOE_ERR_CUDA = 5,                /* a CUDA runtime/driver call failed */
    MOE_ERR_DEVICE = 6,              /* a kernel reported bad data (e.g. an expert id >= E) */
    MOE_ERR_TIMEOUT = 7,             /* a kernel's bounded pipeline wait ran out */
    MOE_ERR_NOT_PREPARED = 8         /* FP4 weights used before moe_prepare_weights */
} moe_status_t;

typedef enum { MOE_ACT_SILU = 0, MOE_ACT_SITU = 1, MOE_ACT_SWIGLUOAI = 2 } moe_act_t;

typedef enum { MOE_W_BF16 = 0, MOE_W_MXFP4 = 1, MOE_W_NVFP4 = 2 } moe_wfmt_t;

/*
 * One projection's weights, G = E + B rows ([E, E+B) are the redundant slots),
 * each an [N, K] matrix with K (the reduction axis) contiguous — the
 * `[G, N, K]` convention of the MoonEP page's moonep_grouped_gemm.
 *
 *   data  : BF16  -> bf16 [G,N,K]
 *           MXFP4 -> uint8 [G,N,K/2] packed e2m1, even k in the low nibble
 *           NVFP4 -> same packing
 *   scale : MXFP4 -> uint8 e8m0 [G,N,K/32] (value 2^(s-127)), the MXFP4 format
 *                    of the TRTLLM MXFP4 page (kMxfp4Static)
 *           NVFP4 -> uint8 fp8-e4m3 [G,N,K/16], the w13/w2_weight_scale planes of
 *                    the DeepSeek-V4 FI page (_realloc_nvfp4_params)
 *           BF16  -> NULL
 *   alpha : NULL (=1) or fp32 [G], a per-row global scale applied in the GEMM
 *           epilogue: NVFP4 weight_scale_2 (FlashInfer MoE-EP page,
 *           epilogue_from_quant_config: finite, > 0, one per expert).
 *   kdata, kscale, kalpha : the kernel-format copy that moe_prepare_weights
 *           writes into caller memory; NULL until then. BF16 needs none.
 *           NVFP4 kdata: tiles of 128 rows x 64 K (codes, then scales) for the GEMM
 *           that stages the weights as f16; kscale: for K % 256 == 0, tiles of 128
 *           rows x 256 K for the block-scaled GEMM (moe_grouped_gemm_nvfp4), else
 *           equal to kdata. MXFP4 kdata: the codes with K padded to a multiple of
 *           128; kscale: the e8m0 scales in 128 x 128 blocks. kalpha: the epilogue
 *           alphas.
 */
typedef struct {
    int32_t fmt;            /* moe_wfmt_t */
    int32_t G, N, K;
    const void* data;
    const void* scale;
    const float* alpha;
    const void* kdata;
    const void* kscale;
    const float* kalpha;
} moe_weight_t;

/* Gated activation. SITU (TRTLLM MXFP4 page, TrtLlmMxfp4ExpertsBase, SITU
 * comment): left = situ_alpha*tanh(g/situ_alpha)*sigmoid(g),
 * right = situ_beta*tanh(u/situ_beta); both must be > 0 (else INVALID_ARG).
 * SILU: silu(g)*u (MoonEP page, module docstring). SWIGLUOAI takes three more
 * parameters and is described with moe_act_ex_t. */
typedef struct {
    int32_t act;            /* moe_act_t */
    float situ_alpha;       /* activation_situ_beta */
    float situ_beta;        /* activation_situ_linear_beta */
} moe_act_params_t;

const char* moe_status_string(moe_status_t s);

/* Library version string and the compute capability the kernels target. */
const char* moe_version(void);

/*
 * S1 — top-k routing, softmax -> top-k -> renormalise ("Renormalize" routing
 * of the TRTLLM MXFP4 page, _invoke_kernel; int32 ids as in the FlashInfer
 * MoE-EP page, apply).
 *   logits      fp32 [T,E], finite.
 *   topk_ids    int32 [T,topk] out: experts by descending logit, ties to the
 *               lower id (selection on the fp32 logits).
 *   topk_w      fp32 [T,topk] out: exp(l_j - l_0) / sum_i exp(l_i - l_0).
 * 1 <= topk <= min(E, 32), 1 <= E <= 1024, else INVALID_ARG/UNSUPPORTED.
 */
moe_status_t moe_route_topk(const float* logits, int T, int E, int topk,
                            int32_t* topk_ids, float* topk_w, moe_stream_t stream);

/*
 * S1 (DeepSeekV3) — group-limited top-k on sigmoid scores, the "DeepSeekV3" routing
 * method of the TRTLLM MXFP4 page (_supports_routing_method; apply passes n_group,
 * topk_group, routing_bias = e_score_correction_bias and routed_scaling_factor). The
 * page names the method only; it is taken as the published DeepSeek-V3 routing:
 *   s_e = sigmoid(l_e), c_e = s_e + bias_e (bias may be NULL = 0; it steers selection only);
 *   the E experts form n_group consecutive groups; a group scores the sum of its two
 *   largest c (its one c for groups of one); the topk_group best groups are kept, ties to
 *   the lower group; the topk largest c among their experts are chosen, ties to the lower
 *   id, in that order; topk_w = routed_scaling_factor * s_j / sum of the chosen s.
 *   Decisions are taken in fp64.
 *   logits fp32 [T,E]; bias fp32 [E] or NULL; topk_ids int32 / topk_w fp32 [T,topk] out.
 * E % n_group, 1 <= topk_group <= n_group, 1 <= topk <= topk_group*E/n_group and a finite
 * positive scaling factor, else INVALID_ARG; E > 512, n_group > 32 or topk > 32: UNSUPPORTED.
 */
moe_status_t moe_route_topk_grouped(const float* logits, const float* bias, int T, int E, int topk,
                                    int n_group, int topk_group, float routed_scaling_factor,
                                    int32_t* topk_ids, float* topk_w, moe_stream_t stream);
/*
 * S2 — permute into expert-contiguous segments (MoonEP page: module docstring
 * and MoonEPExperts.apply; cu_seqlens = cumsum of per-row lengths).
 *   topk_ids/topk_w [T,topk]; replica_src int32 [B] (source expert of each
 *   redundant slot, -1 = unused; may be NULL when B == 0).
 *   Outputs, NvS = T*topk:
 *     cu_seqlens int32 [E+B]: inclusive segment end offsets.
 *     perm_token int32 [NvS]: token of each segment row (ascending per segment).
 *     perm_w     fp32 [NvS]:  its route weight.
 *     inv_perm   int32 [T,topk]: segment row of each (token, k).
 *     x_perm     bf16 [M_alloc,H] or NULL: x rows gathered into segment order;
 *                M_alloc >= NvS, rows >= NvS are left untouched.
 *   A replicated expert's n assignments (ascending token) are cut into
 *   contiguous chunks over [e, its slots ascending], chunk i holding
 *   n/R + (i < n%R) rows. Indices are bit-exact with the oracle.
 *   An expert id outside [0,E), or one expert listed twice by a token, sets MOE_ERR_DEVICE
 *   in the workspace error word; the out-of-range assignment gets inv_perm = -1, and the
 *   rows then left without an assignment (from cu_seqlens[E+B-1] to NvS) get token 0 and
 *   weight 0, so that x_perm reads only rows of x.
 *   ws: at least moe_permute_workspace_size(T, topk, E, B) bytes.
 */
size_t moe_permute_workspace_size(int T, int topk, int E, int B);
moe_status_t moe_permute(const int32_t* topk_ids, const float* topk_w, int T, int topk,
                         int E, int B, const int32_t* replica_src,
                         const void* x, int H,
                         int32_t* cu_seqlens, int32_t* perm_token, float* perm_w,
                         int32_t* inv_perm, void* x_perm, int M_alloc,
                         void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_permute without a workspace argument. The pages have no counterpart: it
 * exists for callers that cannot allocate, such as an operator that is handed only
 * its input and output pointers by another runtime, or a serving loop with a fixed
 * memory plan where cudaMalloc (which also synchronises the device) is not allowed.
 * Arguments and results are those of moe_permute, minus ws/ws_bytes; it calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *   Scratch: a 1 MiB array of device memory inside the library, present on every
 *   GPU that loads it until the process exits. Sizes whose scratch would not fit
 *   (about 2*ceil(T/256)*E*4 bytes plus small tables) return
 *   MOE_ERR_WORKSPACE_TOO_SMALL with nothing launched.
 *   The first call on a device looks up that array's device address (with that
 *   device current); make that first call before any stream capture.
 *   All calls share the one array: calls that overlap on the GPU (two streams,
 *   two host threads) race and must be serialised by the caller.
 *   Bad data is handled as in moe_permute: an expert id outside [0,E), or a token
 *   listing one expert twice, is skipped (its inv_perm entry is -1, and the rows
 *   no assignment reaches get token 0 and weight 0); a replica_src entry outside
 *   [-1,E) is ignored. Each sets the call's error word, which lives in the array,
 *   starts at zero at every call and is read by moe_permute_noalloc_status.
 */
moe_status_t moe_permute_noalloc(const int32_t* topk_ids, const float* topk_w, int T, int topk,
                                 int E, int B, const int32_t* replica_src,
                                 const void* x, int H,
                                 int32_t* cu_seqlens, int32_t* perm_token, float* perm_w,
                                 int32_t* inv_perm, void* x_perm, int M_alloc,
                                 moe_stream_t stream);

/*
 * The device-detected status of the last moe_permute_noalloc call on the current
 * device: synchronises `stream`, returns MOE_OK or the code the kernels recorded
 * (MOE_ERR_DEVICE for the bad data above) and clears it. Allocates nothing. Like the
 * call itself it shares the one array: read it before the next call on the device.
 */
moe_status_t moe_permute_noalloc_status(moe_stream_t stream);

/*
 * S3/S5 — grouped GEMM: out[seg_g] = alpha_g * a[seg_g] @ W[g]^T for every
 * cu_seqlens segment; rows [cu_seqlens[G-1], M_alloc) of out are written as zero
 * (MoonEP page, moonep_grouped_gemm). Empty segments are skipped.
 *   a    bf16 [M_alloc, K];   out bf16 [M_alloc, N];   cu_seqlens int32 [G] on device.
 *   w    BF16 weights, or FP4 weights already prepared (else NOT_PREPARED).
 *   NVFP4: each row of a is converted to f16 times a power of two chosen from the
 *   row's max (exact except below 2^-30 of that max); the products with the
 *   exactly-dequantised weights accumulate in fp32 on the tensor cores.
 *   MXFP4: each 32-value block of a row is staged as two e4m3 terms sharing one
 *   e8m0 scale 2^e (the smallest with block max <= 448 * 2^e): hi = e4m3(v/2^e),
 *   lo = e4m3(v/2^e - hi), within 1.07 * 2^-8 |v| + 2^(e-10) of v; the tensor cores
 *   multiply both terms by the e2m1 weights with both block scales applied
 *   (kind::mxf8f6f4) and accumulate in fp32.
 *   ws: at least moe_grouped_gemm_workspace_size(M_alloc, w) bytes.
 */
size_t moe_grouped_gemm_workspace_size(int M_alloc, const moe_weight_t* w);
moe_status_t moe_grouped_gemm(const void* a, int M_alloc, const moe_weight_t* w,
                              const int32_t* cu_seqlens, void* out,
                              void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * S3/S5 with NVFP4 activations — the block-scaled grouped GEMM (FlashInfer MoE-EP page:
 * NVFP4 experts quantise activations inside the kernel; DeepSeek-V4 FI page: fc1/fc2
 * alphas in the epilogue). For every cu_seqlens segment g and row r in it:
 *   out[r, n] = alpha_g * a_s[r] * sum_k e2m1(a[r,k]) * e4m3(a_sb[r,k/16])
 *                                      * e2m1(W[g][n,k]) * e4m3(W_scale[g][n,k/16])
 * with the products summed in fp32 by the tensor cores (kind::mxf4nvf4), rounded once
 * to bf16; rows [cu_seqlens[G-1], M_alloc) of out are written as zero.
 *   a_codes uint8 [M_alloc, K/2] packed e2m1 (even k in the low nibble);
 *   a_sb    uint8 [M_alloc, K/16] e4m3;  a_s fp32 [M_alloc] — the three outputs of
 *           moe_quantize_nvfp4 for the segment-ordered rows.
 *   w       NVFP4 weights prepared by moe_prepare_weights; K % 256 == 0 (else
 *           MOE_ERR_ALIGNMENT); other formats: MOE_ERR_UNSUPPORTED.
 *   out bf16 [M_alloc, N]; cu_seqlens int32 [G] on device.
 *   ws: at least 256 bytes (the error word).
 */
moe_status_t moe_grouped_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_sb, const float* a_s,
                                    int M_alloc, const moe_weight_t* w, const int32_t* cu_seqlens,
                                    void* out, void* ws, size_t ws_bytes, moe_stream_t stream);
/*
 * S4 — gated activation times route weight: out[r,i] = act(gate[r,i], up[r,i]) * perm_w[r]
 * (MoonEP page, MoonEPExperts.apply). gate/up/out bf16 [M, I]; perm_w fp32 [M]
 * or NULL (no scaling). Computed in fp32, rounded once to bf16.
 */
moe_status_t moe_act_and_mul(const void* gate, const void* up, const float* perm_w,
                             int M, int I, moe_act_params_t act, void* out,
                             moe_stream_t stream);

/*
 * Every gated activation with its parameters. SWIGLUOAI is listed among the MXFP4
 * experts' activations, with gemm1_alpha, gemm1_beta and gemm1_clamp_limit set to one
 * value for every local expert (TRTLLM MXFP4 page, TrtLlmMxfp4ExpertsBase:
 * _supports_activation and __init__). The page gives no formula; it is taken as the
 * published GPT-OSS gated activation:
 *   g = min(gate, swiglu_limit),  u = clamp(up, -swiglu_limit, swiglu_limit),
 *   act = g * sigmoid(swiglu_alpha * g) * (u + swiglu_beta)
 * with swiglu_alpha and swiglu_beta finite and swiglu_limit > 0 (+inf: no clamp), else
 * INVALID_ARG. GPT-OSS uses alpha = 1.702, beta = 1, limit = 7.
 */
typedef struct {
    int32_t act;            /* moe_act_t */
    float situ_alpha;       /* SITU, as in moe_act_params_t */
    float situ_beta;
    float swiglu_alpha;     /* SWIGLUOAI: gemm1_alpha */
    float swiglu_beta;      /* gemm1_beta */
    float swiglu_limit;     /* gemm1_clamp_limit */
} moe_act_ex_t;

/*
 * S4 with per-expert biases (TRTLLM MXFP4 page, TrtLlmMxfp4ExpertsModular._invoke_kernel:
 * gemm1_bias is handed to the gate/up GEMM). For every row r of segment g
 * (cu_seqlens[g-1] <= r < cu_seqlens[g], inclusive ends):
 *   out[r,i] = act(gate[r,i] + bias_gate[g,i], up[r,i] + bias_up[g,i]) * perm_w[r]
 * rows r >= cu_seqlens[G-1] are written as zero.
 *   gate, up   [M,I] bf16 (in_is_f32 = 0) or fp32 (in_is_f32 = 1); out bf16 [M,I].
 *   bias_gate, bias_up  fp32 [G,I], or NULL (no bias); perm_w fp32 [M] or NULL (weight 1).
 *   cu_seqlens int32 [G] on device, non-decreasing; G >= 1.
 *   act: any moe_act_t with its parameters (moe_act_ex_t, a HOST pointer).
 * fp32 arithmetic, one bf16 rounding. I % 8 == 0 and 16-byte aligned gate, up, out and
 * biases, else MOE_ERR_ALIGNMENT. moe_act_and_mul answers SWIGLUOAI with UNSUPPORTED,
 * as moe_act_params_t has no room for its parameters.
 */
moe_status_t moe_bias_act_and_mul(const void* gate, const void* up, int in_is_f32,
                                  const float* bias_gate, const float* bias_up,
                                  const int32_t* cu_seqlens, int G, const float* perm_w,
                                  int M, int I, const moe_act_ex_t* act, void* out,
                                  moe_stream_t stream);

/*
 * S6 — combine: out[t] = sum_k w_k * y_perm[inv_perm[t,k]], summed in fp32 in k
 * order and rounded once to bf16 (TRTLLM MXFP4 page, do_finalize). topk_w fp32
 * [T,topk], or NULL when the route weight was already applied (w_k = 1).
 * y_perm bf16 [>= T*topk, H]; out bf16 [T,H]. A negative inv_perm entry (an assignment
 * the permutation refused) contributes nothing.
 */
moe_status_t moe_combine(const void* y_perm, const int32_t* inv_perm, const float* topk_w,
                         int T, int topk, int H, void* out, moe_stream_t stream);

/*
 * S2q — dynamic NVFP4 quantisation of activation rows (FlashInfer MoE-EP page,
 * epilogue_from_quant_config: activations are quantised inside the kernel and
 * the checkpoint's input scales drop out). Per row r, in fp32 with IEEE
 * division: s_r = amax_r/2688; per 16 values sb = e4m3_rne_satfinite(amax_b/(6 s_r));
 * q = e2m1_rne_satfinite(v/(sb*s_r)). A zero row or a zero block scale gives +0 codes.
 *   in       bf16 (in_is_f32 = 0) or fp32 (in_is_f32 = 1) [R,K], K % 16 == 0.
 *   codes    uint8 [R,K/2] packed e2m1 (even k in the low nibble).
 *   sb       uint8 [R,K/16] e4m3.   s  fp32 [R].
 *   deq_f16  optional f16 [R,K]: e2m1(q)*sb, the GEMM operand (s_r applied later).
 */
moe_status_t moe_quantize_nvfp4(const void* in, int in_is_f32, int R, int K,
                                uint8_t* codes, uint8_t* sb, float* s, void* deq_f16,
                                moe_stream_t stream);

/*
 * S2q — dynamic MXFP8 quantisation of activation rows, the activation side of the W4A8 mode
 * of MXFP4 experts (TRTLLM MXFP4 page, _supports_quant_scheme: (kMxfp4Static,
 * kMxfp8Dynamic)). The page names the mode only; the format and rule are OCP MX v1.0
 * MXFP8: per 32 values, scale 2^e with e = floor(log2 amax) - 8 clamped to [-127, 127]
 * (e = -127 for an all-zero block), q = e4m3_rne_satfinite(v / 2^e).
 *   in      bf16 (in_is_f32 = 0) or fp32 (in_is_f32 = 1) [R,K], K % 32 == 0.
 *   codes   uint8 [R,K] e4m3.   scales  uint8 [R,K/32] e8m0 (value 2^(s-127)).
 */
moe_status_t moe_quantize_mxfp8(const void* in, int in_is_f32, int R, int K, uint8_t* codes,
                                uint8_t* scales, moe_stream_t stream);
/*
 * S0 — one-time conversion of FP4 weights into the kernel's tile layout
 * (FlashInfer MoE-EP page, process_weights_after_loading; DeepSeek-V4 FI page,
 * finalize_weights). Untimed; synchronises `stream`.
 *   dst: caller device memory of moe_prepared_weight_bytes(w) bytes. On success
 *   w->kdata/kscale/kalpha point into dst. BF16 weights: no-op, MOE_OK.
 *   An e8m0 NaN scale (255), or a non-finite or non-positive alpha: INVALID_ARG.
 */
size_t moe_prepared_weight_bytes(const moe_weight_t* w);
moe_status_t moe_prepare_weights(moe_weight_t* w, void* dst, size_t dst_bytes,
                                 moe_stream_t stream);

/*
 * The fused layer: S1 -> S2 (-> S2q) -> S3+S4 -> S5 -> S6, launched back to back
 * on one stream (programmatic dependent launch between kernels), no host sync,
 * no allocation. The DeepSeek-V4 FI page's forward (MoEEpTensors: hidden states,
 * ids, weights, fc1/fc2 alpha) and the TRTLLM monolithic apply (router logits in,
 * finalized output out) are the two shapes this mirrors.
 *   x bf16 [T,H]; router_logits fp32 [T,E]; weights [E+B, I, H] gate/up and
 *   [E+B, H, I] down, all in one format; FP4 weights must be prepared.
 *   act_quant = 1: dynamic NVFP4 activations (NVFP4 weights only); each GEMM whose K
 *   (H for gate/up, I for down) is a multiple of 256 then runs block-scaled as in
 *   moe_grouped_gemm_nvfp4, the other one on f16-staged operands.
 *   MXFP4 weights with act_quant = 0 take bf16 activations, staged for the tensor cores
 *   as two e4m3 terms as in moe_grouped_gemm.
 *   act_quant = 2: dynamic MXFP8 activations (MXFP4 weights only, the W4A8 mode): x and
 *   every activation row are quantised as moe_quantize_mxfp8 does, and both GEMMs take
 *   them as e4m3 with their e8m0 scales. Other act_quant values: INVALID_ARG.
 *   apply_topk_in_fc1 = 1 applies the route weight in the activation (default);
 *   0 applies it in the combine (FlashInfer MoE-EP page, apply_topk_in_fc1).
 *   topk_ids_out/topk_w_out: optional [T,topk] copies of the routing.
 *   T <= T_max given to moe_forward_workspace_size, else INVALID_ARG.
 *   stage_events: optional array of MOE_FWD_STAGE_EVENTS caller-created cudaEvent_t,
 *   recorded on `stream` at the stage boundaries: [0] start, [1] after S1 routing,
 *   [2] after S2 permutation/gather (and x quantisation), [3] after S3+S4 gate/up
 *   GEMM, [4] after the activation row pass (== [3] when there is none),
 *   [5] after S5 down GEMM, [6] after S6 combine. Recording an event between two
 *   kernels stops them overlapping through programmatic dependent launch.
 */
#define MOE_FWD_STAGE_EVENTS 7
typedef struct {
    const void* x;
    const float* router_logits;
    int32_t T, H, I, E, B, topk;
    const int32_t* replica_src;     /* [B] or NULL */
    moe_weight_t w_gate, w_up, w_down;
    moe_act_params_t act;
    int32_t apply_topk_in_fc1;
    int32_t act_quant;
    void* out;                      /* bf16 [T,H] */
    int32_t* topk_ids_out;          /* optional */
    float* topk_w_out;              /* optional */
    int32_t T_max;                  /* capacity the workspace was sized for */
    void* const* stage_events;      /* optional: MOE_FWD_STAGE_EVENTS cudaEvent_t */
    /* routing: 0 = softmax -> top-k -> renormalise (moe_route_topk), 1 = DeepSeekV3
     * (moe_route_topk_grouped with the four fields below), 2 = given: the experts and
     * route weights of every token come in topk_ids_in / topk_w_in and router_logits may
     * be NULL (the modular and routed kernels of the FlashInfer MoE-EP and TRTLLM MXFP4
     * pages take a computed top-k). A token must not list an expert twice: the
     * permutation reports that as MOE_ERR_DEVICE. Other values: INVALID_ARG. */
    int32_t routing;
    const float* routing_bias;      /* [E] or NULL */
    int32_t n_group, topk_group;
    float routed_scaling_factor;
    const int32_t* topk_ids_in;     /* [T,topk] for routing 2 */
    const float* topk_w_in;         /* [T,topk] for routing 2 */
    /* 1: top-1 routing with the route weight on the input: the experts see x * w (rounded
     * once to bf16) and the activation and the combine take no weight (MoonEP experts
     * page, MoonEPExperts.apply). topk != 1: INVALID_ARG. */
    int32_t apply_router_weight_on_input;
    /* SWIGLUOAI parameters, used when act.act == MOE_ACT_SWIGLUOAI (moe_act_ex_t). */
    float swiglu_alpha, swiglu_beta, swiglu_limit;
    /* Per-expert GEMM biases, fp32, each NULL or present (TRTLLM MXFP4 page,
     * TrtLlmMxfp4ExpertsModular._invoke_kernel: gemm1_bias and gemm2_bias):
     * bias_gate, bias_up [E+B, I] are added to the gate and up projections before the
     * activation; bias_down [E+B, H] to the down projection, so it is scaled by the route
     * weight with the rest of the expert's output. A redundant slot reads its own rows. */
    const float* bias_gate;
    const float* bias_up;
    const float* bias_down;
} moe_forward_args_t;

/* SWIGLUOAI and the biases run inside the grouped GEMMs: the gate/up GEMM's epilogue adds
 * the gate and up biases, applies the activation and the route weight; the down GEMM's
 * epilogue adds the down bias (times the route weight when the activation carries it) to
 * the fp32 rows the combine sums. They need no workspace of their own:
 * moe_forward_workspace_size_args (which reads T_max, H, I, E, B, topk, w_gate.fmt and
 * act_quant of `args`) equals moe_forward_workspace_size. */
size_t moe_forward_workspace_size(int T_max, int H, int I, int E, int B, int topk,
                                  int wfmt, int act_quant);
size_t moe_forward_workspace_size_args(const moe_forward_args_t* args);
moe_status_t moe_forward(const moe_forward_args_t* args, void* ws, size_t ws_bytes,
                         moe_stream_t stream);

/* Synchronises `stream`, returns (and clears) the error word a kernel wrote at
 * the start of `ws` (any workspace passed to the entry points above). */
moe_status_t moe_get_device_error(void* ws, moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_MOE_H */
