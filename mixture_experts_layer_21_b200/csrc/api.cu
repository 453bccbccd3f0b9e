// The extern "C" boundary: argument validation, workspace planning and the
// launch sequences. Host code only; kernels live in the other .cu files.
#include <cmath>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "internal.h"

namespace moe {
size_t prepared_weight_bytes(const moe_weight_t* w);
// DeepSeekV3 routing (route_permute.cu); E <= 512, E % n_group == 0, n_group <= 32,
// topk_group <= n_group, topk <= min(32, topk_group * E / n_group), checked here.
cudaError_t launch_route_grouped(const float* logits, const float* bias, int T, int E, int topk, int n_group,
                                 int topk_group, float scale, int32_t* ids, float* w, cudaStream_t st, bool pdl);
// x[t,:] * w[t] rounded to bf16 (elementwise.cu); H % 8 == 0.
cudaError_t launch_scale_rows(const __nv_bfloat16* x, const float* w, int T, int H, __nv_bfloat16* out,
                              cudaStream_t st, bool pdl);
moe_status_t prepare_weights(moe_weight_t* w, void* dst, size_t dst_bytes, cudaStream_t st);
// The bias and gated-activation row pass (bias_act.cu): out = act(gate + bg[seg], up + bu[seg])
// * perm_w over [M, I] (I % 8 == 0; rows past cu[G-1] written as zero).
cudaError_t launch_bias_act(const void* gate, const void* up, bool in_f32, const float* bg, const float* bu,
                            const int32_t* cu, int G, const float* perm_w, int M, int I, int act, float sa, float sb,
                            float oa, float ob, float lim, void* out, bool out_f32, cudaStream_t st, bool pdl);

int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = n > 0 ? n : 148;
    }
    return cached[dev];
}
}  // namespace moe

using namespace moe;

namespace {

inline cudaStream_t S(moe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }
inline size_t up256(size_t b) { return (b + 255) & ~size_t(255); }

// Host-timeline ranges for profilers (NVTX): one around a whole call and one nested range
// per stage, so that e.g. `ncu --nvtx --nvtx-include "moe_forward/gate_up/"` picks out one
// stage's kernels. Without an attached tool each call is a branch.
class Trace {
  public:
    explicit Trace(const char* name) { nvtxRangePushA(name); }
    ~Trace() {
        if (stage_) nvtxRangePop();
        nvtxRangePop();
    }
    Trace(const Trace&) = delete;
    Trace& operator=(const Trace&) = delete;
    void stage(const char* name) {
        if (stage_) nvtxRangePop();
        nvtxRangePushA(name);
        stage_ = true;
    }

  private:
    bool stage_ = false;
};

bool act_ok(const moe_act_params_t& a) {
    if (a.act == MOE_ACT_SILU) return true;
    if (a.act == MOE_ACT_SITU)
        return std::isfinite(a.situ_alpha) && std::isfinite(a.situ_beta) && a.situ_alpha > 0.f && a.situ_beta > 0.f;
    return false;
}

// SWIGLUOAI: finite alpha and beta, a clamp limit > 0 (+inf: none; NaN fails).
bool swiglu_ok(float alpha, float beta, float limit) {
    return std::isfinite(alpha) && std::isfinite(beta) && limit > 0.0f;
}

bool act_ex_ok(const moe_act_ex_t& a) {
    if (a.act == MOE_ACT_SWIGLUOAI) return swiglu_ok(a.swiglu_alpha, a.swiglu_beta, a.swiglu_limit);
    return act_ok(moe_act_params_t{a.act, a.situ_alpha, a.situ_beta});
}

// Checks one projection's descriptor against the expected shape.
moe_status_t check_weight(const moe_weight_t& w, int G, int N, int K) {
    if (w.G != G || w.N != N || w.K != K || !w.data) return MOE_ERR_INVALID_ARG;
    if (w.fmt != MOE_W_BF16 && w.fmt != MOE_W_MXFP4 && w.fmt != MOE_W_NVFP4) return MOE_ERR_UNSUPPORTED;
    if (!aligned16(w.data)) return MOE_ERR_ALIGNMENT;
    if (w.fmt == MOE_W_BF16) {
        if (K % 8) return MOE_ERR_ALIGNMENT;
        return MOE_OK;
    }
    if (!w.scale) return MOE_ERR_INVALID_ARG;
    if (K % (w.fmt == MOE_W_MXFP4 ? 32 : 16)) return MOE_ERR_ALIGNMENT;
    if (!w.kdata || !w.kscale || !w.kalpha) return MOE_ERR_NOT_PREPARED;
    return MOE_OK;
}

const float* weight_alpha(const moe_weight_t& w) { return w.fmt == MOE_W_BF16 ? w.alpha : w.kalpha; }

// ----------------------------------------------------------------- forward workspace
struct FwdWs {
    size_t ids, w, cu, perm_token, perm_w, inv, perm_scratch, xperm, tscale, xq_codes, xq_sb, xq_s,
        xq_deq, xq_rec, xperm_rec, act, act2, act2_scale, act_codes, act_sb, act_rec, mx_xq, mx_xperm, mx_act,
        x_in, y, bytes;
};

// With NVFP4 activations a GEMM whose K is a multiple of 256 runs block-scaled on the
// tensor cores; its operand rows are records of K/2 code bytes followed by K/16 scales.
inline bool nvf4_k(int act_quant, int K) { return act_quant == 1 && K % kNvf4StageK == 0; }
// MXFP4 weights: activations as two e4m3 terms (bf16 staged) or one (act_quant 2, MXFP8).
inline int mx8_terms(int act_quant) { return act_quant == 2 ? 1 : 2; }
inline int nvf4_rec_bytes(int K) { return K / 2 + K / 16; }

FwdWs fwd_layout(int T_max, int H, int I, int E, int B, int topk, int wfmt, int act_quant) {
    FwdWs L{};
    const size_t NvS = (size_t)T_max * topk;
    const int G = E + B;
    size_t off = kErrBytes;
    auto take = [&](size_t b) {
        const size_t o = off;
        off += up256(b);
        return o;
    };
    const bool fp4 = wfmt != MOE_W_BF16;
    L.ids = take(4 * NvS);
    L.w = take(4 * NvS);
    L.cu = take(4 * (size_t)G);
    L.perm_token = take(4 * NvS);
    L.perm_w = take(4 * NvS);
    L.inv = take(4 * NvS);
    L.perm_scratch = take(permute_ws_layout(T_max, topk, E, B).bytes);
    const bool nat1 = nvf4_k(act_quant, H), nat2 = nvf4_k(act_quant, I);
    const bool q1 = act_quant == 1 && !nat1, q2 = act_quant == 1 && !nat2;  // NVFP4, then staged as f16
    L.xperm = take(nat1 || wfmt == MOE_W_MXFP4 ? 0 : 2 * NvS * H);
    L.tscale = take(fp4 ? 4 * NvS : 0);
    L.xq_codes = take(q1 ? (size_t)T_max * H / 2 : 0);
    L.xq_sb = take(q1 ? (size_t)T_max * H / 16 : 0);
    L.xq_s = take(q1 ? 4 * (size_t)T_max : 0);
    L.xq_deq = take(q1 ? 2 * (size_t)T_max * H : 0);
    L.xq_rec = 0;
    L.xperm_rec = take(nat1 ? NvS * nvf4_rec_bytes(H) : 0);
    const bool mx = wfmt == MOE_W_MXFP4;
    // h: bf16 (BF16 weights), fp32 when a row pass follows (NVFP4 weights); the MXFP4 gate/up
    // epilogue writes the down GEMM's records directly
    L.act = take(mx ? 0 : (fp4 ? 4 : 2) * NvS * I);
    L.act2 = take(fp4 && !nat2 && wfmt != MOE_W_MXFP4 ? 2 * NvS * I : 0);
    L.act2_scale = take(fp4 ? 4 * NvS : 0);
    L.act_codes = take(q2 ? NvS * I / 2 : 0);
    L.act_sb = take(q2 ? NvS * I / 16 : 0);
    L.act_rec = take(nat2 ? NvS * nvf4_rec_bytes(I) : 0);
    const int terms = mx8_terms(act_quant);
    L.mx_xq = 0;
    L.mx_xperm = take(mx ? NvS * mx8_rec_bytes(H, terms) : 0);
    L.mx_act = take(mx ? NvS * mx8_rec_bytes(I, terms) : 0);
    L.x_in = take(topk == 1 ? 2 * (size_t)T_max * H : 0);  // x times the top-1 weight (input-side weighting)
    L.y = take(4 * NvS * H);  // fp32: the output is rounded to bf16 once, in the combine
    L.bytes = off;
    return L;
}

const char* kStatusNames[] = {"MOE_OK",
                              "MOE_ERR_INVALID_ARG",
                              "MOE_ERR_UNSUPPORTED",
                              "MOE_ERR_ALIGNMENT",
                              "MOE_ERR_WORKSPACE_TOO_SMALL",
                              "MOE_ERR_CUDA",
                              "MOE_ERR_DEVICE",
                              "MOE_ERR_TIMEOUT",
                              "MOE_ERR_NOT_PREPARED"};

}  // namespace

extern "C" {

const char* moe_status_string(moe_status_t s) {
    const int i = static_cast<int>(s);
    if (i < 0 || i >= (int)(sizeof(kStatusNames) / sizeof(kStatusNames[0]))) return "MOE_ERR_UNKNOWN";
    return kStatusNames[i];
}

const char* moe_version(void) { return "moe_b200 0.1 sm_100a"; }

moe_status_t moe_route_topk(const float* logits, int T, int E, int topk, int32_t* topk_ids, float* topk_w,
                            moe_stream_t stream) {
    if (T < 0 || E < 1 || topk < 1 || topk > E) return MOE_ERR_INVALID_ARG;
    if (E > kMaxExperts || topk > kMaxTopk) return MOE_ERR_UNSUPPORTED;
    if (T == 0) return MOE_OK;
    if (!logits || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_route_topk(logits, T, E, topk, topk_ids, topk_w, S(stream), false));
}

}  // extern "C"

namespace {
// Arguments of the DeepSeekV3 routing; MOE_OK when the kernel supports them.
moe_status_t check_grouped(int E, int topk, int n_group, int topk_group, float scale) {
    if (n_group < 1 || E % n_group || topk_group < 1 || topk_group > n_group) return MOE_ERR_INVALID_ARG;
    if (topk < 1 || topk > topk_group * (E / n_group)) return MOE_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.0f)) return MOE_ERR_INVALID_ARG;
    if (E > 512 || n_group > 32 || topk > kMaxTopk) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}
}  // namespace

extern "C" {

moe_status_t moe_route_topk_grouped(const float* logits, const float* bias, int T, int E, int topk, int n_group,
                                    int topk_group, float routed_scaling_factor, int32_t* topk_ids, float* topk_w,
                                    moe_stream_t stream) {
    if (T < 0 || E < 1) return MOE_ERR_INVALID_ARG;
    moe_status_t s = check_grouped(E, topk, n_group, topk_group, routed_scaling_factor);
    if (s != MOE_OK) return s;
    if (T == 0) return MOE_OK;
    if (!logits || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
    return cuda_status(launch_route_grouped(logits, bias, T, E, topk, n_group, topk_group, routed_scaling_factor,
                                            topk_ids, topk_w, S(stream), false));
}

size_t moe_permute_workspace_size(int T, int topk, int E, int B) {
    if (T < 0 || topk < 1 || E < 1 || B < 0) return 0;
    return kErrBytes + permute_ws_layout(T, topk, E, B).bytes;
}

moe_status_t moe_permute(const int32_t* topk_ids, const float* topk_w, int T, int topk, int E, int B,
                         const int32_t* replica_src, const void* x, int H, int32_t* cu_seqlens, int32_t* perm_token,
                         float* perm_w, int32_t* inv_perm, void* x_perm, int M_alloc, void* ws, size_t ws_bytes,
                         moe_stream_t stream) {
    if (T < 0 || topk < 1 || E < 1 || B < 0 || topk > E) return MOE_ERR_INVALID_ARG;
    if (E > kMaxExperts || E + B > kMaxRows || topk > kMaxTopk) return MOE_ERR_UNSUPPORTED;
    if (B > 0 && !replica_src) return MOE_ERR_INVALID_ARG;
    if (!cu_seqlens || !ws) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < moe_permute_workspace_size(T, topk, E, B)) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (x_perm) {
        if (!x || H <= 0 || M_alloc < T * topk) return MOE_ERR_INVALID_ARG;
        if (H % 8 || !aligned16(x) || !aligned16(x_perm)) return MOE_ERR_ALIGNMENT;
    }
    if (T > 0 && (!topk_ids || !perm_token || !perm_w || !inv_perm)) return MOE_ERR_INVALID_ARG;
    char* w = static_cast<char*>(ws);
    cudaStream_t st = S(stream);
    cudaError_t e = launch_permute(topk_ids, topk_w, T, topk, E, B, replica_src, cu_seqlens, perm_token, perm_w,
                                   inv_perm, reinterpret_cast<DevError*>(w), w + kErrBytes, st, false);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    if (x_perm) e = launch_gather(0, x, H, perm_token, T * topk, x_perm, nullptr, nullptr, st, true);
    return cuda_status(e);
}

size_t moe_grouped_gemm_workspace_size(int M_alloc, const moe_weight_t* w) {
    if (!w || M_alloc < 0) return 0;
    size_t b = kErrBytes;
    if (w->fmt == MOE_W_MXFP4) b += up256((size_t)M_alloc * mx8_rec_bytes(w->K));
    else if (w->fmt != MOE_W_BF16) b += up256(2 * (size_t)M_alloc * w->K) + up256(4 * (size_t)M_alloc);
    return b;
}

moe_status_t moe_grouped_gemm(const void* a, int M_alloc, const moe_weight_t* w, const int32_t* cu_seqlens,
                              void* out, void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (!w || M_alloc < 0 || w->G < 1 || w->N < 1 || w->K < 1) return MOE_ERR_INVALID_ARG;
    if (w->G > 1024) return MOE_ERR_UNSUPPORTED;
    moe_status_t s = check_weight(*w, w->G, w->N, w->K);
    if (s != MOE_OK) return s;
    if (M_alloc == 0) return MOE_OK;
    if (!a || !cu_seqlens || !out || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(out) || w->N % 8) return MOE_ERR_ALIGNMENT;
    if (ws_bytes < moe_grouped_gemm_workspace_size(M_alloc, w)) return MOE_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = S(stream);
    char* wsb = static_cast<char*>(ws);
    GemmProblem p{};
    p.M_alloc = M_alloc;
    p.cu_seqlens = cu_seqlens;
    p.G = w->G;
    p.N = w->N;
    p.K = w->K;
    p.wfmt = w->fmt;
    p.dual = false;
    p.alpha0 = weight_alpha(*w);
    p.out_scale = 1.0f;
    p.out = out;
    p.out_kind = OUT_BF16;
    p.zero_pad = true;
    p.err = reinterpret_cast<DevError*>(wsb);
    bool pdl = false;
    if (w->fmt == MOE_W_BF16) {
        p.x = a;
        p.w0 = w->data;
    } else if (w->fmt == MOE_W_MXFP4) {
        // activations -> e4m3 hi/lo records, then the block-scaled GEMM
        uint8_t* rec = reinterpret_cast<uint8_t*>(wsb + kErrBytes);
        const int rb = mx8_rec_bytes(w->K), Kp = mx8_kpad(w->K);
        cudaError_t e = launch_quant_mx8(a, false, M_alloc, w->K, Kp, true, rec, rec + Kp, rec + 2 * Kp, rb, rb, st,
                                         false);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        p.x = rec;
        p.x_stride = rb;
        p.mx8 = 2;
        p.kdata0 = w->kdata;
        p.kscale0 = w->kscale;
        pdl = true;
    } else {
        __half* a16 = reinterpret_cast<__half*>(wsb + kErrBytes);
        float* sc = reinterpret_cast<float*>(wsb + kErrBytes + up256(2 * (size_t)M_alloc * w->K));
        cudaError_t e = launch_rows_to_f16(a, false, M_alloc, w->K, a16, sc, st, false);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        p.x = a16;
        p.tscale = sc;
        p.kdata0 = w->kdata;
        p.kscale0 = w->kscale;
        pdl = true;
    }
    return cuda_status(launch_grouped_gemm(p, st, pdl));
}

moe_status_t moe_quantize_mxfp8(const void* in, int in_is_f32, int R, int K, uint8_t* codes, uint8_t* scales,
                                moe_stream_t stream) {
    if (R < 0 || K < 0) return MOE_ERR_INVALID_ARG;
    if (K % 32) return MOE_ERR_ALIGNMENT;
    if ((size_t)R * K == 0) return MOE_OK;
    if (!in || !codes || !scales) return MOE_ERR_INVALID_ARG;
    if (!aligned16(in) || !aligned16(codes)) return MOE_ERR_ALIGNMENT;
    return cuda_status(launch_quant_mx8(in, in_is_f32 != 0, R, K, K, false, codes, nullptr, scales, K, K / 32,
                                        S(stream), false));
}

moe_status_t moe_grouped_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_sb, const float* a_s, int M_alloc,
                                    const moe_weight_t* w, const int32_t* cu_seqlens, void* out, void* ws,
                                    size_t ws_bytes, moe_stream_t stream) {
    if (!w || M_alloc < 0 || w->G < 1 || w->N < 1 || w->K < 1) return MOE_ERR_INVALID_ARG;
    if (w->G > 1024) return MOE_ERR_UNSUPPORTED;
    if (w->fmt != MOE_W_NVFP4) return MOE_ERR_UNSUPPORTED;
    moe_status_t s = check_weight(*w, w->G, w->N, w->K);
    if (s != MOE_OK) return s;
    if (w->K % kNvf4StageK) return MOE_ERR_ALIGNMENT;
    if (M_alloc == 0) return MOE_OK;
    if (!a_codes || !a_sb || !a_s || !cu_seqlens || !out || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned16(a_codes) || !aligned16(a_sb) || !aligned16(out) || w->N % 8) return MOE_ERR_ALIGNMENT;
    if (ws_bytes < kErrBytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
    GemmProblem p{};
    p.x = a_codes;
    p.x_stride = w->K / 2;
    p.xsf = a_sb;
    p.xsf_stride = w->K / 16;
    p.nvf4 = true;
    p.tscale = a_s;
    p.M_alloc = M_alloc;
    p.cu_seqlens = cu_seqlens;
    p.G = w->G;
    p.N = w->N;
    p.K = w->K;
    p.wfmt = w->fmt;
    p.dual = false;
    p.kdata0 = w->kdata;
    p.kscale0 = w->kscale;
    p.alpha0 = weight_alpha(*w);
    p.out_scale = 1.0f;
    p.out = out;
    p.out_kind = OUT_BF16;
    p.zero_pad = true;
    p.err = reinterpret_cast<DevError*>(ws);
    return cuda_status(launch_grouped_gemm(p, S(stream), false));
}

moe_status_t moe_act_and_mul(const void* gate, const void* up, const float* perm_w, int M, int I,
                             moe_act_params_t act, void* out, moe_stream_t stream) {
    if (act.act == MOE_ACT_SWIGLUOAI) return MOE_ERR_UNSUPPORTED;  // its parameters: moe_bias_act_and_mul
    if (M < 0 || I < 0 || !act_ok(act)) return MOE_ERR_INVALID_ARG;
    if ((size_t)M * I == 0) return MOE_OK;
    if (!gate || !up || !out) return MOE_ERR_INVALID_ARG;
    if (I % 8 || !aligned16(gate) || !aligned16(up) || !aligned16(out)) return MOE_ERR_ALIGNMENT;
    return cuda_status(launch_act_and_mul(static_cast<const __nv_bfloat16*>(gate),
                                          static_cast<const __nv_bfloat16*>(up), perm_w, M, I, act.act,
                                          act.situ_alpha, act.situ_beta, static_cast<__nv_bfloat16*>(out),
                                          S(stream), false));
}

moe_status_t moe_bias_act_and_mul(const void* gate, const void* up, int in_is_f32, const float* bias_gate,
                                  const float* bias_up, const int32_t* cu_seqlens, int G, const float* perm_w, int M,
                                  int I, const moe_act_ex_t* act, void* out, moe_stream_t stream) {
    if (!act || M < 0 || I < 0 || G < 1) return MOE_ERR_INVALID_ARG;
    if (!act_ex_ok(*act)) return MOE_ERR_INVALID_ARG;
    if ((size_t)M * I == 0) return MOE_OK;
    if (!gate || !up || !out || !cu_seqlens) return MOE_ERR_INVALID_ARG;
    if (I % 8 || !aligned16(gate) || !aligned16(up) || !aligned16(out)) return MOE_ERR_ALIGNMENT;
    if ((bias_gate && !aligned16(bias_gate)) || (bias_up && !aligned16(bias_up))) return MOE_ERR_ALIGNMENT;
    return cuda_status(launch_bias_act(gate, up, in_is_f32 != 0, bias_gate, bias_up, cu_seqlens, G, perm_w, M, I,
                                       act->act, act->situ_alpha, act->situ_beta, act->swiglu_alpha,
                                       act->swiglu_beta, act->swiglu_limit, out, false, S(stream), false));
}

moe_status_t moe_combine(const void* y_perm, const int32_t* inv_perm, const float* topk_w, int T, int topk, int H,
                         void* out, moe_stream_t stream) {
    if (T < 0 || topk < 1 || H < 1) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!y_perm || !inv_perm || !out) return MOE_ERR_INVALID_ARG;
    if (H % 8 || !aligned16(y_perm) || !aligned16(out)) return MOE_ERR_ALIGNMENT;
    return cuda_status(launch_combine(static_cast<const __nv_bfloat16*>(y_perm), inv_perm, topk_w, T, topk, H,
                                      static_cast<__nv_bfloat16*>(out), S(stream), false));
}

moe_status_t moe_quantize_nvfp4(const void* in, int in_is_f32, int R, int K, uint8_t* codes, uint8_t* sb, float* s,
                                void* deq_f16, moe_stream_t stream) {
    if (R < 0 || K < 0) return MOE_ERR_INVALID_ARG;
    if (K % 16) return MOE_ERR_ALIGNMENT;
    if ((size_t)R * K == 0) return MOE_OK;
    if (!in || !codes || !sb || !s) return MOE_ERR_INVALID_ARG;
    if (!aligned16(in) || !aligned16(codes) || (deq_f16 && !aligned16(deq_f16))) return MOE_ERR_ALIGNMENT;
    return cuda_status(launch_quant_nvfp4(in, in_is_f32 != 0, R, K, codes, K / 2, sb, K / 16, s,
                                          static_cast<__half*>(deq_f16), S(stream), false));
}

size_t moe_prepared_weight_bytes(const moe_weight_t* w) {
    if (!w) return 0;
    return prepared_weight_bytes(w);
}

moe_status_t moe_prepare_weights(moe_weight_t* w, void* dst, size_t dst_bytes, moe_stream_t stream) {
    if (!w || w->G < 1 || w->N < 1 || w->K < 1 || !w->data) return MOE_ERR_INVALID_ARG;
    if (w->fmt == MOE_W_BF16) return MOE_OK;
    if (w->fmt != MOE_W_MXFP4 && w->fmt != MOE_W_NVFP4) return MOE_ERR_UNSUPPORTED;
    if (!w->scale || !dst) return MOE_ERR_INVALID_ARG;
    if (w->K % (w->fmt == MOE_W_MXFP4 ? 32 : 16)) return MOE_ERR_ALIGNMENT;
    if (w->alpha) {
        // epilogue alphas must be finite and positive (FlashInfer MoE-EP page,
        // epilogue_from_quant_config -> require_finite_positive_scales)
        std::vector<float> h(w->G);
        if (cudaMemcpy(h.data(), w->alpha, sizeof(float) * w->G, cudaMemcpyDeviceToHost) != cudaSuccess)
            return MOE_ERR_CUDA;
        for (float v : h)
            if (!std::isfinite(v) || !(v > 0.0f)) return MOE_ERR_INVALID_ARG;
    }
    return prepare_weights(w, dst, dst_bytes, S(stream));
}

size_t moe_forward_workspace_size(int T_max, int H, int I, int E, int B, int topk, int wfmt, int act_quant) {
    if (T_max < 0 || H < 1 || I < 1 || E < 1 || B < 0 || topk < 1) return 0;
    return fwd_layout(T_max, H, I, E, B, topk, wfmt, act_quant).bytes;
}

}  // extern "C"

extern "C" {

// The workspace of a given argument set. SWIGLUOAI and the GEMM biases run in the GEMMs'
// epilogues and need nothing extra, so this equals moe_forward_workspace_size.
size_t moe_forward_workspace_size_args(const moe_forward_args_t* a) {
    if (!a || a->T_max < 0 || a->H < 1 || a->I < 1 || a->E < 1 || a->B < 0 || a->topk < 1) return 0;
    return fwd_layout(a->T_max, a->H, a->I, a->E, a->B, a->topk, a->w_gate.fmt, a->act_quant).bytes;
}

moe_status_t moe_forward(const moe_forward_args_t* p, void* ws, size_t ws_bytes, moe_stream_t stream) {
    if (!p) return MOE_ERR_INVALID_ARG;
    const int T = p->T, H = p->H, I = p->I, E = p->E, B = p->B, k = p->topk;
    if (T < 0 || H < 1 || I < 1 || E < 1 || B < 0 || k < 1 || k > E) return MOE_ERR_INVALID_ARG;
    if (T > p->T_max) return MOE_ERR_INVALID_ARG;  // the workspace was sized for T_max tokens
    if (E > kMaxExperts || E + B > 1024 || k > kMaxTopk) return MOE_ERR_UNSUPPORTED;
    if (p->act.act == MOE_ACT_SWIGLUOAI) {
        if (!swiglu_ok(p->swiglu_alpha, p->swiglu_beta, p->swiglu_limit)) return MOE_ERR_INVALID_ARG;
    } else if (!act_ok(p->act)) {
        return MOE_ERR_INVALID_ARG;
    }
    // routing: 0 = softmax -> top-k -> renormalise, 1 = DeepSeekV3 grouped top-k, 2 = given
    if (p->routing < 0 || p->routing > 2) return MOE_ERR_INVALID_ARG;
    if (p->routing == 2 && (!p->topk_ids_in || !p->topk_w_in)) return MOE_ERR_INVALID_ARG;
    if (p->apply_router_weight_on_input && k != 1) return MOE_ERR_INVALID_ARG;
    if (p->routing == 1) {
        const moe_status_t rs = check_grouped(E, k, p->n_group, p->topk_group, p->routed_scaling_factor);
        if (rs != MOE_OK) return rs;
    }
    const int G = E + B;
    const int fmt = p->w_gate.fmt;
    if (p->w_up.fmt != fmt || p->w_down.fmt != fmt) return MOE_ERR_UNSUPPORTED;
    moe_status_t s;
    if ((s = check_weight(p->w_gate, G, I, H)) != MOE_OK) return s;
    if ((s = check_weight(p->w_up, G, I, H)) != MOE_OK) return s;
    if ((s = check_weight(p->w_down, G, H, I)) != MOE_OK) return s;
    // act_quant: 1 = dynamic NVFP4 (NVFP4 weights), 2 = dynamic MXFP8 (MXFP4 weights)
    if (p->act_quant < 0 || p->act_quant > 2) return MOE_ERR_INVALID_ARG;
    if ((p->act_quant == 1 && fmt != MOE_W_NVFP4) || (p->act_quant == 2 && fmt != MOE_W_MXFP4))
        return MOE_ERR_UNSUPPORTED;
    if (H % 16 || I % 16) return MOE_ERR_ALIGNMENT;
    if (B > 0 && !p->replica_src) return MOE_ERR_INVALID_ARG;
    if (!ws) return MOE_ERR_INVALID_ARG;
    const FwdWs L = fwd_layout(p->T_max, H, I, E, B, k, fmt, p->act_quant);
    if (ws_bytes < L.bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (T == 0) return MOE_OK;
    if (!p->x || (!p->router_logits && p->routing != 2) || !p->out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(p->x) || !aligned16(p->out) || !aligned16(ws)) return MOE_ERR_ALIGNMENT;
    for (const float* b : {p->bias_gate, p->bias_up, p->bias_down})
        if (b && !aligned16(b)) return MOE_ERR_ALIGNMENT;

    char* w = static_cast<char*>(ws);
    DevError* err = reinterpret_cast<DevError*>(w);
    const bool given = p->routing == 2;
    const int32_t* ids = given ? p->topk_ids_in
                               : (p->topk_ids_out ? p->topk_ids_out : reinterpret_cast<int32_t*>(w + L.ids));
    const float* tw = given ? p->topk_w_in : (p->topk_w_out ? p->topk_w_out : reinterpret_cast<float*>(w + L.w));
    int32_t* cu = reinterpret_cast<int32_t*>(w + L.cu);
    int32_t* perm_token = reinterpret_cast<int32_t*>(w + L.perm_token);
    float* perm_w = reinterpret_cast<float*>(w + L.perm_w);
    int32_t* inv = reinterpret_cast<int32_t*>(w + L.inv);
    void* xperm = w + L.xperm;
    float* tscale = reinterpret_cast<float*>(w + L.tscale);
    void* act = w + L.act;
    __half* act2 = reinterpret_cast<__half*>(w + L.act2);
    float* act2_scale = reinterpret_cast<float*>(w + L.act2_scale);
    float* y = reinterpret_cast<float*>(w + L.y);
    const int NvS = T * k;
    const bool nat1 = nvf4_k(p->act_quant, H), nat2 = nvf4_k(p->act_quant, I);
    const int terms = mx8_terms(p->act_quant);
    cudaStream_t st = S(stream);
    cudaError_t e;
    // Optional stage events (tracing). An event recorded between two kernels ends their
    // programmatic-dependent-launch overlap, so only that boundary launches without it.
    bool ev = false;
    auto mark = [&](int i) -> bool {
        if (!p->stage_events || !p->stage_events[i]) return true;
        ev = true;
        return cudaEventRecord(static_cast<cudaEvent_t>(p->stage_events[i]), st) == cudaSuccess;
    };
    auto pdl = [&]() {
        const bool r = !ev;
        ev = false;
        return r;
    };

    Trace trace("moe_forward");
    trace.stage("route");
    if (!mark(0)) return MOE_ERR_CUDA;
    // S1 route (or the given top-k, copied to the optional outputs)
    int32_t* ids_w = const_cast<int32_t*>(ids);
    float* tw_w = const_cast<float*>(tw);
    if (given) {
        e = cudaSuccess;
        if (p->topk_ids_out)
            e = cudaMemcpyAsync(p->topk_ids_out, ids, sizeof(int32_t) * (size_t)T * k, cudaMemcpyDeviceToDevice, st);
        if (e == cudaSuccess && p->topk_w_out)
            e = cudaMemcpyAsync(p->topk_w_out, tw, sizeof(float) * (size_t)T * k, cudaMemcpyDeviceToDevice, st);
    } else if (p->routing == 1) {
        e = launch_route_grouped(p->router_logits, p->routing_bias, T, E, k, p->n_group, p->topk_group,
                                 p->routed_scaling_factor, ids_w, tw_w, st, false);
    } else if (T <= 256) {
        // decode batches: the routing and the permutation in one launch
        e = launch_route_permute_one_block(p->router_logits, T, E, k, ids_w, tw_w, B, p->replica_src, cu, perm_token,
                                           perm_w, inv, err, w + L.perm_scratch, st, false);
    } else {
        e = launch_route_topk(p->router_logits, T, E, k, ids_w, tw_w, st, false);
    }
    const bool permuted = !given && p->routing == 0 && T <= 256;
    if (e != cudaSuccess || !mark(1)) return MOE_ERR_CUDA;
    // top-1 weight on the input: the experts see x * w and the activation takes no weight
    const bool in_w = p->apply_router_weight_on_input != 0;
    const void* xin = p->x;
    if (in_w) {
        e = launch_scale_rows(static_cast<const __nv_bfloat16*>(p->x), tw, T, H,
                              reinterpret_cast<__nv_bfloat16*>(w + L.x_in), st, pdl());
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        xin = w + L.x_in;
    }
    // S2 permute
    trace.stage("permute");
    if (!permuted) {
        e = launch_permute(ids, tw, T, k, E, B, p->replica_src, cu, perm_token, perm_w, inv, err, w + L.perm_scratch,
                           st, pdl());
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
    // S2 gather (+ S2q). The BF16 gate/up GEMM with 128-token tiles (or on CTA pairs) can read
    // the token rows of x by perm_token itself (MOE_FUSED_GATHER=1), which saves writing and
    // re-reading x_perm.
    GemmProblem probe{};
    probe.wfmt = fmt;
    probe.dual = true;
    probe.M_alloc = NvS;
    probe.G = G;
    const char* fg = getenv("MOE_FUSED_GATHER");
    const bool fused_gather = fmt == MOE_W_BF16 && fg && fg[0] == '1' && fg[1] == '\0' && gemm_can_gather(probe);
    if (fmt == MOE_W_BF16) {
        e = fused_gather ? cudaSuccess : launch_gather(0, xin, H, perm_token, NvS, xperm, nullptr, nullptr, st, pdl());
    } else if (fmt == MOE_W_MXFP4) {
        // stage the gathered rows as e4m3 records (hi/lo, or MXFP8) in segment order, one pass
        const int rb = mx8_rec_bytes(H, terms), Kp = mx8_kpad(H);
        uint8_t* rec = reinterpret_cast<uint8_t*>(w + L.mx_xperm);
        e = launch_quant_mx8(xin, false, NvS, H, Kp, terms == 2, rec, terms == 2 ? rec + Kp : nullptr,
                             rec + terms * Kp, rb, rb, st, pdl(), perm_token, T);
    } else if (nat1) {
        // quantise the gathered rows into records in segment order, one pass (a row's codes
        // depend on that row alone, so a token quantised twice gives the same bits)
        uint8_t* rec = reinterpret_cast<uint8_t*>(w + L.xperm_rec);
        const int rb = nvf4_rec_bytes(H);
        e = launch_quant_nvfp4(xin, false, NvS, H, rec, rb, rec + H / 2, rb, tscale, nullptr, st, pdl(), perm_token,
                               T);
    } else if (p->act_quant) {
        e = launch_quant_nvfp4(xin, false, T, H, reinterpret_cast<uint8_t*>(w + L.xq_codes), H / 2,
                               reinterpret_cast<uint8_t*>(w + L.xq_sb), H / 16, reinterpret_cast<float*>(w + L.xq_s),
                               reinterpret_cast<__half*>(w + L.xq_deq), st, pdl());
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        e = launch_gather(1, w + L.xq_deq, H, perm_token, NvS, xperm, reinterpret_cast<float*>(w + L.xq_s), tscale,
                          st, pdl());
    } else {
        e = launch_gather(2, xin, H, perm_token, NvS, xperm, nullptr, tscale, st, pdl());
    }
    if (e != cudaSuccess || !mark(2)) return MOE_ERR_CUDA;

    // S3 + S4: gate/up grouped GEMM with the activation epilogue
    trace.stage("gate_up");
    const bool situ = p->act.act == MOE_ACT_SITU;
    GemmProblem g1{};
    g1.x = fused_gather ? xin : xperm;
    g1.gather_idx = fused_gather ? perm_token : nullptr;
    g1.gather_rows = T;
    g1.M_alloc = NvS;
    g1.cu_seqlens = cu;
    g1.G = G;
    g1.N = I;
    g1.K = H;
    g1.wfmt = fmt;
    g1.dual = true;
    g1.w0 = p->w_gate.data;
    g1.w1 = p->w_up.data;
    g1.kdata0 = p->w_gate.kdata;
    g1.kscale0 = p->w_gate.kscale;
    g1.kdata1 = p->w_up.kdata;
    g1.kscale1 = p->w_up.kscale;
    g1.alpha0 = weight_alpha(p->w_gate);
    g1.alpha1 = weight_alpha(p->w_up);
    g1.perm_w = (p->apply_topk_in_fc1 && !in_w) ? perm_w : nullptr;
    g1.tscale = fmt == MOE_W_BF16 ? nullptr : tscale;
    g1.out_scale = 1.0f;
    g1.act = p->act.act;
    g1.situ_a = p->act.situ_alpha;
    g1.situ_b = p->act.situ_beta;
    g1.sw_alpha = p->swiglu_alpha;
    g1.sw_beta = p->swiglu_beta;
    g1.sw_limit = p->swiglu_limit;
    g1.bias0 = p->bias_gate;
    g1.bias1 = p->bias_up;
    g1.out = act;
    g1.err = err;
    if (fmt == MOE_W_MXFP4) {
        g1.mx8 = terms;
        g1.x = w + L.mx_xperm;
        g1.x_stride = mx8_rec_bytes(H, terms);
        g1.tscale = nullptr;
    }
    if (nat1) {
        const int rb = nvf4_rec_bytes(H);
        g1.nvf4 = true;
        g1.x = w + L.xperm_rec;
        g1.x_stride = rb;
        g1.xsf = w + L.xperm_rec + H / 2;
        g1.xsf_stride = rb;
    }
    // The down projection's operand: bf16 for BF16 weights; for FP4 weights f16 with a
    // per-row power-of-two scale (or a fixed one when SITU bounds |h| by alpha*beta),
    // or NVFP4-quantised rows when act_quant.
    float fc2_out_scale = 1.0f;
    const void* fc2_x = act;
    const float* fc2_tscale = nullptr;
    bool row_pass = false;
    if (fmt == MOE_W_BF16) {
        g1.out_kind = OUT_BF16;
    } else if (fmt == MOE_W_MXFP4) {
        // the epilogue writes h straight as the down GEMM's e4m3 records and e8m0 scales
        g1.out_kind = OUT_MX8;
        g1.out = w + L.mx_act;
        g1.out_terms = terms;
        g1.out_stride = mx8_rec_bytes(I, terms);
        fc2_x = w + L.mx_act;
    } else if (situ && !p->act_quant) {
        // |h| <= alpha*beta*|route weight| <= alpha*beta: one fixed power of two keeps it below 2^15
        const double bound = (double)p->act.situ_alpha * p->act.situ_beta;
        int ex = 0;
        std::frexp(bound, &ex);
        const int sh = std::max(0, ex - 15);
        g1.out_scale = std::ldexp(1.0f, -sh);
        fc2_out_scale = std::ldexp(1.0f, sh);
        g1.out_kind = OUT_F16;
    } else {
        g1.out_kind = OUT_F32;
        row_pass = true;
    }
    // S3 + S4 in one launch: gate and up, their biases, the activation (SWIGLUOAI included)
    // and the route weight in the epilogue
    e = launch_grouped_gemm(g1, st, pdl());
    if (e != cudaSuccess || !mark(3)) return MOE_ERR_CUDA;
    const int rb2 = nvf4_rec_bytes(I);
    trace.stage("act_row_pass");
    if (row_pass) {
        if (nat2) {
            uint8_t* rec = reinterpret_cast<uint8_t*>(w + L.act_rec);
            e = launch_quant_nvfp4(act, true, NvS, I, rec, rb2, rec + I / 2, rb2, act2_scale, nullptr, st, pdl());
        } else if (p->act_quant) {
            e = launch_quant_nvfp4(act, true, NvS, I, reinterpret_cast<uint8_t*>(w + L.act_codes), I / 2,
                                   reinterpret_cast<uint8_t*>(w + L.act_sb), I / 16, act2_scale, act2, st, pdl());
        } else {
            e = launch_rows_to_f16(act, true, NvS, I, act2, act2_scale, st, pdl());
        }
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        fc2_x = nat2 ? static_cast<const void*>(w + L.act_rec) : act2;
        fc2_tscale = act2_scale;
    }
    if (!mark(4)) return MOE_ERR_CUDA;
    // S5: down grouped GEMM
    trace.stage("down");
    GemmProblem g2{};
    g2.x = fc2_x;
    g2.M_alloc = NvS;
    g2.cu_seqlens = cu;
    g2.G = G;
    g2.N = H;
    g2.K = I;
    g2.wfmt = fmt;
    g2.dual = false;
    g2.w0 = p->w_down.data;
    g2.kdata0 = p->w_down.kdata;
    g2.kscale0 = p->w_down.kscale;
    g2.alpha0 = weight_alpha(p->w_down);
    g2.tscale = fc2_tscale;
    g2.out_scale = fc2_out_scale;
    g2.out = y;
    g2.out_kind = OUT_F32;
    g2.err = err;
    // the expert's down bias is part of its output: under the route weight when the
    // activation carries the weight, else the combine weights it with the rest
    g2.bias0 = p->bias_down;
    g2.bias_rw = g1.perm_w;
    if (fmt == MOE_W_MXFP4) {
        g2.mx8 = terms;
        g2.x_stride = mx8_rec_bytes(I, terms);
    }
    if (nat2) {
        g2.nvf4 = true;
        g2.x_stride = rb2;
        g2.xsf = w + L.act_rec + I / 2;
        g2.xsf_stride = rb2;
    }
    e = launch_grouped_gemm(g2, st, pdl());
    if (e != cudaSuccess || !mark(5)) return MOE_ERR_CUDA;
    // S6: combine
    trace.stage("combine");
    e = launch_combine_f32(y, inv, (p->apply_topk_in_fc1 || in_w) ? nullptr : tw, T, k, H,
                           static_cast<__nv_bfloat16*>(p->out), st, pdl());
    if (e != cudaSuccess || !mark(6)) return MOE_ERR_CUDA;
    return MOE_OK;
}

moe_status_t moe_get_device_error(void* ws, moe_stream_t stream) {
    if (!ws) return MOE_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return MOE_ERR_CUDA;
    DevError h{0, 0};
    if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    if (h.code != 0) {
        if (cudaMemset(ws, 0, sizeof(h)) != cudaSuccess) return MOE_ERR_CUDA;
        return static_cast<moe_status_t>(h.code);
    }
    return MOE_OK;
}

}  // extern "C"
