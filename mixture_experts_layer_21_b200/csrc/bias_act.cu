// The standalone bias/activation row pass (moe_bias_act_and_mul): per-expert gate/up
// biases and every gated activation, SWIGLUOAI included (TRTLLM MXFP4 experts page:
// SWIGLUOAI among the supported activations, gemm1_alpha, gemm1_beta and
// gemm1_clamp_limit broadcast to every local expert in __init__, gemm1_bias handed to the
// kernel in _invoke_kernel). The fused layer does the same in the gate/up GEMM's epilogue.
//
// bias_act_kernel adds each row's expert bias, applies the gated activation and the route
// weight. The expert of a segment row is found from cu_seqlens (inclusive segment ends) by
// binary search, so redundant slots use their own bias rows.
#include "internal.h"

namespace moe {

// Parameters of every gated activation the row pass applies.
struct ActArgs {
    int act;          // moe_act_t
    float sa, sb;     // SITU caps
    float oa, ob;     // SWIGLUOAI: sigmoid slope alpha and up offset beta
    float lim;        // SWIGLUOAI clamp (+inf: none)
};

// Segment holding row r: the first g with cu[g] > r; G when r >= cu[G-1].
__device__ __forceinline__ int segment_of(const int32_t* __restrict__ cu, int G, int r) {
    int lo = 0, hi = G;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(cu + mid) > r) hi = mid;
        else lo = mid + 1;
    }
    return lo;
}

// SWIGLUOAI as published with GPT-OSS: g = min(gate, lim), u = clamp(up, -lim, lim),
// out = g * sigmoid(alpha * g) * (u + beta).
__device__ __forceinline__ float act_ex(const ActArgs& a, float g, float u) {
    if (a.act == MOE_ACT_SWIGLUOAI) {
        const float gc = fminf(g, a.lim);
        const float uc = fminf(fmaxf(u, -a.lim), a.lim);
        return gc / (1.0f + expf(-a.oa * gc)) * (uc + a.ob);
    }
    return act_apply(a.act, g, u, a.sa, a.sb);
}

template <bool F32>
__device__ __forceinline__ void ld8(const void* p, size_t i, float (&f)[8]) {
    if constexpr (F32) {
        const float4* q = reinterpret_cast<const float4*>(static_cast<const float*>(p) + i);
        const float4 a = q[0], b = q[1];
        f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
        f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    } else {
        const uint4 v = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p) + i);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 t = __bfloat1622float2(h[q]);
            f[2 * q] = t.x;
            f[2 * q + 1] = t.y;
        }
    }
}

template <bool F32>
__device__ __forceinline__ void st8(void* p, size_t i, const float (&f)[8]) {
    if constexpr (F32) {
        float4* q = reinterpret_cast<float4*>(static_cast<float*>(p) + i);
        q[0] = make_float4(f[0], f[1], f[2], f[3]);
        q[1] = make_float4(f[4], f[5], f[6], f[7]);
    } else {
        uint4 v;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
        for (int q = 0; q < 4; ++q) h[q] = __floats2bfloat162_rn(f[2 * q], f[2 * q + 1]);
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p) + i) = v;
    }
}

// out[r,i] = act(gate[r,i] + bg[g,i], up[r,i] + bu[g,i]) * perm_w[r] for the rows of
// segment g < G (bg, bu, perm_w may each be NULL: no term); rows at or past cu[G-1] are
// written as zero. gate/up/out [M, I] row-major, I % 8 == 0; bg/bu fp32 [G, I]. fp32
// arithmetic, one rounding when the output is bf16. Each thread owns 8 consecutive values.
template <bool IN_F32, bool OUT_F32>
__global__ void __launch_bounds__(256) bias_act_kernel(const void* __restrict__ gate, const void* __restrict__ up,
                                                       const float* __restrict__ bg, const float* __restrict__ bu,
                                                       const int32_t* __restrict__ cu, int G,
                                                       const float* __restrict__ perm_w, int M, int I, ActArgs a,
                                                       void* __restrict__ out) {
    pdl_wait();
    const int c8n = I / 8;
    const long long n8 = (long long)M * c8n;
    for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < n8;
         v += (long long)gridDim.x * blockDim.x) {
        const int r = (int)(v / c8n);
        const int c = (int)(v - (long long)r * c8n) * 8;
        const size_t i = (size_t)r * I + c;
        const int g = segment_of(cu, G, r);
        float o[8];
        if (g < G) {
            float gv[8], uv[8];
            ld8<IN_F32>(gate, i, gv);
            ld8<IN_F32>(up, i, uv);
            if (bg) {
                float b[8];
                ld8<true>(bg, (size_t)g * I + c, b);
#pragma unroll
                for (int q = 0; q < 8; ++q) gv[q] += b[q];
            }
            if (bu) {
                float b[8];
                ld8<true>(bu, (size_t)g * I + c, b);
#pragma unroll
                for (int q = 0; q < 8; ++q) uv[q] += b[q];
            }
            const float pw = perm_w ? perm_w[r] : 1.0f;
#pragma unroll
            for (int q = 0; q < 8; ++q) o[q] = act_ex(a, gv[q], uv[q]) * pw;
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) o[q] = 0.0f;
        }
        st8<OUT_F32>(out, i, o);
    }
    pdl_launch();
}

namespace {
inline int row_pass_blocks(long long n8) {
    return (int)std::min<long long>((n8 + 255) / 256, (long long)num_sms() * 16);
}
}  // namespace

cudaError_t launch_bias_act(const void* gate, const void* up, bool in_f32, const float* bg, const float* bu,
                            const int32_t* cu, int G, const float* perm_w, int M, int I, int act, float sa, float sb,
                            float oa, float ob, float lim, void* out, bool out_f32, cudaStream_t st, bool pdl) {
    const long long n8 = (long long)M * (I / 8);
    if (n8 == 0) return cudaSuccess;
    const ActArgs a{act, sa, sb, oa, ob, lim};
    const dim3 grid(row_pass_blocks(n8)), block(256);
    if (in_f32) {
        if (out_f32)
            return launch_k(bias_act_kernel<true, true>, grid, block, 0, st, pdl, gate, up, bg, bu, cu, G, perm_w, M,
                            I, a, out);
        return launch_k(bias_act_kernel<true, false>, grid, block, 0, st, pdl, gate, up, bg, bu, cu, G, perm_w, M, I,
                        a, out);
    }
    if (out_f32)
        return launch_k(bias_act_kernel<false, true>, grid, block, 0, st, pdl, gate, up, bg, bu, cu, G, perm_w, M, I,
                        a, out);
    return launch_k(bias_act_kernel<false, false>, grid, block, 0, st, pdl, gate, up, bg, bu, cu, G, perm_w, M, I, a,
                    out);
}

}  // namespace moe
