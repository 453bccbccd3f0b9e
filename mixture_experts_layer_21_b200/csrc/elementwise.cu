// S4 activation, S6 combine and S2q NVFP4 activation quantisation.
#include "internal.h"

namespace moe {

// ----------------------------------------------------------------- S4
// out[r,i] = act(gate[r,i], up[r,i]) * perm_w[r], fp32 math, one bf16 rounding.
// (MoonEP experts page, MoonEPExperts.apply; SITU form from the TRTLLM MXFP4 page.)
__global__ void __launch_bounds__(256) act_and_mul_kernel(const __nv_bfloat16* __restrict__ gate,
                                                          const __nv_bfloat16* __restrict__ up,
                                                          const float* __restrict__ perm_w, int M,
                                                          int I, int act, float sa, float sb,
                                                          __nv_bfloat16* __restrict__ out) {
    pdl_wait();
    const long long n8 = (long long)M * I / 8;
    for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < n8;
         v += (long long)gridDim.x * blockDim.x) {
        const long long e0 = v * 8;
        const int r = (int)(e0 / I);
        const float pw = perm_w ? perm_w[r] : 1.0f;
        const uint4 g = reinterpret_cast<const uint4*>(gate)[v];
        const uint4 u = reinterpret_cast<const uint4*>(up)[v];
        const __nv_bfloat162* gp = reinterpret_cast<const __nv_bfloat162*>(&g);
        const __nv_bfloat162* up2 = reinterpret_cast<const __nv_bfloat162*>(&u);
        uint4 o;
        __nv_bfloat162* op = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 gf = __bfloat1622float2(gp[q]);
            const float2 uf = __bfloat1622float2(up2[q]);
            op[q] = __floats2bfloat162_rn(act_apply(act, gf.x, uf.x, sa, sb) * pw,
                                          act_apply(act, gf.y, uf.y, sa, sb) * pw);
        }
        reinterpret_cast<uint4*>(out)[v] = o;
    }
    pdl_launch();
}

cudaError_t launch_act_and_mul(const __nv_bfloat16* gate, const __nv_bfloat16* up,
                               const float* perm_w, int M, int I, int act, float sa, float sb,
                               __nv_bfloat16* out, cudaStream_t st, bool pdl) {
    const long long n8 = (long long)M * I / 8;
    if (n8 == 0) return cudaSuccess;
    const int blocks = (int)std::min<long long>((n8 + 255) / 256, (long long)num_sms() * 16);
    return launch_k(act_and_mul_kernel, dim3(blocks), dim3(256), 0, st, pdl, gate, up, perm_w, M, I,
                    act, sa, sb, out);
}

// ----------------------------------------------------------------- input-side route weight
// out[t,:] = x[t,:] * w[t] (top-1 routing with the weight on the input), fp32 product,
// one bf16 rounding. H % 8 == 0.
__global__ void __launch_bounds__(256) scale_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                         const float* __restrict__ w, int T, int H,
                                                         __nv_bfloat16* __restrict__ out) {
    pdl_wait();
    const long long n8 = (long long)T * H / 8;
    for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < n8;
         v += (long long)gridDim.x * blockDim.x) {
        const float s = w[(v * 8) / H];
        const uint4 a = reinterpret_cast<const uint4*>(x)[v];
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&a);
        uint4 o;
        __nv_bfloat162* q = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(p[i]);
            q[i] = __floats2bfloat162_rn(f.x * s, f.y * s);
        }
        reinterpret_cast<uint4*>(out)[v] = o;
    }
    pdl_launch();
}

cudaError_t launch_scale_rows(const __nv_bfloat16* x, const float* w, int T, int H, __nv_bfloat16* out,
                              cudaStream_t st, bool pdl) {
    const long long n8 = (long long)T * H / 8;
    if (n8 == 0) return cudaSuccess;
    const int blocks = (int)std::min<long long>((n8 + 255) / 256, (long long)num_sms() * 16);
    return launch_k(scale_rows_kernel, dim3(blocks), dim3(256), 0, st, pdl, x, w, T, H, out);
}

// ----------------------------------------------------------------- S6
// out[t] = sum_k w[t,k] * y[inv_perm[t,k]], fp32 in k order, one bf16 rounding.
// Grid (T, ceil(H / 1024)); each thread owns 8 contiguous columns. y is bf16 (the
// standalone entry point) or fp32 (the fused layer keeps the down projection's rows
// in fp32 so that the output is rounded to bf16 once).
__device__ __forceinline__ void load8(const __nv_bfloat16* y, size_t row, int H, int c8, float (&f)[8]) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(y + row * H) + c8);
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float2 g = __bfloat1622float2(p[q]);
        f[2 * q] = g.x;
        f[2 * q + 1] = g.y;
    }
}
__device__ __forceinline__ void load8(const float* y, size_t row, int H, int c8, float (&f)[8]) {
    const float4* p = reinterpret_cast<const float4*>(y + row * H) + 2 * c8;
    const float4 a = __ldg(p), b = __ldg(p + 1);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

template <typename YT>
__global__ void __launch_bounds__(128) combine_kernel(const YT* __restrict__ y,
                                                      const int32_t* __restrict__ inv_perm,
                                                      const float* __restrict__ topk_w, int T,
                                                      int topk, int H,
                                                      __nv_bfloat16* __restrict__ out) {
    pdl_wait();
    const int t = blockIdx.x;
    const int c8 = blockIdx.y * 128 + threadIdx.x;  // index of an 8-column chunk
    if (c8 < H / 8) {
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
        for (int j = 0; j < topk; ++j) {
            const int r = inv_perm[(size_t)t * topk + j];
            if (r < 0) continue;  // an assignment the permutation refused (bad expert id)
            const float wj = topk_w ? topk_w[(size_t)t * topk + j] : 1.0f;
            float f[8];
            load8(y, (size_t)r, H, c8, f);
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = topk_w ? fmaf(wj, f[q], acc[q]) : acc[q] + f[q];
        }
        uint4 o;
        __nv_bfloat162* op = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
        for (int q = 0; q < 4; ++q) op[q] = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
        reinterpret_cast<uint4*>(out + (size_t)t * H)[c8] = o;
    }
    (void)T;
    pdl_launch();
}

cudaError_t launch_combine(const __nv_bfloat16* y, const int32_t* inv_perm, const float* topk_w,
                           int T, int topk, int H, __nv_bfloat16* out, cudaStream_t st, bool pdl) {
    if (T == 0) return cudaSuccess;
    dim3 grid(T, (H / 8 + 127) / 128);
    return launch_k(combine_kernel<__nv_bfloat16>, grid, dim3(128), 0, st, pdl, y, inv_perm, topk_w, T, topk,
                    H, out);
}

cudaError_t launch_combine_f32(const float* y, const int32_t* inv_perm, const float* topk_w, int T, int topk,
                               int H, __nv_bfloat16* out, cudaStream_t st, bool pdl) {
    if (T == 0) return cudaSuccess;
    dim3 grid(T, (H / 8 + 127) / 128);
    return launch_k(combine_kernel<float>, grid, dim3(128), 0, st, pdl, y, inv_perm, topk_w, T, topk, H, out);
}

// ----------------------------------------------------------------- S2q
// Dynamic NVFP4 quantisation of rows, one warp per row; every decision in fp32
// with IEEE division:
//   s_r  = amax_r / 2688
//   sb   = e4m3_rne_satfinite(amax_b / (6 s_r))   per 16 values
//   q    = e2m1_rne_satfinite(v / (sb s_r))
// A zero row or a block scale that rounds to zero gives +0 codes.
// Two values -> one byte: `lo` in the low nibble.
__device__ __forceinline__ uint8_t cvt_e2m1x2(float lo, float hi) {
    uint16_t r;
    asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u16.u8 %0, t; }"
        : "=h"(r)
        : "f"(hi), "f"(lo));
    return (uint8_t)r;
}
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint8_t b) {
    uint32_t r;
    asm("{ .reg .b8 t; cvt.u8.u16 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(r) : "h"((uint16_t)b));
    return r;
}

template <bool IN_F32>
__device__ __forceinline__ void load16(const void* base, size_t off, float (&v)[16]) {
    if (IN_F32) {
        const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + off);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 f = p[q];
            v[4 * q] = f.x;
            v[4 * q + 1] = f.y;
            v[4 * q + 2] = f.z;
            v[4 * q + 3] = f.w;
        }
    } else {
        const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(base) + off);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const uint4 u = p[q];
            const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(b[i]);
                v[8 * q + 2 * i] = f.x;
                v[8 * q + 2 * i + 1] = f.y;
            }
        }
    }
}

template <bool IN_F32>
__global__ void __launch_bounds__(256) quant_nvfp4_kernel(const void* __restrict__ in, int R, int K,
                                                          uint8_t* __restrict__ codes, int cstride,
                                                          uint8_t* __restrict__ sbo, int sstride,
                                                          float* __restrict__ so,
                                                          __half* __restrict__ deq,
                                                          const int32_t* __restrict__ row_idx, int in_rows) {
    pdl_wait();
    const int r = blockIdx.x * 8 + warp_id();
    const int lane = lane_id();
    if (r < R) {
        const int nb = K / 16;
        // output row r quantises input row r, or row_idx[r] (clamped into the input)
        const size_t ri = row_idx ? (size_t)min(max(row_idx[r], 0), in_rows - 1) : (size_t)r;
        float amax = 0.0f;
        for (int b = lane; b < nb; b += 32) {
            float v[16];
            load16<IN_F32>(in, ri * K + b * 16, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        const float s = __fdiv_rn(amax, 2688.0f);
        const float six_s = __fmul_rn(6.0f, s);
        for (int b = lane; b < nb; b += 32) {
            float v[16];
            load16<IN_F32>(in, ri * K + b * 16, v);
            float bmax = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(v[i]));
            const uint8_t sbc = six_s > 0.0f ? cvt_e4m3(__fdiv_rn(bmax, six_s)) : (uint8_t)0;
            const float sbv = e4m3_to_f32(sbc);
            const float step = __fmul_rn(sbv, s);
            uint32_t packed[2] = {0u, 0u};
            if (step > 0.0f) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint8_t byte = cvt_e2m1x2(__fdiv_rn(v[2 * i], step), __fdiv_rn(v[2 * i + 1], step));
                    packed[i >> 2] |= (uint32_t)byte << (8 * (i & 3));
                }
            }
            *reinterpret_cast<uint2*>(codes + (size_t)r * cstride + b * 8) = make_uint2(packed[0], packed[1]);
            sbo[(size_t)r * sstride + b] = sbc;
            if (deq) {
                const __half hsb = __float2half_rn(sbv);  // exact: e4m3 values are f16 values
                const __half2 sb2 = __halves2half2(hsb, hsb);
                uint32_t o[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint8_t byte = (uint8_t)(packed[i >> 2] >> (8 * (i & 3)));
                    uint32_t raw = e2m1x2_to_f16x2(byte);
                    __half2 h = __hmul2(*reinterpret_cast<const __half2*>(&raw), sb2);
                    o[i] = *reinterpret_cast<uint32_t*>(&h);
                }
                uint4* d = reinterpret_cast<uint4*>(deq + (size_t)r * K + b * 16);
                d[0] = make_uint4(o[0], o[1], o[2], o[3]);
                d[1] = make_uint4(o[4], o[5], o[6], o[7]);
            }
        }
        if (lane == 0) so[r] = s;
    }
    pdl_launch();
}


// ----------------------------------------------------------------- MXFP8 activations
// Activation rows for the MXFP4-weight GEMM, whose tensor cores take e4m3 activations with
// one e8m0 scale per 32 values. Two forms:
//   hi/lo (bf16 activations): each 32-value block b gets the smallest power of two 2^e
//     with amax_b <= 448 * 2^e, then y = v * 2^-e (exact), hi = e4m3_rne(y) and
//     lo = e4m3_rne(y - hi) (the difference is exact in fp32), so v = (hi + lo) * 2^e to
//     within 1.07 * 2^-8 |v| + 2^(e-10).
//   one term (dynamic MXFP8, the OCP MX v1.0 conversion): 2^e = 2^(floor(log2 amax_b) - 8)
//     and q = e4m3_rne_satfinite(v * 2^-e) (saturating at 448).
// One warp per row, one 32-value block per lane and step; blocks past K (up to Kp) are zero.
// (mx8_block_exp, in common.cuh, picks e.)
template <bool IN_F32, bool TWO>
__global__ void __launch_bounds__(256) quant_mx8_kernel(const void* __restrict__ in, int R, int K, int Kp,
                                                        uint8_t* __restrict__ hi_out, uint8_t* __restrict__ lo_out,
                                                        uint8_t* __restrict__ sc_out, int code_stride,
                                                        int sc_stride, const int32_t* __restrict__ row_idx,
                                                        int in_rows) {
    pdl_wait();
    const int r = blockIdx.x * 8 + warp_id();
    const int lane = lane_id();
    if (r < R) {
        // output row r stages input row r, or row_idx[r] (clamped into the input)
        const size_t ri = row_idx ? (size_t)min(max(row_idx[r], 0), in_rows - 1) : (size_t)r;
        for (int b = lane; b < Kp / 32; b += 32) {
            uint32_t hi[8] = {0, 0, 0, 0, 0, 0, 0, 0}, lo[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            int e = -127;
            if (b * 32 < K) {
                float v[2][16];
                load16<IN_F32>(in, ri * K + b * 32, v[0]);
                load16<IN_F32>(in, ri * K + b * 32 + 16, v[1]);
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i >> 4][i & 15]));
                e = mx8_block_exp(amax, TWO);
                const float inv = mx8_inv_scale(e);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float y = v[i >> 4][i & 15] * inv;
                    const uint8_t h = cvt_e4m3(y);
                    hi[i >> 2] |= (uint32_t)h << (8 * (i & 3));
                    if (TWO) lo[i >> 2] |= (uint32_t)cvt_e4m3(y - e4m3_to_f32(h)) << (8 * (i & 3));
                }
            }
            uint4* ph = reinterpret_cast<uint4*>(hi_out + (size_t)r * code_stride + b * 32);
            ph[0] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            ph[1] = make_uint4(hi[4], hi[5], hi[6], hi[7]);
            if (TWO) {
                uint4* pl = reinterpret_cast<uint4*>(lo_out + (size_t)r * code_stride + b * 32);
                pl[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                pl[1] = make_uint4(lo[4], lo[5], lo[6], lo[7]);
            }
            sc_out[(size_t)r * sc_stride + b] = (uint8_t)(e + 127);
        }
    }
    pdl_launch();
}

cudaError_t launch_quant_mx8(const void* in, bool in_f32, int R, int K, int Kp, bool two, uint8_t* hi, uint8_t* lo,
                             uint8_t* sc, int code_stride, int sc_stride, cudaStream_t st, bool pdl,
                             const int32_t* row_idx, int in_rows) {
    if (R <= 0) return cudaSuccess;
    dim3 grid((R + 7) / 8), block(256);
    if (two) {
        if (in_f32)
            return launch_k(quant_mx8_kernel<true, true>, grid, block, 0, st, pdl, in, R, K, Kp, hi, lo, sc,
                            code_stride, sc_stride, row_idx, in_rows);
        return launch_k(quant_mx8_kernel<false, true>, grid, block, 0, st, pdl, in, R, K, Kp, hi, lo, sc,
                        code_stride, sc_stride, row_idx, in_rows);
    }
    if (in_f32)
        return launch_k(quant_mx8_kernel<true, false>, grid, block, 0, st, pdl, in, R, K, Kp, hi, lo, sc,
                        code_stride, sc_stride, row_idx, in_rows);
    return launch_k(quant_mx8_kernel<false, false>, grid, block, 0, st, pdl, in, R, K, Kp, hi, lo, sc, code_stride,
                    sc_stride, row_idx, in_rows);
}

cudaError_t launch_quant_nvfp4(const void* in, bool in_f32, int R, int K, uint8_t* codes, int codes_stride,
                               uint8_t* sb, int sb_stride, float* s, __half* deq, cudaStream_t st, bool pdl,
                               const int32_t* row_idx, int in_rows) {
    if (R <= 0) return cudaSuccess;
    dim3 grid((R + 7) / 8), block(256);
    if (in_f32)
        return launch_k(quant_nvfp4_kernel<true>, grid, block, 0, st, pdl, in, R, K, codes, codes_stride, sb,
                        sb_stride, s, deq, row_idx, in_rows);
    return launch_k(quant_nvfp4_kernel<false>, grid, block, 0, st, pdl, in, R, K, codes, codes_stride, sb, sb_stride,
                    s, deq, row_idx, in_rows);
}

}  // namespace moe
