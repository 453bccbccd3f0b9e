// S0 — one-time conversion of FP4 weights into the grouped GEMM's tile layout
// (the "kernel format" of the FlashInfer MoE-EP page's
// process_weights_after_loading and the DeepSeek-V4 FI page's finalize_weights).
//
// Layout: chunks [g][nt][kb] for weight row g, 128-row block nt and 64-value K block
// kb, the number of K blocks padded to even (a pipeline stage covers 128 K values);
// each chunk of kFp4ChunkBytes(fmt) = 4096 + 128*S bytes holds
//   128 rows x 32 bytes of packed e2m1 (even k in the low nibble), zero past N and K,
//   then 128 rows x S scale bytes, S = 2 (MXFP4, two e8m0 per 64) or 4 (NVFP4, four e4m3),
// so one stage is one contiguous copy per matrix. kdata points at it.
//   kscale: NVFP4 with K % 256 == 0 -> the block-scaled tiles [g][nt][ks] of 128 rows x
//           256 K values (kNvf4TileBytes each: the swizzled code image, then the scale
//           blocks in tensor-memory copy order), read by the GEMM that takes NVFP4
//           activations; otherwise the same address as kdata.
//   kalpha: fp32 [G]. NVFP4: weight_scale_2 (1 if absent). MXFP4: 2^bias_g, where
//           bias_g re-bases expert g's e8m0 exponents so its largest block scale is
//           2^13; the GEMM stages e2m1 * 2^(e-127-bias) in f16, exact while the
//           expert's scales span at most 36 binades.
#include <vector>

#include "internal.h"

namespace moe {

namespace {

constexpr int kMxTop = 140;   // re-biased exponent of the largest MXFP4 scale (2^13)
constexpr int kMxFloor = 104; // smallest re-biased exponent staged exactly in f16

struct PrepLayout {
    int NT, KB, S, KS;
    size_t data_off, scale_off, alpha_off, scratch_off, bytes;
};

bool has_nvf4_tiles(const moe_weight_t* w) { return w->fmt == MOE_W_NVFP4 && w->K % kNvf4StageK == 0; }

PrepLayout prep_layout(const moe_weight_t* w) {
    PrepLayout L{};
    L.NT = (w->N + kTileN - 1) / kTileN;
    L.KB = 2 * ((w->K + 2 * kTileK - 1) / (2 * kTileK));  // padded to even
    L.S = fp4_scale_bytes_per_row(w->fmt);
    const size_t chunks = (size_t)w->G * L.NT * L.KB;
    size_t off = 0;
    auto take = [&](size_t b) {
        const size_t o = off;
        off += (b + 255) & ~size_t(255);
        return o;
    };
    L.data_off = take(chunks * fp4_chunk_bytes(w->fmt));
    L.KS = w->K / kNvf4StageK;
    L.scale_off = has_nvf4_tiles(w) ? take((size_t)w->G * L.NT * L.KS * kNvf4TileBytes) : L.data_off;
    L.alpha_off = take(sizeof(float) * w->G);
    L.scratch_off = take(sizeof(int) * 2 * w->G + 16);
    L.bytes = off;
    return L;
}

__global__ void mx_scale_range_kernel(const uint8_t* __restrict__ scale, int N, int KS, int* __restrict__ mm) {
    // one block per weight row g: min and max e8m0 exponent, and a NaN (255) flag
    const uint8_t* s = scale + (size_t)blockIdx.x * N * KS;
    int lo = 255, hi = 0, nan = 0;
    for (size_t i = threadIdx.x; i < (size_t)N * KS; i += blockDim.x) {
        const int v = s[i];
        nan |= (v == 255);
        lo = min(lo, v);
        hi = max(hi, v);
    }
    for (int off = 16; off > 0; off >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        nan |= __shfl_xor_sync(0xffffffffu, nan, off);
    }
    __shared__ int slo[32], shi[32], snan[32];
    if ((threadIdx.x & 31) == 0) {
        slo[threadIdx.x >> 5] = lo;
        shi[threadIdx.x >> 5] = hi;
        snan[threadIdx.x >> 5] = nan;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 1; i < (int)(blockDim.x >> 5); ++i) {
            lo = min(lo, slo[i]);
            hi = max(hi, shi[i]);
            nan |= snan[i];
        }
        mm[2 * blockIdx.x] = nan ? -1 : lo;
        mm[2 * blockIdx.x + 1] = hi;
    }
}

// One block per (g, nt, kb) chunk; thread r copies weight row nt*128 + r.
__global__ void __launch_bounds__(128) relayout_kernel(const uint8_t* __restrict__ data,
                                                       const uint8_t* __restrict__ scale, int fmt,
                                                       int G, int N, int K, int NT, int KB,
                                                       const int* __restrict__ bias,
                                                       uint8_t* __restrict__ chunks) {
    const size_t tile = blockIdx.x;
    const int kb = (int)(tile % KB);
    const int nt = (int)((tile / KB) % NT);
    const int g = (int)(tile / ((size_t)KB * NT));
    const int r = threadIdx.x;
    const int n = nt * kTileN + r;
    const int row_bytes = K / 2;
    const int S = fmt == MOE_W_MXFP4 ? 2 : 4;
    const int per = fmt == MOE_W_MXFP4 ? 32 : 16;  // values per scale
    const int KS = K / per;
    uint8_t* chunk = chunks + tile * (size_t)(kTileN * 32 + kTileN * S);
    uint8_t out[32];
    for (int i = 0; i < 32; ++i) {
        const int byte = kb * 32 + i;
        out[i] = (n < N && byte < row_bytes) ? data[((size_t)g * N + n) * row_bytes + byte] : (uint8_t)0;
    }
    uint4* d = reinterpret_cast<uint4*>(chunk + r * 32);
    d[0] = *reinterpret_cast<uint4*>(out);
    d[1] = *reinterpret_cast<uint4*>(out + 16);
    uint8_t* kscale = chunk + kTileN * 32;
    for (int i = 0; i < S; ++i) {
        const int si = kb * S + i;
        uint8_t v = 0;
        if (n < N && si < KS) {
            v = scale[((size_t)g * N + n) * KS + si];
            if (fmt == MOE_W_MXFP4) v = (uint8_t)min(255, max(0, (int)v - bias[g]));
        } else if (fmt == MOE_W_MXFP4) {
            v = 127;  // any finite scale: these codes are zero
        }
        kscale[r * S + i] = v;
    }
    (void)G;
}

// One block per block-scaled tile (g, nt, ks); thread m writes weight row nt*128 + m.
// Rows past N are zero codes with zero scales.
__global__ void __launch_bounds__(128) relayout_nvf4_kernel(const uint8_t* __restrict__ data,
                                                            const uint8_t* __restrict__ scale, int N, int K,
                                                            int NT, int KS, uint8_t* __restrict__ tiles) {
    const size_t tile = blockIdx.x;
    const int ks = (int)(tile % KS);
    const int nt = (int)((tile / KS) % NT);
    const size_t g = tile / ((size_t)KS * NT);
    const int m = threadIdx.x;
    const int n = nt * kTileN + m;
    const bool live = n < N;
    uint8_t* t = tiles + tile * (size_t)kNvf4TileBytes;
    const uint4* src = reinterpret_cast<const uint4*>(data + (g * N + n) * (size_t)(K / 2) + (size_t)ks * 128);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 v = live ? src[c] : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(t + m * 128 + ((c ^ (m & 7)) << 4)) = v;
    }
    // 16 scales of this row for the tile's 256 values: four per 64-value block j
    const uint8_t* srow = scale + (g * N + n) * (size_t)(K / 16) + (size_t)ks * 16;
    uint8_t* sf = t + kNvf4CodeBytes;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t word = 0;
        if (live)  // byte loads: the caller's scale plane need not be 4-byte aligned
            word = (uint32_t)srow[4 * j] | (uint32_t)srow[4 * j + 1] << 8 | (uint32_t)srow[4 * j + 2] << 16 |
                   (uint32_t)srow[4 * j + 3] << 24;
        *reinterpret_cast<uint32_t*>(sf + j * 512 + 16 * (m & 31) + 4 * (m >> 5)) = word;
    }
}

__global__ void alpha_kernel(const float* __restrict__ alpha, const int* __restrict__ bias, int fmt, int G,
                             float* __restrict__ kalpha) {
    for (int g = blockIdx.x * blockDim.x + threadIdx.x; g < G; g += gridDim.x * blockDim.x) {
        float a = alpha ? alpha[g] : 1.0f;
        if (fmt == MOE_W_MXFP4) a *= ldexpf(1.0f, bias[g]);
        kalpha[g] = a;
    }
}

}  // namespace

size_t prepared_weight_bytes(const moe_weight_t* w) {
    if (w->fmt == MOE_W_BF16) return 0;
    return prep_layout(w).bytes;
}

moe_status_t prepare_weights(moe_weight_t* w, void* dst, size_t dst_bytes, cudaStream_t st) {
    if (w->fmt == MOE_W_BF16) return MOE_OK;
    const PrepLayout L = prep_layout(w);
    if (dst_bytes < L.bytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
    char* base = static_cast<char*>(dst);
    int* mm = reinterpret_cast<int*>(base + L.scratch_off);
    std::vector<int> h_mm(2 * (size_t)w->G, 0), h_bias(w->G, 0);
    if (w->fmt == MOE_W_MXFP4) {
        mx_scale_range_kernel<<<w->G, 256, 0, st>>>(static_cast<const uint8_t*>(w->scale), w->N, w->K / 32, mm);
        if (cudaMemcpyAsync(h_mm.data(), mm, sizeof(int) * 2 * w->G, cudaMemcpyDeviceToHost, st) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
        for (int g = 0; g < w->G; ++g) {
            const int lo = h_mm[2 * g], hi = h_mm[2 * g + 1];
            if (lo < 0) return MOE_ERR_INVALID_ARG;  // an e8m0 NaN scale
            h_bias[g] = hi - kMxTop;
            if (lo - h_bias[g] < kMxFloor) return MOE_ERR_UNSUPPORTED;
        }
    }
    // the per-row exponent bias overwrites the (consumed) range scratch
    int* d_bias = mm;
    if (cudaMemcpyAsync(d_bias, h_bias.data(), sizeof(int) * w->G, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    const size_t tiles = (size_t)w->G * L.NT * L.KB;
    uint8_t* kdata = reinterpret_cast<uint8_t*>(base + L.data_off);
    uint8_t* kscale = reinterpret_cast<uint8_t*>(base + L.scale_off);
    float* kalpha = reinterpret_cast<float*>(base + L.alpha_off);
    if (tiles > 0) {
        relayout_kernel<<<(unsigned)tiles, 128, 0, st>>>(static_cast<const uint8_t*>(w->data),
                                                          static_cast<const uint8_t*>(w->scale), w->fmt, w->G, w->N,
                                                          w->K, L.NT, L.KB, d_bias, kdata);
    }
    if (has_nvf4_tiles(w) && w->N > 0) {
        const size_t ntiles = (size_t)w->G * L.NT * L.KS;
        if (ntiles > 0)
            relayout_nvf4_kernel<<<(unsigned)ntiles, 128, 0, st>>>(static_cast<const uint8_t*>(w->data),
                                                                   static_cast<const uint8_t*>(w->scale), w->N,
                                                                   w->K, L.NT, L.KS, kscale);
    }
    alpha_kernel<<<(w->G + 255) / 256, 256, 0, st>>>(w->alpha, d_bias, w->fmt, w->G, kalpha);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    w->kdata = kdata;
    w->kscale = kscale;
    w->kalpha = kalpha;
    return MOE_OK;
}

}  // namespace moe
