// S0 — one-time conversion of FP4 weights into the grouped GEMMs' tile layouts
// (the "kernel format" of the FlashInfer MoE-EP page's
// process_weights_after_loading and the DeepSeek-V4 FI page's finalize_weights).
//
// NVFP4:
//   kdata: chunks [g][nt][kb] for weight row g, 128-row block nt and 64-value K block
//          kb, the number of K blocks padded to even (a pipeline stage covers 128 K
//          values); each chunk of 4096 + 512 bytes holds 128 rows x 32 bytes of packed
//          e2m1 (even k in the low nibble), zero past N and K, then 128 rows x 4 e4m3
//          scales, so one stage is one contiguous copy per matrix (the GEMM that stages
//          the weights as f16 for bf16 activations).
//   kscale: K % 256 == 0 -> the block-scaled tiles [g][nt][ks] of 128 rows x 256 K
//          values (kNvf4TileBytes each: the swizzled code image, then the scale blocks in
//          tensor-memory copy order), read by the GEMM that takes NVFP4 activations;
//          otherwise the same address as kdata.
// MXFP4:
//   kdata: packed codes [g][n][Kp/2], K zero-padded to a multiple of 128;
//   kscale: the e8m0 scale blocks [g][nt][kb], 512 bytes per 128 rows x 128 K values.
// kalpha: fp32 [G], the epilogue alpha (NVFP4 weight_scale_2; 1 if absent).
#include <vector>

#include "internal.h"

namespace moe {

namespace {

struct PrepLayout {
    int NT, KB, KS;
    size_t data_off, scale_off, alpha_off, scratch_off, bytes;
};

bool has_nvf4_tiles(const moe_weight_t* w) { return w->fmt == MOE_W_NVFP4 && w->K % kNvf4StageK == 0; }

PrepLayout prep_layout(const moe_weight_t* w) {
    PrepLayout L{};
    L.NT = (w->N + kTileN - 1) / kTileN;
    L.KB = 2 * ((w->K + 2 * kTileK - 1) / (2 * kTileK));  // padded to even
    const size_t chunks = (size_t)w->G * L.NT * L.KB;
    size_t off = 0;
    auto take = [&](size_t b) {
        const size_t o = off;
        off += (b + 255) & ~size_t(255);
        return o;
    };
    if (w->fmt == MOE_W_MXFP4) {
        // padded codes for the 4-bit tensor map, then the scale blocks
        const int Kp = mx8_kpad(w->K);
        L.KS = Kp / kMx8StageK;
        L.data_off = take((size_t)w->G * w->N * (Kp / 2));
        L.scale_off = take((size_t)w->G * L.NT * L.KS * 512);
    } else {
        L.data_off = take(chunks * fp4_chunk_bytes(w->fmt));
        L.KS = w->K / kNvf4StageK;
        L.scale_off = has_nvf4_tiles(w) ? take((size_t)w->G * L.NT * L.KS * kNvf4TileBytes) : L.data_off;
    }
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

// NVFP4, one block per (g, nt, kb) chunk; thread r copies weight row nt*128 + r.
__global__ void __launch_bounds__(128) relayout_kernel(const uint8_t* __restrict__ data,
                                                       const uint8_t* __restrict__ scale, int N, int K, int NT,
                                                       int KB, uint8_t* __restrict__ chunks) {
    const size_t tile = blockIdx.x;
    const int kb = (int)(tile % KB);
    const int nt = (int)((tile / KB) % NT);
    const size_t g = tile / ((size_t)KB * NT);
    const int r = threadIdx.x;
    const int n = nt * kTileN + r;
    const int row_bytes = K / 2;
    const int KS = K / 16;
    uint8_t* chunk = chunks + tile * (size_t)(kTileN * 32 + kTileN * 4);
    uint8_t out[32];
    for (int i = 0; i < 32; ++i) {
        const int byte = kb * 32 + i;
        out[i] = (n < N && byte < row_bytes) ? data[(g * N + n) * row_bytes + byte] : (uint8_t)0;
    }
    uint4* d = reinterpret_cast<uint4*>(chunk + r * 32);
    d[0] = *reinterpret_cast<uint4*>(out);
    d[1] = *reinterpret_cast<uint4*>(out + 16);
    uint8_t* kscale = chunk + kTileN * 32;
    for (int i = 0; i < 4; ++i) {
        const int si = kb * 4 + i;
        kscale[r * 4 + i] = (n < N && si < KS) ? scale[(g * N + n) * KS + si] : (uint8_t)0;
    }
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

// MXFP4 codes [G, N, K/2] -> [G, N, Kp/2], zero past K; one thread per 16 bytes.
__global__ void mx_codes_pad_kernel(const uint8_t* __restrict__ data, long long rows, int K, int Kp,
                                    uint8_t* __restrict__ dst) {
    const int per_row = Kp / 32;  // 16-byte chunks per padded row
    const long long n = rows * per_row;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const long long r = i / per_row;
        const int c = (int)(i - r * per_row);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (c * 32 < K) v = *reinterpret_cast<const uint4*>(data + r * (K / 2) + (size_t)c * 16);
        *reinterpret_cast<uint4*>(dst + r * (Kp / 2) + (size_t)c * 16) = v;
    }
}

// MXFP4 e8m0 scales [G, N, K/32] -> 512-byte blocks per (g, nt, kb); one thread per
// (block, row m). Rows past N and blocks past K get 127 (their codes are zero).
__global__ void mx_scale_blocks_kernel(const uint8_t* __restrict__ scale, int G, int N, int K, int NT, int KS,
                                       uint8_t* __restrict__ blocks) {
    const long long n = (long long)G * NT * KS * kTileN;
    const int ks_row = K / 32;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const int m = (int)(i % kTileN);
        const long long blk = i / kTileN;
        const int kb = (int)(blk % KS);
        const int nt = (int)((blk / KS) % NT);
        const long long g = blk / ((long long)KS * NT);
        const int row = nt * kTileN + m;
        uint32_t word = 0;
        for (int j = 0; j < 4; ++j) {
            const int si = kb * 4 + j;
            uint32_t v = 127;
            if (row < N && si < ks_row) v = scale[((size_t)g * N + row) * ks_row + si];
            word |= v << (8 * j);
        }
        *reinterpret_cast<uint32_t*>(blocks + blk * 512 + 16 * (m & 31) + 4 * (m >> 5)) = word;
    }
}

__global__ void alpha_kernel(const float* __restrict__ alpha, int G, float* __restrict__ kalpha) {
    for (int g = blockIdx.x * blockDim.x + threadIdx.x; g < G; g += gridDim.x * blockDim.x)
        kalpha[g] = alpha ? alpha[g] : 1.0f;
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
    uint8_t* kdata = reinterpret_cast<uint8_t*>(base + L.data_off);
    uint8_t* kscale = reinterpret_cast<uint8_t*>(base + L.scale_off);
    float* kalpha = reinterpret_cast<float*>(base + L.alpha_off);
    const uint8_t* data = static_cast<const uint8_t*>(w->data);
    const uint8_t* scale = static_cast<const uint8_t*>(w->scale);
    if (w->fmt == MOE_W_MXFP4) {
        // an e8m0 NaN scale (255) is rejected
        int* mm = reinterpret_cast<int*>(base + L.scratch_off);
        std::vector<int> h_mm(2 * (size_t)w->G, 0);
        mx_scale_range_kernel<<<w->G, 256, 0, st>>>(scale, w->N, w->K / 32, mm);
        if (cudaMemcpyAsync(h_mm.data(), mm, sizeof(int) * 2 * w->G, cudaMemcpyDeviceToHost, st) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
        for (int g = 0; g < w->G; ++g)
            if (h_mm[2 * g] < 0) return MOE_ERR_INVALID_ARG;
        const int Kp = mx8_kpad(w->K);
        const long long rows = (long long)w->G * w->N;
        const long long n16 = rows * (Kp / 32), nblk = (long long)w->G * L.NT * L.KS * kTileN;
        const unsigned gb = (unsigned)std::min<long long>((n16 + 255) / 256, 65535LL * 16);
        const unsigned sbk = (unsigned)std::min<long long>((nblk + 255) / 256, 65535LL * 16);
        if (n16 > 0) mx_codes_pad_kernel<<<gb, 256, 0, st>>>(data, rows, w->K, Kp, kdata);
        if (nblk > 0) mx_scale_blocks_kernel<<<sbk, 256, 0, st>>>(scale, w->G, w->N, w->K, L.NT, L.KS, kscale);
    } else {
        const size_t tiles = (size_t)w->G * L.NT * L.KB;
        if (tiles > 0) relayout_kernel<<<(unsigned)tiles, 128, 0, st>>>(data, scale, w->N, w->K, L.NT, L.KB, kdata);
        const size_t ntiles = has_nvf4_tiles(w) ? (size_t)w->G * L.NT * L.KS : 0;
        if (ntiles > 0)
            relayout_nvf4_kernel<<<(unsigned)ntiles, 128, 0, st>>>(data, scale, w->N, w->K, L.NT, L.KS, kscale);
    }
    alpha_kernel<<<(w->G + 255) / 256, 256, 0, st>>>(w->alpha, w->G, kalpha);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    w->kdata = kdata;
    w->kscale = kscale;
    w->kalpha = kalpha;
    return MOE_OK;
}

}  // namespace moe
