// S1 routing and S2 permutation kernels.
//
// Routing: one warp per token; softmax -> top-k -> renormalise, i.e. the
// "Renormalize" routing method of the TRTLLM MXFP4 experts page.
// Permutation: expert-contiguous segments over E experts + B redundant slots as
// in the MoonEP experts page (cu_seqlens = inclusive running sum of segment
// lengths; segments ordered by ascending token id). The order inside a segment
// is decided without atomics: each 256-token block records, per expert, a
// 256-bit mask of the tokens that chose it, and a token's rank is a popcount.
#include "internal.h"

namespace moe {

// ----------------------------------------------------------------- S1 route
// Token t's top-k by one warp (all 32 lanes): ids and renormalised weights, in selection order.
template <int EPL>  // logits per lane (E <= 32*EPL)
__device__ __forceinline__ void route_token(const float* __restrict__ logits, int t, int E, int topk,
                                            int32_t* __restrict__ ids, float* __restrict__ w) {
    const int lane = lane_id();
    {
        float v[EPL];
        const float* row = logits + (size_t)t * E;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = i * 32 + lane;
            v[i] = e < E ? row[e] : 0.0f;
        }
        uint32_t taken = 0;  // bit i: entry i of this lane is selected or absent
#pragma unroll
        for (int i = 0; i < EPL; ++i)
            if (i * 32 + lane >= E) taken |= 1u << i;
        float my_v = 0.0f;
        int my_id = 0;
        for (int j = 0; j < topk; ++j) {
            // lane-local best: larger value, then lower id (lower i is lower id)
            float bv = 0.0f;
            int bid = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                if (!(taken >> i & 1u)) {
                    if (bid == 0x7fffffff || v[i] > bv) {
                        bv = v[i];
                        bid = i * 32 + lane;
                    }
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
                const int oid = __shfl_xor_sync(0xffffffffu, bid, off);
                const bool other_better =
                    oid != 0x7fffffff && (bid == 0x7fffffff || ov > bv || (ov == bv && oid < bid));
                if (other_better) {
                    bv = ov;
                    bid = oid;
                }
            }
            if ((bid & 31) == lane) taken |= 1u << (bid >> 5);
            if (lane == j) {
                my_v = bv;
                my_id = bid;
            }
        }
        const float v0 = __shfl_sync(0xffffffffu, my_v, 0);
        float z = lane < topk ? expf(my_v - v0) : 0.0f;
        float sum = z;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane < topk) {
            ids[(size_t)t * topk + lane] = my_id;
            w[(size_t)t * topk + lane] = z / sum;
        }
    }
}

template <int EPL>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits, int T,
                                                         int E, int topk,
                                                         int32_t* __restrict__ ids,
                                                         float* __restrict__ w) {
    pdl_wait();
    const int t = blockIdx.x * (blockDim.x >> 5) + warp_id();
    if (t < T) route_token<EPL>(logits, t, E, topk, ids, w);
    pdl_launch();
}

cudaError_t launch_route_topk(const float* logits, int T, int E, int topk, int32_t* ids, float* w,
                              cudaStream_t st, bool pdl) {
    const int warps = 8;
    dim3 grid((T + warps - 1) / warps), block(32 * warps);
    const int epl = (E + 31) / 32;
    if (epl <= 1) return launch_k(route_topk_kernel<1>, grid, block, 0, st, pdl, logits, T, E, topk, ids, w);
    if (epl <= 2) return launch_k(route_topk_kernel<2>, grid, block, 0, st, pdl, logits, T, E, topk, ids, w);
    if (epl <= 4) return launch_k(route_topk_kernel<4>, grid, block, 0, st, pdl, logits, T, E, topk, ids, w);
    if (epl <= 8) return launch_k(route_topk_kernel<8>, grid, block, 0, st, pdl, logits, T, E, topk, ids, w);
    if (epl <= 16) return launch_k(route_topk_kernel<16>, grid, block, 0, st, pdl, logits, T, E, topk, ids, w);
    return launch_k(route_topk_kernel<32>, grid, block, 0, st, pdl, logits, T, E, topk, ids, w);
}

// ----------------------------------------------------------------- S1 route, DeepSeekV3
// Grouped top-k on sigmoid scores (the "DeepSeekV3" routing method of the TRTLLM MXFP4
// page): s = sigmoid(l), c = s + bias; groups of E/n_group consecutive experts score the
// sum of their two largest c; the topk_group best groups are kept (ties to the lower
// group); the topk largest c among their experts are chosen (ties to the lower id), and
// w = scale * s / sum of the chosen s. One warp per token; every decision in fp64.
template <int EPL>  // experts per lane (E <= 32*EPL)
__global__ void __launch_bounds__(256) route_grouped_kernel(const float* __restrict__ logits,
                                                            const float* __restrict__ bias, int T, int E,
                                                            int topk, int n_group, int topk_group, float scale,
                                                            int32_t* __restrict__ ids, float* __restrict__ w) {
    constexpr int NONE = 0x7fffffff;
    pdl_wait();
    const int lane = lane_id();
    const int t = blockIdx.x * (blockDim.x >> 5) + warp_id();
    if (t < T) {
        const int gs = E / n_group;
        const double ninf = -(double)INFINITY;
        double sc[EPL], c[EPL];
        const float* row = logits + (size_t)t * E;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = i * 32 + lane;
            sc[i] = 0.0;
            c[i] = ninf;
            if (e < E) {
                sc[i] = 1.0 / (1.0 + exp(-(double)row[e]));
                c[i] = sc[i] + (bias ? (double)bias[e] : 0.0);
            }
        }
        // group scores: each group's two largest c, merged across the warp; lane g keeps group g's
        double my_gs = ninf;
        for (int g = 0; g < n_group; ++g) {
            double a1 = ninf, a2 = ninf;
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                const int e = i * 32 + lane;
                if (e < E && e / gs == g) {
                    if (c[i] > a1) {
                        a2 = a1;
                        a1 = c[i];
                    } else if (c[i] > a2) {
                        a2 = c[i];
                    }
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const double b1 = __shfl_xor_sync(0xffffffffu, a1, off);
                const double b2 = __shfl_xor_sync(0xffffffffu, a2, off);
                const double n2 = fmax(fmin(a1, b1), fmax(a2, b2));
                a1 = fmax(a1, b1);
                a2 = n2;
            }
            if (lane == g) my_gs = a1 + (gs >= 2 ? a2 : 0.0);
        }
        // the topk_group best groups
        uint32_t keep = 0;
        for (int j = 0; j < topk_group; ++j) {
            double bv = my_gs;
            int bg = (lane < n_group && !(keep >> lane & 1u)) ? lane : NONE;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const double ov = __shfl_xor_sync(0xffffffffu, bv, off);
                const int og = __shfl_xor_sync(0xffffffffu, bg, off);
                if (og != NONE && (bg == NONE || ov > bv || (ov == bv && og < bg))) {
                    bv = ov;
                    bg = og;
                }
            }
            keep |= 1u << bg;  // bg is valid: topk_group <= n_group
        }
        // the topk best experts of the kept groups
        uint32_t taken = 0;  // bit i: entry i of this lane is chosen, absent or outside the kept groups
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = i * 32 + lane;
            if (e >= E || !(keep >> (e / gs) & 1u)) taken |= 1u << i;
        }
        double my_s = 0.0;
        int my_id = 0;
        for (int j = 0; j < topk; ++j) {
            double bv = 0.0, bs = 0.0;
            int bid = NONE;
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                if (!(taken >> i & 1u) && (bid == NONE || c[i] > bv)) {
                    bv = c[i];
                    bs = sc[i];
                    bid = i * 32 + lane;
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const double ov = __shfl_xor_sync(0xffffffffu, bv, off);
                const double os = __shfl_xor_sync(0xffffffffu, bs, off);
                const int oid = __shfl_xor_sync(0xffffffffu, bid, off);
                if (oid != NONE && (bid == NONE || ov > bv || (ov == bv && oid < bid))) {
                    bv = ov;
                    bs = os;
                    bid = oid;
                }
            }
            if (bid != NONE && (bid & 31) == lane) taken |= 1u << (bid >> 5);
            if (lane == j) {
                my_s = bs;
                my_id = bid;
            }
        }
        double sum = lane < topk ? my_s : 0.0;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane < topk) {
            ids[(size_t)t * topk + lane] = my_id;
            w[(size_t)t * topk + lane] = (float)((double)scale * my_s / sum);
        }
    }
    pdl_launch();
}

cudaError_t launch_route_grouped(const float* logits, const float* bias, int T, int E, int topk, int n_group,
                                 int topk_group, float scale, int32_t* ids, float* w, cudaStream_t st, bool pdl) {
    const int warps = 8;
    dim3 grid((T + warps - 1) / warps), block(32 * warps);
    const int epl = (E + 31) / 32;
#define MOE_ROUTE_G(N)                                                                                            \
    return launch_k(route_grouped_kernel<N>, grid, block, 0, st, pdl, logits, bias, T, E, topk, n_group, topk_group, \
                    scale, ids, w)
    if (epl <= 1) MOE_ROUTE_G(1);
    if (epl <= 2) MOE_ROUTE_G(2);
    if (epl <= 4) MOE_ROUTE_G(4);
    if (epl <= 8) MOE_ROUTE_G(8);
    MOE_ROUTE_G(16);
#undef MOE_ROUTE_G
}

// ----------------------------------------------------------------- S2 permute
// Token blocks of 256: thread i of block b owns token b*256+i.
constexpr int kPermBlock = 256;

PermuteWs permute_ws_layout(int T, int topk, int E, int B) {
    PermuteWs L;
    const int nblk = (T + kPermBlock - 1) / kPermBlock;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += (bytes + 255) & ~size_t(255);
        return o;
    };
    L.nblk = nblk;
    L.blkcnt = take(sizeof(int) * (size_t)std::max(nblk, 1) * E);
    L.blkoff = take(sizeof(int) * (size_t)std::max(nblk, 1) * E);
    L.total = take(sizeof(int) * E);
    L.nrep = take(sizeof(int) * E);
    L.rep_ptr = take(sizeof(int) * (E + 1));
    L.rep_rows = take(sizeof(int) * (E + B));
    L.rowstart = take(sizeof(int) * (E + B));
    L.bytes = off;
    (void)topk;
    return L;
}

// Builds the block's per-expert token masks; returns false if an id was out of range.
__device__ void build_masks(uint32_t* masks, const int32_t* __restrict__ ids, int T, int topk,
                            int E, int t0, DevError* err) {
    for (int i = threadIdx.x; i < E * (kPermBlock / 32); i += blockDim.x) masks[i] = 0u;
    __syncthreads();
    const int t = t0 + threadIdx.x;
    if (threadIdx.x < kPermBlock && t < T) {
        for (int j = 0; j < topk; ++j) {
            const int e = ids[(size_t)t * topk + j];
            if (e < 0 || e >= E) {
                report_error(err, MOE_ERR_DEVICE, t);
                continue;
            }
            // a token listing one expert twice (possible only with a given top-k) is refused
            const uint32_t bit = 1u << (threadIdx.x & 31);
            if (atomicOr(&masks[e * (kPermBlock / 32) + (threadIdx.x >> 5)], bit) & bit)
                report_error(err, MOE_ERR_DEVICE, t);
        }
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kPermBlock) permute_count_kernel(const int32_t* __restrict__ ids,
                                                                   int T, int topk, int E,
                                                                   int* __restrict__ blkcnt,
                                                                   DevError* err) {
    extern __shared__ uint32_t masks[];
    pdl_wait();
    build_masks(masks, ids, T, topk, E, blockIdx.x * kPermBlock, err);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int c = 0;
#pragma unroll
        for (int q = 0; q < kPermBlock / 32; ++q) c += __popc(masks[e * (kPermBlock / 32) + q]);
        blkcnt[(size_t)blockIdx.x * E + e] = c;
    }
    pdl_launch();
}

// One block: per-expert running sums over token blocks, the replica split and the
// inclusive scan of segment lengths over the G = E + B weight rows. Rows from the last
// segment end up to NvS receive no assignment unless an id was bad (out of range, or an
// expert listed twice by one token; both reported): they get token 0 and weight 0, so that
// a gather over all NvS rows reads only rows of x.
// The scan's work for one block of 1024 threads; sm holds [G] segment sizes, then [1024]
// scan scratch.
__device__ void permute_scan_body(
    int* sm, const int* __restrict__ blkcnt, int nblk, int E, int B, const int32_t* __restrict__ replica_src,
    int* __restrict__ blkoff, int* __restrict__ total, int* __restrict__ nrep,
    int* __restrict__ rep_ptr, int* __restrict__ rep_rows, int* __restrict__ rowstart,
    int32_t* __restrict__ cu_seqlens, int NvS, int32_t* __restrict__ perm_token, float* __restrict__ perm_w,
    DevError* err) {
    const int G = E + B;
    int* seg = sm;
    int* scratch = sm + G;
    // per-expert totals and block offsets; replica counts
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int b = 0; b < nblk; ++b) {
            blkoff[(size_t)b * E + e] = run;
            run += blkcnt[(size_t)b * E + e];
        }
        total[e] = run;
        int m = 1;
        for (int s = 0; s < B; ++s) m += (replica_src[s] == e);
        nrep[e] = m;
    }
    for (int s = threadIdx.x; s < B; s += blockDim.x) {
        const int src = replica_src[s];
        if (src < -1 || src >= E) report_error(err, MOE_ERR_DEVICE, -1 - s);
    }
    __syncthreads();
    // exclusive scan of nrep over experts -> rep_ptr (serial chunks + block scan)
    auto block_exclusive_scan = [&](const int* in, int n, int* out_excl) -> int {
        // each thread owns a contiguous chunk
        const int per = (n + blockDim.x - 1) / blockDim.x;
        const int lo = min(n, (int)threadIdx.x * per), hi = min(n, lo + per);
        int local = 0;
        for (int i = lo; i < hi; ++i) local += in[i];
        scratch[threadIdx.x] = local;
        __syncthreads();
        for (int d = 1; d < (int)blockDim.x; d <<= 1) {
            const int add = threadIdx.x >= (unsigned)d ? scratch[threadIdx.x - d] : 0;
            __syncthreads();
            scratch[threadIdx.x] += add;
            __syncthreads();
        }
        int run = scratch[threadIdx.x] - local;
        for (int i = lo; i < hi; ++i) {
            out_excl[i] = run;
            run += in[i];
        }
        const int tot = scratch[blockDim.x - 1];
        __syncthreads();
        return tot;
    };
    const int nrows = block_exclusive_scan(nrep, E, rep_ptr);
    if (threadIdx.x == 0) rep_ptr[E] = nrows;
    __syncthreads();
    // rows of each expert, and segment sizes
    for (int g = threadIdx.x; g < G; g += blockDim.x) seg[g] = 0;
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int m = nrep[e], n = total[e], base = rep_ptr[e];
        const int q = n / m, r = n % m;
        int i = 0;
        rep_rows[base + i] = e;
        seg[e] = q + (i < r ? 1 : 0);
        ++i;
        for (int s = 0; s < B; ++s) {
            if (replica_src[s] == e) {
                rep_rows[base + i] = E + s;
                seg[E + s] = q + (i < r ? 1 : 0);
                ++i;
            }
        }
    }
    __syncthreads();
    const int filled = block_exclusive_scan(seg, G, rowstart);
    for (int g = threadIdx.x; g < G; g += blockDim.x) cu_seqlens[g] = rowstart[g] + seg[g];
    for (int r = filled + threadIdx.x; r < NvS; r += blockDim.x) {
        perm_token[r] = 0;
        perm_w[r] = 0.0f;
    }
}

__global__ void __launch_bounds__(1024) permute_scan_kernel(
    const int* __restrict__ blkcnt, int nblk, int E, int B, const int32_t* __restrict__ replica_src,
    int* __restrict__ blkoff, int* __restrict__ total, int* __restrict__ nrep,
    int* __restrict__ rep_ptr, int* __restrict__ rep_rows, int* __restrict__ rowstart,
    int32_t* __restrict__ cu_seqlens, int NvS, int32_t* __restrict__ perm_token, float* __restrict__ perm_w,
    DevError* err) {
    extern __shared__ int sm[];  // [G] segment sizes, then [1024] scan scratch
    pdl_wait();
    permute_scan_body(sm, blkcnt, nblk, E, B, replica_src, blkoff, total, nrep, rep_ptr, rep_rows, rowstart,
                      cu_seqlens, NvS, perm_token, perm_w, err);
    pdl_launch();
}

// Token block `blk`'s assignments to their rows, from the block's masks (threads 0..255
// own the block's tokens).
__device__ void permute_scatter_body(
    const uint32_t* masks, int blk, const int32_t* __restrict__ ids, const float* __restrict__ topk_w, int T,
    int topk, int E, const int* __restrict__ blkoff, const int* __restrict__ total, const int* __restrict__ nrep,
    const int* __restrict__ rep_ptr, const int* __restrict__ rep_rows, const int* __restrict__ rowstart,
    int32_t* __restrict__ perm_token, float* __restrict__ perm_w, int32_t* __restrict__ inv_perm) {
    const int t = blk * kPermBlock + threadIdx.x;
    if (threadIdx.x < kPermBlock && t < T) {
        const int word = threadIdx.x >> 5;
        const uint32_t below = (1u << (threadIdx.x & 31)) - 1u;
        for (int j = 0; j < topk; ++j) {
            const int e = ids[(size_t)t * topk + j];
            if (e < 0 || e >= E) {
                inv_perm[(size_t)t * topk + j] = -1;
                continue;
            }
            const uint32_t* m = masks + e * (kPermBlock / 32);
            int rank = __popc(m[word] & below);
            for (int q = 0; q < word; ++q) rank += __popc(m[q]);
            const int r = blkoff[(size_t)blk * E + e] + rank;
            const int n = total[e], R = nrep[e];
            const int q = n / R, rem = n % R, big = rem * (q + 1);
            int chunk, pos;
            if (r < big) {
                chunk = r / (q + 1);
                pos = r - chunk * (q + 1);
            } else {
                chunk = rem + (r - big) / q;
                pos = (r - big) - (chunk - rem) * q;
            }
            const int row = rep_rows[rep_ptr[e] + chunk];
            const int dst = rowstart[row] + pos;
            perm_token[dst] = t;
            perm_w[dst] = topk_w ? topk_w[(size_t)t * topk + j] : 1.0f;
            inv_perm[(size_t)t * topk + j] = dst;
        }
    }
}

__global__ void __launch_bounds__(kPermBlock) permute_scatter_kernel(
    const int32_t* __restrict__ ids, const float* __restrict__ topk_w, int T, int topk, int E,
    const int* __restrict__ blkoff, const int* __restrict__ total, const int* __restrict__ nrep,
    const int* __restrict__ rep_ptr, const int* __restrict__ rep_rows,
    const int* __restrict__ rowstart, int32_t* __restrict__ perm_token, float* __restrict__ perm_w,
    int32_t* __restrict__ inv_perm) {
    extern __shared__ uint32_t masks[];
    pdl_wait();
    build_masks(masks, ids, T, topk, E, blockIdx.x * kPermBlock, nullptr);
    permute_scatter_body(masks, blockIdx.x, ids, topk_w, T, topk, E, blkoff, total, nrep, rep_ptr, rep_rows,
                         rowstart, perm_token, perm_w, inv_perm);
    pdl_launch();
}

__device__ void permute_one_block_body(
    uint32_t* smem_u, const int32_t* __restrict__ ids, const float* __restrict__ topk_w, int T, int topk, int E,
    int B, const int32_t* __restrict__ replica_src, int* __restrict__ blkcnt, int* __restrict__ blkoff,
    int* __restrict__ total, int* __restrict__ nrep, int* __restrict__ rep_ptr, int* __restrict__ rep_rows,
    int* __restrict__ rowstart, int32_t* __restrict__ cu_seqlens, int32_t* __restrict__ perm_token,
    float* __restrict__ perm_w, int32_t* __restrict__ inv_perm, DevError* err);

// At most one token block: the count, the scan and the scatter in one CTA of 1024 threads
// (three launches fewer for decode batches). Shared memory: the block's masks [E * 8], then
// the scan's [G + 1024].
__global__ void __launch_bounds__(1024) permute_one_block_kernel(
    const int32_t* __restrict__ ids, const float* __restrict__ topk_w, int T, int topk, int E, int B,
    const int32_t* __restrict__ replica_src, int* __restrict__ blkcnt, int* __restrict__ blkoff,
    int* __restrict__ total, int* __restrict__ nrep, int* __restrict__ rep_ptr, int* __restrict__ rep_rows,
    int* __restrict__ rowstart, int32_t* __restrict__ cu_seqlens, int32_t* __restrict__ perm_token,
    float* __restrict__ perm_w, int32_t* __restrict__ inv_perm, DevError* err) {
    extern __shared__ uint32_t smem_u[];
    pdl_wait();
    permute_one_block_body(smem_u, ids, topk_w, T, topk, E, B, replica_src, blkcnt, blkoff, total, nrep, rep_ptr,
                           rep_rows, rowstart, cu_seqlens, perm_token, perm_w, inv_perm, err);
    pdl_launch();
}

// Softmax -> top-k -> renormalise for at most 256 tokens (32 warps) and their permutation,
// one CTA: two launches fewer than the routing plus the permutation for decode batches.
template <int EPL>
__global__ void __launch_bounds__(1024) route_permute_one_block_kernel(
    const float* __restrict__ logits, int T, int E, int topk, int32_t* __restrict__ ids, float* __restrict__ topk_w,
    int B, const int32_t* __restrict__ replica_src, int* __restrict__ blkcnt, int* __restrict__ blkoff,
    int* __restrict__ total, int* __restrict__ nrep, int* __restrict__ rep_ptr, int* __restrict__ rep_rows,
    int* __restrict__ rowstart, int32_t* __restrict__ cu_seqlens, int32_t* __restrict__ perm_token,
    float* __restrict__ perm_w, int32_t* __restrict__ inv_perm, DevError* err) {
    extern __shared__ uint32_t smem_u[];
    pdl_wait();
    for (int t = warp_id(); t < T; t += blockDim.x >> 5) route_token<EPL>(logits, t, E, topk, ids, topk_w);
    __syncthreads();
    permute_one_block_body(smem_u, ids, topk_w, T, topk, E, B, replica_src, blkcnt, blkoff, total, nrep, rep_ptr,
                           rep_rows, rowstart, cu_seqlens, perm_token, perm_w, inv_perm, err);
    pdl_launch();
}

__device__ void permute_one_block_body(
    uint32_t* smem_u, const int32_t* __restrict__ ids, const float* __restrict__ topk_w, int T, int topk, int E,
    int B, const int32_t* __restrict__ replica_src, int* __restrict__ blkcnt, int* __restrict__ blkoff,
    int* __restrict__ total, int* __restrict__ nrep, int* __restrict__ rep_ptr, int* __restrict__ rep_rows,
    int* __restrict__ rowstart, int32_t* __restrict__ cu_seqlens, int32_t* __restrict__ perm_token,
    float* __restrict__ perm_w, int32_t* __restrict__ inv_perm, DevError* err) {
    uint32_t* masks = smem_u;
    int* sm = reinterpret_cast<int*>(smem_u + (size_t)E * (kPermBlock / 32));
    build_masks(masks, ids, T, topk, E, 0, err);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int c = 0;
#pragma unroll
        for (int q = 0; q < kPermBlock / 32; ++q) c += __popc(masks[e * (kPermBlock / 32) + q]);
        blkcnt[e] = c;
    }
    __syncthreads();
    permute_scan_body(sm, blkcnt, 1, E, B, replica_src, blkoff, total, nrep, rep_ptr, rep_rows, rowstart,
                      cu_seqlens, T * topk, perm_token, perm_w, err);
    __syncthreads();
    permute_scatter_body(masks, 0, ids, topk_w, T, topk, E, blkoff, total, nrep, rep_ptr, rep_rows, rowstart,
                         perm_token, perm_w, inv_perm);
}

cudaError_t launch_permute(const int32_t* ids, const float* topk_w, int T, int topk, int E, int B,
                           const int32_t* replica_src, int32_t* cu_seqlens, int32_t* perm_token,
                           float* perm_w, int32_t* inv_perm, DevError* err, char* ws, cudaStream_t st,
                           bool pdl) {
    const PermuteWs L = permute_ws_layout(T, topk, E, B);
    int* blkcnt = reinterpret_cast<int*>(ws + L.blkcnt);
    int* blkoff = reinterpret_cast<int*>(ws + L.blkoff);
    int* total = reinterpret_cast<int*>(ws + L.total);
    int* nrep = reinterpret_cast<int*>(ws + L.nrep);
    int* rep_ptr = reinterpret_cast<int*>(ws + L.rep_ptr);
    int* rep_rows = reinterpret_cast<int*>(ws + L.rep_rows);
    int* rowstart = reinterpret_cast<int*>(ws + L.rowstart);
    const size_t mask_smem = sizeof(uint32_t) * E * (kPermBlock / 32);
    cudaError_t e;
    if (L.nblk == 1) {
        const size_t smem = mask_smem + sizeof(int) * (E + B + 1024);
        if (smem > 48 * 1024) {
            static int done[64] = {0};
            int dev = 0;
            e = cudaGetDevice(&dev);
            if (e != cudaSuccess) return e;
            if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
            if (!done[dev]) {
                e = cudaFuncSetAttribute(permute_one_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
                if (e != cudaSuccess) return e;
                done[dev] = 1;
            }
        }
        return launch_k(permute_one_block_kernel, dim3(1), dim3(1024), smem, st, pdl, ids, topk_w, T, topk, E, B,
                        replica_src, blkcnt, blkoff, total, nrep, rep_ptr, rep_rows, rowstart, cu_seqlens,
                        perm_token, perm_w, inv_perm, err);
    }
    if (L.nblk > 0) {
        e = launch_k(permute_count_kernel, dim3(L.nblk), dim3(kPermBlock), mask_smem, st, pdl, ids, T,
                     topk, E, blkcnt, err);
        if (e != cudaSuccess) return e;
    }
    const size_t scan_smem = sizeof(int) * (E + B + 1024);
    // the scan and scatter follow this function's own kernels: they always overlap with them
    e = launch_k(permute_scan_kernel, dim3(1), dim3(1024), scan_smem, st, L.nblk > 0 ? true : pdl,
                 (const int*)blkcnt, L.nblk, E, B, replica_src, blkoff, total, nrep, rep_ptr, rep_rows,
                 rowstart, cu_seqlens, T * topk, perm_token, perm_w, err);
    if (e != cudaSuccess) return e;
    if (L.nblk > 0) {
        e = launch_k(permute_scatter_kernel, dim3(L.nblk), dim3(kPermBlock), mask_smem, st, true, ids,
                     topk_w, T, topk, E, (const int*)blkoff, (const int*)total, (const int*)nrep,
                     (const int*)rep_ptr, (const int*)rep_rows, (const int*)rowstart, perm_token,
                     perm_w, inv_perm);
    }
    return e;
}

cudaError_t launch_route_permute_one_block(const float* logits, int T, int E, int topk, int32_t* ids, float* w,
                                          int B, const int32_t* replica_src, int32_t* cu_seqlens,
                                          int32_t* perm_token, float* perm_w, int32_t* inv_perm, DevError* err,
                                          char* ws, cudaStream_t st, bool pdl) {
    if (T < 1 || T > kPermBlock) return cudaErrorInvalidValue;
    const PermuteWs L = permute_ws_layout(T, topk, E, B);
    int* blkcnt = reinterpret_cast<int*>(ws + L.blkcnt);
    int* blkoff = reinterpret_cast<int*>(ws + L.blkoff);
    int* total = reinterpret_cast<int*>(ws + L.total);
    int* nrep = reinterpret_cast<int*>(ws + L.nrep);
    int* rep_ptr = reinterpret_cast<int*>(ws + L.rep_ptr);
    int* rep_rows = reinterpret_cast<int*>(ws + L.rep_rows);
    int* rowstart = reinterpret_cast<int*>(ws + L.rowstart);
    const size_t smem = sizeof(uint32_t) * E * (kPermBlock / 32) + sizeof(int) * (E + B + 1024);
    const int epl = (E + 31) / 32;
    cudaError_t e = cudaSuccess;
#define MOE_RP(N)                                                                                                  \
    {                                                                                                              \
        auto k = route_permute_one_block_kernel<N>;                                                                \
        if (smem > 48 * 1024) {                                                                                    \
            static int done[64] = {0};                                                                             \
            int dev = 0;                                                                                           \
            if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;                                                \
            if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;                                               \
            if (!done[dev]) {                                                                                      \
                if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=       \
                    cudaSuccess)                                                                                   \
                    return e;                                                                                      \
                done[dev] = 1;                                                                                     \
            }                                                                                                      \
        }                                                                                                          \
        return launch_k(k, dim3(1), dim3(1024), smem, st, pdl, logits, T, E, topk, ids, w, B, replica_src, blkcnt, \
                        blkoff, total, nrep, rep_ptr, rep_rows, rowstart, cu_seqlens, perm_token, perm_w, inv_perm, \
                        err);                                                                                      \
    }
    if (epl <= 1) MOE_RP(1);
    if (epl <= 2) MOE_RP(2);
    if (epl <= 4) MOE_RP(4);
    if (epl <= 8) MOE_RP(8);
    if (epl <= 16) MOE_RP(16);
    MOE_RP(32);
#undef MOE_RP
}

// ----------------------------------------------------------------- row gathers
// dst[r] = src[perm_token[r]] for r < NvS, one warp per row, 16-byte vectors.
// mode 0: bf16 -> bf16 copy. mode 1: f16 -> f16 copy plus a per-row scale copy
// (src_scale[token] -> dst_scale[r]). mode 2: bf16 -> f16 times 2^-e, e chosen
// from the row's max so that the max lands in [2^14, 2^15); dst_scale[r] = 2^e.
__device__ __forceinline__ float pow2_row_shift(float amax, float* inv_scale) {
    if (!(amax > 0.0f)) {
        *inv_scale = 1.0f;
        return 1.0f;
    }
    int ex;
    frexpf(amax, &ex);  // amax = m * 2^ex, m in [0.5, 1)
    const int sh = max(-126, min(127, ex - 15));
    *inv_scale = ldexpf(1.0f, -sh);
    return ldexpf(1.0f, sh);
}

template <int MODE>
__global__ void __launch_bounds__(256) gather_rows_kernel(const void* __restrict__ src, int H,
                                                          const int32_t* __restrict__ perm_token,
                                                          int NvS, void* __restrict__ dst,
                                                          const float* __restrict__ src_scale,
                                                          float* __restrict__ dst_scale) {
    pdl_wait();
    const int r = blockIdx.x * 8 + warp_id();
    const int lane = lane_id();
    if (r < NvS) {
        const int t = perm_token[r];
        const uint4* s = reinterpret_cast<const uint4*>(src) + (size_t)t * (H / 8);
        uint4* d = reinterpret_cast<uint4*>(dst) + (size_t)r * (H / 8);
        const int nv = H / 8;
        if (MODE == 0 || MODE == 1) {
            for (int i = lane; i < nv; i += 32) d[i] = __ldg(s + i);
            if (MODE == 1 && lane == 0) dst_scale[r] = src_scale[t];
        } else {
            float amax = 0.0f;
            for (int i = lane; i < nv; i += 32) {
                uint4 v = __ldg(s + i);
                const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 f = __bfloat1622float2(p[q]);
                    amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
            float inv;
            const float sc = pow2_row_shift(amax, &inv);
            for (int i = lane; i < nv; i += 32) {
                uint4 v = __ldg(s + i);
                const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
                uint4 o;
                __half2* po = reinterpret_cast<__half2*>(&o);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 f = __bfloat1622float2(p[q]);
                    po[q] = __floats2half2_rn(f.x * inv, f.y * inv);
                }
                d[i] = o;
            }
            if (lane == 0) dst_scale[r] = sc;
        }
    }
    pdl_launch();
}

cudaError_t launch_gather(int mode, const void* src, int H, const int32_t* perm_token, int NvS,
                          void* dst, const float* src_scale, float* dst_scale, cudaStream_t st,
                          bool pdl) {
    if (NvS <= 0) return cudaSuccess;
    dim3 grid((NvS + 7) / 8), block(256);
    if (mode == 0)
        return launch_k(gather_rows_kernel<0>, grid, block, 0, st, pdl, src, H, perm_token, NvS, dst,
                        src_scale, dst_scale);
    if (mode == 1)
        return launch_k(gather_rows_kernel<1>, grid, block, 0, st, pdl, src, H, perm_token, NvS, dst,
                        src_scale, dst_scale);
    return launch_k(gather_rows_kernel<2>, grid, block, 0, st, pdl, src, H, perm_token, NvS, dst,
                    src_scale, dst_scale);
}

// Row-wise conversion (no gather): rows of fp32 or bf16 [R,K] -> f16 times 2^-e
// with the per-row scale 2^e, as in gather mode 2.
template <bool IN_F32>
__global__ void __launch_bounds__(256) rows_to_f16_pow2_kernel(const void* __restrict__ src, int R,
                                                               int K, __half* __restrict__ dst,
                                                               float* __restrict__ scale) {
    pdl_wait();
    const int r = blockIdx.x * 8 + warp_id();
    const int lane = lane_id();
    if (r < R) {
        float amax = 0.0f;
        if (IN_F32) {
            const float4* s = reinterpret_cast<const float4*>(src) + (size_t)r * (K / 4);
            for (int i = lane; i < K / 4; i += 32) {
                const float4 v = s[i];
                amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
            }
        } else {
            const __nv_bfloat162* s = reinterpret_cast<const __nv_bfloat162*>(src) + (size_t)r * (K / 2);
            for (int i = lane; i < K / 2; i += 32) {
                const float2 f = __bfloat1622float2(s[i]);
                amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        float inv;
        const float sc = pow2_row_shift(amax, &inv);
        __half2* d = reinterpret_cast<__half2*>(dst) + (size_t)r * (K / 2);
        if (IN_F32) {
            const float2* s = reinterpret_cast<const float2*>(src) + (size_t)r * (K / 2);
            for (int i = lane; i < K / 2; i += 32) {
                const float2 f = s[i];
                d[i] = __floats2half2_rn(f.x * inv, f.y * inv);
            }
        } else {
            const __nv_bfloat162* s = reinterpret_cast<const __nv_bfloat162*>(src) + (size_t)r * (K / 2);
            for (int i = lane; i < K / 2; i += 32) {
                const float2 f = __bfloat1622float2(s[i]);
                d[i] = __floats2half2_rn(f.x * inv, f.y * inv);
            }
        }
        if (lane == 0) scale[r] = sc;
    }
    pdl_launch();
}

cudaError_t launch_rows_to_f16(const void* src, bool in_f32, int R, int K, __half* dst, float* scale,
                               cudaStream_t st, bool pdl) {
    if (R <= 0) return cudaSuccess;
    dim3 grid((R + 7) / 8), block(256);
    if (in_f32) return launch_k(rows_to_f16_pow2_kernel<true>, grid, block, 0, st, pdl, src, R, K, dst, scale);
    return launch_k(rows_to_f16_pow2_kernel<false>, grid, block, 0, st, pdl, src, R, K, dst, scale);
}

}  // namespace moe
