// S3/S4/S5 — persistent grouped GEMM on the 5th-generation tensor cores.
//
// Computes out[seg_g] = alpha_g * x[seg_g] @ W[g]^T over the expert-contiguous
// segments of cu_seqlens (MoonEP experts page, moonep_grouped_gemm), optionally
// as the fused gate+up pair with the gated activation and route weight in the
// epilogue (MoonEP experts page, module docstring: act = silu(gate)*up*route_w;
// SITU from the TRTLLM MXFP4 page).
//
// Tiling ("swap AB"): one tile is 128 weight rows (the MMA M side) by BT token
// rows (the MMA N side, 16..128) of one segment. Decode segments hold a handful
// of tokens, so the token side is the narrow one; the weights stream through
// at full width. Each CTA owns one SM and walks the tile list
// (segment, weight block, token block) with the token block fastest, so the
// CTAs working on one weight block at the same time share it through L2.
//
// Warp roles (one CTA per SM):
//   warp 0       producer (one thread): TMA / bulk copies per K step
//   warp 1       MMA issuer (one thread) + TMEM owner; accumulators double-buffered
//   warps 2..5   epilogue: TMEM -> registers -> alpha / activation / scales -> global
//   warps 6..13  (FP4 weights only) e2m1 -> f16 converters writing the swizzled
//                operand the MMA reads (FP4 dequant fused into the mainloop)
// Pipelines:
//   BF16 weights: one ring of stages {gate tile, [up tile], token tile}.
//   FP4 weights: a deep ring of small raw stages {token tile, packed e2m1 codes,
//   block scales} that keeps enough bytes in flight to stream HBM, feeding a
//   shallow ring of converted f16 weight tiles. The MMA reads weights from the
//   converted ring and tokens straight from the raw stage.
// Every wait is bounded; a timeout records MOE_ERR_TIMEOUT in the error word,
// stops all roles, lets copies in flight land, frees TMEM and returns.
#include <mutex>

#include "internal.h"

namespace moe {

constexpr int kMaxG = 1024;      // segment table capacity (weight rows)
constexpr int kMaxStages = 16;

__host__ __device__ constexpr int round1024(int b) { return (b + 1023) & ~1023; }
__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }

template <int BT, bool DUAL, int WFMT>
struct GemmCfg {
    static constexpr bool FP4 = WFMT != MOE_W_BF16;
    static constexpr int NB = DUAL ? 2 : 1;
    static constexpr int A_BYTES = kTileN * kTileK * 2;      // 16 KB: 128 rows x 64 x 16-bit
    static constexpr int B_BYTES = BT * kTileK * 2;          // BT rows x 64 x 16-bit
    static constexpr int RAW_D = kTileN * kTileK / 2;        // 4 KB of packed e2m1
    static constexpr int RAW_S = WFMT == MOE_W_MXFP4 ? kTileN * 2 : (WFMT == MOE_W_NVFP4 ? kTileN * 4 : 0);
    // operand stage: weights (+ tokens for BF16); raw stage (FP4): tokens, codes, scales
    static constexpr int OP_STAGE = NB * A_BYTES + (FP4 ? 0 : B_BYTES);
    static constexpr int RAW_STAGE = FP4 ? round1024(B_BYTES + NB * (RAW_D + RAW_S)) : 0;
    static constexpr int CTRL_BYTES = 12288;
    static constexpr int SMEM_LIMIT = 232448;
    static constexpr int BUDGET = SMEM_LIMIT - 1024 - CTRL_BYTES;
    static constexpr int STAGES = FP4 ? (BT >= 64 ? 4 : 3) : cmin(kMaxStages, BUDGET / OP_STAGE);
    static constexpr int RSTAGES = FP4 ? cmin(kMaxStages, (BUDGET - STAGES * OP_STAGE) / RAW_STAGE) : 0;
    static constexpr int TMEM_USED = 2 * NB * BT;
    static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 : TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
    static constexpr int CONV_WARPS = FP4 ? 8 : 0;
    static constexpr int CONV_THREADS = CONV_WARPS * 32;
    static constexpr int THREADS = (6 + CONV_WARPS) * 32;
    static constexpr int SMEM_BYTES = 1024 + STAGES * OP_STAGE + RSTAGES * RAW_STAGE + CTRL_BYTES;
    static_assert(STAGES >= 2 && (!FP4 || RSTAGES >= 2), "pipeline needs two stages");
    static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory");
    static_assert(TMEM_USED <= 512, "accumulators exceed TMEM");
    static_assert(BT % 16 == 0 && BT >= 16 && BT <= 256, "MMA N for M=128 is a multiple of 16 in [16,256]");
};

struct GemmArgs {
    const int32_t* cu;
    int G, N, K, KB, NT, M_alloc;
    void* out;
    const float* alpha0;
    const float* alpha1;
    const float* perm_w;
    const float* tscale;
    float out_scale;
    int act;
    float sa, sb;
    const uint8_t* kd0;
    const uint8_t* ks0;
    const uint8_t* kd1;
    const uint8_t* ks1;
    int zero_pad;
    DevError* err;
};

struct CtrlBlock {
    uint64_t full[kMaxStages], empty[kMaxStages];          // operand ring
    uint64_t raw_full[kMaxStages], raw_empty[kMaxStages];  // raw ring (FP4)
    uint64_t tfull[2], tempty[2], drain;
    uint32_t tmem_slot;
    int abort;
    uint16_t lut[256];
    int cu[kMaxG];
    int tpre[kMaxG + 1];
};
static_assert(sizeof(CtrlBlock) <= 12288, "control block");

template <int BT>
__device__ __forceinline__ void decode_tile(int L, const CtrlBlock* c, int G, int NT, int& g, int& nt,
                                            int& row0, int& rows) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (c->tpre[mid] <= L) lo = mid;
        else hi = mid - 1;
    }
    g = lo;
    const int mcount = (c->tpre[g + 1] - c->tpre[g]) / NT;
    const int r = L - c->tpre[g];
    nt = r / mcount;
    const int mt = r - nt * mcount;
    const int start = g ? c->cu[g - 1] : 0;
    row0 = start + mt * BT;
    rows = min(BT, c->cu[g] - row0);
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}
// 8 packed e2m1 values (one 32-bit word, even k in the low nibble) -> 4 x f16x2, times a scale.
__device__ __forceinline__ uint4 e2m1x8_to_f16(uint32_t w, uint32_t sc2) {
    uint32_t o0, o1, o2, o3;
    asm("{ .reg .b8 b0,b1,b2,b3; mov.b32 {b0,b1,b2,b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0; cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2; cvt.rn.f16x2.e2m1x2 %3, b3; }"
        : "=r"(o0), "=r"(o1), "=r"(o2), "=r"(o3)
        : "r"(w));
    return make_uint4(hmul2_u32(o0, sc2), hmul2_u32(o1, sc2), hmul2_u32(o2, sc2), hmul2_u32(o3, sc2));
}
// 32 values (half a 64-value row) -> 4 x 16-byte chunks of the 128-byte-swizzled operand row.
__device__ __forceinline__ void convert_half_row(const uint4 raw, uint32_t sc2_lo, uint32_t sc2_hi,
                                                 uint8_t* row_base, int r, int c_first) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 o = e2m1x8_to_f16(w[i], i < 2 ? sc2_lo : sc2_hi);
        *reinterpret_cast<uint4*>(row_base + (((c_first + i) ^ (r & 7)) << 4)) = o;
    }
}

template <int BT, bool DUAL, int WFMT, int OUT>
__global__ void __launch_bounds__(GemmCfg<BT, DUAL, WFMT>::THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_w0,
                        const __grid_constant__ CUtensorMap tm_w1, const GemmArgs a) {
    using C = GemmCfg<BT, DUAL, WFMT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // operand ring: stage s = [A0][A1 if dual][B if BF16]; raw ring (FP4): [B][D0][D1][S0][S1]
    uint8_t* sOp = smem;
    uint8_t* sRaw = sOp + C::STAGES * C::OP_STAGE;
    CtrlBlock* ctl = reinterpret_cast<CtrlBlock*>(sRaw + C::RSTAGES * C::RAW_STAGE);
    volatile int* abort_flag = &ctl->abort;
    auto opA = [&](int s, int m) { return sOp + s * C::OP_STAGE + m * C::A_BYTES; };
    auto opB = [&](int s) { return sOp + s * C::OP_STAGE + C::NB * C::A_BYTES; };
    auto rawB = [&](int r) { return sRaw + r * C::RAW_STAGE; };
    auto rawD = [&](int r, int m) { return sRaw + r * C::RAW_STAGE + C::B_BYTES + m * C::RAW_D; };
    auto rawS = [&](int r, int m) {
        return sRaw + r * C::RAW_STAGE + C::B_BYTES + C::NB * C::RAW_D + m * C::RAW_S;
    };

    const int warp = warp_id(), lane = lane_id();
    const int G = a.G, NT = a.NT, KB = a.KB;

    // ---------------- prologue: independent of the previous kernel's output
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&ctl->full[s], C::FP4 ? C::CONV_WARPS : 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int r = 0; r < C::RSTAGES; ++r) {
            mbar_init(&ctl->raw_full[r], 1);
            mbar_init(&ctl->raw_empty[r], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tfull[b], 1);
            mbar_init(&ctl->tempty[b], 4);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_barrier_init();
    }
    if (threadIdx.x == 32) {
        tma_prefetch_desc(&tm_x);
        if (!C::FP4) {
            tma_prefetch_desc(&tm_w0);
            if (DUAL) tma_prefetch_desc(&tm_w1);
        }
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    if (WFMT == MOE_W_MXFP4) {
        // e8m0 (already re-biased by the weight preparation) -> f16 bits of 2^(e-127)
        for (int i = threadIdx.x; i < 256; i += blockDim.x) {
            const int e = i - 127;
            uint16_t bits;
            if (e >= -14 && e <= 15) bits = (uint16_t)((e + 15) << 10);
            else if (e >= -24 && e < -14) bits = (uint16_t)(1u << (e + 24));
            else bits = e > 15 ? (uint16_t)0x7C00 : (uint16_t)0;
            ctl->lut[i] = bits;
        }
    }
    pdl_wait();
    if (warp == 0) {
        // segment table: cu (inclusive ends) and the running tile count.
        // Ends are clamped to [0, M_alloc] and a segment whose end lies before the
        // previous end counts as empty, so no tile can touch rows outside the buffers.
        int carry = 0, prev_chunk_end = 0;
        for (int base = 0; base < G; base += 32) {
            const int g = base + lane;
            const int raw = g < G ? a.cu[g] : 0;
            const int end = min(max(raw, 0), a.M_alloc);
            int prev = __shfl_up_sync(0xffffffffu, end, 1);
            if (lane == 0) prev = prev_chunk_end;
            if (g < G && (raw != end || end < prev)) report_error(a.err, MOE_ERR_DEVICE, 1000000 + g);
            const int len = g < G ? max(0, end - prev) : 0;
            const int tiles = ((len + BT - 1) / BT) * NT;
            int incl = tiles;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += n;
            }
            if (g < G) {
                ctl->cu[g] = len > 0 ? end : prev;
                ctl->tpre[g + 1] = carry + incl;
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
            const int eff = g < G ? (len > 0 ? end : prev) : prev;
            prev_chunk_end = __shfl_sync(0xffffffffu, eff, 31);
        }
        if (lane == 0) ctl->tpre[0] = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch();
    const uint32_t tmem_base = ctl->tmem_slot;
    const int total = ctl->tpre[G];

    if (warp == 0) {
        // ---------------- producer
        if (lane == 0) {
            constexpr int NS = C::FP4 ? C::RSTAGES : C::STAGES;
            uint64_t* fullb = C::FP4 ? ctl->raw_full : ctl->full;
            uint64_t* emptyb = C::FP4 ? ctl->raw_empty : ctl->empty;
            int s = 0;
            uint32_t ph = 0, issued_mask = 0, issued_par = 0;
            bool ok = true;
            for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
                int g, nt, row0, rows;
                decode_tile<BT>(L, ctl, G, NT, g, nt, row0, rows);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&emptyb[s], ph ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (!C::FP4) {
                        mbar_arrive_expect_tx(&fullb[s], C::NB * C::A_BYTES + C::B_BYTES);
                        tma_load_3d(opA(s, 0), &tm_w0, &fullb[s], kb * kTileK, nt * kTileN, g);
                        if (DUAL) tma_load_3d(opA(s, 1), &tm_w1, &fullb[s], kb * kTileK, nt * kTileN, g);
                        tma_load_2d(opB(s), &tm_x, &fullb[s], kb * kTileK, row0);
                    } else {
                        const size_t tile = ((size_t)g * NT + nt) * KB + kb;
                        mbar_arrive_expect_tx(&fullb[s], C::B_BYTES + C::NB * (C::RAW_D + C::RAW_S));
                        bulk_load(rawD(s, 0), a.kd0 + tile * C::RAW_D, C::RAW_D, &fullb[s]);
                        bulk_load(rawS(s, 0), a.ks0 + tile * C::RAW_S, C::RAW_S, &fullb[s]);
                        if (DUAL) {
                            bulk_load(rawD(s, 1), a.kd1 + tile * C::RAW_D, C::RAW_D, &fullb[s]);
                            bulk_load(rawS(s, 1), a.ks1 + tile * C::RAW_S, C::RAW_S, &fullb[s]);
                        }
                        tma_load_2d(rawB(s), &tm_x, &fullb[s], kb * kTileK, row0);
                    }
                    issued_mask |= 1u << s;
                    issued_par = (issued_par & ~(1u << s)) | (ph << s);
                    if (++s == NS) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok) {
                report_error(a.err, MOE_ERR_TIMEOUT, 1);
                ctl->abort = 1;
                // let every copy this thread issued land before the CTA exits
                int never = 0;
                for (int q = 0; q < NS; ++q)
                    if (issued_mask >> q & 1u) mbar_wait(&fullb[q], issued_par >> q & 1u, &never);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16(C::FP4 ? 0 : 1, kTileN, BT);
            int s = 0, r = 0, b = 0;
            uint32_t ph = 0, rph = 0, bph = 0;
            bool ok = true, issued = false;
            for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
                if (!mbar_wait(&ctl->tempty[b], bph ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d0 = tmem_base + (uint32_t)(b * C::NB * BT);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&ctl->full[s], ph, abort_flag) ||
                        (C::FP4 && !mbar_wait(&ctl->raw_full[r], rph, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(opA(s, 0));
                    const uint32_t a1 = smem_u32(opA(s, DUAL ? 1 : 0));
                    const uint32_t bb = smem_u32(C::FP4 ? rawB(r) : opB(s));
#pragma unroll
                    for (int kk = 0; kk < kTileK / 16; ++kk) {
                        const uint64_t bdesc = sw128_kmajor_desc(bb + kk * 32);
                        const uint32_t acc = (kb | kk) != 0;
                        mma_f16_ss(d0, sw128_kmajor_desc(a0 + kk * 32), bdesc, idesc, acc);
                        if (DUAL) mma_f16_ss(d0 + BT, sw128_kmajor_desc(a1 + kk * 32), bdesc, idesc, acc);
                    }
                    issued = true;
                    mma_commit(&ctl->empty[s]);
                    if (++s == C::STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                    if (C::FP4) {
                        mma_commit(&ctl->raw_empty[r]);
                        if (++r == C::RSTAGES) {
                            r = 0;
                            rph ^= 1u;
                        }
                    }
                }
                if (!ok) break;
                mma_commit(&ctl->tfull[b]);
                b ^= 1;
                if (b == 0) bph ^= 1u;
            }
            if (!ok) {
                report_error(a.err, MOE_ERR_TIMEOUT, 2);
                ctl->abort = 1;
                if (issued) {
                    // wait (bounded) for the MMAs in flight before TMEM is released
                    int never = 0;
                    mma_commit(&ctl->drain);
                    mbar_wait(&ctl->drain, 0, &never);
                }
            }
        }
    } else if (warp < 6) {
        // ---------------- epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        int b = 0;
        uint32_t bph = 0;
        for (int L = blockIdx.x; L < total; L += gridDim.x) {
            int g, nt, row0, rows;
            decode_tile<BT>(L, ctl, G, NT, g, nt, row0, rows);
            if (!mbar_wait(&ctl->tfull[b], bph, abort_flag)) {
                if (lane == 0) report_error(a.err, MOE_ERR_TIMEOUT, 3);
                ctl->abort = 1;
                break;
            }
            tc_fence_after();
            const int n = nt * kTileN + q * 32 + lane;
            const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * C::NB * BT);
            const float al0 = a.alpha0 ? a.alpha0[g] : 1.0f;
            const float al1 = a.alpha1 ? a.alpha1[g] : 1.0f;
#pragma unroll 1
            for (int c0 = 0; c0 < BT; c0 += 16) {
                if (c0 >= rows) break;
                uint32_t r0[16], r1[16];
                tmem_ld16(tb + c0, r0);
                if (DUAL) tmem_ld16(tb + BT + c0, r1);
                tmem_ld_wait();
                if (n < a.N) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        if (c0 + j < rows) {
                            const int row = row0 + c0 + j;
                            const float ts = a.tscale ? a.tscale[row] : 1.0f;
                            float v;
                            if (DUAL) {
                                const float gv = __uint_as_float(r0[j]) * al0 * ts;
                                const float uv = __uint_as_float(r1[j]) * al1 * ts;
                                v = act_apply(a.act, gv, uv, a.sa, a.sb);
                                if (a.perm_w) v *= a.perm_w[row];
                            } else {
                                v = __uint_as_float(r0[j]) * al0 * ts;
                            }
                            v *= a.out_scale;
                            const size_t idx = (size_t)row * a.N + n;
                            if (OUT == OUT_BF16) reinterpret_cast<__nv_bfloat16*>(a.out)[idx] = __float2bfloat16_rn(v);
                            else if (OUT == OUT_F16) reinterpret_cast<__half*>(a.out)[idx] = __float2half_rn(v);
                            else reinterpret_cast<float*>(a.out)[idx] = v;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->tempty[b]);
            b ^= 1;
            if (b == 0) bph ^= 1u;
        }
        if (a.zero_pad && OUT == OUT_BF16) {
            // rows [cu[G-1], M_alloc) of the output are zero
            const int start = G > 0 ? ctl->cu[G - 1] : 0;
            const long long count = (long long)(a.M_alloc - start) * a.N;
            __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.out) + (size_t)start * a.N;
            const long long tid = (long long)blockIdx.x * 128 + (threadIdx.x - 64);
            const long long stride = (long long)gridDim.x * 128;
            for (long long i = tid; i < count; i += stride) o[i] = __float2bfloat16_rn(0.0f);
        }
    } else if (C::CONV_WARPS > 0) {
        // ---------------- FP4 -> f16 converters (FP4 dequant fused into the mainloop)
        const int ct = threadIdx.x - 6 * 32;  // 0 .. CONV_THREADS-1
        int s = 0, r = 0;
        uint32_t ph = 0, rph = 0;
        bool ok = true;
        for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
            for (int kb = 0; kb < KB; ++kb) {
                if (!mbar_wait(&ctl->raw_full[r], rph, abort_flag) ||
                    !mbar_wait(&ctl->empty[s], ph ^ 1u, abort_flag)) {
                    if (lane == 0) report_error(a.err, MOE_ERR_TIMEOUT, 4);
                    ctl->abort = 1;
                    ok = false;
                    break;
                }
                // items: (matrix m, row, half) -> 16 raw bytes = 32 values each; contiguous reads
                constexpr int ITEMS = C::NB * kTileN * 2;
#pragma unroll
                for (int it = 0; it < ITEMS / C::CONV_THREADS; ++it) {
                    const int item = ct + C::CONV_THREADS * it;
                    const int m = item / (kTileN * 2);
                    const int ri = item - m * (kTileN * 2);
                    const int row = ri >> 1, h = ri & 1;
                    const uint4 v = *reinterpret_cast<const uint4*>(rawD(r, m) + ri * 16);
                    const uint8_t* rs = rawS(r, m);
                    uint32_t lo, hi;
                    if (WFMT == MOE_W_MXFP4) {
                        const uint32_t bits = ctl->lut[rs[row * 2 + h]];
                        lo = hi = bits | (bits << 16);
                    } else {
                        const uint16_t pair = *reinterpret_cast<const uint16_t*>(rs + row * 4 + h * 2);
                        uint32_t s2;
                        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(s2) : "h"(pair));
                        lo = (s2 & 0xFFFFu) | (s2 << 16);
                        hi = (s2 >> 16) | (s2 & 0xFFFF0000u);
                    }
                    convert_half_row(v, lo, hi, opA(s, m) + row * 128, row, h * 4);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->full[s]);
                if (++s == C::STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
                if (++r == C::RSTAGES) {
                    r = 0;
                    rph ^= 1u;
                }
            }
        }
    }

    // ---------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ============================================================ host side

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D map over a row-major [rows, cols] matrix of 16-bit elements; box = 64 cols x box_rows.
bool make_map_2d(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, uint64_t cols,
                 uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kTileK, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over weights [G, N, K] of 16-bit elements; box = 64 (K) x 128 (N) x 1.
bool make_map_3d(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, uint64_t K, uint64_t N,
                 uint64_t G) {
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    const cuuint64_t dims[3] = {K, N, G};
    const cuuint64_t strides[2] = {K * 2, N * K * 2};
    const cuuint32_t box[3] = {(cuuint32_t)kTileK, (cuuint32_t)kTileN, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BT, bool DUAL, int WFMT, int OUT>
cudaError_t run(const GemmProblem& p, const GemmArgs& args, const CUtensorMap& tx, const CUtensorMap& t0,
                const CUtensorMap& t1, cudaStream_t st, bool pdl) {
    using C = GemmCfg<BT, DUAL, WFMT>;
    auto kern = grouped_gemm_kernel<BT, DUAL, WFMT, OUT>;
    static int attr_set[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set[dev] = 1;
    }
    const long long tiles_ub = ((long long)(p.M_alloc + BT - 1) / BT + p.G) * args.NT;
    const int grid = (int)std::max<long long>(1, std::min<long long>(num_sms(), tiles_ub));
    return launch_k(kern, dim3(grid), dim3(C::THREADS), (size_t)C::SMEM_BYTES, st, pdl, tx, t0, t1, args);
}

template <int BT>
cudaError_t dispatch_bt(const GemmProblem& p, const GemmArgs& args, const CUtensorMap& tx,
                        const CUtensorMap& t0, const CUtensorMap& t1, cudaStream_t st, bool pdl) {
    if (p.dual) {
        if (p.wfmt == MOE_W_BF16) return run<BT, true, MOE_W_BF16, OUT_BF16>(p, args, tx, t0, t1, st, pdl);
        if (p.wfmt == MOE_W_MXFP4) {
            if (p.out_kind == OUT_F16) return run<BT, true, MOE_W_MXFP4, OUT_F16>(p, args, tx, t0, t1, st, pdl);
            return run<BT, true, MOE_W_MXFP4, OUT_F32>(p, args, tx, t0, t1, st, pdl);
        }
        if (p.out_kind == OUT_F16) return run<BT, true, MOE_W_NVFP4, OUT_F16>(p, args, tx, t0, t1, st, pdl);
        return run<BT, true, MOE_W_NVFP4, OUT_F32>(p, args, tx, t0, t1, st, pdl);
    }
    if (p.out_kind == OUT_F32) {
        if (p.wfmt == MOE_W_BF16) return run<BT, false, MOE_W_BF16, OUT_F32>(p, args, tx, t0, t1, st, pdl);
        if (p.wfmt == MOE_W_MXFP4) return run<BT, false, MOE_W_MXFP4, OUT_F32>(p, args, tx, t0, t1, st, pdl);
        return run<BT, false, MOE_W_NVFP4, OUT_F32>(p, args, tx, t0, t1, st, pdl);
    }
    if (p.wfmt == MOE_W_BF16) return run<BT, false, MOE_W_BF16, OUT_BF16>(p, args, tx, t0, t1, st, pdl);
    if (p.wfmt == MOE_W_MXFP4) return run<BT, false, MOE_W_MXFP4, OUT_BF16>(p, args, tx, t0, t1, st, pdl);
    return run<BT, false, MOE_W_NVFP4, OUT_BF16>(p, args, tx, t0, t1, st, pdl);
}

}  // namespace

int choose_token_tile(long long NvS, int G) {
    const long long segs = std::max<long long>(1, std::min<long long>(G, NvS));
    const long long avg = (NvS + segs - 1) / segs;
    if (avg <= 16) return 16;
    if (avg <= 32) return 32;
    if (avg <= 64) return 64;
    return 128;
}

cudaError_t launch_grouped_gemm(const GemmProblem& p, cudaStream_t st, bool pdl) {
    if (p.G > kMaxG) return cudaErrorInvalidValue;
    GemmArgs a{};
    a.cu = p.cu_seqlens;
    a.G = p.G;
    a.N = p.N;
    a.K = p.K;
    a.KB = (p.K + kTileK - 1) / kTileK;
    a.NT = (p.N + kTileN - 1) / kTileN;
    a.M_alloc = p.M_alloc;
    a.out = p.out;
    a.alpha0 = p.alpha0;
    a.alpha1 = p.alpha1;
    a.perm_w = p.perm_w;
    a.tscale = p.tscale;
    a.out_scale = p.out_scale;
    a.act = p.act;
    a.sa = p.situ_a;
    a.sb = p.situ_b;
    a.kd0 = static_cast<const uint8_t*>(p.kdata0);
    a.ks0 = static_cast<const uint8_t*>(p.kscale0);
    a.kd1 = static_cast<const uint8_t*>(p.kdata1);
    a.ks1 = static_cast<const uint8_t*>(p.kscale1);
    a.zero_pad = p.zero_pad ? 1 : 0;
    a.err = p.err;
    int bt = p.bt;
    if (!bt) {
        // MOE_TOKEN_TILE=16|32|64|128 overrides the token-tile choice (tests, tuning)
        const char* env = getenv("MOE_TOKEN_TILE");
        const int v = env ? atoi(env) : 0;
        bt = (v == 16 || v == 32 || v == 64 || v == 128) ? v : choose_token_tile(p.M_alloc, p.G);
    }
    const CUtensorMapDataType xdt =
        p.wfmt == MOE_W_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUtensorMap tx, t0, t1;
    memset(&t0, 0, sizeof(t0));
    memset(&t1, 0, sizeof(t1));
    if (!make_map_2d(&tx, p.x, xdt, p.K, p.M_alloc, bt)) return cudaErrorInvalidValue;
    if (p.wfmt == MOE_W_BF16) {
        if (!make_map_3d(&t0, p.w0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.K, p.N, p.G)) return cudaErrorInvalidValue;
        if (p.dual && !make_map_3d(&t1, p.w1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.K, p.N, p.G))
            return cudaErrorInvalidValue;
    }
    switch (bt) {
        case 16: return dispatch_bt<16>(p, a, tx, t0, t1, st, pdl);
        case 32: return dispatch_bt<32>(p, a, tx, t0, t1, st, pdl);
        case 64: return dispatch_bt<64>(p, a, tx, t0, t1, st, pdl);
        default: return dispatch_bt<128>(p, a, tx, t0, t1, st, pdl);
    }
}

}  // namespace moe
