// S3/S4/S5 — persistent grouped GEMMs on the 5th-generation tensor cores.
//
// Computes out[seg_g] = alpha_g * x[seg_g] @ W[g]^T over the expert-contiguous
// segments of cu_seqlens (MoonEP experts page, moonep_grouped_gemm), optionally
// as the fused gate+up pair with the gated activation and route weight in the
// epilogue (MoonEP experts page, module docstring: act = silu(gate)*up*route_w;
// SITU from the TRTLLM MXFP4 page).
//
// Tiling ("swap AB"): one tile is 128 weight rows (the MMA M side) by BT token
// rows (the MMA N side, 16..256) of one segment. Decode segments hold a handful
// of tokens, so the token side is the narrow one; the weights stream through
// at full width. Each CTA owns one SM and walks the tile list
// (segment, weight block, token block) with the token block fastest, so the
// CTAs working on one weight block at the same time share it through L2.
//
// Four kernels share the tile schedule and the epilogue:
//
// grouped_gemm_kernel (BF16 weights): a ring of shared-memory stages
//   {gate tile, [up tile], token tile} filled by TMA; kind::f16 MMAs from smem.
//
// grouped_gemm_nvf4_kernel (NVFP4 weights, NVFP4 activations): block-scaled
//   kind::mxf4nvf4 MMAs. Weights arrive as prepared 128 x 256 tiles (swizzled codes
//   plus e4m3 scale blocks, one bulk copy each), tokens as packed e2m1 rows plus
//   scales (TMA); a scale warp copies both scale sets into tensor memory.
//
// grouped_gemm_mx8_kernel (MXFP4 weights, bf16 activations): block-scaled
//   kind::mxf8f6f4 MMAs of e2m1 weights (4-bit tensor map) against the activations
//   staged as two e4m3 terms with a shared e8m0 scale per 32 values.
//
// grouped_gemm_fp4_kernel (NVFP4 weights, bf16 activations): a deep ring of small
//   raw stages {token tile, packed e2m1 codes, block scales}; converter warps expand
//   the codes to f16 (times the block scale, exact) straight into a ring of weight
//   tiles in tensor memory, and the MMA reads A from TMEM and the tokens from smem.
//
// Warp roles (one CTA per SM): a producer thread (TMA / bulk copies), one or more
// MMA-issuing threads (the first one's warp owns TMEM), four or eight epilogue warps
// (TMEM -> registers -> alpha / activation / scales -> global), and per kernel a
// scale warp or converter warps. Every wait is bounded; a timeout records
// MOE_ERR_TIMEOUT in the error word, stops all roles, lets copies in flight land,
// frees TMEM and returns.
#include <cmath>
#include <mutex>

#include "internal.h"

namespace moe {

constexpr int kMaxG = 1024;      // segment table capacity (weight rows)
constexpr int kMaxStages = 16;
constexpr int kCtrlBytes = 12288;
constexpr int kSmemLimit = 232448;
constexpr int kSmemBudget = kSmemLimit - 1024 - kCtrlBytes;

__host__ __device__ constexpr int round1024(int b) { return (b + 1023) & ~1023; }
__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int tmem_cols_pow2(int c) {
    return c <= 32 ? 32 : c <= 64 ? 64 : c <= 128 ? 128 : c <= 256 ? 256 : 512;
}

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
    int x3d;          // FP4: the token map is 3-D {64, rows, K/64}: one copy per 128-K stage
    DevError* err;
    long long wait_limit;  // cycles a pipeline wait may take before the kernel gives up
    int l2_w, l2_t;        // L2 policy of the weight and of the token copies (see l2_policy)
    // Per-expert fp32 biases [G, N] (or NULL): the gate/up pair adds bias0 / bias1 before the
    // activation; a single GEMM adds bias_rw[row] * bias0 to its output (bias_rw NULL: 1).
    const float* bias0;
    const float* bias1;
    const float* bias_rw;
    float sw_alpha, sw_beta, sw_limit;  // SWIGLUOAI
    int out_terms, out_stride, out_kpad;  // OUT_MX8 records: terms, row stride, codes per term
    // fused gather (CTA pairs): token row r of the GEMM is row gather_idx[r] of gx [gather_rows, K]
    const int32_t* gather_idx;
    const __nv_bfloat16* gx;
    int gather_rows;
};

struct CtrlBlock {
    uint64_t full[kMaxStages], empty[kMaxStages];          // operand ring (smem or TMEM)
    uint64_t raw_full[kMaxStages], raw_empty[kMaxStages];  // raw ring (FP4)
    uint64_t tfull[2], tempty[2], drain[6];
    uint32_t tmem_slot;
    int abort;
    int cu[kMaxG];
    int tpre[kMaxG + 1];
};
static_assert(sizeof(CtrlBlock) <= kCtrlBytes, "control block");

// ------------------------------------------------------------------ shared pieces

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
    // the segment's mcount = ceil(len / BT) token tiles share its rows evenly (in multiples of
    // 16, at most BT each), so that the tiles of one weight block take about the same time and
    // read the weight tile from L2 together; (mcount - 1) * rs < len keeps every tile non-empty
    const int len = c->cu[g] - start;
    const int rs = min(BT, ((len + mcount - 1) / mcount + 15) & ~15);
    row0 = start + mt * rs;
    rows = min(rs, c->cu[g] - row0);
}

// One warp: the segment table (cu, clamped, and the running tile count tpre).
// Ends are clamped to [0, M_alloc] and a segment whose end lies before the previous
// end counts as empty, so no tile can touch rows outside the buffers.
template <int BT>
__device__ __forceinline__ void build_segment_table(const GemmArgs& a, CtrlBlock* ctl, int lane) {
    const int G = a.G, NT = a.NT;
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

// What one thread has in flight: the producer's stages (and the parity of each one's last
// issue), or whether a tcgen05 issuer (MMA or scale copies) issued anything.
struct Issued {
    uint32_t mask = 0, par = 0;
    bool tc = false;
};

// After an abort, before the CTA's shared and tensor memory are released: the producer
// waits for its copies to land, a tcgen05 issuer commits to its own drain barrier and waits
// for it. An abort can come after a role left its loop normally, so this runs for every
// role once all have stopped. These waits take the default limit; nothing aborts them.
__device__ __forceinline__ void drain_in_flight(const Issued& is, uint64_t* full, int stages, uint64_t* drain) {
    int never = 0;
    for (int q = 0; q < stages; ++q)
        if (is.mask >> q & 1u) mbar_wait(&full[q], is.par >> q & 1u, &never);
    if (is.tc && drain) {
        mma_commit(drain);
        mbar_wait(drain, 0, &never);
    }
}

// Epilogue of one tile for the warp owning TMEM lanes [32q, 32q+32). The accumulator
// buffer at column tb holds NPART partial sums per matrix. Partial j of matrix m sits at
// tb + (j*NB + m)*BT (partials of different issuers, PM = false), or at
// tb + (m*NPART + j)*BT (PM = true: one MMA wrote a matrix's partials side by side).
// With EW warps per lane quarter, warp h of a quarter takes the 16-token chunks h, h+EW, ...

// Tokens c0 .. c0+15 of this lane's row, partial sums added: matrix 0 in r0, matrix 1 in r1.
template <int BT, bool DUAL, int NPART, bool PM>
__device__ __forceinline__ void epi_load16(uint32_t tb, int c0, uint32_t (&r0)[16], uint32_t (&r1)[16]) {
    constexpr int NB = DUAL ? 2 : 1;
    auto col = [](int m, int j) { return (PM ? m * NPART + j : j * NB + m) * BT; };
    tmem_ld16(tb + col(0, 0) + c0, r0);
    if (DUAL) tmem_ld16(tb + col(1, 0) + c0, r1);
    tmem_ld_wait();
#pragma unroll
    for (int pj = 1; pj < NPART; ++pj) {
        uint32_t p0[16], p1[16];
        tmem_ld16(tb + col(0, pj) + c0, p0);
        if (DUAL) tmem_ld16(tb + col(1, pj) + c0, p1);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            r0[j] = __float_as_uint(__uint_as_float(r0[j]) + __uint_as_float(p0[j]));
            if (DUAL) r1[j] = __float_as_uint(__uint_as_float(r1[j]) + __uint_as_float(p1[j]));
        }
    }
}

// What a lane's output column n needs for every token of a tile.
struct EpiCol {
    int n;
    float al0, al1, bn0, bn1, inv_sa, inv_sb;
};

template <bool DUAL>
__device__ __forceinline__ EpiCol epi_col(const GemmArgs& a, int g, int nt, int q, int lane) {
    EpiCol c;
    c.n = nt * kTileN + q * 32 + lane;
    c.al0 = a.alpha0 ? a.alpha0[g] : 1.0f;
    c.al1 = a.alpha1 ? a.alpha1[g] : 1.0f;
    c.bn0 = (a.bias0 && c.n < a.N) ? a.bias0[(size_t)g * a.N + c.n] : 0.0f;
    c.bn1 = (DUAL && a.bias1 && c.n < a.N) ? a.bias1[(size_t)g * a.N + c.n] : 0.0f;
    c.inv_sa = 1.0f / a.sa;
    c.inv_sb = 1.0f / a.sb;
    return c;
}

// Per-token factors of a 16-token chunk, loaded by lane (token % 16) and broadcast later:
// the token's activation row scale and the dual GEMM's route weight (a single GEMM's: the
// weight of its bias).
template <bool DUAL>
__device__ __forceinline__ void epi_token_factors(const GemmArgs& a, int row0, int c0, int rows, int lane, float& ts,
                                                  float& pw) {
    const int my_row = row0 + c0 + (lane & 15);
    const bool row_ok = c0 + (lane & 15) < rows;
    ts = (a.tscale && row_ok) ? a.tscale[my_row] : 1.0f;
    const float* rw = DUAL ? a.perm_w : a.bias_rw;
    pw = (rw && row_ok) ? rw[my_row] : 1.0f;
}

// The gated activation of one token (the dual GEMM) times its route weight.
__device__ __forceinline__ float epi_gated(const GemmArgs& a, const EpiCol& c, uint32_t x0, uint32_t x1, float ts,
                                           float pw) {
    const float gv = __uint_as_float(x0) * c.al0 * ts + c.bn0;
    const float uv = __uint_as_float(x1) * c.al1 * ts + c.bn1;
    return (a.act == MOE_ACT_SWIGLUOAI ? swigluoai_fast(gv, uv, a.sw_alpha, a.sw_beta, a.sw_limit)
                                       : act_apply_fast(a.act, gv, uv, a.sa, a.sb, c.inv_sa, c.inv_sb)) *
           pw;
}

// One token's 32-value block of the down GEMM's K (this warp's 32 lanes): its e8m0 scale,
// then the e4m3 code (and the lo term's) of each lane's value. Lanes past N (up to the padded
// K) hold zeros. All lanes take part. For finite values the block exponent is a
// non-decreasing function of the block's largest magnitude, so it is the warp max of the
// lanes' own exponents: one integer reduction instead of a shuffle tree over floats. An
// infinite value makes the block's largest magnitude infinite (key 255), and the block takes
// that magnitude's exponent; NaNs do not count, as in a max over floats.
__device__ __forceinline__ void epi_store_mx8(const GemmArgs& a, int row, int n, int lane, float v) {
    const bool two = a.out_terms == 2;
    const float av = fabsf(v);
    const unsigned key = isinf(av) ? 255u : (unsigned)(mx8_block_exp(av, two) + 127);
    const unsigned kmax = __reduce_max_sync(0xffffffffu, key);
    const int e = kmax == 255u ? mx8_block_exp(__int_as_float(0x7f800000), two) : (int)kmax - 127;
    const float y = v * mx8_inv_scale(e);
    uint8_t* rec = reinterpret_cast<uint8_t*>(a.out) + (size_t)row * a.out_stride;
    const uint8_t hi = cvt_e4m3(y);
    rec[n] = hi;
    if (two) rec[a.out_kpad + n] = cvt_e4m3(y - e4m3_to_f32(hi));
    if (lane == 0) rec[a.out_terms * a.out_kpad + n / 32] = (uint8_t)(e + 127);
}

template <int OUT>
__device__ __forceinline__ void epi_store(const GemmArgs& a, int row, int n, float v) {
    const size_t idx = (size_t)row * a.N + n;
    if (OUT == OUT_BF16) reinterpret_cast<__nv_bfloat16*>(a.out)[idx] = __float2bfloat16_rn(v);
    else if (OUT == OUT_F16) reinterpret_cast<__half*>(a.out)[idx] = __float2half_rn(v);
    else reinterpret_cast<float*>(a.out)[idx] = v;
}

template <int BT, bool DUAL, int OUT, int NPART = 1, bool PM = false, int EW = 1>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& a, uint32_t tb, int g, int nt, int row0, int rows,
                                              int q, int lane, int h = 0) {
    const EpiCol c = epi_col<DUAL>(a, g, nt, q, lane);
    const int n = c.n;
#pragma unroll 1
    for (int c0 = 16 * h; c0 < BT; c0 += 16 * EW) {
        if (c0 >= rows) break;
        uint32_t r0[16], r1[16];
        epi_load16<BT, DUAL, NPART, PM>(tb, c0, r0, r1);
        float my_ts, my_pw;
        epi_token_factors<DUAL>(a, row0, c0, rows, lane, my_ts, my_pw);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            // every lane takes part in the shuffles; only in-range outputs are stored
            const float ts = __shfl_sync(0xffffffffu, my_ts, j);
            const float pw = __shfl_sync(0xffffffffu, my_pw, j);
            const int row = row0 + c0 + j;
            if constexpr (OUT == OUT_MX8) {
                // rows, c0 and j are the same in every lane, so the warp stays whole
                if (c0 + j < rows)
                    epi_store_mx8(a, row, n, lane, DUAL && n < a.N ? epi_gated(a, c, r0[j], r1[j], ts, pw) : 0.0f);
            } else if (n < a.N && c0 + j < rows) {
                const float v = DUAL ? epi_gated(a, c, r0[j], r1[j], ts, pw) * a.out_scale
                                     : __uint_as_float(r0[j]) * c.al0 * ts * a.out_scale + pw * c.bn0;
                epi_store<OUT>(a, row, n, v);
            }
        }
    }
}

// The epilogue of a single-buffered accumulator whose output is the down GEMM's e4m3
// records (the MXFP4 gate/up tile). The next tile's MMAs wait for it, so phase 1 only reads
// this warp's chunks out of tensor memory and applies the activation into registers; then
// `release()` frees the accumulator, and phase 2 encodes and stores while the next tile's
// MMAs run. The values are those of epilogue_tile.
template <int BT, int NPART, bool PM, int EW, typename Rel>
__device__ __forceinline__ void epilogue_tile_mx8_staged(const GemmArgs& a, uint32_t tb, int g, int nt, int row0,
                                                         int rows, int q, int lane, int h, Rel release) {
    constexpr int NCH = BT / (16 * EW);  // this warp's chunks
    const EpiCol c = epi_col<true>(a, g, nt, q, lane);
    const int n = c.n;
    float vals[NCH][16];
#pragma unroll
    for (int ci = 0; ci < NCH; ++ci) {
        const int c0 = 16 * (h + ci * EW);
        if (c0 < rows) {
            uint32_t r0[16], r1[16];
            epi_load16<BT, true, NPART, PM>(tb, c0, r0, r1);
            float my_ts, my_pw;
            epi_token_factors<true>(a, row0, c0, rows, lane, my_ts, my_pw);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float ts = __shfl_sync(0xffffffffu, my_ts, j);
                const float pw = __shfl_sync(0xffffffffu, my_pw, j);
                vals[ci][j] = n < a.N ? epi_gated(a, c, r0[j], r1[j], ts, pw) : 0.0f;
            }
        }
    }
    release();
#pragma unroll
    for (int ci = 0; ci < NCH; ++ci) {
        const int c0 = 16 * (h + ci * EW);
        if (c0 < rows) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                if (c0 + j >= rows) break;  // the same in every lane
                epi_store_mx8(a, row0 + c0 + j, n, lane, vals[ci][j]);
            }
        }
    }
}

// The token half of a stage gathered by the producer warp: 128 rows of 64 K values (128
// bytes), row r of the tile from token tok(r), where lane l holds the tokens of rows l + 32 j
// in tok[j]. Lane 8 rr + c copies chunk c (16 bytes) of rows 4 i + rr, so one warp
// instruction reads four whole 128-byte row segments; chunk c of row r lands at chunk
// position c ^ (r % 8), the 128-byte swizzle the MMA reads. Chunks past K are zero-filled.
__device__ __forceinline__ void gather_stage_rows(uint32_t bb, const __nv_bfloat16* gx, const int (&tok)[4], int K,
                                                  int kb, int lane, uint64_t pol) {
    const int rr = lane >> 3, c = lane & 7;
    const int k = kb * kTileK + c * 8;
    const bool kin = k < K;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int row = 4 * i + rr;
        const int t = __shfl_sync(0xffffffffu, tok[i >> 3], 4 * (i & 7) + rr);
        cp_async16_p(bb + row * 128 + ((c ^ (row & 7)) << 4), kin ? gx + (size_t)t * K + k : gx, kin ? 16u : 0u, pol);
    }
}

// Rows [cu[G-1], M_alloc) of a bf16 output are zero (standalone grouped GEMM).
__device__ __forceinline__ void zero_padding_rows(const GemmArgs& a, const CtrlBlock* ctl, int tid128) {
    const int start = a.G > 0 ? ctl->cu[a.G - 1] : 0;
    const long long count = (long long)(a.M_alloc - start) * a.N;
    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.out) + (size_t)start * a.N;
    const long long stride = (long long)gridDim.x * 128;
    for (long long i = (long long)blockIdx.x * 128 + tid128; i < count; i += stride) o[i] = __float2bfloat16_rn(0.0f);
}

// ------------------------------------------------------------------ BF16 kernel

template <int BT, bool DUAL>
struct Bf16Cfg {
    static constexpr int NB = DUAL ? 2 : 1;
    static constexpr int A_BYTES = kTileN * kTileK * 2;      // 16 KB: 128 rows x 64 bf16
    static constexpr int B_BYTES = BT * kTileK * 2;
    static constexpr int STAGE = NB * A_BYTES + B_BYTES;
    static constexpr int STAGES = cmin(kMaxStages, kSmemBudget / STAGE);
    static constexpr int ACC_COLS = NB * BT;
    // Two accumulator buffers when they fit; the 256-token gate/up tile has one, and two
    // epilogue warps per lane quarter shorten the time the MMAs wait for it.
    static constexpr int ACC_BUFS = 2 * ACC_COLS <= 512 ? 2 : 1;
    static constexpr int EW = ACC_BUFS == 1 ? 2 : 1;
    static constexpr int TMEM_COLS = tmem_cols_pow2(ACC_BUFS * ACC_COLS);
    static constexpr int THREADS = (2 + 4 * EW) * 32;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE + kCtrlBytes;
    static_assert(STAGES >= 2 && SMEM_BYTES <= kSmemLimit && ACC_BUFS * ACC_COLS <= 512, "BF16 GEMM config");
    static_assert(BT % 16 == 0 && BT >= 16 && BT <= 256, "MMA N for M=128 is a multiple of 16 in [16,256]");
};

// GATHER (the 128-token gate/up tile): the token tile of each stage is gathered from gx by
// gather_idx (the permutation's perm_token) by the producer warp's 32 lanes with cp.async, in
// the 128-byte-swizzled layout the MMA reads; stage s is full after lane 0's weight copies and
// 32 cp.async arrivals.
template <int BT, bool DUAL, int OUT, bool GATHER = false>
__global__ void __launch_bounds__(Bf16Cfg<BT, DUAL>::THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_w0,
                        const __grid_constant__ CUtensorMap tm_w1, const GemmArgs a) {
    using C = Bf16Cfg<BT, DUAL>;
    static_assert(!GATHER || BT == 128, "the gather maps 4 rows per lane");
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment by offsetting the shared array itself (no integer round trip),
    // so that every access below stays a shared-memory access
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    CtrlBlock* ctl = reinterpret_cast<CtrlBlock*>(smem + C::STAGES * C::STAGE);
    volatile int* abort_flag = &ctl->abort;
    Issued is;  // this thread's copies or tcgen05 operations in flight
    auto opA = [&](int s, int m) { return smem + s * C::STAGE + m * C::A_BYTES; };
    auto opB = [&](int s) { return smem + s * C::STAGE + C::NB * C::A_BYTES; };
    const int warp = warp_id(), lane = lane_id();
    const int G = a.G, NT = a.NT, KB = a.KB;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&ctl->full[s], GATHER ? 33 : 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tfull[b], 1);
            mbar_init(&ctl->tempty[b], 4 * C::EW);
        }
        mbar_init(&ctl->drain[0], 1);
        ctl->abort = 0;
        fence_barrier_init();
    }
    if (threadIdx.x == 32) {
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_w0);
        if (DUAL) tma_prefetch_desc(&tm_w1);
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    pdl_wait();
    if (warp == 0) build_segment_table<BT>(a, ctl, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch();
    const uint32_t tmem_base = ctl->tmem_slot;
    const int total = ctl->tpre[G];

    if (warp == 0) {
        if (GATHER) {  // ---------------- producer warp: weights by TMA (lane 0), tokens gathered
            const uint64_t pol_w = l2_policy(a.l2_w), pol_t = l2_policy(a.l2_t);
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            const int K = a.K;
            for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
                int g, nt, row0, rows;
                decode_tile<BT>(L, ctl, G, NT, g, nt, row0, rows);
                // the tokens of tile rows lane + 32 i; rows past the GEMM's rows read a valid token
                // (their products are discarded), ids outside [0, gather_rows) too
                int tok[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = min(row0 + lane + 32 * i, a.M_alloc - 1);
                    tok[i] = min(max(a.gather_idx[r], 0), a.gather_rows - 1);
                }
                for (int kb = 0; kb < KB; ++kb) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&ctl->empty[s], ph ^ 1u, abort_flag, a.wait_limit))) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&ctl->full[s], C::NB * C::A_BYTES);
                        tma_load_3d_p(opA(s, 0), &tm_w0, &ctl->full[s], kb * kTileK, nt * kTileN, g, pol_w);
                        if (DUAL) tma_load_3d_p(opA(s, 1), &tm_w1, &ctl->full[s], kb * kTileK, nt * kTileN, g, pol_w);
                    }
                    gather_stage_rows(smem_u32(opB(s)), a.gx, tok, K, kb, lane, pol_t);
                    cp_async_arrive_noinc(&ctl->full[s]);
                    is.mask |= 1u << s;
                    is.par = (is.par & ~(1u << s)) | (ph << s);
                    if (++s == C::STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok && lane == 0) {
                report_error(a.err, MOE_ERR_TIMEOUT, 1);
                ctl->abort = 1;
            }
        } else if (lane == 0) {  // ---------------- TMA producer
            const uint64_t pol_w = l2_policy(a.l2_w), pol_t = l2_policy(a.l2_t);
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
                int g, nt, row0, rows;
                decode_tile<BT>(L, ctl, G, NT, g, nt, row0, rows);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&ctl->empty[s], ph ^ 1u, abort_flag, a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&ctl->full[s], C::NB * C::A_BYTES + C::B_BYTES);
                    tma_load_3d_p(opA(s, 0), &tm_w0, &ctl->full[s], kb * kTileK, nt * kTileN, g, pol_w);
                    if (DUAL) tma_load_3d_p(opA(s, 1), &tm_w1, &ctl->full[s], kb * kTileK, nt * kTileN, g, pol_w);
                    tma_load_2d_p(opB(s), &tm_x, &ctl->full[s], kb * kTileK, row0, pol_t);
                    is.mask |= 1u << s;
                    is.par = (is.par & ~(1u << s)) | (ph << s);
                    if (++s == C::STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok) {
                report_error(a.err, MOE_ERR_TIMEOUT, 1);
                ctl->abort = 1;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {  // ---------------- MMA issuer
            int s = 0, b = 0;
            uint32_t ph = 0, bph = 0;
            bool ok = true;
            for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
                // MMA width: the tile's rows rounded up to 16, so a segment's short last
                // tile does not pay for BT columns
                int g, nt, row0, rows;
                decode_tile<BT>(L, ctl, G, NT, g, nt, row0, rows);
                const uint32_t idesc = idesc_f16(1, kTileN, cmin(BT, (rows + 15) & ~15));
                if (!mbar_wait(&ctl->tempty[b], bph ^ 1u, abort_flag, a.wait_limit)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d0 = tmem_base + (uint32_t)(b * C::ACC_COLS);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&ctl->full[s], ph, abort_flag, a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    if (GATHER) fence_proxy_async_smem();  // the gathered rows came by the generic proxy
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(opA(s, 0));
                    const uint32_t a1 = smem_u32(opA(s, DUAL ? 1 : 0));
                    const uint32_t bb = smem_u32(opB(s));
#pragma unroll
                    for (int kk = 0; kk < kTileK / 16; ++kk) {
                        const uint64_t bdesc = sw128_kmajor_desc(bb + kk * 32);
                        const uint32_t acc = (kb | kk) != 0;
                        mma_f16_ss(d0, sw128_kmajor_desc(a0 + kk * 32), bdesc, idesc, acc);
                        if (DUAL) mma_f16_ss(d0 + BT, sw128_kmajor_desc(a1 + kk * 32), bdesc, idesc, acc);
                    }
                    is.tc = true;
                    mma_commit(&ctl->empty[s]);
                    if (++s == C::STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(&ctl->tfull[b]);
                if (++b == C::ACC_BUFS) {
                    b = 0;
                    bph ^= 1u;
                }
            }
            if (!ok) {
                report_error(a.err, MOE_ERR_TIMEOUT, 2);
                ctl->abort = 1;
            }
        }
    } else {
        // ---------------- epilogue (warps 2 .. 2 + 4 EW)
        const int q = warp & 3, h = (warp - 2) >> 2;  // TMEM lane quarter; chunk phase
        int b = 0;
        uint32_t bph = 0;
        for (int L = blockIdx.x; L < total; L += gridDim.x) {
            int g, nt, row0, rows;
            decode_tile<BT>(L, ctl, G, NT, g, nt, row0, rows);
            if (!mbar_wait(&ctl->tfull[b], bph, abort_flag, a.wait_limit)) {
                if (lane == 0) report_error(a.err, MOE_ERR_TIMEOUT, 3);
                ctl->abort = 1;
                break;
            }
            tc_fence_after();
            const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * C::ACC_COLS);
            auto release = [&] {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->tempty[b]);
            };
            epilogue_tile<BT, DUAL, OUT, 1, false, C::EW>(a, tb, g, nt, row0, rows, q, lane, h);
            release();
            if (++b == C::ACC_BUFS) {
                b = 0;
                bph ^= 1u;
            }
        }
        if (a.zero_pad && OUT == OUT_BF16 && h == 0) zero_padding_rows(a, ctl, threadIdx.x - 64);
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        drain_in_flight(is, ctl->full, C::STAGES, warp == 1 && lane == 0 ? &ctl->drain[0] : nullptr);
        tc_fence_before();
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ BF16 kernel on CTA pairs

// The BF16 GEMM with two SMs per tile (a cluster of two CTAs, cta_group::2 MMAs). A pair tile
// is 256 weight rows (128 from each CTA's shared memory) by up to BT tokens (BT/2 rows in each
// CTA), so each SM moves half the token operand per FLOP of a one-SM tile of the same width.
// The leader (rank 0) issues the MMAs; both CTAs produce their own operands and run the
// epilogue of their own 128 weight rows. Barriers:
//   full[s]   each CTA: its own copies of stage s landed (the leader's MMA thread waits on
//             its own; in the peer, warp 1 waits and forwards to the leader's pfull[s])
//   pfull[s]  leader: the peer's stage s landed
//   empty[s]  each CTA: the MMAs that read stage s completed (commit multicast to both)
//   tfull[b]  each CTA: accumulator buffer b holds a finished tile (commit multicast)
//   tempty[b] leader: both CTAs' epilogue warps have drained buffer b
template <int BT, bool DUAL>
struct PairCfg {
    static constexpr int NB = DUAL ? 2 : 1;
    static constexpr int A_BYTES = kTileN * kTileK * 2;   // this CTA's 128 weight rows x 64 K
    static constexpr int B_ROWS = BT / 2;                 // this CTA's half of the token tile
    static constexpr int B_BYTES = B_ROWS * kTileK * 2;
    static constexpr int STAGE = NB * A_BYTES + B_BYTES;
    static constexpr int STAGES = cmin(kMaxStages, kSmemBudget / STAGE);
    static constexpr int ACC_COLS = NB * BT;
    static constexpr int ACC_BUFS = 2 * ACC_COLS <= 512 ? 2 : 1;
    // with one accumulator buffer the MMAs wait for the epilogue: two warps per lane quarter
    static constexpr int EW = ACC_BUFS == 1 ? 2 : 1;
    static constexpr int EPI_WARPS = 4 * EW;
    static constexpr int TMEM_COLS = tmem_cols_pow2(ACC_BUFS * ACC_COLS);
    static constexpr int THREADS = (2 + EPI_WARPS) * 32;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE + kCtrlBytes;
    static_assert(STAGES >= 3 && SMEM_BYTES <= kSmemLimit && ACC_BUFS * ACC_COLS <= 512, "pair GEMM config");
    static_assert(BT % 32 == 0 && BT >= 32 && BT <= 256, "pair MMA N: a multiple of 32 (16 per CTA) up to 256");
    static_assert(B_BYTES % 1024 == 0, "operands stay 1024-byte aligned");
};

// MMA width of a pair tile: its rows rounded up to 32 (each CTA's half a multiple of 16).
__device__ __forceinline__ int pair_mma_n(int rows, int bt) { return min(bt, (rows + 31) & ~31); }

// GATHER: the token half of each stage is gathered from gx by gather_idx (the permutation's
// perm_token) by the producer warp's 32 lanes with cp.async, in the 128-byte-swizzled layout
// the MMA reads, instead of a TMA box of pre-gathered rows; stage s is full after lane 0's
// weight copies and 32 cp.async arrivals.
// FWD = false (without GATHER): both CTAs' copies of stage s complete on the leader's full[s]
// (cta_group::2 TMA loads), whose expected bytes the leader's producer sets for both, so the
// MMA waits on one local barrier and no stage takes a forwarding hop. The peer cannot watch
// its own copies then; after an abort it lets them settle (a bounded pause) before exiting.
template <int BT, bool DUAL, int OUT, bool GATHER = false, bool FWD = true>
__global__ void __launch_bounds__(PairCfg<BT, DUAL>::THREADS, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w0,
                             const __grid_constant__ CUtensorMap tm_w1, const GemmArgs a) {
    using C = PairCfg<BT, DUAL>;
    static_assert(!GATHER || C::B_ROWS == 128, "the gather maps 4 rows per lane");
    static_assert(FWD || !GATHER, "the gather completes on each CTA's own barriers");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    CtrlBlock* ctl = reinterpret_cast<CtrlBlock*>(smem + C::STAGES * C::STAGE);
    volatile int* abort_flag = &ctl->abort;
    Issued is;  // this thread's copies or tcgen05 operations in flight
    uint64_t* pfull = ctl->raw_full;
    auto opA = [&](int s, int m) { return smem + s * C::STAGE + m * C::A_BYTES; };
    auto opB = [&](int s) { return smem + s * C::STAGE + C::NB * C::A_BYTES; };
    const int warp = warp_id(), lane = lane_id();
    const int G = a.G, NT = a.NT, KB = a.KB;     // NT: blocks of 256 weight rows
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&ctl->full[s], GATHER ? 33 : 1);
            mbar_init(&ctl->empty[s], 1);
            mbar_init(&pfull[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tfull[b], 1);
            mbar_init(&ctl->tempty[b], 2 * C::EPI_WARPS);
        }
        mbar_init(&ctl->drain[0], 1);
        ctl->abort = 0;
        fence_barrier_init();
    }
    if (threadIdx.x == 32) {
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_w0);
        if (DUAL) tma_prefetch_desc(&tm_w1);
    }
    if (warp == 1) {
        tmem_alloc_pair(&ctl->tmem_slot, C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    pdl_wait();
    if (warp == 0) build_segment_table<BT>(a, ctl, lane);
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers initialised and tensor memory allocated
    tc_fence_after();
    pdl_launch();
    const uint32_t tmem_base = ctl->tmem_slot;
    const int total = ctl->tpre[G];

    if (warp == 0) {
        if (GATHER) {  // ---------------- producer warp: weights by TMA (lane 0), tokens gathered
            const uint64_t pol_w = l2_policy(a.l2_w), pol_t = l2_policy(a.l2_t);
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            const int K = a.K;
            for (int L = pair; L < total && ok; L += npairs) {
                int g, nt, row0, rows;
                decode_tile<BT>(L, ctl, G, NT, g, nt, row0, rows);
                const int trow = row0 + (int)rank * (pair_mma_n(rows, BT) / 2);
                const int wrow = (2 * nt + (int)rank) * kTileN;
                // the tokens of the half's rows lane + 32 i; rows past the GEMM's rows read a
                // valid token (their products are discarded), ids outside [0, gather_rows) too
                int tok[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = min(trow + lane + 32 * i, a.M_alloc - 1);
                    tok[i] = min(max(a.gather_idx[r], 0), a.gather_rows - 1);
                }
                for (int kb = 0; kb < KB; ++kb) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&ctl->empty[s], ph ^ 1u, abort_flag, a.wait_limit))) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&ctl->full[s], C::NB * C::A_BYTES);
                        tma_load_3d_p(opA(s, 0), &tm_w0, &ctl->full[s], kb * kTileK, wrow, g, pol_w);
                        if (DUAL) tma_load_3d_p(opA(s, 1), &tm_w1, &ctl->full[s], kb * kTileK, wrow, g, pol_w);
                    }
                    gather_stage_rows(smem_u32(opB(s)), a.gx, tok, K, kb, lane, pol_t);
                    cp_async_arrive_noinc(&ctl->full[s]);
                    is.mask |= 1u << s;
                    is.par = (is.par & ~(1u << s)) | (ph << s);
                    if (++s == C::STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok && lane == 0) {
                report_error(a.err, MOE_ERR_TIMEOUT, 1);
                ctl->abort = 1;
            }
        } else if (lane == 0) {  // ---------------- producer: this CTA's weight rows and token half
            const uint64_t pol_w = l2_policy(a.l2_w), pol_t = l2_policy(a.l2_t);
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int L = pair; L < total && ok; L += npairs) {
                int g, nt, row0, rows;
                decode_tile<BT>(L, ctl, G, NT, g, nt, row0, rows);
                const int trow = row0 + (int)rank * (pair_mma_n(rows, BT) / 2);
                const int wrow = (2 * nt + (int)rank) * kTileN;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&ctl->empty[s], ph ^ 1u, abort_flag, a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    if (FWD) {
                        mbar_arrive_expect_tx(&ctl->full[s], C::NB * C::A_BYTES + C::B_BYTES);
                        tma_load_3d_p(opA(s, 0), &tm_w0, &ctl->full[s], kb * kTileK, wrow, g, pol_w);
                        if (DUAL) tma_load_3d_p(opA(s, 1), &tm_w1, &ctl->full[s], kb * kTileK, wrow, g, pol_w);
                        tma_load_2d_p(opB(s), &tm_x, &ctl->full[s], kb * kTileK, trow, pol_t);
                    } else {
                        const uint32_t bar = mapa_shared(smem_u32(&ctl->full[s]), 0);  // the leader's
                        if (leader) mbar_arrive_expect_tx(&ctl->full[s], 2 * (C::NB * C::A_BYTES + C::B_BYTES));
                        tma_load_3d_pair(opA(s, 0), &tm_w0, bar, kb * kTileK, wrow, g);
                        if (DUAL) tma_load_3d_pair(opA(s, 1), &tm_w1, bar, kb * kTileK, wrow, g);
                        tma_load_2d_pair(opB(s), &tm_x, bar, kb * kTileK, trow);
                    }
                    is.mask |= 1u << s;
                    is.par = (is.par & ~(1u << s)) | (ph << s);
                    if (++s == C::STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok) {
                report_error(a.err, MOE_ERR_TIMEOUT, 1);
                ctl->abort = 1;
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {  // ---------------- MMA issuer of the pair
            int s = 0, b = 0;
            uint32_t ph = 0, bph = 0;
            bool ok = true;
            for (int L = pair; L < total && ok; L += npairs) {
                int g, nt, row0, rows;
                decode_tile<BT>(L, ctl, G, NT, g, nt, row0, rows);
                const uint32_t idesc = idesc_f16(1, 2 * kTileN, pair_mma_n(rows, BT));
                if (!mbar_wait_cluster(&ctl->tempty[b], bph ^ 1u, abort_flag, a.wait_limit)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d0 = tmem_base + (uint32_t)(b * C::ACC_COLS);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_cluster(&ctl->full[s], ph, abort_flag, a.wait_limit) ||
                        (FWD && !mbar_wait_cluster(&pfull[s], ph, abort_flag, a.wait_limit))) {
                        ok = false;
                        break;
                    }
                    if (GATHER) fence_proxy_async_smem();  // the gathered rows came by the generic proxy
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(opA(s, 0));
                    const uint32_t a1 = smem_u32(opA(s, DUAL ? 1 : 0));
                    const uint32_t bb = smem_u32(opB(s));
#pragma unroll
                    for (int kk = 0; kk < kTileK / 16; ++kk) {
                        const uint64_t bdesc = sw128_kmajor_desc(bb + kk * 32);
                        const uint32_t acc = (kb | kk) != 0;
                        mma_f16_ss_pair(d0, sw128_kmajor_desc(a0 + kk * 32), bdesc, idesc, acc);
                        if (DUAL) mma_f16_ss_pair(d0 + BT, sw128_kmajor_desc(a1 + kk * 32), bdesc, idesc, acc);
                    }
                    is.tc = true;
                    mma_commit_pair(&ctl->empty[s], 0x3);
                    if (++s == C::STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit_pair(&ctl->tfull[b], 0x3);
                if (++b == C::ACC_BUFS) {
                    b = 0;
                    bph ^= 1u;
                }
            }
            if (!ok) {
                report_error(a.err, MOE_ERR_TIMEOUT, 2);
                ctl->abort = 1;
            }
        } else if (FWD && lane == 0) {  // ---------------- peer: tells the leader each stage landed
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int L = pair; L < total && ok; L += npairs) {
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&ctl->full[s], ph, abort_flag, a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    if (GATHER) fence_proxy_async_smem();
                    mbar_arrive_cluster(mapa_shared(smem_u32(&pfull[s]), 0));
                    if (++s == C::STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok) {
                report_error(a.err, MOE_ERR_TIMEOUT, 6);
                ctl->abort = 1;
            }
        }
    } else {
        // ---------------- epilogue (warps 2 .. 2 + 4 EW) of this CTA's 128 weight rows
        const int q = warp & 3, h = (warp - 2) >> 2;
        int b = 0;
        uint32_t bph = 0;
        for (int L = pair; L < total; L += npairs) {
            int g, nt, row0, rows;
            decode_tile<BT>(L, ctl, G, NT, g, nt, row0, rows);
            if (!mbar_wait(&ctl->tfull[b], bph, abort_flag, a.wait_limit)) {
                if (lane == 0) report_error(a.err, MOE_ERR_TIMEOUT, 3);
                ctl->abort = 1;
                break;
            }
            tc_fence_after();
            const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * C::ACC_COLS);
            auto release = [&] {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&ctl->tempty[b]), 0));
            };
            epilogue_tile<BT, DUAL, OUT, 1, false, C::EW>(a, tb, g, 2 * nt + (int)rank, row0, rows, q, lane, h);
            release();
            if (++b == C::ACC_BUFS) {
                b = 0;
                bph ^= 1u;
            }
        }
        if (a.zero_pad && OUT == OUT_BF16 && h == 0) zero_padding_rows(a, ctl, threadIdx.x - 64);
    }

    // Every CTA lets what it has in flight finish whether or not anything aborted (in a normal
    // run these waits return at once): the producer's copies, and in the leader the pair's MMAs.
    // Then neither CTA's shared or tensor memory is in use by the other, and both free it.
    tc_fence_before();
    __syncthreads();
    {
        int never = 0;
        // FWD = false: only the leader's full barriers track copies (both CTAs'); the peer's
        // copies of a stage the leader never armed are not tracked: after an abort the peer
        // waits about 100 microseconds, far longer than a copy takes, before it can exit
        if (FWD || leader) {
            for (int q = 0; q < C::STAGES; ++q)
                if (is.mask >> q & 1u) mbar_wait(&ctl->full[q], is.par >> q & 1u, &never);
        } else if (is.mask && *abort_flag) {
            const long long t0 = clock64();
            while (clock64() - t0 < 200000) {
            }
        }
        if (is.tc) {
            mma_commit_pair(&ctl->drain[0], 0x1);
            mbar_wait(&ctl->drain[0], 0, &never);
        }
    }
    tc_fence_before();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ FP4 kernel

template <int BT, bool DUAL>
struct Fp4Cfg {
    static constexpr int NB = DUAL ? 2 : 1;
    static constexpr int KS = kFp4StageK;                    // 128 K values per stage
    static constexpr int BOX_BYTES = BT * kTileK * 2;        // one 64-K token box, f16
    static constexpr int B_BYTES = 2 * BOX_BYTES;            // token tile of a stage
    static constexpr int S = 4;                              // e4m3 scale bytes per row per 64 K
    static constexpr int CHUNK = kTileN * 32 + kTileN * S;   // prepared 128 x 64 chunk
    static constexpr int RAW_M = 2 * CHUNK;                  // one matrix's raw bytes per stage
    static constexpr int RAW_STAGE = round1024(B_BYTES + NB * RAW_M);
    static constexpr int RSTAGES = cmin(kMaxStages, kSmemBudget / RAW_STAGE);
    // MMA-issuing threads. A 128 x N x 16 MMA costs an issuing thread ~45 cycles for any
    // N <= 64, so narrow token tiles are issue-bound with one issuer; four issuers (each
    // with its own partial accumulator: matrix x K-half, or K-quarter for one matrix)
    // reach the tensor pipe's rate. Wide tiles (N = 128) run at full rate with one.
    static constexpr int NI = BT <= 64 ? 4 : 1;
    static constexpr int NPART = NI == 1 ? 1 : (DUAL ? 2 : 4);  // partial sums per matrix
    // TMEM: accumulators [ACC_BUFS x ACC_COLS] then the weight ring [A_STAGES x NB x 64 cols]
    static constexpr int ACC_COLS = NB * NPART * BT;
    static constexpr int ACC_BUFS = 2 * ACC_COLS <= 256 ? 2 : 1;
    static constexpr int A_COLS = KS / 2;                    // 128 rows x 128 f16 = 64 columns
    static constexpr int A_BASE = ACC_BUFS * ACC_COLS;
    static constexpr int A_STAGES = cmin(8, (512 - A_BASE) / (NB * A_COLS));
    static constexpr int CONV_WARPS = 16;
    // warps: 0 producer, [1, 1+NI) issuers, then 4 epilogue, then the converters
    static constexpr int EPI_WARP0 = 1 + NI;
    static constexpr int CONV_WARP0 = EPI_WARP0 + 4;
    static constexpr int THREADS = (CONV_WARP0 + CONV_WARPS) * 32;
    static constexpr int SMEM_BYTES = 1024 + RSTAGES * RAW_STAGE + kCtrlBytes;
    static_assert(RSTAGES >= 2 && A_STAGES >= 2 && SMEM_BYTES <= kSmemLimit, "FP4 GEMM config");
    static_assert(RSTAGES > A_STAGES, "TMEM slot reuse is read from the raw ring's barriers");
    static_assert(BT % 16 == 0 && BT >= 16 && BT <= 256, "MMA N for M=128 is a multiple of 16 in [16,256]");
    static_assert(BOX_BYTES % 1024 == 0, "token boxes must stay 1024-byte aligned");
};

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}
// 8 packed e2m1 values (one 32-bit word, even k in the low nibble) -> 4 x f16x2, times a scale.
__device__ __forceinline__ void e2m1x8_to_f16(uint32_t w, uint32_t sc2, uint32_t* o) {
    uint32_t o0, o1, o2, o3;
    asm("{ .reg .b8 b0,b1,b2,b3; mov.b32 {b0,b1,b2,b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0; cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2; cvt.rn.f16x2.e2m1x2 %3, b3; }"
        : "=r"(o0), "=r"(o1), "=r"(o2), "=r"(o3)
        : "r"(w));
    o[0] = hmul2_u32(o0, sc2);
    o[1] = hmul2_u32(o1, sc2);
    o[2] = hmul2_u32(o2, sc2);
    o[3] = hmul2_u32(o3, sc2);
}
// f16x2 holding `bits` in both halves
__device__ __forceinline__ uint32_t dup16(uint32_t bits) { return (bits & 0xFFFFu) | (bits << 16); }

// One weight row's 64 K values of one prepared NVFP4 chunk -> 32 f16x2 words (e2m1 times
// its e4m3 block scale; exact in f16).
__device__ __forceinline__ void convert_chunk_row(const uint8_t* chunk, int row, uint32_t (&o)[32]) {
    const uint4 v0 = *reinterpret_cast<const uint4*>(chunk + row * 32);
    const uint4 v1 = *reinterpret_cast<const uint4*>(chunk + row * 32 + 16);
    const uint32_t four = *reinterpret_cast<const uint32_t*>(chunk + kTileN * 32 + row * 4);
    uint32_t s01, s23, sc[4];
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(s01) : "h"((uint16_t)(four & 0xFFFF)));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(s23) : "h"((uint16_t)(four >> 16)));
    sc[0] = dup16(s01);
    sc[1] = dup16(s01 >> 16);
    sc[2] = dup16(s23);
    sc[3] = dup16(s23 >> 16);
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) e2m1x8_to_f16(w[i], sc[i >> 1], o + 4 * i);
}

// Half of it: the 32 values [32h, 32h+32) of the chunk row -> 16 f16x2 words.
__device__ __forceinline__ void convert_half_chunk_row(const uint8_t* chunk, int row, int h, uint32_t (&o)[16]) {
    const uint4 v = *reinterpret_cast<const uint4*>(chunk + row * 32 + h * 16);
    const uint16_t pair = *reinterpret_cast<const uint16_t*>(chunk + kTileN * 32 + row * 4 + 2 * h);
    uint32_t s01, sc[2];
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(s01) : "h"(pair));
    sc[0] = dup16(s01);
    sc[1] = dup16(s01 >> 16);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) e2m1x8_to_f16(w[i], sc[i >> 1], o + 4 * i);
}

template <int BT, bool DUAL, int OUT>
__global__ void __launch_bounds__(Fp4Cfg<BT, DUAL>::THREADS, 1)
    grouped_gemm_fp4_kernel(const __grid_constant__ CUtensorMap tm_x, const GemmArgs a) {
    using C = Fp4Cfg<BT, DUAL>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    CtrlBlock* ctl = reinterpret_cast<CtrlBlock*>(smem + C::RSTAGES * C::RAW_STAGE);
    volatile int* abort_flag = &ctl->abort;
    Issued is;  // this thread's copies or tcgen05 operations in flight
    // raw stage r: [token box 0][token box 1][matrix 0: chunk kb, chunk kb+1][matrix 1: ...]
    auto rawB = [&](int r) { return smem + r * C::RAW_STAGE; };
    auto rawM = [&](int r, int m) { return smem + r * C::RAW_STAGE + C::B_BYTES + m * C::RAW_M; };
    const int warp = warp_id(), lane = lane_id();
    const int G = a.G, NT = a.NT, KB = a.KB;   // KB: stages of 128 K per tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::A_STAGES; ++s) {
            mbar_init(&ctl->full[s], C::CONV_WARPS);
            mbar_init(&ctl->empty[s], C::NI);       // every issuer commits once per stage
        }
        for (int r = 0; r < C::RSTAGES; ++r) {
            mbar_init(&ctl->raw_full[r], 1);
            mbar_init(&ctl->raw_empty[r], C::NI);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tfull[b], C::NI);
            mbar_init(&ctl->tempty[b], 4);
        }
        for (int i = 0; i < 4; ++i) mbar_init(&ctl->drain[i], 1);
        ctl->abort = 0;
        fence_barrier_init();
    }
    if (threadIdx.x == 0) tma_prefetch_desc(&tm_x);
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_slot, 512);
        tmem_relinquish();
    }
    pdl_wait();
    if (warp == 0) build_segment_table<BT>(a, ctl, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch();
    const uint32_t tmem_base = ctl->tmem_slot;
    const int total = ctl->tpre[G];

    if (warp == 0) {
        if (lane == 0) {  // ---------------- producer: two token boxes (TMA) + one copy per matrix
            const uint64_t pol_w = l2_policy(a.l2_w), pol_t = l2_policy(a.l2_t);
            int r = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
                int g, nt, row0, rows;
                decode_tile<BT>(L, ctl, G, NT, g, nt, row0, rows);
                const size_t chunk0 = ((size_t)g * NT + nt) * (2 * KB);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&ctl->raw_empty[r], ph ^ 1u, abort_flag, a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&ctl->raw_full[r], C::B_BYTES + C::NB * C::RAW_M);
                    const size_t off = (chunk0 + 2 * kb) * C::CHUNK;
                    bulk_load_p(rawM(r, 0), a.kd0 + off, C::RAW_M, &ctl->raw_full[r], pol_w);
                    if (DUAL) bulk_load_p(rawM(r, 1), a.kd1 + off, C::RAW_M, &ctl->raw_full[r], pol_w);
                    if (a.x3d) {  // both 64-K boxes of the token tile in one copy: {64, rows, chunks}
                        tma_load_3d_p(rawB(r), &tm_x, &ctl->raw_full[r], 0, row0, 2 * kb, pol_t);
                    } else {
                        tma_load_2d_p(rawB(r), &tm_x, &ctl->raw_full[r], kb * C::KS, row0, pol_t);
                        tma_load_2d_p(rawB(r) + C::BOX_BYTES, &tm_x, &ctl->raw_full[r], kb * C::KS + kTileK, row0, pol_t);
                    }
                    is.mask |= 1u << r;
                    is.par = (is.par & ~(1u << r)) | (ph << r);
                    if (++r == C::RSTAGES) {
                        r = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok) {
                report_error(a.err, MOE_ERR_TIMEOUT, 1);
                ctl->abort = 1;
            }
        }
    } else if (warp < C::EPI_WARP0) {
        if (lane == 0) {  // ---------------- MMA issuers: A from TMEM, B (tokens) from smem
            // A stage: matrix m at columns (s*NB + m)*64, K step kk (0..7) at +8*kk.
            // B: K step kk in token box kk/4 at byte offset (kk%4)*32.
            // Issuer i with NI == 4: two matrices -> matrix i&1, K steps 4(i>>1)..+3,
            // partial i>>1; one matrix -> K steps 2i, 2i+1, partial i. Partial p of matrix m
            // at column (p*NB + m)*BT of the accumulator buffer.
            const int i = warp - 1;
            constexpr uint32_t idesc = idesc_f16(0, kTileN, BT);
            constexpr int KSTEPS = C::KS / 16;
            constexpr int KPI = C::NI == 1 ? KSTEPS : (DUAL ? KSTEPS / 2 : KSTEPS / 4);
            const int m_i = (C::NI == 1 || !DUAL) ? 0 : (i & 1);
            const int p_i = C::NI == 1 ? 0 : (DUAL ? (i >> 1) : i);
            const int kk0 = p_i * KPI;
            int s = 0, r = 0, b = 0;
            uint32_t ph = 0, rph = 0, bph = 0;
            bool ok = true;
            for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
                if (!mbar_wait(&ctl->tempty[b], bph ^ 1u, abort_flag, a.wait_limit)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d0 = tmem_base + (uint32_t)(b * C::ACC_COLS);
                for (int kb = 0; kb < KB; ++kb) {
                    // the converters arrive on full[s] only after they saw raw stage r land, so
                    // this one wait also orders the token tile before the MMA
                    if (!mbar_wait(&ctl->full[s], ph, abort_flag, a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t bb = smem_u32(rawB(r));
                    const uint32_t a0 = tmem_base + (uint32_t)(C::A_BASE + (s * C::NB) * C::A_COLS);
                    auto bdesc = [&](int kk) {
                        return sw128_kmajor_desc(bb + (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32);
                    };
                    if (C::NI == 1) {
#pragma unroll
                        for (int kk = 0; kk < KSTEPS; ++kk) {
                            const uint32_t acc = (kb | kk) != 0;
                            mma_f16_ts(d0, a0 + kk * 8, bdesc(kk), idesc, acc);
                            if (DUAL) mma_f16_ts(d0 + BT, a0 + C::A_COLS + kk * 8, bdesc(kk), idesc, acc);
                        }
                    } else {
                        const uint32_t dm = d0 + (uint32_t)((p_i * C::NB + m_i) * BT);
#pragma unroll
                        for (int j = 0; j < KPI; ++j) {
                            const int kk = kk0 + j;
                            mma_f16_ts(dm, a0 + m_i * C::A_COLS + kk * 8, bdesc(kk), idesc,
                                       (kb > 0 || j > 0) ? 1u : 0u);
                        }
                    }
                    is.tc = true;
                    // one commit per stage: it frees raw stage r and, for the converters, the
                    // TMEM weight slot of this stage
                    mma_commit(&ctl->raw_empty[r]);
                    if (++s == C::A_STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                    if (++r == C::RSTAGES) {
                        r = 0;
                        rph ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(&ctl->tfull[b]);
                if (++b == C::ACC_BUFS) {
                    b = 0;
                    bph ^= 1u;
                }
            }
            if (!ok) {
                report_error(a.err, MOE_ERR_TIMEOUT, 2);
                ctl->abort = 1;
            }
        }
    } else if (warp < C::CONV_WARP0) {
        // ---------------- epilogue (4 warps)
        const int q = warp & 3;
        int b = 0;
        uint32_t bph = 0;
        for (int L = blockIdx.x; L < total; L += gridDim.x) {
            int g, nt, row0, rows;
            decode_tile<BT>(L, ctl, G, NT, g, nt, row0, rows);
            if (!mbar_wait(&ctl->tfull[b], bph, abort_flag, a.wait_limit)) {
                if (lane == 0) report_error(a.err, MOE_ERR_TIMEOUT, 3);
                ctl->abort = 1;
                break;
            }
            tc_fence_after();
            epilogue_tile<BT, DUAL, OUT, C::NPART>(
                a, tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * C::ACC_COLS), g, nt, row0, rows, q, lane);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->tempty[b]);
            if (++b == C::ACC_BUFS) {
                b = 0;
                bph ^= 1u;
            }
        }
        if (a.zero_pad && OUT == OUT_BF16) zero_padding_rows(a, ctl, threadIdx.x - 32 * C::EPI_WARP0);
    } else {
        // ---------------- converters (16 warps): e2m1 x block scale -> f16 rows in TMEM.
        // Warp w owns TMEM lanes [32q, 32q+32), q = w % 4, so thread `lane` converts weight
        // row 32q + lane; the four warps of a quarter split a stage's row into four units
        // (two matrices x two 64-K chunks, or two chunks x two halves).
        const int q = warp & 3, grp = (warp - C::CONV_WARP0) >> 2;
        const int row = q * 32 + lane;
        const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
        int s = 0, r = 0;
        uint32_t ph = 0, rph = 0;
        long long it = 0;  // stages converted so far
        bool ok = true;
        for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
            for (int kb = 0; kb < KB; ++kb, ++it) {
                // The TMEM weight slot s is free once the MMAs of stage it - A_STAGES are done,
                // which the issuers' commit on that stage's raw barrier records. That barrier
                // cannot run a phase ahead: it would need stage it - A_STAGES + RSTAGES > it.
                bool got = mbar_wait(&ctl->raw_full[r], rph, abort_flag, a.wait_limit);
                if (got && it >= C::A_STAGES) {
                    const long long j = it - C::A_STAGES;
                    got = mbar_wait(&ctl->raw_empty[j % C::RSTAGES], (uint32_t)((j / C::RSTAGES) & 1), abort_flag, a.wait_limit);
                }
                if (!got) {
                    if (lane == 0) report_error(a.err, MOE_ERR_TIMEOUT, 4);
                    ctl->abort = 1;
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acol = (uint32_t)(C::A_BASE + s * C::NB * C::A_COLS);
                if (DUAL) {  // unit grp: matrix grp>>1, chunk grp&1 (64 values)
                    const int m = grp >> 1, c = grp & 1;
                    uint32_t o[32];
                    convert_chunk_row(rawM(r, m) + c * C::CHUNK, row, o);
                    tmem_st32(lane_base + acol + m * C::A_COLS + c * 32, o);
                } else {     // unit grp: chunk grp>>1, half grp&1 (32 values)
                    const int c = grp >> 1, h = grp & 1;
                    uint32_t o[16];
                    convert_half_chunk_row(rawM(r, 0) + c * C::CHUNK, row, h, o);
                    tmem_st16(lane_base + acol + c * 32 + h * 16, o);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->full[s]);
                if (++s == C::A_STAGES) {
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

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        drain_in_flight(is, ctl->raw_full, C::RSTAGES,
                        warp >= 1 && warp < C::EPI_WARP0 && lane == 0 ? &ctl->drain[warp - 1] : nullptr);
        tc_fence_before();
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

// ------------------------------------------------------------------ block-scaled NVFP4 kernel

template <int BT, bool DUAL>
struct Nvf4Cfg {
    static constexpr int NB = DUAL ? 2 : 1;
    static constexpr int A_BYTES = kNvf4TileBytes;              // codes image + 4 scale blocks
    static constexpr int B_OFF = NB * A_BYTES;                  // token codes: BT rows x 128 bytes
    static constexpr int B_BYTES = BT * kNvf4StageK / 2;
    static constexpr int SFR_OFF = B_OFF + B_BYTES;             // token scales as loaded: BT x 16 bytes
    static constexpr int SFR_BYTES = BT * 16;
    static constexpr int SFB_OFF = SFR_OFF + (SFR_BYTES < 128 ? 128 : SFR_BYTES);  // 4 copy blocks
    static constexpr int STAGE = round1024(SFB_OFF + 4 * 512);
    // TMEM: two accumulator buffers, then one scale-factor slot per pipeline stage (four
    // 4-column groups per matrix, then four for the tokens)
    static constexpr int ACC_COLS = NB * BT;
    static constexpr int SF_BASE = 2 * ACC_COLS;
    static constexpr int SF_SLOT = NB * 16 + 16;
    static constexpr int STAGES = cmin(cmin(kMaxStages, kSmemBudget / STAGE), (512 - SF_BASE) / SF_SLOT);
    static constexpr int TMEM_COLS = tmem_cols_pow2(SF_BASE + STAGES * SF_SLOT);
    static constexpr int THREADS = 7 * 32;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE + kCtrlBytes;
    static_assert(STAGES >= 3 && SMEM_BYTES <= kSmemLimit && SF_BASE + STAGES * SF_SLOT <= 512, "NVFP4 GEMM config");
    static_assert(BT == 16 || BT == 32 || BT == 64 || BT == 128, "token tile");
    static_assert(B_OFF % 1024 == 0 && SFR_OFF % 128 == 0 && SFB_OFF % 128 == 0, "operand alignment");
};

// The token tile's scales arrive as BT rows of 16 bytes (one 32-bit word of four scales
// per 64 K values j). The scale-factor copy wants, per j, a 512-byte block whose byte
// 16*(r % 32) + 4*(r / 32) + i is scale i of row r. Lane l moves rows l, l+32, ...
template <int BT>
__device__ __forceinline__ void build_sfb_blocks(const uint8_t* raw, uint8_t* blk, int lane) {
    constexpr int G32 = BT >= 32 ? BT / 32 : 1;
    if (BT < 32 && lane >= BT) return;
    uint32_t w[G32][4];
#pragma unroll
    for (int m1 = 0; m1 < G32; ++m1) {
        const uint4 v = *reinterpret_cast<const uint4*>(raw + (32 * m1 + lane) * 16);
        w[m1][0] = v.x;
        w[m1][1] = v.y;
        w[m1][2] = v.z;
        w[m1][3] = v.w;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint8_t* d = blk + j * 512 + lane * 16;
        if (G32 == 4) *reinterpret_cast<uint4*>(d) = make_uint4(w[0][j], w[1 % G32][j], w[2 % G32][j], w[3 % G32][j]);
        else if (G32 == 2) *reinterpret_cast<uint2*>(d) = make_uint2(w[0][j], w[1 % G32][j]);
        else *reinterpret_cast<uint32_t*>(d) = w[0][j];
    }
}

// Weights in block-scaled tiles (bulk copies), tokens as packed e2m1 rows plus their
// e4m3 scales (TMA); the tensor cores apply both scales. Warp roles: 0 producer, 1 MMA
// issuer (one thread), 2..5 epilogue, 6 scale warp: it rearranges the token scales and
// one of its threads copies the stage's scale factors into that stage's TMEM slot, so
// the MMA thread issues nothing but MMAs.
template <int BT, bool DUAL, int OUT>
__global__ void __launch_bounds__(Nvf4Cfg<BT, DUAL>::THREADS, 1)
    grouped_gemm_nvf4_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_sf,
                             const GemmArgs a) {
    using C = Nvf4Cfg<BT, DUAL>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    CtrlBlock* ctl = reinterpret_cast<CtrlBlock*>(smem + C::STAGES * C::STAGE);
    volatile int* abort_flag = &ctl->abort;
    Issued is;  // this thread's copies or tcgen05 operations in flight
    auto opA = [&](int s, int m) { return smem + s * C::STAGE + m * C::A_BYTES; };
    auto opB = [&](int s) { return smem + s * C::STAGE + C::B_OFF; };
    auto sfRaw = [&](int s) { return smem + s * C::STAGE + C::SFR_OFF; };
    auto sfBlk = [&](int s) { return smem + s * C::STAGE + C::SFB_OFF; };
    uint64_t* sf_full = ctl->raw_full;   // scale factors of stage s are in TMEM
    const int warp = warp_id(), lane = lane_id();
    const int G = a.G, NT = a.NT, KB = a.KB;   // KB: 256-K stages per tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
            mbar_init(&sf_full[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tfull[b], 1);
            mbar_init(&ctl->tempty[b], 4);
        }
        mbar_init(&ctl->drain[0], 1);
        mbar_init(&ctl->drain[1], 1);
        ctl->abort = 0;
        fence_barrier_init();
    }
    if (threadIdx.x == 32) {
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_sf);
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    pdl_wait();
    if (warp == 0) build_segment_table<BT>(a, ctl, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch();
    const uint32_t tmem_base = ctl->tmem_slot;
    const int total = ctl->tpre[G];
    // scale-factor slot of stage s: matrix m's 64-K block j at + m*16 + 4j, tokens' at + NB*16 + 4j
    auto sf_slot = [&](int s) { return tmem_base + (uint32_t)(C::SF_BASE + s * C::SF_SLOT); };

    if (warp == 0) {
        if (lane == 0) {  // ---------------- producer
            const uint64_t pol_w = l2_policy(a.l2_w), pol_t = l2_policy(a.l2_t);
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
                int g, nt, row0, rows;
                decode_tile<BT>(L, ctl, G, NT, g, nt, row0, rows);
                const size_t tile0 = ((size_t)g * NT + nt) * KB;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&ctl->empty[s], ph ^ 1u, abort_flag, a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&ctl->full[s], C::NB * C::A_BYTES + C::B_BYTES + C::SFR_BYTES);
                    const size_t off = (tile0 + kb) * (size_t)kNvf4TileBytes;
                    bulk_load_p(opA(s, 0), a.ks0 + off, kNvf4TileBytes, &ctl->full[s], pol_w);
                    if (DUAL) bulk_load_p(opA(s, 1), a.ks1 + off, kNvf4TileBytes, &ctl->full[s], pol_w);
                    tma_load_2d_p(opB(s), &tm_x, &ctl->full[s], kb * (kNvf4StageK / 2), row0, pol_t);
                    tma_load_2d_p(sfRaw(s), &tm_sf, &ctl->full[s], kb * (kNvf4StageK / 16), row0, pol_t);
                    is.mask |= 1u << s;
                    is.par = (is.par & ~(1u << s)) | (ph << s);
                    if (++s == C::STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok) {
                report_error(a.err, MOE_ERR_TIMEOUT, 1);
                ctl->abort = 1;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {  // ---------------- MMA issuer
            constexpr uint32_t idesc = idesc_nvf4(kTileN, BT);
            int s = 0, b = 0;
            uint32_t ph = 0, bph = 0;
            bool ok = true;
            for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
                if (!mbar_wait(&ctl->tempty[b], bph ^ 1u, abort_flag, a.wait_limit)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d0 = tmem_base + (uint32_t)(b * C::ACC_COLS);
                for (int kb = 0; kb < KB; ++kb) {
                    // operands landed (full) and their scale factors are in TMEM (sf_full)
                    if (!mbar_wait(&ctl->full[s], ph, abort_flag, a.wait_limit) || !mbar_wait(&sf_full[s], ph, abort_flag, a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t bb = smem_u32(opB(s));
                    const uint32_t sfs = sf_slot(s);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint64_t bdesc = sw128_kmajor_desc(bb + 32 * j);
                        const uint32_t acc = (kb | j) != 0;
#pragma unroll
                        for (int m = 0; m < C::NB; ++m)
                            mma_nvf4_ss(d0 + m * BT, sw128_kmajor_desc(smem_u32(opA(s, m)) + 32 * j), bdesc, idesc,
                                        sfs + m * 16 + 4 * j, sfs + C::NB * 16 + 4 * j, acc);
                    }
                    is.tc = true;
                    mma_commit(&ctl->empty[s]);
                    if (++s == C::STAGES) {
                        s = 0;
                        ph ^= 1u;
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
            }
        }
    } else if (warp == 6) {
        // ---------------- scale warp: token scales -> copy blocks (all lanes), then lane 0
        // copies the weights' and the tokens' scale blocks into the stage's TMEM slot. The
        // slot is free: the stage's previous MMAs completed before the producer refilled it.
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
            for (int kb = 0; kb < KB; ++kb) {
                if (!__all_sync(0xffffffffu, mbar_wait(&ctl->full[s], ph, abort_flag, a.wait_limit))) {
                    ok = false;
                    break;
                }
                build_sfb_blocks<BT>(sfRaw(s), sfBlk(s), lane);
                fence_proxy_async_smem();  // the copies read these bytes through the async proxy
                __syncwarp();
                if (lane == 0) {
                    tc_fence_after();
                    const uint32_t sfs = sf_slot(s);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
#pragma unroll
                        for (int m = 0; m < C::NB; ++m)
                            tmem_cp_32x128b_x4(sfs + m * 16 + 4 * j,
                                               sf_block_desc(smem_u32(opA(s, m)) + kNvf4CodeBytes + 512 * j));
                        tmem_cp_32x128b_x4(sfs + C::NB * 16 + 4 * j, sf_block_desc(smem_u32(sfBlk(s)) + 512 * j));
                    }
                    mma_commit(&sf_full[s]);
                }
                __syncwarp();
                is.tc = true;
                if (++s == C::STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {
            report_error(a.err, MOE_ERR_TIMEOUT, 5);
            ctl->abort = 1;
        }
    } else {
        // ---------------- epilogue (warps 2..5)
        const int q = warp & 3;
        int b = 0;
        uint32_t bph = 0;
        for (int L = blockIdx.x; L < total; L += gridDim.x) {
            int g, nt, row0, rows;
            decode_tile<BT>(L, ctl, G, NT, g, nt, row0, rows);
            if (!mbar_wait(&ctl->tfull[b], bph, abort_flag, a.wait_limit)) {
                if (lane == 0) report_error(a.err, MOE_ERR_TIMEOUT, 3);
                ctl->abort = 1;
                break;
            }
            tc_fence_after();
            epilogue_tile<BT, DUAL, OUT>(a, tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * C::ACC_COLS), g,
                                         nt, row0, rows, q, lane);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->tempty[b]);
            b ^= 1;
            if (b == 0) bph ^= 1u;
        }
        if (a.zero_pad && OUT == OUT_BF16) zero_padding_rows(a, ctl, threadIdx.x - 64);
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        drain_in_flight(is, ctl->full, C::STAGES,
                        lane != 0 ? nullptr : warp == 1 ? &ctl->drain[0] : warp == 6 ? &ctl->drain[1] : nullptr);
        tc_fence_before();
        __syncthreads();
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ MXFP4 x MXFP8 kernel

template <int BT, bool DUAL, bool TWO>
struct Mx8Cfg {
    static constexpr int NB = DUAL ? 2 : 1;
    // TWO: the activations are two e4m3 terms (hi/lo staging of bf16); else one (MXFP8).
    // The hi and lo token rows sit one after the other in shared memory, so while the
    // accumulators fit, one MMA of N = 2*BT covers both terms (MERGE): half the MMAs, and
    // the weight tile is read once for both. Its two column halves are partial sums the
    // epilogue adds. Otherwise (two 128-token tiles) each term is its own MMA.
    static constexpr bool MERGE = TWO && NB * 2 * BT <= 256;
    static constexpr int TERMS = MERGE ? 2 : 1;            // partials one MMA writes side by side
    // A thread issues a block-scaled MMA about every 145 cycles, so narrow tiles split each
    // stage's four K steps between two issuers with their own partial sums where TMEM allows.
    static constexpr int KSPLIT = NB * TERMS * 2 * BT <= 128 ? 2 : 1;
    static constexpr int NPART = TERMS * KSPLIT;
    static constexpr int NI = NB * KSPLIT;                 // issuer i: matrix i % NB, K half i / NB
    static constexpr int N_MMA = TERMS * BT;
    static constexpr int A_BYTES = kTileN * kMx8StageK;   // 128 rows x 128 e2m1, a byte each in smem
    static constexpr int A_TX = A_BYTES / 2;              // what the 4-bit load counts: the packed bytes
    static constexpr int B_BYTES = BT * kMx8StageK;       // one e4m3 term
    static constexpr int BH_OFF = NB * A_BYTES;
    static constexpr int BL_OFF = BH_OFF + B_BYTES;
    static constexpr int SFA_OFF = BH_OFF + (TWO ? 2 : 1) * B_BYTES;  // one 512-byte block per matrix
    static constexpr int SFR_OFF = SFA_OFF + NB * 512;     // token scales as loaded: BT x 16 bytes
    static constexpr int SFR_BYTES = BT * 16;
    static constexpr int SFB_OFF = SFR_OFF + (SFR_BYTES < 128 ? 128 : SFR_BYTES);
    static constexpr int STAGE = round1024(SFB_OFF + 512);
    static constexpr int ACC_COLS = NB * NPART * BT;
    static constexpr int SFB_COLS = N_MMA > 128 ? 8 : 4;  // token scales: 4 columns per 128 MMA rows
    static constexpr int SF_SLOT = 4 * NB + SFB_COLS;
    static constexpr int ACC_BUFS = 2 * ACC_COLS + 3 * SF_SLOT <= 512 ? 2 : 1;
    static constexpr int SF_BASE = ACC_BUFS * ACC_COLS;
    static constexpr int STAGES = cmin(cmin(kMaxStages, kSmemBudget / STAGE), (512 - SF_BASE) / SF_SLOT);
    static constexpr int TMEM_COLS = tmem_cols_pow2(SF_BASE + STAGES * SF_SLOT);
    // Epilogue warps per TMEM lane quarter. With one accumulator buffer the MMAs wait for
    // the epilogue, whose instruction chains are latency-bound: four warps per quarter
    // (the MXFP4 prefill gate/up GEMM measured about 1.1 ms with two, 0.8 with four), else two.
    static constexpr int EW = ACC_BUFS == 1 ? 4 : 2;
    static constexpr int EPI_WARP0 = 1 + NI;
    static constexpr int SCALE_WARP = EPI_WARP0 + 4 * EW;
    static constexpr int THREADS = (SCALE_WARP + 1) * 32;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE + kCtrlBytes;
    static_assert(STAGES >= 3 && SMEM_BYTES <= kSmemLimit && SF_BASE + STAGES * SF_SLOT <= 512, "MX GEMM config");
    static_assert(BT == 16 || BT == 32 || BT == 64 || BT == 128, "token tile");
    static_assert(BH_OFF % 1024 == 0 && BL_OFF % 1024 == 0 && SFR_OFF % 128 == 0 && SFB_OFF % 128 == 0,
                  "operand alignment");
    static_assert(KSPLIT == 1 || MERGE || !TWO, "split K steps only with merged or single terms");
};

// The token tile's scales arrive as BT rows of 16 bytes covering 512 K values; word w of
// a row holds the four scales of this stage's 128 values. The copy block wants byte
// 16*(r % 32) + 4*(r / 32) + i = scale i of MMA row r, and MMA row r is token r % BT
// (rows [BT, 2BT) are the lo terms of the same tokens when the terms are merged).
template <int BT, bool MERGE>
__device__ __forceinline__ void build_sfb_block_mx8(const uint8_t* raw, uint8_t* blk, int w, int lane) {
    constexpr int R = MERGE ? (2 * BT < 128 ? 2 * BT : 128) : BT;  // rows one copy block covers
    const uint32_t* rw = reinterpret_cast<const uint32_t*>(raw);
    auto word = [&](int r) { return rw[(r % BT) * 4 + w]; };
    uint8_t* d = blk + lane * 16;
    if (R <= 32) {
        if (lane < R) *reinterpret_cast<uint32_t*>(d) = word(lane);
    } else if (R == 64) {
        *reinterpret_cast<uint2*>(d) = make_uint2(word(lane), word(lane + 32));
    } else {
        *reinterpret_cast<uint4*>(d) = make_uint4(word(lane), word(lane + 32), word(lane + 64), word(lane + 96));
    }
}

// MXFP4 weights (4-bit tensor map, expanded to a byte per value in smem, plus their
// e8m0 scale blocks) against MXFP8 activations given as two e4m3 terms that share one
// e8m0 scale per 32 values; the tensor cores apply both scales. Warp roles: 0 producer,
// 1..NI MMA issuers, then 4 epilogue warps, then the scale warp (token scales into copy
// blocks, scale-factor copies into the stage's TMEM slot).
// WIDE (single matrix): a tile is two consecutive 128-row weight blocks, handled like the
// gate/up pair (two weight tiles per stage), so a stage of a decode tile streams as many
// weight bytes per fixed per-stage cost as the pair does; the epilogue writes both blocks.
template <int BT, bool DUAL, bool TWO, int OUT, bool WIDE = false>
__global__ void __launch_bounds__(Mx8Cfg<BT, DUAL || WIDE, TWO>::THREADS, 1)
    grouped_gemm_mx8_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_sf,
                            const __grid_constant__ CUtensorMap tm_w0, const __grid_constant__ CUtensorMap tm_w1,
                            const GemmArgs a, int Kp) {
    static_assert(!(DUAL && WIDE), "WIDE is a single-matrix mode");
    using C = Mx8Cfg<BT, DUAL || WIDE, TWO>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    CtrlBlock* ctl = reinterpret_cast<CtrlBlock*>(smem + C::STAGES * C::STAGE);
    volatile int* abort_flag = &ctl->abort;
    Issued is;  // this thread's copies or tcgen05 operations in flight
    auto opA = [&](int s, int m) { return smem + s * C::STAGE + m * C::A_BYTES; };
    auto opB = [&](int s, int t) { return smem + s * C::STAGE + (t ? C::BL_OFF : C::BH_OFF); };
    auto sfA = [&](int s, int m) { return smem + s * C::STAGE + C::SFA_OFF + m * 512; };
    auto sfRaw = [&](int s) { return smem + s * C::STAGE + C::SFR_OFF; };
    auto sfBlk = [&](int s) { return smem + s * C::STAGE + C::SFB_OFF; };
    uint64_t* sf_full = ctl->raw_full;
    const int warp = warp_id(), lane = lane_id();
    const int G = a.G, NT = a.NT, KB = a.KB;   // KB: 128-K stages per tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], C::NI);
            mbar_init(&sf_full[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tfull[b], C::NI);
            mbar_init(&ctl->tempty[b], 4 * C::EW);
        }
        for (int i = 0; i < 6; ++i) mbar_init(&ctl->drain[i], 1);
        ctl->abort = 0;
        fence_barrier_init();
    }
    if (threadIdx.x == 32) {
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_sf);
        tma_prefetch_desc(&tm_w0);
        if (DUAL) tma_prefetch_desc(&tm_w1);
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    pdl_wait();
    if (warp == 0) build_segment_table<BT>(a, ctl, lane);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_launch();
    const uint32_t tmem_base = ctl->tmem_slot;
    const int total = ctl->tpre[G];
    // scale-factor slot of stage s: matrix m's block at + 4m, the tokens' at + 4 NB
    auto sf_slot = [&](int s) { return tmem_base + (uint32_t)(C::SF_BASE + s * C::SF_SLOT); };

    if (warp == 0) {
        if (lane == 0) {  // ---------------- producer
            const uint64_t pol_w = l2_policy(a.l2_w), pol_t = l2_policy(a.l2_t);
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
                int g, nt, row0, rows;
                decode_tile<BT>(L, ctl, G, NT, g, nt, row0, rows);
                // 128-row weight blocks of this tile: nt (and nt for up), or 2nt and 2nt + 1.
                // A second block past the last one is zero-filled by the tensor map; its
                // scale copy repeats the last block's (times zero weights: no effect).
                const int NT1 = WIDE ? (a.N + kTileN - 1) / kTileN : NT;
                const int wb0 = WIDE ? 2 * nt : nt, wb1 = WIDE ? 2 * nt + 1 : nt;
                const size_t blk0 = ((size_t)g * NT1 + wb0) * KB;
                const size_t blk1 = ((size_t)g * NT1 + min(wb1, NT1 - 1)) * KB;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&ctl->empty[s], ph ^ 1u, abort_flag, a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&ctl->full[s],
                                          C::NB * (C::A_TX + 512) + (TWO ? 2 : 1) * C::B_BYTES + C::SFR_BYTES);
                    tma_load_3d_p(opA(s, 0), &tm_w0, &ctl->full[s], kb * kMx8StageK, wb0 * kTileN, g, pol_w);
                    bulk_load_p(sfA(s, 0), a.ks0 + (blk0 + kb) * 512, 512, &ctl->full[s], pol_w);
                    if (DUAL || WIDE) {
                        tma_load_3d_p(opA(s, 1), &tm_w1, &ctl->full[s], kb * kMx8StageK, wb1 * kTileN, g, pol_w);
                        bulk_load_p(sfA(s, 1), a.ks1 + (blk1 + kb) * 512, 512, &ctl->full[s], pol_w);
                    }
                    tma_load_2d_p(opB(s, 0), &tm_x, &ctl->full[s], kb * kMx8StageK, row0, pol_t);
                    if (TWO) tma_load_2d_p(opB(s, 1), &tm_x, &ctl->full[s], Kp + kb * kMx8StageK, row0, pol_t);
                    tma_load_2d_p(sfRaw(s), &tm_sf, &ctl->full[s], (kb >> 2) * 16, row0, pol_t);
                    is.mask |= 1u << s;
                    is.par = (is.par & ~(1u << s)) | (ph << s);
                    if (++s == C::STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok) {
                report_error(a.err, MOE_ERR_TIMEOUT, 1);
                ctl->abort = 1;
            }
        }
    } else if (warp < C::EPI_WARP0) {
        if (lane == 0) {  // ---------------- MMA issuers
            const int i = warp - 1;
            const int m = i % C::NB, kh = i / C::NB;
            constexpr int KPI = (kMx8StageK / 32) / C::KSPLIT;  // K steps per issuer and stage
            int s = 0, b = 0;
            uint32_t ph = 0, bph = 0;
            bool ok = true;
            for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
                if (!mbar_wait(&ctl->tempty[b], bph ^ 1u, abort_flag, a.wait_limit)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(b * C::ACC_COLS + (m * C::NPART + kh * C::TERMS) * BT);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&ctl->full[s], ph, abort_flag, a.wait_limit) || !mbar_wait(&sf_full[s], ph, abort_flag, a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t aa = smem_u32(opA(s, m));
                    const uint32_t sfa = sf_slot(s) + 4 * m, sfb = sf_slot(s) + 4 * C::NB;
#pragma unroll
                    for (int j = 0; j < KPI; ++j) {
                        const int kk = kh * KPI + j;
                        const uint64_t adesc = sw128_kmajor_desc(aa + 32 * kk);
                        const uint32_t id = (uint32_t)kk, idb = id << 30;
                        if (C::MERGE || !TWO) {  // one MMA; merged: hi and lo partials at d and d + BT
                            mma_mx8_ss(d, adesc, sw128_kmajor_desc(smem_u32(opB(s, 0)) + 32 * kk),
                                       idesc_mx8(kTileN, C::N_MMA, id), sfa | idb, sfb | idb, (kb | j) != 0);
                        } else {
#pragma unroll
                            for (int t = 0; t < 2; ++t)
                                mma_mx8_ss(d, adesc, sw128_kmajor_desc(smem_u32(opB(s, t)) + 32 * kk),
                                           idesc_mx8(kTileN, BT, id), sfa | idb, sfb | idb, (kb | j | t) != 0);
                        }
                    }
                    is.tc = true;
                    mma_commit(&ctl->empty[s]);
                    if (++s == C::STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(&ctl->tfull[b]);
                if (++b == C::ACC_BUFS) {
                    b = 0;
                    bph ^= 1u;
                }
            }
            if (!ok) {
                report_error(a.err, MOE_ERR_TIMEOUT, 2);
                ctl->abort = 1;
            }
        }
    } else if (warp == C::SCALE_WARP) {
        // ---------------- scale warp (see the NVFP4 kernel); the slot of stage s is free once
        // the producer refilled s, i.e. after the MMAs that read it completed
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
            for (int kb = 0; kb < KB; ++kb) {
                if (!__all_sync(0xffffffffu, mbar_wait(&ctl->full[s], ph, abort_flag, a.wait_limit))) {
                    ok = false;
                    break;
                }
                build_sfb_block_mx8<BT, C::MERGE>(sfRaw(s), sfBlk(s), kb & 3, lane);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tc_fence_after();
                    const uint32_t sfs = sf_slot(s);
#pragma unroll
                    for (int mm = 0; mm < C::NB; ++mm) tmem_cp_32x128b_x4(sfs + 4 * mm, sf_block_desc(smem_u32(sfA(s, mm))));
                    // MMA rows [128, 256) (the lo terms of a 128-token tile) repeat rows [0, 128)
#pragma unroll
                    for (int h = 0; h < C::SFB_COLS / 4; ++h)
                        tmem_cp_32x128b_x4(sfs + 4 * C::NB + 4 * h, sf_block_desc(smem_u32(sfBlk(s))));
                    mma_commit(&sf_full[s]);
                }
                __syncwarp();
                is.tc = true;
                if (++s == C::STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {
            report_error(a.err, MOE_ERR_TIMEOUT, 5);
            ctl->abort = 1;
        }
    } else {
        // ---------------- epilogue (4 * EW warps)
        const int q = warp & 3, h = (warp - C::EPI_WARP0) >> 2;
        int b = 0;
        uint32_t bph = 0;
        for (int L = blockIdx.x; L < total; L += gridDim.x) {
            int g, nt, row0, rows;
            decode_tile<BT>(L, ctl, G, NT, g, nt, row0, rows);
            if (!mbar_wait(&ctl->tfull[b], bph, abort_flag, a.wait_limit)) {
                if (lane == 0) report_error(a.err, MOE_ERR_TIMEOUT, 3);
                ctl->abort = 1;
                break;
            }
            tc_fence_after();
            const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * C::ACC_COLS);
            auto release = [&] {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->tempty[b]);
            };
            if constexpr (WIDE) {  // block 2nt, then block 2nt + 1 (its partials NPART * BT columns on)
                epilogue_tile<BT, false, OUT, C::NPART, true, C::EW>(a, tb, g, 2 * nt, row0, rows, q, lane, h);
                epilogue_tile<BT, false, OUT, C::NPART, true, C::EW>(a, tb + C::NPART * BT, g, 2 * nt + 1, row0, rows,
                                                                     q, lane, h);
                release();
            } else if constexpr (DUAL && C::ACC_BUFS == 1 && OUT == OUT_MX8) {
                epilogue_tile_mx8_staged<BT, C::NPART, true, C::EW>(a, tb, g, nt, row0, rows, q, lane, h, release);
            } else {
                epilogue_tile<BT, DUAL, OUT, C::NPART, true, C::EW>(a, tb, g, nt, row0, rows, q, lane, h);
                release();
            }
            if (++b == C::ACC_BUFS) {
                b = 0;
                bph ^= 1u;
            }
        }
        if (a.zero_pad && OUT == OUT_BF16 && h == 0) zero_padding_rows(a, ctl, threadIdx.x - 32 * C::EPI_WARP0);
    }

    tc_fence_before();
    __syncthreads();
    if (*abort_flag) {
        drain_in_flight(is, ctl->full, C::STAGES,
                        lane != 0                         ? nullptr
                        : warp >= 1 && warp < C::EPI_WARP0 ? &ctl->drain[warp - 1]
                        : warp == C::SCALE_WARP           ? &ctl->drain[5]
                                                          : nullptr);
        tc_fence_before();
        __syncthreads();
    }
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

// A row-major [rows, K] matrix of 16-bit elements seen as {64 columns, rows, K/64 chunks}
// (chunk stride 128 bytes); box = 64 x box_rows x 2 lands as two consecutive 64-column
// boxes, i.e. a 128-K token tile in one copy. Needs K % 64 == 0 (no column past K is read).
bool make_map_3d_chunks(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, uint64_t K, uint64_t rows,
                        uint32_t box_rows) {
    EncodeTiledFn enc = get_encode();
    if (!enc || K % kTileK) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)kTileK, rows, K / kTileK};
    const cuuint64_t strides[2] = {K * 2, (cuuint64_t)kTileK * 2};
    const cuuint32_t box[3] = {(cuuint32_t)kTileK, box_rows, 2};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
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

// 2-D map over rows of bytes: [rows, cols] with rows `stride` bytes apart; box = box_cols
// bytes x box_rows. Rows and columns past the ends read as zero.
bool make_map_u8(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint64_t stride,
                 uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
    EncodeTiledFn enc = get_encode();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {stride};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over MXFP4 codes [G, N, Kp/2] (packed, 4-bit elements); box = 128 values x
// 128 rows x 1, each 16 values landing in 16 bytes of shared memory (8 bytes of codes,
// then 8 unused) with the 128-byte swizzle. Kp % 128 == 0; rows past N read as zero.
bool make_map_w_u4(CUtensorMap* m, const void* ptr, uint64_t Kp, uint64_t N, uint64_t G) {
    EncodeTiledFn enc = get_encode();
    if (!enc || Kp % 128) return false;
    const cuuint64_t dims[3] = {Kp, N, G};
    const cuuint64_t strides[2] = {Kp / 2, N * Kp / 2};
    const cuuint32_t box[3] = {128, (cuuint32_t)kTileN, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, const_cast<void*>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// `done` belongs to the caller's instantiation: kernels of one signature share a
// function-pointer type, so the flag cannot live in a template on that type.
template <typename Kern>
cudaError_t set_smem_once(Kern kern, int bytes, int (&done)[64]) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!done[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return e;
        done[dev] = 1;
    }
    return cudaSuccess;
}

int grid_for(const GemmProblem& p, const GemmArgs& args, int bt) {
    const long long tiles_ub = ((long long)(p.M_alloc + bt - 1) / bt + p.G) * args.NT;
    return (int)std::max<long long>(1, std::min<long long>(num_sms(), tiles_ub));
}

template <int BT, bool DUAL, int OUT, bool GATHER = false>
cudaError_t run_bf16(const GemmProblem& p, const GemmArgs& args, const CUtensorMap& tx, const CUtensorMap& t0,
                     const CUtensorMap& t1, cudaStream_t st, bool pdl) {
    using C = Bf16Cfg<BT, DUAL>;
    auto kern = grouped_gemm_kernel<BT, DUAL, OUT, GATHER>;
    static int done[64] = {0};
    cudaError_t e = set_smem_once(kern, C::SMEM_BYTES, done);
    if (e != cudaSuccess) return e;
    return launch_k(kern, dim3(grid_for(p, args, BT)), dim3(C::THREADS), (size_t)C::SMEM_BYTES, st, pdl, tx, t0, t1,
                    args);
}

// Pairs that can be resident at once (clusters of two CTAs, one CTA per SM), per device.
template <typename Kern>
int max_pairs_once(Kern kern, int smem, int threads, int (&cache)[64]) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (!cache[dev]) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (num_sms() / 2));
        cfg.blockDim = dim3(threads);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) return 0;
        cache[dev] = n;
    }
    return cache[dev];
}

template <int BT, bool DUAL, int OUT, bool GATHER = false, bool FWD = true>
cudaError_t run_pair(const GemmProblem& p, GemmArgs args, const CUtensorMap& tx, const CUtensorMap& t0,
                     const CUtensorMap& t1, cudaStream_t st, bool pdl) {
    using C = PairCfg<BT, DUAL>;
    auto kern = grouped_gemm_pair_kernel<BT, DUAL, OUT, GATHER, FWD>;
    static int done[64] = {0};
    static int pairs_cache[64] = {0};
    cudaError_t e = set_smem_once(kern, C::SMEM_BYTES, done);
    if (e != cudaSuccess) return e;
    const int maxp = max_pairs_once(kern, C::SMEM_BYTES, C::THREADS, pairs_cache);
    if (maxp < 1) return cudaErrorInvalidConfiguration;
    args.NT = (p.N + 2 * kTileN - 1) / (2 * kTileN);
    const long long tiles_ub = ((long long)(p.M_alloc + BT - 1) / BT + p.G) * args.NT;
    const int pairs = (int)std::max<long long>(1, std::min<long long>(maxp, tiles_ub));
    return launch_k_pairs(kern, dim3(2 * pairs), dim3(C::THREADS), (size_t)C::SMEM_BYTES, st, pdl, tx, t0, t1,
                          args);
}

template <int BT, bool DUAL, int OUT>
cudaError_t run_fp4(const GemmProblem& p, const GemmArgs& args, const CUtensorMap& tx, cudaStream_t st, bool pdl) {
    using C = Fp4Cfg<BT, DUAL>;
    auto kern = grouped_gemm_fp4_kernel<BT, DUAL, OUT>;
    static int done[64] = {0};
    cudaError_t e = set_smem_once(kern, C::SMEM_BYTES, done);
    if (e != cudaSuccess) return e;
    return launch_k(kern, dim3(grid_for(p, args, BT)), dim3(C::THREADS), (size_t)C::SMEM_BYTES, st, pdl, tx, args);
}

template <int BT, bool DUAL, int OUT>
cudaError_t run_nvf4(const GemmProblem& p, const GemmArgs& args, const CUtensorMap& tx, const CUtensorMap& tsf,
                     cudaStream_t st, bool pdl) {
    using C = Nvf4Cfg<BT, DUAL>;
    auto kern = grouped_gemm_nvf4_kernel<BT, DUAL, OUT>;
    static int done[64] = {0};
    cudaError_t e = set_smem_once(kern, C::SMEM_BYTES, done);
    if (e != cudaSuccess) return e;
    return launch_k(kern, dim3(grid_for(p, args, BT)), dim3(C::THREADS), (size_t)C::SMEM_BYTES, st, pdl, tx, tsf,
                    args);
}

template <int BT>
cudaError_t dispatch_nvf4(const GemmProblem& p, const GemmArgs& args, const CUtensorMap& tx, const CUtensorMap& tsf,
                          cudaStream_t st, bool pdl) {
    if constexpr (BT <= 64) {
        if (p.dual) return run_nvf4<BT, true, OUT_F32>(p, args, tx, tsf, st, pdl);
    }
    if (p.dual) return cudaErrorInvalidValue;
    if (p.out_kind == OUT_F32) return run_nvf4<BT, false, OUT_F32>(p, args, tx, tsf, st, pdl);
    return run_nvf4<BT, false, OUT_BF16>(p, args, tx, tsf, st, pdl);
}

// Token tile of the block-scaled GEMM. Its cost is one pipeline stage per (token tile,
// weight tile, 256 K) whatever the tile's width, so the tile should hold a whole segment:
// a width of at least mean + 2 sqrt(mean) covers nearly every segment once.
int choose_token_tile_nvf4(long long NvS, int G) {
    const long long segs = std::max<long long>(1, std::min<long long>(G, NvS));
    const double avg = (double)NvS / (double)segs;
    const double want = avg + 2.0 * std::sqrt(avg);
    return want <= 16 ? 16 : want <= 32 ? 32 : want <= 64 ? 64 : 128;
}

// The block-scaled NVFP4 GEMM. Token tile as above, at most 64 for the
// gate/up pair (two 2 x 64-column accumulator buffers plus the scale factors fill TMEM).
cudaError_t launch_nvf4(const GemmProblem& p, GemmArgs& a, cudaStream_t st, bool pdl) {
    if (p.K % kNvf4StageK || !p.kscale0 || (p.dual && !p.kscale1) || !p.xsf) return cudaErrorInvalidValue;
    if (p.dual && p.out_kind != OUT_F32) return cudaErrorInvalidValue;
    a.KB = p.K / kNvf4StageK;
    int bt = p.bt;
    if (!bt) {
        const char* env = getenv("MOE_TOKEN_TILE");
        const int v = env ? atoi(env) : 0;
        bt = (v == 16 || v == 32 || v == 64 || v == 128) ? v : choose_token_tile_nvf4(p.M_alloc, p.G);
    }
    if (bt > 128) bt = 128;
    if (p.dual && bt > 64) bt = 64;
    CUtensorMap tx, tsf;
    if (!make_map_u8(&tx, p.x, (uint64_t)p.K / 2, p.M_alloc, p.x_stride, kNvf4StageK / 2, bt,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_u8(&tsf, p.xsf, (uint64_t)p.K / 16, p.M_alloc, p.xsf_stride, kNvf4StageK / 16, bt,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    switch (bt) {
        case 16: return dispatch_nvf4<16>(p, a, tx, tsf, st, pdl);
        case 32: return dispatch_nvf4<32>(p, a, tx, tsf, st, pdl);
        case 64: return dispatch_nvf4<64>(p, a, tx, tsf, st, pdl);
        default: return dispatch_nvf4<128>(p, a, tx, tsf, st, pdl);
    }
}

template <int BT, bool DUAL, bool TWO, int OUT, bool WIDE = false>
cudaError_t run_mx8(const GemmProblem& p, GemmArgs args, const CUtensorMap& tx, const CUtensorMap& tsf,
                    const CUtensorMap& t0, const CUtensorMap& t1, int Kp, cudaStream_t st, bool pdl) {
    using C = Mx8Cfg<BT, DUAL || WIDE, TWO>;
    auto kern = grouped_gemm_mx8_kernel<BT, DUAL, TWO, OUT, WIDE>;
    static int done[64] = {0};
    cudaError_t e = set_smem_once(kern, C::SMEM_BYTES, done);
    if (e != cudaSuccess) return e;
    if (WIDE) {  // tiles of two 128-row blocks of the one matrix
        args.NT = (p.N + 2 * kTileN - 1) / (2 * kTileN);
        args.ks1 = args.ks0;
    }
    return launch_k(kern, dim3(grid_for(p, args, BT)), dim3(C::THREADS), (size_t)C::SMEM_BYTES, st, pdl, tx, tsf, t0,
                    t1, args, Kp);
}

// The single-matrix MXFP4 GEMM streams two weight blocks per stage for decode-sized token
// tiles (MOE_MX8_WIDE=0 keeps one).
bool mx8_wide(int bt) {
    const char* env = getenv("MOE_MX8_WIDE");
    if (env && env[0] == '0' && env[1] == '\0') return false;
    return bt <= 32;
}

template <int BT, bool TWO>
cudaError_t dispatch_mx8_terms(const GemmProblem& p, const GemmArgs& args, const CUtensorMap& tx,
                               const CUtensorMap& tsf, const CUtensorMap& t0, const CUtensorMap& t1, int Kp,
                               cudaStream_t st, bool pdl) {
    if (p.dual) {
        if (p.out_kind == OUT_MX8) return run_mx8<BT, true, TWO, OUT_MX8>(p, args, tx, tsf, t0, t1, Kp, st, pdl);
        if (p.out_kind != OUT_F32) return cudaErrorInvalidValue;
        return run_mx8<BT, true, TWO, OUT_F32>(p, args, tx, tsf, t0, t1, Kp, st, pdl);
    }
    if constexpr (BT <= 32) {
        if (mx8_wide(BT)) {
            if (p.out_kind == OUT_F32) return run_mx8<BT, false, TWO, OUT_F32, true>(p, args, tx, tsf, t0, t1, Kp, st, pdl);
            if (!TWO) return cudaErrorInvalidValue;
            return run_mx8<BT, false, TWO, OUT_BF16, true>(p, args, tx, tsf, t0, t1, Kp, st, pdl);
        }
    }
    if (p.out_kind == OUT_F32) return run_mx8<BT, false, TWO, OUT_F32>(p, args, tx, tsf, t0, t1, Kp, st, pdl);
    if (!TWO) return cudaErrorInvalidValue;  // the standalone bf16-output GEMM stages hi/lo
    return run_mx8<BT, false, TWO, OUT_BF16>(p, args, tx, tsf, t0, t1, Kp, st, pdl);
}

template <int BT>
cudaError_t dispatch_mx8(const GemmProblem& p, const GemmArgs& args, const CUtensorMap& tx, const CUtensorMap& tsf,
                         const CUtensorMap& t0, const CUtensorMap& t1, int Kp, cudaStream_t st, bool pdl) {
    if (p.mx8 == 1) return dispatch_mx8_terms<BT, false>(p, args, tx, tsf, t0, t1, Kp, st, pdl);
    return dispatch_mx8_terms<BT, true>(p, args, tx, tsf, t0, t1, Kp, st, pdl);
}

// The MXFP4 x MXFP8 GEMM; token tile as for the NVFP4 one.
cudaError_t launch_mx8(const GemmProblem& p, GemmArgs& a, cudaStream_t st, bool pdl) {
    if (!p.kdata0 || !p.kscale0 || (p.dual && (!p.kdata1 || !p.kscale1))) return cudaErrorInvalidValue;
    const int Kp = mx8_kpad(p.K);
    a.KB = Kp / kMx8StageK;
    int bt = p.bt;
    if (!bt) {
        const char* env = getenv("MOE_TOKEN_TILE");
        const int v = env ? atoi(env) : 0;
        bt = (v == 16 || v == 32 || v == 64 || v == 128) ? v : choose_token_tile_nvf4(p.M_alloc, p.G);
    }
    if (bt > 128) bt = 128;
    const uint8_t* rec = static_cast<const uint8_t*>(p.x);
    CUtensorMap tx, tsf, t0, t1;
    memset(&t1, 0, sizeof(t1));
    const int terms = p.mx8 == 1 ? 1 : 2;
    if (!make_map_u8(&tx, rec, (uint64_t)terms * Kp, p.M_alloc, p.x_stride, kMx8StageK, bt,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_u8(&tsf, rec + (size_t)terms * Kp, mx8_scale_bytes(p.K), p.M_alloc, p.x_stride, 16, bt,
                     CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map_w_u4(&t0, p.kdata0, Kp, p.N, p.G) || (p.dual && !make_map_w_u4(&t1, p.kdata1, Kp, p.N, p.G)))
        return cudaErrorInvalidValue;
    if (!p.dual) t1 = t0;
    a.ks0 = static_cast<const uint8_t*>(p.kscale0);
    a.ks1 = static_cast<const uint8_t*>(p.kscale1);
    switch (bt) {
        case 16: return dispatch_mx8<16>(p, a, tx, tsf, t0, t1, Kp, st, pdl);
        case 32: return dispatch_mx8<32>(p, a, tx, tsf, t0, t1, Kp, st, pdl);
        case 64: return dispatch_mx8<64>(p, a, tx, tsf, t0, t1, Kp, st, pdl);
        default: return dispatch_mx8<128>(p, a, tx, tsf, t0, t1, Kp, st, pdl);
    }
}

template <int BT>
cudaError_t dispatch_fp4(const GemmProblem& p, const GemmArgs& args, const CUtensorMap& tx, cudaStream_t st,
                         bool pdl) {
    if (p.dual) {
        if (p.out_kind == OUT_F16) return run_fp4<BT, true, OUT_F16>(p, args, tx, st, pdl);
        return run_fp4<BT, true, OUT_F32>(p, args, tx, st, pdl);
    }
    if (p.out_kind == OUT_F32) return run_fp4<BT, false, OUT_F32>(p, args, tx, st, pdl);
    return run_fp4<BT, false, OUT_BF16>(p, args, tx, st, pdl);
}

template <int BT>
cudaError_t dispatch_bt(const GemmProblem& p, const GemmArgs& args, const CUtensorMap& tx,
                        const CUtensorMap& t0, const CUtensorMap& t1, cudaStream_t st, bool pdl) {
    if (p.wfmt == MOE_W_NVFP4) return dispatch_fp4<BT>(p, args, tx, st, pdl);
    if (p.dual) return run_bf16<BT, true, OUT_BF16>(p, args, tx, t0, t1, st, pdl);
    if (p.out_kind == OUT_F32) return run_bf16<BT, false, OUT_F32>(p, args, tx, t0, t1, st, pdl);
    return run_bf16<BT, false, OUT_BF16>(p, args, tx, t0, t1, st, pdl);
}

}  // namespace

// Token tile from the mean segment length. 256-token tiles exist for the BF16 GEMMs only:
// at 128 x 128 a tile needs more shared-memory bandwidth per FLOP than an SM has, and a
// 256-wide tile halves the weight-tile traffic per FLOP. They are chosen for the single
// matrix (double-buffered accumulators still fit); the gate/up pair's 256-token tile has
// one accumulator buffer and is used only when MOE_TOKEN_TILE asks for it. The MMA width
// follows each tile's rows, so a wide tile costs a short segment little.
int choose_token_tile(long long NvS, int G, bool wide_ok) {
    const long long segs = std::max<long long>(1, std::min<long long>(G, NvS));
    const long long avg = (NvS + segs - 1) / segs;
    if (avg <= 16) return 16;
    if (avg <= 32) return 32;
    if (avg <= 64) return 64;
    if (avg <= 128 || !wide_ok) return 128;
    return 256;
}

// The pipeline-wait limit of a launch: MOE_WAIT_LIMIT_CYCLES (a positive integer, read at
// every launch) or the default of about one second. A shorter limit is for tests of the
// timeout path; the waits for copies and MMAs in flight after an abort keep the default.
long long wait_limit_cycles() {
    const char* env = getenv("MOE_WAIT_LIMIT_CYCLES");
    if (env) {
        char* end = nullptr;
        const long long v = strtoll(env, &end, 10);
        if (end != env && *end == '\0' && v > 0) return std::min(v, kWaitLimitCycles);
    }
    return kWaitLimitCycles;
}

// Whether a BF16 GEMM runs on CTA pairs. MOE_GEMM_PAIRS=0: never; 1: always; 2: when the
// segments average more than 96 rows. Unset: when they average more than 512 rows and no
// token tile was forced. Long segments fill the pair's 256-token tiles; the pair measured
// faster than one SM per tile there (the Mixtral-shaped prefill) and not at DeepSeek-shaped
// segments of about 250 rows.
bool use_pairs(const GemmProblem& p) {
    const char* env = getenv("MOE_GEMM_PAIRS");
    int mode = 3;
    if (env) {
        if (env[0] < '0' || env[0] > '2' || env[1] != '\0') return false;
        mode = env[0] - '0';
    }
    if (mode == 0) return false;
    if (mode == 1) return true;
    if (p.bt || getenv("MOE_TOKEN_TILE")) return false;
    const long long segs = std::max<long long>(1, std::min<long long>(p.G, p.M_alloc));
    return p.M_alloc > (mode == 2 ? 96 : 512) * segs;
}

// Whether launch_grouped_gemm can gather this problem's token rows itself (BF16 gate/up with
// 128-token tiles on one SM, or on CTA pairs).
bool gemm_can_gather(const GemmProblem& p) {
    if (p.wfmt != MOE_W_BF16 || !p.dual) return false;
    if (use_pairs(p)) return true;
    const char* env = getenv("MOE_TOKEN_TILE");
    const int v = env ? atoi(env) : 0;
    const int bt = p.bt ? p.bt : (v ? v : choose_token_tile(p.M_alloc, p.G, false));
    return bt == 128;
}

// L2 policies of the copies: MOE_L2_HINTS = 0 none, 1 token rows evict-last, 2 also the
// weights evict-first (default 1). Token rows are re-read by every weight block of their
// segment; weight tiles by the few token tiles of a segment, close together in time.
void l2_policies(int* w, int* t) {
    const char* env = getenv("MOE_L2_HINTS");
    const int m = env && env[0] >= '0' && env[0] <= '2' && env[1] == '\0' ? env[0] - '0' : 1;
    *t = m >= 1 ? 2 : 0;
    *w = m >= 2 ? 1 : 0;
}

cudaError_t launch_grouped_gemm(const GemmProblem& p, cudaStream_t st, bool pdl) {
    if (p.G > kMaxG) return cudaErrorInvalidValue;
    GemmArgs a{};
    a.wait_limit = wait_limit_cycles();
    l2_policies(&a.l2_w, &a.l2_t);
    a.cu = p.cu_seqlens;
    a.G = p.G;
    a.N = p.N;
    a.K = p.K;
    // pipeline stages per tile: 64 K values (BF16) or 128 (FP4, two prepared chunks)
    a.KB = p.wfmt == MOE_W_BF16 ? (p.K + kTileK - 1) / kTileK : (p.K + kFp4StageK - 1) / kFp4StageK;
    a.NT = (p.N + kTileN - 1) / kTileN;
    a.M_alloc = p.M_alloc;
    a.out = p.out;
    a.alpha0 = p.alpha0;
    a.alpha1 = p.alpha1;
    a.perm_w = p.perm_w;
    a.tscale = p.tscale;
    a.out_scale = p.out_scale;
    a.bias0 = p.bias0;
    a.bias1 = p.bias1;
    a.bias_rw = p.bias_rw;
    a.sw_alpha = p.sw_alpha;
    a.sw_beta = p.sw_beta;
    a.sw_limit = p.sw_limit;
    a.out_terms = p.out_terms;
    a.out_stride = p.out_stride;
    a.out_kpad = p.out_kind == OUT_MX8 ? mx8_kpad(p.N) : 0;
    // the records cover the padded K of the down GEMM: N_tiles * 128 = mx8_kpad(N)
    if (p.out_kind == OUT_MX8 && (p.wfmt != MOE_W_MXFP4 || !p.dual || p.N % 32 ||
                                  (p.out_terms != 1 && p.out_terms != 2)))
        return cudaErrorInvalidValue;
    a.act = p.act;
    a.sa = p.situ_a;
    a.sb = p.situ_b;
    a.kd0 = static_cast<const uint8_t*>(p.kdata0);
    a.ks0 = static_cast<const uint8_t*>(p.kscale0);
    a.kd1 = static_cast<const uint8_t*>(p.kdata1);
    a.ks1 = static_cast<const uint8_t*>(p.kscale1);
    a.zero_pad = p.zero_pad ? 1 : 0;
    a.err = p.err;
    if (p.nvf4) return launch_nvf4(p, a, st, pdl);
    if (p.wfmt == MOE_W_MXFP4) return p.mx8 ? launch_mx8(p, a, st, pdl) : cudaErrorInvalidValue;
    // The gate/up pair's 256-token tile (one accumulator buffer, three pipeline stages)
    // measured slower than two 128-token tiles; it is used only on request.
    const bool wide_ok = p.wfmt == MOE_W_BF16 && !p.dual;
    const bool wide_req = p.wfmt == MOE_W_BF16;
    int bt = p.bt;
    if (!bt) {
        // MOE_TOKEN_TILE=16|32|64|128|256 overrides the token-tile choice (tests, tuning)
        const char* env = getenv("MOE_TOKEN_TILE");
        const int v = env ? atoi(env) : 0;
        bt = (v == 16 || v == 32 || v == 64 || v == 128 || (v == 256 && wide_req))
                 ? v
                 : choose_token_tile(p.M_alloc, p.G, wide_ok);
    }
    if (bt == 256 && !wide_req) bt = 128;
    // BF16 prefill shapes run on CTA pairs: 256 weight rows x up to 256 tokens per pair tile
    // (MOE_GEMM_PAIRS=0 keeps the one-SM kernel, e.g. to compare the two)
    if (p.wfmt == MOE_W_BF16 && p.gather_idx && !use_pairs(p)) {
        // the 128-token gate/up tile gathering its own token rows from x
        if (!p.dual || p.K % 8 || p.gather_rows < 1) return cudaErrorInvalidValue;
        CUtensorMap tx, t0, t1;
        if (!make_map_2d(&tx, p.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.K, p.gather_rows, 128) ||
            !make_map_3d(&t0, p.w0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.K, p.N, p.G) ||
            !make_map_3d(&t1, p.w1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.K, p.N, p.G))
            return cudaErrorInvalidValue;
        a.gather_idx = p.gather_idx;
        a.gx = static_cast<const __nv_bfloat16*>(p.x);
        a.gather_rows = p.gather_rows;
        return run_bf16<128, true, OUT_BF16, true>(p, a, tx, t0, t1, st, pdl);
    }
    if (p.wfmt == MOE_W_BF16 && use_pairs(p)) {
        CUtensorMap tx, t0, t1;
        memset(&t1, 0, sizeof(t1));
        if (!make_map_2d(&tx, p.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.K, p.gather_idx ? p.gather_rows : p.M_alloc,
                         128) ||
            !make_map_3d(&t0, p.w0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.K, p.N, p.G) ||
            (p.dual && !make_map_3d(&t1, p.w1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.K, p.N, p.G)))
            return cudaErrorInvalidValue;
        if (!p.dual) t1 = t0;
        if (p.gather_idx) {
            // token rows straight from x: K % 8 == 0 keeps each 16-byte chunk inside a row
            if (!p.dual || p.K % 8 || p.gather_rows < 1) return cudaErrorInvalidValue;
            a.gather_idx = p.gather_idx;
            a.gx = static_cast<const __nv_bfloat16*>(p.x);
            a.gather_rows = p.gather_rows;
            return run_pair<256, true, OUT_BF16, true, true>(p, a, tx, t0, t1, st, pdl);
        }
        // MOE_PAIR_FWD=1: the peer forwards each stage instead of completing the leader's barrier
        const char* fwd = getenv("MOE_PAIR_FWD");
        if (fwd && fwd[0] == '1' && fwd[1] == '\0') {
            if (p.dual) return run_pair<256, true, OUT_BF16, false, true>(p, a, tx, t0, t1, st, pdl);
            if (p.out_kind == OUT_F32) return run_pair<256, false, OUT_F32, false, true>(p, a, tx, t0, t1, st, pdl);
            return run_pair<256, false, OUT_BF16, false, true>(p, a, tx, t0, t1, st, pdl);
        }
        if (p.dual) return run_pair<256, true, OUT_BF16, false, false>(p, a, tx, t0, t1, st, pdl);
        if (p.out_kind == OUT_F32) return run_pair<256, false, OUT_F32, false, false>(p, a, tx, t0, t1, st, pdl);
        return run_pair<256, false, OUT_BF16, false, false>(p, a, tx, t0, t1, st, pdl);
    }
    const CUtensorMapDataType xdt =
        p.wfmt == MOE_W_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUtensorMap tx, t0, t1;
    memset(&t0, 0, sizeof(t0));
    memset(&t1, 0, sizeof(t1));
    a.x3d = p.wfmt != MOE_W_BF16 && p.K % kTileK == 0;
    if (a.x3d) {
        if (!make_map_3d_chunks(&tx, p.x, xdt, p.K, p.M_alloc, bt)) return cudaErrorInvalidValue;
    } else if (!make_map_2d(&tx, p.x, xdt, p.K, p.M_alloc, bt)) {
        return cudaErrorInvalidValue;
    }
    if (p.wfmt == MOE_W_BF16) {
        if (!make_map_3d(&t0, p.w0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.K, p.N, p.G)) return cudaErrorInvalidValue;
        if (p.dual && !make_map_3d(&t1, p.w1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.K, p.N, p.G))
            return cudaErrorInvalidValue;
    }
    switch (bt) {
        case 16: return dispatch_bt<16>(p, a, tx, t0, t1, st, pdl);
        case 32: return dispatch_bt<32>(p, a, tx, t0, t1, st, pdl);
        case 64: return dispatch_bt<64>(p, a, tx, t0, t1, st, pdl);
        case 256:
            if (p.dual) return run_bf16<256, true, OUT_BF16>(p, a, tx, t0, t1, st, pdl);
            if (p.out_kind == OUT_F32) return run_bf16<256, false, OUT_F32>(p, a, tx, t0, t1, st, pdl);
            return run_bf16<256, false, OUT_BF16>(p, a, tx, t0, t1, st, pdl);
        default: return dispatch_bt<128>(p, a, tx, t0, t1, st, pdl);
    }
}

}  // namespace moe
