"""CPU oracle for the fused MoE expert layer.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module. The CUDA
library never calls it, and it shares no code with the library: no kernels, no
headers, no tables, no helpers. Its inputs come from ``workloads.py``.

It is written to be read against the pages, not to be fast:

* fp64 everywhere, with a BLAS matmul as the only library step;
* intermediates are never rounded to bf16;
* the one place where floating point decides an integer (the dynamic NVFP4
  activation codes) takes that decision in fp32 with IEEE division, the
  precision the CUDA kernels use.

Page citations name the page's module and the class, method or docstring:

* [moonep]   vllm.model_executor.layers.fused_moe.experts.moonep_experts
* [fi_ep]    vllm.model_executor.layers.fused_moe.experts.flashinfer_moe_ep
* [dsv4_fi]  vllm.models.deepseek_v4.nvidia.fi_moe (DeepseekV4MegaMoEExpertsFI)
* [trtllm]   vllm.model_executor.layers.fused_moe.experts.trtllm_mxfp4_moe

Readings taken where the pages are silent are stated at the function that takes
them.
"""
from __future__ import annotations

import numpy as np
import torch

# --------------------------------------------------------------------------------------
# FP4 / FP8 codecs. The pages name the formats (MXFP4: e2m1 values with an e8m0 scale per
# 32 along K [trtllm: _supports_quant_scheme, kMxfp4Static]; NVFP4: e2m1 values with an
# fp8-e4m3 scale per 16 along K plus an fp32 weight_scale_2 [dsv4_fi: _realloc_nvfp4_params])
# but not the bit-level codes. Those are the public OCP Microscaling (MX) v1.0 element
# formats, written out here from their definitions.
# --------------------------------------------------------------------------------------

# e2m1: 1 sign bit (bit 3), 2 exponent bits (bias 1), 1 mantissa bit; no inf/NaN.
# Exponent field 0 is subnormal: value = m * 0.5. Otherwise 2^(e-1) * (1 + m/2).
def _e2m1_magnitudes() -> np.ndarray:
    mags = []
    for code in range(8):
        e, m = code >> 1, code & 1
        mags.append(m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1.0 + m / 2.0))
    return np.array(mags, dtype=np.float64)


E2M1_MAG = _e2m1_magnitudes()          # [0, .5, 1, 1.5, 2, 3, 4, 6]
E2M1_MAX = 6.0


E2M1_VALUES = np.concatenate([E2M1_MAG, -E2M1_MAG])   # by code: bit 3 is the sign


def e2m1_decode(codes) -> np.ndarray:
    """e2m1 code (0..15) -> value, fp64: bit 3 the sign, bits 0-2 the magnitude above."""
    return E2M1_VALUES[np.asarray(codes).astype(np.uint8) & 15]


def unpack_e2m1(packed) -> np.ndarray:
    """Packed bytes ``[..., K/2]`` -> codes ``[..., K]``; the even-K value sits in the low nibble."""
    p = np.asarray(packed).astype(np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0x0F
    out[..., 1::2] = p >> 4
    return out


# e4m3 (the "fn" variant): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, no inf;
# exponent 15 with mantissa 7 is NaN, so the largest finite value is 448.
def _e4m3_value(codes) -> np.ndarray:
    c = np.asarray(codes).astype(np.int64)
    s, e, m = (c >> 7) & 1, (c >> 3) & 0xF, c & 7
    mag = np.where(e == 0, m * 2.0 ** -9, 2.0 ** (e - 7.0) * (1.0 + m / 8.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


E4M3_TABLE = _e4m3_value(np.arange(256))   # the value of every code


def e4m3_decode(codes) -> np.ndarray:
    """e4m3 code (a byte) -> value, fp64, from the table of all 256 codes."""
    return E4M3_TABLE[np.asarray(codes).astype(np.uint8)]


E4M3_MAX = 448.0


def e8m0_decode(codes) -> np.ndarray:
    """e8m0 (MX shared scale): an unsigned biased exponent, value 2^(s-127); 255 is NaN."""
    s = np.asarray(codes).astype(np.int64)
    return np.where(s == 255, np.nan, np.ldexp(1.0, s - 127))


def _encode_rne_satfinite(v, table_vals: np.ndarray, sign_bit: int) -> np.ndarray:
    """Round |v| to the nearest entry of ``table_vals`` (non-negative, ascending, index = code),
    ties to the even code (even mantissa), saturating to the largest entry; the sign of v
    (including -0) goes to ``sign_bit``. NaN inputs are not expected and not handled."""
    x = np.asarray(v, dtype=np.float64)
    neg = np.signbit(x)
    a = np.minimum(np.abs(x), table_vals[-1])
    hi = np.clip(np.searchsorted(table_vals, a, side="left"), 0, len(table_vals) - 1)
    lo = np.clip(hi - 1, 0, len(table_vals) - 1)
    dlo, dhi = a - table_vals[lo], table_vals[hi] - a
    pick = np.where(dhi < dlo, hi, np.where(dlo < dhi, lo, np.where(lo % 2 == 0, lo, hi)))
    return (pick | (neg.astype(np.int64) << sign_bit)).astype(np.uint8)


_E4M3_POS = e4m3_decode(np.arange(0, 127))      # codes 0..126: the non-negative finite values


def e2m1_encode(v) -> np.ndarray:
    """Real -> e2m1 code, round to nearest even, saturate to +-6."""
    return _encode_rne_satfinite(v, E2M1_MAG, 3)


def e4m3_encode(v) -> np.ndarray:
    """Real -> e4m3 code, round to nearest even, saturate to +-448."""
    return _encode_rne_satfinite(v, _E4M3_POS, 7)


# --------------------------------------------------------------------------------------
# Weights
# --------------------------------------------------------------------------------------

def to_f64(t) -> np.ndarray:
    """bf16 / fp32 torch tensor (or array) -> fp64 numpy, exactly."""
    if isinstance(t, torch.Tensor):
        return t.detach().to(torch.float64).cpu().numpy()
    return np.asarray(t, dtype=np.float64)


def weight_rows(ws, g: int) -> np.ndarray:
    """Dequantised weights of row ``g`` of a projection, fp64 ``[N,K]``, without its global alpha.

    BF16 as stored. MXFP4: e2m1(q) * 2^(s-127), one e8m0 scale per 32 along K
    [trtllm: TrtLlmMxfp4ExpertsBase]. NVFP4: e2m1(q) * e4m3(s), one scale per 16 along K;
    the per-expert fp32 ``weight_scale_2`` stays a separate epilogue alpha
    [dsv4_fi: _realloc_nvfp4_params; fi_ep: epilogue_from_quant_config].
    Every product is exact in fp64.
    """
    if ws.fmt == "bf16":
        return to_f64(ws.data[g])
    q = e2m1_decode(unpack_e2m1(ws.data[g].numpy()))
    blk = {"mxfp4": 32, "nvfp4": 16}.get(ws.fmt)
    if blk is None:
        raise ValueError(ws.fmt)
    sc = (e8m0_decode if ws.fmt == "mxfp4" else e4m3_decode)(ws.scale[g].numpy())
    # each scale multiplies its block of blk consecutive values along K
    return (q.reshape(q.shape[0], -1, blk) * sc[..., None]).reshape(q.shape)


def weight_alpha(ws) -> np.ndarray:
    """Per-row global scale (fc1/fc2 epilogue alpha): NVFP4 ``weight_scale_2``, else 1.

    [fi_ep: epilogue_from_quant_config] MXFP4 carries no global scale and keeps the default
    epilogue; NVFP4's per-expert globals become the alphas [dsv4_fi: finalize_weights].
    """
    if ws.alpha is None:
        return np.ones(ws.G, dtype=np.float64)
    return to_f64(ws.alpha)


# --------------------------------------------------------------------------------------
# S1 routing
# --------------------------------------------------------------------------------------

def route_topk(logits, topk: int):
    """Softmax -> top-k -> renormalise ("Renormalize" routing [trtllm: _invoke_kernel,
    routing_method_type]; int32 ids [fi_ep: FlashInferMoeEpExperts.apply]).

    Selection is on the fp32 logits: experts ordered by (logit descending, id ascending), so
    ties go to the lower expert id and -0 ties +0. Over the selected k, with l_0 the largest,
    ``w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0)``, which equals the softmax over all E
    experts restricted to the k and renormalised (the common factor cancels).
    Returns ``ids [T,k] int32`` (in selection order) and ``w [T,k]`` fp64.
    """
    L = np.asarray(logits, dtype=np.float32).astype(np.float64)
    T, E = L.shape
    if not (1 <= topk <= E):
        raise ValueError("need 1 <= topk <= E")
    if T == 0:
        return np.zeros((0, topk), np.int32), np.zeros((0, topk), np.float64)
    eid = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((eid, -L), axis=-1)          # primary key last: -logit, then id
    ids = order[:, :topk]
    sel = np.take_along_axis(L, ids, axis=1)
    z = np.exp(sel - sel[:, :1])
    w = z / z.sum(axis=1, keepdims=True)
    return ids.astype(np.int32), w


def route_topk_grouped(logits, topk: int, n_group: int, topk_group: int, bias=None,
                       routed_scaling_factor: float = 1.0):
    """DeepSeekV3 routing: group-limited top-k on sigmoid scores with a selection bias.

    The TRTLLM MXFP4 page lists ``RoutingMethodType.DeepSeekV3`` among its routing methods
    and passes ``n_group``, ``topk_group``, ``routing_bias=e_score_correction_bias`` and
    ``routed_scaling_factor`` to the kernel [trtllm: _supports_routing_method, apply]; it does
    not spell the method out. Reading taken: the published DeepSeek-V3 routing.

      s_e = sigmoid(l_e);  c_e = s_e + bias_e          (the bias steers selection only)
      the E experts form n_group consecutive groups of E/n_group; a group's score is the
      sum of its two largest c (its one c when a group has a single expert)
      keep the topk_group groups of largest score (ties to the lower group id)
      among their experts take the topk of largest c (ties to the lower id), in that order
      w_j = routed_scaling_factor * s_j / sum over the chosen s

    Every decision is taken in fp64 (so is the CUDA kernel's).
    Returns ``ids [T,k] int32`` (in selection order) and ``w [T,k]`` fp64.
    """
    L = np.asarray(logits, dtype=np.float32).astype(np.float64)
    T, E = L.shape
    if n_group < 1 or E % n_group or not (1 <= topk_group <= n_group):
        raise ValueError("need E % n_group == 0 and 1 <= topk_group <= n_group")
    gs = E // n_group
    if not (1 <= topk <= topk_group * gs):
        raise ValueError("need 1 <= topk <= topk_group * E / n_group")
    b = np.zeros(E) if bias is None else np.asarray(bias, dtype=np.float32).astype(np.float64)
    if T == 0:
        return np.zeros((0, topk), np.int32), np.zeros((0, topk), np.float64)
    s = 1.0 / (1.0 + np.exp(-L))
    c = s + b[None, :]
    top = -np.sort(-c.reshape(T, n_group, gs), axis=2)           # descending within each group
    gscore = top[:, :, 0] + (top[:, :, 1] if gs >= 2 else 0.0)
    gid = np.broadcast_to(np.arange(n_group), (T, n_group))
    gorder = np.lexsort((gid, -gscore), axis=-1)[:, :topk_group]
    keep = np.zeros((T, n_group), dtype=bool)
    np.put_along_axis(keep, gorder, True, axis=1)
    allowed = np.repeat(keep, gs, axis=1)
    eid = np.broadcast_to(np.arange(E), (T, E))
    key = np.where(allowed, -c, np.inf)
    ids = np.lexsort((eid, key), axis=-1)[:, :topk]
    sel = np.take_along_axis(s, ids, axis=1)
    w = routed_scaling_factor * sel / sel.sum(axis=1, keepdims=True)
    return ids.astype(np.int32), w


def route(cfg, logits, bias=None):
    """The routing method a workload names: "renormalize" (``route_topk``) or "deepseek_v3"
    (``route_topk_grouped`` with the workload's n_group, topk_group and scaling factor)."""
    if getattr(cfg, "routing", "renormalize") == "deepseek_v3":
        return route_topk_grouped(logits, cfg.topk, cfg.n_group, cfg.topk_group, bias, cfg.routed_scaling_factor)
    return route_topk(logits, cfg.topk)


# --------------------------------------------------------------------------------------
# S2 permutation into expert-contiguous segments
# --------------------------------------------------------------------------------------

def assign_rows(ids, E: int, B: int, replica_src):
    """Expert-contiguous segments over G = E + B weight rows [moonep: module docstring, apply].

    Segment g lists its (token, k) assignments in ascending token order. ``cu_seqlens[g]`` is
    the inclusive running sum of the segment lengths, as ``torch.cumsum(expert_num_tokens)``
    [moonep: MoonEPExperts.apply]. Rows [E, E+B) are redundant copies of hot experts; the pages
    do not say how a replicated expert's tokens are shared out (that lives in the unseen
    MoonEPPrepareAndFinalize), so this reading is taken: let R(e) be e followed by the slots s
    with replica_src[s] == e in ascending s; e's n assignments (ascending token order) are cut
    into |R(e)| contiguous chunks, chunk i holding n // |R| + (i < n % |R|) of them, and chunk i
    goes to row R(e)[i]. Unused slots (replica_src = -1) stay empty.

    Returns dict with ``row [T,k]`` (weight row of each assignment), ``cu_seqlens [G]``,
    ``perm_token [NvS]``, ``perm_k [NvS]`` and ``inv_perm [T,k]`` (position of (t,k) in NvS).
    """
    ids = np.asarray(ids, dtype=np.int64)
    T, k = ids.shape
    G = E + B
    src = np.asarray(replica_src, dtype=np.int64).reshape(-1) if B else np.zeros(0, np.int64)
    if src.shape[0] != B:
        raise ValueError("replica_src must have B entries")
    reps = [[e] for e in range(E)]
    for s in range(B):
        if src[s] >= 0:
            reps[int(src[s])].append(E + s)
    per_expert = [[] for _ in range(E)]
    for t in range(T):
        for j in range(k):
            per_expert[int(ids[t, j])].append((t, j))
    segments = [[] for _ in range(G)]
    for e in range(E):
        lst, R = per_expert[e], reps[e]
        q, r = divmod(len(lst), len(R))
        pos = 0
        for i, row in enumerate(R):
            size = q + (1 if i < r else 0)
            segments[row] = lst[pos:pos + size]
            pos += size
    counts = np.array([len(s) for s in segments], dtype=np.int64)
    cu = np.cumsum(counts).astype(np.int32) if G else np.zeros(0, np.int32)
    NvS = T * k
    perm_token = np.empty(NvS, np.int32)
    perm_k = np.empty(NvS, np.int32)
    inv_perm = np.empty((T, k), np.int32)
    row = np.empty((T, k), np.int32)
    p = 0
    for g, seg in enumerate(segments):
        for (t, j) in seg:
            perm_token[p], perm_k[p], inv_perm[t, j], row[t, j] = t, j, p, g
            p += 1
    return dict(row=row, cu_seqlens=cu, perm_token=perm_token, perm_k=perm_k, inv_perm=inv_perm)


def segment_bounds(cu_seqlens):
    """(start, end) of every segment from inclusive end offsets."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    starts = np.concatenate([[0], cu[:-1]]) if len(cu) else cu
    return list(zip(starts.tolist(), cu.tolist()))


# --------------------------------------------------------------------------------------
# S3 / S5 grouped GEMM
# --------------------------------------------------------------------------------------

def grouped_gemm(a, ws, cu_seqlens, M_alloc: int | None = None):
    """``out[seg_g] = alpha_g * a[seg_g] @ W[g].T`` for every segment; rows past the last
    segment end are zero [moonep: moonep_grouped_gemm]. ``a`` is fp64 ``[M,K]``."""
    a = np.asarray(a, dtype=np.float64)
    M = a.shape[0] if M_alloc is None else M_alloc
    alpha = weight_alpha(ws)
    out = np.zeros((M, ws.N), dtype=np.float64)
    for g, (s, e) in enumerate(segment_bounds(cu_seqlens)):
        if e > s:  # empty segments are skipped
            out[s:e] = alpha[g] * (a[s:e] @ weight_rows(ws, g).T)
    return out


# --------------------------------------------------------------------------------------
# S4 activation
# --------------------------------------------------------------------------------------

def silu_and_mul(gate, up):
    """silu(gate) * up = gate / (1 + e^-gate) * up [moonep: module docstring, apply]."""
    with np.errstate(over="ignore"):
        return gate / (1.0 + np.exp(-gate)) * up


def situ_and_mul(gate, up, alpha: float, beta: float):
    """SITU gated activation [trtllm: TrtLlmMxfp4ExpertsBase.__init__, SITU comment]:
    left = alpha * tanh(x0/alpha) * sigmoid(x0) on the gate, right = beta * tanh(x1/beta) on the
    up projection, output left * right; alpha = situ_beta, beta = situ_linear_beta, both > 0.
    The sigmoid takes the raw gate, as written."""
    if not (alpha > 0 and beta > 0):
        raise ValueError("SITU needs alpha > 0 and beta > 0")
    with np.errstate(over="ignore"):
        sig = 1.0 / (1.0 + np.exp(-gate))
    return alpha * np.tanh(gate / alpha) * sig * (beta * np.tanh(up / beta))


def swigluoai_and_mul(gate, up, alpha: float, beta: float, limit=None):
    """SWIGLUOAI gated activation. The TRTLLM MXFP4 page lists SWIGLUOAI among its
    activations and hands per-expert gemm1_alpha, gemm1_beta and gemm1_clamp_limit to the
    kernel [trtllm: TrtLlmMxfp4ExpertsBase._supports_activation and __init__,
    TrtLlmMxfp4ExpertsModular._invoke_kernel], without the formula. Reading taken: the
    published GPT-OSS gated activation,

      g = min(gate, limit),  u = clamp(up, -limit, limit)     (no clamp when limit is None)
      out = g * sigmoid(alpha * g) * (u + beta)

    (GPT-OSS itself uses alpha = 1.702, beta = 1, limit = 7)."""
    g = np.asarray(gate, dtype=np.float64)
    u = np.asarray(up, dtype=np.float64)
    if limit is not None:
        g = np.minimum(g, limit)
        u = np.clip(u, -limit, limit)
    with np.errstate(over="ignore"):
        sig = 1.0 / (1.0 + np.exp(-alpha * g))
    return g * sig * (u + beta)


def act_and_mul(gate, up, act: str = "silu", situ_alpha: float = 1.0, situ_beta: float = 1.0,
                route_w=None, swiglu_alpha: float = 1.702, swiglu_beta: float = 1.0, swiglu_limit=7.0):
    """Gated activation times the per-row route weight (``act *= route_weight``
    [moonep: MoonEPExperts.apply])."""
    if act == "silu":
        h = silu_and_mul(gate, up)
    elif act == "situ":
        h = situ_and_mul(gate, up, situ_alpha, situ_beta)
    elif act == "swigluoai":
        h = swigluoai_and_mul(gate, up, swiglu_alpha, swiglu_beta, swiglu_limit)
    else:
        raise ValueError(act)
    if route_w is not None:
        h = h * np.asarray(route_w, dtype=np.float64)[:, None]
    return h


# --------------------------------------------------------------------------------------
# S2q dynamic NVFP4 activation quantisation
# --------------------------------------------------------------------------------------

NVFP4_ROW_DIV = np.float32(6.0 * 448.0)   # 2688: e2m1 max times e4m3 max


def nvfp4_quantize_rows(v):
    """Dynamic NVFP4 quantisation of activation rows.

    The pages only say the megakernel quantises activations dynamically and drops the
    checkpoint's input scales [fi_ep: epilogue_from_quant_config; dsv4_fi: forward,
    stage_inputs(..., quantize_input=True)]. Reading taken: e2m1 codes with one e4m3 scale per
    16 values and one fp32 scale per row, all decisions in fp32 with IEEE division:

      s_r  = amax_r / 2688
      sb_b = e4m3_rne_satfinite(amax_b / (6 * s_r))        per 16-value block b
      q    = e2m1_rne_satfinite(v / (sb_b * s_r))           (sb_b * s_r rounded to fp32)
      value = e2m1(q) * sb_b * s_r

    A zero row, and any block whose scale rounds to zero, quantises to +0 codes.
    Returns ``codes [R,K] uint8``, ``sb [R,K/16] uint8`` (e4m3 codes), ``s [R] float32``.
    """
    x = np.asarray(v, dtype=np.float32)
    R, K = x.shape
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    ax = np.abs(x)
    amax = ax.max(axis=1) if K else np.zeros(R, np.float32)
    s = (amax / NVFP4_ROW_DIV).astype(np.float32)
    six_s = (np.float32(6.0) * s).astype(np.float32)
    bmax = ax.reshape(R, K // 16, 16).max(axis=2)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(six_s[:, None] > 0, bmax / six_s[:, None], np.float32(0)).astype(np.float32)
    sb = e4m3_encode(ratio)
    step = (e4m3_decode(sb).astype(np.float32) * s[:, None]).astype(np.float32)
    step_k = np.repeat(step, 16, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = np.where(step_k > 0, x / step_k, np.float32(0)).astype(np.float32)
    codes = e2m1_encode(y)
    codes = np.where(step_k > 0, codes, 0).astype(np.uint8)
    return codes, sb, s


def nvfp4_dequantize_rows(codes, sb, s):
    """Value of quantised rows: e2m1(q) * e4m3(sb) * s_r, fp64 (exact)."""
    return (e2m1_decode(codes) * np.repeat(e4m3_decode(sb), 16, axis=1)
            * np.asarray(s, dtype=np.float64)[:, None])


# --------------------------------------------------------------------------------------
# S2q dynamic MXFP8 activation quantisation (the W4A8 mode of MXFP4 experts)
# --------------------------------------------------------------------------------------

E4M3_EMAX = 8   # exponent of e4m3's largest normal value, 448 = 1.75 * 2^8


def mxfp8_quantize_rows(v):
    """Dynamic MXFP8 quantisation of activation rows for MXFP4 weights.

    The page lists ``(kMxfp4Static, kMxfp8Dynamic)`` as a supported weight/activation pair
    [trtllm: _supports_quant_scheme] and says nothing more. Reading taken: the OCP MX v1.0
    MXFP8 format with its conversion rule, per 32-value block b of a row:

      X_b  = 2^(floor(log2 amax_b) - 8), the exponent clamped to e8m0's [-127, 127]
      q    = e4m3_rne_satfinite(v / X_b)
      value = e4m3(q) * X_b

    An all-zero block takes X_b = 2^-127 and +0 codes. X_b is a power of two, so v / X_b is
    exact and no decision depends on the arithmetic's precision. Applied, like the NVFP4
    mode, to x in token order and to every activation row before the down GEMM.
    Returns ``codes [R,K] uint8`` (e4m3) and ``scales [R,K/32] uint8`` (e8m0).
    """
    x = np.asarray(v, dtype=np.float32).astype(np.float64)
    R, K = x.shape
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    amax = np.abs(x).reshape(R, K // 32, 32).max(axis=2)
    _, ex = np.frexp(amax)                       # amax = m * 2^ex, m in [0.5, 1): floor(log2) = ex - 1
    e = np.where(amax > 0, ex - 1 - E4M3_EMAX, -127)
    e = np.clip(e, -127, 127).astype(np.int64)
    codes = e4m3_encode(x / np.repeat(np.ldexp(1.0, e), 32, axis=1))
    return codes, (e + 127).astype(np.uint8)


def mxfp8_dequantize_rows(codes, scales):
    """Value of MXFP8 rows: e4m3(q) * 2^(s - 127), fp64 (exact)."""
    return e4m3_decode(codes) * np.repeat(e8m0_decode(scales), 32, axis=1)


# --------------------------------------------------------------------------------------
# S6 combine
# --------------------------------------------------------------------------------------

def combine(y, inv_perm, topk_w=None):
    """``out[t] = sum_k y[inv_perm[t,k]]`` in k order (times ``topk_w[t,k]`` when the route
    weight was not already applied in the activation) [trtllm: do_finalize; fi_ep: module
    docstring, the megakernel combines]."""
    y = np.asarray(y, dtype=np.float64)
    inv = np.asarray(inv_perm, dtype=np.int64)
    T, k = inv.shape
    out = np.zeros((T, y.shape[1]), dtype=np.float64)
    for j in range(k):
        rows = y[inv[:, j]]
        out += rows if topk_w is None else rows * np.asarray(topk_w, np.float64)[:, j:j + 1]
    return out


# --------------------------------------------------------------------------------------
# The whole layer
# --------------------------------------------------------------------------------------

def weighted_input(x, w_top1):
    """The experts' input when the top-1 route weight is applied on the input side.

    With ``apply_router_weight_on_input`` the MoonEP experts skip their own weight multiply
    because the weighting already happened before dispatch [moonep: MoonEPExperts.apply], so
    what the experts receive is an activation tensor in the model's dtype: x scaled by its
    weight. Reading taken: the product of the bf16 x and the fp32 weight is formed in fp32 and
    rounded once to bf16 (RNE). The dynamic activation quantisation of the experts' input
    [fi_ep: FlashInferMoeEpExperts docstring; dsv4_fi: forward, quantize_input] then applies
    to this tensor, like to any other input of the experts. Returns bf16 ``[T,H]``.
    """
    wt = torch.from_numpy(np.asarray(w_top1, dtype=np.float32).reshape(-1, 1))
    return (x.float() * wt).to(torch.bfloat16)


def moe_forward(cfg, x, logits, replica_src, w_gate, w_up, w_down, *,
                tokens=None, apply_topk_in_fc1: bool = True, keep: bool = False, routing_bias=None,
                given_topk=None, apply_router_weight_on_input: bool = False, biases=None):
    """The fused expert layer: route -> permute -> gate/up grouped GEMMs -> activation times
    route weight -> down grouped GEMM -> combine [moonep: module docstring and apply;
    trtllm: _invoke_kernel; fi_ep: apply].

    ``cfg`` supplies E, B, topk, act, situ_alpha, situ_beta, act_quant and the routing method
    (``route``; ``routing_bias`` is the DeepSeekV3 method's selection bias). With act_quant = 1,
    x (in token order) and every activation row are NVFP4-quantised (``nvfp4_quantize_rows``)
    before their GEMM; with act_quant = 2 they are MXFP8-quantised (``mxfp8_quantize_rows``). ``tokens`` restricts the expert maths to the rows those tokens need
    (routing and permutation are always computed in full). With ``apply_topk_in_fc1`` false
    the route weight moves from the activation to the combine [fi_ep: apply_topk_in_fc1].

    ``biases = (b_gate [G,I], b_up [G,I], b_down [G,H])`` adds per-row biases to the GEMM
    outputs (gemm1_bias / gemm2_bias [trtllm: TrtLlmMxfp4ExpertsModular._invoke_kernel]):
    gate and up get theirs before the activation, and the down projection's is part of the
    expert's output, so it is scaled by the route weight with it.

    ``given_topk = (ids, w)`` skips the routing: the experts and route weights are given, as
    in the modular and routed kernels that take a computed top-k [fi_ep: apply, topk_ids and
    topk_weights; trtllm: _invoke_kernel]. ``apply_router_weight_on_input`` (top-1 only)
    scales x by its route weight before the experts and leaves the activation unweighted:
    the MoonEP experts skip their weight multiply in that case because the weighting
    happened before dispatch [moonep: MoonEPExperts.apply].

    Returns a dict: ids, w, row, cu_seqlens, perm_token, perm_k, perm_w, inv_perm, tokens and
    out (fp64 ``[len(tokens), H]``); with ``keep``, also xq (codes/sb/s), the experts' input
    x_exp (token order, after any input weighting and quantisation), the activation rows
    h_pre (before their quantisation) and h (as the down GEMM takes them), and y rows.
    """
    if given_topk is not None:
        ids = np.asarray(given_topk[0], dtype=np.int32)
        w = np.asarray(given_topk[1], dtype=np.float32).astype(np.float64)
    else:
        ids, w = route(cfg, logits, routing_bias)
    if apply_router_weight_on_input and ids.shape[1] != 1:
        raise ValueError("apply_router_weight_on_input needs top-1 routing")
    perm = assign_rows(ids, cfg.E, cfg.B, replica_src)
    T, k = ids.shape
    inv = perm["inv_perm"]
    perm_w = w[perm["perm_token"], perm["perm_k"]] if T else np.zeros(0)
    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    need = np.zeros(T * k, dtype=bool)
    need[inv[tok].reshape(-1)] = True

    x_in = x
    if apply_router_weight_on_input:
        x_in = weighted_input(x, w[:, 0])
        apply_topk_in_fc1 = True          # the activation takes no weight (perm_w below is ignored)
        perm_w = np.ones_like(perm_w)
    x64 = to_f64(x_in)
    res = dict(ids=ids, w=w, perm_w=perm_w, tokens=tok, **perm)
    # the dynamic activation quantisers see what the experts see: x, or x times its weight
    if cfg.act_quant == 1:
        codes, sb, s = nvfp4_quantize_rows(np.asarray(x_in.float().numpy(), np.float32))
        x64 = nvfp4_dequantize_rows(codes, sb, s)
        if keep:
            res.update(xq_codes=codes, xq_sb=sb, xq_s=s)
    elif cfg.act_quant == 2:
        codes, sc = mxfp8_quantize_rows(np.asarray(x_in.float().numpy(), np.float32))
        x64 = mxfp8_dequantize_rows(codes, sc)
        if keep:
            res.update(xq_codes=codes, xq_scales=sc)

    a_g, a_u, a_d = weight_alpha(w_gate), weight_alpha(w_up), weight_alpha(w_down)
    y = np.zeros((T * k, w_down.N), dtype=np.float64)
    h_keep = np.zeros((T * k, w_gate.N), dtype=np.float64) if keep else None
    h_pre_keep = np.zeros((T * k, w_gate.N), dtype=np.float64) if keep else None
    for g, (s0, s1) in enumerate(segment_bounds(perm["cu_seqlens"])):
        rows = np.nonzero(need[s0:s1])[0] + s0
        if len(rows) == 0:
            continue
        a = x64[perm["perm_token"][rows]]
        gate = a_g[g] * (a @ weight_rows(w_gate, g).T)
        up = a_u[g] * (a @ weight_rows(w_up, g).T)
        if biases is not None:
            gate = gate + to_f64(biases[0][g])[None, :]
            up = up + to_f64(biases[1][g])[None, :]
        h = act_and_mul(gate, up, cfg.act, cfg.situ_alpha, cfg.situ_beta,
                        perm_w[rows] if apply_topk_in_fc1 else None, cfg.swiglu_alpha, cfg.swiglu_beta,
                        cfg.swiglu_limit)
        if keep:
            h_pre_keep[rows] = h
        if cfg.act_quant == 1:
            hc, hsb, hs = nvfp4_quantize_rows(h.astype(np.float32))
            h = nvfp4_dequantize_rows(hc, hsb, hs)
        elif cfg.act_quant == 2:
            hc, hsc = mxfp8_quantize_rows(h.astype(np.float32))
            h = mxfp8_dequantize_rows(hc, hsc)
        if keep:
            h_keep[rows] = h
        y[rows] = a_d[g] * (h @ weight_rows(w_down, g).T)
        if biases is not None:   # the expert's own bias, under the route weight when it is in h
            wb = perm_w[rows] if apply_topk_in_fc1 else np.ones(len(rows))
            y[rows] += wb[:, None] * to_f64(biases[2][g])[None, :]
    out = combine(y, inv[tok], None if apply_topk_in_fc1 else w[tok])
    res["out"] = out
    res["apply_topk_in_fc1"] = apply_topk_in_fc1
    if keep:
        res.update(h=h_keep, h_pre=h_pre_keep, y=y, x_exp=x64)
    return res
