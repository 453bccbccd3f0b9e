"""Shared helpers of the GPU parity tests: tolerances and comparisons against the oracle.

Tolerances (written out in the tests that use them):
* indices (topk ids, cu_seqlens, perm_token, inv_perm, quantised codes): bit-exact;
* BF16 outputs: |gpu - ref| <= 2e-2 + 2^-8 |ref| elementwise and rel-L2 <= 1e-2. The 2^-8|ref|
  term is the bf16 rounding of the output itself (round to nearest with 8 significant bits:
  at most 2^-8 of the value), which alone exceeds an absolute 2e-2 at |ref| > 5; the absolute
  term covers the bf16 rounding of the intermediate activation;
* FP4-weight layers: an element-wise bound derived from the layer's arithmetic
  (fp4_layer_bound, below) and rel-L2 <= 3e-2;
* MXFP4-weight GEMMs stage the bf16 activations as two e4m3 terms with one e8m0 scale per
  32 values: every activation x is carried to within 1.07 * 2^-8 |x| + 2^(e-10), where
  2^e < 2 amax_b / 448 for the amax of its 32-value block. An output then lies within
  sum_k |W[n,k]| (0.0042 |x_k| + 5e-6 amax_b(k)) of the exact result, plus its own bf16
  rounding (mx8_staging_bound).
"""
import numpy as np
import torch

BF16_ATOL = 2e-2
BF16_RTOL = 2.0 ** -8
BF16_REL_L2 = 1e-2
FP4_REL_L2 = 3e-2


def to_dev(t):
    return None if t is None else t.cuda().contiguous()


def rel_l2(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def check_bf16(got, ref, atol=BF16_ATOL, rtol=BF16_RTOL, rel=BF16_REL_L2, what=""):
    got = got.float().cpu().numpy().astype(np.float64) if isinstance(got, torch.Tensor) else got
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    worst = np.unravel_index(np.argmax(err - bound), err.shape) if err.size else None
    assert err.size == 0 or np.all(err <= bound), \
        f"{what}: max excess {np.max(err - bound):.3e} at {worst}: got {got[worst]} ref {ref[worst]}"
    r = rel_l2(got, ref)
    assert r <= rel, f"{what}: rel-L2 {r:.3e} > {rel}"
    return float(np.max(err)) if err.size else 0.0, r


def mx8_staging_bound(a, ws, cu_seqlens, M_alloc):
    """Per-output bound of the MXFP4 GEMM's activation staging error (module docstring):
    sum_k |W_g[n,k]| * (0.0042 |a[r,k]| + 5e-6 amax of a[r]'s 32-value block holding k)."""
    from oracle import moe_oracle as O

    a = np.asarray(a, np.float64)
    M, K = a.shape
    amax = np.repeat(np.abs(a).reshape(M, K // 32, 32).max(axis=2), 32, axis=1)
    per = 0.0042 * np.abs(a) + 5e-6 * amax
    alpha = O.weight_alpha(ws)
    out = np.zeros((M_alloc, ws.N))
    for g, (s, e) in enumerate(O.segment_bounds(cu_seqlens)):
        if e > s:
            out[s:e] = alpha[g] * (per[s:e] @ np.abs(O.weight_rows(ws, g)).T)
    return out


def check_mx8(got, ref, bound, what=""):
    """|got - ref| <= staging bound + 2^-8 |ref| (the bf16 output) + 1e-6 max|ref|."""
    got = got.float().cpu().numpy().astype(np.float64) if isinstance(got, torch.Tensor) else got
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    lim = bound + 2.0 ** -8 * np.abs(ref) + 1e-6 * max(np.abs(ref).max(), 1e-30)
    worst = np.unravel_index(np.argmax(err - lim), err.shape) if err.size else None
    assert err.size == 0 or np.all(err <= lim), \
        f"{what}: max excess {np.max(err - lim):.3e} at {worst}: got {got[worst]} ref {ref[worst]}"
    return rel_l2(got, ref)


def routing_kwargs(cfg, inp):
    """MoEForward's routing arguments for a workload (the DeepSeekV3 method's bias on the GPU)."""
    bias = inp.extra.get("routing_bias")
    return dict(routing=cfg.routing, routing_bias=None if bias is None else to_dev(bias), n_group=cfg.n_group,
                topk_group=cfg.topk_group, routed_scaling_factor=cfg.routed_scaling_factor)


def oracle_bias(inp):
    """The DeepSeekV3 selection bias for the oracle, or None."""
    bias = inp.extra.get("routing_bias")
    return None if bias is None else bias.numpy()


# ------------------------------------------------------------------ FP4-weight layers, element-wise
#
# An FP4-weight layer on the GPU differs from the oracle (same dequantised weights, fp64, no
# intermediate rounding) only where its arithmetic differs. Walking the layer once:
#
#   x -> a1       the gate/up operand. Dynamic NVFP4 / MXFP8 codes and the f16 staging of
#                 NVFP4-weight rows are exact; the MXFP4 hi/lo staging carries each value to
#                 within b = 0.0042|v| + 5e-6 amax_b (module docstring).
#   gate, up      fp32 accumulation of exact products: within GAMMA * sum_k |W||a1| of the
#                 exact sum (GAMMA: a generous multiple of fp32's rounding), plus the operand
#                 error carried by W.
#   h = act(g,u)  the activation's local Lipschitz constants in g and u (bounds below), plus
#                 ~1e-6 |h| from the epilogue's exp/division; times the route weight when the
#                 activation carries it.
#   h -> a2       the down operand: hi/lo staging or f16 rounding, or dynamic NVFP4 / MXFP8
#                 codes, where fp32 decides an integer. For the codes, the quantiser's inputs
#                 are known only to within the band TAIL * sigma_h, so its scales and codes are
#                 taken over that band: a code can differ from the oracle's only where the band
#                 straddles a rounding boundary, and then by one grid step (a "flip").
#   y = h W_d^T   as for gate/up.
#   out           the sum over the token's k rows (times the route weight when the combine
#                 carries it) in fp32, then one bf16 rounding (at most 2^-8 of the value).
#
# Rounding and staging errors are independent and zero-mean, each within its bound b, so they
# are tracked as standard deviations (sigma <= b / sqrt(3) for a uniform error, and b itself is
# used where the distribution is unknown) combined in quadrature through every dot product and
# linearly through the activation. The check allows TAIL = 6 standard deviations (a normal tail
# of 2e-9 per element) plus, in full, the flips' worst-case effect and the output rounding, and
# also requires rel-L2 <= 3e-2 overall (the stated FP4 tolerance).

GAMMA = 2.0 ** -18           # fp32 accumulation of a dot product, relative to sum |W||a|
TAIL = 6.0


def _block_amax(v, n):
    R, K = v.shape
    return np.repeat(np.abs(v).reshape(R, K // n, n).max(axis=2), n, axis=1)


def _hilo_err(v):
    return 0.0042 * np.abs(v) + 5e-6 * _block_amax(v, 32)


def _grid_round(z, grid, up):
    """z (fp64, >= 0, may be inf) rounded to the nearest entry of an ascending grid,
    saturating; an exact tie goes up when ``up`` else down (the conservative end of an
    interval whichever way the quantiser breaks ties)."""
    z = np.minimum(z, grid[-1])
    hi = np.clip(np.searchsorted(grid, z, side="left"), 0, len(grid) - 1)
    lo = np.clip(hi - 1, 0, len(grid) - 1)
    dlo, dhi = z - grid[lo], grid[hi] - z
    pick_hi = (dhi < dlo) | ((dhi == dlo) & up)
    return np.where(pick_hi, grid[hi], grid[lo])


def _quant_interval_err(v, e, ref_deq, mode):
    """Largest |q(v') - ref_deq| over quantiser inputs v' within e of v (row-wise NVFP4 when
    mode == 1, MXFP8 when mode == 2): scales and codes taken over the interval."""
    from oracle import moe_oracle as O

    slack = 1.0 + 2.0 ** -20                      # fp32 rounding of the scale arithmetic
    av = np.abs(v)
    lo_v, hi_v = np.maximum(av - e, 0.0) / slack, (av + e) * slack
    e4 = O.e4m3_decode(np.arange(0, 127))
    if mode == 1:
        A_lo, A_hi = lo_v.max(axis=1, keepdims=True), hi_v.max(axis=1, keepdims=True)
        s_lo, s_hi = A_lo / 2688.0, A_hi / 2688.0
        b_lo, b_hi = _block_amax(lo_v, 16), _block_amax(hi_v, 16)
        with np.errstate(divide="ignore", invalid="ignore"):
            r_lo = np.where(s_hi > 0, b_lo / (6.0 * s_hi), 0.0) / slack
            r_hi = np.where(s_lo > 0, b_hi / (6.0 * s_lo), np.inf) * slack
        P_lo = _grid_round(r_lo, e4, False) * s_lo / slack
        P_hi = _grid_round(r_hi, e4, True) * s_hi * slack
        grid = O.E2M1_MAG
    else:
        b_lo, b_hi = _block_amax(lo_v, 32), _block_amax(hi_v, 32)
        E_lo = np.where(b_lo > 0, np.floor(np.log2(np.where(b_lo > 0, b_lo, 1.0))), -127.0)
        E_hi = np.where(b_hi > 0, np.floor(np.log2(np.where(b_hi > 0, b_hi, 1.0))), -127.0)
        P_lo = np.ldexp(1.0, np.clip(E_lo - 8, -127, 127).astype(np.int64))
        P_hi = np.ldexp(1.0, np.clip(E_hi - 8, -127, 127).astype(np.int64))
        grid = e4
    with np.errstate(divide="ignore", invalid="ignore"):
        z_lo = np.where(P_hi > 0, lo_v / P_hi, 0.0)
        z_hi = np.where(P_lo > 0, hi_v / P_lo, np.inf)
    d_lo = _grid_round(z_lo, grid, False) * P_lo
    d_hi = _grid_round(z_hi, grid, True) * P_hi
    sgn = np.sign(v)
    err = np.maximum(np.abs(sgn * d_lo - ref_deq), np.abs(sgn * d_hi - ref_deq))
    # an input that may cross zero may take either sign
    return np.where(av <= e, np.abs(ref_deq) + d_hi, err)


def _sd(e, W2):
    """Standard deviation of sum_k W[n,k] d[r,k] for independent errors of sd e[r,k]
    (``W2`` = W * W)."""
    return np.sqrt((np.asarray(e, np.float32) ** 2) @ W2.T).astype(np.float64)


class _Dequant:
    """Dequantised weight rows in fp32 through 256-entry tables built from the oracle's pinned
    codecs (the bound needs magnitudes, not fp64 sums; this is several times faster than the
    oracle's own per-code decoding at full size)."""

    def __init__(self, ws):
        from oracle import moe_oracle as O

        self.ws = ws
        b = np.arange(256)
        self.lut = np.stack([O.e2m1_decode(b & 15), O.e2m1_decode(b >> 4)], axis=1).astype(np.float32)
        if ws.fmt == "mxfp4":
            self.slut, self.blk = O.e8m0_decode(b).astype(np.float32), 32
        elif ws.fmt == "nvfp4":
            self.slut, self.blk = np.nan_to_num(O.e4m3_decode(b)).astype(np.float32), 16

    def __call__(self, g):
        ws = self.ws
        if ws.fmt == "bf16":
            return ws.data[g].float().numpy()
        q = self.lut[ws.data[g].numpy()].reshape(ws.N, ws.K)
        return q * np.repeat(self.slut[ws.scale[g].numpy()], self.blk, axis=-1)


def fp4_layer_bound(cfg, inp, ref, gamma=GAMMA, tail=TAIL):
    """Element-wise bound on |gpu - oracle| for the rows ``ref["tokens"]`` of an FP4-weight
    layer (see the walk above). ``ref`` is the oracle's result with keep=True."""
    from oracle import moe_oracle as O

    r3 = 1.0 / np.sqrt(3.0)
    wg, wu, wd = inp.w_gate, inp.w_up, inp.w_down
    ag, au, ad = O.weight_alpha(wg), O.weight_alpha(wu), O.weight_alpha(wd)
    x_exp = np.asarray(ref["x_exp"], np.float64)
    perm_token, cu = ref["perm_token"], ref["cu_seqlens"]
    inv, tok = np.asarray(ref["inv_perm"]), np.asarray(ref["tokens"])
    k = inv.shape[1]
    in_fc1 = ref["apply_topk_in_fc1"]
    pw = np.asarray(ref["perm_w"], np.float64)
    need = np.zeros(len(perm_token), dtype=bool)
    need[inv[tok].reshape(-1)] = True
    sd_y = np.zeros((len(perm_token), wd.N))        # standard deviation of y's error
    fl_y = np.zeros((len(perm_token), wd.N))        # worst-case effect of code flips on y
    y_abs = np.zeros((len(perm_token), wd.N))
    biases = inp.extra.get("biases") if getattr(cfg, "bias", False) else None
    dq = [_Dequant(w) for w in (wg, wu, wd)]

    def segment(g, s0, s1):
        rows = np.nonzero(need[s0:s1])[0] + s0
        if len(rows) == 0:
            return
        a1 = x_exp[perm_token[rows]].astype(np.float32)
        if cfg.wfmt == "mxfp4" and cfg.act_quant == 0:
            sd_a1 = r3 * _hilo_err(a1)
        elif cfg.wfmt == "nvfp4" and cfg.act_quant == 0:
            sd_a1 = 2.0 ** -29 * np.abs(a1).max(axis=1, keepdims=True) * np.ones_like(a1)
        else:
            sd_a1 = np.zeros_like(a1)
        Wg, Wu, Wd = (d(g) for d in dq)
        Wg2, Wu2, Wd2 = Wg * Wg, Wu * Wu, Wd * Wd
        G = ag[g] * (a1 @ Wg.T)
        U = au[g] * (a1 @ Wu.T)
        if biases is not None:
            G = G + O.to_f64(biases[0][g])[None, :]
            U = U + O.to_f64(biases[1][g])[None, :]
        # accumulation: GAMMA * sum_k |W||a| <= GAMMA * sqrt(K) * sqrt(sum_k W^2 a^2) (Cauchy-Schwarz)
        rk1 = np.sqrt(a1.shape[1])
        sd_g = np.sqrt((ag[g] * _sd(sd_a1, Wg2)) ** 2 + (ag[g] * gamma * rk1 * _sd(a1, Wg2) + 2.0 ** -23 * np.abs(G)) ** 2)
        sd_u = np.sqrt((au[g] * _sd(sd_a1, Wu2)) ** 2 + (au[g] * gamma * rk1 * _sd(a1, Wu2) + 2.0 ** -23 * np.abs(U)) ** 2)
        e_g, e_u = tail * sd_g, tail * sd_u            # the band the activation's inputs lie in
        Gm, Um = np.abs(G) + e_g, np.abs(U) + e_u
        # local Lipschitz constants of the activation in g and in u over that band
        if cfg.act == "silu":                          # |silu'| <= 1.1, |silu(g)| <= |g|
            d_g, d_u = 1.1 * Um, Gm
        elif cfg.act == "situ":
            # d/dg [a tanh(g/a) sigmoid(g)] <= sech^2(g/a) + a sigmoid'(g) and d/du [b tanh(u/b)]
            # = sech^2(u/b) both fall with |g|, |u|: their values at the band's point nearest
            # zero bound them on the band (a saturated gate is flat)
            a_, b_ = cfg.situ_alpha, cfg.situ_beta
            mg, mu = np.maximum(np.abs(G) - e_g, 0.0), np.maximum(np.abs(U) - e_u, 0.0)
            sg = 1.0 / (1.0 + np.exp(-mg))
            d_g = (1.0 / np.cosh(np.minimum(mg / a_, 300.0)) ** 2 + a_ * sg * (1.0 - sg)) * np.minimum(b_, Um)
            d_u = np.minimum(a_, Gm) / np.cosh(np.minimum(mu / b_, 300.0)) ** 2
        else:
            # swigluoai: g' = min(g, lim), u' = clamp(u, +-lim), h = g' sigmoid(al g') (u' + be).
            # d/dg' [g' sigmoid(al g')] <= 1.224 and is 0 where g is clamped; |u' + be| <=
            # min(|u|, lim) + |be|; |g' sigmoid(al g')| <= min(|g|, lim) for g > 0 and
            # <= min(|g|, 0.2785 / al) for g < 0 (the largest of y sigmoid(-y) is 0.2785)
            lim = np.inf if cfg.swiglu_limit is None else cfg.swiglu_limit
            al, be = cfg.swiglu_alpha, cfg.swiglu_beta
            clamped = (G - e_g) > lim
            d_g = np.where(clamped, 0.0, 1.224 * (np.minimum(Um, lim) + abs(be)))
            neg = np.minimum(Gm, 0.2785 / al) if al > 0 else Gm
            d_u = np.maximum(np.where(G + e_g > 0, np.minimum(Gm, lim), 0.0), np.where(G - e_g < 0, neg, 0.0))
        w_row = np.abs(pw[rows][:, None]) if in_fc1 else 1.0
        h_pre = np.asarray(ref["h_pre"][rows], np.float64)
        sd_h = w_row * np.sqrt((d_g * sd_g) ** 2 + (d_u * sd_u) ** 2) + 4e-6 * np.abs(h_pre) + 1e-30
        a2 = np.asarray(ref["h"][rows], np.float64)
        flips = np.zeros_like(a2)
        if cfg.act_quant in (1, 2):
            dev = _quant_interval_err(h_pre, tail * sd_h, a2, cfg.act_quant)
            # within the band the dequantised value follows h continuously (up to the scale's
            # own motion, already in `dev`) unless a code flips; count a flip where `dev` is
            # more than the band itself
            flip = dev > tail * sd_h * (1.0 + 2.0 ** -10) + 2.0 ** -20 * np.abs(a2)
            flips = np.where(flip, dev, 0.0)
            sd_a2 = np.where(flip, 0.0, np.maximum(sd_h, dev / tail))
        elif cfg.wfmt == "mxfp4":
            sd_a2 = np.sqrt(sd_h ** 2 + (r3 * _hilo_err(np.abs(h_pre) + tail * sd_h)) ** 2)
        else:                                          # f16 rows with a power-of-two scale
            sd_a2 = sd_h + 2.0 ** -11 * (np.abs(h_pre) + tail * sd_h) + \
                2.0 ** -25 * max(1.0, cfg.situ_alpha * cfg.situ_beta) + \
                2.0 ** -29 * np.abs(h_pre).max(axis=1, keepdims=True)
        rk2 = np.sqrt(a2.shape[1])
        sd_y[rows] = ad[g] * np.sqrt(_sd(sd_a2, Wd2) ** 2 + (gamma * rk2 * _sd(a2, Wd2)) ** 2)
        # the flips: their worst case, or the Hoeffding form (their signs against W's are
        # independent), whichever is smaller
        if np.any(flips):
            fl_y[rows] = ad[g] * np.minimum(flips @ np.abs(Wd).T, tail * _sd(flips, Wd2))
        y_abs[rows] = np.abs(ref["y"][rows])

    # segments write disjoint rows; numpy releases the GIL in the matmuls and large array ops
    import concurrent.futures as cf
    import os
    with cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(lambda t: segment(t[0], *t[1]), enumerate(O.segment_bounds(cu))))
    wt = np.ones((len(tok), k)) if in_fc1 else np.abs(np.asarray(ref["w"], np.float64)[tok])
    var = np.zeros((len(tok), wd.N))
    fl = np.zeros((len(tok), wd.N))
    for j in range(k):
        r = inv[tok, j]
        var += (wt[:, j:j + 1] * sd_y[r]) ** 2
        fl += wt[:, j:j + 1] * (fl_y[r] + 2.0 ** -22 * y_abs[r])
    # the output's bf16 rounding: at most 2^-8 of the value it rounds (8 significant bits)
    pre = tail * np.sqrt(var) + fl + 1e-6 * max(np.abs(ref["out"]).max(), 1e-30)
    return (1.0 + 2.0 ** -8) * pre + 2.0 ** -8 * np.abs(ref["out"])


def check_fp4_layer(out, ref, cfg, inp, what="", rel=FP4_REL_L2, gamma=GAMMA):
    """Element-wise |gpu - oracle| <= fp4_layer_bound, and rel-L2 <= 3e-2 (the stated FP4
    tolerance). ``out`` holds the rows ``ref["tokens"]``. Returns (rel-L2, the largest
    err/bound ratio)."""
    got = out.float().cpu().numpy().astype(np.float64) if isinstance(out, torch.Tensor) else np.asarray(out)
    refo = np.asarray(ref["out"], np.float64)
    assert got.shape == refo.shape, (got.shape, refo.shape)
    bound = fp4_layer_bound(cfg, inp, ref, gamma)
    err = np.abs(got - refo)
    ratio = err / bound
    worst = np.unravel_index(np.argmax(ratio), ratio.shape)
    assert np.all(err <= bound), \
        f"{what}: err {err[worst]:.3e} > bound {bound[worst]:.3e} at {worst}: got {got[worst]} ref {refo[worst]}"
    r = rel_l2(got, refo)
    assert r <= rel, f"{what}: rel-L2 {r:.3e} > {rel}"
    return r, float(ratio.max())
