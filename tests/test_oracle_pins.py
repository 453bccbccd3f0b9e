"""Pins for the CPU oracle: each checks it against something other than itself.

Codecs against the OCP MX element tables (tests/golden) and torch's float8 types; routing
against a brute-force loop written differently (repeated argmax, softmax over all experts);
the grouped GEMM against pure-Python dot products; activations against closed forms and
limits; the whole layer against a per-token loop with no permutation and against a dense
SwiGLU MLP; the NVFP4 activation quantiser against a brute-force nearest-grid-point search.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import workloads as W
from oracle import moe_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _read_pairs(name):
    rows = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                a, b = line.split()
                rows.append((float(a), float(b)))
    return rows


# ------------------------------------------------------------------ codecs

def test_e2m1_decode_matches_ocp_table():
    for code, val in _read_pairs("e2m1_ocp_mx_v1.txt"):
        got = O.e2m1_decode(np.array([int(code)]))[0]
        assert got == val and math.copysign(1, got) == math.copysign(1, val), (code, got, val)


def test_e2m1_encode_ties_and_saturation():
    for v, expect in _read_pairs("rne_ties.txt"):
        c = O.e2m1_encode(np.array([v], np.float32))[0]
        got = O.e2m1_decode(np.array([c]))[0]
        assert got == expect and math.copysign(1, got) == math.copysign(1, expect), (v, got, expect)


def test_e4m3_decode_matches_torch_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_decode(np.arange(256))
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.all(both_nan | (ref == got))
    assert O.e4m3_decode(np.array([0x7E]))[0] == 448.0


def test_e8m0_decode_matches_torch():
    if not hasattr(torch, "float8_e8m0fnu"):
        pytest.skip("torch without float8_e8m0fnu")
    codes = torch.arange(255, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    assert np.array_equal(ref, O.e8m0_decode(np.arange(255)))
    assert np.isnan(O.e8m0_decode(np.array([255]))[0])


def test_e4m3_encode_matches_torch_rne():
    g = torch.Generator().manual_seed(3)
    v = torch.cat([torch.rand(20000, generator=g) * 448.0,
                   torch.rand(20000, generator=g) * 0.02,          # subnormal range
                   torch.tensor([0.0, 2.0 ** -10, 3 * 2.0 ** -11, 448.0, 464.0 - 1e-3])])
    ref = v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_encode(v.numpy())
    assert np.array_equal(ref, got)
    assert O.e4m3_encode(np.array([1e6], np.float32))[0] == 0x7E       # satfinite
    assert O.e4m3_encode(np.array([-1e6], np.float32))[0] == 0xFE


@pytest.mark.parametrize("enc,dec,n", [(O.e2m1_encode, O.e2m1_decode, 16),
                                       (O.e4m3_encode, O.e4m3_decode, 256)])
def test_encode_is_nearest_grid_point(enc, dec, n):
    grid = dec(np.arange(n))
    grid = grid[np.isfinite(grid)]
    vmax = np.max(grid)
    rng = np.random.default_rng(0)
    v = (rng.standard_normal(5000) * vmax / 3).astype(np.float32)
    c = enc(v)
    got = dec(c)
    best = np.min(np.abs(np.minimum(np.abs(v), vmax)[:, None] - np.abs(grid)[None, :]), axis=1)
    assert np.allclose(np.abs(np.minimum(np.abs(v), vmax) - np.abs(got)), best, rtol=0, atol=0)
    assert np.all(np.signbit(got) == np.signbit(v))


def test_unpack_nibble_order():
    p = np.array([[0x21, 0xF0]], dtype=np.uint8)
    assert O.unpack_e2m1(p).tolist() == [[1, 2, 0, 15]]


# ------------------------------------------------------------------ routing

def _route_brute(logits, k):
    """Repeated argmax (first maximum = lowest id) and a full softmax, renormalised."""
    L = np.asarray(logits, np.float32).astype(np.float64)
    T, E = L.shape
    ids = np.zeros((T, k), np.int64)
    w = np.zeros((T, k))
    for t in range(T):
        avail = list(range(E))
        for j in range(k):
            best = avail[0]
            for e in avail[1:]:
                if L[t, e] > L[t, best]:
                    best = e
            ids[t, j] = best
            avail.remove(best)
        p = [math.exp(L[t, e]) for e in range(E)]
        tot = sum(p)
        sel = [p[e] / tot for e in ids[t]]
        w[t] = [q / sum(sel) for q in sel]
    return ids, w


@pytest.mark.parametrize("T,E,k,int_logits", [(64, 8, 2, False), (64, 8, 2, True),
                                              (33, 16, 5, True), (20, 64, 8, False), (7, 4, 4, True)])
def test_route_matches_bruteforce(T, E, k, int_logits):
    g = torch.Generator().manual_seed(T * E + k)
    L = torch.randn(T, E, generator=g)
    if int_logits:
        L = torch.randint(-2, 3, (T, E), generator=g).float()
        L[0, :] = 0.0
        L[1, ::2] = -0.0        # -0 ties +0
    ids, w = O.route_topk(L.numpy(), k)
    bids, bw = _route_brute(L.numpy(), k)
    assert np.array_equal(ids, bids)
    assert np.allclose(w, bw, rtol=1e-13, atol=1e-15)
    assert np.allclose(w.sum(1), 1.0, atol=1e-14)
    for t in range(T):
        assert len(set(ids[t].tolist())) == k
        sl = L.numpy()[t, ids[t]]
        assert np.all(np.diff(sl) <= 0)


def test_route_empty_and_full_k():
    ids, w = O.route_topk(np.zeros((0, 8), np.float32), 2)
    assert ids.shape == (0, 2)
    ids, w = O.route_topk(np.zeros((3, 4), np.float32), 4)
    assert ids.tolist() == [[0, 1, 2, 3]] * 3 and np.allclose(w, 0.25)


# ------------------------------------------------------------------ permutation

def _perm_case(T, E, k, B, used, seed):
    g = torch.Generator().manual_seed(seed)
    L = torch.randn(T, E, generator=g) * 2
    ids, w = O.route_topk(L.numpy(), k)
    src = -np.ones(B, np.int64)
    if B:
        src[:used] = torch.randperm(E, generator=g)[:used].numpy()
    return ids, w, src


def _grouped_brute(logits, bias, k, n_group, topk_group, scale):
    """DeepSeekV3 routing by exhaustion: the group subset of size topk_group with the largest
    total group score (ties: the lexicographically smallest ids), then repeated argmax of
    sigmoid + bias over its experts; weights from the plain sigmoid, pure Python."""
    L = np.asarray(logits, np.float32).astype(np.float64)
    b = np.asarray(bias, np.float32).astype(np.float64)
    T, E = L.shape
    gs = E // n_group
    ids = np.zeros((T, k), np.int64)
    w = np.zeros((T, k))
    for t in range(T):
        sg = [1.0 / (1.0 + math.exp(-L[t, e])) for e in range(E)]
        c = [sg[e] + b[e] for e in range(E)]
        gscore = []
        for g in range(n_group):
            vals = sorted(c[g * gs:(g + 1) * gs], reverse=True)
            gscore.append(vals[0] + (vals[1] if gs >= 2 else 0.0))
        best = None
        for sub in itertools.combinations(range(n_group), topk_group):
            tot = sum(gscore[g] for g in sub)
            if best is None or tot > best[0]:
                best = (tot, sub)
        avail = [e for g in best[1] for e in range(g * gs, (g + 1) * gs)]
        for j in range(k):
            pick = avail[0]
            for e in avail[1:]:
                if c[e] > c[pick] or (c[e] == c[pick] and e < pick):
                    pick = e
            ids[t, j] = pick
            avail.remove(pick)
        tot = sum(sg[e] for e in ids[t])
        w[t] = [scale * sg[e] / tot for e in ids[t]]
    return ids, w


@pytest.mark.parametrize("E,n_group,topk_group,k,ints", [(12, 4, 2, 3, False), (16, 4, 1, 4, False),
                                                         (24, 6, 3, 5, True), (8, 8, 3, 3, False),
                                                         (10, 1, 1, 4, False)])
def test_grouped_routing_matches_bruteforce(E, n_group, topk_group, k, ints):
    g = np.random.default_rng(E + k)
    L = g.normal(0, 2, (7, E)).astype(np.float32)
    if ints:
        L = np.round(L).astype(np.float32)      # many ties
    bias = (g.normal(0, 0.05, E)).astype(np.float32)
    ids, w = O.route_topk_grouped(L, k, n_group, topk_group, bias, 2.5)
    bi, bw = _grouped_brute(L, bias, k, n_group, topk_group, 2.5)
    assert np.array_equal(ids, bi)
    assert np.allclose(w, bw, rtol=1e-12, atol=0)


def test_grouped_routing_reductions_and_invariants():
    g = np.random.default_rng(3)
    L = g.normal(0, 2, (50, 64)).astype(np.float32)
    bias = g.normal(0, 0.05, 64).astype(np.float32)
    # one group, no bias: sigmoid is monotone, so the choice is the plain top-k of the logits
    ids, w = O.route_topk_grouped(L, 6, 1, 1, None, 1.0)
    ref_ids, _ = O.route_topk(L, 6)
    assert np.array_equal(ids, ref_ids)
    s = 1.0 / (1.0 + np.exp(-np.take_along_axis(L.astype(np.float64), ids.astype(np.int64), 1)))
    assert np.allclose(w, s / s.sum(1, keepdims=True), rtol=1e-12)
    # groups: every choice lies in at most topk_group groups, weights sum to the scaling factor
    ids, w = O.route_topk_grouped(L, 8, 8, 3, bias, 2.5)
    assert all(len(set((r // 8).tolist())) <= 3 for r in ids)
    assert np.allclose(w.sum(1), 2.5)
    # a constant added to every bias moves every group score alike: the choice is unchanged
    ids2, w2 = O.route_topk_grouped(L, 8, 8, 3, bias + np.float32(0.25), 2.5)
    assert np.array_equal(ids, ids2) and np.allclose(w, w2, rtol=1e-12)
    # all logits equal: the lowest groups, then the lowest ids
    ids, _ = O.route_topk_grouped(np.zeros((2, 8), np.float32), 3, 4, 2, None, 1.0)
    assert ids.tolist() == [[0, 1, 2], [0, 1, 2]]


@pytest.mark.parametrize("T,E,k,B,used", [(16, 8, 2, 0, 0), (50, 8, 3, 4, 2), (64, 16, 4, 6, 6),
                                          (1, 4, 1, 2, 1), (0, 4, 2, 2, 1)])
def test_permute_invariants(T, E, k, B, used):
    ids, w, src = _perm_case(T, E, k, B, used, seed=T + 7 * B)
    p = O.assign_rows(ids, E, B, src)
    cu, pt, pk, inv, row = p["cu_seqlens"], p["perm_token"], p["perm_k"], p["inv_perm"], p["row"]
    G = E + B
    assert cu.shape == (G,) and (G == 0 or cu[-1] == T * k)
    assert np.all(np.diff(np.concatenate([[0], cu])) >= 0)
    # every (t, j) appears exactly once; the permutation inverts
    assert sorted(zip(pt.tolist(), pk.tolist())) == [(t, j) for t in range(T) for j in range(k)]
    for t in range(T):
        for j in range(k):
            assert pt[inv[t, j]] == t and pk[inv[t, j]] == j
    # each segment: ascending token ids, rows of a replica serve only their source expert
    for g, (s0, s1) in enumerate(O.segment_bounds(cu)):
        toks = pt[s0:s1]
        assert np.all(np.diff(toks) > 0)
        expert = g if g < E else src[g - E]
        if g >= E and src[g - E] < 0:
            assert s1 == s0                           # unused slot is empty
        for q in range(s0, s1):
            assert ids[pt[q], pk[q]] == expert and row[pt[q], pk[q]] == g
    # replica split is balanced: sizes of an expert's rows differ by at most one, larger first
    for e in range(E):
        rows = [e] + [E + s for s in range(B) if src[s] == e]
        sizes = [cu[r] - (cu[r - 1] if r else 0) for r in rows]
        assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    # permute-then-unpermute identity on a payload
    x = np.arange(T * 3, dtype=np.float64).reshape(T, 3)
    xp = x[pt]
    for t in range(T):
        for j in range(k):
            assert np.array_equal(xp[inv[t, j]], x[t])


# ------------------------------------------------------------------ grouped GEMM

def test_grouped_gemm_matches_python_dots():
    seg = [3, 0, 4, 1]
    cu = np.cumsum(seg).astype(np.int32)
    a, wt, _ = W.gen_grouped_gemm_case(10, seg, 5, 6, seed=1)
    ws = W.WeightSet("bf16", wt)
    out = O.grouped_gemm(O.to_f64(a), ws, cu, M_alloc=10)
    A, Wf = a.double().tolist(), wt.double().tolist()
    start = 0
    for g, n in enumerate(seg):
        for r in range(start, start + n):
            for c in range(5):
                ref = sum(A[r][kk] * Wf[g][c][kk] for kk in range(6))
                assert abs(out[r, c] - ref) <= 1e-15 * max(1.0, abs(ref))
        start += n
    assert np.all(out[8:] == 0)                       # padding rows past cu[-1] are zero


def test_grouped_gemm_fp4_weights_scale_and_alpha():
    # NVFP4 codes for +1 (0x2) everywhere, block scales 1.0 (e4m3 0x38), alpha 2 -> a row sum times 2
    G, N, K = 2, 3, 32
    data = torch.full((G, N, K // 2), 0x22, dtype=torch.uint8)
    scale = torch.full((G, N, K // 16), 0x38, dtype=torch.uint8)
    ws = W.WeightSet("nvfp4", data, scale, torch.tensor([2.0, 0.5]))
    a = np.arange(4 * K, dtype=np.float64).reshape(4, K) / 7
    out = O.grouped_gemm(a, ws, np.array([1, 4], np.int32))
    assert np.allclose(out[0], 2.0 * a[0].sum()) and np.allclose(out[1:], 0.5 * a[1:].sum(1)[:, None])
    # MXFP4: code 0x7 (6.0) with e8m0 126 (0.5) -> every weight 3.0
    ws = W.WeightSet("mxfp4", torch.full((1, 2, K // 2), 0x77, dtype=torch.uint8),
                     torch.full((1, 2, K // 32), 126, dtype=torch.uint8))
    out = O.grouped_gemm(a[:2], ws, np.array([2], np.int32))
    assert np.allclose(out, 3.0 * a[:2].sum(1)[:, None])


# ------------------------------------------------------------------ activations

def test_silu_closed_forms():
    x = np.linspace(-30, 30, 601)
    one = np.ones_like(x)
    assert O.silu_and_mul(np.zeros(1), np.ones(1))[0] == 0.0
    # silu(x) - silu(-x) = x * (sigmoid(x) + sigmoid(-x)) = x
    assert np.allclose(O.silu_and_mul(x, one) - O.silu_and_mul(-x, one), x, atol=1e-12)
    assert np.allclose(O.silu_and_mul(x, 3 * one), 3 * O.silu_and_mul(x, one))
    assert np.all(O.silu_and_mul(x, one) >= -0.2785)   # global minimum of x*sigmoid(x)


def test_situ_limits_and_symmetries():
    rng = np.random.default_rng(1)
    g, u = rng.standard_normal(1000) * 3, rng.standard_normal(1000) * 3
    # alpha, beta -> infinity: alpha*tanh(x/alpha) -> x, so SITU -> silu(gate) * up
    big = O.situ_and_mul(g, u, 1e4, 1e4)
    assert np.allclose(big, O.silu_and_mul(g, u), rtol=1e-6, atol=1e-9)
    s = O.situ_and_mul(g, u, 1.0, 1.0)
    assert np.allclose(O.situ_and_mul(g, -u, 1.0, 1.0), -s)        # odd in the up input
    assert np.all(np.abs(O.situ_and_mul(g, u, 0.7, 1.3)) <= 0.7 * 1.3 + 1e-15)
    # gate -> +inf: left factor -> alpha; gate -> -inf: -> 0
    assert np.allclose(O.situ_and_mul(np.full(3, 50.0), np.array([0.1, 1, 9]), 2.0, 1.5),
                       2.0 * 1.5 * np.tanh(np.array([0.1, 1, 9]) / 1.5))
    assert np.allclose(O.situ_and_mul(np.full(3, -60.0), np.ones(3), 2.0, 1.5), 0.0, atol=1e-20)
    with pytest.raises(ValueError):
        O.situ_and_mul(g, u, 0.0, 1.0)


# ------------------------------------------------------------------ NVFP4 activation quant

def _quant_brute(row):
    """Per element: nearest point of the block's grid e2m1 * step, ties to the even code."""
    row = np.asarray(row, np.float32)
    amax = np.float32(np.max(np.abs(row)))
    s = np.float32(amax / np.float32(2688.0))
    codes = []
    for b in range(len(row) // 16):
        blk = row[16 * b:16 * b + 16]
        r = np.float32(np.float32(np.max(np.abs(blk))) / np.float32(np.float32(6.0) * s)) if s > 0 else 0.0
        sb = O.e4m3_encode(np.array([r], np.float32))[0]
        step = np.float32(np.float32(O.e4m3_decode(np.array([sb]))[0]) * s)
        for v in blk:
            if step == 0:
                codes.append(0)
                continue
            y = float(np.float32(v / step))
            best = min(range(16), key=lambda c: (abs(min(abs(y), 6.0) - O.E2M1_MAG[c & 7]), c & 1)
                       if (c >> 3) == (1 if math.copysign(1, y) < 0 else 0) else (1e9, 0))
            codes.append(best)
    return np.array(codes, np.uint8)


def test_nvfp4_quant_matches_bruteforce_and_bounds():
    x = W.gen_rows(6, 64, seed=5, dtype=torch.float32).numpy()
    x[2, 16:32] = 0.0                                   # an all-zero block
    x[3] *= 1e-3
    x[4, 5] = 40.0                                      # an outlier
    x[5] = 0.0                                          # an all-zero row
    codes, sb, s = O.nvfp4_quantize_rows(x)
    for r in range(6):
        assert np.array_equal(codes[r], _quant_brute(x[r])), r
    deq = O.nvfp4_dequantize_rows(codes, sb, s)
    assert np.all(deq[5] == 0) and s[5] == 0
    # the largest element of a row lands near the top of its block's range
    for r in range(5):
        i = int(np.argmax(np.abs(x[r])))
        assert abs(deq[r, i] - x[r, i]) <= 0.25 * abs(x[r, i])
    # values already on the grid quantise to themselves
    codes2, sb2, s2 = O.nvfp4_quantize_rows(deq.astype(np.float32))
    assert np.allclose(O.nvfp4_dequantize_rows(codes2, sb2, s2), deq, rtol=1e-6, atol=0)


def _mxfp8_brute(row):
    """Per element: the block's power-of-two scale from a loop over exponents, then the
    nearest point of the whole e4m3 grid times that scale (ties to the even code, beyond 448
    clamped to 448)."""
    grid = [float(O.e4m3_decode(np.array([c]))[0]) for c in range(127)]   # non-negative finite
    codes, scales = [], []
    for b in range(len(row) // 32):
        blk = [float(v) for v in row[32 * b:32 * b + 32]]
        amax = max(abs(v) for v in blk)
        if amax == 0:
            k = -127
        else:
            k = 0
            while 2.0 ** k > amax:
                k -= 1
            while 2.0 ** (k + 1) <= amax:
                k += 1
            k = max(-127, min(127, k - 8))
        scales.append(k + 127)
        X = 2.0 ** k
        for v in blk:
            a = min(abs(v) / X, 448.0)
            best = min(range(127), key=lambda c: (abs(grid[c] - a), c % 2))
            codes.append(best | (128 if math.copysign(1.0, v) < 0 else 0))
    return np.array(codes, np.uint8), np.array(scales, np.uint8)


def test_mxfp8_quant_matches_bruteforce_and_special_cases():
    x = W.gen_rows(4, 96, seed=7, dtype=torch.float32).numpy()
    x[1, 32:64] = 0.0                                   # an all-zero block
    x[2] *= 1e-4
    x[3, 0:32] = np.linspace(-1.0, 1.0, 32) * 1.9 * 8.0  # amax 15.2 -> v/X reaches 486 > 448: saturates
    codes, sc = O.mxfp8_quantize_rows(x)
    for r in range(4):
        bc, bs = _mxfp8_brute(x[r])
        assert np.array_equal(codes[r], bc), r
        assert np.array_equal(sc[r], bs), r
    assert sc[1, 1] == 0 and np.all(codes[1, 32:64] == 0)
    deq = O.mxfp8_dequantize_rows(codes, sc)
    assert sc[3, 0] == 127 + 3 - 8 and deq[3, 31] == 448.0 * 2.0 ** -5 and deq[3, 0] == -448.0 * 2.0 ** -5
    # a power of two is its block's amax exactly: scale 2^(k-8), code of 256
    y = np.zeros((1, 32), np.float32)
    y[0, 3] = 2.0 ** 5
    c1, s1 = O.mxfp8_quantize_rows(y)
    assert s1[0, 0] == 127 + 5 - 8 and O.e4m3_decode(c1[0, 3:4])[0] == 256.0
    # values already on the grid quantise to themselves
    c2, s2 = O.mxfp8_quantize_rows(deq.astype(np.float32))
    assert np.array_equal(O.mxfp8_dequantize_rows(c2, s2), deq)


# ------------------------------------------------------------------ the whole layer

def _layer_brute(cfg, inp, apply_topk_in_fc1=True, given=None, input_weight=False, biases=None):
    """Per token, per chosen expert, the expert MLP on that token alone: no permutation,
    own routing (or the given ids and weights), pure-Python dot products. With
    input_weight the token is scaled by its weight before the MLP, which is then unweighted."""
    if given is not None:
        ids, w = np.asarray(given[0]), np.asarray(given[1], np.float32).astype(np.float64)
    elif cfg.routing == "deepseek_v3":
        ids, w = _grouped_brute(inp.logits.numpy(), inp.extra["routing_bias"].numpy(), cfg.topk, cfg.n_group,
                                cfg.topk_group, cfg.routed_scaling_factor)
    else:
        ids, w = _route_brute(inp.logits.numpy(), cfg.topk)
    def expert_input(t, j):
        # with the weight on the input: bf16 x times the fp32 weight in fp32, rounded to
        # bf16, and only then quantised, one token row at a time
        row = inp.x[t:t + 1].float()
        if input_weight:
            row = torch.tensor([[float(np.float32(v) * np.float32(w[t, j])) for v in row[0].tolist()]],
                               dtype=torch.float32).to(torch.bfloat16).float()
        r = row.numpy()
        if cfg.act_quant == 1:
            c, sb, s = O.nvfp4_quantize_rows(r)
            return O.nvfp4_dequantize_rows(c, sb, s)[0].tolist()
        if cfg.act_quant == 2:
            c, sc = O.mxfp8_quantize_rows(r)
            return O.mxfp8_dequantize_rows(c, sc)[0].tolist()
        return r[0].astype(np.float64).tolist()

    ag, au, ad = (O.weight_alpha(inp.w_gate), O.weight_alpha(inp.w_up), O.weight_alpha(inp.w_down))
    out = np.zeros((cfg.T, cfg.H))
    Wg = [O.weight_rows(inp.w_gate, e).tolist() for e in range(cfg.E)]
    Wu = [O.weight_rows(inp.w_up, e).tolist() for e in range(cfg.E)]
    Wd = [O.weight_rows(inp.w_down, e).tolist() for e in range(cfg.E)]
    for t in range(cfg.T):
        for j in range(cfg.topk):
            xt = expert_input(t, j)
            e = int(ids[t, j])
            gate = [ag[e] * sum(a * b for a, b in zip(row, xt)) for row in Wg[e]]
            up = [au[e] * sum(a * b for a, b in zip(row, xt)) for row in Wu[e]]
            if biases is not None:
                gate = [v + float(b) for v, b in zip(gate, biases[0][e])]
                up = [v + float(b) for v, b in zip(up, biases[1][e])]
            if cfg.act == "silu":
                h = [gg / (1 + math.exp(-gg)) * uu for gg, uu in zip(gate, up)]
            elif cfg.act == "swigluoai":
                lim, al, be = cfg.swiglu_limit, cfg.swiglu_alpha, cfg.swiglu_beta
                h = []
                for gg, uu in zip(gate, up):
                    if lim is not None:
                        gg, uu = min(gg, lim), max(-lim, min(uu, lim))
                    h.append(gg / (1 + math.exp(-al * gg)) * (uu + be))
            else:
                al, be = cfg.situ_alpha, cfg.situ_beta
                h = [al * math.tanh(gg / al) / (1 + math.exp(-gg)) * be * math.tanh(uu / be)
                     for gg, uu in zip(gate, up)]
            if apply_topk_in_fc1 and not input_weight:
                h = [v * w[t, j] for v in h]
            if cfg.act_quant == 1:
                c, sb, s = O.nvfp4_quantize_rows(np.array([h], np.float32))
                h = O.nvfp4_dequantize_rows(c, sb, s)[0].tolist()
            elif cfg.act_quant == 2:
                c, sc = O.mxfp8_quantize_rows(np.array([h], np.float32))
                h = O.mxfp8_dequantize_rows(c, sc)[0].tolist()
            y = [ad[e] * sum(a * b for a, b in zip(row, h)) for row in Wd[e]]
            if biases is not None:   # the bias is part of the expert's output, under its weight
                bw = w[t, j] if (apply_topk_in_fc1 and not input_weight) else 1.0
                y = [v + bw * float(b) for v, b in zip(y, biases[2][e])]
            wt = 1.0 if (apply_topk_in_fc1 or input_weight) else w[t, j]
            out[t] += wt * np.array(y)
    return out


SMALL = {
    "tiny": W.CONFIGS["tiny"],
    "replicas": W.MoEConfig("replicas", T=12, H=32, I=48, E=6, topk=3, B=4, B_used=3, logit_std=2.0),
    "mxfp4_situ": W.MoEConfig("mxfp4_situ", T=8, H=64, I=64, E=4, topk=2, act="situ",
                              situ_alpha=0.8, situ_beta=1.7, wfmt="mxfp4"),
    "nvfp4_quant": W.MoEConfig("nvfp4_quant", T=8, H=64, I=32, E=4, topk=2, wfmt="nvfp4",
                               act_quant=1),
    "mxfp4_w4a8": W.MoEConfig("mxfp4_w4a8", T=8, H=64, I=64, E=4, topk=2, act="situ", wfmt="mxfp4",
                              act_quant=2),
    "grouped_routing": W.MoEConfig("grouped_routing", T=10, H=32, I=48, E=8, topk=3, routing="deepseek_v3",
                                   n_group=4, topk_group=2, routed_scaling_factor=2.5, logit_std=2.0),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_layer_matches_per_token_loop(name):
    cfg = SMALL[name]
    inp = W.gen_inputs(cfg)
    bias = inp.extra.get("routing_bias")
    res = O.moe_forward(cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(),
                        inp.w_gate, inp.w_up, inp.w_down, routing_bias=None if bias is None else bias.numpy())
    ref = _layer_brute(cfg, inp)
    scale = np.max(np.abs(ref))
    if cfg.act_quant:
        # the activation codes are decided in fp32 on values whose fp64 rounding order
        # differs between the two loops; a flipped code moves one element by one step
        assert np.linalg.norm(res["out"] - ref) <= 1e-3 * np.linalg.norm(ref)
    else:
        assert np.max(np.abs(res["out"] - ref)) <= 1e-12 * scale


def test_layer_weight_in_combine_equals_weight_in_activation():
    cfg = SMALL["replicas"]
    inp = W.gen_inputs(cfg)
    args = (cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up, inp.w_down)
    a = O.moe_forward(*args)["out"]
    b = O.moe_forward(*args, apply_topk_in_fc1=False)["out"]
    assert np.allclose(a, b, rtol=1e-12, atol=1e-14)


def test_layer_redundant_slots_do_not_change_output():
    cfg = SMALL["replicas"]
    inp = W.gen_inputs(cfg)
    a = O.moe_forward(cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(),
                      inp.w_gate, inp.w_up, inp.w_down)["out"]
    cfg0 = cfg.with_(B=0, B_used=0)
    strip = lambda ws: W.WeightSet(ws.fmt, ws.data[:cfg.E])
    b = O.moe_forward(cfg0, inp.x, inp.logits.numpy(), np.zeros(0, np.int32),
                      strip(inp.w_gate), strip(inp.w_up), strip(inp.w_down))["out"]
    assert np.allclose(a, b, rtol=1e-12, atol=1e-14)


def test_layer_single_expert_is_dense_swiglu():
    cfg = W.MoEConfig("dense", T=9, H=40, I=24, E=1, topk=1)
    inp = W.gen_inputs(cfg)
    res = O.moe_forward(cfg, inp.x, inp.logits.numpy(), np.zeros(0, np.int32),
                        inp.w_gate, inp.w_up, inp.w_down)
    x = inp.x.double()
    wg, wu, wd = (inp.w_gate.data[0].double(), inp.w_up.data[0].double(), inp.w_down.data[0].double())
    ref = torch.nn.functional.silu(x @ wg.T) * (x @ wu.T) @ wd.T       # textbook SwiGLU MLP
    assert np.allclose(res["w"], 1.0)
    assert np.allclose(res["out"], ref.numpy(), rtol=1e-12, atol=1e-14)


def test_layer_token_subset_matches_full():
    cfg = SMALL["replicas"]
    inp = W.gen_inputs(cfg)
    args = (cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up, inp.w_down)
    full = O.moe_forward(*args)["out"]
    sub = O.moe_forward(*args, tokens=[0, 5, 11])["out"]
    assert np.allclose(sub, full[[0, 5, 11]], rtol=1e-13, atol=1e-16)   # BLAS order may differ


def test_workload_generator_is_deterministic_and_replicas_copy():
    cfg = SMALL["replicas"]
    a, b = W.gen_inputs(cfg), W.gen_inputs(cfg)
    assert torch.equal(a.x, b.x) and torch.equal(a.w_down.data, b.w_down.data)
    src, copy_of = W.gen_replica_src(cfg)
    for s in range(cfg.B):
        assert torch.equal(a.w_gate.data[cfg.E + s], a.w_gate.data[int(copy_of[s])])
    assert (src[cfg.B_used:] == -1).all() and (src[:cfg.B_used] >= 0).all()


def test_given_topk_and_input_weighting():
    cfg = W.MoEConfig("given", T=9, H=32, I=48, E=6, topk=2, logit_std=2.0)
    inp = W.gen_inputs(cfg)
    args = (cfg, inp.x, inp.logits.numpy(), np.zeros(0, np.int32), inp.w_gate, inp.w_up, inp.w_down)
    # the computed routing, given back, changes nothing
    ids, w = O.route_topk(inp.logits.numpy(), cfg.topk)
    a = O.moe_forward(*args)["out"]
    b = O.moe_forward(*args, given_topk=(ids, w.astype(np.float32)))["out"]
    assert np.allclose(a, b, rtol=1e-6, atol=1e-9)
    # arbitrary given experts and weights (a repeated expert for one token included)
    g = np.random.default_rng(5)
    gid = g.integers(0, cfg.E, (cfg.T, cfg.topk)).astype(np.int32)
    gw = g.uniform(0.1, 2.0, (cfg.T, cfg.topk)).astype(np.float32)
    res = O.moe_forward(*args, given_topk=(gid, gw))["out"]
    ref = _layer_brute(cfg, inp, given=(gid, gw))
    assert np.allclose(res, ref, rtol=1e-9, atol=1e-12 * np.abs(ref).max())
    # top-1 with the weight on the input: x scaled before the MLP, no weight after it
    cfg1 = cfg.with_(topk=1)
    args1 = (cfg1,) + args[1:]
    w1 = g.uniform(0.2, 3.0, (cfg.T, 1)).astype(np.float32)
    res = O.moe_forward(*args1, given_topk=(gid[:, :1], w1), apply_router_weight_on_input=True)["out"]
    ref = _layer_brute(cfg1, inp, given=(gid[:, :1], w1), input_weight=True)
    assert np.allclose(res, ref, rtol=1e-9, atol=1e-12 * np.abs(ref).max())
    # unit weights: weighting the input or the output is the same
    ones = np.ones((cfg.T, 1), np.float32)
    u1 = O.moe_forward(*args1, given_topk=(gid[:, :1], ones), apply_router_weight_on_input=True)["out"]
    u2 = O.moe_forward(*args1, given_topk=(gid[:, :1], ones))["out"]
    assert np.allclose(u1, u2, rtol=1e-12)
    with pytest.raises(ValueError):
        O.moe_forward(*args, given_topk=(gid, gw), apply_router_weight_on_input=True)


@pytest.mark.parametrize("wfmt,aq", [("nvfp4", 1), ("mxfp4", 2)])
def test_input_weighting_reaches_the_activation_quantiser(wfmt, aq):
    """Top-1 weight on the input with dynamic activation quantisation: the quantiser sees the
    weighted input (what the experts receive when the weighting happens before dispatch)."""
    cfg = W.MoEConfig("given_q", T=8, H=64, I=64, E=4, topk=1, wfmt=wfmt, act_quant=aq)
    inp = W.gen_inputs(cfg)
    args = (cfg, inp.x, inp.logits.numpy(), np.zeros(0, np.int32), inp.w_gate, inp.w_up, inp.w_down)
    g = np.random.default_rng(11)
    gid = g.integers(0, cfg.E, (cfg.T, 1)).astype(np.int32)
    ones = np.ones((cfg.T, 1), np.float32)
    outs = {}
    for v in (0.25, 4.0):
        full = np.full((cfg.T, 1), v, np.float32)
        outs[v] = O.moe_forward(*args, given_topk=(gid, full), apply_router_weight_on_input=True)["out"]
        # a power of two scales x exactly in bf16 and moves both quantisers' scales by the same
        # power, so this is the unweighted layer on the input x * v
        xs = inp.x * v
        assert torch.equal(xs.float(), inp.x.float() * v)
        ref = O.moe_forward(cfg, xs, *args[2:], given_topk=(gid, ones))["out"]
        assert np.array_equal(outs[v], ref)
    # the weight is not dropped: the layer is nonlinear, so the two differ
    assert np.linalg.norm(outs[0.25] - outs[4.0]) > 0.5 * np.linalg.norm(outs[4.0])
    # other weights: the codes are those of bf16(x * w), not of x
    w1 = g.uniform(0.2, 3.0, (cfg.T, 1)).astype(np.float32)
    res = O.moe_forward(*args, given_topk=(gid, w1), apply_router_weight_on_input=True, keep=True)
    xw = torch.tensor(inp.x.float().numpy() * w1, dtype=torch.float32).to(torch.bfloat16).float().numpy()
    quant = O.nvfp4_quantize_rows if aq == 1 else O.mxfp8_quantize_rows
    assert np.array_equal(res["xq_codes"], quant(xw)[0])
    assert not np.array_equal(res["xq_codes"], quant(inp.x.float().numpy())[0])
    # and the per-token loop, which weights, rounds and then quantises each token by itself
    ref = _layer_brute(cfg, inp, given=(gid, w1), input_weight=True)
    assert np.linalg.norm(res["out"] - ref) <= 1e-3 * np.linalg.norm(ref)


def test_swigluoai_reductions_and_clamps():
    g = np.random.default_rng(9)
    gate, up = g.normal(0, 4, (5, 64)), g.normal(0, 4, (5, 64))
    # no clamp, alpha 1, beta 0: silu-and-mul exactly
    assert np.allclose(O.swigluoai_and_mul(gate, up, 1.0, 0.0, None), O.silu_and_mul(gate, up), rtol=1e-14)
    # the clamp: a gate above the limit acts as the limit, up is clipped on both sides
    lim = 7.0
    assert np.allclose(O.swigluoai_and_mul(np.array([10.0]), np.array([2.0]), 1.702, 1.0, lim),
                       O.swigluoai_and_mul(np.array([lim]), np.array([2.0]), 1.702, 1.0, lim))
    assert np.allclose(O.swigluoai_and_mul(np.array([1.5]), np.array([-50.0]), 1.702, 1.0, lim),
                       O.swigluoai_and_mul(np.array([1.5]), np.array([-lim]), 1.702, 1.0, lim))
    # a gate below -limit is not clamped (the gate has an upper clamp only)
    v = O.swigluoai_and_mul(np.array([-9.0]), np.array([0.5]), 1.0, 1.0, lim)[0]
    assert v == -9.0 / (1.0 + math.exp(9.0)) * 1.5
    # an infinite limit (the C ABI's "no clamp") is no clamp
    assert np.array_equal(O.swigluoai_and_mul(gate, up, 1.702, 1.0, np.inf),
                          O.swigluoai_and_mul(gate, up, 1.702, 1.0, None))


def test_biases_closed_form_and_layer_loop():
    # all-zero weights: gate = b_gate, up = b_up, and the expert output is its down bias, so
    # out[t] = sum_k w_k b_down[e_k] whatever the activation
    cfg = W.MoEConfig("bias0", T=6, H=32, I=48, E=5, topk=2, act="swigluoai", bias=True, w_std=0.0)
    inp = W.gen_inputs(cfg)
    bg, bu, bd = inp.extra["biases"]
    res = O.moe_forward(cfg, inp.x, inp.logits.numpy(), np.zeros(0, np.int32), inp.w_gate, inp.w_up,
                        inp.w_down, biases=(bg, bu, bd))
    ids, w = O.route_topk(inp.logits.numpy(), cfg.topk)
    ref = np.einsum("tk,tkh->th", w, bd.double().numpy()[ids])
    assert np.allclose(res["out"], ref, rtol=1e-12, atol=1e-15)
    # random weights, SWIGLUOAI with its clamp, biases: the per-token loop
    cfg = W.MoEConfig("bias1", T=8, H=32, I=48, E=5, topk=2, act="swigluoai", bias=True, logit_std=2.0,
                      swiglu_limit=1.0)
    inp = W.gen_inputs(cfg)
    b = inp.extra["biases"]
    res = O.moe_forward(cfg, inp.x, inp.logits.numpy(), np.zeros(0, np.int32), inp.w_gate, inp.w_up,
                        inp.w_down, biases=b)["out"]
    ref = _layer_brute(cfg, inp, biases=b)
    assert np.allclose(res, ref, rtol=1e-9, atol=1e-12 * np.abs(ref).max())
    res2 = O.moe_forward(cfg, inp.x, inp.logits.numpy(), np.zeros(0, np.int32), inp.w_gate, inp.w_up,
                         inp.w_down, biases=b, apply_topk_in_fc1=False)["out"]
    ref2 = _layer_brute(cfg, inp, apply_topk_in_fc1=False, biases=b)
    assert np.allclose(res2, ref2, rtol=1e-9, atol=1e-12 * np.abs(ref2).max())


# ------------------------------------------------------------------ the FP4 parity bound itself

@pytest.mark.parametrize("name", ["nvfp4_quant", "mxfp4_situ", "mxfp4_w4a8"])
def test_fp4_layer_bound_passes_rounding_and_catches_a_wrong_block(name):
    """The element-wise FP4 bound of the GPU tests admits the oracle's own output rounded to
    bf16 (RNE, as the combine rounds) and rejects one token's 16 outputs off by 30 %."""
    from tests.parity import check_fp4_layer, fp4_layer_bound

    cfg = SMALL[name].with_(T=24, H=128, I=128)
    inp = W.gen_inputs(cfg)
    ref = O.moe_forward(cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up,
                        inp.w_down, keep=True)
    rounded = torch.from_numpy(ref["out"]).float().to(torch.bfloat16)
    check_fp4_layer(rounded, ref, cfg, inp, what=name)
    bad = ref["out"].copy()
    bad[5, 16:32] *= 0.7
    with pytest.raises(AssertionError):
        check_fp4_layer(torch.from_numpy(bad).float().to(torch.bfloat16), ref, cfg, inp, what=name)
    # and it is not vacuous: typically a few percent of the output's mean magnitude
    b = fp4_layer_bound(cfg, inp, ref)
    assert np.median(b) < 0.2 * np.abs(ref["out"]).mean()
