"""GPU parity of each C-ABI entry point against the oracle, on small seeded cases that still
span several tiles and a ragged tail."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import moe_oracle as O
from tests.parity import (FP4_REL_L2, check_bf16, check_fp4_layer, check_mx8, mx8_staging_bound, oracle_bias, rel_l2,
                          routing_kwargs, to_dev)

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ S1 routing

@pytest.mark.parametrize("T,E,k,std,ints", [(16, 8, 2, 1.0, False), (300, 8, 2, 1.0, True),
                                            (64, 256, 8, 2.0, False), (513, 128, 4, 1.0, False),
                                            (37, 33, 32, 1.0, True), (5, 1024, 8, 3.0, False),
                                            (1, 4, 4, 1.0, True)])
def test_route_topk_matches_oracle(lib, T, E, k, std, ints):
    g = torch.Generator().manual_seed(T + E)
    L = torch.randn(T, E, generator=g) * std
    if ints:
        L = torch.randint(-2, 3, (T, E), generator=g).float()
        L[0] = -0.0
    ids, w = lib.moe_route_topk(to_dev(L), k)
    torch.cuda.synchronize()
    rids, rw = O.route_topk(L.numpy(), k)
    assert np.array_equal(ids.cpu().numpy(), rids)
    assert np.allclose(w.cpu().numpy(), rw, rtol=2e-6, atol=1e-7)


# ------------------------------------------------------------------ S2 permutation

@pytest.mark.parametrize("T,E,k,n_group,topk_group,bias,ints",
                         [(64, 256, 8, 8, 4, True, False), (300, 24, 4, 6, 2, True, True),
                          (37, 512, 8, 16, 3, False, False), (5, 32, 32, 2, 2, True, False),
                          (9, 64, 6, 1, 1, True, False), (17, 96, 3, 32, 3, False, True)])
def test_route_grouped_matches_oracle(lib, T, E, k, n_group, topk_group, bias, ints):
    g = torch.Generator().manual_seed(T + E)
    L = torch.randn(T, E, generator=g) * 2.0
    if ints:
        L = torch.round(L)                      # ties between experts and between groups
    b = (torch.randn(E, generator=g) * 0.05) if bias else None
    ids, w = lib.moe_route_topk_grouped(to_dev(L), k, n_group, topk_group, to_dev(b), 2.5)
    torch.cuda.synchronize()
    rids, rw = O.route_topk_grouped(L.numpy(), k, n_group, topk_group, None if b is None else b.numpy(), 2.5)
    assert np.array_equal(ids.cpu().numpy(), rids)
    assert np.allclose(w.cpu().numpy(), rw, rtol=2e-7, atol=1e-7)


def _perm_inputs(T, E, k, B, used, seed, skew=None):
    g = torch.Generator().manual_seed(seed)
    L = torch.randn(T, E, generator=g) * 2
    if skew == "one_expert":
        L[:, 3] += 100.0
    src = -torch.ones(B, dtype=torch.int32)
    if B:
        src[:used] = torch.randperm(E, generator=g)[:used].to(torch.int32)
    ids, w = O.route_topk(L.numpy(), k)
    return torch.from_numpy(ids), torch.from_numpy(w.astype(np.float32)), src


@pytest.mark.parametrize("T,E,k,B,used,skew", [(16, 8, 2, 0, 0, None), (300, 8, 3, 4, 3, None),
                                               (64, 256, 8, 16, 8, None), (1029, 64, 6, 10, 10, None),
                                               (257, 16, 2, 3, 1, "one_expert"), (1, 4, 1, 2, 1, None),
                                               (8192, 256, 8, 16, 8, None)])
def test_permute_matches_oracle_bitexact(lib, T, E, k, B, used, skew):
    ids, w, src = _perm_inputs(T, E, k, B, used, seed=T * 7 + B, skew=skew)
    H = 64
    x = W.gen_rows(T, H, seed=T)
    r = lib.moe_permute(to_dev(ids), to_dev(w), E, B, to_dev(src) if B else None, x=to_dev(x),
                        M_alloc=T * k + 5)
    torch.cuda.synchronize()
    ref = O.assign_rows(ids.numpy(), E, B, src.numpy())
    assert np.array_equal(r["cu_seqlens"].cpu().numpy(), ref["cu_seqlens"])
    assert np.array_equal(r["perm_token"].cpu().numpy(), ref["perm_token"])
    assert np.array_equal(r["inv_perm"].cpu().numpy(), ref["inv_perm"])
    pw = w.numpy()[ref["perm_token"], ref["perm_k"]]
    assert np.array_equal(r["perm_w"].cpu().numpy(), pw)
    xp = r["x_perm"].cpu()
    assert torch.equal(xp[:T * k], x[torch.from_numpy(ref["perm_token"]).long()])
    assert torch.count_nonzero(xp[T * k:]) == 0            # rows past NvS untouched (zeros here)
    assert lib.moe_get_device_error(r["ws"]) == 0


def test_permute_out_of_range_id_sets_device_error(lib):
    ids = torch.tensor([[0, 1], [2, 9], [3, 1]], dtype=torch.int32)   # 9 >= E
    w = torch.full((3, 2), 0.5)
    r = lib.moe_permute(to_dev(ids), to_dev(w), 4, 0)
    assert lib.moe_get_device_error(r["ws"]) == 6           # MOE_ERR_DEVICE
    assert lib.moe_get_device_error(r["ws"]) == 0           # the word was cleared


def test_permute_empty(lib):
    ids = torch.zeros(0, 2, dtype=torch.int32)
    r = lib.moe_permute(to_dev(ids), to_dev(torch.zeros(0, 2)), 8, 0)
    torch.cuda.synchronize()
    assert torch.count_nonzero(r["cu_seqlens"]) == 0


# ------------------------------------------------------------------ S3/S5 grouped GEMM

GEMM_CASES = [
    ([3, 0, 130, 17, 0, 1, 64], 320, 192, 4),        # ragged N tile, one segment spans 2+ tiles
    ([1, 2, 1, 3, 2, 1, 1, 5], 128, 512, 0),         # decode-like: tiny segments
    ([600, 0, 300], 256, 256, 40),                   # prefill-like, padding rows
    ([0, 0, 0], 128, 64, 8),                         # all empty: output is all padding
    ([37], 136, 200, 3),                             # K not a multiple of 64, N % 128 = 8
]


@pytest.mark.parametrize("seg,N,K,pad", GEMM_CASES)
def test_grouped_gemm_bf16(lib, seg, N, K, pad):
    M = sum(seg) + pad
    a, wt, lens = W.gen_grouped_gemm_case(M, seg, N, K, seed=N + K)
    cu = np.cumsum(seg).astype(np.int32)
    w = lib.Weight("bf16", to_dev(wt))
    out = lib.moe_grouped_gemm(to_dev(a), w, to_dev(torch.from_numpy(cu)),
                               out=torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    ref = O.grouped_gemm(O.to_f64(a), W.WeightSet("bf16", wt), cu, M_alloc=M)
    check_bf16(out, ref, atol=1e-5 * max(1.0, np.abs(ref).max()), rtol=2.0 ** -8, rel=4e-3, what="gemm")


@pytest.mark.parametrize("fmt", ["bf16", "mxfp4", "nvfp4"])
@pytest.mark.parametrize("bt", [16, 32, 64, 128])
def test_grouped_gemm_every_token_tile(lib, bt, fmt, monkeypatch):
    # the same problem through each token-tile width the kernel is built for
    monkeypatch.setenv("MOE_TOKEN_TILE", str(bt))
    seg = [5, 40, 0, 130, 1]
    M, N, K = sum(seg), 256, 128
    a, wt, _ = W.gen_grouped_gemm_case(M, seg, N, K, seed=bt)
    cu = np.cumsum(seg).astype(np.int32)
    ws = W.WeightSet("bf16", wt) if fmt == "bf16" else _fp4_weightset(fmt, len(seg), N, K, seed=bt)
    w = lib.moe_prepare_weights(lib.Weight.from_host(ws))
    out = lib.moe_grouped_gemm(to_dev(a), w, to_dev(torch.from_numpy(cu)))
    torch.cuda.synchronize()
    ref = O.grouped_gemm(O.to_f64(a), ws, cu)
    if fmt == "mxfp4":
        r = check_mx8(out, ref, mx8_staging_bound(O.to_f64(a), ws, cu, M), what=f"bt{bt}")
        assert r <= 4e-3, r
    else:
        check_bf16(out, ref, atol=1e-4 * np.abs(ref).max(), rtol=2.0 ** -8, rel=4e-3, what=f"bt{bt}")


def test_grouped_gemm_bf16_256_token_tile(lib, monkeypatch):
    # the wide tile of the single-matrix BF16 GEMM: segments spanning 1, 2 and 3 tiles, ragged N
    monkeypatch.setenv("MOE_TOKEN_TILE", "256")
    seg = [300, 0, 17, 600, 1]
    M, N, K = sum(seg) + 9, 200, 192
    a, wt, _ = W.gen_grouped_gemm_case(M, seg, N, K, seed=256)
    cu = np.cumsum(seg).astype(np.int32)
    w = lib.Weight("bf16", to_dev(wt))
    out = lib.moe_grouped_gemm(to_dev(a), w, to_dev(torch.from_numpy(cu)))
    torch.cuda.synchronize()
    ref = O.grouped_gemm(O.to_f64(a), W.WeightSet("bf16", wt), cu, M_alloc=M)
    check_bf16(out, ref, atol=1e-4 * np.abs(ref).max(), rtol=2.0 ** -8, rel=4e-3, what="bt256")


@pytest.mark.parametrize("fwd", ["0", "1"])
def test_grouped_gemm_bf16_pairs_ragged(lib, fwd, monkeypatch):
    # the CTA-pair kernel on segments of every awkward length (1, one under and over a tile of
    # 256, several tiles, empty), N not a multiple of the 256-row pair block, K not of 64,
    # padding rows after the last segment; both ways of completing a stage (on the leader's
    # barrier, or forwarded by the peer)
    monkeypatch.setenv("MOE_GEMM_PAIRS", "1")
    monkeypatch.setenv("MOE_PAIR_FWD", fwd)
    seg = [1, 17, 0, 33, 100, 255, 256, 257, 600, 31]
    M, N, K = sum(seg) + 5, 200, 136
    a, wt, _ = W.gen_grouped_gemm_case(M, seg, N, K, seed=77)
    cu = np.cumsum(seg).astype(np.int32)
    w = lib.Weight("bf16", to_dev(wt))
    out = lib.moe_grouped_gemm(to_dev(a), w, to_dev(torch.from_numpy(cu)),
                               out=torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    ref = O.grouped_gemm(O.to_f64(a), W.WeightSet("bf16", wt), cu, M_alloc=M)
    check_bf16(out, ref, atol=1e-5 * max(1.0, np.abs(ref).max()), rtol=2.0 ** -8, rel=4e-3, what="pairs")


@pytest.mark.parametrize("fused_gather", ["0", "1"])
def test_forward_bf16_pairs_ragged(lib, fused_gather, monkeypatch):
    # the fused layer with both GEMMs on CTA pairs: a given top-1 routing that gives the
    # experts 0, 1, 17, 33, 100, 255, 256, 257 and 300 tokens; I = 384 leaves the second pair
    # block of the gate/up GEMM half empty, H = 208 is not a multiple of 64. With the fused
    # gather the gate/up GEMM reads the token rows of x by the permutation itself.
    monkeypatch.setenv("MOE_GEMM_PAIRS", "1")
    monkeypatch.setenv("MOE_FUSED_GATHER", fused_gather)
    lens = [0, 1, 17, 33, 100, 255, 256, 257, 300]
    cfg = W.MoEConfig("pairs", T=sum(lens), H=208, I=384, E=len(lens), topk=1)
    inp = W.gen_inputs(cfg)
    gid = np.concatenate([np.full(n, e, np.int32) for e, n in enumerate(lens)])
    gid = np.random.default_rng(4).permutation(gid).reshape(-1, 1)
    gw = np.random.default_rng(5).uniform(0.2, 1.0, (cfg.T, 1)).astype(np.float32)
    dev = lambda ws: lib.Weight.from_host(ws)
    layer = lib.MoEForward(dev(inp.w_gate), dev(inp.w_up), dev(inp.w_down), cfg.E, 1, routing="given", T_max=cfg.T)
    out = layer(to_dev(inp.x), None, topk_ids_in=to_dev(torch.from_numpy(gid)), topk_w_in=to_dev(torch.from_numpy(gw)))
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    ref = O.moe_forward(cfg, inp.x, None, np.zeros(0, np.int32), inp.w_gate, inp.w_up, inp.w_down,
                        given_topk=(gid, gw))
    check_bf16(out, ref["out"], what="pairs forward")


def test_forward_bf16_fused_gather_one_sm(lib, monkeypatch):
    # the one-SM gate/up GEMM with 128-token tiles reading its token rows of x by the
    # permutation (segments of about 150 rows, H = 208 not a multiple of 64): the oracle's
    # output, and the same bits as the pre-gathered form
    cfg = W.MoEConfig("gather1", T=600, H=208, I=256, E=8, topk=2, B=3, B_used=2)
    inp = W.gen_inputs(cfg)
    outs = {}
    monkeypatch.setenv("MOE_GEMM_PAIRS", "0")
    for fg in ("1", "0"):
        monkeypatch.setenv("MOE_FUSED_GATHER", fg)
        outs[fg], _, _, _ = run_layer(lib, cfg, inp)
    ref = O.moe_forward(cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up, inp.w_down)
    check_bf16(outs["1"], ref["out"], what="fused gather")
    assert torch.equal(outs["1"], outs["0"])


def test_grouped_gemm_bf16_matches_torch_grouped_mm(lib):
    if not hasattr(torch, "_grouped_mm"):
        pytest.skip("torch._grouped_mm unavailable")
    seg = [16, 48, 32, 64]
    M, N, K = sum(seg), 256, 256
    a, wt, _ = W.gen_grouped_gemm_case(M, seg, N, K, seed=11)
    cu = torch.tensor(np.cumsum(seg), dtype=torch.int32, device="cuda")
    w = lib.Weight("bf16", to_dev(wt))
    out = lib.moe_grouped_gemm(to_dev(a), w, cu)
    try:
        ref = torch._grouped_mm(to_dev(a), to_dev(wt).transpose(1, 2), offs=cu)
    except Exception as e:  # library kernel not available for this build
        pytest.skip(f"torch._grouped_mm: {e}")
    torch.cuda.synchronize()
    assert (out.float() - ref.float()).abs().max().item() <= 2.0 ** -7 * ref.float().abs().max().item()


def _fp4_weightset(fmt, G, N, K, seed):
    cfg = W.MoEConfig("w", T=1, H=K, I=N, E=G, topk=1, wfmt=fmt)
    wg, _, _, _ = W.gen_weights(cfg)
    return wg


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("seg,N,K", [([3, 0, 130, 17], 320, 192), ([1, 2, 1, 3], 128, 512),
                                     ([77, 5], 224, 96)])
def test_grouped_gemm_fp4(lib, fmt, seg, N, K):
    ws = _fp4_weightset(fmt, len(seg), N, K, seed=N)
    M = sum(seg) + 3
    a, _, _ = W.gen_grouped_gemm_case(M, seg, 8, K, seed=K)
    cu = np.cumsum(seg).astype(np.int32)
    w = lib.moe_prepare_weights(lib.Weight.from_host(ws))
    out = lib.moe_grouped_gemm(to_dev(a), w, to_dev(torch.from_numpy(cu)))
    torch.cuda.synchronize()
    ref = O.grouped_gemm(O.to_f64(a), ws, cu, M_alloc=M)
    if fmt == "mxfp4":
        r = check_mx8(out, ref, mx8_staging_bound(O.to_f64(a), ws, cu, M), what=fmt)
        assert r <= 4e-3, r
    else:
        check_bf16(out, ref, atol=1e-4 * np.abs(ref).max(), rtol=2.0 ** -8, rel=4e-3, what=fmt)


@pytest.mark.parametrize("bt", [16, 32])
def test_grouped_gemm_mxfp4_wide_matches_narrow(lib, bt, monkeypatch):
    # the single-matrix MXFP4 GEMM with two weight blocks per tile (the decode form): N = 384
    # is three 128-row blocks, so the second wide tile is half past the end; against the
    # staging bound and bit for bit against one block per tile
    monkeypatch.setenv("MOE_TOKEN_TILE", str(bt))
    seg, N, K = [3, 0, 20, 1, 37], 384, 256
    ws = _fp4_weightset("mxfp4", len(seg), N, K, seed=bt + 1)
    M = sum(seg) + 3
    a, _, _ = W.gen_grouped_gemm_case(M, seg, 8, K, seed=bt)
    cu = np.cumsum(seg).astype(np.int32)
    w = lib.moe_prepare_weights(lib.Weight.from_host(ws))
    outs = {}
    for wide in ("1", "0"):
        monkeypatch.setenv("MOE_MX8_WIDE", wide)
        outs[wide] = lib.moe_grouped_gemm(to_dev(a), w, to_dev(torch.from_numpy(cu)))
        torch.cuda.synchronize()
    ref = O.grouped_gemm(O.to_f64(a), ws, cu, M_alloc=M)
    r = check_mx8(outs["1"], ref, mx8_staging_bound(O.to_f64(a), ws, cu, M), what=f"wide bt{bt}")
    assert r <= 4e-3, r
    assert torch.equal(outs["1"], outs["0"])


def _nvfp4_rows(a):
    """The oracle's NVFP4 quantisation of rows a (bf16 [M,K]): packed codes, e4m3 block
    scales, fp32 row scales, and the exact values they stand for."""
    codes, sb, s = O.nvfp4_quantize_rows(a.float().numpy())
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return (torch.from_numpy(packed), torch.from_numpy(sb), torch.from_numpy(s),
            O.nvfp4_dequantize_rows(codes, sb, s))


# K a multiple of 256 (one pipeline stage); ragged N, empty segments, padding rows, and
# segments spanning one to three token tiles of every width
NVF4_CASES = [([5, 40, 0, 130, 1], 256, 256, 0), ([3, 0, 130, 17], 320, 512, 3),
              ([1, 2, 1, 3], 128, 1024, 0), ([77, 5], 208, 256, 9)]


@pytest.mark.parametrize("seg,N,K,pad", NVF4_CASES)
@pytest.mark.parametrize("bt", [16, 32, 64, 128])
def test_grouped_gemm_nvfp4_block_scaled(lib, seg, N, K, pad, bt, monkeypatch):
    monkeypatch.setenv("MOE_TOKEN_TILE", str(bt))
    ws = _fp4_weightset("nvfp4", len(seg), N, K, seed=N + bt)
    M = sum(seg) + pad
    a, _, _ = W.gen_grouped_gemm_case(M, seg, 8, K, seed=K + bt)
    codes, sb, s, deq = _nvfp4_rows(a)
    cu = np.cumsum(seg).astype(np.int32)
    w = lib.moe_prepare_weights(lib.Weight.from_host(ws))
    out = lib.moe_grouped_gemm_nvfp4(to_dev(codes), to_dev(sb), to_dev(s), w, to_dev(torch.from_numpy(cu)),
                                     out=torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    ref = O.grouped_gemm(deq, ws, cu, M_alloc=M)
    check_bf16(out, ref, atol=1e-4 * np.abs(ref).max(), rtol=2.0 ** -8, rel=4e-3, what=f"nvf4 bt{bt}")


# ------------------------------------------------------------------ S4 activation

@pytest.mark.parametrize("act,sa,sb", [("silu", 1.0, 1.0), ("situ", 1.0, 1.0), ("situ", 0.7, 2.5)])
def test_act_and_mul(lib, act, sa, sb):
    M, I = 37, 136
    gate = W.gen_rows(M, I, seed=1, std=3.0)
    up = W.gen_rows(M, I, seed=2, std=3.0)
    pw = torch.rand(M, generator=torch.Generator().manual_seed(3))
    out = lib.moe_act_and_mul(to_dev(gate), to_dev(up), to_dev(pw), act, sa, sb)
    torch.cuda.synchronize()
    ref = O.act_and_mul(O.to_f64(gate), O.to_f64(up), act, sa, sb, pw.double().numpy())
    check_bf16(out, ref, atol=1e-6, rtol=2.0 ** -8, rel=4e-3, what=act)


# ------------------------------------------------------------------ S6 combine

@pytest.mark.parametrize("weighted", [False, True])
def test_combine(lib, weighted):
    T, k, H = 33, 4, 1032
    ids, w, _ = _perm_inputs(T, 16, k, 0, 0, seed=5)
    ref_p = O.assign_rows(ids.numpy(), 16, 0, np.zeros(0))
    y = W.gen_rows(T * k, H, seed=6)
    out = lib.moe_combine(to_dev(y), to_dev(torch.from_numpy(ref_p["inv_perm"])),
                          to_dev(w) if weighted else None)
    torch.cuda.synchronize()
    ref = O.combine(O.to_f64(y), ref_p["inv_perm"], w.double().numpy() if weighted else None)
    check_bf16(out, ref, atol=1e-6, rtol=2.0 ** -8, rel=4e-3, what="combine")


# ------------------------------------------------------------------ S2q NVFP4 quantisation

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantize_nvfp4_bitexact(lib, dtype):
    R, K = 70, 7168
    x = W.gen_rows(R, K, seed=9, dtype=torch.float32)
    x[1] *= 1e-3
    x[2, 32:48] = 0.0                          # a zero block
    x[3] = 0.0                                 # a zero row
    x[4, 100] = 75.0                           # an outlier
    x[5, :16] = -1e-30                         # negatives that round to zero
    x = x.to(dtype)
    codes, sb, s, deq = lib.moe_quantize_nvfp4(to_dev(x))
    torch.cuda.synchronize()
    rc, rsb, rs = O.nvfp4_quantize_rows(x.float().numpy())
    packed = (rc[:, 0::2] | (rc[:, 1::2] << 4)).astype(np.uint8)
    assert np.array_equal(s.cpu().numpy(), rs)
    assert np.array_equal(sb.cpu().numpy(), rsb)
    assert np.array_equal(codes.cpu().numpy(), packed)
    ref_deq = O.e2m1_decode(rc) * np.repeat(O.e4m3_decode(rsb), 16, axis=1)
    assert np.array_equal(deq.cpu().double().numpy(), ref_deq)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantize_mxfp8_bitexact(lib, dtype):
    R, K = 37, 2880
    x = W.gen_rows(R, K, seed=11, dtype=torch.float32)
    x[1] *= 1e-3
    x[2, 64:96] = 0.0                          # a zero block
    x[3] = 0.0                                 # a zero row
    x[4, 100] = 75.0                           # an outlier
    x[5, :32] = torch.linspace(-1, 1, 32) * 15.2   # saturates at 448 * 2^-5
    x[6, :32] = 2.0 ** 5                       # a power of two
    x = x.to(dtype)
    codes, scales = lib.moe_quantize_mxfp8(to_dev(x))
    torch.cuda.synchronize()
    rc, rs = O.mxfp8_quantize_rows(x.float().numpy())
    assert np.array_equal(scales.cpu().numpy(), rs)
    assert np.array_equal(codes.cpu().numpy(), rc)


# ------------------------------------------------------------------ the fused layer, small

SMALL = {
    "tiny": W.CONFIGS["tiny"],
    "replicas": W.MoEConfig("replicas", T=300, H=128, I=256, E=16, topk=4, B=6, B_used=4, logit_std=2.0),
    "situ_bf16": W.MoEConfig("situ_bf16", T=70, H=256, I=384, E=8, topk=2, act="situ",
                             situ_alpha=0.8, situ_beta=1.7),
    "mxfp4": W.MoEConfig("mxfp4", T=40, H=256, I=320, E=8, topk=4, act="situ", wfmt="mxfp4"),
    "mxfp4_silu": W.MoEConfig("mxfp4_silu", T=40, H=256, I=192, E=8, topk=2, wfmt="mxfp4"),
    "nvfp4": W.MoEConfig("nvfp4", T=50, H=512, I=256, E=16, topk=8, wfmt="nvfp4", act_quant=1),
    # gate/up K = 272 staged in f16, down K = 512 block-scaled
    "nvfp4_mixed": W.MoEConfig("nvfp4_mixed", T=33, H=272, I=512, E=8, topk=4, wfmt="nvfp4", act_quant=1),
    # neither K a multiple of 256: both staged in f16
    "nvfp4_f16": W.MoEConfig("nvfp4_f16", T=40, H=272, I=304, E=8, topk=2, wfmt="nvfp4", act_quant=1),
    # DeepSeekV3 grouped routing with replicas: 6 groups of 4, 2 kept, scaling 2.5
    "grouped_routing": W.MoEConfig("grouped_routing", T=130, H=128, I=192, E=24, topk=4, B=4, B_used=3,
                                   logit_std=2.0, routing="deepseek_v3", n_group=6, topk_group=2,
                                   routed_scaling_factor=2.5),
    # W4A8: MXFP4 weights with dynamic MXFP8 activations (K padded to 128 in both GEMMs)
    "mxfp4_w4a8": W.MoEConfig("mxfp4_w4a8", T=40, H=256, I=320, E=8, topk=4, act="situ", wfmt="mxfp4",
                              act_quant=2),
    "mxfp4_w4a8_silu": W.MoEConfig("mxfp4_w4a8_silu", T=300, H=192, I=256, E=8, topk=2, wfmt="mxfp4",
                                   act_quant=2),
}


def run_layer(lib, cfg, inp, apply_topk_in_fc1=True):
    dev = lambda ws: lib.Weight.from_host(ws)
    layer = lib.MoEForward(dev(inp.w_gate), dev(inp.w_up), dev(inp.w_down), cfg.E, cfg.topk, cfg.B,
                           to_dev(inp.replica_src) if cfg.B else None, cfg.act, cfg.situ_alpha,
                           cfg.situ_beta, cfg.act_quant, apply_topk_in_fc1, T_max=cfg.T,
                           **routing_kwargs(cfg, inp))
    ids = torch.empty(cfg.T, cfg.topk, dtype=torch.int32, device="cuda")
    tw = torch.empty(cfg.T, cfg.topk, dtype=torch.float32, device="cuda")
    out = layer(to_dev(inp.x), to_dev(inp.logits), topk_ids=ids, topk_w=tw)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    return out, ids, tw, layer


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_small_matches_oracle(lib, name):
    cfg = SMALL[name]
    inp = W.gen_inputs(cfg)
    out, ids, tw, _ = run_layer(lib, cfg, inp)
    ref = O.moe_forward(cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up,
                        inp.w_down, routing_bias=oracle_bias(inp), keep=cfg.wfmt != "bf16")
    assert np.array_equal(ids.cpu().numpy(), ref["ids"])
    if cfg.wfmt == "bf16":
        check_bf16(out, ref["out"], what=name)
    else:
        check_fp4_layer(out, ref, cfg, inp, what=name)


@pytest.mark.parametrize("bt", [16, 32, 64, 128])
@pytest.mark.parametrize("act_quant", [0, 2])
def test_forward_mxfp4_every_token_tile(lib, bt, act_quant, monkeypatch):
    # the MXFP4 layer with each token tile forced, hi/lo and W4A8: the 64- and 128-token
    # gate/up tiles have one accumulator buffer (four epilogue warps per lane quarter, the
    # staged record epilogue); segments of about 56 rows leave every width ragged, and
    # I = 320 ends in half a weight block
    monkeypatch.setenv("MOE_TOKEN_TILE", str(bt))
    cfg = W.MoEConfig("mx_tiles", T=140, H=192, I=320, E=10, topk=4, act="situ", wfmt="mxfp4",
                      act_quant=act_quant)
    inp = W.gen_inputs(cfg)
    out, ids, _, _ = run_layer(lib, cfg, inp)
    ref = O.moe_forward(cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up,
                        inp.w_down, keep=True)
    assert np.array_equal(ids.cpu().numpy(), ref["ids"])
    check_fp4_layer(out, ref, cfg, inp, what=f"mxfp4 bt{bt} act_quant {act_quant}")


def test_forward_bf16_256_token_tiles(lib, monkeypatch):
    # the 256-token gate/up tile (one accumulator buffer, eight epilogue warps) and the
    # per-tile MMA width: segments of about 75 rows use a fraction of each tile
    monkeypatch.setenv("MOE_TOKEN_TILE", "256")
    cfg = SMALL["replicas"]
    inp = W.gen_inputs(cfg)
    out, ids, _, _ = run_layer(lib, cfg, inp)
    ref = O.moe_forward(cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up,
                        inp.w_down)
    assert np.array_equal(ids.cpu().numpy(), ref["ids"])
    check_bf16(out, ref["out"], what="bt256")


def test_forward_given_topk_and_input_weight(lib):
    # routing on a given top-k (distinct experts per token, arbitrary weights), and top-1 with
    # the route weight on the input
    cfg = W.MoEConfig("given", T=90, H=128, I=192, E=8, topk=2)
    inp = W.gen_inputs(cfg)
    g = np.random.default_rng(2)
    gid = np.stack([g.permutation(cfg.E)[:cfg.topk] for _ in range(cfg.T)]).astype(np.int32)
    gw = g.uniform(0.1, 2.0, (cfg.T, cfg.topk)).astype(np.float32)
    dev = lambda ws: lib.Weight.from_host(ws)
    for k, in_w in ((2, False), (1, True)):
        c = cfg.with_(topk=k)
        layer = lib.MoEForward(dev(inp.w_gate), dev(inp.w_up), dev(inp.w_down), c.E, c.topk, routing="given",
                               apply_router_weight_on_input=in_w, T_max=c.T)
        ids_d, w_d = to_dev(torch.from_numpy(gid[:, :k].copy())), to_dev(torch.from_numpy(gw[:, :k].copy()))
        out = layer(to_dev(inp.x), None, topk_ids_in=ids_d, topk_w_in=w_d)
        torch.cuda.synchronize()
        assert layer.device_error() == 0
        ref = O.moe_forward(c, inp.x, None, np.zeros(0, np.int32), inp.w_gate, inp.w_up, inp.w_down,
                            given_topk=(gid[:, :k], gw[:, :k]), apply_router_weight_on_input=in_w)
        check_bf16(out, ref["out"], what=f"given k={k} input-weight={in_w}")


@pytest.mark.parametrize("wfmt,aq,H,I", [("nvfp4", 1, 512, 256), ("nvfp4", 1, 160, 96), ("mxfp4", 2, 256, 320)])
def test_forward_input_weight_with_activation_quant(lib, wfmt, aq, H, I):
    # top-1 weight on the input with dynamic activation quantisation: the quantiser sees x
    # times the weight, rounded to bf16 (both the block-scaled NVFP4 path, K % 256 == 0, and
    # its f16-staged fallback, and the W4A8 path)
    cfg = W.MoEConfig("given_q", T=70, H=H, I=I, E=8, topk=1, wfmt=wfmt, act_quant=aq)
    inp = W.gen_inputs(cfg)
    g = np.random.default_rng(3)
    gid = g.integers(0, cfg.E, (cfg.T, 1)).astype(np.int32)
    dev = lambda ws: lib.Weight.from_host(ws)
    layer = lib.MoEForward(dev(inp.w_gate), dev(inp.w_up), dev(inp.w_down), cfg.E, 1, routing="given",
                           act_quant=aq, apply_router_weight_on_input=True, T_max=cfg.T)
    outs = {}
    for name, gw in (("uniform", g.uniform(0.2, 3.0, (cfg.T, 1))), ("x0.25", np.full((cfg.T, 1), 0.25)),
                     ("x4", np.full((cfg.T, 1), 4.0))):
        gw = gw.astype(np.float32)
        out = layer(to_dev(inp.x), None, topk_ids_in=to_dev(torch.from_numpy(gid)),
                    topk_w_in=to_dev(torch.from_numpy(gw)))
        torch.cuda.synchronize()
        assert layer.device_error() == 0
        ref = O.moe_forward(cfg, inp.x, None, np.zeros(0, np.int32), inp.w_gate, inp.w_up, inp.w_down,
                            given_topk=(gid, gw), apply_router_weight_on_input=True, keep=True)
        check_fp4_layer(out, ref, cfg, inp, what=f"{wfmt} input weight {name}")
        outs[name] = out.float().cpu().numpy()
    # the weight reached the experts' quantised input
    assert rel_l2(outs["x0.25"], outs["x4"]) > 0.5


def test_forward_given_topk_repeated_expert_is_refused(lib):
    cfg = W.MoEConfig("given", T=20, H=128, I=192, E=8, topk=2)
    inp = W.gen_inputs(cfg)
    gid = np.tile(np.array([[1, 3]], np.int32), (cfg.T, 1))
    gid[7] = [5, 5]                            # the same expert twice for token 7
    gw = np.ones((cfg.T, 2), np.float32)
    dev = lambda ws: lib.Weight.from_host(ws)
    layer = lib.MoEForward(dev(inp.w_gate), dev(inp.w_up), dev(inp.w_down), cfg.E, cfg.topk, routing="given",
                           T_max=cfg.T)
    layer(to_dev(inp.x), None, topk_ids_in=to_dev(torch.from_numpy(gid)), topk_w_in=to_dev(torch.from_numpy(gw)))
    torch.cuda.synchronize()
    assert layer.device_error() == 6          # MOE_ERR_DEVICE


def test_forward_weight_in_combine(lib):
    cfg = SMALL["replicas"]
    inp = W.gen_inputs(cfg)
    out, _, _, _ = run_layer(lib, cfg, inp, apply_topk_in_fc1=False)
    ref = O.moe_forward(cfg, inp.x, inp.logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up,
                        inp.w_down, apply_topk_in_fc1=False)
    check_bf16(out, ref["out"], what="weight in combine")


def test_forward_reuse_and_fewer_tokens(lib):
    # one workspace sized for T_max serves a smaller batch; repeated calls agree bitwise
    cfg = SMALL["replicas"]
    inp = W.gen_inputs(cfg)
    out1, _, _, layer = run_layer(lib, cfg, inp)
    out2 = layer(to_dev(inp.x), to_dev(inp.logits))
    half = layer(to_dev(inp.x[:77]), to_dev(inp.logits[:77]))
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)
    ref = O.moe_forward(cfg.with_(T=77), inp.x[:77], inp.logits[:77].numpy(), inp.replica_src.numpy(),
                        inp.w_gate, inp.w_up, inp.w_down)
    check_bf16(half, ref["out"], what="T<T_max")
