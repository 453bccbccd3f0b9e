"""GPU parity of the fused layer at the edges of its argument ranges: one token, one expert
(a dense SwiGLU MLP), every expert chosen by every token, the largest top-k, the largest number
of weight rows (E + B = 1024) and every token sending its first choice to one expert. Also the
NVFP4-weight layer with bf16 activations (act_quant = 0), whose f16 staging of x (a gather
with a per-row power-of-two scale) and of h (a row pass, or SITU's fixed-scale f16 epilogue)
no other forward case takes.

Routing ids are compared bit-exactly and outputs with the BF16 tolerance of tests/parity.py
(|d| <= 2e-2 + 2^-8 |ref| elementwise, rel-L2 <= 1e-2); the FP4 case with rel-L2 <= 3e-2.
The file name sorts after the GPU files whose kernels these cases reuse, so a run that stops at
its first failure has run those first.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import moe_oracle as O
from tests.parity import check_bf16, check_fp4_layer, to_dev

pytestmark = pytest.mark.gpu

EDGES = {
    "one_token": W.MoEConfig("one_token", T=1, H=128, I=256, E=8, topk=2),
    "one_token_mxfp4": W.MoEConfig("one_token_mxfp4", T=1, H=256, I=320, E=8, topk=4, act="situ", wfmt="mxfp4"),
    "one_token_nvfp4": W.MoEConfig("one_token_nvfp4", T=1, H=512, I=256, E=16, topk=8, wfmt="nvfp4",
                                   act_quant=1),
    "dense": W.MoEConfig("dense", T=77, H=128, I=192, E=1, topk=1),
    "topk_is_E": W.MoEConfig("topk_is_E", T=50, H=128, I=128, E=4, topk=4),
    "topk_32": W.MoEConfig("topk_32", T=20, H=128, I=128, E=64, topk=32),
    "max_rows": W.MoEConfig("max_rows", T=64, H=128, I=128, E=1000, topk=8, B=24, B_used=12, logit_std=2.0),
    "nvfp4_w4a16_silu": W.MoEConfig("nvfp4_w4a16_silu", T=50, H=512, I=256, E=16, topk=8, wfmt="nvfp4"),
    # K = 272 and 304: neither a multiple of the 64-value chunk, so x and h take 2-D tensor maps
    "nvfp4_w4a16_situ": W.MoEConfig("nvfp4_w4a16_situ", T=40, H=272, I=304, E=8, topk=2, wfmt="nvfp4", act="situ",
                                    situ_alpha=0.8, situ_beta=1.7),
}


def _run(lib, cfg, inp, logits):
    dev = lambda ws: lib.Weight.from_host(ws)
    layer = lib.MoEForward(dev(inp.w_gate), dev(inp.w_up), dev(inp.w_down), cfg.E, cfg.topk, cfg.B,
                           to_dev(inp.replica_src) if cfg.B else None, cfg.act, cfg.situ_alpha, cfg.situ_beta,
                           cfg.act_quant, True, T_max=cfg.T)
    ids = torch.empty(cfg.T, cfg.topk, dtype=torch.int32, device="cuda")
    out = layer(to_dev(inp.x), to_dev(logits), topk_ids=ids)
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    ref = O.moe_forward(cfg, inp.x, logits.numpy(), inp.replica_src.numpy(), inp.w_gate, inp.w_up, inp.w_down,
                        keep=cfg.wfmt != "bf16")
    assert np.array_equal(ids.cpu().numpy(), ref["ids"])
    if cfg.wfmt == "bf16":
        check_bf16(out, ref["out"], what=cfg.name)
    else:
        check_fp4_layer(out, ref, cfg, inp, what=cfg.name)
    return ref


@pytest.mark.parametrize("name", list(EDGES))
def test_forward_edges_match_oracle(lib, name):
    cfg = EDGES[name]
    inp = W.gen_inputs(cfg)
    ref = _run(lib, cfg, inp, inp.logits)
    if name == "max_rows":       # the replica slots are used and the last weight rows are reached
        cu = ref["cu_seqlens"]
        assert np.count_nonzero(np.diff(np.concatenate([[0], cu]))[cfg.E:]) > 0


def test_forward_one_expert_takes_every_first_choice(lib):
    # expert 3's logit is raised for every token: its segment holds all T rows (three token
    # tiles, the last with one row) while the second choices spread over the rest
    cfg = W.MoEConfig("skew", T=257, H=128, I=256, E=8, topk=2)
    inp = W.gen_inputs(cfg)
    logits = inp.logits.clone()
    logits[:, 3] += 100.0
    ref = _run(lib, cfg, inp, logits)
    assert np.all(ref["ids"][:, 0] == 3)
    assert int(ref["cu_seqlens"][3] - ref["cu_seqlens"][2]) == cfg.T


# ------------------------------------------------------------------ bad ids and output margins
# Set up so that every access stays in bounds whatever the kernels do with the bad rows:
# perm_token starts at 0 (a valid token), and the combine's y_perm is a view that starts
# inside a larger buffer.

def test_permute_bad_ids_fill_unassigned_rows(lib):
    # token 2 names expert 9 (E = 4) and token 5 names expert 1 twice: both are reported, the
    # out-of-range assignment gets inv_perm = -1, and the two rows no assignment reaches get
    # token 0 and weight 0; x_perm rows past M_alloc's NvS keep their canary
    T, k, E, H = 8, 2, 4, 64
    ids = torch.tensor([[0, 1], [2, 3], [9, 0], [1, 2], [3, 0], [1, 1], [2, 0], [3, 1]], dtype=torch.int32)
    w = torch.full((T, k), 0.5)
    x = W.gen_rows(T, H, seed=5)
    canary_w = 7.0
    canary_x = torch.full((T * k + 4, H), -3.0, dtype=torch.bfloat16)
    out = dict(perm_token=torch.zeros(T * k, dtype=torch.int32, device="cuda"),
               perm_w=torch.full((T * k,), canary_w, device="cuda"), x_perm=canary_x.cuda())
    r = lib.moe_permute(to_dev(ids), to_dev(w), E, 0, x=to_dev(x), out=out)
    assert lib.moe_get_device_error(r["ws"]) == 6             # MOE_ERR_DEVICE
    cu = r["cu_seqlens"].cpu().numpy()
    assert cu[-1] == T * k - 2
    inv = r["inv_perm"].cpu().numpy()
    assert inv[2, 0] == -1 and inv[5, 0] == inv[5, 1] >= 0
    pt, pw = r["perm_token"].cpu().numpy(), r["perm_w"].cpu().numpy()
    assert np.all(pt[cu[-1]:] == 0) and np.all(pw[cu[-1]:] == 0.0)
    xp = r["x_perm"].cpu()
    assert torch.equal(xp[cu[-1]:T * k], x[:1].expand(int(T * k - cu[-1]), H))
    assert torch.equal(xp[T * k:], canary_x[T * k:])
    # every valid assignment still lands on a row of its expert holding its token
    for t in range(T):
        for j in range(k):
            e = int(ids[t, j])
            if 0 <= e < E:
                row = int(inv[t, j])
                assert (cu[e - 1] if e else 0) <= row < cu[e] and pt[row] == t


def test_combine_skips_refused_assignments(lib):
    T, k, H = 5, 3, 64
    rows = T * k
    big = W.gen_rows(rows + 8, H, seed=9)
    big[:8] = 1000.0                                          # canary rows before y_perm
    y = big.cuda()[8:]
    inv = torch.arange(rows, dtype=torch.int32).reshape(T, k)
    inv[1, 2] = -1
    inv[4, 0] = -1
    tw = W.gen_rows(T, k, seed=10, dtype=torch.float32)
    out = lib.moe_combine(y, to_dev(inv), to_dev(tw))
    torch.cuda.synchronize()
    yk = big[8:].double().numpy()
    ref = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            if inv[t, j] >= 0:
                ref[t] += float(tw[t, j]) * yk[int(inv[t, j])]
    check_bf16(out, ref, what="combine with refused rows")


# ------------------------------------------------------------------ CUDA graph capture

@pytest.mark.parametrize("name", ["replicas_bf16", "mxfp4", "nvfp4"])
def test_forward_graph_replay_matches_eager(lib, name):
    # the forward (programmatic dependent launches, no host sync, no allocation) captured once
    # and replayed: bitwise the eager result, also after new inputs are copied into the
    # captured buffers
    cfg = {"replicas_bf16": W.MoEConfig("g_bf16", T=300, H=128, I=256, E=16, topk=4, B=6, B_used=4),
           "mxfp4": W.MoEConfig("g_mxfp4", T=40, H=256, I=320, E=8, topk=4, act="situ", wfmt="mxfp4"),
           "nvfp4": W.MoEConfig("g_nvfp4", T=50, H=512, I=256, E=16, topk=8, wfmt="nvfp4", act_quant=1)}[name]
    inp = W.gen_inputs(cfg)
    inp2 = W.gen_inputs(cfg.with_(seed=1))
    dev = lambda ws: lib.Weight.from_host(ws)
    layer = lib.MoEForward(dev(inp.w_gate), dev(inp.w_up), dev(inp.w_down), cfg.E, cfg.topk, cfg.B,
                           to_dev(inp.replica_src) if cfg.B else None, cfg.act, cfg.situ_alpha, cfg.situ_beta,
                           cfg.act_quant, True, T_max=cfg.T)
    x, logits = to_dev(inp.x), to_dev(inp.logits)
    eager1 = layer(x, logits).clone()
    eager2 = layer(to_dev(inp2.x), to_dev(inp2.logits)).clone()
    g, out = layer.graph(x, logits)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager1)
    x.copy_(to_dev(inp2.x))
    logits.copy_(to_dev(inp2.logits))
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager2)
    assert layer.device_error() == 0
    del g
