"""The C ABI on the CPU: the library loads, exports every symbol include/moe.h declares,
and rejects bad arguments on the host (status codes, nothing launched, no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

import mixture_experts_layer_21_b200 as m

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
L = m.lib()
INVALID, UNSUP, ALIGN, WS_SMALL, NOT_PREP = 1, 2, 3, 4, 8


def _declared():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 15
    out = subprocess.run(["nm", "-D", "--defined-only", m.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (moe_\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    assert sorted(m.EXPORTS) == names


def test_status_strings_and_version():
    assert m.status_string(0) == "MOE_OK"
    assert m.status_string(8) == "MOE_ERR_NOT_PREPARED"
    assert m.status_string(99) == "MOE_ERR_UNKNOWN"
    assert "sm_100a" in m.version()


def test_workspace_sizes():
    assert L.moe_permute_workspace_size(64, 8, 256, 16) > 0
    assert L.moe_permute_workspace_size(8192, 8, 256, 16) > L.moe_permute_workspace_size(64, 8, 256, 16)
    a = L.moe_forward_workspace_size(64, 7168, 2048, 256, 16, 8, 0, 0)
    b = L.moe_forward_workspace_size(8192, 7168, 2048, 256, 16, 8, 0, 0)
    assert 0 < a < b
    # NVFP4 activations: the fp32 gate/up and down outputs plus the quantised row records
    nvs, H, I = 1024 * 8, 7168, 2048
    assert L.moe_forward_workspace_size(1024, H, I, 256, 0, 8, 2, 1) >= \
        4 * nvs * (H + I) + nvs * (H + I) * 9 // 16
    assert L.moe_forward_workspace_size(-1, 1, 1, 1, 0, 1, 0, 0) == 0


def test_prepared_bytes():
    w = m.moe_weight_t(1, 4, 300, 96)         # MXFP4, G=4, N=300 (3 row tiles), K=96 -> padded 128
    # codes with K padded to 128, then one 512-byte scale block per (g, row tile, 128 K)
    assert L.moe_prepared_weight_bytes(ctypes.byref(w)) >= 4 * 300 * 64 + 4 * 3 * 1 * 512
    w.fmt = 0
    assert L.moe_prepared_weight_bytes(ctypes.byref(w)) == 0


def test_route_validation():
    f = L.moe_route_topk
    assert f(None, -1, 8, 2, None, None, None) == INVALID
    assert f(None, 4, 8, 9, None, None, None) == INVALID       # topk > E
    assert f(None, 4, 8, 0, None, None, None) == INVALID
    assert f(None, 4, 2048, 2, None, None, None) == UNSUP      # E > 1024
    assert f(None, 4, 64, 33, None, None, None) == UNSUP      # topk > 32
    assert f(None, 0, 8, 2, None, None, None) == 0             # no tokens: no-op
    assert f(None, 4, 8, 2, None, None, None) == INVALID       # null pointers


def test_permute_validation():
    f = L.moe_permute
    args = lambda **kw: dict(dict(ids=None, w=None, T=4, k=2, E=8, B=0, src=None, x=None, H=0, cu=1,
                                  pt=None, pw=None, inv=None, xp=None, M=0, ws=1, nws=1 << 20), **kw)
    call = lambda d: f(d["ids"], d["w"], d["T"], d["k"], d["E"], d["B"], d["src"], d["x"], d["H"],
                       d["cu"], d["pt"], d["pw"], d["inv"], d["xp"], d["M"], d["ws"], d["nws"], None)
    assert call(args(k=9)) == INVALID
    assert call(args(B=2)) == INVALID                         # B > 0 needs replica_src
    assert call(args(nws=16)) == WS_SMALL
    assert call(args(xp=16, x=16, H=12, M=8)) == ALIGN        # H % 8
    assert call(args(xp=16, x=16, H=16, M=4)) == INVALID      # M_alloc < T*k
    assert call(args()) == INVALID                            # T > 0 with null outputs


def _w(fmt, G, N, K, data=16, scale=16, kdata=None):
    w = m.moe_weight_t(fmt, G, N, K, data, scale if fmt else None, None)
    if kdata:
        w.kdata, w.kscale, w.kalpha = kdata, kdata, kdata
    return w


def _fwd(**kw):
    p = m.moe_forward_args_t()
    d = dict(T=8, H=64, I=128, E=4, B=0, topk=2, fmt=0, act=0, sa=1.0, sb=1.0, aq=0, T_max=8)
    d.update(kw)
    p.x, p.router_logits, p.out = 16, 16, 16
    p.T, p.H, p.I, p.E, p.B, p.topk, p.T_max = d["T"], d["H"], d["I"], d["E"], d["B"], d["topk"], d["T_max"]
    G = d["E"] + d["B"]
    kd = kw.get("kdata")
    p.w_gate = _w(d["fmt"], G, d["I"], d["H"], kdata=kd)
    p.w_up = _w(d["fmt"], G, d["I"], d["H"], kdata=kd)
    p.w_down = _w(d["fmt"], G, d["H"], d["I"], kdata=kd)
    p.act = m.moe_act_params_t(d["act"], d["sa"], d["sb"])
    p.act_quant = d["aq"]
    p.routing = kw.get("routing", 0)
    p.n_group, p.topk_group = kw.get("n_group", 1), kw.get("topk_group", 1)
    p.routed_scaling_factor = kw.get("scale", 1.0)
    p.apply_router_weight_on_input = kw.get("in_w", 0)
    p.apply_topk_in_fc1 = 1
    p.swiglu_alpha, p.swiglu_beta, p.swiglu_limit = kw.get("oa", 1.702), kw.get("ob", 1.0), kw.get("lim", 7.0)
    p.bias_gate, p.bias_up, p.bias_down = kw.get("bias_gate"), kw.get("bias_up"), kw.get("bias_down")
    nws = L.moe_forward_workspace_size(d["T_max"], d["H"], d["I"], d["E"], d["B"], d["topk"], d["fmt"], d["aq"])
    return p, nws


@pytest.mark.parametrize("kw,expect", [
    (dict(act=1, sa=0.0), INVALID),                 # SITU needs alpha > 0
    (dict(act=1, sb=-1.0), INVALID),
    (dict(act=7), INVALID),
    (dict(T=9), INVALID),                           # T > T_max: buffer sized for fewer tokens
    (dict(topk=5), INVALID),                        # topk > E
    (dict(fmt=1), NOT_PREP),                        # FP4 weights not prepared
    (dict(fmt=1, H=48, kdata=16), ALIGN),           # MXFP4 needs K % 32
    (dict(aq=1), UNSUP),                            # dynamic NVFP4 activations need NVFP4 weights
    (dict(aq=2), UNSUP),                            # dynamic MXFP8 activations need MXFP4 weights
    (dict(fmt=2, aq=2, kdata=16), UNSUP),
    (dict(aq=3), INVALID),                          # no such activation quantisation
    (dict(H=72, I=128), ALIGN),                     # H % 16
    (dict(B=2), INVALID),                           # replicas without replica_src
    (dict(E=1100, topk=2), UNSUP),
    (dict(routing=3), INVALID),                     # no such routing method
    (dict(routing=2), INVALID),                     # given routing without the given top-k
    (dict(in_w=1), INVALID),                        # input-side weight needs top-1
    (dict(routing=1, n_group=3), INVALID),          # E % n_group
    (dict(routing=1, n_group=2, topk_group=1, scale=0.0), INVALID),
    (dict(act=2, oa=float("nan")), INVALID),        # SWIGLUOAI: finite alpha and beta,
    (dict(act=2, ob=float("inf")), INVALID),
    (dict(act=2, lim=0.0), INVALID),                # a clamp limit > 0
    (dict(act=2, lim=float("nan")), INVALID),
    (dict(bias_gate=8), ALIGN),                     # biases 16-byte aligned
    (dict(bias_down=24), ALIGN),
])
def test_forward_validation(kw, expect):
    p, nws = _fwd(**kw)
    assert L.moe_forward(ctypes.byref(p), 16, max(nws, 1 << 30), None) == expect


def test_forward_small_workspace_and_empty():
    p, nws = _fwd()
    assert L.moe_forward(ctypes.byref(p), 16, nws - 1, None) == WS_SMALL
    p, nws = _fwd(T=0)
    assert L.moe_forward(ctypes.byref(p), 16, nws, None) == 0   # no tokens: nothing launched
    p.w_down.N = 63
    assert L.moe_forward(ctypes.byref(p), 16, nws, None) == INVALID


def test_grouped_gemm_and_misc_validation():
    w = _w(2, 4, 128, 64)
    assert L.moe_grouped_gemm(16, 8, ctypes.byref(w), 16, 16, 16, 1 << 20, None) == NOT_PREP
    w = _w(0, 4, 128, 60)
    assert L.moe_grouped_gemm(16, 8, ctypes.byref(w), 16, 16, 16, 1 << 20, None) == ALIGN
    w = _w(0, 4, 128, 64)
    assert L.moe_grouped_gemm(16, 0, ctypes.byref(w), 16, 16, 16, 1 << 20, None) == 0   # no rows
    assert L.moe_grouped_gemm(16, 8, ctypes.byref(w), 16, 16, 16, 100, None) == WS_SMALL
    assert L.moe_quantize_nvfp4(16, 0, 4, 24, 16, 16, 16, None, None) == ALIGN
    assert L.moe_quantize_nvfp4(16, 0, 0, 32, 16, 16, 16, None, None) == 0
    assert L.moe_combine(16, 16, None, 4, 2, 12, 16, None) == ALIGN
    assert L.moe_act_and_mul(16, 16, None, 4, 16, m.moe_act_params_t(1, 0.0, 1.0), 16, None) == INVALID
    wb = _w(0, 4, 128, 64)
    assert L.moe_prepare_weights(ctypes.byref(wb), None, 0, None) == 0                   # BF16: no-op
    wm = _w(1, 4, 128, 48)
    assert L.moe_prepare_weights(ctypes.byref(wm), 16, 1 << 20, None) == ALIGN


def test_route_grouped_validation():
    f = L.moe_route_topk_grouped
    ok = dict(E=256, k=8, ng=8, tg=4, sc=2.5)
    def call(**kw):
        d = dict(ok, **kw)
        return f(16, None, 4, d["E"], d["k"], d["ng"], d["tg"], ctypes.c_float(d["sc"]), 16, 16, None)
    assert f(16, None, 0, 256, 8, 8, 4, ctypes.c_float(2.5), 16, 16, None) == 0    # no tokens
    assert call(E=250) == INVALID                 # E % n_group
    assert call(tg=9) == INVALID                  # topk_group > n_group
    assert call(tg=0) == INVALID
    assert call(k=129) == INVALID                 # more than the kept groups hold
    assert call(sc=0.0) == INVALID
    assert call(sc=float("nan")) == INVALID
    assert call(E=1024, ng=8) == UNSUP            # E > 512
    assert call(E=256, ng=64, tg=4) == UNSUP      # n_group > 32
    assert f(None, None, 4, 256, 8, 8, 4, ctypes.c_float(2.5), 16, 16, None) == INVALID


def test_quantize_mxfp8_validation():
    f = L.moe_quantize_mxfp8
    assert f(16, 0, 4, 48, 16, 16, None) == ALIGN                 # K % 32
    assert f(16, 0, 0, 64, 16, 16, None) == 0                     # no rows: nothing launched
    assert f(None, 0, 4, 64, 16, 16, None) == INVALID
    assert f(16, 0, 4, 64, 8, 16, None) == ALIGN                  # codes not 16-byte aligned
    assert f(16, 0, -1, 64, 16, 16, None) == INVALID


def test_grouped_gemm_nvfp4_validation():
    f = L.moe_grouped_gemm_nvfp4
    wn = _w(2, 4, 128, 512, kdata=16)
    assert f(16, 16, 16, 0, ctypes.byref(wn), 16, 16, 16, 256, None) == 0            # no rows
    assert f(16, 16, 16, 8, ctypes.byref(wn), 16, 16, 16, 100, None) == WS_SMALL
    assert f(None, 16, 16, 8, ctypes.byref(wn), 16, 16, 16, 256, None) == INVALID
    assert f(16, 8, 16, 8, ctypes.byref(wn), 16, 16, 16, 256, None) == ALIGN         # scales misaligned
    assert f(16, 16, 16, 8, ctypes.byref(_w(2, 4, 128, 512)), 16, 16, 16, 256, None) == NOT_PREP
    assert f(16, 16, 16, 8, ctypes.byref(_w(2, 4, 128, 384, kdata=16)), 16, 16, 16, 256, None) == ALIGN
    assert f(16, 16, 16, 8, ctypes.byref(_w(1, 4, 128, 512, kdata=16)), 16, 16, 16, 256, None) == UNSUP
    assert f(16, 16, 16, 8, ctypes.byref(_w(0, 4, 128, 512)), 16, 16, 16, 256, None) == UNSUP


def test_nvfp4_prepared_bytes_hold_both_tile_layouts():
    # K % 256 == 0: the f16-staging tiles plus the block-scaled tiles; otherwise the first only
    G, N = 3, 200
    one = L.moe_prepared_weight_bytes(ctypes.byref(_w(2, G, N, 272)))
    both = L.moe_prepared_weight_bytes(ctypes.byref(_w(2, G, N, 512)))
    NT = 2
    assert one >= G * NT * 6 * (4096 + 512)
    assert both >= G * NT * 8 * (4096 + 512) + G * NT * 2 * (16384 + 2048)


def _c_struct(name):
    """(field, kind) of a typedef struct in moe.h, in declaration order; kind is i32, f32, ptr
    or the name of a nested struct."""
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    body = re.search(r"typedef struct \{([^{}]*)\}\s*" + name + r"\s*;", src).group(1)
    out = []
    for decl in filter(None, (d.strip() for d in body.split(";"))):
        first, *rest = decl.split(",")
        fname = re.findall(r"\w+", first)[-1]
        base = first[: first.rindex(fname)]
        btype = [t for t in re.findall(r"\w+", base) if t != "const"][0]
        for d, nm in [(first, fname)] + [(r, re.findall(r"\w+", r)[-1]) for r in rest]:
            ptr = "*" in base or "*" in d[len(base):]
            out.append((nm, "ptr" if ptr else {"int32_t": "i32", "float": "f32"}.get(btype, btype)))
    return out


def _ctypes_struct(cls):
    kinds = {ctypes.c_int32: "i32", ctypes.c_float: "f32", ctypes.c_void_p: "ptr"}
    return [(n, kinds.get(t, t.__name__)) for n, t in cls._fields_]


@pytest.mark.parametrize("name", ["moe_weight_t", "moe_act_params_t", "moe_act_ex_t", "moe_forward_args_t"])
def test_binding_structs_match_the_header(name):
    # the ctypes mirrors must list the header's fields in its order with the same kinds,
    # so that both compilers lay them out alike
    assert _ctypes_struct(getattr(m, name)) == _c_struct(name)


def test_forward_workspace_with_biases_or_swigluoai():
    # SWIGLUOAI and the biases run in the GEMM epilogues: no workspace of their own
    p, nws = _fwd()
    assert L.moe_forward_workspace_size_args(ctypes.byref(p)) == nws
    p, _ = _fwd(act=2)
    assert L.moe_forward_workspace_size_args(ctypes.byref(p)) == nws
    assert L.moe_forward(ctypes.byref(p), 16, nws - 1, None) == WS_SMALL
    for b in ("bias_gate", "bias_up", "bias_down"):
        p, _ = _fwd(**{b: 16})
        assert L.moe_forward_workspace_size_args(ctypes.byref(p)) == nws
        p.T = 0
        assert L.moe_forward(ctypes.byref(p), 16, nws, None) == 0          # no tokens: nothing launched
    assert L.moe_forward_workspace_size_args(None) == 0


def test_bias_act_validation():
    f = L.moe_bias_act_and_mul

    def call(act, M=4, I=16, G=2, gate=16, bg=None, cu=16):
        return f(gate, 16, 0, bg, None, cu, G, None, M, I, ctypes.byref(act), 16, None)

    ok = m.act_ex()
    assert call(m.act_ex("swigluoai", swiglu_limit=0.0)) == INVALID
    assert call(m.act_ex("swigluoai", swiglu_alpha=float("inf"))) == INVALID
    assert call(m.act_ex("situ", situ_alpha=-1.0)) == INVALID
    assert call(m.moe_act_ex_t(7, 1.0, 1.0, 1.0, 1.0, 1.0)) == INVALID
    assert call(ok, G=0) == INVALID
    assert call(ok, M=0) == 0                                     # no rows: nothing launched
    assert call(ok, I=12) == ALIGN                                # I % 8
    assert call(ok, bg=8) == ALIGN                                # bias not 16-byte aligned
    assert call(ok, gate=None) == INVALID
    assert call(ok, cu=None) == INVALID
    assert f(16, 16, 0, None, None, 16, 2, None, 4, 16, None, 16, None) == INVALID   # no activation
    # moe_act_params_t has no room for SWIGLUOAI's parameters
    assert L.moe_act_and_mul(16, 16, None, 4, 16, m.moe_act_params_t(2, 1.0, 1.0), 16, None) == UNSUP


def test_binding_struct_offsets_match_gcc(tmp_path):
    # the header compiled by the host C compiler: every field's offset and every struct's
    # size equal the ctypes mirror's
    names = ["moe_weight_t", "moe_act_params_t", "moe_act_ex_t", "moe_forward_args_t"]
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "moe.h"', "int main(void) {"]
    for n in names:
        lines.append(f'printf("{n} sizeof %zu\\n", sizeof({n}));')
        for f, _ in _c_struct(n):
            lines.append(f'printf("{n} {f} %zu\\n", offsetof({n}, {f}));')
    lines += ["return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines():
        n, f, v = line.split()
        got[(n, f)] = int(v)
    for n in names:
        cls = getattr(m, n)
        assert got[(n, "sizeof")] == ctypes.sizeof(cls), n
        for f, _ in cls._fields_:
            assert got[(n, f)] == getattr(cls, f).offset, (n, f)
