"""moe_permute_noalloc, the permutation for callers that cannot allocate.

Some callers hold only their input and output buffers: an operator handed bare pointers by
another runtime, or a loop with a fixed memory plan where cudaMalloc is not allowed. This
entry point keeps its scratch in a device array inside the library. The checks, through the
C ABI: indices bit-exact with the oracle's permutation on two calls in a row (and equal to
moe_permute's), the bad-id handling and its status, and the refusal of sizes beyond the
array, which must launch nothing.

The file name sorts late so that a run stopping at the first failure has run the other
tests first.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu

MOE_ERR_WORKSPACE_TOO_SMALL = 4
MOE_ERR_DEVICE = 6


def _case(T, E, k, B, used, seed):
    g = torch.Generator().manual_seed(seed)
    L = torch.randn(T, E, generator=g) * 2
    ids, w = O.route_topk(L.numpy(), k)
    src = -np.ones(B, np.int32)
    if B:
        src[:used] = torch.randperm(E, generator=g)[:used].numpy()
    return ids, w.astype(np.float32), src


def _outputs(T, k, E, B, H, dev="cuda"):
    NvS = T * k
    return dict(cu_seqlens=torch.full((E + B,), -7, dtype=torch.int32, device=dev),
                perm_token=torch.full((NvS,), -7, dtype=torch.int32, device=dev),
                perm_w=torch.full((NvS,), -7.0, dtype=torch.float32, device=dev),
                inv_perm=torch.full((T, k), -7, dtype=torch.int32, device=dev),
                x_perm=torch.zeros(NvS, H, dtype=torch.bfloat16, device=dev))


def _noalloc(lib, ids, w, E, B, src, x, out=None):
    T, k = ids.shape
    H = x.shape[1]
    o = out if out is not None else _outputs(T, k, E, B, H)
    st = torch.cuda.current_stream().cuda_stream
    rc = lib.lib().moe_permute_noalloc(ids.data_ptr(), w.data_ptr(), T, k, E, B,
                                       src.data_ptr() if B else None, x.data_ptr(), H, o["cu_seqlens"].data_ptr(),
                                       o["perm_token"].data_ptr(), o["perm_w"].data_ptr(), o["inv_perm"].data_ptr(),
                                       o["x_perm"].data_ptr(), T * k, st)
    return rc, o


def _status(lib):
    return lib.lib().moe_permute_noalloc_status(torch.cuda.current_stream().cuda_stream)


def test_permute_noalloc_matches_oracle_twice(lib):
    cases = [(300, 64, 6, 10, 7, 1), (64, 256, 8, 16, 8, 2)]   # two calls in a row, different sizes
    for T, E, k, B, used, seed in cases:
        ids, w, src = _case(T, E, k, B, used, seed)
        x = W.gen_rows(T, 128, seed=seed)
        d_ids, d_w, d_src, d_x = (torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(),
                                  torch.from_numpy(src).cuda(), x.cuda())
        rc, got = _noalloc(lib, d_ids, d_w, E, B, d_src, d_x)
        assert rc == 0, lib.status_string(rc)
        assert _status(lib) == 0
        ref = O.assign_rows(ids, E, B, src)
        for key in ("cu_seqlens", "perm_token", "inv_perm"):
            assert np.array_equal(got[key].cpu().numpy(), ref[key]), key
        assert np.array_equal(got["perm_w"].cpu().numpy(), w[ref["perm_token"], ref["perm_k"]])
        assert torch.equal(got["x_perm"].cpu(), x[torch.from_numpy(ref["perm_token"]).long()])
        # and the same bits as the workspace-taking entry point
        other = lib.moe_permute(d_ids, d_w, E, B, d_src if B else None, x=d_x)
        torch.cuda.synchronize()
        for key in ("cu_seqlens", "perm_token", "perm_w", "inv_perm", "x_perm"):
            assert torch.equal(got[key], other[key]), key


def test_permute_noalloc_bad_id_is_reported_then_cleared(lib):
    # token 1 lists expert 9 >= E = 4; every access stays inside the buffers
    ids = np.array([[0, 1], [2, 9], [3, 1]], np.int32)
    w = np.full((3, 2), 0.5, np.float32)
    x = W.gen_rows(3, 64, seed=5)
    rc, got = _noalloc(lib, torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(), 4, 0,
                       torch.zeros(0, dtype=torch.int32, device="cuda"), x.cuda())
    assert rc == 0
    assert _status(lib) == MOE_ERR_DEVICE
    assert _status(lib) == 0                                   # read once, then cleared
    inv = got["inv_perm"].cpu().numpy()
    assert inv[1, 1] == -1
    cu = got["cu_seqlens"].cpu().numpy()
    assert cu[-1] == 5                                         # five good assignments
    pt, pw = got["perm_token"].cpu().numpy(), got["perm_w"].cpu().numpy()
    assert pt[5] == 0 and pw[5] == 0.0                         # the row no assignment reached
    for t in range(3):
        for j in range(2):
            if inv[t, j] >= 0:
                assert pt[inv[t, j]] == t
    # a clean call right after gives the oracle's permutation and a clean status
    ids2, w2, src2 = _case(40, 8, 2, 0, 0, 9)
    rc, got2 = _noalloc(lib, torch.from_numpy(ids2).cuda(), torch.from_numpy(w2).cuda(), 8, 0,
                        torch.zeros(0, dtype=torch.int32, device="cuda"), W.gen_rows(40, 64, seed=9).cuda())
    assert rc == 0 and _status(lib) == 0
    ref = O.assign_rows(ids2, 8, 0, src2)
    for key in ("cu_seqlens", "perm_token", "inv_perm"):
        assert np.array_equal(got2[key].cpu().numpy(), ref[key]), key


def test_permute_noalloc_rejects_sizes_beyond_its_scratch(lib):
    # 65536 tokens x 1024 experts needs about 2 MiB of scratch: refused with nothing launched,
    # so the (real, small) output buffers keep their fill
    T, k, E, H = 65536, 8, 1024, 8
    ids = torch.zeros(T, k, dtype=torch.int32, device="cuda")
    w = torch.zeros(T, k, dtype=torch.float32, device="cuda")
    x = torch.zeros(T, H, dtype=torch.bfloat16, device="cuda")
    out = _outputs(T, k, E, 0, H)
    before = {key: v.clone() for key, v in out.items()}
    rc, _ = _noalloc(lib, ids, w, E, 0, torch.zeros(0, dtype=torch.int32, device="cuda"), x, out)
    assert rc == MOE_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
    for key in out:
        assert torch.equal(out[key], before[key]), key
