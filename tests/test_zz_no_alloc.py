"""moe_permute_noalloc against moe_permute.

The allocation-free variant serves callers that hold only their input and output
buffers (an operator handed bare pointers by another runtime, or a loop with a fixed
memory plan where cudaMalloc is not allowed). It keeps its scratch in a device array
inside the library; this checks, through the C ABI, that two calls in a row give the
same results as the workspace-taking entry point. Indices and gathered rows are
integer/byte data, so the comparison is bit-exact.

The file name sorts late so that a run stopping at the first failure has run the
other tests first.
"""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


def _case(T, E, k, B, used, seed):
    g = torch.Generator().manual_seed(seed)
    L = torch.randn(T, E, generator=g) * 2
    ids, w = O.route_topk(L.numpy(), k)
    src = -torch.ones(B, dtype=torch.int32)
    if B:
        src[:used] = torch.randperm(E, generator=g)[:used].to(torch.int32)
    return torch.from_numpy(ids).cuda(), torch.from_numpy(w.astype(np.float32)).cuda(), src.cuda()


def _noalloc(lib, ids, w, E, B, src, x):
    T, k = ids.shape
    H = x.shape[1]
    dev = ids.device
    NvS = T * k
    cu = torch.empty(E + B, dtype=torch.int32, device=dev)
    pt = torch.empty(NvS, dtype=torch.int32, device=dev)
    pw = torch.empty(NvS, dtype=torch.float32, device=dev)
    inv = torch.empty(T, k, dtype=torch.int32, device=dev)
    xp = torch.zeros(NvS, H, dtype=x.dtype, device=dev)
    st = torch.cuda.current_stream().cuda_stream
    rc = lib.lib().moe_permute_noalloc(ids.data_ptr(), w.data_ptr(), T, k, E, B,
                                       src.data_ptr() if B else None, x.data_ptr(), H, cu.data_ptr(),
                                       pt.data_ptr(), pw.data_ptr(), inv.data_ptr(), xp.data_ptr(), NvS, st)
    assert rc == 0, lib.status_string(rc)
    return dict(cu_seqlens=cu, perm_token=pt, perm_w=pw, inv_perm=inv, x_perm=xp)


def test_permute_noalloc_matches_permute_twice(lib):
    cases = [(300, 64, 6, 10, 7, 1), (64, 256, 8, 16, 8, 2)]   # two calls in a row, different sizes
    for T, E, k, B, used, seed in cases:
        ids, w, src = _case(T, E, k, B, used, seed)
        x = W.gen_rows(T, 128, seed=seed).cuda()
        got = _noalloc(lib, ids, w, E, B, src, x)
        ref = lib.moe_permute(ids, w, E, B, src if B else None, x=x)
        torch.cuda.synchronize()
        for key in ("cu_seqlens", "perm_token", "perm_w", "inv_perm", "x_perm"):
            assert torch.equal(got[key], ref[key]), key


def test_permute_noalloc_rejects_sizes_beyond_its_scratch(lib):
    # 65536 tokens x 1024 experts needs about 2 MiB of scratch: refused, nothing launched
    rc = lib.lib().moe_permute_noalloc(None, None, 65536, 8, 1024, 0, None, None, 0, 16, 16, 16, 16,
                                       None, 0, None)
    assert rc == 4   # MOE_ERR_WORKSPACE_TOO_SMALL
