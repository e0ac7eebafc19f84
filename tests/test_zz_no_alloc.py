"""The allocation-free entry point nf4_lora_linear_fwd_noalloc, for callers that
cannot give the library a device workspace (a framework that keeps all device
memory in its own pool, or a caller that cannot afford the synchronisation an
allocation may cause).  It must give the same result as nf4_lora_linear_fwd with
a caller workspace, call after call, reusing its built-in scratch.

Collected last on purpose (tests/test_zz_*), and self-contained so that it also
passes alone in a fresh process.
"""
import numpy as np
import pytest

from layer_streamed_qlora_nf4_b200 import synth

pytestmark = pytest.mark.gpu
TOL = 2e-2


def test_noalloc_matches_workspace_entry_point_twice():
    import torch
    from layer_streamed_qlora_nf4_b200 import lib as L
    L.load()
    N, K, T, r, s = 1024, 1024, 128, 16, 2.0
    case = synth.linear_case(7, N, K, T, r)
    W = torch.from_numpy(case["W"]).cuda()
    codes = torch.empty(N * K // 2, dtype=torch.uint8, device="cuda")
    absmax = torch.empty(N * K // 64, dtype=torch.float32, device="cuda")
    L.nf4_quantize(W, codes, absmax)
    x = torch.from_numpy(case["x"].view(np.int16)).cuda().view(torch.bfloat16)
    A, B = torch.from_numpy(case["A"]).cuda(), torch.from_numpy(case["B"]).cuda()
    res = torch.from_numpy(synth.normal_bf16(synth.rng(8), (T, N)).view(np.int16)).cuda().view(torch.bfloat16)
    ws = torch.empty(L.nf4_lora_linear_workspace_bytes(T, K, N, r), dtype=torch.uint8, device="cuda")
    ref = torch.empty(T, N, dtype=torch.bfloat16, device="cuda")
    ref_u = torch.empty(T, r, dtype=torch.float32, device="cuda")
    L.nf4_lora_linear_fwd(x, codes, absmax, A, B, s, ref, residual=res, u_out=ref_u, ws=ws)
    for _ in range(2):   # two calls in a row share (and reuse) the built-in scratch
        y = torch.full((T, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        u = torch.full((T, r), float("nan"), dtype=torch.float32, device="cuda")
        L.nf4_lora_linear_fwd_noalloc(x, codes, absmax, A, B, s, y, residual=res, u_out=u)
        torch.cuda.synchronize()
        rf = ref.float()
        err = ((y.float() - rf).abs().max() / rf.abs().max()).item()
        assert err <= TOL, err
        assert torch.isfinite(y.float()).all()
        assert ((u - ref_u).abs().max() / ref_u.abs().max()).item() <= 1e-6
    assert L.lsq_device_status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import torch
    from layer_streamed_qlora_nf4_b200 import lib as L
    L.load()
    N, K, T, r = 1024, 4096, 2048, 16      # split-K partials alone need 32 MiB here
    assert L.nf4_lora_linear_workspace_bytes(T, K, N, r) > (32 << 20)
    x = torch.zeros(T, K, dtype=torch.bfloat16, device="cuda")
    y = torch.zeros(T, N, dtype=torch.bfloat16, device="cuda")
    codes = torch.zeros(N * K // 2, dtype=torch.uint8, device="cuda")
    absmax = torch.zeros(N * K // 64, device="cuda")
    A, B = torch.zeros(r, K, device="cuda"), torch.zeros(N, r, device="cuda")
    with pytest.raises(L.LsqError) as e:
        L.nf4_lora_linear_fwd_noalloc(x, codes, absmax, A, B, 2.0, y)
    assert e.value.code == L.LSQ_ERR_WORKSPACE
    assert "built-in" in str(e.value)
