"""The allocation-free entry point nf4_lora_linear_fwd_noalloc, for callers that
cannot give the library a device workspace (a framework that keeps all device
memory in its own pool, or a caller that cannot afford the synchronisation an
allocation may cause).  It runs the same deterministic kernels as
nf4_lora_linear_fwd with a caller workspace, so its output must be identical,
call after call, while it reuses its built-in scratch; after its first call on
the device (which loads the scratch array) it must not change the device's free
memory.

Collected last on purpose (tests/test_zz_*), and self-contained so that it also
passes alone in a fresh process.
"""
import pytest

from layer_streamed_qlora_nf4_b200 import synth

pytestmark = pytest.mark.gpu


def _case(L, seed):
    import torch
    N, K, T, r = 1024, 1024, 128, 16
    case = synth.linear_case(seed, N, K, T, r)
    W = torch.from_numpy(case["W"]).cuda()
    codes = torch.empty(N * K // 2, dtype=torch.uint8, device="cuda")
    absmax = torch.empty(N * K // 64, dtype=torch.float32, device="cuda")
    L.nf4_quantize(W, codes, absmax)
    x = torch.from_numpy(synth.to_f16(synth.bf16_bits_to_f32(case["x"]))).cuda()
    A, B = torch.from_numpy(case["A"]).cuda(), torch.from_numpy(case["B"]).cuda()
    return N, K, T, r, codes, absmax, x, A, B


@pytest.mark.parametrize("with_residual", [True, False])
def test_noalloc_matches_workspace_entry_point_twice(with_residual):
    import torch
    from layer_streamed_qlora_nf4_b200 import lib as L
    L.load()
    N, K, T, r, codes, absmax, x, A, B = _case(L, 7)
    s = 2.0
    res = None
    if with_residual:    # fp32 residual stream, fp32 output
        res = torch.from_numpy(synth.bf16_bits_to_f32(synth.normal_bf16(synth.rng(8), (T, N)))).cuda()
    ydt = torch.float32 if with_residual else torch.float16
    ws = torch.empty(L.nf4_lora_linear_workspace_bytes(T, K, N, r), dtype=torch.uint8, device="cuda")
    ref = torch.empty(T, N, dtype=ydt, device="cuda")
    ref_u = torch.empty(T, r, dtype=torch.float32, device="cuda")
    L.nf4_lora_linear_fwd(x, codes, absmax, A, B, s, ref, residual=res, u_out=ref_u, ws=ws)
    torch.cuda.synchronize()
    assert torch.isfinite(ref.float()).all()
    for i in range(3):   # the first call may load the scratch; the next two reuse it
        y = torch.full((T, N), float("nan"), dtype=ydt, device="cuda")
        u = torch.full((T, r), float("nan"), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        L.nf4_lora_linear_fwd_noalloc(x, codes, absmax, A, B, s, y, residual=res, u_out=u)
        torch.cuda.synchronize()
        if i > 0:
            assert torch.cuda.mem_get_info()[0] == free0
        assert torch.equal(y, ref), i
        assert torch.equal(u, ref_u), i
    assert L.lsq_device_status() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import torch
    from layer_streamed_qlora_nf4_b200 import lib as L
    L.load()
    N, K, T, r = 1024, 4096, 2048, 16      # split-K partials alone need 32 MiB here
    assert L.nf4_lora_linear_workspace_bytes(T, K, N, r) > (32 << 20)
    x = torch.zeros(T, K, dtype=torch.float16, device="cuda")
    y = torch.zeros(T, N, dtype=torch.float16, device="cuda")
    codes = torch.zeros(N * K // 2, dtype=torch.uint8, device="cuda")
    absmax = torch.zeros(N * K // 64, device="cuda")
    A, B = torch.zeros(r, K, device="cuda"), torch.zeros(N, r, device="cuda")
    with pytest.raises(L.LsqError) as e:
        L.nf4_lora_linear_fwd_noalloc(x, codes, absmax, A, B, 2.0, y)
    assert e.value.code == L.LSQ_ERR_WORKSPACE
    assert "built-in" in str(e.value)
