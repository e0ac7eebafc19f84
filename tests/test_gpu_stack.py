"""GPU parity for the streamed stack step: against the fp64 oracle (loss within
1e-3 relative, logits within normwise 2e-2, every LoRA gradient within 2e-2 by
the max-element reading and in the Frobenius norm (gpu_util.check_stack_grad),
post-AdamW parameters within 2*lr), over several seeds, and streamed vs resident
bit-equality (max |dlogit| = 0.0, identical gradients), at a small Llama-shaped
stack and at the full 32-layer Llama-3.1-8B-shaped stack."""
import math

import numpy as np
import pytest

from oracle import model as om
from oracle import nf4 as onf4
from layer_streamed_qlora_nf4_b200 import synth

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module")
def L():
    from layer_streamed_qlora_nf4_b200 import lib
    lib.load()
    return lib


class Stack:
    """Host-generated small stack, packed on the device, pinned copies for streaming."""

    def __init__(self, L, cfg, seed, tied=False):
        import torch
        from gpu_util import dev, dev_bf16
        from layer_streamed_qlora_nf4_b200 import pack
        self.cfg = cfg
        nl = cfg["n_layers"]
        self.lw = [synth.layer_weights(seed + 100 + i, cfg) for i in range(nl)]
        emb, head = synth.embeddings(seed + 1, cfg["vocab"], cfg["hidden"])
        if tied:                       # one matrix is both the embedding and the lm_head
            head = emb
        self.emb_bits, self.head_bits = emb, head
        self.gf_bits = synth.to_bf16_bits(np.ones(cfg["hidden"], np.float32))
        lay = L.lsq_layer_layout_get(cfg)
        self.blob_bytes = lay.bytes
        self.dev_blobs, self.host_blobs = [], []
        for lw in self.lw:
            b = torch.zeros(lay.bytes, dtype=torch.uint8, device="cuda")
            pack.pack_layer(cfg, {p: dev(lw["W"][p]) for p in synth.PROJ}, dev_bf16(lw["g1"]),
                            dev_bf16(lw["g2"]), b)
            self.dev_blobs.append(b)
            self.host_blobs.append(b.cpu().pin_memory())
        self.lora = torch.cat([pack.lora_block(cfg, lw["A"], lw["B"]) for lw in self.lw])
        self.emb, self.head, self.gf = dev_bf16(emb), dev_bf16(head), dev_bf16(self.gf_bits)
        self.bufs = [torch.empty(lay.bytes, dtype=torch.uint8, device="cuda") for _ in range(2)]

    def handle(self, L, resident):
        blobs = self.dev_blobs if resident else self.host_blobs
        return L.StreamStack(self.cfg, blobs, self.bufs[0], self.bufs[1], resident)

    def oracle_layers(self):
        out = []
        bits = self.cfg.get("absmax_bits", 32)
        for lw in self.lw:
            W = {}
            for p in synth.PROJ:
                N, K = lw["W"][p].shape
                if self.cfg.get("weight_bits", 4) == 16:
                    W[p] = synth.bf16_bits_to_f32(synth.to_bf16_bits(lw["W"][p]))
                    continue
                codes, am = onf4.quantize(lw["W"][p])
                if bits == 8:
                    W[p] = onf4.dequantize_dq(codes, *onf4.quantize_absmax8(am), N, K)
                else:
                    W[p] = onf4.dequantize(codes, am, N, K)
            out.append(dict(W=W, A=lw["A"], B=lw["B"], g1=synth.bf16_bits_to_f32(lw["g1"]),
                            g2=synth.bf16_bits_to_f32(lw["g2"])))
        return out


def _step(L, st, h, tokens_np, mb, batch, seq, opt=None, lora=None):
    import torch
    from gpu_util import workspace
    cfg = st.cfg
    T = batch * seq
    ws = workspace(L.stream_stack_workspace_bytes(cfg, batch, seq))
    tokens = torch.from_numpy(tokens_np.astype(np.int32)).cuda()
    lora = st.lora.clone() if lora is None else lora
    grad = torch.full_like(lora, float("nan"))
    logits = torch.empty(T, cfg["vocab"], dtype=torch.float32, device="cuda")
    loss = L.stream_stack_step(h, tokens, mb, batch, seq, st.emb, st.head, st.gf, lora, grad, opt,
                               ws, logits_out=logits)
    return loss, logits, grad, lora


@pytest.fixture(scope="module")
def small(L):
    return Stack(L, synth.SMALL, 5)


@pytest.fixture(scope="module")
def small8(L):
    # the same weights as `small`, stored with the 8-bit absmax
    return Stack(L, dict(synth.SMALL, absmax_bits=8), 5)


def test_stack_matches_oracle(L, small):
    _check_against_oracle(L, small)


@pytest.mark.parametrize("seed", [6, 8])
def test_stack_matches_oracle_more_seeds(L, seed):
    _check_against_oracle(L, Stack(L, synth.SMALL, seed))


def test_stack_absmax8_matches_oracle(L, small8):
    _check_against_oracle(L, small8)


@pytest.mark.parametrize("seed", [6, 9])
def test_stack_absmax8_matches_oracle_more_seeds(L, seed):
    _check_against_oracle(L, Stack(L, dict(synth.SMALL, absmax_bits=8), seed))


@pytest.fixture(scope="module")
def small_bf16(L):
    # unquantised bf16 stack, tied embedding, LoRA rank 64 (Qwen2.5-3B-style)
    return Stack(L, dict(synth.SMALL, weight_bits=16, lora_r=64, lora_alpha=128.0), 7, tied=True)


def test_stack_bf16_tied_matches_oracle(L, small_bf16):
    _check_against_oracle(L, small_bf16)


@pytest.mark.parametrize("seed", [8, 10])
def test_stack_bf16_tied_matches_oracle_more_seeds(L, seed):
    cfg = dict(synth.SMALL, weight_bits=16, lora_r=64, lora_alpha=128.0)
    _check_against_oracle(L, Stack(L, cfg, seed, tied=True))


def test_stack_bf16_streamed_equals_resident_bitwise(L, small_bf16):
    import torch
    tokens = synth.tokens(35, 2, 64, small_bf16.cfg["vocab"])
    hs = small_bf16.handle(L, resident=False)
    hr = small_bf16.handle(L, resident=True)
    ls, lgs, gs, _ = _step(L, small_bf16, hs, tokens, 1, 2, 64)
    lr_, lgr, gr, _ = _step(L, small_bf16, hr, tokens, 1, 2, 64)
    hs.close()
    hr.close()
    assert ls == lr_ and torch.equal(lgs, lgr) and torch.equal(gs, gr)


def test_stack_absmax8_streamed_equals_resident_bitwise(L, small8):
    import torch
    tokens = synth.tokens(34, 1, 96, small8.cfg["vocab"])
    hs = small8.handle(L, resident=False)
    hr = small8.handle(L, resident=True)
    ls, lgs, gs, _ = _step(L, small8, hs, tokens, 1, 1, 96)
    st = L.stream_stack_last_stats(hs)
    lr_, lgr, gr, _ = _step(L, small8, hr, tokens, 1, 1, 96)
    hs.close()
    hr.close()
    assert ls == lr_ and torch.equal(lgs, lgr) and torch.equal(gs, gr)
    assert st["h2d_bytes"] == st["layer_copies"] * small8.blob_bytes
    assert small8.blob_bytes < L.lsq_layer_layout_get(synth.SMALL).bytes


def _check_against_oracle(L, small):
    from gpu_util import check_stack_grad, normwise_err
    from layer_streamed_qlora_nf4_b200 import pack
    cfg = small.cfg
    batch, seq = 2, 80
    tokens = synth.tokens(31, batch, seq, cfg["vocab"])
    h = small.handle(L, resident=False)
    loss, logits, grad, _ = _step(L, small, h, tokens, 1, batch, seq)
    h.close()
    layers = small.oracle_layers()
    rloss, rlogits, rgrads = om.stack_loss_and_grads(
        layers, synth.bf16_bits_to_f32(small.emb_bits), synth.bf16_bits_to_f32(small.head_bits),
        synth.bf16_bits_to_f32(small.gf_bits), tokens, cfg)
    assert abs(loss - rloss) <= 1e-3 * abs(rloss), (loss, rloss)
    assert normwise_err(logits.cpu().numpy(), rlogits) <= TOL
    nf = L.lsq_lora_layout_get(cfg).floats_per_layer
    for i in range(cfg["n_layers"]):
        gv = pack.lora_views(cfg, grad[i * nf:(i + 1) * nf])
        for name in synth.PROJ:
            check_stack_grad(gv[name][0].cpu().numpy(), rgrads[i][name][0], name, (i, "A"))
            check_stack_grad(gv[name][1].cpu().numpy(), rgrads[i][name][1], name, (i, "B"))


def test_stack_streamed_equals_resident_bitwise(L, small):
    import torch
    cfg = small.cfg
    batch, seq = 1, 128
    tokens = synth.tokens(32, batch, seq, cfg["vocab"])
    hs = small.handle(L, resident=False)
    hr = small.handle(L, resident=True)
    ls, lgs, gs, _ = _step(L, small, hs, tokens, 1, batch, seq)
    st1 = L.stream_stack_last_stats(hs)
    lr_, lgr, gr, _ = _step(L, small, hr, tokens, 1, batch, seq)
    ls2, lgs2, gs2, _ = _step(L, small, hs, tokens, 1, batch, seq)   # buffers carried over
    st2 = L.stream_stack_last_stats(hs)
    hs.close()
    hr.close()
    assert ls == lr_ == ls2
    assert torch.equal(lgs, lgr) and torch.equal(lgs, lgs2)       # max |dlogit| = 0.0
    assert torch.equal(gs, gr) and torch.equal(gs, gs2)
    nl = cfg["n_layers"]
    assert st1["layer_copies"] == 2 * nl - 2
    assert st2["layer_copies"] == 2 * nl - 4
    assert st1["h2d_bytes"] == st1["layer_copies"] * small.blob_bytes


def test_stack_head_chunks_equal_one_chunk(L, small, monkeypatch):
    # lm_head, cross-entropy and the head's input gradient over chunks of one
    # sequence each give the same step as over the whole batch at once (every
    # row's products and loss are computed the same way in both)
    import torch
    cfg = small.cfg
    batch, seq = 3, 48
    tokens = synth.tokens(36, batch, seq, cfg["vocab"])
    h = small.handle(L, resident=True)
    monkeypatch.setenv("LSQ_HEAD_CHUNK_SEQS", "1")
    l1, lg1, g1, _ = _step(L, small, h, tokens, 1, batch, seq)
    monkeypatch.delenv("LSQ_HEAD_CHUNK_SEQS")
    l0, lg0, g0, _ = _step(L, small, h, tokens, 1, batch, seq)
    h.close()
    assert L.stream_stack_workspace_bytes(cfg, batch, seq) > 0
    assert l1 == l0 and torch.equal(lg1, lg0) and torch.equal(g1, g0)


def test_stack_grad_accumulation_and_adamw(L, small):
    import torch
    from gpu_util import check_stack_grad
    cfg = small.cfg
    batch, seq, mb = 1, 64, 2
    tokens = synth.tokens(33, mb * batch, seq, cfg["vocab"]).reshape(mb, batch, seq)
    h = small.handle(L, resident=False)
    lr = 2e-4
    m = torch.zeros_like(small.lora)
    v = torch.zeros_like(small.lora)
    opt = dict(lr=lr, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, step=1, m=m, v=v)
    loss, _, grad, new_lora = _step(L, small, h, tokens, mb, batch, seq, opt=opt)
    h.close()
    layers = small.oracle_layers()
    emb = synth.bf16_bits_to_f32(small.emb_bits)
    head = synth.bf16_bits_to_f32(small.head_bits)
    gf = synth.bf16_bits_to_f32(small.gf_bits)
    r0 = om.stack_loss_and_grads(layers, emb, head, gf, tokens[0], cfg)
    r1 = om.stack_loss_and_grads(layers, emb, head, gf, tokens[1], cfg)
    rloss = 0.5 * (r0[0] + r1[0])
    assert abs(loss - rloss) <= 1e-3 * abs(rloss)
    from layer_streamed_qlora_nf4_b200 import pack
    nf = L.lsq_lora_layout_get(cfg).floats_per_layer
    for i in range(cfg["n_layers"]):
        gv = pack.lora_views(cfg, grad[i * nf:(i + 1) * nf])
        pv = pack.lora_views(cfg, new_lora[i * nf:(i + 1) * nf])
        for j, name in enumerate(synth.PROJ):
            for k, key in ((0, "A"), (1, "B")):
                rg = 0.5 * (r0[2][i][name][k] + r1[2][i][name][k])
                check_stack_grad(gv[name][k].cpu().numpy(), rg, name, (i, key))
                p0 = layers[i][key][name]
                rp, _, _ = om.adamw_step(p0, rg, np.zeros_like(rg), np.zeros_like(rg), 1, lr=lr)
                got = pv[name][k].cpu().numpy()
                assert np.max(np.abs(got - rp)) <= 2 * lr + 1e-6, (i, name, key)


def test_stack_rejects_bad_arguments(L, small):
    import torch
    cfg = dict(small.cfg, n_layers=small.cfg["n_layers"] + 1)
    with pytest.raises(L.LsqError) as e:
        L.StreamStack(cfg, small.host_blobs, small.bufs[0], small.bufs[1], False)
    assert e.value.code == L.LSQ_ERR_SHAPE
    pageable = [b.cpu() for b in small.dev_blobs]      # not page-locked
    with pytest.raises(L.LsqError) as e:
        L.StreamStack(small.cfg, pageable, small.bufs[0], small.bufs[1], False)
    assert e.value.code == L.LSQ_ERR_INVALID
    h = small.handle(L, resident=False)
    from gpu_util import workspace
    tokens = torch.zeros(1, 16, dtype=torch.int32, device="cuda")
    with pytest.raises(L.LsqError) as e:
        L.stream_stack_step(h, tokens, 1, 1, 16, small.emb, small.head, small.gf, small.lora.clone(),
                            torch.empty_like(small.lora), None, workspace(1024))
    assert e.value.code == L.LSQ_ERR_WORKSPACE
    h.close()


def test_stack_llama8b_streamed_equals_resident(L):
    """The 32-layer Llama-3.1-8B-shaped stack (batch 1, seq 512): streamed and
    resident steps are bit-identical; the loss is finite and near ln V."""
    import torch
    from layer_streamed_qlora_nf4_b200 import pack
    from gpu_util import workspace
    cfg = synth.LLAMA8B
    lay = L.lsq_layer_layout_get(cfg)
    g = torch.Generator(device="cuda").manual_seed(2)
    shapes = synth.proj_shapes(cfg)
    ones = torch.ones(cfg["hidden"], dtype=torch.bfloat16, device="cuda")
    dev_blobs, host_blobs = [], []
    for i in range(cfg["n_layers"]):
        W = {p: torch.randn(shapes[p], generator=g, device="cuda") * 0.02 for p in synth.PROJ}
        b = torch.empty(lay.bytes, dtype=torch.uint8, device="cuda")
        pack.pack_layer(cfg, W, ones, ones, b)
        dev_blobs.append(b)
        host_blobs.append(b.cpu().pin_memory())
        del W
    r = cfg["lora_r"]
    A = {p: torch.randn(r, shapes[p][1], generator=g, device="cuda") / r for p in synth.PROJ}
    B = {p: torch.randn(shapes[p][0], r, generator=g, device="cuda") * 0.01 for p in synth.PROJ}
    lora = torch.cat([pack.lora_block(cfg, A, B) for _ in range(cfg["n_layers"])])
    emb = (torch.randn(cfg["vocab"], cfg["hidden"], generator=g, device="cuda") * 0.02).bfloat16()
    head = (torch.randn(cfg["vocab"], cfg["hidden"], generator=g, device="cuda") * 0.02).bfloat16()
    bufs = [torch.empty(lay.bytes, dtype=torch.uint8, device="cuda") for _ in range(2)]
    batch, seq = 1, 512
    tokens = torch.randint(0, cfg["vocab"], (batch, seq), generator=g, device="cuda",
                           dtype=torch.int32)
    ws = workspace(L.stream_stack_workspace_bytes(cfg, batch, seq))
    out = []
    for resident, blobs in ((False, host_blobs), (True, dev_blobs)):
        h = L.StreamStack(cfg, blobs, bufs[0], bufs[1], resident)
        grad = torch.empty_like(lora)
        logits = torch.empty(batch * seq, cfg["vocab"], device="cuda")
        loss = L.stream_stack_step(h, tokens, 1, batch, seq, emb, head, ones, lora, grad, None, ws,
                                   logits_out=logits)
        out.append((loss, logits, grad))
        h.close()
    (ls, lgs, gs), (lr_, lgr, gr) = out
    assert ls == lr_
    assert torch.equal(lgs, lgr)
    assert torch.equal(gs, gr)
    assert math.isfinite(ls) and math.log(cfg["vocab"]) - 1 < ls < math.log(cfg["vocab"]) + 3
    assert torch.isfinite(gs).all()
