"""Pins for the oracle's LoRA linear, decoder layer, stack loss and AdamW (CPU only).

The references here are independent of the oracle's code: fp64 central finite
differences, torch autograd, explicit per-query attention loops, closed forms
(RoPE identities, ln V), the HF transformers Llama implementation, and
torch.optim.AdamW.
"""

import math

import numpy as np
import pytest
import torch

from oracle import model as om

TINY = dict(hidden=64, ffn=128, n_heads=4, n_kv_heads=2, head_dim=16, rope_theta=500000.0,
            rms_eps=1e-5, lora_r=2, lora_alpha=4.0)


def _layer_params(seed, cfg, b_std=0.3):
    g = np.random.default_rng(seed)
    D, F = cfg["hidden"], cfg["ffn"]
    qd = cfg["n_heads"] * cfg["head_dim"]
    kvd = cfg["n_kv_heads"] * cfg["head_dim"]
    shapes = dict(q=(qd, D), k=(kvd, D), v=(kvd, D), o=(D, qd), gate=(F, D), up=(F, D), down=(D, F))
    r = cfg["lora_r"]
    W = {n: g.standard_normal(s) * 0.15 for n, s in shapes.items()}
    A = {n: g.standard_normal((r, s[1])) / r for n, s in shapes.items()}
    B = {n: g.standard_normal((s[0], r)) * b_std for n, s in shapes.items()}
    return dict(W=W, A=A, B=B, g1=1.0 + 0.1 * g.standard_normal(D), g2=1.0 + 0.1 * g.standard_normal(D))


# ------------------------------------------------------------------ LoRA linear
def test_lora_b_zero_and_s_zero_give_base():
    g = np.random.default_rng(0)
    x, W = g.standard_normal((5, 64)), g.standard_normal((32, 64))
    A, B = g.standard_normal((4, 64)), np.zeros((32, 4))
    base = x @ W.T
    assert np.array_equal(om.lora_linear_fwd(x, W, A, B, 2.0), base)
    assert np.array_equal(om.lora_linear_fwd(x, W, A, g.standard_normal((32, 4)), 0.0), base)
    _, dA, _ = om.lora_linear_bwd(g.standard_normal((5, 32)), x, W, A, B, 2.0)
    assert np.all(dA == 0)


def test_lora_linearity_in_x():
    g = np.random.default_rng(1)
    W, A, B = g.standard_normal((16, 64)), g.standard_normal((2, 64)), g.standard_normal((16, 2))
    x1, x2 = g.standard_normal((3, 64)), g.standard_normal((3, 64))
    lhs = om.lora_linear_fwd(2.5 * x1 - x2, W, A, B, 2.0)
    rhs = 2.5 * om.lora_linear_fwd(x1, W, A, B, 2.0) - om.lora_linear_fwd(x2, W, A, B, 2.0)
    assert np.max(np.abs(lhs - rhs)) < 1e-12


def test_lora_bwd_finite_differences():
    g = np.random.default_rng(2)
    T, K, N, r, s = 3, 64, 64, 2, 2.0
    x, W = g.standard_normal((T, K)), g.standard_normal((N, K))
    A, B, dy = g.standard_normal((r, K)), g.standard_normal((N, r)), g.standard_normal((T, N))
    dx, dA, dB = om.lora_linear_bwd(dy, x, W, A, B, s)
    h = 1e-4

    def L(x_, A_, B_):
        return float(np.sum(om.lora_linear_fwd(x_, W, A_, B_, s) * dy))

    for arr, grad, which in ((x, dx, 0), (A, dA, 1), (B, dB, 2)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            p, m = arr.copy(), arr.copy()
            p[idx] += h
            m[idx] -= h
            args_p = [x, A, B]
            args_m = [x, A, B]
            args_p[which], args_m[which] = p, m
            num[idx] = (L(*args_p) - L(*args_m)) / (2 * h)
        assert np.max(np.abs(num - grad)) / np.max(np.abs(grad)) < 1e-6


def test_lora_bwd_matches_torch_autograd():
    g = np.random.default_rng(3)
    T, K, N, r, s = 7, 96, 80, 4, 1.5
    x, W = g.standard_normal((T, K)), g.standard_normal((N, K))
    A, B, dy = g.standard_normal((r, K)), g.standard_normal((N, r)), g.standard_normal((T, N))
    tx = torch.tensor(x, requires_grad=True)
    tA = torch.tensor(A, requires_grad=True)
    tB = torch.tensor(B, requires_grad=True)
    y = torch.nn.functional.linear(tx, torch.tensor(W)) + s * torch.nn.functional.linear(
        torch.nn.functional.linear(tx, tA), tB)
    y.backward(torch.tensor(dy))
    dx, dA, dB = om.lora_linear_bwd(dy, x, W, A, B, s)
    assert np.allclose(y.detach().numpy(), om.lora_linear_fwd(x, W, A, B, s), rtol=0, atol=1e-11)
    for a, b in ((dx, tx.grad), (dA, tA.grad), (dB, tB.grad)):
        assert np.allclose(a, b.numpy(), rtol=0, atol=1e-10)


# ------------------------------------------------------------------ pieces
def test_attention_matches_brute_force_loops():
    g = np.random.default_rng(4)
    S, H, Hkv, d = 9, 4, 2, 8
    q, k, v = g.standard_normal((S, H, d)), g.standard_normal((S, Hkv, d)), g.standard_normal((S, Hkv, d))
    o, lse = om.attention(q, k, v)
    for h in range(H):
        kv = h // (H // Hkv)
        for i in range(S):
            sc = [sum(q[i, h, e] * k[j, kv, e] for e in range(d)) / math.sqrt(d) for j in range(i + 1)]
            mx = max(sc)
            w = [math.exp(x - mx) for x in sc]
            z = sum(w)
            ref = [sum(w[j] * v[j, kv, e] for j in range(i + 1)) / z for e in range(d)]
            assert np.max(np.abs(np.array(ref) - o[i, h])) < 1e-12
            assert abs(mx + math.log(z) - lse[h, i]) < 1e-12


def test_attention_bwd_matches_torch_autograd():
    g = np.random.default_rng(5)
    S, H, Hkv, d = 11, 4, 1, 8
    q, k, v = g.standard_normal((S, H, d)), g.standard_normal((S, Hkv, d)), g.standard_normal((S, Hkv, d))
    do = g.standard_normal((S, H, d))
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    kk = tk.repeat_interleave(H // Hkv, dim=1).permute(1, 0, 2)
    vv = tv.repeat_interleave(H // Hkv, dim=1).permute(1, 0, 2)
    sc = tq.permute(1, 0, 2) @ kk.transpose(1, 2) / math.sqrt(d)
    sc = sc.masked_fill(torch.triu(torch.ones(S, S, dtype=torch.bool), 1), float("-inf"))
    o = (torch.softmax(sc, -1) @ vv).permute(1, 0, 2)
    o.backward(torch.tensor(do))
    dq, dk, dv = om.attention_bwd(do, q, k, v)
    for a, b in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.allclose(a, b.numpy(), rtol=0, atol=1e-11)


def test_rope_identities():
    g = np.random.default_rng(6)
    S, d = 40, 16
    ang = om.rope_angles(S, d, 500000.0)
    x = g.standard_normal((S, 3, d))
    y = om.rope(x, ang)
    assert np.allclose(y[0], x[0], rtol=0, atol=0)                       # pos 0 = identity
    h = d // 2
    assert np.allclose(x[..., :h] ** 2 + x[..., h:] ** 2, y[..., :h] ** 2 + y[..., h:] ** 2, atol=1e-12)
    qv, kv = g.standard_normal(d), g.standard_normal(d)
    def dot(m, n):
        return float(om.rope(np.tile(qv, (S, 1, 1)), ang)[m, 0] @ om.rope(np.tile(kv, (S, 1, 1)), ang)[n, 0])
    assert abs(dot(7, 3) - dot(30, 26)) < 1e-10 and abs(dot(5, 5) - dot(0, 0)) < 1e-10
    # inverse frequencies: theta^(-2i/d)
    assert abs(ang[1, 1] - 500000.0 ** (-2.0 / d)) < 1e-15
    assert np.allclose(om.rope_bwd(y, ang), x, atol=1e-12)              # rotation is orthogonal


def test_rmsnorm_and_silu_closed_forms():
    g = np.random.default_rng(7)
    x = g.standard_normal((4, 256)) * 3
    y = om.rmsnorm(x, np.ones(256), 0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, -1)), 1.0, atol=1e-12)
    assert om.silu(np.array([0.0]))[0] == 0.0
    assert abs(om.silu(np.array([1.0]))[0] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-15


def test_rmsnorm_and_swiglu_bwd_torch_autograd():
    g = np.random.default_rng(8)
    x, gg, dy = g.standard_normal((5, 32)), g.standard_normal(32), g.standard_normal((5, 32))
    tx = torch.tensor(x, requires_grad=True)
    y = tx * torch.rsqrt(torch.mean(tx * tx, -1, keepdim=True) + 1e-5) * torch.tensor(gg)
    y.backward(torch.tensor(dy))
    assert np.allclose(om.rmsnorm_bwd(dy, x, gg, 1e-5), tx.grad.numpy(), atol=1e-12)
    a, b, dm = g.standard_normal((5, 32)), g.standard_normal((5, 32)), g.standard_normal((5, 32))
    ta, tb = torch.tensor(a, requires_grad=True), torch.tensor(b, requires_grad=True)
    (torch.nn.functional.silu(ta) * tb).backward(torch.tensor(dm))
    dg, du = om.swiglu_bwd(dm, a, b)
    assert np.allclose(dg, ta.grad.numpy(), atol=1e-12) and np.allclose(du, tb.grad.numpy(), atol=1e-12)


# ------------------------------------------------------------------ HF Llama pins
# HF's Llama runs RMSNorm and the rotary tables in fp32 even inside a float64
# model, so these comparisons are normwise at fp32 level (1e-5); an error in the
# layer's wiring (a transposed operand, a wrong sign, a dropped term) is O(1).
def _close(a, b, tol=1e-5):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return np.max(np.abs(a - b)) <= tol * np.max(np.abs(b))


class _LoraLinear(torch.nn.Module):
    def __init__(self, W, A, B, s):
        super().__init__()
        self.register_buffer("W", torch.tensor(W))
        self.A = torch.nn.Parameter(torch.tensor(A))
        self.B = torch.nn.Parameter(torch.tensor(B))
        self.s = s

    def forward(self, x):
        return x @ self.W.T + self.s * ((x @ self.A.T) @ self.B.T)


def _hf_model(cfg, layers, n_layers, vocab=97, emb=None, head=None, gf=None):
    from transformers import LlamaConfig, LlamaForCausalLM
    hc = LlamaConfig(hidden_size=cfg["hidden"], intermediate_size=cfg["ffn"],
                     num_attention_heads=cfg["n_heads"], num_key_value_heads=cfg["n_kv_heads"],
                     head_dim=cfg["head_dim"], rms_norm_eps=cfg["rms_eps"], vocab_size=vocab,
                     num_hidden_layers=n_layers, tie_word_embeddings=False,
                     rope_parameters={"rope_theta": cfg["rope_theta"], "rope_type": "default"},
                     attention_bias=False, mlp_bias=False, hidden_act="silu",
                     max_position_embeddings=4096)
    hc._attn_implementation = "eager"
    m = LlamaForCausalLM(hc).double().eval()
    s = cfg["lora_alpha"] / cfg["lora_r"]
    for L, p in zip(m.model.layers, layers):
        at, mlp = L.self_attn, L.mlp
        at.q_proj, at.k_proj = _LoraLinear(p["W"]["q"], p["A"]["q"], p["B"]["q"], s), _LoraLinear(p["W"]["k"], p["A"]["k"], p["B"]["k"], s)
        at.v_proj, at.o_proj = _LoraLinear(p["W"]["v"], p["A"]["v"], p["B"]["v"], s), _LoraLinear(p["W"]["o"], p["A"]["o"], p["B"]["o"], s)
        mlp.gate_proj = _LoraLinear(p["W"]["gate"], p["A"]["gate"], p["B"]["gate"], s)
        mlp.up_proj = _LoraLinear(p["W"]["up"], p["A"]["up"], p["B"]["up"], s)
        mlp.down_proj = _LoraLinear(p["W"]["down"], p["A"]["down"], p["B"]["down"], s)
        with torch.no_grad():
            L.input_layernorm.weight.copy_(torch.tensor(p["g1"]))
            L.post_attention_layernorm.weight.copy_(torch.tensor(p["g2"]))
    if emb is not None:
        with torch.no_grad():
            m.model.embed_tokens.weight.copy_(torch.tensor(emb))
            m.lm_head.weight.copy_(torch.tensor(head))
            m.model.norm.weight.copy_(torch.tensor(gf))
    return m


def test_decoder_layer_matches_hf_llama_forward_and_backward():
    cfg = TINY
    p = _layer_params(20, cfg)
    g = np.random.default_rng(21)
    Bsz, S = 2, 8
    x = g.standard_normal((Bsz * S, cfg["hidden"]))
    dout = g.standard_normal((Bsz * S, cfg["hidden"]))
    m = _hf_model(cfg, [p], 1)
    captured = {}
    m.model.layers[0].register_forward_hook(lambda mod, i, o: captured.__setitem__("o", o[0] if isinstance(o, tuple) else o))
    tx = torch.tensor(x.reshape(Bsz, S, -1), requires_grad=True)
    m.model(inputs_embeds=tx)
    out_hf = captured["o"]
    (out_hf * torch.tensor(dout.reshape(Bsz, S, -1))).sum().backward()
    out, _ = om.decoder_layer_fwd(p, x, cfg, S)
    assert _close(out, out_hf.detach().numpy().reshape(Bsz * S, -1))
    dx, grads = om.decoder_layer_bwd(p, x, dout, cfg, S)
    assert _close(dx, tx.grad.numpy().reshape(Bsz * S, -1))
    L = m.model.layers[0]
    mods = dict(q=L.self_attn.q_proj, k=L.self_attn.k_proj, v=L.self_attn.v_proj, o=L.self_attn.o_proj,
                gate=L.mlp.gate_proj, up=L.mlp.up_proj, down=L.mlp.down_proj)
    for n, mod in mods.items():
        assert _close(grads[n][0], mod.A.grad.numpy()), n
        assert _close(grads[n][1], mod.B.grad.numpy()), n


def test_decoder_layer_finite_differences():
    cfg = dict(TINY, hidden=64, ffn=128)
    p = _layer_params(22, cfg, b_std=0.2)
    g = np.random.default_rng(23)
    S = 8
    x = g.standard_normal((S, cfg["hidden"]))
    dout = g.standard_normal((S, cfg["hidden"]))
    dx, grads = om.decoder_layer_bwd(p, x, dout, cfg, S)
    h = 1e-5

    def L():
        return float(np.sum(om.decoder_layer_fwd(p, x, cfg, S)[0] * dout))

    for (arr, grad) in ((x, dx), (p["A"]["q"], grads["q"][0]), (p["B"]["down"], grads["down"][1]),
                        (p["A"]["gate"], grads["gate"][0]), (p["B"]["v"], grads["v"][1])):
        gi = np.random.default_rng(24)
        for _ in range(6):
            idx = tuple(int(gi.integers(0, n)) for n in arr.shape)
            old = arr[idx]
            arr[idx] = old + h
            lp = L()
            arr[idx] = old - h
            lm = L()
            arr[idx] = old
            num = (lp - lm) / (2 * h)
            assert abs(num - grad[idx]) <= 1e-6 * max(1.0, np.max(np.abs(grad))), (num, grad[idx])


def test_stack_matches_hf_llama_causal_lm_loss_and_grads():
    cfg = TINY
    V, nl = 97, 2
    layers = [_layer_params(30 + i, cfg) for i in range(nl)]
    g = np.random.default_rng(31)
    emb, head = g.standard_normal((V, cfg["hidden"])) * 0.5, g.standard_normal((V, cfg["hidden"])) * 0.5
    gf = 1.0 + 0.1 * g.standard_normal(cfg["hidden"])
    tokens = g.integers(0, V, size=(2, 8))
    m = _hf_model(cfg, layers, nl, V, emb, head, gf)
    ids = torch.tensor(tokens, dtype=torch.long)
    out = m(input_ids=ids, labels=ids)
    out.loss.backward()
    loss, logits, grads = om.stack_loss_and_grads(layers, emb, head, gf, tokens, cfg)
    assert abs(loss - out.loss.item()) < 1e-5 * abs(loss)
    assert _close(logits, out.logits.detach().numpy().reshape(16, V))
    # two layers of HF's fp32-internal norms/rotary: observed <= 2e-5 normwise
    for i, L in enumerate(m.model.layers):
        mods = dict(q=L.self_attn.q_proj, k=L.self_attn.k_proj, v=L.self_attn.v_proj, o=L.self_attn.o_proj,
                    gate=L.mlp.gate_proj, up=L.mlp.up_proj, down=L.mlp.down_proj)
        for n, mod in mods.items():
            assert _close(grads[i][n][0], mod.A.grad.numpy(), 1e-4), (i, n)
            assert _close(grads[i][n][1], mod.B.grad.numpy(), 1e-4), (i, n)


def test_loss_is_ln_v_for_equal_logits():
    tokens = np.random.default_rng(32).integers(0, 50, size=(3, 6))
    loss, dl = om.sft_loss_and_dlogits(np.zeros((18, 50)), tokens)
    assert abs(loss - math.log(50)) < 1e-14
    assert np.allclose(dl.reshape(3, 6, 50)[:, -1], 0.0)
    assert np.allclose(dl.reshape(3, 6, 50)[:, :-1].sum(-1), 0.0, atol=1e-15)


def test_adamw_matches_torch():
    g = np.random.default_rng(33)
    p0 = g.standard_normal(50)
    tp = torch.nn.Parameter(torch.tensor(p0))
    opt = torch.optim.AdamW([tp], lr=2e-4, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.01)
    p, m, v = p0.copy(), np.zeros(50), np.zeros(50)
    for step in range(1, 4):
        grad = g.standard_normal(50)
        tp.grad = torch.tensor(grad)
        opt.step()
        p, m, v = om.adamw_step(p, grad, m, v, step, wd=0.01)
    assert np.max(np.abs(p - tp.detach().numpy())) < 1e-14


# ------------------------------------------------------------------ DPO step
def _dpo_case(seed, P=2, S=7, V=97, nl=2):
    cfg = TINY
    layers = [_layer_params(seed + i, cfg) for i in range(nl)]
    g = np.random.default_rng(seed + 50)
    emb, head = g.standard_normal((V, cfg["hidden"])) * 0.5, g.standard_normal((V, cfg["hidden"])) * 0.5
    gf = 1.0 + 0.1 * g.standard_normal(cfg["hidden"])
    tokens = g.integers(0, V, size=(P, 2, S))
    return cfg, layers, emb, head, gf, tokens


def test_sequence_logprobs_brute_force_loops():
    g = np.random.default_rng(60)
    lg = g.standard_normal((2 * 5, 11))
    tok = g.integers(0, 11, size=(2, 5))
    got = om.sequence_logprobs(lg, tok)
    for b in range(2):
        want = 0.0
        for t in range(4):
            row = lg[b * 5 + t]
            want += math.log(math.exp(row[tok[b, t + 1]]) / sum(math.exp(v) for v in row))
        assert abs(got[b] - want) < 1e-12


def test_dpo_matches_hf_llama_autograd():
    # Policy: the HF Llama with LoRA on all seven projections; reference: the same
    # model with every LoRA branch removed; the DPO loss written with torch ops.
    cfg, layers, emb, head, gf, tokens = _dpo_case(70)
    V, nl, beta = 97, 2, 0.1
    pol = _hf_model(cfg, layers, nl, V, emb, head, gf)
    ref = _hf_model(cfg, om.adapter_off(layers), nl, V, emb, head, gf)
    ids = torch.tensor(tokens.reshape(-1, tokens.shape[-1]), dtype=torch.long)

    def seq_lp(model):
        lp = torch.log_softmax(model(input_ids=ids).logits, dim=-1)
        return torch.gather(lp[:, :-1], 2, ids[:, 1:, None])[..., 0].sum(1).reshape(-1, 2)
    with torch.no_grad():
        lr = seq_lp(ref)
    lpp = seq_lp(pol)
    z = beta * ((lpp[:, 0] - lr[:, 0]) - (lpp[:, 1] - lr[:, 1]))
    tloss = -torch.nn.functional.logsigmoid(z).mean()
    tloss.backward()
    loss, logits, grads, aux = om.dpo_loss_and_grads(layers, emb, head, gf, tokens, cfg, beta)
    assert abs(loss - tloss.item()) < 1e-5 * abs(loss)
    assert _close(aux["lp_ref"], lr.numpy()) and _close(aux["lp_pol"], lpp.detach().numpy())
    for i, L in enumerate(pol.model.layers):
        mods = dict(q=L.self_attn.q_proj, k=L.self_attn.k_proj, v=L.self_attn.v_proj, o=L.self_attn.o_proj,
                    gate=L.mlp.gate_proj, up=L.mlp.up_proj, down=L.mlp.down_proj)
        for n, mod in mods.items():
            assert _close(grads[i][n][0], mod.A.grad.numpy(), 1e-4), (i, n)
            assert _close(grads[i][n][1], mod.B.grad.numpy(), 1e-4), (i, n)


def test_dpo_with_the_adapter_at_zero_is_log2_and_swaps_sign():
    cfg, layers, emb, head, gf, tokens = _dpo_case(80)
    zero = om.adapter_off(layers)           # policy == reference
    loss, _, grads, aux = om.dpo_loss_and_grads(zero, emb, head, gf, tokens, cfg, 0.1)
    assert abs(loss - math.log(2.0)) < 1e-12 and np.allclose(aux["z"], 0.0, atol=1e-12)
    for gl in grads:                        # B = 0: no gradient can reach A
        for n in om.PROJ:
            assert np.max(np.abs(gl[n][0])) == 0.0
    # swapping chosen and rejected flips z: softplus(z) - softplus(-z) = z
    l1, _, _, a1 = om.dpo_loss_and_grads(layers, emb, head, gf, tokens, cfg, 0.1)
    l2, _, _, a2 = om.dpo_loss_and_grads(layers, emb, head, gf, tokens[:, ::-1, :], cfg, 0.1)
    assert np.allclose(a2["z"], -a1["z"], atol=1e-12)
    assert abs((l2 - l1) - np.mean(a1["z"])) < 1e-12


def test_dpo_finite_differences():
    cfg, layers, emb, head, gf, tokens = _dpo_case(90, P=1, S=5)
    beta = 0.5
    _, _, grads, _ = om.dpo_loss_and_grads(layers, emb, head, gf, tokens, cfg, beta)
    g = np.random.default_rng(91)
    h = 1e-6
    for (li, n, k) in ((0, "q", "A"), (1, "down", "B"), (0, "gate", "B"), (1, "v", "A")):
        arr = layers[li][k][n]
        idx = tuple(int(g.integers(0, d)) for d in arr.shape)
        old = arr[idx]
        arr[idx] = old + h
        lp = om.dpo_loss_and_grads(layers, emb, head, gf, tokens, cfg, beta)[0]
        arr[idx] = old - h
        lm = om.dpo_loss_and_grads(layers, emb, head, gf, tokens, cfg, beta)[0]
        arr[idx] = old
        fd = (lp - lm) / (2 * h)
        an = grads[li][n][0 if k == "A" else 1][idx]
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)) + 1e-8, (li, n, k, fd, an)
