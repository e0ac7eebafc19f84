"""LoRA linear, Llama-style decoder layer and the streamed-stack SFT step (CPU oracle).

Test infrastructure only (see the package docstring).  All arithmetic is fp64 on
inputs that are exactly representable (bf16 activations, fp32 dequantised NF4
weights, fp32 LoRA masters).

What the pages fix, and the readings taken where they are silent:

  * LoRA linear, y = x W~^T + s (x A^T) B^T with s = alpha / r; only A [r, K] and
    B [N, r] are trained, the NF4 base W~ is frozen (Soup layer-streaming tutorial,
    "四段資料路徑" part 1; YAML "lora: r, alpha, dropout: 0").  Dropout is 0.
  * Backward still reads the frozen W: dX = dY W~ + s (dY B) A, dA = s (dY B)^T X,
    dB = s dY^T (X A^T) (tutorial, part 3 "Forward＋backward" and FAQ 4).
  * The layer is recomputed in backward from its saved input (tutorial, part 3
    and the "gradient_checkpointing: true" bullet: the streaming wrapper forces
    per-layer checkpointing).  Recomputation gives the same fp program, so the
    oracle's backward simply runs the forward again.
  * The model is only named (Llama-3.1-8B, tutorial "維護者的 4GB／8B 成績").  Reading:
    the HF Llama decoder layer - RMSNorm (eps 1e-5, fp32/fp64 math, gain g) ->
    q/k/v -> rotate-half RoPE (theta 500000, no frequency scaling, positions
    0..S-1 per sequence) -> causal grouped-query attention (scale 1/sqrt(d),
    query head h reads kv head h // (H/Hkv)) -> o, residual; RMSNorm -> SwiGLU
    MLP silu(gate) * up -> down, residual.  No biases.
  * SFT loss: mean token cross-entropy over positions 0..S-2 of every sequence
    with target tokens[t+1] (synthetic data: no prompt mask, no padding).
  * Optimiser: AdamW on the LoRA masters only (the pages' run uses a paged 8-bit
    variant; the reading here is plain fp32 AdamW, lr 2e-4 from the tutorial's
    YAML, betas (0.9, 0.999), eps 1e-8, decoupled weight decay 0, bias-corrected,
    step counter starting at 1).

  * DPO step (Soup release notes "Layer streaming ... 扩展到偏好损失" and the Layer
    Streaming blog, "無記憶體消耗的參考模型"): the reference model is the same
    streamed base with its adapter turned off, i.e. every LoRA branch removed
    (y = x W~^T).  The pages name DPO but print no formula; the reading is the
    published Direct Preference Optimization loss: for a pair (chosen c,
    rejected r), z = beta * ((log pi(c) - log ref(c)) - (log pi(r) - log ref(r))),
    loss = mean over pairs of -log sigmoid(z).  A sequence's log-probability is
    the sum over positions 0..S-2 of log softmax(logits)[tokens[t+1]] (synthetic
    pairs: no prompt mask).

Projection order everywhere: q, k, v, o, gate, up, down.
"""

import math

import numpy as np

PROJ = ("q", "k", "v", "o", "gate", "up", "down")


# --------------------------------------------------------------------------- LoRA
def lora_linear_fwd(x, W, A, B, s):
    """y = x W^T + s (x A^T) B^T ; x [T, K], W [N, K], A [r, K], B [N, r]."""
    x = np.asarray(x, np.float64)
    u = x @ np.asarray(A, np.float64).T
    return x @ np.asarray(W, np.float64).T + s * (u @ np.asarray(B, np.float64).T)


def lora_linear_bwd(dy, x, W, A, B, s):
    """Returns (dx, dA, dB) for y = x W^T + s (x A^T) B^T; W gets no gradient."""
    dy = np.asarray(dy, np.float64)
    x = np.asarray(x, np.float64)
    W = np.asarray(W, np.float64)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    v = dy @ B                     # [T, r]
    u = x @ A.T                    # [T, r]
    dx = dy @ W + s * (v @ A)
    dA = s * (v.T @ x)             # [r, K]
    dB = s * (dy.T @ u)            # [N, r]
    return dx, dA, dB


# --------------------------------------------------------------------------- pieces
def rmsnorm(x, g, eps):
    x = np.asarray(x, np.float64)
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * r * np.asarray(g, np.float64)


def rmsnorm_bwd(dy, x, g, eps):
    """d/dx of x * r(x) * g with r = (mean(x^2) + eps)^-1/2 (g is frozen)."""
    x = np.asarray(x, np.float64)
    D = x.shape[-1]
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    gdy = np.asarray(dy, np.float64) * np.asarray(g, np.float64)
    return r * gdy - x * (r ** 3) * np.sum(gdy * x, axis=-1, keepdims=True) / D


def rope_angles(S, d, theta):
    """angle[pos, i] = pos * theta^(-2i/d), pos in [0, S), i in [0, d/2)."""
    i = np.arange(d // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / d)
    return np.arange(S, dtype=np.float64)[:, None] * inv_freq[None, :]


def rope(x, pos_angles):
    """Rotate-half RoPE on x [T, heads, d]; dims i and i + d/2 form a pair."""
    x = np.asarray(x, np.float64)
    h = x.shape[-1] // 2
    c = np.cos(pos_angles)[:, None, :]
    s = np.sin(pos_angles)[:, None, :]
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def rope_bwd(dy, pos_angles):
    """Transpose of the rotation: rotate by -angle."""
    dy = np.asarray(dy, np.float64)
    h = dy.shape[-1] // 2
    c = np.cos(pos_angles)[:, None, :]
    s = np.sin(pos_angles)[:, None, :]
    d1, d2 = dy[..., :h], dy[..., h:]
    return np.concatenate([d1 * c + d2 * s, d2 * c - d1 * s], axis=-1)


def attention(q, k, v):
    """Causal GQA for one sequence. q [S, H, d], k/v [S, Hkv, d] -> (o [S, H, d], lse [H, S])."""
    S, H, d = q.shape
    Hkv = k.shape[1]
    rep = H // Hkv
    scale = 1.0 / math.sqrt(d)
    o = np.empty((S, H, d), np.float64)
    lse = np.empty((H, S), np.float64)
    mask = np.triu(np.ones((S, S), dtype=bool), k=1)
    for h in range(H):
        g = h // rep
        sc = (q[:, h, :] @ k[:, g, :].T) * scale
        sc[mask] = -np.inf
        m = np.max(sc, axis=-1, keepdims=True)
        p = np.exp(sc - m)
        z = np.sum(p, axis=-1, keepdims=True)
        o[:, h, :] = (p / z) @ v[:, g, :]
        lse[h] = (m + np.log(z))[:, 0]
    return o, lse


def attention_bwd(do, q, k, v):
    """Gradients of causal GQA for one sequence: (dq, dk, dv)."""
    S, H, d = q.shape
    Hkv = k.shape[1]
    rep = H // Hkv
    scale = 1.0 / math.sqrt(d)
    dq = np.zeros_like(q, dtype=np.float64)
    dk = np.zeros_like(k, dtype=np.float64)
    dv = np.zeros_like(v, dtype=np.float64)
    mask = np.triu(np.ones((S, S), dtype=bool), k=1)
    for h in range(H):
        g = h // rep
        sc = (q[:, h, :] @ k[:, g, :].T) * scale
        sc[mask] = -np.inf
        p = np.exp(sc - np.max(sc, axis=-1, keepdims=True))
        p /= np.sum(p, axis=-1, keepdims=True)
        dp = do[:, h, :] @ v[:, g, :].T
        ds = p * (dp - np.sum(dp * p, axis=-1, keepdims=True))
        dv[:, g, :] += p.T @ do[:, h, :]
        dq[:, h, :] = (ds @ k[:, g, :]) * scale
        dk[:, g, :] += (ds.T @ q[:, h, :]) * scale
    return dq, dk, dv


def silu(z):
    return z / (1.0 + np.exp(-z))


def swiglu_bwd(dm, g, u):
    sg = 1.0 / (1.0 + np.exp(-g))
    dg = dm * u * sg * (1.0 + g * (1.0 - sg))
    du = dm * g * sg
    return dg, du


# --------------------------------------------------------------------------- layer
def _lin(p, name, x, s):
    return lora_linear_fwd(x, p["W"][name], p["A"][name], p["B"][name], s)


def decoder_layer_fwd(p, x, cfg, seq_len):
    """One decoder layer on x [T, D] (T = batch * seq_len); returns (out, cache)."""
    H, Hkv, d = cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    eps, s = cfg["rms_eps"], cfg["lora_alpha"] / cfg["lora_r"]
    x = np.asarray(x, np.float64)
    T = x.shape[0]
    nb = T // seq_len
    ang = rope_angles(seq_len, d, cfg["rope_theta"])
    n1 = rmsnorm(x, p["g1"], eps)
    q = _lin(p, "q", n1, s).reshape(T, H, d)
    k = _lin(p, "k", n1, s).reshape(T, Hkv, d)
    v = _lin(p, "v", n1, s).reshape(T, Hkv, d)
    qr = np.empty_like(q)
    kr = np.empty_like(k)
    a = np.empty((T, H, d), np.float64)
    for b in range(nb):
        sl = slice(b * seq_len, (b + 1) * seq_len)
        qr[sl] = rope(q[sl], ang)
        kr[sl] = rope(k[sl], ang)
        a[sl], _ = attention(qr[sl], kr[sl], v[sl])
    a2 = a.reshape(T, H * d)
    h = x + _lin(p, "o", a2, s)
    n2 = rmsnorm(h, p["g2"], eps)
    gt = _lin(p, "gate", n2, s)
    up = _lin(p, "up", n2, s)
    m = silu(gt) * up
    out = h + _lin(p, "down", m, s)
    cache = dict(x=x, n1=n1, qr=qr, kr=kr, v=v, a=a2, h=h, n2=n2, gt=gt, up=up, m=m, ang=ang)
    return out, cache


def decoder_layer_bwd(p, x, dout, cfg, seq_len):
    """Recompute the layer from x, then backpropagate dout [T, D].

    Returns (dx [T, D], grads) with grads[name] = (dA, dB) for the 7 projections.
    """
    H, Hkv, d = cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    eps, s = cfg["rms_eps"], cfg["lora_alpha"] / cfg["lora_r"]
    _, c = decoder_layer_fwd(p, x, cfg, seq_len)
    dout = np.asarray(dout, np.float64)
    T = dout.shape[0]
    nb = T // seq_len
    grads = {}

    def lin_bwd(name, dy, xin):
        dx, dA, dB = lora_linear_bwd(dy, xin, p["W"][name], p["A"][name], p["B"][name], s)
        grads[name] = (dA, dB)
        return dx

    dm = lin_bwd("down", dout, c["m"])
    dg, du = swiglu_bwd(dm, c["gt"], c["up"])
    dn2 = lin_bwd("gate", dg, c["n2"]) + lin_bwd("up", du, c["n2"])
    dh = dout + rmsnorm_bwd(dn2, c["h"], p["g2"], eps)
    da = lin_bwd("o", dh, c["a"]).reshape(T, H, d)
    dq = np.empty((T, H, d))
    dk = np.empty((T, Hkv, d))
    dv = np.empty((T, Hkv, d))
    for b in range(nb):
        sl = slice(b * seq_len, (b + 1) * seq_len)
        dqr, dkr, dv[sl] = attention_bwd(da[sl], c["qr"][sl], c["kr"][sl], c["v"][sl])
        dq[sl] = rope_bwd(dqr, c["ang"])
        dk[sl] = rope_bwd(dkr, c["ang"])
    dn1 = (lin_bwd("q", dq.reshape(T, H * d), c["n1"])
           + lin_bwd("k", dk.reshape(T, Hkv * d), c["n1"])
           + lin_bwd("v", dv.reshape(T, Hkv * d), c["n1"]))
    dx = dh + rmsnorm_bwd(dn1, c["x"], p["g1"], eps)
    return dx, grads


# --------------------------------------------------------------------------- stack
def stack_forward(layers, emb, lm_head, g_final, tokens, cfg):
    """Embedding -> layers -> final RMSNorm -> logits; tokens [B, S]."""
    tokens = np.asarray(tokens)
    Bsz, S = tokens.shape
    h = np.asarray(emb, np.float64)[tokens.reshape(-1)]
    xs = []
    for p in layers:
        xs.append(h)
        h, _ = decoder_layer_fwd(p, h, cfg, S)
    hf = rmsnorm(h, g_final, cfg["rms_eps"])
    logits = hf @ np.asarray(lm_head, np.float64).T
    return logits, dict(xs=xs, h=h, hf=hf)


def sft_loss_and_dlogits(logits, tokens):
    """Mean CE over positions 0..S-2 of each sequence; returns (loss, dlogits)."""
    tokens = np.asarray(tokens)
    Bsz, S = tokens.shape
    lg = np.asarray(logits, np.float64).reshape(Bsz, S, -1)
    m = np.max(lg, axis=-1, keepdims=True)
    z = np.exp(lg - m)
    lse = (m + np.log(np.sum(z, axis=-1, keepdims=True)))[..., 0]
    n = Bsz * (S - 1)
    tgt = tokens[:, 1:]
    picked = np.take_along_axis(lg[:, :-1, :], tgt[..., None], axis=-1)[..., 0]
    loss = float(np.sum(lse[:, :-1] - picked) / n)
    dl = z / np.sum(z, axis=-1, keepdims=True)
    dl[:, -1, :] = 0.0
    bi, ti = np.meshgrid(np.arange(Bsz), np.arange(S - 1), indexing="ij")
    dl[bi, ti, tgt] -= 1.0
    dl[:, :-1, :] /= n
    return loss, dl.reshape(Bsz * S, -1)


def stack_loss_and_grads(layers, emb, lm_head, g_final, tokens, cfg):
    """One SFT forward + backward through the stack; grads only for LoRA A, B."""
    tokens = np.asarray(tokens)
    S = tokens.shape[1]
    logits, c = stack_forward(layers, emb, lm_head, g_final, tokens, cfg)
    loss, dlogits = sft_loss_and_dlogits(logits, tokens)
    dhf = dlogits @ np.asarray(lm_head, np.float64)
    dh = rmsnorm_bwd(dhf, c["h"], g_final, cfg["rms_eps"])
    grads = [None] * len(layers)
    for i in range(len(layers) - 1, -1, -1):
        dh, grads[i] = decoder_layer_bwd(layers[i], c["xs"][i], dh, cfg, S)
    return loss, logits, grads


def adapter_off(layers):
    """The reference model of the DPO step: the same layers with the LoRA branch removed."""
    out = []
    for p in layers:
        q = dict(p)
        q["B"] = {n: np.zeros_like(np.asarray(b, np.float64)) for n, b in p["B"].items()}
        out.append(q)
    return out


def sequence_logprobs(logits, tokens):
    """Sum over positions 0..S-2 of log softmax(logits[t])[tokens[t+1]] -> [B]."""
    tokens = np.asarray(tokens)
    Bsz, S = tokens.shape
    lg = np.asarray(logits, np.float64).reshape(Bsz, S, -1)
    m = np.max(lg, axis=-1, keepdims=True)
    lse = (m + np.log(np.sum(np.exp(lg - m), axis=-1, keepdims=True)))[..., 0]
    picked = np.take_along_axis(lg[:, :-1, :], tokens[:, 1:, None], axis=-1)[..., 0]
    return np.sum(picked - lse[:, :-1], axis=1)


def dpo_loss(lp_pol, lp_ref, beta):
    """lp_* [P, 2] (chosen, rejected) -> (loss, dloss/dlp_pol [P, 2], z [P])."""
    lp_pol = np.asarray(lp_pol, np.float64)
    lp_ref = np.asarray(lp_ref, np.float64)
    P = lp_pol.shape[0]
    z = beta * ((lp_pol[:, 0] - lp_ref[:, 0]) - (lp_pol[:, 1] - lp_ref[:, 1]))
    # -log sigmoid(z) = softplus(-z), written to stay finite for large |z|
    loss = float(np.mean(np.maximum(-z, 0.0) + np.log1p(np.exp(-np.abs(z)))))
    sig_neg = 1.0 / (1.0 + np.exp(z))            # sigmoid(-z) = -d softplus(-z) / dz
    g = np.empty((P, 2))
    g[:, 0] = -beta * sig_neg / P
    g[:, 1] = beta * sig_neg / P
    return loss, g, z


def dpo_loss_and_grads(layers, emb, lm_head, g_final, tokens, cfg, beta):
    """One DPO forward + backward; tokens [P, 2, S] (pair, chosen/rejected, position).

    Returns (loss, policy logits [2P*S, V], LoRA grads per layer, dict(lp_pol, lp_ref, z)).
    """
    tokens = np.asarray(tokens)
    P, two, S = tokens.shape
    assert two == 2
    flat = tokens.reshape(2 * P, S)
    ref_logits, _ = stack_forward(adapter_off(layers), emb, lm_head, g_final, flat, cfg)
    logits, c = stack_forward(layers, emb, lm_head, g_final, flat, cfg)
    lp_ref = sequence_logprobs(ref_logits, flat).reshape(P, 2)
    lp_pol = sequence_logprobs(logits, flat).reshape(P, 2)
    loss, g, z = dpo_loss(lp_pol, lp_ref, beta)
    # d lp_b / d logits[b, t] = onehot(tokens[b, t+1]) - softmax(logits[b, t]), t < S-1
    lg = logits.reshape(2 * P, S, -1)
    sm = np.exp(lg - np.max(lg, axis=-1, keepdims=True))
    sm /= np.sum(sm, axis=-1, keepdims=True)
    dlp = -sm
    dlp[:, -1, :] = 0.0
    bi, ti = np.meshgrid(np.arange(2 * P), np.arange(S - 1), indexing="ij")
    dlp[bi, ti, flat[:, 1:]] += 1.0
    dlogits = (dlp * g.reshape(2 * P)[:, None, None]).reshape(2 * P * S, -1)
    dhf = dlogits @ np.asarray(lm_head, np.float64)
    dh = rmsnorm_bwd(dhf, c["h"], g_final, cfg["rms_eps"])
    grads = [None] * len(layers)
    for i in range(len(layers) - 1, -1, -1):
        dh, grads[i] = decoder_layer_bwd(layers[i], c["xs"][i], dh, cfg, S)
    return loss, logits, grads, dict(lp_pol=lp_pol, lp_ref=lp_ref, z=z)


def adamw_step(param, grad, m, v, step, lr=2e-4, beta1=0.9, beta2=0.999, eps=1e-8, wd=0.0):
    """Decoupled-weight-decay Adam, bias-corrected; step counts from 1.

    Returns (param, m, v) as new fp64 arrays.
    """
    param = np.asarray(param, np.float64) * (1.0 - lr * wd)
    g = np.asarray(grad, np.float64)
    m = beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * g
    v = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * g * g
    mhat = m / (1.0 - beta1 ** step)
    vhat = v / (1.0 - beta2 ** step)
    return param - lr * mhat / (np.sqrt(vhat) + eps), m, v
