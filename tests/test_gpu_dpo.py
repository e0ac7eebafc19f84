"""GPU parity for the DPO step (the same streamed base with its adapter off as the
reference model): the adapter-off layer forward against the oracle, the DPO step
against the fp64 oracle (sequence log-probabilities within 1e-3 relative, the
DPO loss within the bound those errors imply, policy logits and LoRA gradients
within normwise 2e-2), and streamed vs resident bit-equality with the same layer
copies as an SFT step."""
import numpy as np
import pytest

from oracle import model as om
from layer_streamed_qlora_nf4_b200 import synth

pytestmark = pytest.mark.gpu
TOL = 2e-2
BETA = 0.1


@pytest.fixture(scope="module")
def L():
    from layer_streamed_qlora_nf4_b200 import lib
    lib.load()
    return lib


@pytest.fixture(scope="module")
def small(L):
    from test_gpu_stack import Stack
    return Stack(L, synth.SMALL, 5)


def _dpo(L, st, h, tokens_np, pairs, seq, opt=None):
    import torch
    from gpu_util import workspace
    cfg = st.cfg
    ws = workspace(L.stream_stack_dpo_workspace_bytes(cfg, pairs, seq))
    tokens = torch.from_numpy(tokens_np.astype(np.int32)).cuda()
    lora = st.lora.clone()
    grad = torch.full_like(lora, float("nan"))
    logits = torch.empty(2 * pairs * seq, cfg["vocab"], dtype=torch.float32, device="cuda")
    loss, lps = L.stream_stack_dpo_step(h, tokens, pairs, seq, BETA, st.emb, st.head, st.gf, lora,
                                        grad, opt, ws, logits_out=logits)
    return loss, np.array(lps, np.float64), logits, grad


def test_layer_forward_with_the_adapter_off(L):
    import torch
    from gpu_util import dev, normwise_err, workspace
    from test_gpu_layer import _device_layer, _oracle_params
    cfg, batch, seq = synth.SMALL, 2, 100
    lw = synth.layer_weights(12, cfg)
    x = synth.bf16_bits_to_f32(synth.activations(13, batch * seq, cfg["hidden"]))
    blob, _ = _device_layer(L, cfg, lw)
    y = torch.empty(batch * seq, cfg["hidden"], dtype=torch.float32, device="cuda")
    L.decoder_layer_fwd(cfg, blob, None, dev(x), batch, seq, y,
                        workspace(L.decoder_layer_workspace_bytes(cfg, batch, seq)))
    torch.cuda.synchronize()
    p = om.adapter_off([_oracle_params(lw, cfg)])[0]
    ref, _ = om.decoder_layer_fwd(p, x, cfg, seq)
    assert normwise_err(y.cpu().numpy(), ref) <= TOL


def test_dpo_step_matches_oracle(L, small):
    from gpu_util import check_stack_grad, normwise_err
    from layer_streamed_qlora_nf4_b200 import pack
    cfg = small.cfg
    pairs, seq = 2, 64
    tokens = synth.tokens(40, 2 * pairs, seq, cfg["vocab"]).reshape(pairs, 2, seq)
    h = small.handle(L, resident=False)
    loss, lps, logits, grad = _dpo(L, small, h, tokens, pairs, seq)
    h.close()
    rloss, rlogits, rgrads, aux = om.dpo_loss_and_grads(
        small.oracle_layers(), synth.bf16_bits_to_f32(small.emb_bits),
        synth.bf16_bits_to_f32(small.head_bits), synth.bf16_bits_to_f32(small.gf_bits), tokens,
        cfg, BETA)
    ref_lps = np.concatenate([aux["lp_pol"], aux["lp_ref"]], axis=1)   # per pair: pc, pr, rc, rr
    assert np.all(np.abs(lps - ref_lps) <= 1e-3 * np.abs(ref_lps)), (lps, ref_lps)
    # |d loss / d lp| <= beta / pairs for every sequence, so the loss error is bounded
    # by the log-probability errors it is computed from (plus fp32 rounding)
    bound = BETA / pairs * np.sum(np.abs(lps - ref_lps)) + 1e-5
    assert abs(loss - rloss) <= bound, (loss, rloss, bound)
    assert normwise_err(logits.cpu().numpy(), rlogits) <= TOL
    nf = L.lsq_lora_layout_get(cfg).floats_per_layer
    for i in range(cfg["n_layers"]):
        gv = pack.lora_views(cfg, grad[i * nf:(i + 1) * nf])
        for name in synth.PROJ:
            check_stack_grad(gv[name][0].cpu().numpy(), rgrads[i][name][0], name, (i, "A"))
            check_stack_grad(gv[name][1].cpu().numpy(), rgrads[i][name][1], name, (i, "B"))
    assert L.lsq_device_status() == 0


def test_dpo_streamed_equals_resident_bitwise(L, small):
    import torch
    cfg = small.cfg
    pairs, seq = 1, 96
    tokens = synth.tokens(41, 2 * pairs, seq, cfg["vocab"]).reshape(pairs, 2, seq)
    hs = small.handle(L, resident=False)
    hr = small.handle(L, resident=True)
    ls, lps_s, lgs, gs = _dpo(L, small, hs, tokens, pairs, seq)
    st = L.stream_stack_last_stats(hs)
    lr_, lps_r, lgr, gr = _dpo(L, small, hr, tokens, pairs, seq)
    hs.close()
    hr.close()
    assert ls == lr_ and np.array_equal(lps_s, lps_r)
    assert torch.equal(lgs, lgr) and torch.equal(gs, gr)
    nl = cfg["n_layers"]
    assert st["layer_copies"] == 2 * nl - 2      # the reference costs no extra layer copies


def test_dpo_rejects_bad_arguments(L, small):
    import torch
    from gpu_util import workspace
    h = small.handle(L, resident=False)
    tok = torch.zeros(1, 2, 16, dtype=torch.int32, device="cuda")
    ws = workspace(L.stream_stack_dpo_workspace_bytes(small.cfg, 1, 16))
    for pairs, beta, code in ((0, 0.1, L.LSQ_ERR_SHAPE), (33, 0.1, L.LSQ_ERR_SHAPE),
                              (1, 0.0, L.LSQ_ERR_INVALID), (1, float("nan"), L.LSQ_ERR_INVALID)):
        with pytest.raises(L.LsqError) as e:
            L.stream_stack_dpo_step(h, tok, pairs, 16, beta, small.emb, small.head, small.gf,
                                    small.lora.clone(), torch.empty_like(small.lora), None, ws)
        assert e.value.code == code
    h.close()
