"""Run by test_gpu_zz_shard.py in a fresh process (NCCL lives only there).

A streamed stack sharded over a one-rank NCCL communicator (the layer slice is
the whole layer, the in-place all-gather a local no-op) must give the same step,
bit for bit, as the unsharded stack; stream_stack_shard's argument checks hold.
Likewise a stack whose steps average the LoRA gradients over a one-rank
communicator (stream_stack_reduce_grads: per-layer all-reduces on their own
stream, the optimiser waiting for them) must give the same gradients and the
same AdamW update, bit for bit, as one without.
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path[:0] = [os.path.dirname(HERE), HERE]


def _expect(fn, code):
    from layer_streamed_qlora_nf4_b200 import lib as L
    try:
        fn()
    except L.LsqError as e:
        assert e.code == code, (e.code, code, str(e))
        return
    raise AssertionError("no error, expected code %d" % code)


def main():
    import torch
    from layer_streamed_qlora_nf4_b200 import lib as L
    from layer_streamed_qlora_nf4_b200 import synth
    from test_gpu_stack import Stack, _step
    L.load()
    st = Stack(L, synth.SMALL, 5)
    batch, seq = 1, 128
    tokens = synth.tokens(33, batch, seq, st.cfg["vocab"])
    h0 = st.handle(L, resident=False)
    loss0, logits0, grad0, _ = _step(L, st, h0, tokens, 1, batch, seq)
    s0 = L.stream_stack_last_stats(h0)
    h0.close()

    S = L.lsq_shard_bytes(st.blob_bytes, 1)
    assert S >= st.blob_bytes and S % 256 == 0
    bufs = [torch.empty(S, dtype=torch.uint8, device="cuda") for _ in range(2)]
    h1 = L.StreamStack(st.cfg, st.host_blobs, bufs[0], bufs[1], False)
    nid = L.lsq_nccl_unique_id()
    assert len(nid) == L.LSQ_NCCL_ID_BYTES
    _expect(lambda: h1.shard(nid, 1, 0, S - 256), L.LSQ_ERR_WORKSPACE)
    _expect(lambda: h1.shard(nid, 1, 1, S), L.LSQ_ERR_INVALID)
    _expect(lambda: h1.shard(nid, 0, 0, S), L.LSQ_ERR_INVALID)
    _expect(lambda: L.stream_stack_shard(h1, nid[:64] + bytes(64), 1, -1, S), L.LSQ_ERR_INVALID)
    hr = st.handle(L, resident=True)
    _expect(lambda: hr.shard(nid, 1, 0, S), L.LSQ_ERR_INVALID)
    hr.close()
    h1.shard(nid, 1, 0, S)
    _expect(lambda: h1.shard(nid, 1, 0, S), L.LSQ_ERR_INVALID)   # already sharded
    loss1, logits1, grad1, _ = _step(L, st, h1, tokens, 1, batch, seq)
    s1 = L.stream_stack_last_stats(h1)
    loss2, _, grad2, _ = _step(L, st, h1, tokens, 1, batch, seq)   # buffers carried over
    h1.close()
    assert loss1 == loss0 == loss2, (loss0, loss1, loss2)
    assert torch.equal(logits1, logits0)
    assert torch.equal(grad1, grad0) and torch.equal(grad2, grad0)
    assert s1["layer_copies"] == s0["layer_copies"]
    assert s1["h2d_bytes"] == s0["h2d_bytes"] == s0["layer_copies"] * st.blob_bytes

    # gradient averaging inside the step, one rank, with the optimiser update
    def opt_state():
        return dict(lr=2e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, step=1,
                    m=torch.zeros_like(st.lora), v=torch.zeros_like(st.lora))
    tok2 = synth.tokens(34, 2 * batch, seq, st.cfg["vocab"]).reshape(2, batch, seq)
    h2 = st.handle(L, resident=False)
    la, lg_a, ga, pa = _step(L, st, h2, tok2, 2, batch, seq, opt=opt_state())
    h2.close()
    h3 = st.handle(L, resident=False)
    gid = L.lsq_nccl_unique_id()
    _expect(lambda: h3.reduce_grads(gid, 1, 1), L.LSQ_ERR_INVALID)
    _expect(lambda: h3.reduce_grads(gid, 0, 0), L.LSQ_ERR_INVALID)
    h3.reduce_grads(gid, 1, 0)
    _expect(lambda: h3.reduce_grads(gid, 1, 0), L.LSQ_ERR_INVALID)   # already set up
    lb, lg_b, gb, pb = _step(L, st, h3, tok2, 2, batch, seq, opt=opt_state())
    h3.close()
    assert la == lb and torch.equal(lg_a, lg_b)
    assert torch.equal(ga, gb) and torch.equal(pa, pb)
    assert L.lsq_device_status() == 0
    print("shard ok")


if __name__ == "__main__":
    main()
