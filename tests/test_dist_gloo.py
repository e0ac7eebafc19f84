"""Data-parallel host logic with two gloo ranks on the CPU: every rank ends a
step with the same averaged LoRA gradient, hence the same AdamW update, and the
step time reported is the maximum over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from layer_streamed_qlora_nf4_b200 import dp
    from oracle import model as om
    r, w = dp.init("gloo", timeout_s=60)
    assert (r, w) == (rank, world)
    g = np.random.default_rng(dp.token_seed(5, rank))
    grad = torch.from_numpy(g.standard_normal(1000))          # this rank's gradient
    mine = grad.clone()
    dp.average_(grad)
    gathered = [torch.zeros_like(mine) for _ in range(world)]
    torch.distributed.all_gather(gathered, mine)
    p0 = np.linspace(-1, 1, 1000)
    p1, _, _ = om.adamw_step(p0, grad.numpy(), np.zeros(1000), np.zeros(1000), 1)
    t = dp.max_over_ranks(10.0 + rank, "cpu")
    out[rank] = (grad.numpy().copy(), torch.stack(gathered).mean(0).numpy(), p1, t)
    dp.barrier()
    torch.distributed.destroy_process_group()


def test_two_rank_gradient_average_and_timing():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    g0, mean0, p0, t0 = out[0]
    g1, mean1, p1, t1 = out[1]
    assert np.array_equal(g0, g1)                  # identical averaged gradient on both ranks
    assert np.allclose(g0, mean0, atol=1e-15)      # equal to the mean of the ranks' gradients
    assert np.array_equal(p0, p1)                  # hence identical parameters after AdamW
    assert t0 == t1 == 11.0                        # max over ranks


def _dp_sft_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from layer_streamed_qlora_nf4_b200 import dp
    from oracle import model as om
    from test_oracle_model import TINY, _layer_params
    dp.init("gloo", timeout_s=60)
    layers = [_layer_params(40 + i, TINY) for i in range(2)]
    g = np.random.default_rng(41)
    V = 97
    emb, head = g.standard_normal((V, 64)) * 0.5, g.standard_normal((V, 64)) * 0.5
    gf = np.ones(64)
    tokens = g.integers(0, V, size=(world, 6))          # one sequence per rank
    loss, _, grads = om.stack_loss_and_grads(layers, emb, head, gf, tokens[rank:rank + 1], TINY)
    flat = torch.from_numpy(np.concatenate([np.concatenate([grads[i][n][0].ravel(),
                                                            grads[i][n][1].ravel()])
                                            for i in range(2) for n in om.PROJ]))
    dp.average_(flat)
    lt = torch.tensor([loss], dtype=torch.float64)
    dp.average_(lt)
    out[rank] = (flat.numpy().copy(), float(lt[0]), tokens)
    dp.barrier()
    torch.distributed.destroy_process_group()


def test_two_rank_sft_step_equals_the_union_batch():
    # Data-parallel replicas (one sequence per rank), gradients averaged across the
    # ranks: the same loss and LoRA gradient as one step on both sequences together.
    import sys
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    from oracle import model as om
    from test_oracle_model import TINY, _layer_params
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_dp_sft_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    f0, l0, tokens = out[0]
    f1, l1, _ = out[1]
    assert np.array_equal(f0, f1) and l0 == l1
    layers = [_layer_params(40 + i, TINY) for i in range(2)]
    g = np.random.default_rng(41)
    emb, head = g.standard_normal((97, 64)) * 0.5, g.standard_normal((97, 64)) * 0.5
    loss, _, grads = om.stack_loss_and_grads(layers, emb, head, np.ones(64), tokens, TINY)
    ref = np.concatenate([np.concatenate([grads[i][n][0].ravel(), grads[i][n][1].ravel()])
                          for i in range(2) for n in om.PROJ])
    assert abs(l0 - loss) <= 1e-12 * abs(loss)
    assert np.max(np.abs(f0 - ref)) <= 1e-12 * np.max(np.abs(ref))


def _shard_worker(rank, world, port, sizes, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from layer_streamed_qlora_nf4_b200 import dp
    from layer_streamed_qlora_nf4_b200 import lib as L
    L.load()                     # lsq_shard_bytes is host-only
    dp.init("gloo", timeout_s=60)
    nid = dp.broadcast_bytes(lambda: os.urandom(L.LSQ_NCCL_ID_BYTES))
    res = []
    for nbytes in sizes:
        S = L.lsq_shard_bytes(nbytes, world)
        # every rank holds the same frozen layer in host memory
        blob = torch.from_numpy(np.random.default_rng(nbytes).integers(0, 256, nbytes, np.uint8))
        buf = torch.zeros(world * S, dtype=torch.uint8)             # this rank's layer buffer
        off = rank * S
        ln = max(0, min(S, nbytes - off))
        buf[off:off + ln] = blob[off:off + ln]                       # its host->device slice
        parts = [torch.empty(S, dtype=torch.uint8) for _ in range(world)]
        torch.distributed.all_gather(parts, buf[off:off + S].clone())  # the in-place all-gather
        buf = torch.cat(parts)
        res.append((S, ln, bool(torch.equal(buf[:nbytes], blob))))
    out[rank] = (nid, res)
    dp.barrier()
    torch.distributed.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_layer_shard_plan_reassembles_the_layer(world):
    """Each rank copies only bytes [r S, min((r+1) S, bytes)) of a layer (the
    slice stream_stack_shard documents, S from lsq_shard_bytes) and the
    all-gather of the ranks' S-byte slots rebuilds the layer on every rank; the
    NCCL id made on rank 0 reaches every rank unchanged."""
    sizes = [300, 1000, 3 * 4096 + 17, 122_699_776]   # the last: one 8B NF4 layer
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, sizes, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    ids = {out[r][0] for r in range(world)}
    assert len(ids) == 1 and len(ids.pop()) == 128
    for k, nbytes in enumerate(sizes):
        S = out[0][1][k][0]
        assert S % 256 == 0 and S * world >= nbytes and (S - 256) * world < nbytes
        assert sum(out[r][1][k][1] for r in range(world)) == nbytes   # every byte read once
        assert all(out[r][1][k][2] for r in range(world))


def _absent_peer_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import time
    from layer_streamed_qlora_nf4_b200 import dp
    dp.init("gloo", timeout_s=5)
    if rank == 1:
        out[rank] = "left"          # this rank leaves between steps, before the id exchange
        os._exit(0)
    t0 = time.time()
    try:
        dp.broadcast_bytes(lambda: os.urandom(128))
        out[rank] = ("no error", time.time() - t0)
    except Exception as e:      # the process group's timeout, or the peer's closed connection
        out[rank] = (type(e).__name__, time.time() - t0)
    os._exit(0)


def test_id_exchange_fails_instead_of_hanging_when_a_rank_is_gone():
    """stream_stack_shard's NCCL id reaches the ranks through dp.broadcast_bytes: if a
    rank has left, the others get an error within the process group's timeout."""
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_absent_peer_worker, args=(r, world, port, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[1] == "left"
    err, secs = out[0]
    assert err != "no error" and secs < 60, (err, secs)
