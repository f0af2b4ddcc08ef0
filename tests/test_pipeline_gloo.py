"""Layer pipeline over ranks (world size 2-3, gloo, CPU): stages of contiguous layers, micro-batches
passed point to point.  The stages run real OPT layers (the CPU oracle's float64 evaluation,
fp16 activations between layers), so the pipeline's output must equal, bit for bit, the same
layers run one after another in one process; a stage that leaves is detected by the next one
through the process group's timeout."""
import os
import socket
import time

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from bit_compressed_decode_b200 import pipeline

H_, HID, FFN, NL, S, P = 2, 128, 256, 7, 10, 3


def _port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _env(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))


def _layers_and_caches(first, count):
    """Oracle layers [first, first+count) with their caches, filled by a P-token prompt."""
    import oracle
    import seeded_inputs as si
    ws, cs = [], []
    prompt = si.hidden_block(40, si.STREAM["prompt"], S, P, HID).reshape(S * P, HID)
    seq, pos = np.repeat(np.arange(S), P), np.tile(np.arange(P), S)
    rows = prompt
    for l in range(first + count):
        w = oracle.LayerWeights(si.layer_weights_f16(50 + l, HID, FFN, std=0.05, bias_std=0.05, ln_random=True))
        c = oracle.KVCache(S, H_, HID // H_, 64)
        r, _ = oracle.layer_rows(w, H_, c, rows, seq, pos)
        rows = oracle.f64_to_f16(r)
        if l >= first:
            ws.append(w)
            cs.append(c)
    return ws, cs


def _oracle_runner(ws, cs):
    import oracle

    def run(x, s0, n):
        cur = x.numpy().view(np.float16)
        for w, c in zip(ws, cs):
            r, _ = oracle.layer_rows(w, H_, c, cur, np.arange(s0, s0 + n), np.full(n, P))
            cur = oracle.f64_to_f16(r)
        return torch.from_numpy(np.ascontiguousarray(cur).view(np.int16))

    return run


def _decode_input():
    import seeded_inputs as si
    return si.decode_inputs(41, 0, S, HID)


def _worker(rank, world, port, parts, q):
    _env(rank, world, port)
    from bit_compressed_decode_b200 import replicas
    replicas.init("gloo", timeout_s=60)
    import torch.distributed as dist
    first, count = pipeline.split_layers(NL, world, rank)
    ws, cs = _layers_and_caches(first, count)
    stage = pipeline.PipelineStage(_oracle_runner(ws, cs), HID, rank, world)
    # fp16 activations travel as their 16-bit patterns
    x = torch.from_numpy(_decode_input().view(np.int16)) if rank == 0 else None
    y = stage.step(x, pipeline.micro_batches(S, parts), dtype=torch.int16, device=torch.device("cpu"))
    if y is not None:
        q.put((rank, y.numpy().view(np.float16).copy()))
    dist.barrier()
    dist.destroy_process_group()


def _sequential():
    import oracle
    ws, cs = _layers_and_caches(0, NL)
    cur = _decode_input()
    for w, c in zip(ws, cs):
        r, _ = oracle.layer_rows(w, H_, c, cur, np.arange(S), np.full(S, P))
        cur = oracle.f64_to_f16(r)
    return cur


def test_split_layers_and_micro_batches():
    for nl in (1, 7, 48, 96):
        for world in (1, 2, 3, 8):
            parts = [pipeline.split_layers(nl, world, r) for r in range(world)]
            assert sum(c for _, c in parts) == nl
            assert all(parts[r][0] + parts[r][1] == parts[r + 1][0] for r in range(world - 1))
    assert pipeline.micro_batches(10, 4) == [(0, 3), (3, 3), (6, 2), (8, 2)]
    assert pipeline.micro_batches(2, 4) == [(0, 1), (1, 1)]
    with pytest.raises(ValueError):
        pipeline.micro_batches(5, 0)


@pytest.mark.parametrize("world,parts", [(3, 4), (2, 1)])
def test_pipeline_equals_layers_in_one_process(world, parts):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    ps = [ctx.Process(target=_worker, args=(r, world, port, parts, q)) for r in range(world)]
    for p in ps:
        p.start()
    rank, y = q.get(timeout=300)
    for p in ps:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert rank == world - 1
    assert np.array_equal(y.view(np.uint16), _sequential().view(np.uint16))


def _worker_leaves(rank, world, port, q):
    _env(rank, world, port)
    from bit_compressed_decode_b200 import replicas
    replicas.init("gloo", timeout_s=3)
    if rank == 0:                                    # stage 0 leaves before sending anything
        q.put((rank, "left"))
        q.close()
        q.join_thread()
        os._exit(0)
    stage = pipeline.PipelineStage(lambda x, s0, n: x, HID, rank, world)
    t0 = time.time()
    try:
        stage.step(None, pipeline.micro_batches(S, 2), dtype=torch.int16, device=torch.device("cpu"))
        q.put((rank, "no error"))
    except Exception as e:                           # the receive ends with an error on the host
        q.put((rank, "error", type(e).__name__, time.time() - t0))


def test_stage_that_leaves_is_detected_by_the_next():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    ps = [ctx.Process(target=_worker_leaves, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(2)), key=lambda t: t[0])
    for p in ps:
        p.join(timeout=60)
    assert res[0][1] == "left"
    assert res[1][1] == "error" and res[1][3] < 60
