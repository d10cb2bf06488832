"""Sharded deployments on CPU: two gloo ranks run the orchestration of the expert-parallel
and tensor-parallel layers (w4a16_int4_mixture_align_b200.shard) for real -- the count
exchange, the all-to-all legs and the all-reduce -- with the per-rank layer computed by
the oracle, and the result checked against the oracle's unsharded layer.

The device steps (send plan, packing, combine, FP32 output, rounding) run on the GPU in
tests/test_gpu_shard.py; here the send buffers and the final sum come from the plain
definitions below, which the GPU test checks those kernels against bit for bit."""
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def ep_send_plan(ids, E_rank, W):
    """One send row per (token, rank owning >= 1 of its experts), rank-major, token order."""
    rows = [(t, d) for d in range(W) for t in range(ids.shape[0])
            if np.any((ids[t] >= d * E_rank) & (ids[t] < (d + 1) * E_rank))]
    counts = [sum(1 for _, d in rows if d == r) for r in range(W)]
    return rows, counts


def ep_send_buffers(x, ids, w, rows, E_rank):
    sx = np.stack([x[t] for t, _ in rows]) if rows else np.zeros((0, x.shape[1]), np.uint16)
    sids = np.full((len(rows), ids.shape[1]), -1, np.int32)
    sw = np.zeros((len(rows), ids.shape[1]), np.float32)
    for i, (t, d) in enumerate(rows):
        here = (ids[t] >= d * E_rank) & (ids[t] < (d + 1) * E_rank)
        sids[i][here] = ids[t][here] - d * E_rank
        sw[i][here] = w[t][here]
    return sx, sids, sw


def ep_sum(back_f32, rows, T, H):
    """Per token, the returned rows summed in FP32 in rank order (rows are rank-major)."""
    acc = np.zeros((T, H), np.float32)
    for i, (t, _) in enumerate(rows):
        acc[t] = acc[t] + back_f32[i]
    return acc


def small_cfg(rank):
    from w4a16_int4_mixture_align_b200 import inputs
    return inputs.MoEConfig("shard", 24, 256, 256, 8, 8, 3, "normal", 7 + rank)


def _worker(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        import oracle
        from helpers import close_report
        from w4a16_int4_mixture_align_b200 import inputs, shard
        cfg = small_cfg(rank)
        gw = inputs.make_weights(small_cfg(0))          # the same global weights on every rank
        x = inputs.make_hidden(cfg)
        logits = np.random.default_rng(100 + rank).standard_normal((cfg.T, cfg.E_global)).astype(np.float32)
        ids, w = oracle.router_topk(logits, cfg.topk)  # global ids
        ref = oracle.moe_forward(x, ids, w, *gw)        # the unsharded layer
        res = {}

        # ---- expert parallel: rank r owns experts [r*E_rank, (r+1)*E_rank)
        E_rank = cfg.E_global // world
        mine = [a[rank * E_rank:(rank + 1) * E_rank] for a in gw]
        rows, counts = ep_send_plan(ids, E_rank, world)
        sx, sids, sw = ep_send_buffers(x, ids, w, rows, E_rank)

        def local(rx, rids, rw):
            out = oracle.moe_forward(rx.view(torch.int16).numpy().view(np.uint16), rids.numpy(), rw.numpy(), *mine)
            return torch.from_numpy(out.view(np.int16)).view(torch.bfloat16)

        back = shard.ep_exchange(torch.from_numpy(sx.view(np.int16)).view(torch.bfloat16), torch.from_numpy(sids),
                                 torch.from_numpy(sw), counts, local)
        back_f32 = oracle.bf16_to_f32(back.view(torch.int16).numpy().view(np.uint16))
        ep_out = oracle.f32_to_bf16(ep_sum(back_f32, rows, cfg.T, cfg.H))
        res["ep"] = close_report(ep_out, ref)

        # ---- tensor parallel: every rank sees the same tokens and owns a slice of every
        # expert's intermediate dimension
        cfg0 = small_cfg(0)
        x0 = inputs.make_hidden(cfg0)
        lg0 = np.random.default_rng(100).standard_normal((cfg0.T, cfg0.E_global)).astype(np.float32)
        ids0, w0 = oracle.router_topk(lg0, cfg0.topk)
        ref0 = oracle.moe_forward(x0, ids0, w0, *gw)
        part = oracle.moe_forward(x0, ids0, w0, *shard.tp_shard_weights(*gw, rank, world))
        partial = torch.from_numpy(oracle.bf16_to_f32(part).copy())
        shard.tp_reduce(partial)
        res["tp"] = close_report(oracle.f32_to_bf16(partial.numpy()), ref0)
        res["tp_slices"] = [a.shape for a in shard.tp_shard_weights(*gw, rank, world)]
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_ep_and_tp_orchestration_gloo_world2():
    import torch.multiprocessing as mp
    sys.path.insert(0, ROOT)
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        for kind in ("ep", "tp"):
            r = out[rank][kind]
            assert r["finite"] and r["max_err"] <= 2e-2 * r["max_ref"] and r["mean_rel"] <= 5e-3, (rank, kind, r)
        # rank r's slice: half of gate + half of up rows, half of W2's K (packed / scales)
        assert out[rank]["tp_slices"] == [(8, 256, 32), (8, 256, 8), (8, 256, 16), (8, 256, 4)]


def test_tp_shard_weights_partition_the_intermediate_dimension():
    sys.path.insert(0, ROOT)
    from w4a16_int4_mixture_align_b200 import inputs, shard
    qw13, s13, qw2, s2 = inputs.make_weights(inputs.MoEConfig("s", 4, 256, 512, 2, 2, 1, "normal", 0))
    parts = [shard.tp_shard_weights(qw13, s13, qw2, s2, r, 4) for r in range(4)]
    # gate and up halves reassemble exactly, W2 columns concatenate back
    gate = np.concatenate([p[0][:, :128] for p in parts], axis=1)
    up = np.concatenate([p[0][:, 128:] for p in parts], axis=1)
    assert np.array_equal(np.concatenate([gate, up], axis=1), qw13)
    assert np.array_equal(np.concatenate([p[2] for p in parts], axis=2), qw2)
    assert np.array_equal(np.concatenate([p[3] for p in parts], axis=2), s2)
    with pytest.raises(ValueError):
        shard.tp_shard_weights(qw13, s13, qw2, s2, 0, 3)   # 512 / 3 is not a multiple of 128


def test_ep_send_plan_definition():
    ids = np.array([[0, 5], [6, 7], [-1, 2], [9, 3]], np.int32)   # 2 ranks x 4 experts; 9 is on no rank
    rows, counts = ep_send_plan(ids, 4, 2)
    assert rows == [(0, 0), (2, 0), (3, 0), (0, 1), (1, 1)] and counts == [3, 2]


def test_global_ids_restrict_to_the_local_ids():
    # an expert-parallel rank's router output by global id: its own experts keep their ids,
    # the others are the ids the layer's local view marks -1
    sys.path.insert(0, ROOT)
    from w4a16_int4_mixture_align_b200 import inputs
    for name in ("ep8_decode", "skew"):
        cfg = inputs.CONFIGS[name]
        g, wg = inputs.make_routing(cfg, global_ids=True)
        loc, wl = inputs.make_routing(cfg)
        assert g.min() >= 0 and g.max() < cfg.E_global
        assert np.array_equal(np.where(g < cfg.E, g, -1), loc) and np.array_equal(wg, wl)
        # every token's top-k experts are distinct
        assert all(len(set(row)) == cfg.topk for row in g[:64])
