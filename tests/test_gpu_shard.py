"""Exchange kernels of sharded deployments on one GPU, ranks emulated in one process.

Expert parallel: chord_ep_plan / chord_ep_pack / chord_ep_combine against the plain
definitions (bit for bit), and a whole layer over 4 emulated ranks -- every rank's send
buffers routed to the owners of their experts by slicing, each owner running the layer
on its experts -- against the oracle's unsharded layer. Tensor parallel: the FP32 partial
outputs (CHORD_FLAG_OUTPUT_FP32) of 2 emulated ranks summed and rounded by
chord_round_bf16 against the unsharded layer; the rounding itself bit for bit against the
oracle's. (The collectives between real ranks are covered by tests/test_shard_ranks.py.)"""
import numpy as np
import pytest

import oracle
from helpers import assert_layer_close, ensure_built
from test_shard_ranks import ep_send_buffers, ep_send_plan, ep_sum
from w4a16_int4_mixture_align_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def chord():
    ensure_built()
    from w4a16_int4_mixture_align_b200 import chord as c
    return c


def _dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _bf16(a):
    import torch
    return _dev(a.view(np.int16)).view(torch.bfloat16)


def _bits(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def plan_and_pack(chord, x, ids, w, E_rank, W):
    import torch
    T, k = ids.shape
    H = x.shape[1]
    send_rows = torch.full((max(T * W, 1),), -7, dtype=torch.int32, device="cuda")
    offsets = torch.full((W + 1,), -7, dtype=torch.int32, device="cuda")
    row_of = torch.full((max(T * W, 1),), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(chord.chord_ep_plan_workspace_bytes(T, W), 256), dtype=torch.uint8, device="cuda")
    d_ids = _dev(ids)
    chord.chord_ep_plan(d_ids, E_rank, W, send_rows, offsets, row_of, ws)
    sx = torch.zeros((max(T * W, 1), H), dtype=torch.bfloat16, device="cuda")
    sids = torch.full((max(T * W, 1), k), -7, dtype=torch.int32, device="cuda")
    sw = torch.full((max(T * W, 1), k), -7.0, dtype=torch.float32, device="cuda")
    chord.chord_ep_pack(_bf16(x), d_ids, _dev(w), E_rank, W, send_rows, offsets, row_of, sx, sids, sw)
    torch.cuda.synchronize()
    off = offsets.cpu().numpy()
    n = int(off[W])
    return (send_rows.cpu().numpy()[:n], off, row_of, sx[:n], sids[:n], sw[:n])


@pytest.mark.parametrize("T,E_rank,W,k,seed", [(37, 4, 4, 4, 0), (600, 8, 8, 8, 1), (1, 2, 3, 2, 2), (0, 4, 2, 2, 3)])
def test_ep_plan_and_pack_match_the_definition(chord, T, E_rank, W, k, seed):
    rng = np.random.default_rng(seed)
    ids = rng.integers(-1, E_rank * W + 2, size=(T, k)).astype(np.int32)   # some on no rank
    x = rng.integers(0, 1 << 16, size=(T, 64)).astype(np.uint16)
    w = rng.random((T, k), dtype=np.float32)
    rows, counts = ep_send_plan(ids, E_rank, W)
    send_rows, off, row_of, sx, sids, sw = plan_and_pack(chord, x, ids, w, E_rank, W)
    assert list(send_rows) == [t * W + d for t, d in rows]
    assert list(np.diff(off)) == counts and off[0] == 0
    ex, eids, ew = ep_send_buffers(x, ids, w, rows, E_rank)
    assert np.array_equal(_bits(sx).reshape(ex.shape), ex)
    assert np.array_equal(sids.cpu().numpy(), eids) and np.array_equal(sw.cpu().numpy(), ew)
    ro = row_of.cpu().numpy()[:T * W]
    exp = np.full(T * W, -1, np.int32)
    for i, (t, d) in enumerate(rows):
        exp[t * W + d] = i
    assert np.array_equal(ro, exp)


def test_ep_combine_matches_the_definition(chord):
    import torch
    rng = np.random.default_rng(5)
    T, W, H = 50, 4, 128
    ids = rng.integers(-1, 4 * W, size=(T, 3)).astype(np.int32)
    rows, _ = ep_send_plan(ids, 4, W)
    back = rng.standard_normal((len(rows), H)).astype(np.float32)
    back_bits = oracle.f32_to_bf16(back)
    row_of = np.full(T * W, -1, np.int32)
    for i, (t, d) in enumerate(rows):
        row_of[t * W + d] = i
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    chord.chord_ep_combine(_bf16(back_bits), _dev(row_of), W, out)
    torch.cuda.synchronize()
    exp = oracle.f32_to_bf16(ep_sum(oracle.bf16_to_f32(back_bits), rows, T, H))
    assert np.array_equal(_bits(out), exp)   # FP32 sum in rank order, one rounding


@pytest.mark.parametrize("path", [0, "stream", "tensor"])
def test_expert_parallel_layer_over_four_ranks(chord, path):
    import torch
    W, E_rank = 4, 4
    E = W * E_rank
    cfg = inputs.MoEConfig("ep", 40, 256, 128, E, E, 4, "normal", 11)
    gw = inputs.make_weights(cfg)
    flags = {0: 0, "stream": chord.CHORD_FLAG_FORCE_STREAM, "tensor": chord.CHORD_FLAG_FORCE_TENSOR}[path]
    layers = [chord.ChordMoE(gw[0][d * E_rank:(d + 1) * E_rank], gw[1][d * E_rank:(d + 1) * E_rank].view(np.int16),
                             gw[2][d * E_rank:(d + 1) * E_rank], gw[3][d * E_rank:(d + 1) * E_rank].view(np.int16),
                             topk=cfg.topk, E_global=E, max_tokens=64) for d in range(W)]
    # each rank's own tokens and their global routing
    toks = []
    for r in range(W):
        c = inputs.MoEConfig("ep", 33 + 7 * r, 256, 128, E, E, 4, "normal", 20 + r)
        ids, w = inputs.make_routing(c)
        toks.append((inputs.make_hidden(c), ids, w))
    sent = [plan_and_pack(chord, x, ids, w, E_rank, W) for x, ids, w in toks]
    # all-to-all by slicing: owner d receives, in source order, the rows each source sent it
    back_parts = [[None] * W for _ in range(W)]
    for d in range(W):
        pieces = [(r, slice(int(s[1][d]), int(s[1][d + 1]))) for r, s in enumerate(sent)]
        rx = torch.cat([sent[r][3][sl] for r, sl in pieces])
        rids = torch.cat([sent[r][4][sl] for r, sl in pieces])
        rw = torch.cat([sent[r][5][sl] for r, sl in pieces])
        out = layers[d](rx, rids, rw, flags=flags)
        assert layers[d].check_status() == 0
        start = 0
        for r, sl in pieces:
            n = sl.stop - sl.start
            back_parts[r][d] = out[start:start + n]
            start += n
    for r, (x, ids, w) in enumerate(toks):
        back = torch.cat(back_parts[r])
        out = torch.empty((x.shape[0], cfg.H), dtype=torch.bfloat16, device="cuda")
        chord.chord_ep_combine(back, sent[r][2], W, out)
        torch.cuda.synchronize()
        assert_layer_close(_bits(out), oracle.moe_forward(x, ids, w, *gw))


@pytest.mark.parametrize("path", [0, "stream", "tensor"])
def test_tensor_parallel_layer_over_two_ranks(chord, path):
    import torch
    from w4a16_int4_mixture_align_b200 import shard
    cfg = inputs.MoEConfig("tp", 45, 256, 256, 8, 8, 2, "normal", 13)
    d = inputs.make_inputs(cfg)
    flags = {0: 0, "stream": chord.CHORD_FLAG_FORCE_STREAM, "tensor": chord.CHORD_FLAG_FORCE_TENSOR}[path]
    x, ids, w = _bf16(d["x"]), _dev(d["topk_ids"]), _dev(d["topk_weights"])
    total = torch.zeros((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
    for r in range(2):
        q13, s13, q2, s2 = shard.tp_shard_weights(d["qw13"], d["s13"], d["qw2"], d["s2"], r, 2)
        L = chord.ChordMoE(q13, s13.view(np.int16), q2, s2.view(np.int16), topk=cfg.topk, max_tokens=cfg.T)
        part = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device="cuda")
        L.align(ids)
        chord.chord_moe_forward(x, ids, w, L.sorted_ids, L.expert_ids, L.ntp, L.block_m, L.w13, L.w2, L.I, L.E,
                                part, L.workspace, flags | chord.CHORD_FLAG_OUTPUT_FP32)
        torch.cuda.synchronize()
        assert L.check_status() == 0
        total += part   # the all-reduce of the ranks' partials
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device="cuda")
    chord.chord_round_bf16(total, out)
    torch.cuda.synchronize()
    assert_layer_close(_bits(out), oracle.moe_forward(d["x"], d["topk_ids"], d["topk_weights"], d["qw13"], d["s13"],
                                                      d["qw2"], d["s2"]))


@pytest.mark.parametrize("path", ["stream", "tensor"])
def test_fp32_output_rounds_to_the_bf16_output(chord, path):
    # the FP32 output is the sum the BF16 output rounds: rounding it gives the same bits
    import torch
    d = inputs.make_inputs(inputs.CONFIGS["tiny"])
    flags = chord.CHORD_FLAG_FORCE_STREAM if path == "stream" else chord.CHORD_FLAG_FORCE_TENSOR
    L = chord.ChordMoE(d["qw13"], d["s13"].view(np.int16), d["qw2"], d["s2"].view(np.int16), topk=2, max_tokens=16,
                       block_m=16)
    x, ids, w = _bf16(d["x"]), _dev(d["topk_ids"]), _dev(d["topk_weights"])
    ref = L(x, ids, w, flags=flags)
    f32 = torch.empty((16, 256), dtype=torch.float32, device="cuda")
    chord.chord_moe_forward(x, ids, w, L.sorted_ids, L.expert_ids, L.ntp, L.block_m, L.w13, L.w2, L.I, L.E, f32,
                            L.workspace, flags | chord.CHORD_FLAG_OUTPUT_FP32)
    out = torch.empty((16, 256), dtype=torch.bfloat16, device="cuda")
    chord.chord_round_bf16(f32, out)
    torch.cuda.synchronize()
    assert L.check_status() == 0
    assert np.array_equal(_bits(out), _bits(ref))


def test_round_bf16_matches_the_oracle(chord):
    import torch
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(4000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 4000),
                        # exact ties between two bf16 values (both parities of the kept bit), signs
                        (((np.arange(64, dtype=np.uint32) + 0x3F00) << 16) | 0x8000).view(np.float32),
                        (((np.arange(64, dtype=np.uint32) + 0xBF00) << 16) | 0x8000).view(np.float32),
                        np.array([3.3895314e38, -3.3895314e38, 0.0, -0.0], np.float32)]).astype(np.float32)
    out = torch.empty(v.size, dtype=torch.bfloat16, device="cuda")
    chord.chord_round_bf16(_dev(v), out)
    torch.cuda.synchronize()
    assert np.array_equal(_bits(out), oracle.f32_to_bf16(v))


@pytest.mark.parametrize("W,n", [(4, 4096 * 64), (8, 7168 * 33), (3, 4 * 5), (1, 7168)])
def test_tp_reduce_round_over_rank_buffers(chord, W, n):
    # W ranks' buffers on one GPU stand in for peer memory: each rank's call reduces its
    # slice of all partials in rank order and writes every rank's output; after all W
    # calls every output is bf16 of the rank-ordered FP32 sum, bit for bit
    import torch
    rng = np.random.default_rng(W * 1000 + n % 997)
    parts = [(rng.standard_normal(n) * 10.0 ** rng.integers(-3, 4, n)).astype(np.float32) for _ in range(W)]
    ref = parts[0].copy()
    for p_ in parts[1:]:
        ref = (ref + p_).astype(np.float32)   # FP32 sums in rank order
    exp = oracle.f32_to_bf16(ref)
    d_parts = [_dev(p_) for p_ in parts]
    outs = [torch.full((n,), 7, dtype=torch.int16, device="cuda").view(torch.bfloat16) for _ in range(W)]
    for r in range(W):
        chord.chord_tp_reduce_round(d_parts, outs, r)
    torch.cuda.synchronize()
    for o in outs:
        assert np.array_equal(_bits(o), exp)
