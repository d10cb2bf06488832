"""The whole layer on the GPU vs the CPU oracle.

Tiny workload: every output element. Kimi-K2-shaped workloads at full size: a seeded
sample of 512 token rows among those with a local slot (all such rows when fewer),
computed one by one by the oracle, in the same launch configuration the benchmark
times. Both schedules (weight streaming and tensor core) are checked where they apply.
"""
import numpy as np
import pytest

import oracle
from helpers import assert_layer_close, bf16_bits_to_f64, ensure_built
from w4a16_int4_mixture_align_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def chord():
    ensure_built()
    from w4a16_int4_mixture_align_b200 import chord as c
    return c


def to_dev(d):
    import torch
    dev = torch.device("cuda")
    return {
        "x": torch.from_numpy(d["x"].view(np.int16)).to(dev).view(torch.bfloat16),
        "ids": torch.from_numpy(d["topk_ids"]).to(dev),
        "w": torch.from_numpy(d["topk_weights"]).to(dev),
    }


def make_layer(chord, d, block_m=None, max_tokens=None):
    cfg = d["cfg"]
    return chord.ChordMoE(d["qw13"], d["s13"].view(np.int16), d["qw2"], d["s2"].view(np.int16),
                          topk=cfg.topk, E_global=cfg.E_global,
                          max_tokens=max_tokens or cfg.T, block_m=block_m)


def run_layer(layer, d, flags=0):
    import torch
    t = to_dev(d)
    out = layer(t["x"], t["ids"], t["w"], flags=flags)
    torch.cuda.synchronize()
    st = layer.check_status()
    assert st == 0, hex(st)
    return out.view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_rows(d, rows):
    return oracle.moe_forward(d["x"], d["topk_ids"], d["topk_weights"], d["qw13"], d["s13"],
                              d["qw2"], d["s2"], rows=rows)


# ------------------------------------------------------------------------------ tiny

@pytest.fixture(scope="module")
def tiny():
    return inputs.make_inputs(inputs.CONFIGS["tiny"])


@pytest.mark.parametrize("block_m", [1, 8, 16, 32, 64, 144, 240, 256])
@pytest.mark.parametrize("path", ["stream", "tensor"])
def test_tiny_full_output(chord, tiny, block_m, path):
    flags = chord.CHORD_FLAG_FORCE_STREAM if path == "stream" else chord.CHORD_FLAG_FORCE_TENSOR
    layer = make_layer(chord, tiny, block_m=block_m)
    got = run_layer(layer, tiny, flags)
    ref = oracle_rows(tiny, None)
    assert_layer_close(got, ref)


def test_tiny_matches_golden_fixture_within_tolerance(chord, tiny):
    import os
    g = {}
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.txt")
    rows = []
    for line in open(path):
        if line.startswith("out "):
            rows.append([int(v, 16) for v in line.split()[2:]])
    ref = np.array(rows, dtype=np.uint16)
    got = run_layer(make_layer(chord, tiny), tiny)
    assert_layer_close(got, ref)


# ------------------------------------------------------------------------------ full size

BIG = ["ep8_decode", "ep8_prefill", "tp8_decode", "tp8_prefill", "skew"]


@pytest.fixture(scope="module")
def big_inputs():
    cache = {}

    def get(name):
        if name not in cache:
            cache.clear()
            cache[name] = inputs.make_inputs(inputs.CONFIGS[name])
        return cache[name]
    return get


@pytest.mark.parametrize("name", BIG)
def test_full_size_sampled_rows(chord, big_inputs, name):
    d = big_inputs(name)
    cfg = d["cfg"]
    layer = make_layer(chord, d)
    got = run_layer(layer, d)
    rows = inputs.sample_rows(d["topk_ids"], cfg.E, 512, seed=1)
    ref = oracle_rows(d, rows)
    r = assert_layer_close(got[rows], ref)
    # rows without a local slot are exactly zero
    none = ~((d["topk_ids"] >= 0) & (d["topk_ids"] < cfg.E)).any(axis=1)
    assert np.all(bf16_bits_to_f64(got[none]) == 0)
    print(name, "block_m", layer.block_m, r)


# ------------------------------------------------------------------------------ edges

def small_inputs(T, E=8, E_global=None, topk=2, H=256, I=128, seed=3):
    cfg = inputs.MoEConfig("edge", T, H, I, E, E_global or E, topk, "normal", seed)
    return inputs.make_inputs(cfg)


@pytest.mark.parametrize("T", [1, 3, 37, 129])
@pytest.mark.parametrize("path", ["stream", "tensor"])
def test_ragged_token_counts(chord, T, path):
    d = small_inputs(T, E=6, E_global=10, topk=3, H=384, I=256)
    flags = chord.CHORD_FLAG_FORCE_STREAM if path == "stream" else chord.CHORD_FLAG_FORCE_TENSOR
    got = run_layer(make_layer(chord, d, block_m=16), d, flags)
    assert_layer_close(got, oracle_rows(d, None))


# Weight streaming with stream-K (K of at least 512): with fewer (item, stage) units than
# workers every worker holds about one stage, so an item is split over up to KS workers and
# its owner adds up to KS - 1 partial sums from other CTAs; mid-size unit counts cut items
# at arbitrary stages. A second call must give the same bits (the partial sums' flags are
# reset by the kernel that reads them).
@pytest.mark.parametrize("T,E,topk,H,I,block_m", [
    (4, 4, 2, 2048, 256, 8),     # gate_up KS = 4, RU < workers; down K = 256 (short kernel)
    (5, 3, 3, 3584, 1024, 16),   # KS = 7 and 2, token chunks of 16
    (16, 8, 2, 7168, 512, 8),    # KS = 14, ranges cut items at any stage
    (33, 6, 4, 1024, 2048, 32),  # token chunks of 32, down KS = 4
])
def test_stream_k_splits_match_the_oracle(chord, T, E, topk, H, I, block_m):
    d = small_inputs(T, E=E, topk=topk, H=H, I=I, seed=17)
    layer = make_layer(chord, d, block_m=block_m)
    first = run_layer(layer, d, chord.CHORD_FLAG_FORCE_STREAM)
    assert_layer_close(first, oracle_rows(d, None))
    again = run_layer(layer, d, chord.CHORD_FLAG_FORCE_STREAM)
    assert np.array_equal(first, again)


@pytest.mark.parametrize("path", ["stream", "tensor"])
def test_no_local_slot_gives_zero_rows(chord, path):
    d = small_inputs(20)
    d["topk_ids"][:] = -1
    flags = chord.CHORD_FLAG_FORCE_STREAM if path == "stream" else chord.CHORD_FLAG_FORCE_TENSOR
    got = run_layer(make_layer(chord, d, block_m=8), d, flags)
    assert np.all(bf16_bits_to_f64(got) == 0)


@pytest.mark.parametrize("path", ["stream", "tensor"])
def test_topk_above_one_warp(chord, path):
    # top-k 40 of 64 experts: the combine holds slots 32..39 in a second lane set
    d = small_inputs(9, E=64, topk=40, H=256, I=128)
    flags = chord.CHORD_FLAG_FORCE_STREAM if path == "stream" else chord.CHORD_FLAG_FORCE_TENSOR
    got = run_layer(make_layer(chord, d, block_m=16), d, flags)
    assert_layer_close(got, oracle_rows(d, None))


def test_single_expert_topk1(chord):
    d = small_inputs(33, E=1, topk=1)
    got = run_layer(make_layer(chord, d, block_m=8), d)
    assert_layer_close(got, oracle_rows(d, None))


def test_one_expert_takes_everything(chord):
    d = small_inputs(300, E=4, topk=2)
    d["topk_ids"][:, 0] = 2
    d["topk_ids"][:, 1] = -1
    for bm in (8, 256):
        got = run_layer(make_layer(chord, d, block_m=bm), d)
        assert_layer_close(got, oracle_rows(d, None))


def test_repeated_calls_are_deterministic_in_routing_and_stable(chord, tiny):
    layer = make_layer(chord, tiny, block_m=8)
    a = run_layer(layer, tiny)
    b = run_layer(layer, tiny)
    assert np.array_equal(a, b)


# ------------------------------------------------------------------------------ errors

def test_swapped_weight_roles_fail_on_host(chord, tiny):
    import torch
    layer = make_layer(chord, tiny, block_m=8)
    t = to_dev(tiny)
    layer.align(t["ids"])
    out = torch.empty((16, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(chord.ChordError) as ei:
        chord.chord_moe_forward(t["x"], t["ids"], t["w"], layer.sorted_ids, layer.expert_ids, layer.ntp,
                                layer.block_m, layer.w2, layer.w13, layer.I, layer.E, out, layer.workspace)
    assert ei.value.status == chord.CHORD_ERR_LAYOUT_MISMATCH


def test_foreign_blob_header_checked_on_device(chord, tiny):
    import torch
    layer = make_layer(chord, tiny, block_m=8)
    t = to_dev(tiny)
    layer.align(t["ids"])
    # copies the host registry does not know: the kernels check the header themselves
    w13c, w2c = layer.w2.clone(), layer.w13.clone()          # roles swapped
    out = torch.zeros((16, 256), dtype=torch.bfloat16, device="cuda")
    chord.chord_moe_forward(t["x"], t["ids"], t["w"], layer.sorted_ids, layer.expert_ids, layer.ntp,
                            layer.block_m, w13c, w2c, layer.I, layer.E, out, layer.workspace,
                            chord.CHORD_FLAG_FORCE_STREAM)
    st = layer.check_status()
    assert st & chord.CHORD_DEV_BLOB_MISMATCH
    assert layer.check_status() == 0  # cleared by the read


def test_routing_validation_flags_corrupt_tensors(chord, tiny):
    import torch
    layer = make_layer(chord, tiny, block_m=8)
    t = to_dev(tiny)
    layer.align(t["ids"])
    out = torch.zeros((16, 256), dtype=torch.bfloat16, device="cuda")
    bad = layer.expert_ids.clone()
    bad[0] = 1000
    chord.chord_moe_forward(t["x"], t["ids"], t["w"], layer.sorted_ids, bad, layer.ntp,
                            layer.block_m, layer.w13, layer.w2, layer.I, layer.E, out, layer.workspace,
                            chord.CHORD_FLAG_VALIDATE_ROUTING | chord.CHORD_FLAG_FORCE_STREAM)
    assert layer.check_status() & chord.CHORD_DEV_ROUTING_INVALID
    # valid routing passes validation
    chord.chord_moe_forward(t["x"], t["ids"], t["w"], layer.sorted_ids, layer.expert_ids, layer.ntp,
                            layer.block_m, layer.w13, layer.w2, layer.I, layer.E, out, layer.workspace,
                            chord.CHORD_FLAG_VALIDATE_ROUTING)
    assert layer.check_status() == 0


@pytest.mark.parametrize("path", ["stream", "tensor"])
@pytest.mark.parametrize("bm_align,bm_forward", [(16, 8), (8, 16), (8, 64), (64, 8)])
def test_block_m_mismatch_is_caught_on_the_device(chord, tiny, path, bm_align, bm_forward):
    # routing sorted for one block_m, forward called with another: the kernels check the
    # tag in num_tokens_padded[1] before reading expert_ids, compute nothing, write zero
    # rows and raise CHORD_DEV_BLOCK_M_MISMATCH (no host readback)
    import torch
    src = make_layer(chord, tiny, block_m=bm_align)
    dst = make_layer(chord, tiny, block_m=bm_forward)  # workspace sized for bm_forward
    t = to_dev(tiny)
    src.align(t["ids"])
    flags = chord.CHORD_FLAG_FORCE_STREAM if path == "stream" else chord.CHORD_FLAG_FORCE_TENSOR
    out = torch.full((16, 256), 1.0, dtype=torch.bfloat16, device="cuda")
    chord.chord_moe_forward(t["x"], t["ids"], t["w"], src.sorted_ids, src.expert_ids, src.ntp, bm_forward,
                            dst.w13, dst.w2, dst.I, dst.E, out, dst.workspace, flags)
    assert dst.check_status() == chord.CHORD_DEV_BLOCK_M_MISMATCH
    assert torch.count_nonzero(out.float()).item() == 0
    # the matching block_m on the same buffers still computes the layer
    got = run_layer(dst, tiny, flags)
    assert_layer_close(got, oracle_rows(tiny, None))


# ------------------------------------------------------------------------------ full size, other schedules

@pytest.mark.parametrize("name,block_m,flags", [
    ("tp8_prefill", 64, 0),     # tensor cores, an expert's ~85 rows in two 64-row blocks
    ("tp8_prefill", 96, 0),     # tensor cores, MMA N of a block not a power of two
    ("ep8_prefill", 64, 0),     # tensor cores, ~171 rows per expert in three blocks
    ("ep8_prefill", 96, 0),
    ("tp8_prefill", 128, "stream"),  # weight streaming at a prefill shape: 32-token chunks
    ("ep8_decode", 32, "tensor"),    # tensor cores at a decode shape
])
def test_full_size_other_block_m_and_forced_schedules(chord, big_inputs, name, block_m, flags):
    # the selector's own choice is covered by test_full_size_sampled_rows; these are the
    # block sizes and schedules a caller may pick at Kimi-K2 sizes
    d = big_inputs(name)
    cfg = d["cfg"]
    f = {0: 0, "stream": chord.CHORD_FLAG_FORCE_STREAM, "tensor": chord.CHORD_FLAG_FORCE_TENSOR}[flags]
    layer = make_layer(chord, d, block_m=block_m)
    got = run_layer(layer, d, f)
    rows = inputs.sample_rows(d["topk_ids"], cfg.E, 512, seed=1)
    assert_layer_close(got[rows], oracle_rows(d, rows))
    none = ~((d["topk_ids"] >= 0) & (d["topk_ids"] < cfg.E)).any(axis=1)
    assert np.all(bf16_bits_to_f64(got[none]) == 0)
