"""Grouped operators on the GPU (chord_grouped_contiguous / chord_grouped_masked) vs the
oracle's grouped GEMM.

Small cases compare every output element, including rows that must stay unwritten
(padding rows, rows past masked_m), on both schedules and both unit sizes (128 and 256
rows). The EP8 shapes the benchmark times are checked on a seeded sample of rows, in the
benchmark's launch configuration. Edge cases: empty experts, masked_m of 0, 1 and
max_m, max_m not a multiple of 128, a block mixing experts, masked_m out of range, a
weight prepared for the other mode, zero rows.

Tolerance, from the arithmetic: both sides sum exact bf16 x bf16 products in FP32 (in
different orders) and round once to bf16, so each is within acc + 2^-8 (|exact| + acc)
of the exact sum, acc = c K 2^-24 sum_k |x_k w_k| (c = 1 for the oracle's sequential
sum, 2 for the tensor-core accumulation); the check allows the sum of the two.
"""
import numpy as np
import pytest

import oracle
from helpers import assert_layer_close, bf16_bits_to_f64, ensure_built
from w4a16_int4_mixture_align_b200 import inputs

pytestmark = pytest.mark.gpu

SENTINEL = np.uint16(0x7FC1)


@pytest.fixture(scope="module")
def chord():
    ensure_built()
    from w4a16_int4_mixture_align_b200 import chord as c
    return c


def gcfg(mode, E, N, K, rows, max_m=0, balance="random", seed=0):
    return inputs.GroupedConfig("t", mode, E, N, K, rows, max_m, balance, seed)


def rows_expert(d):
    cfg = d["cfg"]
    if cfg.mode == "contiguous":
        return d["m_indices"].astype(np.int64)
    r = np.arange(cfg.E * cfg.max_m)
    e = r // cfg.max_m
    return np.where(r % cfg.max_m < np.clip(d["masked_m"][e], 0, cfg.max_m), e, -1)


def bf16_dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def prepare(chord, d):
    cfg = d["cfg"]
    return chord.pack_w4a16_grouped(d["qweight"], d["scales"].view(np.int16), cfg.mode)


def run_gpu(chord, d, w, flags=0, expected=None, x2d=False, check=True):
    import torch
    cfg = d["cfg"]
    x = bf16_dev(d["x"])
    M = d["x"].size // cfg.K
    out = torch.full((M, cfg.N), int(SENTINEL.view(np.int16)), dtype=torch.int16, device="cuda").view(torch.bfloat16)
    if cfg.mode == "contiguous":
        chord.contiguous(x, w, torch.from_numpy(d["m_indices"]).cuda(), out=out, flags=flags)
    else:
        if x2d:
            x = x.view(-1, cfg.K)
        chord.masked(x, w, torch.from_numpy(d["masked_m"]).cuda(), expected or max(cfg.rows, 1), out=out,
                     flags=flags)
    torch.cuda.synchronize()
    st = w.check_status()
    if check:
        assert st == 0, hex(st)
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    return (got, st) if not check else got


def oracle_full(d):
    cfg = d["cfg"]
    M = d["x"].size // cfg.K
    out = np.full((M, cfg.N), SENTINEL, np.uint16)
    if cfg.mode == "contiguous":
        return oracle.grouped_gemm(d["x"], d["qweight"], d["scales"], m_indices=d["m_indices"], out=out)
    return oracle.grouped_gemm(d["x"], d["qweight"], d["scales"], masked_m=d["masked_m"], out=out)


def abs_products(d, rows, ex):
    """sum_k |x[m,k] w[e_m][n,k]| for the given flat rows (float32 is ample for a bound)."""
    cfg = d["cfg"]
    x = np.abs(bf16_bits_to_f64(d["x"].reshape(-1, cfg.K)[rows]).astype(np.float32))
    A = np.zeros((len(rows), cfg.N), np.float32)
    for e in np.unique(ex):
        w = np.abs(oracle.dequant(d["qweight"][e], d["scales"][e]))
        sel = ex == e
        A[sel] = x[sel] @ w.T
    return A.astype(np.float64)


def assert_grouped_close(got_bits, ref_bits, A, K):
    got, ref = bf16_bits_to_f64(got_bits), bf16_bits_to_f64(ref_bits)
    acc_o, acc_g = 1.01 * K * 2.0 ** -24 * A, 2.02 * K * 2.0 ** -24 * A
    # |exact| <= 1.004 (|ref| + 1.004 acc_o), so the two roundings add at most this much
    bound = 1.01 * (acc_o + acc_g) + 1.01 * 2.0 ** -7 * (np.abs(ref) + acc_o)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), "non-finite output"
    bad = err > bound
    assert not bad.any(), (int(bad.sum()), float(err.max()), float(err[bad].max()))
    assert_layer_close(got_bits, ref_bits)


def check_full(chord, d, flags=0, expected=None, x2d=False):
    w = prepare(chord, d)
    got = run_gpu(chord, d, w, flags, expected, x2d)
    ref = oracle_full(d)
    ex = rows_expert(d)
    valid = ex >= 0
    assert np.all(got[~valid] == SENTINEL), "a row without an expert was written"
    rows = np.nonzero(valid)[0]
    assert_grouped_close(got[rows], ref[rows], abs_products(d, rows, ex[rows]), d["cfg"].K)


PATHS = ["default", "stream", "tensor"]


def path_flags(chord, path):
    return {"default": 0, "stream": chord.CHORD_FLAG_FORCE_STREAM, "tensor": chord.CHORD_FLAG_FORCE_TENSOR}[path]


# ------------------------------------------------------------------------------ contiguous

@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("E,N,K,rows,seed", [
    (5, 256, 512, 50, 1),     # mostly partial 128-row blocks, some empty experts
    (3, 384, 256, 200, 2),    # runs of 0..400 rows: 256-row units, split blocks
    (8, 128, 1024, 9, 3),     # few rows per expert: 16-row MMAs on the tensor path
])
def test_contiguous_full_output(chord, path, E, N, K, rows, seed):
    check_full(chord, inputs.make_grouped(gcfg("contiguous", E, N, K, rows, seed=seed)), path_flags(chord, path))


def test_contiguous_single_expert_many_blocks(chord):
    d = inputs.make_grouped(gcfg("contiguous", 1, 256, 256, 700, balance="balanced", seed=4))
    check_full(chord, d)


@pytest.mark.parametrize("path", PATHS)
def test_contiguous_few_experts_small_units(chord, path):
    # 64 experts, three of them with rows: M / E = 6 selects 8-row units on the stream path
    d = inputs.make_grouped(gcfg("contiguous", 64, 256, 512, 10, seed=16))
    counts = np.zeros(64, np.int64)
    counts[[3, 40, 41]] = [20, 150, 1]
    runs = [np.concatenate([np.full(c, e, np.int32), np.full((c + 127) // 128 * 128 - c, -1, np.int32)])
            for e, c in enumerate(counts) if c]
    d["m_indices"] = np.concatenate(runs)
    rng = np.random.default_rng(16)
    d["x"] = (rng.standard_normal((d["m_indices"].size, 512), dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)
    check_full(chord, d, path_flags(chord, path))


def test_contiguous_mixed_block_is_flagged_and_skipped(chord):
    d = inputs.make_grouped(gcfg("contiguous", 4, 128, 256, 128, balance="balanced", seed=5))
    d["m_indices"][130] = 2  # block 1 (expert 1) now also names expert 2
    w = prepare(chord, d)
    got, st = run_gpu(chord, d, w, check=False)
    assert st & chord.CHORD_DEV_ROUTING_INVALID
    assert np.all(got[128:256] == SENTINEL)
    ref = oracle_full(d)
    keep = np.r_[0:128, 256:512]
    ex = d["m_indices"][keep].astype(np.int64)
    assert_grouped_close(got[keep], ref[keep], abs_products(d, keep, ex), 256)


def test_contiguous_zero_rows(chord):
    import torch
    d = inputs.make_grouped(gcfg("contiguous", 2, 128, 128, 10, seed=6))
    w = prepare(chord, d)
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    out = chord.contiguous(x, w, torch.empty(0, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert out.shape == (0, 128) and w.check_status() == 0


# ------------------------------------------------------------------------------ masked

@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("E,N,K,rows,max_m,seed", [
    (4, 256, 512, 40, 64, 7),      # budget 64: one 128-row unit per expert
    (3, 256, 256, 150, 200, 8),    # max_m not a multiple of 128, 256-row units
    (6, 128, 768, 5, 24, 9),       # tiny counts
])
def test_masked_full_output(chord, path, E, N, K, rows, max_m, seed):
    check_full(chord, inputs.make_grouped(gcfg("masked", E, N, K, rows, max_m, seed=seed)), path_flags(chord, path))


@pytest.mark.parametrize("path", PATHS)
def test_masked_edge_counts(chord, path):
    d = inputs.make_grouped(gcfg("masked", 5, 128, 256, 64, 130, seed=10))
    d["masked_m"][:] = [0, 1, 130, 128, 129]
    check_full(chord, d, path_flags(chord, path), expected=64)


def test_masked_flat_input(chord):
    check_full(chord, inputs.make_grouped(gcfg("masked", 3, 128, 256, 30, 40, seed=11)), x2d=True)


def test_masked_expected_m_changes_no_result(chord):
    d = inputs.make_grouped(gcfg("masked", 4, 256, 256, 60, 128, seed=12))
    w = prepare(chord, d)
    a = run_gpu(chord, d, w, expected=8)
    b = run_gpu(chord, d, w, expected=8)
    assert np.array_equal(a, b)  # deterministic
    ex = rows_expert(d)
    rows = np.nonzero(ex >= 0)[0]
    for e_m in (8, 16, 32, 64, 256):  # 8-, 16-, 32-row stream units; 128-, 256-row tensor units
        c = run_gpu(chord, d, w, expected=e_m)
        assert np.all(c[ex < 0] == SENTINEL)
        assert_grouped_close(c[rows], oracle_full(d)[rows], abs_products(d, rows, ex[rows]), 256)


def test_masked_out_of_range_counts_are_clamped_and_flagged(chord):
    d = inputs.make_grouped(gcfg("masked", 3, 128, 128, 20, 32, seed=13))
    d["masked_m"][:] = [-4, 40, 7]
    w = prepare(chord, d)
    got, st = run_gpu(chord, d, w, check=False)
    assert st & chord.CHORD_DEV_ROUTING_INVALID
    d["masked_m"][:] = [0, 32, 7]  # what the clamp means
    ref = oracle_full(d)
    ex = rows_expert(d)
    assert np.all(got[ex < 0] == SENTINEL)
    rows = np.nonzero(ex >= 0)[0]
    assert_grouped_close(got[rows], ref[rows], abs_products(d, rows, ex[rows]), 128)


# ------------------------------------------------------------------------------ contract

def test_weight_of_the_other_mode_fails_loudly(chord):
    import torch
    d = inputs.make_grouped(gcfg("masked", 2, 128, 128, 8, 16, seed=14))
    w = chord.pack_w4a16_grouped(d["qweight"], d["scales"].view(np.int16), "contiguous")
    with pytest.raises(chord.ChordError) as ei:
        chord.masked(bf16_dev(d["x"]), w, torch.from_numpy(d["masked_m"]).cuda(), 8)
    assert ei.value.status == chord.CHORD_ERR_LAYOUT_MISMATCH


def test_bad_shapes_are_rejected(chord):
    import torch
    d = inputs.make_grouped(gcfg("contiguous", 2, 128, 128, 8, seed=15))
    w = prepare(chord, d)
    x = torch.zeros((128, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((128, 128), dtype=torch.bfloat16, device="cuda")
    mi = torch.zeros(128, dtype=torch.int32, device="cuda")
    ws = w._workspace(128)
    with pytest.raises(chord.ChordError):  # N not a multiple of 128
        chord.chord_grouped_contiguous(x, mi, w.blob, 2, 100, out, ws)
    with pytest.raises(chord.ChordError):  # workspace too small
        chord.chord_grouped_contiguous(x, mi, w.blob, 2, 128, out, ws[:256])
    with pytest.raises(chord.ChordError):  # both schedules forced
        chord.chord_grouped_contiguous(x, mi, w.blob, 2, 128, out, ws,
                                       chord.CHORD_FLAG_FORCE_STREAM | chord.CHORD_FLAG_FORCE_TENSOR)


# ------------------------------------------------------------------------------ EP8 shapes

@pytest.mark.parametrize("name", sorted(inputs.GROUPED_CONFIGS))
def test_ep8_shapes_sampled_rows(chord, name):
    """The benchmark's workloads and launch configuration; 2 seeded rows per expert."""
    d = inputs.make_grouped(inputs.GROUPED_CONFIGS[name])
    cfg = d["cfg"]
    w = prepare(chord, d)
    got = run_gpu(chord, d, w)
    ex = rows_expert(d)
    assert np.all(got[ex < 0] == SENTINEL)
    rng = np.random.default_rng(1)
    rows = np.sort(np.concatenate([rng.choice(np.nonzero(ex == e)[0], 2, replace=False)
                                   for e in range(cfg.E) if (ex == e).sum() >= 2]))
    x_rows = d["x"].reshape(-1, cfg.K)[rows]
    ref = oracle.grouped_gemm(x_rows, d["qweight"], d["scales"], m_indices=ex[rows].astype(np.int32))
    assert_grouped_close(got[rows], ref, abs_products(d, rows, ex[rows]), cfg.K)
