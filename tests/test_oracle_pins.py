"""Pins for the CPU oracle: it is checked here against things other than itself.

* closed forms and special cases of the layer's definition (all-equal codes, zero scale,
  a single expert reducing to a dense gated MLP, top-k weights summing to one);
* an independent brute force written here in numpy float64 (own unpacking, own
  round-to-nearest-even, no routing sort) on tiny inputs;
* invariants: exact doubling, token permutation, routing-tensor structure;
* an exhaustive check of the dequantisation over every code and every finite bf16 scale.

The layer's definition follows the Chord blog (Novita/vLLM, German edition): subtract
then scale in BF16 ("H200 und Blackwell indexierter Decode"), uint4 group-32 weights
with BF16 scales ("vLLM-Integration"), block-padded sorted routing with sentinels
("Zwei Kernel-Familien", Figure 3).
"""
import numpy as np
import pytest

import oracle
from w4a16_int4_mixture_align_b200 import inputs

TOL_MAX = 2e-2   # max |a - b| <= TOL_MAX * max |b|
TOL_MEAN = 5e-3  # sum |a - b| / sum |b| <= TOL_MEAN


def f32(bits):
    return oracle.bf16_to_f32(bits).astype(np.float64)


# ----------------------------------------------------------------------------------
# independent helpers (float64; no code shared with oracle.c)

def bf16_nearest_even(v: np.ndarray) -> np.ndarray:
    """Nearest bf16 value to each float64 in v (values exactly representable in binary32),
    ties to the even mantissa, overflow to +-inf: chosen between the two neighbours."""
    v = np.asarray(v, dtype=np.float64)
    with np.errstate(over="ignore", invalid="ignore"):
        return _bf16_nearest_even(v)


def _bf16_nearest_even(v):
    f = v.astype(np.float32)
    assert np.all((f.astype(np.float64) == v) | ~np.isfinite(f))
    bits = f.view(np.uint32)
    lo_bits = bits & np.uint32(0xFFFF0000)
    hi_bits = lo_bits + np.uint32(0x10000)
    lo = lo_bits.view(np.float32).astype(np.float64)
    hi_is_inf = (hi_bits & np.uint32(0x7FFFFFFF)) == np.uint32(0x7F800000)
    hi = np.where(hi_is_inf, np.copysign(2.0 ** 128, v), hi_bits.view(np.float32).astype(np.float64))
    d_lo, d_hi = np.abs(v - lo), np.abs(hi - v)
    lo_even = ((lo_bits >> np.uint32(16)) & np.uint32(1)) == 0
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ~lo_even)
    out = np.where(take_hi, np.where(hi_is_inf, np.copysign(np.inf, v), hi), lo)
    return out


def unpack_codes(qw: np.ndarray) -> np.ndarray:
    """int32 [..., K/8] -> uint8 codes [..., K], code k%8 at bit 4*(k%8)."""
    w = qw.view(np.uint32)
    sh = (4 * np.arange(8, dtype=np.uint32))
    c = (w[..., None] >> sh) & np.uint32(0xF)
    return c.reshape(*qw.shape[:-1], qw.shape[-1] * 8).astype(np.int64)


def dequant_f64(qw, s, rounded: bool):
    q = unpack_codes(qw)
    sc = np.repeat(f32(s), 32, axis=-1)
    w = (q - 8).astype(np.float64) * sc
    return bf16_nearest_even(w) if rounded else w


def silu(g):
    return g / (1.0 + np.exp(-g))


def brute_force(d, rounded: bool):
    """Per-token loop, no routing sort, float64 accumulation."""
    x = f32(d["x"])
    ids, tw = d["topk_ids"], d["topk_weights"].astype(np.float64)
    E, N13, _ = d["qw13"].shape
    I = N13 // 2
    T, H = x.shape
    out = np.zeros((T, H))
    w13 = [dequant_f64(d["qw13"][e], d["s13"][e], rounded) for e in range(E)]
    w2 = [dequant_f64(d["qw2"][e], d["s2"][e], rounded) for e in range(E)]
    for t in range(T):
        for j in range(ids.shape[1]):
            e = ids[t, j]
            if not (0 <= e < E):
                continue
            h = w13[e] @ x[t]
            a = silu(h[:I]) * h[I:]
            if rounded:
                a = bf16_nearest_even(a.astype(np.float32).astype(np.float64))
            out[t] += tw[t, j] * (w2[e] @ a)
    return out


def run_oracle(d, rows=None):
    return oracle.moe_forward(d["x"], d["topk_ids"], d["topk_weights"], d["qw13"], d["s13"],
                              d["qw2"], d["s2"], rows=rows)


def assert_close(got_bits, ref, tol_max=TOL_MAX, tol_mean=TOL_MEAN):
    got = f32(got_bits)
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.abs(ref).max()
    assert scale > 0
    err = np.abs(got - ref)
    assert err.max() <= tol_max * scale, (err.max(), scale)
    assert err.sum() <= tol_mean * np.abs(ref).sum(), (err.sum(), np.abs(ref).sum())


# ----------------------------------------------------------------------------------
# bf16 rounding and dequantisation

def test_bf16_rounding_matches_nearest_even_on_random_binary32():
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 2 ** 32, size=20000, dtype=np.uint32)
    vals = bits.view(np.float32)
    vals = vals[np.isfinite(vals)]
    # include exact ties and overflow boundaries
    ties = (np.arange(0, 4000, dtype=np.uint32) << np.uint32(16)) | np.uint32(0x8000)
    extra = np.concatenate([ties.view(np.float32), np.float32([3.3961776e38, 3.3961775e38, -3.3961776e38, 0.0, -0.0])])
    vals = np.concatenate([vals, extra[np.isfinite(extra)]])
    got = f32(oracle.f32_to_bf16(vals))
    ref = bf16_nearest_even(vals.astype(np.float64))
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all(), vals[~same][:5]


def test_dequant_exhaustive_all_codes_all_finite_bf16_scales():
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = (pats & 0x7F80) != 0x7F80
    scales = pats[finite]
    n = scales.shape[0]
    words = np.array([0x76543210, 0xFEDCBA98, 0x76543210, 0xFEDCBA98], dtype=np.uint32)
    qw = np.tile(words.view(np.int32), (n, 1))
    s = scales.reshape(n, 1)
    got = oracle.dequant(qw, s).astype(np.float64)
    q = np.tile(np.concatenate([np.arange(16), np.arange(16)]), (n, 1))
    exact = (q - 8) * f32(s)
    ref = bf16_nearest_even(exact)
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()
    # signed zeros too: (q-8)*s == 0 only for q == 8
    assert np.all(np.signbit(got[:, 8]) == np.signbit(f32(s)[:, 0] * 0.0))


def test_nibble_order_low_nibble_first():
    # word 0x89ABCDEF holds codes F,E,D,C,B,A,9,8 for k = 0..7
    qw = np.array([[0x89ABCDEF, 0x01234567, 0, 0]], dtype=np.uint32).view(np.int32)
    one = np.array([[0x3F80]], dtype=np.uint16)  # bf16 1.0
    w = oracle.dequant(qw, one)[0]
    expect = [15 - k for k in range(8)] + [7 - k for k in range(8)] + [0] * 16
    assert list(w.astype(int)) == [c - 8 for c in expect]


def test_group_index_is_k_over_32():
    rng = np.random.default_rng(3)
    qw = rng.integers(0, 2 ** 32, size=(4, 16), dtype=np.uint32).view(np.int32)  # K = 128
    s = inputs._f32_to_bf16_bits_trunc(rng.uniform(0.5, 2.0, size=(4, 4)).astype(np.float32))
    got = oracle.dequant(qw, s).astype(np.float64)
    assert np.array_equal(got, dequant_f64(qw, s, rounded=True))


# ----------------------------------------------------------------------------------
# routing sort

def brute_align(ids, E, BM):
    T, k = ids.shape
    n = T * k
    flat = ids.reshape(-1)
    cap = n + E * (BM - 1)
    sorted_ids = [n] * cap
    expert_ids = [-1] * ((cap + BM - 1) // BM)
    pos = 0
    for e in range(E):
        mine = [f for f in range(n) if flat[f] == e]
        start = pos
        for r, f in enumerate(mine):
            sorted_ids[start + r] = f
        blocks = -(-len(mine) // BM)
        for b in range(blocks):
            expert_ids[start // BM + b] = e
        pos += blocks * BM
    return np.array(sorted_ids, np.int32), np.array(expert_ids, np.int32), pos


@pytest.mark.parametrize("T,k,E,BM,seed", [
    (16, 2, 8, 16, 0), (37, 8, 48, 8, 1), (5, 3, 4, 1, 2), (64, 8, 1, 16, 3),
    (0, 8, 48, 16, 4), (100, 8, 384, 64, 5), (33, 4, 6, 256, 6), (7, 1, 3, 5, 7),
])
def test_align_matches_brute_force(T, k, E, BM, seed):
    rng = np.random.default_rng(seed)
    ids = rng.integers(-1, E + 3, size=(T, k)).astype(np.int32)  # -1 and ids >= E are not local
    s, eids, ntp, offs = oracle.moe_align(ids, E, BM)
    bs, beids, bntp = brute_align(ids, E, BM)
    assert ntp == bntp
    assert np.array_equal(s, bs)
    assert np.array_equal(eids, beids)
    assert offs[-1] == ntp and np.all(np.diff(offs) % BM == 0)


def test_align_invariants_on_generated_routing():
    cfg = inputs.CONFIGS["ep8_decode"]
    ids, _ = inputs.make_routing(cfg)
    BM = 8
    s, eids, ntp, offs = oracle.moe_align(ids, cfg.E, BM)
    n = ids.size
    flat = ids.reshape(-1)
    local = np.nonzero((flat >= 0) & (flat < cfg.E))[0]
    real = s[s < n]
    assert sorted(real.tolist()) == local.tolist()           # a permutation of local slots
    assert ntp % BM == 0 and np.all(s[ntp:] == n)
    for b in range(ntp // BM):                                 # one expert per block
        blk = s[b * BM:(b + 1) * BM]
        blk = blk[blk < n]
        assert blk.size > 0 and np.all(flat[blk] == eids[b])
        assert np.all(np.diff(blk) > 0)                        # increasing flat index
    assert np.all(eids[ntp // BM:] == -1)


def test_align_single_expert_block_one():
    ids = np.array([[0, -1], [0, 0], [-1, 0]], dtype=np.int32)
    s, eids, ntp, _ = oracle.moe_align(ids, 1, 1)
    assert ntp == 4 and list(s[:4]) == [0, 2, 3, 5] and list(eids[:4]) == [0, 0, 0, 0]


# ----------------------------------------------------------------------------------
# the layer

def tiny_inputs(seed=0, **over):
    cfg = inputs.MoEConfig("t", over.get("T", 16), over.get("H", 256), over.get("I", 128),
                           over.get("E", 8), over.get("E_global", over.get("E", 8)),
                           over.get("topk", 2), over.get("routing", "normal"), seed)
    return inputs.make_inputs(cfg)


def test_forward_matches_brute_force_with_same_roundings():
    d = tiny_inputs()
    got = f32(run_oracle(d))
    ref = brute_force(d, rounded=True)
    # only fp32-vs-fp64 accumulation and the final bf16 rounding differ
    assert np.abs(got - ref).max() <= 8e-3 * np.abs(ref).max()


def test_forward_matches_exact_brute_force_within_layer_tolerance():
    d = tiny_inputs(seed=1, T=24, E=6, topk=3)
    assert_close(run_oracle(d), brute_force(d, rounded=False))


def test_forward_ep_shard_with_nonlocal_slots():
    d = tiny_inputs(seed=2, T=20, E=4, E_global=12, topk=3)
    assert (d["topk_ids"] == -1).any()
    got = run_oracle(d)
    ref = brute_force(d, rounded=True)
    no_local = ~((d["topk_ids"] >= 0).any(axis=1))
    assert np.all(f32(got)[no_local] == 0)
    assert np.abs(f32(got) - ref).max() <= 8e-3 * np.abs(ref).max()


def test_ep_shards_add_up_to_the_unsharded_layer():
    """Expert parallelism splits the experts over shards and each shard keeps the global
    top-k weights (not renormalised over its local experts), so the shard outputs add up
    to the unsharded layer, up to one bf16 rounding per shard. Renormalising the weights
    per shard, or dropping slots that carry another shard's global id, would break this."""
    E_all, shards, topk = 12, 3, 3
    d = tiny_inputs(seed=7, T=24, E=E_all, topk=topk)
    full = f32(run_oracle(d))
    per = E_all // shards
    total = np.zeros_like(full)
    for r in range(shards):
        lo = r * per
        ids = d["topk_ids"].copy()
        local = (ids >= lo) & (ids < lo + per)
        # local slots renumbered to this shard's experts; the others keep a global id
        # at or past the shard's E, which marks a slot of another shard
        ids = np.where(local, ids - lo, ids + per)
        shard = dict(d, topk_ids=ids.astype(np.int32),
                     qw13=np.ascontiguousarray(d["qw13"][lo:lo + per]), s13=np.ascontiguousarray(d["s13"][lo:lo + per]),
                     qw2=np.ascontiguousarray(d["qw2"][lo:lo + per]), s2=np.ascontiguousarray(d["s2"][lo:lo + per]))
        total += f32(run_oracle(shard))
    assert np.abs(total - full).max() <= 4 * 2.0 ** -8 * np.abs(full).max()
    # renormalising the weights over each shard's local slots does not add up
    wrong = np.zeros_like(full)
    for r in range(shards):
        lo = r * per
        local = (d["topk_ids"] >= lo) & (d["topk_ids"] < lo + per)
        w = np.where(local, d["topk_weights"], 0.0)
        w = (w / np.maximum(w.sum(axis=1, keepdims=True), 1e-30)).astype(np.float32)
        ids = np.where(local, d["topk_ids"] - lo, -1).astype(np.int32)
        shard = dict(d, topk_ids=ids, topk_weights=w,
                     qw13=np.ascontiguousarray(d["qw13"][lo:lo + per]), s13=np.ascontiguousarray(d["s13"][lo:lo + per]),
                     qw2=np.ascontiguousarray(d["qw2"][lo:lo + per]), s2=np.ascontiguousarray(d["s2"][lo:lo + per]))
        wrong += f32(run_oracle(shard))
    assert np.abs(wrong - full).max() > 0.1 * np.abs(full).max()


def test_subset_rows_equal_full_rows():
    d = tiny_inputs(seed=3)
    full = run_oracle(d)
    rows = np.array([1, 5, 6, 15])
    assert np.array_equal(run_oracle(d, rows=rows), full[rows])


def test_single_expert_is_dense_gated_mlp():
    d = tiny_inputs(seed=4, E=1, topk=1)
    d["topk_ids"][:] = 0
    d["topk_weights"][:] = 1.0
    w13 = oracle.dequant(d["qw13"][0], d["s13"][0]).astype(np.float64)
    w2 = oracle.dequant(d["qw2"][0], d["s2"][0]).astype(np.float64)
    x = f32(d["x"])
    h = x @ w13.T
    I = w2.shape[1]
    dense = (silu(h[:, :I]) * h[:, I:]) @ w2.T
    assert_close(run_oracle(d), dense)


def test_all_equal_codes_closed_form():
    d = tiny_inputs(seed=5)
    c, s_bits = 11, np.uint16(0x3C23)  # code 11, scale ~0.00995
    word = np.uint32(sum(c << (4 * i) for i in range(8)))
    for k in ("qw13", "qw2"):
        d[k][:] = np.array(word).view(np.int32)
    for k in ("s13", "s2"):
        d[k][:] = s_bits
    w0 = bf16_nearest_even(np.array([(c - 8) * float(f32(s_bits))]))[0]
    x = f32(d["x"])
    I = d["qw2"].shape[2] * 8
    h = w0 * x.sum(axis=1)                       # every gate and up row equals this
    a = bf16_nearest_even((silu(h) * h).astype(np.float32).astype(np.float64))
    y = w0 * I * a                               # every output column
    ref = np.zeros_like(x)
    for t in range(x.shape[0]):
        for j in range(d["topk_ids"].shape[1]):
            if d["topk_ids"][t, j] >= 0:
                ref[t] += d["topk_weights"][t, j] * y[t]
    assert_close(run_oracle(d), ref, tol_max=1e-2, tol_mean=2e-3)


def test_code_eight_gives_exact_zero():
    d = tiny_inputs(seed=6)
    d["qw13"][:] = np.array(np.uint32(0x88888888)).view(np.int32)
    assert np.all(f32(run_oracle(d)) == 0)


def test_zero_scale_gives_exact_zero():
    d = tiny_inputs(seed=7)
    d["s2"][:] = 0
    assert np.all(f32(run_oracle(d)) == 0)


def test_weights_summing_to_one_over_identical_experts_is_dense_mlp():
    d = tiny_inputs(seed=8, topk=4)
    for k in ("qw13", "s13", "qw2", "s2"):
        d[k][:] = d[k][0:1]
    w13 = oracle.dequant(d["qw13"][0], d["s13"][0]).astype(np.float64)
    w2 = oracle.dequant(d["qw2"][0], d["s2"][0]).astype(np.float64)
    x = f32(d["x"])
    h = x @ w13.T
    I = w2.shape[1]
    dense = (silu(h[:, :I]) * h[:, I:]) @ w2.T
    assert np.allclose(d["topk_weights"].sum(axis=1), 1.0, atol=1e-6)
    assert_close(run_oracle(d), dense)


def test_doubling_down_scales_doubles_output_exactly():
    d = tiny_inputs(seed=9)
    base = f32(run_oracle(d))
    d["s2"] = (d["s2"].astype(np.uint32) + 0x80).astype(np.uint16)  # exponent + 1
    assert np.array_equal(f32(run_oracle(d)), 2 * base)


def test_doubling_topk_weights_doubles_output_exactly():
    d = tiny_inputs(seed=10)
    base = f32(run_oracle(d))
    d["topk_weights"] = d["topk_weights"] * np.float32(2)
    assert np.array_equal(f32(run_oracle(d)), 2 * base)


def test_token_permutation_permutes_rows_bit_exactly():
    d = tiny_inputs(seed=11)
    base = run_oracle(d)
    perm = np.random.default_rng(0).permutation(d["x"].shape[0])
    for k in ("x", "topk_ids", "topk_weights"):
        d[k] = np.ascontiguousarray(d[k][perm])
    assert np.array_equal(run_oracle(d), base[perm])


def test_swapped_gate_and_up_would_be_caught():
    """A plausible mistake (gate and up halves swapped) fails the brute-force pin."""
    d = tiny_inputs(seed=12)
    ref = brute_force(d, rounded=True)
    I = d["qw13"].shape[1] // 2
    for k in ("qw13", "s13"):
        d[k] = np.ascontiguousarray(np.concatenate([d[k][:, I:], d[k][:, :I]], axis=1))
    wrong = f32(run_oracle(d))
    assert np.abs(wrong - ref).max() > 0.1 * np.abs(ref).max()


def load_golden():
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_oracle.txt")
    g = {"out": []}
    with open(path) as fh:
        for line in fh:
            if line.startswith("#"):
                continue
            key, *vals = line.split()
            if key == "out":
                g["out"].append([int(v, 16) for v in vals[1:]])
            else:
                g[key] = [int(v) for v in vals]
    g["out"] = np.array(g["out"], dtype=np.uint16)
    return g


def test_oracle_reproduces_golden_fixture():
    g = load_golden()
    d = inputs.make_inputs(inputs.CONFIGS["tiny"])
    s, eids, ntp, offs = oracle.moe_align(d["topk_ids"], 8, 16)
    assert ntp == g["num_tokens_padded"][0]
    assert s.tolist() == g["sorted_ids"] and eids.tolist() == g["expert_ids"]
    assert offs.tolist() == g["expert_offsets"]
    assert np.array_equal(run_oracle(d), g["out"])


# ------------------------------------------------------------------------------ router

def _router_brute(logits, k):
    """Library routines only: a stable argsort of the negated logits (ties keep the lower
    expert id) and scipy's softmax over the chosen logits."""
    from scipy.special import softmax
    order = np.argsort(-logits.astype(np.float64), axis=1, kind="stable")[:, :k]
    chosen = np.take_along_axis(logits.astype(np.float64), order, axis=1)
    return order.astype(np.int32), softmax(chosen, axis=1)


@pytest.mark.parametrize("G,k", [(384, 8), (100, 3), (64, 64), (7, 1)])
def test_router_matches_sort_and_softmax(G, k):
    rng = np.random.default_rng(11 + G + k)
    logits = rng.standard_normal((257, G)).astype(np.float32)
    # coarse values in some rows create ties, which must go to the lower id
    logits[::5] = np.round(logits[::5] * 2) / 2
    ids, w = oracle.router_topk(logits, k)
    ref_ids, ref_w = _router_brute(logits, k)
    np.testing.assert_array_equal(ids, ref_ids)
    np.testing.assert_allclose(w, ref_w, rtol=2e-7, atol=0)


def test_router_closed_forms():
    # all logits equal: the k lowest ids, weight exactly 1/k each
    ids, w = oracle.router_topk(np.full((3, 40), 0.25, np.float32), 5)
    assert np.all(ids == np.arange(5)) and np.all(w == np.float32(1 / 5))
    # k = number of experts: the full softmax, experts by descending logit
    lg = np.array([[0.0, 1.0, -2.0, 3.0]], np.float32)
    ids, w = oracle.router_topk(lg, 4)
    e = np.exp(lg[0].astype(np.float64))
    np.testing.assert_array_equal(ids[0], [3, 1, 0, 2])
    np.testing.assert_allclose(w[0], (e / e.sum())[[3, 1, 0, 2]], rtol=2e-7)
    # adding a constant to every logit (exactly, here) changes nothing
    rng = np.random.default_rng(5)
    base = (rng.integers(-64, 64, (50, 96)) / 8).astype(np.float32)
    i0, w0 = oracle.router_topk(base, 8)
    i1, w1 = oracle.router_topk(base + np.float32(4.0), 8)
    np.testing.assert_array_equal(i0, i1)
    np.testing.assert_allclose(w0, w1, rtol=2e-7)
    # weights of a row sum to one
    np.testing.assert_allclose(w0.astype(np.float64).sum(axis=1), 1.0, rtol=1e-6)


# ------------------------------------------------------------------------------ grouped GEMM

SENTINEL = np.uint16(0x7FC1)  # a NaN pattern no computed bf16 value takes


def gcfg(mode, E, N, K, rows, max_m=0, balance="random", seed=0):
    return inputs.GroupedConfig("t", mode, E, N, K, rows, max_m, balance, seed)


def grouped_rows_expert(d):
    """The expert of each flat row of x, or -1 (read off the layout's definition)."""
    cfg = d["cfg"]
    if cfg.mode == "contiguous":
        return d["m_indices"].astype(np.int64)
    r = np.arange(cfg.E * cfg.max_m)
    e = r // cfg.max_m
    return np.where(r % cfg.max_m < d["masked_m"][e], e, -1)


def grouped_brute(d):
    """Float64, weights rounded to bf16 as the method does; NaN where no expert."""
    cfg = d["cfg"]
    x = f32(d["x"]).reshape(-1, cfg.K)
    ex = grouped_rows_expert(d)
    ref = np.full((x.shape[0], cfg.N), np.nan)
    absum = np.full_like(ref, np.nan)  # sum_k |x_k w_k|, for the rounding bound
    for e in np.unique(ex[ex >= 0]):
        w = dequant_f64(d["qweight"][e], d["scales"][e], rounded=True)
        rows = ex == e
        ref[rows] = x[rows] @ w.T
        absum[rows] = np.abs(x[rows]) @ np.abs(w).T
    return ref, absum


def run_grouped_oracle(d):
    cfg = d["cfg"]
    M = d["x"].size // cfg.K
    out = np.full((M, cfg.N), SENTINEL, np.uint16)
    if cfg.mode == "contiguous":
        return oracle.grouped_gemm(d["x"], d["qweight"], d["scales"], m_indices=d["m_indices"], out=out)
    return oracle.grouped_gemm(d["x"], d["qweight"], d["scales"], masked_m=d["masked_m"], out=out)


def assert_fp32_then_bf16(got_bits, ref, absum, K):
    """A sequential FP32 sum of exact products is within (K-1) 2^-24 sum|x w| of the exact
    sum; one bf16 rounding adds at most 2^-8 of the value."""
    got = f32(got_bits)
    acc = 1.01 * (K - 1) * 2.0 ** -24 * absum
    bound = 2.0 ** -8 * (np.abs(ref) + acc) + acc
    err = np.abs(got - ref)
    assert np.all(err <= bound), (err.max(), np.argmax(err - bound))


@pytest.mark.parametrize("mode,E,N,K,rows,max_m,seed", [
    ("contiguous", 5, 256, 512, 50, 0, 1),
    ("contiguous", 3, 384, 256, 200, 0, 2),
    ("masked", 4, 256, 512, 40, 64, 3),
    ("masked", 6, 128, 384, 10, 24, 4),
])
def test_grouped_matches_brute_force(mode, E, N, K, rows, max_m, seed):
    d = inputs.make_grouped(gcfg(mode, E, N, K, rows, max_m, seed=seed))
    got = run_grouped_oracle(d)
    ref, absum = grouped_brute(d)
    valid = grouped_rows_expert(d) >= 0
    assert valid.any() and (~valid).any()
    assert_fp32_then_bf16(got[valid], ref[valid], absum[valid], K)
    assert np.all(got[~valid] == SENTINEL)  # rows without an expert are not written


def test_grouped_masked_equals_contiguous_layout():
    # the same valid rows in the two layouts give bit-identical results
    d = inputs.make_grouped(gcfg("masked", 5, 256, 256, 30, 48, seed=5))
    cfg = d["cfg"]
    xm = d["x"].reshape(cfg.E, cfg.max_m, cfg.K)
    got_m = run_grouped_oracle(d).reshape(cfg.E, cfg.max_m, cfg.N)
    xs, ids = [], []
    for e in range(cfg.E):
        c = int(d["masked_m"][e])
        pad = (c + 127) // 128 * 128 - c
        xs += [xm[e, :c], np.zeros((pad, cfg.K), np.uint16)]
        ids += [np.full(c, e, np.int32), np.full(pad, -1, np.int32)]
    dc = {"cfg": gcfg("contiguous", cfg.E, cfg.N, cfg.K, 0), "x": np.concatenate(xs), "m_indices": np.concatenate(ids),
          "qweight": d["qweight"], "scales": d["scales"]}
    got_c = run_grouped_oracle(dc)
    at = 0
    for e in range(cfg.E):
        c = int(d["masked_m"][e])
        assert np.array_equal(got_c[at:at + c], got_m[e, :c])
        at += (c + 127) // 128 * 128


def test_grouped_relabelled_experts_give_identical_rows():
    d = inputs.make_grouped(gcfg("contiguous", 6, 128, 256, 40, seed=6))
    base = run_grouped_oracle(d)
    perm = np.array([3, 5, 0, 1, 4, 2])  # expert e's weights move to slot perm[e]
    qw, sc = np.empty_like(d["qweight"]), np.empty_like(d["scales"])
    qw[perm], sc[perm] = d["qweight"], d["scales"]
    mi = np.where(d["m_indices"] >= 0, perm[np.maximum(d["m_indices"], 0)], -1).astype(np.int32)
    d2 = dict(d, qweight=qw, scales=sc, m_indices=mi)
    assert np.array_equal(run_grouped_oracle(d2), base)


def test_grouped_single_expert_is_dense_gemm():
    d = inputs.make_grouped(gcfg("contiguous", 1, 256, 384, 128, balance="balanced", seed=7))
    assert np.all(d["m_indices"] == 0)
    w = oracle.dequant(d["qweight"][0], d["scales"][0]).astype(np.float64)
    x = f32(d["x"])
    ref = x @ w.T  # numpy's matmul over the oracle's own (separately pinned) dequantisation
    assert_fp32_then_bf16(run_grouped_oracle(d), ref, np.abs(x) @ np.abs(w).T, 384)


def test_grouped_all_equal_codes_closed_form():
    d = inputs.make_grouped(gcfg("masked", 3, 128, 256, 20, 32, seed=8))
    c, s_bits = 3, np.uint16(0x3CA0)  # code 3, scale 0.01953125 (exact)
    word = np.uint32(sum(c << (4 * i) for i in range(8)))
    d["qweight"][:] = np.array(word).view(np.int32)
    d["scales"][:] = s_bits
    w0 = (c - 8) * float(f32(s_bits))  # -0.09765625, a bf16 value: rounding keeps it
    x = f32(d["x"]).reshape(-1, 256)
    got = run_grouped_oracle(d)
    valid = grouped_rows_expert(d) >= 0
    ref = np.repeat((w0 * x.sum(axis=1))[:, None], 128, axis=1)  # every column the same
    absum = np.repeat((abs(w0) * np.abs(x).sum(axis=1))[:, None], 128, axis=1)
    assert_fp32_then_bf16(got[valid], ref[valid], absum[valid], 256)
    assert np.all(got[valid] == got[valid][:, :1])


def test_grouped_out_of_range_rows_are_skipped():
    d = inputs.make_grouped(gcfg("contiguous", 4, 128, 128, 30, seed=9))
    d["m_indices"][:7] = 4   # not an expert of this weight
    d["m_indices"][7:9] = -3  # any negative id is padding
    got = run_grouped_oracle(d)
    assert np.all(got[:9] == SENTINEL)
    assert not np.any(got[9:][d["m_indices"][9:] >= 0] == SENTINEL)
