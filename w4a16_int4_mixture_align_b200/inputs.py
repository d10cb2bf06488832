"""Seeded synthetic inputs for the W4A16 mixture-of-experts layer.

This module is shared by the tests, the benchmark and the oracle's callers. It holds
none of the layer's arithmetic: it draws random numbers, runs the router that sits
*upstream* of the layer (softmax top-k over router logits, which the pages exclude
from the layer; "Messungen" section of the Novita Chord blog), and stores random codes
and scales in the layer's input formats:

* activations ``x``: bf16 bit patterns ``uint16 [T, H]``, drawn N(0, 1) in fp32 and
  truncated to bf16 (the rounding used to *make* test data is irrelevant to the layer);
* ``topk_ids``: ``int32 [T, topk]``, the local expert id, or -1 when the routed expert
  lives on another shard; ``topk_weights``: ``float32 [T, topk]``, renormalised over
  all ``topk`` slots (global renormalisation, so they sum to <= 1 over local slots);
* packed int4 weights: ``int32 [E, N, K/8]``, eight uniform 4-bit codes per word with
  code ``k % 8`` in bits ``4*(k%8) .. 4*(k%8)+3`` (low nibble first);
* group scales: bf16 bit patterns ``uint16 [E, N, K/32]``, U[0.005, 0.02) truncated.

Shapes follow Kimi-K2 serving shards (hidden 7168, moe_intermediate 2048, 384 experts,
top-8), the workloads the Chord blog measures ("Messungen" table: EP8 prefill/decode,
TP8 single instance). Each part (routing, x, codes, scales) draws from its own child
stream of ``numpy.random.SeedSequence(seed)``, so any part can be regenerated alone.
"""
from __future__ import annotations

import dataclasses

import numpy as np

GROUP = 32  # K elements per scale group


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int  # tokens
    H: int  # hidden size (K of gate_up, N of down)
    I: int  # moe_intermediate size (gate_up N = 2*I, down K = I)
    E: int  # experts resident on this GPU (local ids 0..E-1)
    E_global: int  # experts the router chooses from
    topk: int
    routing: str  # 'normal' | 'uniform' | 'zipf'
    seed: int = 0

    def with_tokens(self, T: int) -> "MoEConfig":
        return dataclasses.replace(self, T=T)


CONFIGS = {
    # Tiny correctness MoE: 16 tokens, hidden 256, intermediate 128, 8 experts, top-2.
    "tiny": MoEConfig("tiny", 16, 256, 128, 8, 8, 2, "normal"),
    # Kimi-K2 EP8 decode shard: 128 tokens, local experts 0..47 of 384, top-8,
    # uniform router logits (distinct random top-8 per token).
    "ep8_decode": MoEConfig("ep8_decode", 128, 7168, 2048, 48, 384, 8, "uniform"),
    # Kimi-K2 EP8 prefill shard: 8192 tokens, N(0,1) router logits.
    "ep8_prefill": MoEConfig("ep8_prefill", 8192, 7168, 2048, 48, 384, 8, "normal"),
    # Kimi-K2 TP8 single instance: all 384 experts resident, intermediate sharded to 256.
    "tp8_decode": MoEConfig("tp8_decode", 32, 7168, 256, 384, 384, 8, "normal"),
    "tp8_prefill": MoEConfig("tp8_prefill", 4096, 7168, 256, 384, 384, 8, "normal"),
    # Skewed routing: Zipf(1.2) expert popularity over 384 experts, 48 local.
    "skew": MoEConfig("skew", 16384, 7168, 2048, 48, 384, 8, "zipf"),
}

ZIPF_S = 1.2
ZIPF_ZERO_LOCAL = 4  # local experts forced to popularity 0 in the skewed workload


def _streams(seed: int):
    routing, x, codes, scales = np.random.SeedSequence(seed).spawn(4)
    return (np.random.default_rng(routing), np.random.default_rng(x),
            np.random.default_rng(codes), np.random.default_rng(scales))


def _f32_to_bf16_bits_trunc(a: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(a, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _topk_desc(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest logits per row, largest first (ties: lower index first)."""
    idx = np.argsort(-logits, axis=1, kind="stable")[:, :k]
    return idx.astype(np.int64)


def zipf_popularity(cfg: MoEConfig) -> np.ndarray:
    """Per-global-expert popularity for the skewed workload (float64, sums to 1)."""
    rng = np.random.default_rng(np.random.SeedSequence([cfg.seed, 1]))
    ranks = np.arange(1, cfg.E_global + 1, dtype=np.float64)
    p_rank = ranks ** (-ZIPF_S)
    perm = rng.permutation(cfg.E_global)  # expert perm[r-1] gets rank r
    p = np.empty(cfg.E_global, dtype=np.float64)
    p[perm] = p_rank
    zero = rng.choice(cfg.E, size=min(ZIPF_ZERO_LOCAL, cfg.E), replace=False)
    p[zero] = 0.0
    return p / p.sum()


def make_routing(cfg: MoEConfig, global_ids: bool = False):
    """Router output: (topk_ids int32 [T,k] local ids or -1, topk_weights float32 [T,k]);
    with global_ids, the ids over all E_global experts (an expert-parallel rank's input
    to the dispatch)."""
    rng = _streams(cfg.seed)[0]
    T, G, k = cfg.T, cfg.E_global, cfg.topk
    if cfg.routing == "normal":
        logits = rng.standard_normal((T, G), dtype=np.float32).astype(np.float64)
    elif cfg.routing == "uniform":
        logits = rng.random((T, G), dtype=np.float32).astype(np.float64)
    elif cfg.routing == "zipf":
        p = zipf_popularity(cfg)
        with np.errstate(divide="ignore"):
            logp = np.log(p)
        logits = logp[None, :] + rng.gumbel(size=(T, G))
    else:
        raise ValueError(cfg.routing)
    sel = _topk_desc(logits, k)
    chosen = np.take_along_axis(logits, sel, axis=1)
    # softmax over all logits then renormalised over the top-k == softmax over the top-k
    z = np.exp(chosen - chosen.max(axis=1, keepdims=True))
    w = (z / z.sum(axis=1, keepdims=True)).astype(np.float32)
    ids = (sel if global_ids else np.where(sel < cfg.E, sel, -1)).astype(np.int32)
    return np.ascontiguousarray(ids), np.ascontiguousarray(w)


def make_hidden(cfg: MoEConfig) -> np.ndarray:
    rng = _streams(cfg.seed)[1]
    return _f32_to_bf16_bits_trunc(rng.standard_normal((cfg.T, cfg.H), dtype=np.float32))


def _codes(rng, E, N, K) -> np.ndarray:
    words = rng.integers(0, 2 ** 32, size=(E, N, K // 8), dtype=np.uint32)
    return words.view(np.int32)


def _scales(rng, E, N, K) -> np.ndarray:
    s = rng.uniform(0.005, 0.02, size=(E, N, K // GROUP)).astype(np.float32)
    return _f32_to_bf16_bits_trunc(s)


def make_weights(cfg: MoEConfig):
    """(qw13 int32 [E,2I,H/8], s13 u16 [E,2I,H/32], qw2 int32 [E,H,I/8], s2 u16 [E,H,I/32]).

    gate_up rows [0, I) are the gate projection and rows [I, 2I) the up projection.
    """
    _, _, rc, rs = _streams(cfg.seed)
    E, H, I = cfg.E, cfg.H, cfg.I
    qw13 = _codes(rc, E, 2 * I, H)
    qw2 = _codes(rc, E, H, I)
    s13 = _scales(rs, E, 2 * I, H)
    s2 = _scales(rs, E, H, I)
    return qw13, s13, qw2, s2


def make_inputs(cfg: MoEConfig, weights: bool = True) -> dict:
    ids, w = make_routing(cfg)
    d = {"cfg": cfg, "x": make_hidden(cfg), "topk_ids": ids, "topk_weights": w}
    if weights:
        d["qw13"], d["s13"], d["qw2"], d["s2"] = make_weights(cfg)
    return d


def sample_rows(topk_ids: np.ndarray, E: int, n: int = 512, seed: int = 1) -> np.ndarray:
    """``n`` token rows drawn uniformly (seeded) among tokens with at least one local slot,
    sorted ascending; all such rows when there are at most ``n``."""
    local = ((topk_ids >= 0) & (topk_ids < E)).any(axis=1)
    cand = np.nonzero(local)[0]
    if cand.size <= n:
        return cand.astype(np.int64)
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(cand, size=n, replace=False)).astype(np.int64)


# ----------------------------------------------------------------------------------
# Grouped operator layouts ("Gruppierte SM90-Kernel"): one projection [E, N, K] applied to
# rows already grouped by expert. Contiguous: each expert's rows consecutive, the run
# padded to a multiple of 128 rows, m_indices = expert id or -1 for padding. Masked: a
# fixed budget of max_m rows per expert, masked_m = valid rows. The blog measures both
# with the same rows per expert on each side ("Messungen": grouped rows matched per expert,
# EP8 prefill at 128 rows/expert, decode at 32 tokens/expert).

@dataclasses.dataclass(frozen=True)
class GroupedConfig:
    name: str
    mode: str      # 'contiguous' | 'masked'
    E: int         # experts
    N: int         # output columns (weight rows)
    K: int         # reduction length
    rows: int      # mean valid rows per expert (masked: also the expected_m hint)
    max_m: int     # masked row budget per expert (0 for contiguous)
    balance: str   # 'balanced': every expert has `rows`; 'random': uniform in [0, 2*rows]
    seed: int = 0


GROUPED_CONFIGS = {
    # EP8 shards of Kimi-K2 (48 local experts): gate_up [4096, 7168] and down [7168, 2048]
    "grouped_contiguous_ep8_gate_up": GroupedConfig("grouped_contiguous_ep8_gate_up", "contiguous", 48, 4096,
                                                    7168, 128, 0, "balanced"),
    "grouped_contiguous_ep8_down": GroupedConfig("grouped_contiguous_ep8_down", "contiguous", 48, 7168, 2048,
                                                 128, 0, "balanced"),
    "grouped_masked_ep8_gate_up": GroupedConfig("grouped_masked_ep8_gate_up", "masked", 48, 4096, 7168, 32, 256,
                                                "balanced"),
    "grouped_masked_ep8_down": GroupedConfig("grouped_masked_ep8_down", "masked", 48, 7168, 2048, 32, 256,
                                             "balanced"),
}


def grouped_counts(cfg: GroupedConfig) -> np.ndarray:
    """Valid rows per expert, int32 [E] (masked: at most max_m)."""
    if cfg.balance == "balanced":
        c = np.full(cfg.E, cfg.rows, dtype=np.int64)
    elif cfg.balance == "random":
        rng = _streams(cfg.seed)[0]
        c = rng.integers(0, 2 * cfg.rows + 1, size=cfg.E)
    else:
        raise ValueError(cfg.balance)
    if cfg.mode == "masked":
        c = np.minimum(c, cfg.max_m)
    return c.astype(np.int32)


def make_grouped(cfg: GroupedConfig, weights: bool = True) -> dict:
    """x (bf16 bits; [M, K] contiguous, [E, max_m, K] masked), m_indices int32 [M] or
    masked_m int32 [E], and qweight int32 [E, N, K/8] / scales bf16 bits [E, N, K/32].
    Padding rows and rows past masked_m hold random values like the rest."""
    counts = grouped_counts(cfg)
    _, rx, rc, rs = _streams(cfg.seed)
    d = {"cfg": cfg, "counts": counts}
    if cfg.mode == "contiguous":
        runs = []
        for e, c in enumerate(counts):
            padded = (int(c) + 127) // 128 * 128
            runs.append(np.concatenate([np.full(c, e, np.int32), np.full(padded - c, -1, np.int32)]))
        m_idx = np.concatenate(runs) if runs else np.zeros(0, np.int32)
        d["m_indices"] = m_idx.astype(np.int32)
        shape = (m_idx.size, cfg.K)
    elif cfg.mode == "masked":
        d["masked_m"] = counts
        shape = (cfg.E, cfg.max_m, cfg.K)
    else:
        raise ValueError(cfg.mode)
    d["x"] = _f32_to_bf16_bits_trunc(rx.standard_normal(shape, dtype=np.float32))
    if weights:
        d["qweight"] = _codes(rc, cfg.E, cfg.N, cfg.K)
        d["scales"] = _scales(rs, cfg.E, cfg.N, cfg.K)
    return d
