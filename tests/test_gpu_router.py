"""GPU router + routing sort (chord_router_topk_align) vs the oracle: topk_ids and every
routing tensor bit-exact, topk_weights within float rounding (the GPU exponentiates in
fp32, the oracle in double). Covers the one-launch path (up to 8 tokens), the routing
kernel + single-CTA sort and routing kernel + multi-CTA sort paths, ties, E_global not a
multiple of 32, topk = E_global and the largest E_global."""
import numpy as np
import pytest

import oracle
from helpers import ensure_built

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def chord():
    ensure_built()
    import torch  # noqa: F401
    from w4a16_int4_mixture_align_b200 import chord as c
    return c


def make_logits(T, G, kind, seed):
    rng = np.random.default_rng(seed)
    if kind == "normal":
        lg = rng.standard_normal((T, G), dtype=np.float32)
    elif kind == "uniform":
        lg = rng.random((T, G), dtype=np.float32)
    elif kind == "ties":
        lg = (rng.integers(-4, 5, (T, G)) / 2).astype(np.float32)
    else:
        raise ValueError(kind)
    return np.ascontiguousarray(lg)


def run_router(chord, logits, topk, E, bm):
    import torch
    T, G = logits.shape
    dev = torch.device("cuda")
    cap = chord.chord_moe_align_capacity(T, topk, E, bm)
    nb = chord.chord_moe_align_num_blocks(T, topk, E, bm)
    lg = torch.from_numpy(logits).to(dev) if T else torch.empty((0, G), dtype=torch.float32, device=dev)
    ids = torch.full((T, topk), -7, dtype=torch.int32, device=dev)
    w = torch.full((T, topk), -7.0, dtype=torch.float32, device=dev)
    s = torch.full((max(cap, 1),), -7, dtype=torch.int32, device=dev)
    e = torch.full((max(nb, 1),), -7, dtype=torch.int32, device=dev)
    n = torch.full((2,), -7, dtype=torch.int32, device=dev)
    o = torch.full((E + 1,), -7, dtype=torch.int32, device=dev)
    wsb = chord.chord_moe_align_workspace_bytes(T, topk, E)
    ws = torch.full((max(wsb, 1),), 0x5A, dtype=torch.uint8, device=dev) if wsb else None
    chord.chord_router_topk_align(lg, topk, E, bm, ids, w, s, e, n, o, ws)
    torch.cuda.synchronize()
    assert int(n.cpu()[1]) == chord.routing_tag(bm)
    return (ids.cpu().numpy(), w.cpu().numpy(), s.cpu().numpy()[:cap], e.cpu().numpy()[:nb],
            int(n.cpu()[0]), o.cpu().numpy())


CASES = [
    # T, E_global, topk, E local, block_m, logits
    (1, 384, 8, 48, 8, "normal"),        # one launch
    (8, 384, 8, 48, 8, "uniform"),       # one launch, largest batch
    (9, 384, 8, 48, 8, "uniform"),       # routing kernel + single-CTA sort
    (128, 384, 8, 48, 8, "uniform"),     # EP8 decode shape
    (32, 384, 8, 384, 8, "normal"),      # TP8 decode shape
    (512, 384, 8, 48, 16, "normal"),     # 4096 slots: the largest single-CTA sort
    (513, 384, 8, 48, 16, "normal"),     # 4104 slots: multi-CTA sort
    (4096, 384, 8, 384, 128, "normal"),  # TP8 prefill shape
    (8192, 384, 8, 48, 256, "normal"),   # EP8 prefill shape
    (64, 100, 3, 10, 4, "normal"),       # E_global not a multiple of 32
    (20, 64, 64, 64, 8, "normal"),       # topk = E_global
    (50, 1024, 1, 16, 1, "normal"),      # largest E_global, topk 1
    (300, 384, 8, 48, 8, "ties"),        # many equal logits: ties to the lower id
    (700, 384, 8, 48, 8, "ties"),
]


@pytest.mark.parametrize("T,G,k,E,bm,kind", CASES)
def test_router_align_matches_oracle(chord, T, G, k, E, bm, kind):
    logits = make_logits(T, G, kind, seed=T * 7 + G + k)
    ids, w, s, e, n, o = run_router(chord, logits, k, E, bm)
    ref_ids, ref_w = oracle.router_topk(logits, k)
    np.testing.assert_array_equal(ids, ref_ids)
    np.testing.assert_allclose(w, ref_w, rtol=1e-6, atol=1e-7)
    rs, re_, rn, ro = oracle.moe_align(ref_ids, E, bm)
    np.testing.assert_array_equal(s, rs)
    np.testing.assert_array_equal(e, re_)
    assert n == rn
    np.testing.assert_array_equal(o, ro)


def test_router_align_empty_batch(chord):
    ids, w, s, e, n, o = run_router(chord, np.zeros((0, 384), np.float32), 8, 48, 8)
    rs, re_, rn, ro = oracle.moe_align(np.zeros((0, 8), np.int32), 48, 8)
    assert n == rn == 0
    np.testing.assert_array_equal(e, re_)
    np.testing.assert_array_equal(o, ro)


def test_router_rejects_bad_expert_counts(chord):
    import torch
    lg = torch.zeros((4, 8), dtype=torch.float32, device="cuda")
    ids = torch.empty((4, 16), dtype=torch.int32, device="cuda")
    w = torch.empty((4, 16), dtype=torch.float32, device="cuda")
    s = torch.empty(64, dtype=torch.int32, device="cuda")
    with pytest.raises(chord.ChordError):  # topk 16 > E_global 8
        chord.chord_router_topk_align(lg, 16, 8, 1, ids, w, s, s, s)
