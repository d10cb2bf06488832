"""GPU routing sort vs the oracle: bit-exact sorted_ids / expert_ids / num_tokens_padded /
expert_offsets, on generated workloads of every configuration and on edge cases."""
import numpy as np
import pytest

import oracle
from helpers import ensure_built
from w4a16_int4_mixture_align_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def chord():
    ensure_built()
    import torch  # noqa: F401
    from w4a16_int4_mixture_align_b200 import chord as c
    return c


def run_align(chord, ids: np.ndarray, E: int, bm: int):
    import torch
    T, k = ids.shape
    cap = chord.chord_moe_align_capacity(T, k, E, bm)
    nb = chord.chord_moe_align_num_blocks(T, k, E, bm)
    dev = torch.device("cuda")
    d_ids = torch.from_numpy(np.ascontiguousarray(ids)).to(dev) if ids.size else torch.empty((T, k), dtype=torch.int32, device=dev)
    # poison outputs so unwritten entries are caught
    s = torch.full((max(cap, 1),), -7, dtype=torch.int32, device=dev)
    e = torch.full((max(nb, 1),), -7, dtype=torch.int32, device=dev)
    n = torch.full((2,), -7, dtype=torch.int32, device=dev)
    o = torch.full((E + 1,), -7, dtype=torch.int32, device=dev)
    wsb = chord.chord_moe_align_workspace_bytes(T, k, E)
    ws = torch.full((max(wsb, 1),), 0x5A, dtype=torch.uint8, device=dev) if wsb else None
    chord.chord_moe_align(d_ids, E, bm, s, e, n, o, ws)
    torch.cuda.synchronize()
    assert int(n.cpu()[1]) == chord.routing_tag(bm)  # the block_m the forward checks
    return s.cpu().numpy()[:cap], e.cpu().numpy()[:nb], int(n.cpu()[0]), o.cpu().numpy()


def check(chord, ids, E, bm):
    gs, ge, gn, go = run_align(chord, ids, E, bm)
    rs, re_, rn, ro = oracle.moe_align(ids, E, bm)
    assert gn == rn
    assert np.array_equal(gs, rs), np.nonzero(gs != rs)[0][:10]
    assert np.array_equal(ge, re_), np.nonzero(ge != re_)[0][:10]
    assert np.array_equal(go, ro)


@pytest.mark.parametrize("name", list(inputs.CONFIGS))
@pytest.mark.parametrize("bm", [8, 16, 64, 256])
def test_align_configs(chord, name, bm):
    cfg = inputs.CONFIGS[name]
    ids, _ = inputs.make_routing(cfg)
    check(chord, ids, cfg.E, bm)


@pytest.mark.parametrize("T,k,E,bm,seed", [
    (1, 1, 1, 1, 0), (5, 3, 4, 1, 1), (37, 8, 48, 8, 2), (100, 8, 1, 16, 3),
    (4095, 8, 384, 5, 4),        # 32760 slots: last single-CTA size
    (4097, 8, 384, 7, 5),        # 32776 slots: multi-CTA path with a ragged last chunk
    (20000, 6, 1024, 256, 6), (3000, 8, 2, 3, 7),
])
def test_align_random(chord, T, k, E, bm, seed):
    rng = np.random.default_rng(seed)
    ids = rng.integers(-2, E + 3, size=(T, k)).astype(np.int32)
    check(chord, ids, E, bm)


def test_align_no_local_slots(chord):
    ids = np.full((64, 8), -1, dtype=np.int32)
    gs, ge, gn, _ = run_align(chord, ids, 48, 16)
    assert gn == 0 and np.all(gs == 64 * 8) and np.all(ge == -1)


def test_align_empty_batch(chord):
    ids = np.zeros((0, 8), dtype=np.int32)
    gs, ge, gn, go = run_align(chord, ids, 48, 16)
    assert gn == 0 and np.all(gs == 0) and np.all(ge == -1) and np.all(go == 0)


def test_align_one_hot_expert(chord):
    # every slot to one expert: a single long run, many blocks
    ids = np.full((9000, 8), 17, dtype=np.int32)
    check(chord, ids, 48, 8)
