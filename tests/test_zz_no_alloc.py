"""chord_moe_align_noalloc: the routing sort for callers that cannot allocate device
memory when they route a batch (an engine that reserved all free memory up front, code
under stream capture with no workspace at hand). Its scratch is a static device array
inside the library, so this checks, through the C ABI, that two calls in a row give
exactly what chord_moe_align gives with a caller workspace, on batches small enough for
the single-CTA path and large enough to use the static scratch, and that a batch past
the array's limit is refused. Kept in its own file, collected last."""
import numpy as np
import pytest

from helpers import ensure_built
from w4a16_int4_mixture_align_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def chord():
    ensure_built()
    from w4a16_int4_mixture_align_b200 import chord as c
    return c


def _buffers(chord, T, k, E, bm):
    import torch
    cap = chord.chord_moe_align_capacity(T, k, E, bm)
    nb = chord.chord_moe_align_num_blocks(T, k, E, bm)
    mk = lambda n: torch.full((max(n, 1),), -7, dtype=torch.int32, device="cuda")  # noqa: E731
    return mk(cap), mk(nb), mk(2), mk(E + 1), cap, nb


def _with_workspace(chord, ids, E, bm):
    import torch
    T, k = ids.shape
    s, e, n, o, cap, nb = _buffers(chord, T, k, E, bm)
    wsb = chord.chord_moe_align_workspace_bytes(T, k, E)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda") if wsb else None
    chord.chord_moe_align(ids, E, bm, s, e, n, o, ws)
    torch.cuda.synchronize()
    return [t.cpu().numpy()[:m] for t, m in ((s, cap), (e, nb), (n, 2), (o, E + 1))]


def _noalloc(chord, ids, E, bm):
    import torch
    T, k = ids.shape
    s, e, n, o, cap, nb = _buffers(chord, T, k, E, bm)
    chord.chord_moe_align_noalloc(ids, E, bm, s, e, n, o)
    torch.cuda.synchronize()
    return [t.cpu().numpy()[:m] for t, m in ((s, cap), (e, nb), (n, 2), (o, E + 1))]


@pytest.mark.parametrize("name,bm", [("ep8_decode", 8), ("skew", 256), ("ep8_prefill", 16), ("tp8_prefill", 64)])
def test_noalloc_matches_workspace_path_twice(chord, name, bm):
    import torch
    cfg = inputs.CONFIGS[name]
    ids_np, _ = inputs.make_routing(cfg)
    ids = torch.from_numpy(ids_np).cuda()
    ref = _with_workspace(chord, ids, cfg.E, bm)
    for _ in range(2):  # the static scratch keeps the previous call's contents
        got = _noalloc(chord, ids, cfg.E, bm)
        for g, r in zip(got, ref):
            assert np.array_equal(g, r)


def test_noalloc_two_different_batches_in_a_row(chord):
    import torch
    rng = np.random.default_rng(11)
    for T, E in ((9000, 384), (12000, 48)):
        ids = torch.from_numpy(rng.integers(-1, E, size=(T, 8)).astype(np.int32)).cuda()
        assert all(np.array_equal(g, r) for g, r in zip(_noalloc(chord, ids, E, 32), _with_workspace(chord, ids, E, 32)))


def test_noalloc_refuses_batches_past_the_static_limit(chord):
    import torch
    ids = torch.zeros((16385, 8), dtype=torch.int32, device="cuda")  # 131080 slots > 2^17
    s, e, n, o, _, _ = _buffers(chord, 16385, 8, 48, 16)
    with pytest.raises(chord.ChordError) as ei:
        chord.chord_moe_align_noalloc(ids, 48, 16, s, e, n, o)
    assert ei.value.status == chord.CHORD_ERR_UNSUPPORTED
    assert "static scratch" in chord.chord_last_error_detail()
