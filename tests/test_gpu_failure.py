"""Failure detection on the device, without a GPU fault.

Every pipeline wait of the GEMM kernels is bounded in time. The library's self-test
kernel runs that same wait on an mbarrier that nothing completes: with a short limit
it must give up and report CHORD_DEV_TIMEOUT, a second waiter with the kernels' own
1 s limit must see the CTA's abort flag and return early, and the context must stay
usable afterwards (a layer call right after still matches the oracle)."""
import numpy as np
import pytest

import oracle
from helpers import assert_layer_close, ensure_built
from w4a16_int4_mixture_align_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def chord():
    ensure_built()
    from w4a16_int4_mixture_align_b200 import chord as c
    return c


@pytest.mark.parametrize("limit_us", [2000, 20000])
def test_bounded_wait_times_out_and_aborts_peers(chord, limit_us):
    import torch
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    elapsed = torch.zeros(2, dtype=torch.int64, device="cuda")
    chord.chord_selftest_wait_timeout(status, elapsed, limit_us)
    torch.cuda.synchronize()
    st = int(status.item()) & 0xffffffff
    waited = elapsed.cpu().numpy()
    assert st == chord.CHORD_DEV_TIMEOUT, hex(st)
    # the short wait ran out after its limit (plus at most a few suspend intervals)
    assert limit_us * 1000 <= waited[0] < limit_us * 1000 + 50_000_000, waited
    # the 1 s waiter left on the abort flag, long before its own limit
    assert waited[1] < limit_us * 1000 + 50_000_000, waited


def test_context_usable_after_timeout(chord):
    import torch
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    elapsed = torch.zeros(2, dtype=torch.int64, device="cuda")
    chord.chord_selftest_wait_timeout(status, elapsed, 1000)
    torch.cuda.synchronize()
    d = inputs.make_inputs(inputs.CONFIGS["tiny"])
    cfg = d["cfg"]
    layer = chord.ChordMoE(d["qw13"], d["s13"].view(np.int16), d["qw2"], d["s2"].view(np.int16),
                           topk=cfg.topk, max_tokens=cfg.T, block_m=8)
    x = torch.from_numpy(d["x"].view(np.int16)).cuda().view(torch.bfloat16)
    out = layer(x, torch.from_numpy(d["topk_ids"]).cuda(), torch.from_numpy(d["topk_weights"]).cuda())
    torch.cuda.synchronize()
    assert layer.check_status() == 0
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    ref = oracle.moe_forward(d["x"], d["topk_ids"], d["topk_weights"], d["qw13"], d["s13"], d["qw2"], d["s2"])
    assert_layer_close(got, ref)


def test_selftest_rejects_bad_arguments(chord):
    import torch
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    elapsed = torch.zeros(2, dtype=torch.int64, device="cuda")
    for bad in (0, 2_000_000):
        with pytest.raises(chord.ChordError) as ei:
            chord.chord_selftest_wait_timeout(status, elapsed, bad)
        assert ei.value.status == chord.CHORD_ERR_INVALID_ARG
