"""The C-ABI library loads and exports every symbol include/*.h declares; host-only
logic (sizes, selector, argument checks made before any device access) behaves."""
import ctypes

import pytest

from helpers import ensure_built, header_symbols


@pytest.fixture(scope="module")
def lib():
    ensure_built()
    from w4a16_int4_mixture_align_b200 import chord
    return chord


def test_exports_every_declared_symbol(lib):
    names = header_symbols()
    assert len(names) >= 13
    h = ctypes.CDLL(lib.LIB_PATH)
    for n in names:
        assert hasattr(h, n), n
    assert set(names) == set(lib.SIGNATURES), set(names) ^ set(lib.SIGNATURES)


def test_status_strings(lib):
    assert lib.chord_status_string(0) == "CHORD_OK"
    assert lib.chord_status_string(3) == "CHORD_ERR_LAYOUT_MISMATCH"
    assert lib.chord_status_string(99) == "CHORD_ERR_UNKNOWN"


def test_align_sizes(lib):
    assert lib.chord_moe_align_capacity(16, 2, 8, 16) == 32 + 8 * 15
    assert lib.chord_moe_align_num_blocks(16, 2, 8, 16) == (32 + 120 + 15) // 16
    assert lib.chord_moe_align_capacity(0, 8, 48, 8) == 48 * 7
    assert lib.chord_moe_align_capacity(-1, 8, 48, 8) == -1
    assert lib.chord_moe_align_workspace_bytes(128, 8, 48) == 0      # single-CTA path
    assert lib.chord_moe_align_workspace_bytes(16384, 8, 48) > 0     # multi-CTA path


def test_repacked_bytes(lib):
    E, N, K = 48, 4096, 7168
    codes, scales = E * N * K // 2, E * N * K // 32 * 2
    b = lib.chord_repacked_bytes(E, N, K, 32)
    assert b >= 256 + codes + scales and b - (256 + codes + scales) < 512
    assert lib.chord_repacked_bytes(E, N, K, 64) == 0   # only group-32
    assert lib.chord_repacked_bytes(E, 100, K, 32) == 0  # N % 128


def test_workspace_bytes(lib):
    T, k, E, H, I, bm = 128, 8, 48, 7168, 2048, 8
    ws = lib.chord_moe_workspace_bytes(T, k, E, H, I, bm)
    cap = T * k + E * (bm - 1)
    assert ws >= 256 + cap * I * 2 + T * k * H * 4


def test_selector_keys_on_tokens_per_expert(lib):
    # EP8 decode (128 tokens, top-8 of 384): ~2.7 tokens per expert -> streaming schedule
    assert lib.chord_select_block_m(128, 8, 48, 384, 7168, 2048) <= 32
    assert lib.chord_select_block_m(32, 8, 384, 384, 7168, 256) <= 32
    # prefill: ~171 tokens per expert -> tensor-core schedule
    assert lib.chord_select_block_m(8192, 8, 48, 384, 7168, 2048) > 32
    # same total tokens, far fewer per expert -> the smaller schedule
    assert lib.chord_select_block_m(1024, 8, 384, 384 * 8, 7168, 2048) <= 32
    # memoised: same answer twice
    assert lib.chord_select_block_m(4096, 8, 384, 384, 7168, 256) == lib.chord_select_block_m(4096, 8, 384, 384, 7168, 256)


def _raw(lib):
    return lib.lib()


def test_repack_rejects_unsupported_group_before_touching_memory(lib):
    fake = ctypes.c_void_p(0x1000)
    st = _raw(lib).chord_repack_weights(fake, fake, 1, 128, 128, 64, 1, ctypes.c_void_p(0x100000), 1 << 20, None)
    assert st == lib.CHORD_ERR_UNSUPPORTED
    assert "group" in lib.chord_last_error_detail()
    st = _raw(lib).chord_repack_weights(fake, fake, 1, 128, 100, 32, 1, ctypes.c_void_p(0x100000), 1 << 20, None)
    assert st == lib.CHORD_ERR_UNSUPPORTED
    st = _raw(lib).chord_repack_weights(fake, fake, 1, 128, 128, 32, 7, ctypes.c_void_p(0x100000), 1 << 20, None)
    assert st == lib.CHORD_ERR_INVALID_ARG
    st = _raw(lib).chord_repack_weights(fake, fake, 1, 128, 128, 32, 1, ctypes.c_void_p(0x100010), 1 << 20, None)
    assert st == lib.CHORD_ERR_INVALID_ARG  # misaligned blob


def test_forward_rejects_bad_shapes_and_small_workspace(lib):
    f = ctypes.c_void_p(0x100000)
    call = _raw(lib).chord_moe_forward
    # H not a multiple of 128
    st = call(f, f, f, f, f, f, 8, f, f, 16, 200, 128, 8, 2, f, f, 1 << 30, 0, None)
    assert st == lib.CHORD_ERR_UNSUPPORTED
    # block_m out of range
    st = call(f, f, f, f, f, f, 300, f, f, 16, 256, 128, 8, 2, f, f, 1 << 30, 0, None)
    assert st == lib.CHORD_ERR_UNSUPPORTED
    # workspace too small
    st = call(f, f, f, f, f, f, 8, f, f, 16, 256, 128, 8, 2, f, f, 1024, 0, None)
    assert st == lib.CHORD_ERR_WORKSPACE_TOO_SMALL
    # exclusive flags
    st = call(f, f, f, f, f, f, 8, f, f, 16, 256, 128, 8, 2, f, f, 1 << 30, 6, None)
    assert st == lib.CHORD_ERR_INVALID_ARG


def test_align_rejects_bad_args(lib):
    f = ctypes.c_void_p(0x100000)
    call = _raw(lib).chord_moe_align
    assert call(f, 16, 2, 0, 8, f, f, f, None, None, 0, None) == lib.CHORD_ERR_UNSUPPORTED      # E = 0
    assert call(f, 16, 2, 2000, 8, f, f, f, None, None, 0, None) == lib.CHORD_ERR_UNSUPPORTED   # E > 1024
    assert call(f, 16, 2, 8, 0, f, f, f, None, None, 0, None) == lib.CHORD_ERR_UNSUPPORTED      # block_m = 0
    assert call(f, 16384, 8, 48, 8, f, f, f, None, None, 0, None) == lib.CHORD_ERR_WORKSPACE_TOO_SMALL


def test_wait_selftest_rejects_bad_args_before_touching_the_device(lib):
    f = ctypes.c_void_p(0x100000)
    call = _raw(lib).chord_selftest_wait_timeout
    assert call(None, f, 1000, None) == lib.CHORD_ERR_INVALID_ARG
    assert call(f, None, 1000, None) == lib.CHORD_ERR_INVALID_ARG
    assert call(f, f, 0, None) == lib.CHORD_ERR_INVALID_ARG          # limit below 1 us
    assert call(f, f, 1000001, None) == lib.CHORD_ERR_INVALID_ARG    # limit above 1 s
    assert "limit_us" in lib.chord_last_error_detail()


def test_align_workspace_follows_run_size(lib):
    # multi-CTA routing sort: 256-slot runs while E x runs stays within 2^17 histogram
    # entries, else 1024-slot runs (so the no-allocation variant's static scratch of
    # 576 KiB always suffices up to 2^17 slots)
    def runs_bytes(n, E, run):
        g = -(-n // run)
        a = lambda x: (x + 255) // 256 * 256
        return a(E * g * 4) + a(E * 4)
    assert lib.chord_moe_align_workspace_bytes(8192, 8, 48) == runs_bytes(8192 * 8, 48, 256)
    assert lib.chord_moe_align_workspace_bytes(16384, 8, 1024) == runs_bytes(16384 * 8, 1024, 1024)
    assert lib.chord_moe_align_workspace_bytes(16384, 8, 1024) <= 576 * 1024


def test_noalloc_reports_what_chord_moe_align_reports(lib):
    # the no-allocation routing sort shares chord_moe_align's checks, statuses and detail
    # texts; these fail before any device access
    f = ctypes.c_void_p(0x100000)
    ws = _raw(lib).chord_moe_align
    na = _raw(lib).chord_moe_align_noalloc
    cases = [(16, 2, 0, 8), (16, 2, 2000, 8), (16, 2, 8, 0), (16, 2, 8, 300), (-1, 2, 8, 8), (16, 0, 8, 8),
             (1 << 62, 8, 48, 8), (1 << 28, 8, 48, 8)]
    for T, k, E, bm in cases:
        a = ws(f, T, k, E, bm, f, f, f, None, f, 1 << 40, None)
        da = lib.chord_last_error_detail()
        b = na(f, T, k, E, bm, f, f, f, None, None)
        db = lib.chord_last_error_detail()
        assert a == b != lib.CHORD_OK and da == db, (T, k, E, bm, a, b, da, db)
    assert na(None, 16, 2, 8, 8, f, f, f, None, None) == lib.CHORD_ERR_INVALID_ARG  # null ids
    assert "null" in lib.chord_last_error_detail()
    # its own limit: the static scratch holds the histograms of up to 2^17 slots
    assert na(f, 16385, 8, 48, 16, f, f, f, None, None) == lib.CHORD_ERR_UNSUPPORTED
    assert "static scratch" in lib.chord_last_error_detail()


def test_align_size_checks_do_not_overflow(lib):
    # T * topk is bounded before it is formed: T near 2^62 must be refused, not wrap
    f = ctypes.c_void_p(0x100000)
    st = _raw(lib).chord_moe_align(f, (1 << 62) + 1, 64, 48, 8, f, f, f, None, f, 1 << 40, None)
    assert st == lib.CHORD_ERR_UNSUPPORTED and "2^31" in lib.chord_last_error_detail()


def test_tp_reduce_round_checks_its_arguments_before_touching_memory(lib):
    # every rejection happens on the host, before any device access
    raw = _raw(lib)
    P = ctypes.c_void_p
    good_in = (P * 2)(0x100000, 0x200000)
    good_out = (P * 2)(0x300000, 0x400000)
    st = raw.chord_tp_reduce_round(good_in, good_out, 0, 0, 64, None)           # W = 0
    assert st == lib.CHORD_ERR_INVALID_ARG and "W=0" in lib.chord_last_error_detail()
    assert raw.chord_tp_reduce_round(good_in, good_out, 2, 2, 64, None) == lib.CHORD_ERR_INVALID_ARG   # rank >= W
    assert raw.chord_tp_reduce_round(good_in, good_out, 65, 0, 64, None) == lib.CHORD_ERR_INVALID_ARG  # W > 64
    assert raw.chord_tp_reduce_round(good_in, good_out, 2, 0, 6, None) == lib.CHORD_ERR_INVALID_ARG    # n % 4
    assert raw.chord_tp_reduce_round(None, good_out, 2, 0, 64, None) == lib.CHORD_ERR_INVALID_ARG
    assert raw.chord_tp_reduce_round((P * 2)(0x100000, None), good_out, 2, 0, 64, None) == lib.CHORD_ERR_INVALID_ARG
    st = raw.chord_tp_reduce_round((P * 2)(0x100000, 0x200008), good_out, 2, 0, 64, None)   # 8-byte aligned input
    assert st == lib.CHORD_ERR_INVALID_ARG and "aligned" in lib.chord_last_error_detail()
    # nothing to do: returns before looking for a device
    assert raw.chord_tp_reduce_round(good_in, good_out, 2, 1, 0, None) == lib.CHORD_OK
