"""Weight repack and dequantisation on the GPU.

* the blob layout, inverted here in numpy from the layout's specification, returns the
  input codes and scales bit-exactly (gate/up interleave included);
* the kernels' own dequantisation, run over every code and every finite bf16 scale,
  matches the oracle's bf16((q - 8) * s) bit for bit;
* a blob of the wrong role or shape fails loudly (host registry) or raises the device
  status bit (header check) without touching the output.
"""
import numpy as np
import pytest

import oracle
from helpers import ensure_built

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def chord():
    ensure_built()
    from w4a16_int4_mixture_align_b200 import chord as c
    return c


def repack(chord, qw, s, role):
    import torch
    E, N, K8 = qw.shape
    blob = torch.zeros(chord.chord_repacked_bytes(E, N, K8 * 8), dtype=torch.uint8, device="cuda")
    chord.chord_repack_weights(torch.from_numpy(qw).cuda(), torch.from_numpy(s.view(np.int16)).cuda(), role, blob)
    torch.cuda.synchronize()
    return blob


def invert_layout(blob: np.ndarray, E, N, K, role):
    """Numpy inverse of the tile layout -> (qweight [E,N,K/8] int32, scales [E,N,K/32] u16).

    Tiles of 9216 bytes after a 256-byte header, tile (e, nt, kt) in that order; each
    tile is 8192 bytes of codes then 1024 bytes of scales."""
    NT, KT = N // 128, K // 128
    tiles = blob[256:256 + E * NT * KT * 9216].reshape(E, NT, KT, 9216)
    codes = np.ascontiguousarray(tiles[..., :8192]).view(np.uint32)
    codes = codes.reshape(E, NT, KT, 8, 2, 8, 4, 4)          # e nt kt rb h g slot j
    # the 16-byte vector of K slice t of row g sits in slot t ^ ((g >> 1) & 3)
    g = np.arange(8)[:, None].repeat(4, axis=1)
    t = np.arange(4)[None, :].repeat(8, axis=0)
    codes = codes[..., g, t ^ ((g >> 1) & 3), :]             # e nt kt rb h g t j
    # un-permute nibbles: K offset u sits in nibble (u>>1) + 4*(u&1)
    slot = [(u >> 1) + 4 * (u & 1) for u in range(8)]
    words = np.zeros(codes.shape, dtype=np.uint32)
    for u in range(8):
        words |= ((codes >> np.uint32(4 * slot[u])) & np.uint32(0xF)) << np.uint32(4 * u)
    # physical row p = nt*128 + rb*16 + 8h + g ; k/8 = kt*16 + 4j + t
    w = words.transpose(0, 1, 3, 4, 5, 2, 7, 6).reshape(E, N, K // 8)
    sc = np.ascontiguousarray(tiles[..., 8192:]).view(np.uint16)
    sc = sc.reshape(E, NT, KT, 8, 8, 2, 4)                     # e nt kt rb g h j
    sc = sc.transpose(0, 1, 3, 5, 4, 2, 6).reshape(E, N, K // 32)
    if role == 1:  # gate_up: physical block of 16 = 8 gate rows then 8 up rows
        p = np.arange(N)
        blk, r = p // 16, p % 16
        logical = np.where(r < 8, blk * 8 + r, N // 2 + blk * 8 + (r - 8))
        inv = np.empty_like(w)
        inv[:, logical] = w
        sinv = np.empty_like(sc)
        sinv[:, logical] = sc
        w, sc = inv, sinv
    return w.view(np.int32), sc


@pytest.mark.parametrize("role,E,N,K", [(1, 2, 256, 384), (2, 3, 384, 256), (1, 1, 512, 128)])
def test_repack_layout_round_trip(chord, role, E, N, K):
    rng = np.random.default_rng(role * 100 + E)
    qw = rng.integers(0, 2 ** 32, size=(E, N, K // 8), dtype=np.uint32).view(np.int32)
    s = rng.integers(0, 2 ** 16, size=(E, N, K // 32), dtype=np.uint16)
    blob = repack(chord, qw, s, role).cpu().numpy()
    hdr = blob[:48].view(np.uint32)
    assert hdr[0] == 0x34574843 and hdr[1] == 3 and hdr[2] == 2 and hdr[3] == role
    assert list(hdr[4:8].view(np.int32)) == [E, N, K, 32]
    qw2, s2 = invert_layout(blob, E, N, K, role)
    assert np.array_equal(qw2, qw)
    assert np.array_equal(s2, s)


def test_dequant_exhaustive_matches_oracle(chord):
    """Every code x every finite bf16 scale through the kernels' dequant8."""
    import torch
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    scales = pats[(pats & 0x7F80) != 0x7F80]          # 65280 finite patterns = 510 * 128 rows
    N, K = scales.size, 128
    words = np.array([0x76543210, 0xFEDCBA98] * (K // 16), dtype=np.uint32)
    qw = np.tile(words.view(np.int32), (N, 1))[None]
    s = np.repeat(scales[:, None], K // 32, axis=1)[None]
    blob = repack(chord, np.ascontiguousarray(qw), np.ascontiguousarray(s), 2)
    w = torch.empty((1, N, K), dtype=torch.int16, device="cuda")
    chord.chord_dequant_weights(blob, w)
    got = w.cpu().numpy().view(np.uint16)[0]
    ref = oracle.dequant(qw[0], s[0])
    ref_bits = ref.view(np.uint32) >> 16
    assert np.all(ref.view(np.uint32) & 0xFFFF == 0)
    mism = got != ref_bits.astype(np.uint16)
    assert not mism.any(), (np.nonzero(mism)[0][:5], got[mism][:5], ref_bits[mism][:5])


def test_dequant_random_weights_match_oracle(chord):
    import torch
    rng = np.random.default_rng(5)
    E, N, K = 2, 256, 512
    qw = rng.integers(0, 2 ** 32, size=(E, N, K // 8), dtype=np.uint32).view(np.int32)
    s = (rng.uniform(0.005, 0.02, size=(E, N, K // 32)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    for role in (1, 2):
        blob = repack(chord, qw, s, role)
        w = torch.empty((E, N, K), dtype=torch.int16, device="cuda")
        chord.chord_dequant_weights(blob, w)
        got = w.cpu().numpy().view(np.uint16)
        for e in range(E):
            ref = (oracle.dequant(qw[e], s[e]).view(np.uint32) >> 16).astype(np.uint16)
            assert np.array_equal(got[e], ref)
