"""CPU oracle for the W4A16 mixture-of-experts layer (ctypes wrapper over ``oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg are the only callers. The CUDA path never imports this package, and
this package imports nothing from the CUDA path.

Each function follows the step of the layer named in its docstring; ``oracle.c``
carries the citations of the Chord blog sections the steps come from.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

CFLAGS = ["-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
          "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (plain gcc, no GPU)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, i32p, u16p, f32p = ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
        lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f32.restype = ctypes.c_float
        lib.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
        lib.oracle_dequant.argtypes = [i32p, u16p, i64, i64, f32p]
        lib.oracle_dequant.restype = None
        lib.oracle_align_capacity.argtypes = [i64, i64, i64, i64]
        lib.oracle_align_capacity.restype = i64
        lib.oracle_align_blocks.argtypes = [i64, i64, i64, i64]
        lib.oracle_align_blocks.restype = i64
        lib.oracle_moe_align.argtypes = [i32p, i64, i64, i64, i64, i32p, i32p, i32p, i32p]
        lib.oracle_grouped_gemm.restype = ctypes.c_int
        lib.oracle_grouped_gemm.argtypes = [u16p, i64, i64, i32p, u16p, i64, i64, i32p, i32p, i64, u16p,
                                            ctypes.c_int]
        lib.oracle_router_topk.restype = ctypes.c_int
        lib.oracle_router_topk.argtypes = [f32p, i64, i64, i64, i32p, f32p]
        lib.oracle_moe_align.restype = ctypes.c_int
        lib.oracle_moe_forward.argtypes = [u16p, i32p, f32p, i32p, u16p, i32p, u16p,
                                           i64, i64, i64, i64, i64, ctypes.c_void_p, i64,
                                           u16p, ctypes.c_int]
        lib.oracle_moe_forward.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def f32_to_bf16(x) -> np.ndarray:
    """Round-to-nearest-even binary32 -> bfloat16 bit patterns, element by element."""
    lib = _load()
    x = np.asarray(x, dtype=np.float32)
    flat = [lib.oracle_f32_to_bf16(float(v)) for v in x.reshape(-1)]
    return np.array(flat, dtype=np.uint16).reshape(x.shape)


def dequant(qweight: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Unpack + dequantise one expert: float32 [N, K] holding bf16((q - 8) * s)."""
    lib = _load()
    qweight = np.ascontiguousarray(qweight, dtype=np.int32)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    N, K8 = qweight.shape
    K = K8 * 8
    assert scales.shape == (N, K // 32)
    w = np.empty((N, K), dtype=np.float32)
    lib.oracle_dequant(_ptr(qweight), _ptr(scales), N, K, _ptr(w))
    return w


def align_capacity(T: int, topk: int, E: int, block_m: int) -> int:
    return int(_load().oracle_align_capacity(T, topk, E, block_m))


def align_blocks(T: int, topk: int, E: int, block_m: int) -> int:
    return int(_load().oracle_align_blocks(T, topk, E, block_m))


def moe_align(topk_ids: np.ndarray, E: int, block_m: int):
    """Routing sort: (sorted_ids, expert_ids, num_tokens_padded, expert_offsets)."""
    lib = _load()
    ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    T, topk = ids.shape
    sorted_ids = np.empty(align_capacity(T, topk, E, block_m), dtype=np.int32)
    expert_ids = np.empty(align_blocks(T, topk, E, block_m), dtype=np.int32)
    ntp = np.zeros(1, dtype=np.int32)
    offs = np.zeros(E + 1, dtype=np.int32)
    rc = lib.oracle_moe_align(_ptr(ids), T, topk, E, block_m, _ptr(sorted_ids),
                              _ptr(expert_ids), _ptr(ntp), _ptr(offs))
    if rc != 0:
        raise ValueError(f"oracle_moe_align failed ({rc})")
    return sorted_ids, expert_ids, int(ntp[0]), offs


def grouped_gemm(x, qweight, scales, m_indices=None, masked_m=None, out=None, n_threads=0):
    """Grouped GEMM: out[m] = bf16(x[m] . W[e_m]^T), FP32 accumulation; e_m from m_indices
    (contiguous layout, -1 = no expert) or from masked_m (masked layout, x viewed as
    [E * max_m, K]). Rows without an expert keep the contents of `out` (zeros if None)."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.uint16)
    qw = np.ascontiguousarray(qweight, dtype=np.int32)
    sc = np.ascontiguousarray(scales, dtype=np.uint16)
    E, N, _ = qw.shape
    if masked_m is not None:
        E_, max_m, K = x.shape
        M = E_ * max_m
        x2 = x.reshape(M, K)
    else:
        M, K = x.shape
        max_m = 0
        x2 = x
    res = np.zeros((M, N), dtype=np.uint16) if out is None else np.ascontiguousarray(out, dtype=np.uint16).reshape(M, N).copy()
    mi = None if m_indices is None else np.ascontiguousarray(m_indices, dtype=np.int32)
    mm = None if masked_m is None else np.ascontiguousarray(masked_m, dtype=np.int32)
    rc = lib.oracle_grouped_gemm(_ptr(x2), M, K, _ptr(qw), _ptr(sc), E, N,
                                 None if mi is None else _ptr(mi), None if mm is None else _ptr(mm),
                                 max_m, _ptr(res), int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle_grouped_gemm failed ({rc})")
    return res


def router_topk(logits: np.ndarray, topk: int):
    """Router upstream of the routing sort: (topk_ids int32 [T, k] global expert ids,
    topk_weights float32 [T, k]), the top-k logits (ties to the lower id) and their
    softmax renormalised over the chosen ones."""
    lib = _load()
    lg = np.ascontiguousarray(logits, dtype=np.float32)
    T, G = lg.shape
    ids = np.empty((T, topk), dtype=np.int32)
    w = np.empty((T, topk), dtype=np.float32)
    rc = lib.oracle_router_topk(_ptr(lg), T, G, topk, _ptr(ids), _ptr(w))
    if rc != 0:
        raise ValueError(f"oracle_router_topk failed ({rc})")
    return ids, w


def moe_forward(x, topk_ids, topk_weights, qw13, s13, qw2, s2, rows=None, n_threads=0):
    """The layer's output rows (bf16 bits [len(rows), H]; all T rows when rows is None)."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.uint16)
    ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    tw = np.ascontiguousarray(topk_weights, dtype=np.float32)
    qw13 = np.ascontiguousarray(qw13, dtype=np.int32)
    qw2 = np.ascontiguousarray(qw2, dtype=np.int32)
    s13 = np.ascontiguousarray(s13, dtype=np.uint16)
    s2 = np.ascontiguousarray(s2, dtype=np.uint16)
    T, H = x.shape
    E, N13, _ = qw13.shape
    I = N13 // 2
    topk = ids.shape[1]
    assert qw2.shape == (E, H, I // 8) and s13.shape == (E, N13, H // 32)
    assert s2.shape == (E, H, I // 32) and ids.shape == tw.shape == (T, topk)
    if rows is None:
        rows_arr, n = None, T
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        n = rows_arr.shape[0]
    out = np.empty((n, H), dtype=np.uint16)
    rc = lib.oracle_moe_forward(_ptr(x), _ptr(ids), _ptr(tw), _ptr(qw13), _ptr(s13),
                                _ptr(qw2), _ptr(s2), T, H, I, E, topk,
                                None if rows_arr is None else _ptr(rows_arr), n, _ptr(out),
                                int(n_threads))
    if rc != 0:
        raise ValueError(f"oracle_moe_forward failed ({rc})")
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 values (exact widening)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
