"""Python binding of libchord.so (include/chord.h): argument marshalling only.

Every function keeps its C name and forwards torch CUDA tensors as raw device pointers
on the current torch stream. Nothing here computes any part of the layer; when the
library is missing the import fails loudly (there is no fallback path).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libchord.so")

CHORD_OK = 0
CHORD_ERR_INVALID_ARG = 1
CHORD_ERR_UNSUPPORTED = 2
CHORD_ERR_LAYOUT_MISMATCH = 3
CHORD_ERR_WORKSPACE_TOO_SMALL = 4
CHORD_ERR_CUDA = 5
CHORD_ERR_DEVICE = 6

CHORD_DEV_ROUTING_INVALID = 0x1
CHORD_DEV_BLOB_MISMATCH = 0x2
CHORD_DEV_TIMEOUT = 0x4
CHORD_DEV_BLOCK_M_MISMATCH = 0x8


def routing_tag(block_m: int) -> int:
    """num_tokens_padded[1] as the routing entry points write it (CHORD_ROUTING_TAG)."""
    v = 0x52540000 | int(block_m)
    return v - (1 << 32) if v >= 1 << 31 else v

CHORD_ROLE_GATE_UP = 1
CHORD_ROLE_DOWN = 2
CHORD_ROLE_GROUPED_CONTIGUOUS = 3
CHORD_ROLE_GROUPED_MASKED = 4

CHORD_FLAG_VALIDATE_ROUTING = 0x1
CHORD_FLAG_FORCE_STREAM = 0x2
CHORD_FLAG_FORCE_TENSOR = 0x4
CHORD_FLAG_OUTPUT_FP32 = 0x8

# every symbol include/chord.h declares: (name, restype, argtypes)
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_SZ = ctypes.c_size_t
SIGNATURES = {
    "chord_status_string": (ctypes.c_char_p, [_I]),
    "chord_last_error_detail": (ctypes.c_char_p, []),
    "chord_moe_align_capacity": (_I64, [_I64, _I, _I, _I]),
    "chord_moe_align_num_blocks": (_I64, [_I64, _I, _I, _I]),
    "chord_moe_align_workspace_bytes": (_SZ, [_I64, _I, _I]),
    "chord_moe_align": (_I, [_P, _I64, _I, _I, _I, _P, _P, _P, _P, _P, _SZ, _P]),
    "chord_repacked_bytes": (_SZ, [_I, _I, _I, _I]),
    "chord_repack_weights": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _SZ, _P]),
    "chord_dequant_weights": (_I, [_P, _SZ, _P, _P]),
    "chord_select_block_m": (_I, [_I64, _I, _I, _I, _I, _I]),
    "chord_moe_workspace_bytes": (_SZ, [_I64, _I, _I, _I, _I, _I]),
    "chord_moe_forward": (_I, [_P, _P, _P, _P, _P, _P, _I, _P, _P, _I64, _I, _I, _I, _I, _P, _P,
                               _SZ, _I, _P]),
    "chord_moe_check_status": (_I, [_P, _P, ctypes.POINTER(ctypes.c_uint32)]),
    "chord_moe_align_noalloc": (_I, [_P, _I64, _I, _I, _I, _P, _P, _P, _P, _P]),
    "chord_router_topk_align": (_I, [_P, _I64, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "chord_grouped_workspace_bytes": (_SZ, [_I64, _I]),
    "chord_grouped_contiguous": (_I, [_P, _I64, _I, _P, _P, _I, _I, _P, _P, _SZ, _I, _P]),
    "chord_grouped_masked": (_I, [_P, _I, _I64, _I, _P, _I64, _P, _I, _P, _P, _SZ, _I, _P]),
    "chord_ep_plan_workspace_bytes": (_SZ, [_I64, _I]),
    "chord_ep_plan": (_I, [_P, _I64, _I, _I, _I, _P, _P, _P, _P, _SZ, _P]),
    "chord_ep_pack": (_I, [_P, _P, _P, _I64, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P]),
    "chord_ep_combine": (_I, [_P, _P, _I64, _I, _I, _P, _P]),
    "chord_round_bf16": (_I, [_P, _I64, _P, _P]),
    "chord_tp_reduce_round": (_I, [ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_void_p), _I, _I, _I64, _P]),
    "chord_set_timing_events": (_I, [ctypes.POINTER(ctypes.c_void_p), _I]),
    "chord_launch_count": (ctypes.c_uint64, []),
    "chord_selftest_wait_timeout": (_I, [_P, _P, ctypes.c_uint32, _P]),
}

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is not built; run `python -m w4a16_int4_mixture_align_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _lib = h
    return _lib


class ChordError(RuntimeError):
    def __init__(self, status: int, what: str):
        detail = lib().chord_last_error_detail().decode()
        name = lib().chord_status_string(status).decode()
        super().__init__(f"{what}: {name}: {detail}")
        self.status = status


def _check(status: int, what: str):
    if status != CHORD_OK:
        raise ChordError(status, what)


def _ptr(t):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "device tensors must be contiguous CUDA tensors"
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def _routing_header(t):
    # num_tokens_padded holds two int32: the padded count and the routing tag
    assert t.dtype == torch.int32 and t.numel() >= 2, "num_tokens_padded must be an int32 tensor of 2 elements"
    return t


# --------------------------------------------------------------------------- sizes

def chord_moe_align_capacity(T, topk, E, block_m) -> int:
    return int(lib().chord_moe_align_capacity(T, topk, E, block_m))


def chord_moe_align_num_blocks(T, topk, E, block_m) -> int:
    return int(lib().chord_moe_align_num_blocks(T, topk, E, block_m))


def chord_moe_align_workspace_bytes(T, topk, E) -> int:
    return int(lib().chord_moe_align_workspace_bytes(T, topk, E))


def chord_repacked_bytes(E, N, K, group_size=32) -> int:
    return int(lib().chord_repacked_bytes(E, N, K, group_size))


def chord_select_block_m(T, topk, E_local, E_global, H, I) -> int:
    return int(lib().chord_select_block_m(T, topk, E_local, E_global, H, I))


def chord_moe_workspace_bytes(T, topk, E, H, I, block_m) -> int:
    return int(lib().chord_moe_workspace_bytes(T, topk, E, H, I, block_m))


def chord_status_string(status: int) -> str:
    return lib().chord_status_string(status).decode()


def chord_last_error_detail() -> str:
    return lib().chord_last_error_detail().decode()


# --------------------------------------------------------------------------- calls

def chord_moe_align(topk_ids, E, block_m, sorted_ids, expert_ids, num_tokens_padded,
                    expert_offsets=None, workspace=None, stream=None):
    T, topk = topk_ids.shape
    ws_bytes = 0 if workspace is None else _nbytes(workspace)
    _check(lib().chord_moe_align(_ptr(topk_ids), T, topk, E, block_m, _ptr(sorted_ids),
                                 _ptr(expert_ids), _ptr(_routing_header(num_tokens_padded)), _ptr(expert_offsets),
                                 _ptr(workspace), ws_bytes, _stream(stream)), "chord_moe_align")


def chord_moe_align_noalloc(topk_ids, E, block_m, sorted_ids, expert_ids, num_tokens_padded,
                            expert_offsets=None, stream=None):
    """chord_moe_align without a workspace: its scratch is a static device array in the
    library (for callers that cannot allocate device memory when they route)."""
    T, topk = topk_ids.shape
    _check(lib().chord_moe_align_noalloc(_ptr(topk_ids), T, topk, E, block_m, _ptr(sorted_ids),
                                         _ptr(expert_ids), _ptr(_routing_header(num_tokens_padded)),
                                         _ptr(expert_offsets), _stream(stream)),
           "chord_moe_align_noalloc")


def chord_router_topk_align(logits, topk, E, block_m, topk_ids, topk_weights, sorted_ids, expert_ids,
                            num_tokens_padded, expert_offsets=None, workspace=None, stream=None):
    """Top-k softmax router (fp32 logits [T, E_global] -> global topk_ids, renormalised
    topk_weights) fused with the routing sort over the local experts [0, E)."""
    T, E_global = logits.shape
    ws_bytes = 0 if workspace is None else _nbytes(workspace)
    _check(lib().chord_router_topk_align(_ptr(logits), T, E_global, topk, E, block_m, _ptr(topk_ids),
                                         _ptr(topk_weights), _ptr(sorted_ids), _ptr(expert_ids),
                                         _ptr(_routing_header(num_tokens_padded)), _ptr(expert_offsets), _ptr(workspace),
                                         ws_bytes, _stream(stream)), "chord_router_topk_align")


def chord_repack_weights(qweight, scales, role, out, group_size=32, stream=None):
    E, N, K8 = qweight.shape
    _check(lib().chord_repack_weights(_ptr(qweight), _ptr(scales), E, N, K8 * 8, group_size, role,
                                      _ptr(out), _nbytes(out), _stream(stream)),
           "chord_repack_weights")


def chord_dequant_weights(blob, w_out, stream=None):
    _check(lib().chord_dequant_weights(_ptr(blob), _nbytes(blob), _ptr(w_out), _stream(stream)),
           "chord_dequant_weights")


def chord_moe_forward(hidden, topk_ids, topk_weights, sorted_ids, expert_ids, num_tokens_padded,
                      block_m, w13, w2, I, E, out, workspace, flags=0, stream=None):
    T, H = hidden.shape
    topk = topk_ids.shape[1]
    _check(lib().chord_moe_forward(_ptr(hidden), _ptr(topk_ids), _ptr(topk_weights),
                                   _ptr(sorted_ids), _ptr(expert_ids), _ptr(_routing_header(num_tokens_padded)),
                                   block_m, _ptr(w13), _ptr(w2), T, H, I, E, topk, _ptr(out),
                                   _ptr(workspace), _nbytes(workspace), flags, _stream(stream)),
           "chord_moe_forward")


def chord_grouped_workspace_bytes(rows, E) -> int:
    return int(lib().chord_grouped_workspace_bytes(rows, E))


def chord_grouped_contiguous(x, m_indices, w, E, N, out, workspace, flags=0, stream=None):
    M, K = x.shape
    _check(lib().chord_grouped_contiguous(_ptr(x), M, K, _ptr(m_indices), _ptr(w), E, N, _ptr(out),
                                          _ptr(workspace), _nbytes(workspace), flags, _stream(stream)),
           "chord_grouped_contiguous")


def chord_grouped_masked(x, masked_m, expected_m, w, N, out, workspace, flags=0, stream=None):
    E = masked_m.shape[0]
    K = x.shape[-1]
    max_m = x.shape[1] if x.dim() == 3 else x.shape[0] // E  # [E, max_m, K] or [E * max_m, K]
    _check(lib().chord_grouped_masked(_ptr(x), E, max_m, K, _ptr(masked_m), int(expected_m), _ptr(w), N,
                                      _ptr(out), _ptr(workspace), _nbytes(workspace), flags, _stream(stream)),
           "chord_grouped_masked")


def chord_ep_plan_workspace_bytes(T, W) -> int:
    return int(lib().chord_ep_plan_workspace_bytes(T, W))


def chord_ep_plan(topk_ids, E_rank, W, send_rows, rank_offsets, row_of, workspace, stream=None):
    """Expert-parallel send plan: one row per (token, rank owning >= 1 of its experts),
    grouped by rank; rank_offsets [W+1]; row_of [T*W] reset to -1."""
    T, topk = topk_ids.shape
    _check(lib().chord_ep_plan(_ptr(topk_ids), T, topk, E_rank, W, _ptr(send_rows), _ptr(rank_offsets), _ptr(row_of),
                               _ptr(workspace), _nbytes(workspace), _stream(stream)), "chord_ep_plan")


def chord_ep_pack(hidden, topk_ids, topk_weights, E_rank, W, send_rows, rank_offsets, row_of, send_x, send_ids,
                  send_w, stream=None):
    T, H = hidden.shape
    topk = topk_ids.shape[1]
    _check(lib().chord_ep_pack(_ptr(hidden), _ptr(topk_ids), _ptr(topk_weights), T, H, topk, E_rank, W,
                               _ptr(send_rows), _ptr(rank_offsets), _ptr(row_of), _ptr(send_x), _ptr(send_ids),
                               _ptr(send_w), _stream(stream)), "chord_ep_pack")


def chord_ep_combine(back, row_of, W, out, stream=None):
    T, H = out.shape
    _check(lib().chord_ep_combine(_ptr(back) if back.numel() else None, _ptr(row_of), T, H, W, _ptr(out),
                                  _stream(stream)), "chord_ep_combine")


def chord_round_bf16(x_f32, out_bf16, stream=None):
    assert x_f32.dtype == torch.float32 and x_f32.numel() == out_bf16.numel()
    _check(lib().chord_round_bf16(_ptr(x_f32), x_f32.numel(), _ptr(out_bf16), _stream(stream)), "chord_round_bf16")


def chord_tp_reduce_round(partials, outs, rank, stream=None):
    """Rank `rank`'s slice of the tensor-parallel all-reduce of the FP32 `partials` (one
    tensor per rank, readable from this device), rounded to BF16 and stored into every
    rank's tensor in `outs`."""
    W = len(partials)
    assert W == len(outs) and all(p.dtype == torch.float32 and p.numel() == partials[0].numel() for p in partials)
    assert all(o.numel() == partials[0].numel() for o in outs)
    ins = (ctypes.c_void_p * W)(*[p.data_ptr() for p in partials])
    ous = (ctypes.c_void_p * W)(*[o.data_ptr() for o in outs])
    _check(lib().chord_tp_reduce_round(ins, ous, W, rank, partials[0].numel(), _stream(stream)), "chord_tp_reduce_round")


def chord_moe_check_status(workspace, stream=None) -> int:
    v = ctypes.c_uint32(0)
    st = lib().chord_moe_check_status(_ptr(workspace), _stream(stream), ctypes.byref(v))
    if st not in (CHORD_OK, CHORD_ERR_DEVICE):
        _check(st, "chord_moe_check_status")
    return int(v.value)


def chord_set_timing_events(events=None):
    """events: four torch.cuda.Event (already recorded once, so their handles exist) or None."""
    if not events:
        _check(lib().chord_set_timing_events(None, 0), "chord_set_timing_events")
        return
    arr = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(lib().chord_set_timing_events(arr, 4), "chord_set_timing_events")


def chord_launch_count() -> int:
    return int(lib().chord_launch_count())


def chord_selftest_wait_timeout(status, elapsed_ns, limit_us: int, stream=None):
    """status: int32 device tensor [1] (OR-ed); elapsed_ns: int64 device tensor [2]."""
    _check(lib().chord_selftest_wait_timeout(_ptr(status), _ptr(elapsed_ns), ctypes.c_uint32(limit_us),
                                             _stream(stream)), "chord_selftest_wait_timeout")


# --------------------------------------------------------------------------- convenience

def _alloc_bytes(n: int, device) -> torch.Tensor:
    # 256-byte alignment: the torch caching allocator returns 512-byte aligned blocks
    t = torch.empty(max(n, 1), dtype=torch.uint8, device=device)
    assert t.data_ptr() % 256 == 0
    return t


class ChordMoE:
    """A prepared layer: repacked weights plus reusable routing and workspace buffers.

    Buffers are sized for up to ``max_tokens`` tokens; call with any T <= max_tokens.
    ``block_m`` defaults to the library's selector for ``max_tokens``.
    """

    def __init__(self, qw13, s13, qw2, s2, topk, E_global=None, max_tokens=1, block_m=None,
                 device="cuda"):
        E, N13, H8 = qw13.shape
        self.E, self.I, self.H, self.topk = E, N13 // 2, H8 * 8, topk
        self.E_global = E if E_global is None else E_global
        self.device = torch.device(device)
        self.w13 = _alloc_bytes(chord_repacked_bytes(E, N13, self.H), self.device)
        self.w2 = _alloc_bytes(chord_repacked_bytes(E, self.H, self.I), self.device)
        dev = lambda a: torch.as_tensor(a).to(self.device).contiguous()  # noqa: E731
        chord_repack_weights(dev(qw13), dev(s13), CHORD_ROLE_GATE_UP, self.w13)
        chord_repack_weights(dev(qw2), dev(s2), CHORD_ROLE_DOWN, self.w2)
        torch.cuda.current_stream().synchronize()
        self.max_tokens = 0
        self.block_m = block_m
        self.reserve(max_tokens)

    def reserve(self, T: int, block_m=None):
        if block_m is not None:
            self.block_m = block_m
        elif self.block_m is None:
            self.block_m = chord_select_block_m(T, self.topk, self.E, self.E_global, self.H, self.I)
        bm = self.block_m
        cap = chord_moe_align_capacity(T, self.topk, self.E, bm)
        nb = chord_moe_align_num_blocks(T, self.topk, self.E, bm)
        d = self.device
        self.sorted_ids = torch.empty(max(cap, 1), dtype=torch.int32, device=d)
        self.expert_ids = torch.empty(max(nb, 1), dtype=torch.int32, device=d)
        self.ntp = torch.zeros(2, dtype=torch.int32, device=d)  # padded count, routing tag
        self.offsets = torch.empty(self.E + 1, dtype=torch.int32, device=d)
        aw = chord_moe_align_workspace_bytes(T, self.topk, self.E)
        self.align_ws = _alloc_bytes(aw, d) if aw else None
        self.workspace = torch.zeros(chord_moe_workspace_bytes(T, self.topk, self.E, self.H, self.I, bm),
                                     dtype=torch.uint8, device=d)
        self.max_tokens = T

    def align(self, topk_ids):
        chord_moe_align(topk_ids, self.E, self.block_m, self.sorted_ids, self.expert_ids, self.ntp,
                        self.offsets, self.align_ws)

    def forward(self, hidden, topk_ids, topk_weights, out=None, flags=0):
        T = hidden.shape[0]
        if T > self.max_tokens:
            self.reserve(T)
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.bfloat16, device=self.device)
        self.align(topk_ids)
        chord_moe_forward(hidden, topk_ids, topk_weights, self.sorted_ids, self.expert_ids, self.ntp,
                          self.block_m, self.w13, self.w2, self.I, self.E, out, self.workspace, flags)
        return out

    __call__ = forward

    def check_status(self) -> int:
        return chord_moe_check_status(self.workspace)


class GroupedWeight:
    """A weight prepared for one grouped operator ("Gruppierte Operatoreintrittspunkte":
    the mode is part of the prepared weight and checked when the operator runs).

    qweight int32 [E, N, K/8] (eight codes per word, low nibble first), scales bf16 bits
    [E, N, K/32]; mode "contiguous" or "masked". Keeps a workspace for its calls.
    """

    def __init__(self, qweight, scales, mode, device="cuda"):
        roles = {"contiguous": CHORD_ROLE_GROUPED_CONTIGUOUS, "masked": CHORD_ROLE_GROUPED_MASKED}
        if mode not in roles:
            raise ValueError(f"mode must be 'contiguous' or 'masked', not {mode!r}")
        self.mode, self.role = mode, roles[mode]
        self.E, self.N, K8 = qweight.shape
        self.K = K8 * 8
        self.device = torch.device(device)
        self.blob = _alloc_bytes(chord_repacked_bytes(self.E, self.N, self.K), self.device)
        dev = lambda a: torch.as_tensor(a).to(self.device).contiguous()  # noqa: E731
        chord_repack_weights(dev(qweight), dev(scales), self.role, self.blob)
        self.workspace = None

    def _workspace(self, rows):
        need = chord_grouped_workspace_bytes(rows, self.E)
        if self.workspace is None or self.workspace.numel() < need:
            self.workspace = torch.zeros(max(need, 1), dtype=torch.uint8, device=self.device)
        return self.workspace

    def check_status(self) -> int:
        return 0 if self.workspace is None else chord_moe_check_status(self.workspace)


def pack_w4a16_grouped(qweight, scales, mode, device="cuda") -> GroupedWeight:
    return GroupedWeight(qweight, scales, mode, device)


def contiguous(a2, weight: GroupedWeight, m_indices, out=None, flags=0):
    """out [M, N] bf16 for rows grouped by expert (m_indices: expert or -1 per row)."""
    M = a2.shape[0]
    if out is None:
        out = torch.empty((M, weight.N), dtype=torch.bfloat16, device=a2.device)
    chord_grouped_contiguous(a2, m_indices, weight.blob, weight.E, weight.N, out, weight._workspace(M), flags)
    return out


def masked(a3, weight: GroupedWeight, masked_m, expected_m, out=None, flags=0):
    """out [E * max_m, N] bf16 (flat); rows past masked_m[e] in each expert are not written.
    a3 is [E, max_m, K] or [E * max_m, K]."""
    E = weight.E
    max_m = a3.shape[1] if a3.dim() == 3 else a3.shape[0] // E
    if out is None:
        out = torch.empty((E * max_m, weight.N), dtype=torch.bfloat16, device=a3.device)
    chord_grouped_masked(a3, masked_m, expected_m, weight.blob, weight.N, out, weight._workspace(E * max_m), flags)
    return out
