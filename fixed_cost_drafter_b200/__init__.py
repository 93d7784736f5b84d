"""Python binding of the LongSpark fixed-cost drafting round (C ABI: include/longspark.h).

Argument marshalling only: every function forwards to the entry point of the same name
in ``liblongspark.so``; every step of the path runs in the library's CUDA kernels.
Device buffers may be given as torch tensors (their ``data_ptr()`` is passed) or as raw
integer addresses; streams as ``torch.cuda.Stream`` or raw handles. A non-zero status
raises :class:`LsError`. There is no fallback: if the library is missing, importing this
package raises.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liblongspark.so")

LS_OK = 0
LS_ERR_INVALID_ARG = -1
LS_ERR_SHAPE = -2
LS_ERR_UNSUPPORTED = -3
LS_ERR_CUDA = -4
LS_ERR_DEVICE = -5
LS_ERR_DEVICE_TIMEOUT = -6
LS_ERR_SCRATCH_LIMIT = -7
LS_DEVERR_PREFIX_LEN = 0x1
LS_DEVERR_WAIT_TIMEOUT = 0x2
LS_DEVERR_ORDER = 0x4
LS_DEVERR_SAMPLE = 0x8
LS_DEVERR_PAGE = 0x10
LS_MAX_PAGED_LAYERS = 64
LS_F32 = 0
LS_BF16 = 1
LS_FLAG_FORCE_SIMT = 0x1
LS_FLAG_OUT_F32 = 0x2
LS_MAX_SCALES = 4
LS_VIEW_BOUNDARY = 0x1
LS_VIEW_WINDOW = 0x2
LS_VIEW_SUMMARY = 0x4
LS_VIEW_ALL = 0x7
LS_ATTEND_INPUTS_READY = 0x100

EXPORTED = (
    "ls_state_bytes", "ls_get_layout", "ls_init_state", "ls_prefill_workspace_bytes",
    "ls_prefill_summary", "ls_prefill_summary_noalloc", "ls_commit_round", "ls_draft_attend",
    "ls_draft_attend_views", "ls_view_state_bytes", "ls_round", "ls_accept_sampled", "ls_commit_accepted",
    "ls_draft_prologue", "ls_prefill_paged", "ls_commit_round_paged", "ls_commit_accepted_paged", "ls_round_paged",
    "ls_clear_error", "ls_check_wait_timeout", "ls_round_overlaps", "ls_attend_uses_tensor_cores",
    "ls_read_state", "ls_get_error", "ls_destroy_state", "ls_status_string",
)


class LsError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} failed: {status} ({ls_status_string(status)})")
        self.status = status


class ls_config(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("n_layers", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("hidden", ctypes.c_int32),
        ("block", ctypes.c_int32), ("window", ctypes.c_int32), ("n_scales", ctypes.c_int32),
        ("scales", ctypes.c_int32 * LS_MAX_SCALES), ("slots_per_scale", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("flags", ctypes.c_int32),
    ]


class ls_layout(ctypes.Structure):
    _fields_ = [
        ("total_bytes", ctypes.c_size_t), ("off_counters", ctypes.c_size_t),
        ("off_error", ctypes.c_size_t), ("off_sync", ctypes.c_size_t), ("off_kv", ctypes.c_size_t),
        ("off_seg_mean", ctypes.c_size_t), ("off_part_sum", ctypes.c_size_t),
        ("off_glob_sum", ctypes.c_size_t), ("off_boundary", ctypes.c_size_t),
        ("kv_rows", ctypes.c_int32), ("elem_bytes", ctypes.c_int32), ("off_sample", ctypes.c_size_t),
        ("off_prologue", ctypes.c_size_t),
    ]


class ls_paged_kv(ctypes.Structure):
    """A target's paged KV cache: per tapped layer the base of its key and value pages;
    element (page, offset, h, d) at base[page * page_stride + offset * slot_stride + h * D + d];
    position p of sequence b in page block_table[b][p // page_size] at offset p % page_size."""
    _fields_ = [
        ("k_layers", ctypes.c_void_p * LS_MAX_PAGED_LAYERS), ("v_layers", ctypes.c_void_p * LS_MAX_PAGED_LAYERS),
        ("page_stride", ctypes.c_int64), ("slot_stride", ctypes.c_int64), ("block_table", ctypes.c_void_p),
        ("max_blocks", ctypes.c_int32), ("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int64),
        ("verify_slots", ctypes.c_void_p),
    ]


def make_paged_kv(k_layers, v_layers, page_stride, slot_stride, block_table, max_blocks, page_size,
                  num_pages, verify_slots=None) -> ls_paged_kv:
    """Descriptor from per-layer page buffers (tensors or addresses), an int32 block table and,
    optionally, the verify rows' int64 slots [b][B+1]."""
    if len(k_layers) != len(v_layers) or len(k_layers) > LS_MAX_PAGED_LAYERS:
        raise ValueError("one key and one value page buffer per tapped layer, at most LS_MAX_PAGED_LAYERS")
    kv = ls_paged_kv()
    for l, (k, v) in enumerate(zip(k_layers, v_layers)):
        kv.k_layers[l] = _ptr(k)
        kv.v_layers[l] = _ptr(v)
    kv.page_stride, kv.slot_stride = page_stride, slot_stride
    kv.block_table = _ptr(block_table)
    kv.max_blocks, kv.page_size, kv.num_pages = max_blocks, page_size, num_pages
    kv.verify_slots = _ptr(verify_slots)
    return kv


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with __graft_entry__.build()")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    cfgp = ctypes.POINTER(ls_config)
    pkvp = ctypes.POINTER(ls_paged_kv)
    sig = {
        "ls_prefill_paged": (ctypes.c_int, [vp, pkvp, vp, i64, i64, vp, vp, sz, vp]),
        "ls_commit_round_paged": (ctypes.c_int, [vp, vp, vp, pkvp, vp, vp, vp, vp]),
        "ls_commit_accepted_paged": (ctypes.c_int, [vp, vp, pkvp, vp, vp]),
        "ls_round_paged": (ctypes.c_int, [vp, vp, vp, pkvp, vp, vp, vp, vp, i64, i64, ctypes.c_float, vp, vp]),
        "ls_state_bytes": (sz, [cfgp]),
        "ls_view_state_bytes": (sz, [cfgp, i32]),
        "ls_accept_sampled": (ctypes.c_int, [vp, vp, vp, vp, i32, vp, vp, vp, vp]),
        "ls_commit_accepted": (ctypes.c_int, [vp, vp, vp, vp, vp, vp]),
        "ls_draft_prologue": (ctypes.c_int, [vp, vp, vp, vp, vp, vp, vp]),
        "ls_get_layout": (ctypes.c_int, [cfgp, ctypes.POINTER(ls_layout)]),
        "ls_init_state": (ctypes.c_int, [cfgp, vp, sz, ctypes.POINTER(vp), vp]),
        "ls_prefill_workspace_bytes": (sz, [cfgp, i64, i64]),
        "ls_prefill_summary": (ctypes.c_int, [vp, vp, vp, i64, i64, vp, i64, i64, vp, vp, sz, vp]),
        "ls_prefill_summary_noalloc": (ctypes.c_int, [vp, vp, vp, i64, i64, vp, i64, i64, vp, vp]),
        "ls_commit_round": (ctypes.c_int, [vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "ls_draft_attend": (ctypes.c_int, [vp, i32, i32, vp, vp, vp, i64, ctypes.c_float, vp, vp]),
        "ls_draft_attend_views": (ctypes.c_int, [vp, i32, i32, vp, vp, vp, i64, ctypes.c_float, i32, vp, vp]),
        "ls_round": (ctypes.c_int, [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, ctypes.c_float, vp, vp]),
        "ls_round_overlaps": (ctypes.c_int, [vp]),
        "ls_clear_error": (ctypes.c_int, [vp, vp]),
        "ls_check_wait_timeout": (ctypes.c_int, [vp, ctypes.c_uint32, vp]),
        "ls_attend_uses_tensor_cores": (ctypes.c_int, [vp]),
        "ls_read_state": (ctypes.c_int, [vp, vp, sz, vp]),
        "ls_get_error": (ctypes.c_int, [vp, ctypes.POINTER(i32)]),
        "ls_destroy_state": (None, [vp]),
        "ls_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def library_path() -> str:
    return _LIB_PATH


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    raise TypeError(f"expected a tensor or an address, got {type(x)}")


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(fn, status):
    if status != LS_OK:
        raise LsError(fn, status)


def make_config(batch, n_layers, n_kv_heads, n_q_heads, head_dim, hidden, block, window, scales,
                slots_per_scale, dtype=LS_BF16, flags=0) -> ls_config:
    c = ls_config()
    c.batch, c.n_layers, c.n_kv_heads, c.n_q_heads = batch, n_layers, n_kv_heads, n_q_heads
    c.head_dim, c.hidden, c.block, c.window = head_dim, hidden, block, window
    c.n_scales = len(scales)
    for i, s in enumerate(scales):
        c.scales[i] = s
    c.slots_per_scale, c.dtype, c.flags = slots_per_scale, dtype, flags
    return c


def ls_status_string(status: int) -> str:
    return _lib.ls_status_string(status).decode()


def ls_state_bytes(cfg: ls_config) -> int:
    return int(_lib.ls_state_bytes(ctypes.byref(cfg)))


def ls_view_state_bytes(cfg: ls_config, views: int) -> int:
    return int(_lib.ls_view_state_bytes(ctypes.byref(cfg), views))


def ls_get_layout(cfg: ls_config) -> ls_layout:
    out = ls_layout()
    _check("ls_get_layout", _lib.ls_get_layout(ctypes.byref(cfg), ctypes.byref(out)))
    return out


def ls_init_state(cfg: ls_config, arena, arena_bytes: int, stream=None) -> int:
    """Returns the opaque state handle (an address)."""
    h = ctypes.c_void_p()
    _check("ls_init_state", _lib.ls_init_state(ctypes.byref(cfg), _ptr(arena), arena_bytes,
                                               ctypes.byref(h), _stream(stream)))
    return h.value


def ls_prefill_workspace_bytes(cfg: ls_config, row_begin: int, row_end: int) -> int:
    return int(_lib.ls_prefill_workspace_bytes(ctypes.byref(cfg), row_begin, row_end))


def ls_prefill_summary(state, k, v, plane_stride, row_stride, prefix_len, row_begin, row_end,
                       last_hidden, workspace, workspace_bytes, stream=None) -> None:
    _check("ls_prefill_summary", _lib.ls_prefill_summary(
        state, _ptr(k), _ptr(v), plane_stride, row_stride, _ptr(prefix_len), row_begin, row_end,
        _ptr(last_hidden), _ptr(workspace), workspace_bytes, _stream(stream)))


def ls_prefill_summary_noalloc(state, k, v, plane_stride, row_stride, prefix_len, row_begin, row_end,
                               last_hidden, stream=None) -> None:
    """ls_prefill_summary without a workspace argument: the library's fixed 16 MiB scratch
    is used instead, for callers that cannot allocate device memory."""
    _check("ls_prefill_summary_noalloc", _lib.ls_prefill_summary_noalloc(
        state, _ptr(k), _ptr(v), plane_stride, row_stride, _ptr(prefix_len), row_begin, row_end,
        _ptr(last_hidden), _stream(stream)))


def ls_commit_round(state, draft_ids, target_ids, verify_k, verify_v, verify_hidden, accept_len,
                    next_token, stream=None) -> None:
    _check("ls_commit_round", _lib.ls_commit_round(
        state, _ptr(draft_ids), _ptr(target_ids), _ptr(verify_k), _ptr(verify_v),
        _ptr(verify_hidden), _ptr(accept_len), _ptr(next_token), _stream(stream)))


def ls_draft_attend(state, layer_begin, layer_count, q, boundary_k, boundary_v, boundary_stride,
                    softmax_scale, out, stream=None) -> None:
    _check("ls_draft_attend", _lib.ls_draft_attend(
        state, layer_begin, layer_count, _ptr(q), _ptr(boundary_k), _ptr(boundary_v),
        boundary_stride, float(softmax_scale), _ptr(out), _stream(stream)))


def ls_draft_attend_views(state, layer_begin, layer_count, q, boundary_k, boundary_v, boundary_stride,
                          softmax_scale, views, out, stream=None) -> None:
    _check("ls_draft_attend_views", _lib.ls_draft_attend_views(
        state, layer_begin, layer_count, _ptr(q), _ptr(boundary_k), _ptr(boundary_v),
        boundary_stride, float(softmax_scale), views, _ptr(out), _stream(stream)))


def ls_accept_sampled(state, draft_ids, draft_probs, target_probs, vocab, uniforms, accept_len, next_token,
                      stream=None) -> None:
    _check("ls_accept_sampled", _lib.ls_accept_sampled(
        state, _ptr(draft_ids), _ptr(draft_probs), _ptr(target_probs), vocab, _ptr(uniforms), _ptr(accept_len),
        _ptr(next_token), _stream(stream)))


def ls_draft_prologue(state, w_kv, w_q, x, bkv, q, stream=None) -> None:
    _check("ls_draft_prologue", _lib.ls_draft_prologue(
        state, _ptr(w_kv), _ptr(w_q), _ptr(x), _ptr(bkv), _ptr(q), _stream(stream)))


def ls_commit_accepted(state, accept_len, verify_k, verify_v, verify_hidden, stream=None) -> None:
    _check("ls_commit_accepted", _lib.ls_commit_accepted(
        state, _ptr(accept_len), _ptr(verify_k), _ptr(verify_v), _ptr(verify_hidden), _stream(stream)))


def ls_round(state, draft_ids, target_ids, verify_k, verify_v, verify_hidden, accept_len, next_token, q,
             boundary_k_offset, boundary_v_offset, softmax_scale, out, stream=None) -> None:
    _check("ls_round", _lib.ls_round(
        state, _ptr(draft_ids), _ptr(target_ids), _ptr(verify_k), _ptr(verify_v), _ptr(verify_hidden),
        _ptr(accept_len), _ptr(next_token), _ptr(q), boundary_k_offset, boundary_v_offset,
        float(softmax_scale), _ptr(out), _stream(stream)))


def ls_prefill_paged(state, kv: ls_paged_kv, prefix_len, row_begin, row_end, last_hidden, workspace=None,
                     workspace_bytes=0, stream=None) -> None:
    """Prefill reading the prefix from the paged cache; workspace None uses the library's fixed scratch."""
    _check("ls_prefill_paged", _lib.ls_prefill_paged(
        state, ctypes.byref(kv), _ptr(prefix_len), row_begin, row_end, _ptr(last_hidden), _ptr(workspace),
        workspace_bytes, _stream(stream)))


def ls_commit_round_paged(state, draft_ids, target_ids, kv: ls_paged_kv, verify_hidden, accept_len, next_token,
                          stream=None) -> None:
    _check("ls_commit_round_paged", _lib.ls_commit_round_paged(
        state, _ptr(draft_ids), _ptr(target_ids), ctypes.byref(kv), _ptr(verify_hidden), _ptr(accept_len),
        _ptr(next_token), _stream(stream)))


def ls_commit_accepted_paged(state, accept_len, kv: ls_paged_kv, verify_hidden, stream=None) -> None:
    _check("ls_commit_accepted_paged", _lib.ls_commit_accepted_paged(
        state, _ptr(accept_len), ctypes.byref(kv), _ptr(verify_hidden), _stream(stream)))


def ls_round_paged(state, draft_ids, target_ids, kv: ls_paged_kv, verify_hidden, accept_len, next_token, q,
                   boundary_k_offset, boundary_v_offset, softmax_scale, out, stream=None) -> None:
    _check("ls_round_paged", _lib.ls_round_paged(
        state, _ptr(draft_ids), _ptr(target_ids), ctypes.byref(kv), _ptr(verify_hidden), _ptr(accept_len),
        _ptr(next_token), _ptr(q), boundary_k_offset, boundary_v_offset, float(softmax_scale), _ptr(out),
        _stream(stream)))


def ls_round_overlaps(state) -> bool:
    return bool(_lib.ls_round_overlaps(state))


def ls_attend_uses_tensor_cores(state) -> bool:
    return bool(_lib.ls_attend_uses_tensor_cores(state))


def ls_read_state(state, host_dst, nbytes, stream=None) -> None:
    _check("ls_read_state", _lib.ls_read_state(state, _ptr(host_dst), nbytes, _stream(stream)))


def ls_get_error(state) -> tuple[int, int]:
    """(status, device error word). Synchronises the device."""
    code = ctypes.c_int32(0)
    st = _lib.ls_get_error(state, ctypes.byref(code))
    return st, code.value


def ls_clear_error(state, stream=None) -> None:
    _check("ls_clear_error", _lib.ls_clear_error(state, _stream(stream)))


def ls_check_wait_timeout(state, polls, stream=None) -> None:
    """One bounded wait that nothing signals: sets LS_DEVERR_WAIT_TIMEOUT (see the header)."""
    _check("ls_check_wait_timeout", _lib.ls_check_wait_timeout(state, polls, _stream(stream)))


def ls_destroy_state(state) -> None:
    _lib.ls_destroy_state(state)
