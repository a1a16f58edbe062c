"""ctypes binding of the C ABI in include/pa.h (argument marshalling only).

Every function here has the name of the C entry point it calls. Tensors are
torch CUDA tensors (PyTorch only provides device memory and streams); all
computation happens in the sm_100a kernels of libpa_b200.so. Importing this
module fails loudly when the library is missing -- there is no CPU fallback.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpa_b200.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"CUDA library {_LIB_PATH} is not built: run "
                      "`python -m paged_kv_cache_399_b200.build` (there is no CPU fallback)")
_lib = ctypes.CDLL(_LIB_PATH)

PA_OK = 0
PA_ERR_INVALID_ARG = 1
PA_ERR_UNSUPPORTED = 2
PA_ERR_WORKSPACE = 3
PA_ERR_OUT_OF_RANGE = 4
PA_ERR_CUDA = 5
PA_ERR_DEVICE = 6

PA_PATH_AUTO = 0
PA_PATH_SINGLE = 1
PA_PATH_TILE = 2
PA_PATH_TCGEN05 = 3

EXPORTED = ["pa_reshape_and_cache", "pa_decode_plan", "pa_decode_workspace_size", "pa_decode", "pa_decode_fp8",
            "pa_prefill", "pa_decode_partial", "pa_decode_partial_pieces", "pa_combine_partials",
            "pa_merge_partials",
            "pa_decode_static_scratch", "pa_validate", "pa_get_device_error",
            "pa_selftest_bounded_wait", "pa_copy_blocks", "pa_reshape_and_cache_fp8", "pa_status_string",
            "pa_version"]

PA_STATIC_SCRATCH_BYTES = 16 * 1024 * 1024


PA_SCHEDULE_AUTO = 0
PA_SCHEDULE_GRID = 1
PA_SCHEDULE_PERSISTENT = 2

PA_KV_BF16 = 0
PA_KV_FP8_E4M3 = 1


class pa_plan_hints_t(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("schedule", ctypes.c_int32),
                ("split_blocks", ctypes.c_int32), ("share_prefix", ctypes.c_int32),
                ("sliding_window", ctypes.c_int32), ("kv_cache_dtype", ctypes.c_int32)]


class pa_plan_t(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("schedule", ctypes.c_int32),
                ("split_blocks", ctypes.c_int32), ("num_splits", ctypes.c_int32),
                ("rows_per_cta", ctypes.c_int32), ("num_ctas", ctypes.c_int32),
                ("share_cap", ctypes.c_int32), ("share_split_blocks", ctypes.c_int32),
                ("sliding_window", ctypes.c_int32), ("kv_cache_dtype", ctypes.c_int32)]

    def as_dict(self) -> dict:
        return {"path": {1: "single", 2: "tile", 3: "tcgen05"}.get(self.path, self.path),
                "schedule": {1: "grid", 2: "persistent"}.get(self.schedule, self.schedule),
                "split_blocks": self.split_blocks, "num_splits": self.num_splits,
                "rows_per_cta": self.rows_per_cta, "num_ctas": self.num_ctas,
                "share_cap": self.share_cap, "share_split_blocks": self.share_split_blocks,
                "sliding_window": self.sliding_window,
                "kv_cache_dtype": {0: "bf16", 1: "fp8_e4m3"}.get(self.kv_cache_dtype, self.kv_cache_dtype)}

    def __repr__(self):
        return f"pa_plan_t({self.as_dict()})"


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64

_lib.pa_reshape_and_cache_fp8.restype = _I32
_lib.pa_reshape_and_cache_fp8.argtypes = [_P, _P, _I64, _I64, _P, _P, _P, _I64, _I32, _I32, _I64, _I32,
                                          ctypes.c_float, ctypes.c_float, _P]
_lib.pa_copy_blocks.restype = _I32
_lib.pa_copy_blocks.argtypes = [_P, _P, _I64, _I32, _I32, _I32, _P, _I64, _P]
_lib.pa_reshape_and_cache.restype = _I32
_lib.pa_reshape_and_cache.argtypes = [_P, _P, _I64, _I64, _P, _P, _P, _I64, _I32, _I32, _I64, _I32, _P]
_lib.pa_decode_plan.restype = _I32
_lib.pa_decode_plan.argtypes = [_I32, _I32, _I32, _I32, _I32, _I32, ctypes.POINTER(pa_plan_hints_t),
                                ctypes.POINTER(pa_plan_t)]
_lib.pa_decode_workspace_size.restype = ctypes.c_size_t
_lib.pa_decode_workspace_size.argtypes = [ctypes.POINTER(pa_plan_t), _I32, _I32, _I32, _I32, _I32, _I32]
_lib.pa_decode.restype = _I32
_lib.pa_decode.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _I64,
                           ctypes.c_float, ctypes.POINTER(pa_plan_t), _P, ctypes.c_size_t, _P]
_lib.pa_decode_fp8.restype = _I32
_lib.pa_decode_fp8.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _I64,
                               ctypes.c_float, ctypes.c_float, ctypes.c_float, ctypes.POINTER(pa_plan_t), _P,
                               ctypes.c_size_t, _P]
_lib.pa_prefill.restype = _I32
_lib.pa_prefill.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _I64,
                            ctypes.c_float, _P]
_lib.pa_decode_partial.restype = _I32
_lib.pa_decode_partial.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _I64,
                                   ctypes.c_float, _I32, _I32, _I32, _P]
_lib.pa_decode_partial_pieces.restype = _I32
_lib.pa_decode_partial_pieces.argtypes = [_I32, _I32, _I32, _I32, _I32, _I32]
_lib.pa_combine_partials.restype = _I32
_lib.pa_combine_partials.argtypes = [_P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _P]
_lib.pa_merge_partials.restype = _I32
_lib.pa_merge_partials.argtypes = [_P, _P, _P, _I32, _I32, _I32, _I32, _I32, _P]
_lib.pa_decode_static_scratch.restype = _I32
_lib.pa_decode_static_scratch.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32,
                                          _I32, _I64, ctypes.c_float, ctypes.POINTER(pa_plan_t), _P]
_lib.pa_validate.restype = _I32
_lib.pa_validate.argtypes = [_P, _P, _P, _I32, _I32, _I32, _I64, _I64, _I32, ctypes.POINTER(_I64), _P]
_lib.pa_get_device_error.restype = _I32
_lib.pa_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), _I32, _P]
_lib.pa_selftest_bounded_wait.argtypes = [_P]
_lib.pa_selftest_bounded_wait.restype = _I32
_lib.pa_status_string.restype = ctypes.c_char_p
_lib.pa_status_string.argtypes = [_I32]
_lib.pa_version.restype = _I32
_lib.pa_version.argtypes = []


class PAError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {pa_status_string(status)}")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def pa_status_string(status: int) -> str:
    return _lib.pa_status_string(status).decode()


def pa_version() -> int:
    return _lib.pa_version()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _check(status: int, where: str) -> None:
    if status != PA_OK:
        raise PAError(status, where)


# The per-step calls below (cache write, decode) check dtypes and layouts with as few calls
# into torch as they can: their host time sits between a step's kernels.
_BF16, _U8, _INT32, _INT64 = torch.bfloat16, torch.uint8, torch.int32, torch.int64


def _require(ok: bool, what: str) -> None:
    if not ok:
        raise ValueError(what)


def _decode_args(out, query, key_cache, value_cache, block_tables, context_lens, q_per_seq, cache_dtype, where):
    """The C arguments of pa_decode(_fp8) up to num_blocks, after the layout checks."""
    if not (out.dtype is _BF16 and query.dtype is _BF16 and key_cache.dtype is cache_dtype and
            value_cache.dtype is cache_dtype and block_tables.dtype is _INT32 and context_lens.dtype is _INT32):
        raise TypeError(f"{where}: out/query bf16, caches {cache_dtype}, block_tables/context_lens int32")
    _require(out.is_contiguous() and query.is_contiguous() and key_cache.is_contiguous() and
             value_cache.is_contiguous() and block_tables.is_contiguous() and context_lens.is_contiguous(),
             f"{where}: every tensor must be contiguous")
    B, QS, HQ, D = query.shape
    _require(QS == q_per_seq and out.shape == query.shape, f"{where}: out/query [B, q_per_seq, H_q, D]")
    NB, BS, HKV = key_cache.shape[:3]
    return (out.data_ptr(), query.data_ptr(), key_cache.data_ptr(), value_cache.data_ptr(),
            block_tables.data_ptr(), context_lens.data_ptr(), B, QS, HQ, HKV, D, BS, block_tables.shape[1], NB)


def pa_reshape_and_cache(key: torch.Tensor, value: torch.Tensor, key_cache: torch.Tensor,
                         value_cache: torch.Tensor, slot_mapping: torch.Tensor,
                         stream=None) -> None:
    """key/value [T, H_kv, D] bf16 (token stride may exceed H_kv*D); caches
    [NB, 16, H_kv, D] bf16; slot_mapping [T] int64."""
    if not (key.dtype is _BF16 and value.dtype is _BF16 and key_cache.dtype is _BF16 and
            value_cache.dtype is _BF16 and slot_mapping.dtype is _INT64):
        raise TypeError("pa_reshape_and_cache: key/value/caches bf16, slot_mapping int64")
    T, H, D = key.shape
    ks, vs = key.stride(), value.stride()
    _require(ks[2] == 1 and ks[1] == D and vs[2] == 1 and vs[1] == D and value.shape == key.shape and
             slot_mapping.is_contiguous() and key_cache.is_contiguous() and value_cache.is_contiguous(),
             "pa_reshape_and_cache: rows of key/value contiguous, caches and slot_mapping contiguous")
    NB, BS = key_cache.shape[:2]
    st = _lib.pa_reshape_and_cache(key.data_ptr(), value.data_ptr(), ks[0], vs[0], key_cache.data_ptr(),
                                   value_cache.data_ptr(), slot_mapping.data_ptr(), T, H, D, NB, BS,
                                   _stream(stream))
    _check(st, "pa_reshape_and_cache")


def pa_copy_blocks(key_cache: torch.Tensor, value_cache: torch.Tensor, block_mapping,
                   stream=None) -> None:
    """Copy-on-write block copy. Caches [NB, 16, H_kv, D] bf16 on the device;
    block_mapping [n, 2] int64 {source, destination} block ids, a HOST array (CPU tensor
    or numpy), read during the call."""
    assert key_cache.dtype == value_cache.dtype == torch.bfloat16
    assert key_cache.is_contiguous() and value_cache.is_contiguous()
    assert key_cache.shape == value_cache.shape
    if isinstance(block_mapping, torch.Tensor):
        assert block_mapping.device.type == "cpu", "block_mapping is a host array"
        block_mapping = block_mapping.numpy()
    m = np.ascontiguousarray(np.asarray(block_mapping, dtype=np.int64).reshape(-1, 2))
    NB, BS, H, D = key_cache.shape
    st = _lib.pa_copy_blocks(_ptr(key_cache), _ptr(value_cache), NB, H, D, BS,
                             m.ctypes.data if m.shape[0] else None, m.shape[0], _stream(stream))
    _check(st, "pa_copy_blocks")


def pa_reshape_and_cache_fp8(key: torch.Tensor, value: torch.Tensor, key_cache: torch.Tensor,
                             value_cache: torch.Tensor, slot_mapping: torch.Tensor, k_scale: float,
                             v_scale: float, stream=None) -> None:
    """FP8 cache write. key/value [T, H_kv, D] bf16 (token stride may exceed H_kv*D);
    caches [NB, 16, H_kv, D] uint8 (E4M3 codes); slot_mapping [T] int64; one scale per pool."""
    if not (key.dtype is _BF16 and value.dtype is _BF16 and key_cache.dtype is _U8 and
            value_cache.dtype is _U8 and slot_mapping.dtype is _INT64):
        raise TypeError("pa_reshape_and_cache_fp8: key/value bf16, caches uint8, slot_mapping int64")
    T, H, D = key.shape
    ks, vs = key.stride(), value.stride()
    _require(ks[2] == 1 and ks[1] == D and vs[2] == 1 and vs[1] == D and value.shape == key.shape and
             slot_mapping.is_contiguous() and key_cache.is_contiguous() and value_cache.is_contiguous(),
             "pa_reshape_and_cache_fp8: rows of key/value contiguous, caches and slot_mapping contiguous")
    NB, BS = key_cache.shape[:2]
    st = _lib.pa_reshape_and_cache_fp8(key.data_ptr(), value.data_ptr(), ks[0], vs[0], key_cache.data_ptr(),
                                       value_cache.data_ptr(), slot_mapping.data_ptr(), T, H, D, NB, BS,
                                       float(k_scale), float(v_scale), _stream(stream))
    _check(st, "pa_reshape_and_cache_fp8")


def pa_decode_plan(num_seqs: int, q_per_seq: int, num_q_heads: int, num_kv_heads: int,
                   head_dim: int, max_blocks_per_seq: int, path: int = PA_PATH_AUTO,
                   split_blocks: int = 0, schedule: int = PA_SCHEDULE_AUTO,
                   share_prefix: bool = False, sliding_window: int = 0,
                   kv_cache_dtype: int = PA_KV_BF16) -> pa_plan_t:
    """A forced split length implies the grid schedule (the tcgen05 path has no split
    length: its schedule cuts the work into equal tile ranges, and ignores it)."""
    if split_blocks and schedule == PA_SCHEDULE_AUTO and path != PA_PATH_TCGEN05:
        schedule = PA_SCHEDULE_GRID
    hints = pa_plan_hints_t(path, schedule, split_blocks, int(bool(share_prefix)), int(sliding_window),
                            int(kv_cache_dtype))
    plan = pa_plan_t()
    st = _lib.pa_decode_plan(num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim,
                             max_blocks_per_seq, ctypes.byref(hints), ctypes.byref(plan))
    _check(st, "pa_decode_plan")
    return plan


def pa_decode_workspace_size(plan: pa_plan_t | None, num_seqs: int, q_per_seq: int,
                             num_q_heads: int, num_kv_heads: int, head_dim: int,
                             max_blocks_per_seq: int) -> int:
    return int(_lib.pa_decode_workspace_size(None if plan is None else ctypes.byref(plan), num_seqs,
                                             q_per_seq, num_q_heads, num_kv_heads, head_dim,
                                             max_blocks_per_seq))


def pa_decode(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
              value_cache: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor,
              q_per_seq: int, scale: float, plan: pa_plan_t | None = None,
              workspace: torch.Tensor | None = None, stream=None) -> None:
    """out/query [B, q, H_q, D] bf16; caches [NB, 16, H_kv, D] bf16; block_tables
    [B, max_blocks] int32; context_lens [B] int32. workspace: any contiguous CUDA
    tensor of at least pa_decode_workspace_size(plan, ...) bytes (None when 0)."""
    args = _decode_args(out, query, key_cache, value_cache, block_tables, context_lens, q_per_seq, _BF16,
                        "pa_decode")
    st = _lib.pa_decode(*args, float(scale), None if plan is None else ctypes.byref(plan),
                        None if workspace is None else workspace.data_ptr(),
                        0 if workspace is None else workspace.nbytes, _stream(stream))
    _check(st, "pa_decode")


def pa_decode_fp8(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                  value_cache: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor,
                  q_per_seq: int, scale: float, k_scale: float, v_scale: float,
                  plan: pa_plan_t | None = None, workspace: torch.Tensor | None = None, stream=None) -> None:
    """pa_decode over FP8 pools: caches [NB, 16, H_kv, D] uint8 (E4M3 codes, values code *
    k_scale / code * v_scale); everything else as pa_decode. plan: None or one made with
    kv_cache_dtype=PA_KV_FP8_E4M3."""
    args = _decode_args(out, query, key_cache, value_cache, block_tables, context_lens, q_per_seq, _U8,
                        "pa_decode_fp8")
    st = _lib.pa_decode_fp8(*args, float(scale), float(k_scale), float(v_scale),
                            None if plan is None else ctypes.byref(plan),
                            None if workspace is None else workspace.data_ptr(),
                            0 if workspace is None else workspace.nbytes, _stream(stream))
    _check(st, "pa_decode_fp8")


class PreparedDecode:
    """pa_decode (bf16 pools) or pa_decode_fp8 (uint8 pools: give k_scale and v_scale) with its
    tensors checked and its C arguments built once; each call launches the decode on the same
    buffers and stream. For a step loop that reuses its buffers: a call then costs the C entry
    point alone, not the per-call checks of the tensors. The tensors must keep their storage,
    shapes and layout while the object is used (it holds references to them)."""

    def __init__(self, out, query, key_cache, value_cache, block_tables, context_lens, q_per_seq, scale,
                 plan: pa_plan_t | None = None, workspace: torch.Tensor | None = None, stream=None,
                 k_scale: float | None = None, v_scale: float | None = None):
        fp8 = key_cache.dtype is _U8
        if fp8 != (k_scale is not None and v_scale is not None):
            raise ValueError("PreparedDecode: k_scale and v_scale go with uint8 (E4M3) pools, and only with them")
        where = "pa_decode_fp8" if fp8 else "pa_decode"
        args = _decode_args(out, query, key_cache, value_cache, block_tables, context_lens, q_per_seq,
                            _U8 if fp8 else _BF16, where)
        scales = (float(scale), float(k_scale), float(v_scale)) if fp8 else (float(scale),)
        self._keep = (out, query, key_cache, value_cache, block_tables, context_lens, plan, workspace)
        self._fn = _lib.pa_decode_fp8 if fp8 else _lib.pa_decode
        self._where = where
        self._args = args + scales + (None if plan is None else ctypes.byref(plan),
                                      None if workspace is None else workspace.data_ptr(),
                                      0 if workspace is None else workspace.nbytes, _stream(stream))

    def __call__(self) -> None:
        st = self._fn(*self._args)
        if st != PA_OK:
            raise PAError(st, self._where)


class PreparedCacheWrite:
    """pa_reshape_and_cache (bf16 pools) or pa_reshape_and_cache_fp8 (uint8 pools: give k_scale
    and v_scale) prepared like PreparedDecode."""

    def __init__(self, key, value, key_cache, value_cache, slot_mapping, stream=None,
                 k_scale: float | None = None, v_scale: float | None = None):
        fp8 = key_cache.dtype is _U8
        if fp8 != (k_scale is not None and v_scale is not None):
            raise ValueError("PreparedCacheWrite: k_scale and v_scale go with uint8 (E4M3) pools, and only with them")
        where = "pa_reshape_and_cache_fp8" if fp8 else "pa_reshape_and_cache"
        cdt = _U8 if fp8 else _BF16
        if not (key.dtype is _BF16 and value.dtype is _BF16 and key_cache.dtype is cdt and
                value_cache.dtype is cdt and slot_mapping.dtype is _INT64):
            raise TypeError(f"{where}: key/value bf16, caches {cdt}, slot_mapping int64")
        T, H, D = key.shape
        ks, vs = key.stride(), value.stride()
        _require(ks[2] == 1 and ks[1] == D and vs[2] == 1 and vs[1] == D and value.shape == key.shape and
                 slot_mapping.is_contiguous() and key_cache.is_contiguous() and value_cache.is_contiguous(),
                 f"{where}: rows of key/value contiguous, caches and slot_mapping contiguous")
        NB, BS = key_cache.shape[:2]
        self._keep = (key, value, key_cache, value_cache, slot_mapping)
        self._fn = _lib.pa_reshape_and_cache_fp8 if fp8 else _lib.pa_reshape_and_cache
        self._where = where
        self._args = ((key.data_ptr(), value.data_ptr(), ks[0], vs[0], key_cache.data_ptr(), value_cache.data_ptr(),
                       slot_mapping.data_ptr(), T, H, D, NB, BS) +
                      ((float(k_scale), float(v_scale)) if fp8 else ()) + (_stream(stream),))

    def __call__(self) -> None:
        st = self._fn(*self._args)
        if st != PA_OK:
            raise PAError(st, self._where)


def pa_prefill(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor, value_cache: torch.Tensor,
               block_tables: torch.Tensor, context_lens: torch.Tensor, query_start: torch.Tensor,
               max_query_len: int, scale: float, stream=None) -> None:
    """Chunked-prefill attention. out/query [T, H_q, D] bf16 (the chunks of all sequences,
    concatenated); query_start [B + 1] int32 on the device; caches, block_tables and
    context_lens as pa_decode; max_query_len bounds every chunk length."""
    assert out.dtype == query.dtype == key_cache.dtype == value_cache.dtype == torch.bfloat16
    assert block_tables.dtype == context_lens.dtype == query_start.dtype == torch.int32
    for t in (out, query, key_cache, value_cache, block_tables, context_lens, query_start):
        assert t.is_contiguous()
    T, HQ, D = query.shape
    assert tuple(out.shape) == tuple(query.shape)
    B = block_tables.shape[0]
    assert query_start.numel() == B + 1 and context_lens.numel() == B
    NB, BS, HKV = key_cache.shape[0], key_cache.shape[1], key_cache.shape[2]
    st = _lib.pa_prefill(_ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables),
                         _ptr(context_lens), _ptr(query_start), B, T, int(max_query_len), HQ, HKV, D, BS,
                         block_tables.shape[1], NB, float(scale), _stream(stream))
    _check(st, "pa_prefill")


def pa_decode_partial(part_o: torch.Tensor, part_ml: torch.Tensor, query: torch.Tensor,
                      key_cache: torch.Tensor, value_cache: torch.Tensor, block_tables: torch.Tensor,
                      context_lens: torch.Tensor, q_per_seq: int, scale: float, block_begin: int,
                      block_end: int, stream=None) -> None:
    """The attention over table entries [block_begin, block_end) of every sequence, cut into
    part_o.shape[0] pieces, as unnormalised records: part_o [S, B, q, H_q, D] fp32, part_ml
    [S, B, q, H_q, 2] fp32 {m, l} (m in log2 units). Other arguments as pa_decode."""
    assert query.dtype == key_cache.dtype == value_cache.dtype == torch.bfloat16
    assert part_o.dtype == part_ml.dtype == torch.float32
    assert block_tables.dtype == torch.int32 and context_lens.dtype == torch.int32
    for t in (part_o, part_ml, query, key_cache, value_cache, block_tables, context_lens):
        assert t.is_contiguous()
    B, QS, HQ, D = query.shape
    S = part_o.shape[0]
    assert QS == q_per_seq and tuple(part_o.shape) == (S, B, QS, HQ, D) and tuple(part_ml.shape) == (S, B, QS, HQ, 2)
    NB, BS, HKV = key_cache.shape[0], key_cache.shape[1], key_cache.shape[2]
    st = _lib.pa_decode_partial(_ptr(part_o), _ptr(part_ml), _ptr(query), _ptr(key_cache), _ptr(value_cache),
                                _ptr(block_tables), _ptr(context_lens), B, QS, HQ, HKV, D, BS,
                                block_tables.shape[1], NB, float(scale), int(block_begin), int(block_end), S,
                                _stream(stream))
    _check(st, "pa_decode_partial")


def pa_decode_partial_pieces(num_seqs: int, q_per_seq: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                             range_blocks: int) -> int:
    """Pieces the decode heuristic takes for ranges of range_blocks table entries (0: bad shapes)."""
    return int(_lib.pa_decode_partial_pieces(num_seqs, q_per_seq, num_q_heads, num_kv_heads, head_dim,
                                             range_blocks))


def pa_combine_partials(rec_o: torch.Tensor, rec_ml: torch.Tensor, part_o: torch.Tensor, part_ml: torch.Tensor,
                        stream=None) -> None:
    """One record per row, rec_o [B, q, H_q, D] and rec_ml [B, q, H_q, 2] fp32, from the pieces
    part_o [P, B, q, H_q, D] and part_ml [P, B, q, H_q, 2]."""
    assert rec_o.dtype == rec_ml.dtype == part_o.dtype == part_ml.dtype == torch.float32
    for t in (rec_o, rec_ml, part_o, part_ml):
        assert t.is_contiguous()
    P, B, QS, HQ, D = part_o.shape
    assert tuple(rec_o.shape) == (B, QS, HQ, D) and tuple(rec_ml.shape) == (B, QS, HQ, 2)
    assert tuple(part_ml.shape) == (P, B, QS, HQ, 2)
    st = _lib.pa_combine_partials(_ptr(rec_o), _ptr(rec_ml), _ptr(part_o), _ptr(part_ml), P, B, QS, HQ, D,
                                  _stream(stream))
    _check(st, "pa_combine_partials")


def pa_merge_partials(out: torch.Tensor, part_o: torch.Tensor, part_ml: torch.Tensor, stream=None) -> None:
    """out [B, q, H_q, D] bf16 from the pieces part_o [P, B, q, H_q, D] and part_ml
    [P, B, q, H_q, 2] fp32 (an all-gather of pa_decode_partial outputs)."""
    assert out.dtype == torch.bfloat16 and part_o.dtype == part_ml.dtype == torch.float32
    for t in (out, part_o, part_ml):
        assert t.is_contiguous()
    P, B, QS, HQ, D = part_o.shape
    assert tuple(out.shape) == (B, QS, HQ, D) and tuple(part_ml.shape) == (P, B, QS, HQ, 2)
    st = _lib.pa_merge_partials(_ptr(out), _ptr(part_o), _ptr(part_ml), P, B, QS, HQ, D, _stream(stream))
    _check(st, "pa_merge_partials")


def pa_decode_static_scratch(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                             value_cache: torch.Tensor, block_tables: torch.Tensor,
                             context_lens: torch.Tensor, q_per_seq: int, scale: float,
                             plan: pa_plan_t | None = None, stream=None) -> None:
    """pa_decode without a caller workspace: for callers that cannot allocate device
    memory where they decode. Split partials go to the library's fixed
    PA_STATIC_SCRATCH_BYTES array; calls must not overlap on the GPU."""
    assert out.dtype == query.dtype == key_cache.dtype == value_cache.dtype == torch.bfloat16
    assert block_tables.dtype == torch.int32 and context_lens.dtype == torch.int32
    for t in (out, query, key_cache, value_cache, block_tables, context_lens):
        assert t.is_contiguous()
    B, QS, HQ, D = query.shape
    assert QS == q_per_seq and tuple(out.shape) == tuple(query.shape)
    NB, BS, HKV = key_cache.shape[0], key_cache.shape[1], key_cache.shape[2]
    st = _lib.pa_decode_static_scratch(_ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache),
                                       _ptr(block_tables), _ptr(context_lens), B, QS, HQ, HKV, D, BS,
                                       block_tables.shape[1], NB, float(scale),
                                       None if plan is None else ctypes.byref(plan), _stream(stream))
    _check(st, "pa_decode_static_scratch")


def pa_validate(block_tables: torch.Tensor, context_lens: torch.Tensor,
                slot_mapping: torch.Tensor | None, q_per_seq: int, num_blocks: int,
                block_size: int = 16, stream=None) -> int:
    """Returns the number of out-of-range entries (0 = all preconditions hold)."""
    bad = _I64(0)
    T = 0 if slot_mapping is None else slot_mapping.numel()
    st = _lib.pa_validate(_ptr(block_tables), _ptr(context_lens), _ptr(slot_mapping),
                          block_tables.shape[0], block_tables.shape[1], q_per_seq, T, num_blocks,
                          block_size, ctypes.byref(bad), _stream(stream))
    if st not in (PA_OK, PA_ERR_OUT_OF_RANGE):
        _check(st, "pa_validate")
    return int(bad.value)


def pa_selftest_bounded_wait(stream=None) -> None:
    """Enqueue the failure-path self-test: about one wait limit later the device error
    word holds 0x600 (read it with pa_get_device_error)."""
    _check(_lib.pa_selftest_bounded_wait(_stream(stream)), "pa_selftest_bounded_wait")


def pa_get_device_error(reset: bool = True, stream=None) -> int:
    code = ctypes.c_uint32(0)
    st = _lib.pa_get_device_error(ctypes.byref(code), int(reset), _stream(stream))
    if st not in (PA_OK, PA_ERR_DEVICE):
        _check(st, "pa_get_device_error")
    return int(code.value)


def raw_library() -> ctypes.CDLL:
    """The loaded ctypes handle (tests call entry points with raw pointers through it)."""
    return _lib
