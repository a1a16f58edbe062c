"""fp64 CPU oracle for the paged KV-cache hot path (cache write + paged decode) and the
copy-on-write block copy.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use it. The
CUDA library and its Python binding never import it.

The arithmetic lives in ``pa_oracle.cpp`` (plain C++17, fp64, std::thread);
this module only compiles it with g++ and marshals numpy/torch CPU arrays.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(HERE, "pa_oracle.cpp")


def library_path(mutant: int = 0) -> str:
    name = "libpa_oracle.so" if mutant == 0 else f"libpa_oracle_mutant{mutant}.so"
    return os.path.join(HERE, name)


def build(mutant: int = 0, force: bool = False, out_dir: str | None = None) -> str:
    """Compile the oracle (or a mutant with one planted mistake) into a .so."""
    path = library_path(mutant)
    if out_dir is not None:
        path = os.path.join(out_dir, os.path.basename(path))
    if not force and os.path.exists(path) and os.path.getmtime(path) >= os.path.getmtime(SOURCE):
        return path
    tmp = path + f".tmp{os.getpid()}"
    cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
           f"-DORACLE_MUTANT={mutant}", SOURCE, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, path)
    return path


_I64 = ctypes.c_int64
_I32 = ctypes.c_int
_P = ctypes.c_void_p


def _declare(lib: ctypes.CDLL) -> ctypes.CDLL:
    lib.oracle_bf16_to_f64.restype = ctypes.c_double
    lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
    lib.oracle_blocks_for_tokens.restype = _I64
    lib.oracle_blocks_for_tokens.argtypes = [_I64, _I64]
    lib.oracle_kv_bytes_per_token.restype = _I64
    lib.oracle_kv_bytes_per_token.argtypes = [_I64, _I64, _I64, _I64]
    lib.oracle_reshape_and_cache.restype = _I32
    lib.oracle_reshape_and_cache.argtypes = [_P, _P, _I64, _I64, _P, _P, _P, _I64,
                                             _I32, _I32, _I64, _I32]
    lib.oracle_decode.restype = _I32
    lib.oracle_decode.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32,
                                  _I32, _I32, _I64, ctypes.c_double, _I32]
    lib.oracle_decode_rows.restype = _I32
    lib.oracle_decode_rows.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32,
                                       _I32, _I32, _I32, _I64, ctypes.c_double, _P, _I64,
                                       _I32]
    lib.oracle_decode_window.restype = _I32
    lib.oracle_decode_window.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32,
                                         _I32, _I32, _I64, ctypes.c_double, _I32, _I32]
    lib.oracle_decode_rows_window.restype = _I32
    lib.oracle_decode_rows_window.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32,
                                              _I32, _I32, _I32, _I64, ctypes.c_double, _P, _I64,
                                              _I32, _I32]
    lib.oracle_fp8_encode.restype = None
    lib.oracle_fp8_encode.argtypes = [_P, _P, _I64]
    lib.oracle_fp8_decode.restype = None
    lib.oracle_fp8_decode.argtypes = [_P, _P, _I64]
    lib.oracle_reshape_and_cache_fp8.restype = _I32
    lib.oracle_reshape_and_cache_fp8.argtypes = [_P, _P, _I64, _I64, _P, _P, _P, _I64, _I32, _I32, _I64, _I32,
                                                 ctypes.c_float, ctypes.c_float]
    lib.oracle_decode_fp8.restype = _I32
    lib.oracle_decode_fp8.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _I32, _I32, _I64,
                                      ctypes.c_double, ctypes.c_double, ctypes.c_double, _I32, _I32]
    lib.oracle_copy_blocks.restype = _I32
    lib.oracle_copy_blocks.argtypes = [_P, _P, _I64, _I64, _P, _I64]
    lib.oracle_threads_used.restype = _I32
    lib.oracle_mutant_id.restype = _I32
    return lib


_LIBS: dict[int, ctypes.CDLL] = {}


def load(mutant: int = 0, out_dir: str | None = None) -> ctypes.CDLL:
    key = mutant if out_dir is None else (mutant, out_dir)
    if key not in _LIBS:
        _LIBS[key] = _declare(ctypes.CDLL(build(mutant, out_dir=out_dir)))
    return _LIBS[key]


def _u16(a) -> np.ndarray:
    """bf16 data as a contiguous uint16 numpy array (bit patterns)."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            assert a.dtype == torch.bfloat16
            return a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16
    return a


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


class Oracle:
    """Thin wrapper over one compiled oracle library (the real one by default)."""

    def __init__(self, mutant: int = 0, out_dir: str | None = None):
        self.lib = load(mutant, out_dir)

    def bf16_to_f64(self, bits: int) -> float:
        return self.lib.oracle_bf16_to_f64(bits)

    def blocks_for_tokens(self, n: int, block_size: int = 16) -> int:
        return self.lib.oracle_blocks_for_tokens(n, block_size)

    def kv_bytes_per_token(self, layers: int, kv_heads: int, head_dim: int,
                           bytes_per_value: int = 2) -> int:
        return self.lib.oracle_kv_bytes_per_token(layers, kv_heads, head_dim, bytes_per_value)

    def reshape_and_cache(self, key, value, key_cache, value_cache, slot_mapping):
        """Returns new (key_cache, value_cache) uint16 arrays; inputs untouched."""
        k = _u16(key)
        v = _u16(value)
        kc = _u16(key_cache).copy()
        vc = _u16(value_cache).copy()
        slots = np.ascontiguousarray(np.asarray(slot_mapping, dtype=np.int64))
        T, H, D = k.shape
        NB, BS = kc.shape[0], kc.shape[1]
        st = self.lib.oracle_reshape_and_cache(_ptr(k), _ptr(v), H * D, H * D, _ptr(kc),
                                               _ptr(vc), _ptr(slots), T, H, D, NB, BS)
        if st != 0:
            raise ValueError(f"oracle_reshape_and_cache status {st}")
        return kc, vc

    def decode(self, query, key_cache, value_cache, block_tables, context_lens,
               q_per_seq: int, scale: float, num_threads: int = 0, window: int = 0) -> np.ndarray:
        """fp64 output [B, q_per_seq, H_q, D]. query is [B, q_per_seq, H_q, D] bf16.
        window > 0: sliding window of that many tokens (table entries before every
        row's window are not read)."""
        q = _u16(query)
        kc = _u16(key_cache)
        vc = _u16(value_cache)
        bt = np.ascontiguousarray(np.asarray(block_tables, dtype=np.int32))
        cl = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32))
        B, QS, HQ, D = q.shape
        assert QS == q_per_seq
        NB, BS, HKV = kc.shape[0], kc.shape[1], kc.shape[2]
        out = np.zeros((B, QS, HQ, D), dtype=np.float64)
        if window > 0:
            st = self.lib.oracle_decode_window(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _ptr(bt),
                                               _ptr(cl), B, QS, HQ, HKV, D, BS, bt.shape[1], NB,
                                               float(scale), int(window), num_threads)
        else:
            st = self.lib.oracle_decode(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _ptr(bt),
                                        _ptr(cl), B, QS, HQ, HKV, D, BS, bt.shape[1], NB,
                                        float(scale), num_threads)
        if st != 0:
            raise ValueError(f"oracle_decode status {st}")
        return out

    def decode_rows(self, rows, query, key_cache, value_cache, block_tables, context_lens,
                    q_per_seq: int, scale: float, num_threads: int = 0, window: int = 0) -> np.ndarray:
        """fp64 outputs [len(rows), D] for the (b, i, h) triples in rows."""
        q = _u16(query)
        kc = _u16(key_cache)
        vc = _u16(value_cache)
        bt = np.ascontiguousarray(np.asarray(block_tables, dtype=np.int32))
        cl = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32))
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
        B, QS, HQ, D = q.shape
        NB, BS, HKV = kc.shape[0], kc.shape[1], kc.shape[2]
        out = np.zeros((r.shape[0], D), dtype=np.float64)
        st = self.lib.oracle_decode_rows_window(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _ptr(bt),
                                                _ptr(cl), B, QS, HQ, HKV, D, BS, bt.shape[1], NB,
                                                float(scale), _ptr(r), r.shape[0], int(window),
                                                num_threads)
        if st != 0:
            raise ValueError(f"oracle_decode_rows status {st}")
        return out

    def fp8_encode(self, x) -> np.ndarray:
        """E4M3 codes (uint8) of fp32 values (ties to even, saturating at +-448)."""
        xf = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
        out = np.empty(xf.shape, dtype=np.uint8)
        self.lib.oracle_fp8_encode(_ptr(xf), _ptr(out), xf.size)
        return out

    def fp8_decode(self, codes) -> np.ndarray:
        """fp64 values of E4M3 codes (NaN for S.1111.111)."""
        c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
        out = np.empty(c.shape, dtype=np.float64)
        self.lib.oracle_fp8_decode(_ptr(c), _ptr(out), c.size)
        return out

    def reshape_and_cache_fp8(self, key, value, key_cache, value_cache, slot_mapping,
                              k_scale: float, v_scale: float):
        """FP8 cache write. key/value bf16 [T, H_kv, D]; caches uint8 [NB, bs, H_kv, D].
        Returns new (key_cache, value_cache) uint8 arrays; inputs untouched."""
        k = _u16(key)
        v = _u16(value)
        kc = np.ascontiguousarray(np.asarray(key_cache, dtype=np.uint8)).copy()
        vc = np.ascontiguousarray(np.asarray(value_cache, dtype=np.uint8)).copy()
        slots = np.ascontiguousarray(np.asarray(slot_mapping, dtype=np.int64))
        T, H, D = k.shape
        NB, BS = kc.shape[0], kc.shape[1]
        st = self.lib.oracle_reshape_and_cache_fp8(_ptr(k), _ptr(v), H * D, H * D, _ptr(kc), _ptr(vc),
                                                   _ptr(slots), T, H, D, NB, BS, float(k_scale), float(v_scale))
        if st != 0:
            raise ValueError(f"oracle_reshape_and_cache_fp8 status {st}")
        return kc, vc

    def decode_fp8(self, query, key_cache, value_cache, block_tables, context_lens, q_per_seq: int,
                   scale: float, k_scale: float, v_scale: float, window: int = 0,
                   num_threads: int = 0) -> np.ndarray:
        """fp64 output [B, q, H_q, D] over FP8 pools (uint8 [NB, bs, H_kv, D]) and their scales."""
        q = _u16(query)
        kc = np.ascontiguousarray(np.asarray(key_cache, dtype=np.uint8))
        vc = np.ascontiguousarray(np.asarray(value_cache, dtype=np.uint8))
        bt = np.ascontiguousarray(np.asarray(block_tables, dtype=np.int32))
        cl = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32))
        B, QS, HQ, D = q.shape
        NB, BS, HKV = kc.shape[0], kc.shape[1], kc.shape[2]
        out = np.zeros((B, QS, HQ, D), dtype=np.float64)
        st = self.lib.oracle_decode_fp8(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _ptr(bt), _ptr(cl), B, QS, HQ,
                                        HKV, D, BS, bt.shape[1], NB, float(scale), float(k_scale), float(v_scale),
                                        int(window), num_threads)
        if st != 0:
            raise ValueError(f"oracle_decode_fp8 status {st}")
        return out

    def copy_blocks(self, key_cache, value_cache, block_mapping):
        """Copy-on-write block copy. block_mapping is [n][2] {source, destination}.
        Returns new (key_cache, value_cache) uint16 arrays; inputs untouched."""
        kc = _u16(key_cache).copy()
        vc = _u16(value_cache).copy()
        m = np.ascontiguousarray(np.asarray(block_mapping, dtype=np.int64).reshape(-1, 2))
        NB = kc.shape[0]
        block_elems = int(np.prod(kc.shape[1:]))
        st = self.lib.oracle_copy_blocks(_ptr(kc), _ptr(vc), NB, block_elems, _ptr(m), m.shape[0])
        if st != 0:
            raise ValueError(f"oracle_copy_blocks status {st}")
        return kc, vc

    def threads_used(self) -> int:
        return self.lib.oracle_threads_used()
