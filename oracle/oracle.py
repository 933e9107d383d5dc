"""ctypes front end of the fp64 C oracle (``kvring_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg use it; the product never does.  It imports nothing from the product
package; inputs arrive as numpy arrays from the seeded generators.

The arithmetic lives in the C file; this module only owns the host arrays of an oracle
ring and marshals pointers.  See the C file's header for the definitions it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvring_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

# gcc flags: no contraction into FMA, no fast-math, so every binary64 op is IEEE.
GCC_FLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
             "-std=c11", "-Wall", "-Wno-unknown-pragmas"]


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (skipped when up to date)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        P = ctypes.c_void_p
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_bf16_round.restype = ctypes.c_float
        L.orc_bf16_round.argtypes = [ctypes.c_float]
        L.orc_rope_cs.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_double, P, P]
        L.orc_rope_apply.argtypes = [P, ctypes.c_int, P, P, P]
        L.orc_rope_apply_f64.argtypes = [P, ctypes.c_int, ctypes.c_int64, ctypes.c_double, P]
        L.orc_quant_row.argtypes = [P, ctypes.c_int, P, P]
        L.orc_slot_of_age.restype = ctypes.c_int64
        L.orc_slot_of_age.argtypes = [P, ctypes.c_int64]
        L.orc_ring_commit.argtypes = [P]
        L.orc_ring_write.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int]
        L.orc_ring_delta_rotate.argtypes = [P, ctypes.c_int64]
        L.orc_ring_delta_rotate.restype = ctypes.c_int
        L.orc_rope_cs_ring.argtypes = [P, ctypes.c_int64, P, P]
        L.orc_chunk_attention.argtypes = [
            P, P, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_float, ctypes.c_int, P,
            ctypes.c_int, P, P]
        L.orc_chunk_attention_multi.argtypes = [
            P, ctypes.c_int, P, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_float,
            ctypes.c_int, P, ctypes.c_int, P, P]
        L.orc_key_mass.argtypes = [
            P, ctypes.c_int, P, ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_float,
            ctypes.c_int, P, ctypes.c_int, P]
        L.orc_memory_select.argtypes = [P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_double, P]
        L.orc_memory_select.restype = ctypes.c_int
        L.orc_e4m3_encode_n.argtypes = [P, ctypes.c_int64, P]
        L.orc_e4m3_decode_n.argtypes = [P, ctypes.c_int64, P]
        L.orc_bf16_round_n.argtypes = [P, ctypes.c_int64, P]
        L.orc_quant_rows.argtypes = [P, ctypes.c_int64, ctypes.c_int, P, P]
        L.orc_struct_size.restype = ctypes.c_int
    return _lib


def _p(a: np.ndarray) -> ctypes.c_void_p:
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


# ------------------------------------------------------------------ scalar/array helpers

def e4m3_encode(v) -> np.ndarray:
    v = _f32(v)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e4m3_encode_n(_p(v), v.size, _p(out))
    return out


def e4m3_decode(c) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(c, dtype=np.uint8))
    out = np.empty(c.shape, np.float64)
    lib().orc_e4m3_decode_n(_p(c), c.size, _p(out))
    return out


def bf16_round(v) -> np.ndarray:
    v = _f32(v)
    out = np.empty(v.shape, np.float32)
    lib().orc_bf16_round_n(_p(v), v.size, _p(out))
    return out


def rope_cs(p: int, D: int, base: float = 10000.0):
    c = np.empty(D // 2, np.float32)
    s = np.empty(D // 2, np.float32)
    lib().orc_rope_cs(int(p), D, float(base), _p(c), _p(s))
    return c, s


def rope_apply(x, p: int, base: float = 10000.0) -> np.ndarray:
    """binary32 RoPE of one row at position p."""
    x = _f32(x)
    c, s = rope_cs(p, x.shape[-1], base)
    y = np.empty_like(x)
    lib().orc_rope_apply(_p(x), x.shape[-1], _p(c), _p(s), _p(y))
    return y


def rope_apply_f64(x, p: int, base: float = 10000.0) -> np.ndarray:
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    y = np.empty_like(x)
    lib().orc_rope_apply_f64(_p(x), x.shape[-1], int(p), float(base), _p(y))
    return y


def quant_rows(y) -> tuple[np.ndarray, np.ndarray]:
    """Per-row e4m3 quantisation of a [rows][D] binary32 array -> (codes, scales)."""
    y = _f32(y)
    rows, D = y.reshape(-1, y.shape[-1]).shape
    codes = np.empty((rows, D), np.uint8)
    scales = np.empty(rows, np.float32)
    lib().orc_quant_rows(_p(y), rows, D, _p(codes), _p(scales))
    return codes.reshape(y.shape), scales.reshape(y.shape[:-1])


# ------------------------------------------------------------------ ring

class _RingStruct(ctypes.Structure):
    _fields_ = [("C", ctypes.c_int32), ("H", ctypes.c_int32), ("D", ctypes.c_int32),
                ("_pad", ctypes.c_int32), ("base", ctypes.c_double),
                ("pairs_t", ctypes.c_int32), ("pairs_h", ctypes.c_int32),
                ("pairs_w", ctypes.c_int32), ("grid_h", ctypes.c_int32),
                ("grid_w", ctypes.c_int32), ("_pad2", ctypes.c_int32),
                ("write_slot", ctypes.c_int64), ("live", ctypes.c_int64),
                ("pending", ctypes.c_int64), ("next_pos", ctypes.c_int64),
                ("kc", ctypes.c_void_p), ("vc", ctypes.c_void_p), ("ks", ctypes.c_void_p),
                ("vs", ctypes.c_void_p), ("slot_pos", ctypes.c_void_p)]


class OracleRing:
    """Host-side oracle ring: codes [H][C][D] u8, scales [H][C] f32, slot_pos [C] i32.

    rope3d = (pairs_t, pairs_h, pairs_w, grid_h, grid_w) selects 3-D RoPE (see
    ``orc_rope_cs_ring`` in the C file); None is 1-D RoPE."""

    def __init__(self, capacity: int, n_heads: int, head_dim: int, base: float = 10000.0,
                 next_pos: int = 0, rope3d=None):
        assert head_dim % 2 == 0 and head_dim <= 512
        self.C, self.H, self.D = capacity, n_heads, head_dim
        self.kc = np.zeros((n_heads, capacity, head_dim), np.uint8)
        self.vc = np.zeros((n_heads, capacity, head_dim), np.uint8)
        self.ks = np.zeros((n_heads, capacity), np.float32)
        self.vs = np.zeros((n_heads, capacity), np.float32)
        self.slot_pos = np.zeros(capacity, np.int32)
        r3 = (0, 0, 0, 0, 0) if rope3d is None else tuple(int(x) for x in rope3d)
        if rope3d is not None:
            assert sum(r3[:3]) == head_dim // 2 and min(r3) >= 0 and r3[3] >= 1 and r3[4] >= 1
        self.rope3d = rope3d
        self._s = _RingStruct(capacity, n_heads, head_dim, 0, float(base), *r3, 0, 0, 0, 0,
                              int(next_pos), self.kc.ctypes.data, self.vc.ctypes.data,
                              self.ks.ctypes.data, self.vs.ctypes.data,
                              self.slot_pos.ctypes.data)
        assert lib().orc_struct_size() == ctypes.sizeof(_RingStruct)

    # state integers
    @property
    def write_slot(self): return self._s.write_slot

    @property
    def live(self): return self._s.live

    @property
    def pending(self): return self._s.pending

    @property
    def next_pos(self): return self._s.next_pos

    def state(self) -> tuple[int, int, int, int]:
        return (self._s.write_slot, self._s.live, self._s.pending, self._s.next_pos)

    def _ptr(self):
        return ctypes.byref(self._s)

    def slot_of_age(self, age: int) -> int:
        return lib().orc_slot_of_age(self._ptr(), int(age))

    def write(self, k, v, commit: bool = False) -> None:
        k, v = _f32(k), _f32(v)
        n = k.shape[0]
        assert k.shape == (n, self.H, self.D) and v.shape == k.shape and 0 < n <= self.C
        lib().orc_ring_write(self._ptr(), _p(k), _p(v), n, int(bool(commit)))

    def commit(self) -> None:
        lib().orc_ring_commit(self._ptr())

    def delta_rotate(self, delta: int) -> None:
        rc = lib().orc_ring_delta_rotate(self._ptr(), int(delta))
        if rc != 0:
            raise ValueError(f"3-D RoPE resets move whole frames: {delta} is not a multiple "
                             f"of the frame size")

    def rope_cs(self, p: int):
        """(cos, sin) of token position p under this ring's RoPE rule, binary32."""
        c = np.empty(self.D // 2, np.float32)
        s = np.empty(self.D // 2, np.float32)
        lib().orc_rope_cs_ring(self._ptr(), int(p), _p(c), _p(s))
        return c, s

    def attention(self, q, q_pos0: int, n_current: int, mask=(1 << 30, 1 << 30, 1 << 30, 1 << 30),
                  cache_bias: float = 0.0, softmax_scale: float | None = None, rows=None,
                  mode_b: bool = False):
        """Returns (out [rows][H][D] f64, lse [H][rows] f64).

        mask = (q_first_len, q_block_len, k_first_len, k_block_len)."""
        q, n_q, softmax_scale, rows_arr, n_rows, rp, out, lse = _attn_io(
            self, q, softmax_scale, rows)
        qf, qb, kf, kb = (int(x) for x in mask)
        lib().orc_chunk_attention(self._ptr(), _p(q), n_q, int(q_pos0), int(n_current), qf, qb,
                                  kf, kb, float(cache_bias), float(softmax_scale),
                                  int(bool(mode_b)), rp, n_rows, _p(out), _p(lse))
        return out, lse


def _attn_io(ring: "OracleRing", q, softmax_scale, rows):
    """Shared marshalling of the attention calls: query array, scale, row list, outputs."""
    q = _f32(q)
    n_q = q.shape[0]
    assert q.shape == (n_q, ring.H, ring.D)
    if softmax_scale is None:
        softmax_scale = float(np.float32(1.0 / np.sqrt(ring.D)))
    if rows is None:
        rows_arr, n_rows, rp = None, n_q, None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        assert rows_arr.min() >= 0 and rows_arr.max() < n_q
        n_rows, rp = rows_arr.size, _p(rows_arr)
    out = np.zeros((n_rows, ring.H, ring.D), np.float64)
    lse = np.zeros((ring.H, n_rows), np.float64)
    return q, n_q, softmax_scale, rows_arr, n_rows, rp, out, lse


def attention_multi(main: OracleRing, history_rings, q, q_pos0: int, n_current: int,
                    mask=(1 << 30, 1 << 30, 1 << 30, 1 << 30), cache_bias: float = 0.0,
                    softmax_scale: float | None = None, rows=None, mode_b: bool = False):
    """Attention over the valid slots of ``main`` and of every ring in ``history_rings``.

    ``main`` holds the current chunk (its newest ``n_current`` slots); every slot of the
    other rings is history (always visible, ``cache_bias`` added), e.g. a persistent
    anchor chunk kept beside the sliding window.  Same return values as
    ``OracleRing.attention``."""
    rings = [main, *history_rings]
    for r in rings:
        assert (r.H, r.D, r._s.base) == (main.H, main.D, main._s.base)
    q, n_q, softmax_scale, rows_arr, n_rows, rp, out, lse = _attn_io(
        main, q, softmax_scale, rows)
    ptrs = (ctypes.c_void_p * len(rings))(*[ctypes.addressof(r._s) for r in rings])
    qf, qb, kf, kb = (int(x) for x in mask)
    lib().orc_chunk_attention_multi(ctypes.cast(ptrs, ctypes.c_void_p), len(rings), _p(q), n_q,
                                    int(q_pos0), int(n_current), qf, qb, kf, kb,
                                    float(cache_bias), float(softmax_scale), int(bool(mode_b)),
                                    rp, n_rows, _p(out), _p(lse))
    return out, lse


def key_mass(main: OracleRing, history_rings, q, q_pos0: int, n_current: int, ring_index: int,
             ages, mask=(1 << 30, 1 << 30, 1 << 30, 1 << 30), cache_bias: float = 0.0,
             softmax_scale: float | None = None) -> np.ndarray:
    """Attention mass (sum over heads and query rows of the softmax probability) that the
    history slots of ring ``ring_index`` at the given ages receive in the attention call
    over ``main`` and ``history_rings`` (see ``orc_key_mass``)."""
    rings = [main, *history_rings]
    q = _f32(q)
    n_q = q.shape[0]
    if softmax_scale is None:
        softmax_scale = float(np.float32(1.0 / np.sqrt(main.D)))
    ages = np.ascontiguousarray(np.asarray(ages, dtype=np.int64))
    out = np.zeros(ages.size, np.float64)
    ptrs = (ctypes.c_void_p * len(rings))(*[ctypes.addressof(r._s) for r in rings])
    qf, qb, kf, kb = (int(x) for x in mask)
    lib().orc_key_mass(ctypes.cast(ptrs, ctypes.c_void_p), len(rings), _p(q), n_q, int(q_pos0),
                       int(n_current), qf, qb, kf, kb, float(cache_bias), float(softmax_scale),
                       int(ring_index), _p(ages), ages.size, _p(out))
    return out


def memory_select(quality, frame, pos, M: int, gamma: float = 0.5) -> np.ndarray:
    """Indices (ascending) of the candidates kept by the top-M rule with temporal
    diversity (see ``orc_memory_select``)."""
    qv = np.ascontiguousarray(np.asarray(quality, dtype=np.float64))
    fr = np.ascontiguousarray(np.asarray(frame, dtype=np.int64))
    ps = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    kept = np.zeros(max(1, qv.size), np.int32)
    m = lib().orc_memory_select(_p(qv), _p(fr), _p(ps), qv.size, int(M), float(gamma), _p(kept))
    return kept[:m].copy()
