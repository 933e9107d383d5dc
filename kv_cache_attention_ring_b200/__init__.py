"""Ring KV-cache attention for chunk-wise video diffusion on B200 (sm_100a).

Thin ctypes binding of ``libkvring.so`` (C ABI in ``include/kvring.h``).  The binding
only marshals arguments: every step of the path runs in the library's CUDA kernels.
PyTorch provides device memory and streams.  There is no fallback: if the library is
missing or the device is not sm_100, calls raise.

Entry points (same names as the C ABI): ``kv_rope_table_build``, ``KvRing`` (fills a
``kv_ring_t`` and calls ``kv_ring_init``), ``kv_ring_write``, ``kv_ring_commit``,
``kv_ring_delta_rotate``, ``chunk_attention``, ``chunk_attention_workspace_size``,
``chunk_attention_split``, ``chunk_attention_split_noalloc``, ``chunk_attention_multi``,
``chunk_attention_rows``, ``kv_status_string``, ``kv_wait_timeout_count``.
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvring.so")

KV_OK, KV_EINVAL, KV_ERANGE, KV_EUNSUPPORTED, KV_ECUDA, KV_ESTATE = 0, -1, -2, -3, -4, -5
KV_DTYPE_BF16, KV_DTYPE_FP32 = 1, 2
KV_COMMIT = 1
KV_QK_FP8 = 1
KV_PV_FP8 = 2

EXPORTS = ("kv_rope_table_build", "kv_rope3d_table_build", "kv_ring_init", "kv_ring_write", "kv_ring_commit",
           "kv_ring_delta_rotate", "chunk_attention", "chunk_attention_workspace_size",
           "chunk_attention_split", "chunk_attention_split_noalloc", "chunk_attention_multi",
           "chunk_attention_rows", "chunk_attention_suggest_splits", "chunk_key_mass", "chunk_key_mass_multi", "chunk_key_mass_workspace_size",
           "kv_memory_select", "kv_status_string",
           "kv_wait_timeout_count")
KV_NOALLOC_SCRATCH_BYTES = 16 << 20
KV_MEMORY_MAX_CANDIDATES = 8192
KV_MAX_RINGS = 8


class KvError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {kv_status_string(status)} (status {status})")
        self.status = status


class kv_ring_t(ctypes.Structure):
    _fields_ = [("capacity", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("initialized", ctypes.c_int32),
                ("write_slot", ctypes.c_int64), ("live", ctypes.c_int64),
                ("pending", ctypes.c_int64), ("next_pos", ctypes.c_int64),
                ("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
                ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
                ("slot_pos", ctypes.c_void_p), ("rope_table", ctypes.c_void_p),
                ("rope_pos_min", ctypes.c_int64), ("rope_pos_max", ctypes.c_int64),
                ("rope_base", ctypes.c_double),
                ("rope_pairs_t", ctypes.c_int32), ("rope_pairs_h", ctypes.c_int32),
                ("rope_pairs_w", ctypes.c_int32), ("rope_grid_h", ctypes.c_int32),
                ("rope_grid_w", ctypes.c_int32), ("rope_reserved", ctypes.c_int32),
                ("opaque", ctypes.c_uint64 * 96)]


class kv_block_mask_t(ctypes.Structure):
    _fields_ = [("q_first_len", ctypes.c_int32), ("q_block_len", ctypes.c_int32),
                ("k_first_len", ctypes.c_int32), ("k_block_len", ctypes.c_int32)]


class kv_cache_bias_t(ctypes.Structure):
    _fields_ = [("history_bias", ctypes.c_float)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libkvring.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m kv_cache_attention_ring_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        L.kv_rope_table_build.argtypes = [P, I64, I64, I, ctypes.c_double]
        L.kv_rope3d_table_build.argtypes = [P, I64, I64, I, ctypes.c_double, I, I, I, I, I]
        L.kv_ring_init.argtypes = [P]
        L.kv_ring_write.argtypes = [P, P, P, I, I, ctypes.c_uint32, P]
        L.kv_ring_commit.argtypes = [P]
        L.kv_ring_delta_rotate.argtypes = [P, I64, P]
        L.chunk_attention.argtypes = [P, P, I, I64, I, P, P, ctypes.c_float, P, P,
                                      ctypes.c_uint32, P]
        L.chunk_attention_rows.argtypes = [P, P, I, I64, I, P, I, P, P, ctypes.c_float, P, P,
                                           I, P, ctypes.c_size_t, ctypes.c_uint32, P]
        L.chunk_attention_suggest_splits.argtypes = [I, I, I64, I]
        L.chunk_attention_suggest_splits.restype = I
        L.chunk_key_mass.argtypes = [P, P, P, I, I64, P, P, ctypes.c_float, I64, I, P, P]
        L.chunk_key_mass_multi.argtypes = [P, I, P, P, I, I64, P, P, ctypes.c_float, P, P, P,
                                           P, ctypes.c_size_t, P]
        L.chunk_key_mass_workspace_size.argtypes = [I, I]
        L.chunk_key_mass_workspace_size.restype = ctypes.c_size_t
        L.kv_memory_select.argtypes = [P, P, P, P, I64, I, I, I64, ctypes.c_float, P, P, P]
        L.kv_status_string.argtypes = [I]
        L.kv_status_string.restype = ctypes.c_char_p
        L.kv_wait_timeout_count.argtypes = [P]
        L.chunk_attention_workspace_size.argtypes = [I, I, I, I]
        L.chunk_attention_workspace_size.restype = ctypes.c_size_t
        L.chunk_attention_split.argtypes = [P, P, I, I64, I, P, P, ctypes.c_float, P, P, I, P,
                                            ctypes.c_size_t, ctypes.c_uint32, P]
        L.chunk_attention_split_noalloc.argtypes = [P, P, I, I64, I, P, P, ctypes.c_float, P,
                                                    P, I, ctypes.c_uint32, P]
        L.chunk_attention_multi.argtypes = [P, I, P, I, I64, I, P, P, ctypes.c_float, P, P, I,
                                            P, ctypes.c_size_t, ctypes.c_uint32, P]
        _lib = L
    return _lib


def kv_status_string(status: int) -> str:
    return lib().kv_status_string(int(status)).decode()


def _check(rc: int, what: str) -> None:
    if rc != KV_OK:
        raise KvError(rc, what)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def kv_rope_table_build(pos_min: int, pos_max: int, head_dim: int,
                        base: float = 10000.0) -> np.ndarray:
    """Host RoPE table [(pos_max-pos_min+1)][head_dim/2][2] float32 (cos, sin)."""
    out = np.empty((pos_max - pos_min + 1, head_dim // 2, 2), np.float32)
    _check(lib().kv_rope_table_build(ctypes.c_void_p(out.ctypes.data), int(pos_min),
                                     int(pos_max), int(head_dim), float(base)),
           "kv_rope_table_build")
    return out


def kv_rope3d_table_build(pos_min: int, pos_max: int, head_dim: int, rope3d,
                          base: float = 10000.0) -> np.ndarray:
    """Host 3-D RoPE table [(pos_max-pos_min+1)][head_dim/2][2] float32; rope3d =
    (pairs_t, pairs_h, pairs_w, grid_h, grid_w)."""
    out = np.empty((pos_max - pos_min + 1, head_dim // 2, 2), np.float32)
    _check(lib().kv_rope3d_table_build(ctypes.c_void_p(out.ctypes.data), int(pos_min),
                                       int(pos_max), int(head_dim), float(base),
                                       *(int(x) for x in rope3d)),
           "kv_rope3d_table_build")
    return out


class KvRing:
    """A ring with its caller-owned device buffers (torch tensors) and its kv_ring_t.

    rope3d = (pairs_t, pairs_h, pairs_w, grid_h, grid_w) selects 3-D RoPE (the table is
    then built with kv_rope3d_table_build); None is 1-D RoPE."""

    def __init__(self, capacity: int, n_heads: int, head_dim: int, pos_min: int, pos_max: int,
                 base: float = 10000.0, next_pos: int = 0, device=None, rope_table=None,
                 rope3d=None):
        import torch
        dev = torch.device("cuda") if device is None else torch.device(device)
        C, H, D = int(capacity), int(n_heads), int(head_dim)
        self.C, self.H, self.D = C, H, D
        self.k_codes = torch.zeros((H, C, D), dtype=torch.uint8, device=dev)
        self.v_codes = torch.zeros((H, C, D), dtype=torch.uint8, device=dev)
        self.k_scale = torch.zeros((H, C), dtype=torch.float32, device=dev)
        self.v_scale = torch.zeros((H, C), dtype=torch.float32, device=dev)
        self.slot_pos = torch.zeros((C,), dtype=torch.int32, device=dev)
        if rope_table is None:
            host = (kv_rope_table_build(pos_min, pos_max, D, base) if rope3d is None else
                    kv_rope3d_table_build(pos_min, pos_max, D, rope3d, base))
            rope_table = torch.from_numpy(host).to(dev)
        self.rope_table = rope_table
        s = kv_ring_t()
        s.capacity, s.n_heads, s.head_dim = C, H, D
        s.next_pos = int(next_pos)
        s.k_codes, s.v_codes = self.k_codes.data_ptr(), self.v_codes.data_ptr()
        s.k_scale, s.v_scale = self.k_scale.data_ptr(), self.v_scale.data_ptr()
        s.slot_pos = self.slot_pos.data_ptr()
        s.rope_table = self.rope_table.data_ptr()
        s.rope_pos_min, s.rope_pos_max, s.rope_base = int(pos_min), int(pos_max), float(base)
        if rope3d is not None:
            (s.rope_pairs_t, s.rope_pairs_h, s.rope_pairs_w, s.rope_grid_h,
             s.rope_grid_w) = (int(x) for x in rope3d)
        self.s = s
        _check(lib().kv_ring_init(ctypes.byref(s)), "kv_ring_init")

    @property
    def ref(self):
        return ctypes.byref(self.s)

    def state(self) -> tuple[int, int, int, int]:
        return (self.s.write_slot, self.s.live, self.s.pending, self.s.next_pos)

    @property
    def next_pos(self) -> int:
        return self.s.next_pos

    @property
    def n_valid(self) -> int:
        return min(self.s.live + self.s.pending, self.C)


def kv_ring_write(ring: KvRing, k, v, commit: bool = False, stream=None) -> None:
    import torch
    assert k.is_cuda and v.is_cuda and k.is_contiguous() and v.is_contiguous()
    assert k.shape == v.shape and k.dim() == 3 and k.shape[1:] == (ring.H, ring.D)
    dt = {torch.bfloat16: KV_DTYPE_BF16, torch.float32: KV_DTYPE_FP32}.get(k.dtype)
    assert dt is not None and v.dtype == k.dtype
    _check(lib().kv_ring_write(ring.ref, _ptr(k), _ptr(v), dt, int(k.shape[0]),
                               KV_COMMIT if commit else 0, _stream(stream)), "kv_ring_write")


def kv_ring_commit(ring: KvRing) -> None:
    _check(lib().kv_ring_commit(ring.ref), "kv_ring_commit")


def kv_ring_delta_rotate(ring: KvRing, delta: int, stream=None) -> None:
    _check(lib().kv_ring_delta_rotate(ring.ref, int(delta), _stream(stream)),
           "kv_ring_delta_rotate")


def _flags(mode_b: bool, pv_fp8: bool) -> int:
    return (KV_QK_FP8 if mode_b else 0) | (KV_PV_FP8 if pv_fp8 else 0)


def chunk_attention(ring: KvRing, q, q_pos0: int, n_current: int, mask=None,
                    cache_bias: float = 0.0, softmax_scale: float | None = None, out=None,
                    lse=None, want_lse: bool = True, stream=None, mode_b: bool = False,
                    pv_fp8: bool = False):
    """q: bf16 [n_q][H][D] on the GPU.  mask: (q_first, q_block, k_first, k_block) or None.
    Returns (out bf16 [n_q][H][D], lse fp32 [H][n_q] or None)."""
    import torch
    assert q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous()
    n_q = int(q.shape[0])
    assert q.shape == (n_q, ring.H, ring.D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((ring.H, n_q), dtype=torch.float32, device=q.device)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(ring.D)
    m = None if mask is None else kv_block_mask_t(*(int(x) for x in mask))
    b = kv_cache_bias_t(float(cache_bias))
    _check(lib().chunk_attention(ring.ref, _ptr(q), n_q, int(q_pos0), int(n_current),
                                 None if m is None else ctypes.byref(m), ctypes.byref(b),
                                 float(softmax_scale), _ptr(out),
                                 None if lse is None else _ptr(lse),
                                 _flags(mode_b, pv_fp8), _stream(stream)),
           "chunk_attention")
    return out, lse


def chunk_attention_rows(ring: KvRing, q, q_pos0: int, n_current: int, rows, out, lse=None,
                         mask=None, cache_bias: float = 0.0, softmax_scale: float | None = None,
                         stream=None, mode_b: bool = False, n_splits: int = 1, workspace=None):
    """chunk_attention for the listed query rows only: q is the whole chunk (bf16
    [n_q][H][D]); rows is a device int32 tensor of chunk indices; out (bf16 [n_q][H][D])
    and lse (fp32 [H][n_q], optional) receive the listed rows and keep every other row.
    n_splits > 1 splits the keys (workspace: a device tensor of at least
    chunk_attention_workspace_size(len(rows), H, D, n_splits) bytes)."""
    import torch
    assert q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous()
    n_q = int(q.shape[0])
    assert q.shape == (n_q, ring.H, ring.D)
    assert rows.is_cuda and rows.dtype == torch.int32 and rows.is_contiguous() and rows.dim() == 1
    assert out.is_cuda and out.dtype == torch.bfloat16 and out.is_contiguous()
    assert out.shape == q.shape
    if lse is not None:
        assert lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous()
        assert lse.shape == (ring.H, n_q)
    if workspace is not None:
        assert workspace.is_cuda and workspace.is_contiguous()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(ring.D)
    m = None if mask is None else kv_block_mask_t(*(int(x) for x in mask))
    b = kv_cache_bias_t(float(cache_bias))
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().chunk_attention_rows(ring.ref, _ptr(q), n_q, int(q_pos0), int(n_current),
                                      _ptr(rows), int(rows.numel()),
                                      None if m is None else ctypes.byref(m), ctypes.byref(b),
                                      float(softmax_scale), _ptr(out),
                                      None if lse is None else _ptr(lse), int(n_splits),
                                      None if workspace is None else _ptr(workspace), nbytes,
                                      KV_QK_FP8 if mode_b else 0, _stream(stream)),
           "chunk_attention_rows")
    return out, lse


def chunk_attention_suggest_splits(n_q: int, n_heads: int, n_keys: int, n_sms: int = 148) -> int:
    """Key splits for chunk_attention_split that fill the GPU in whole waves."""
    return int(lib().chunk_attention_suggest_splits(int(n_q), int(n_heads), int(n_keys), int(n_sms)))


def chunk_attention_workspace_size(n_q: int, n_heads: int, head_dim: int, n_splits: int) -> int:
    return int(lib().chunk_attention_workspace_size(int(n_q), int(n_heads), int(head_dim),
                                                    int(n_splits)))


def chunk_attention_split(ring: KvRing, q, q_pos0: int, n_current: int, n_splits: int,
                          workspace, mask=None, cache_bias: float = 0.0,
                          softmax_scale: float | None = None, out=None, lse=None,
                          want_lse: bool = True, stream=None, mode_b: bool = False,
                          pv_fp8: bool = False):
    """chunk_attention with the keys split over n_splits groups; `workspace` is a device
    tensor of at least chunk_attention_workspace_size(...) bytes."""
    import torch
    assert q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous()
    n_q = int(q.shape[0])
    assert q.shape == (n_q, ring.H, ring.D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((ring.H, n_q), dtype=torch.float32, device=q.device)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(ring.D)
    m = None if mask is None else kv_block_mask_t(*(int(x) for x in mask))
    b = kv_cache_bias_t(float(cache_bias))
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().chunk_attention_split(ring.ref, _ptr(q), n_q, int(q_pos0), int(n_current),
                                       None if m is None else ctypes.byref(m), ctypes.byref(b),
                                       float(softmax_scale), _ptr(out),
                                       None if lse is None else _ptr(lse), int(n_splits),
                                       _ptr(workspace), nbytes, _flags(mode_b, pv_fp8),
                                       _stream(stream)),
           "chunk_attention_split")
    return out, lse


def chunk_attention_multi(rings, q, q_pos0: int, n_current: int, n_splits: int, workspace,
                          mask=None, cache_bias: float = 0.0, softmax_scale: float | None = None,
                          out=None, lse=None, want_lse: bool = True, stream=None,
                          mode_b: bool = False):
    """chunk_attention over rings[0], the stream's ring that holds the current chunk, and
    the history-only rings[1:] (a persistent anchor, for instance).  `workspace` is a
    device tensor of at least chunk_attention_workspace_size(n_q, H, D, len(rings) *
    n_splits) bytes."""
    import torch
    rings = list(rings)
    r0 = rings[0]
    assert q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous()
    n_q = int(q.shape[0])
    assert q.shape == (n_q, r0.H, r0.D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((r0.H, n_q), dtype=torch.float32, device=q.device)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(r0.D)
    m = None if mask is None else kv_block_mask_t(*(int(x) for x in mask))
    b = kv_cache_bias_t(float(cache_bias))
    arr = (ctypes.c_void_p * len(rings))(*[ctypes.addressof(r.s) for r in rings])
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().chunk_attention_multi(arr, len(rings), _ptr(q), n_q, int(q_pos0),
                                       int(n_current), None if m is None else ctypes.byref(m),
                                       ctypes.byref(b), float(softmax_scale), _ptr(out),
                                       None if lse is None else _ptr(lse), int(n_splits),
                                       _ptr(workspace), nbytes, KV_QK_FP8 if mode_b else 0,
                                       _stream(stream)),
           "chunk_attention_multi")
    return out, lse


def chunk_attention_split_noalloc(ring: KvRing, q, q_pos0: int, n_current: int, n_splits: int,
                                  out, lse=None, mask=None, cache_bias: float = 0.0,
                                  softmax_scale: float | None = None, stream=None,
                                  mode_b: bool = False):
    """chunk_attention_split with the library's static per-device scratch instead of a
    workspace; `out` (and `lse`, if wanted) are caller-allocated, so the call allocates
    nothing.  Calls that overlap in time on one device race on the scratch."""
    import torch
    assert q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous()
    n_q = int(q.shape[0])
    assert q.shape == (n_q, ring.H, ring.D)
    assert out.is_cuda and out.dtype == torch.bfloat16 and out.is_contiguous()
    assert out.shape == q.shape and out.device == q.device
    if lse is not None:
        assert lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous()
        assert lse.shape == (ring.H, n_q) and lse.device == q.device
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(ring.D)
    m = None if mask is None else kv_block_mask_t(*(int(x) for x in mask))
    b = kv_cache_bias_t(float(cache_bias))
    _check(lib().chunk_attention_split_noalloc(
        ring.ref, _ptr(q), n_q, int(q_pos0), int(n_current),
        None if m is None else ctypes.byref(m), ctypes.byref(b), float(softmax_scale),
        _ptr(out), None if lse is None else _ptr(lse), int(n_splits),
        KV_QK_FP8 if mode_b else 0, _stream(stream)),
        "chunk_attention_split_noalloc")
    return out, lse


def kv_wait_timeout_count() -> int:
    v = ctypes.c_uint32(0)
    _check(lib().kv_wait_timeout_count(ctypes.byref(v)), "kv_wait_timeout_count")
    return int(v.value)


def chunk_key_mass(main: KvRing, cand: KvRing, q, q_pos0: int, lse, slot_first: int,
                   n_cand: int, cache_bias: float = 0.0, softmax_scale: float | None = None,
                   mass=None, stream=None):
    """Attention mass [H][n_cand] (fp32, device) that slots (slot_first + c) mod C of
    `cand` receive in the attention call with these q, q_pos0, bias and its lse [H][n_q]."""
    import torch
    assert q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous()
    assert lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous()
    n_q = int(q.shape[0])
    if mass is None:
        mass = torch.empty((main.H, int(n_cand)), dtype=torch.float32, device=q.device)
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(main.D)
    b = kv_cache_bias_t(float(cache_bias))
    _check(lib().chunk_key_mass(main.ref, cand.ref, _ptr(q), n_q, int(q_pos0), _ptr(lse),
                                ctypes.byref(b), float(softmax_scale), int(slot_first),
                                int(n_cand), _ptr(mass), _stream(stream)),
           "chunk_key_mass")
    return mass


def chunk_key_mass_workspace_size(n_q: int, n_heads: int) -> int:
    return int(lib().chunk_key_mass_workspace_size(int(n_q), int(n_heads)))


def chunk_key_mass_multi(main: KvRing, cands, q, q_pos0: int, lse, slot_firsts, n_cands,
                         cache_bias: float = 0.0, softmax_scale: float | None = None,
                         masses=None, workspace=None, stream=None):
    """chunk_key_mass for several candidate sets (rings `cands`, first slots, counts) of
    one attention call in one launch.  `workspace` (device, at least
    chunk_key_mass_workspace_size bytes) lets the queries be split once per call.
    Returns the list of masses [H][n_cand] (fp32, device), one per set."""
    import torch
    assert q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous()
    assert lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous()
    n = len(cands)
    assert n == len(slot_firsts) == len(n_cands)
    if masses is None:
        masses = [torch.empty((main.H, int(c)), dtype=torch.float32, device=q.device)
                  for c in n_cands]
    assert len(masses) == n
    for m, c in zip(masses, n_cands):
        assert m.is_cuda and m.dtype == torch.float32 and m.is_contiguous()
        assert m.numel() >= main.H * int(c)
    if workspace is not None:
        assert workspace.is_cuda and workspace.is_contiguous()
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(main.D)
    b = kv_cache_bias_t(float(cache_bias))
    rings = (ctypes.c_void_p * n)(*[ctypes.addressof(c.s) for c in cands])
    firsts = (ctypes.c_int64 * n)(*[int(f) for f in slot_firsts])
    counts = (ctypes.c_int * n)(*[int(c) for c in n_cands])
    outs = (ctypes.c_void_p * n)(*[_ptr(m) for m in masses])
    ws = None if workspace is None else _ptr(workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().chunk_key_mass_multi(main.ref, n, rings, _ptr(q), int(q.shape[0]), int(q_pos0),
                                      _ptr(lse), ctypes.byref(b), float(softmax_scale), firsts,
                                      counts, outs, ws, ws_bytes, _stream(stream)),
           "chunk_key_mass_multi")
    return masses


def kv_memory_select(memory, mass_memory, fifo: KvRing, mass_fifo, fifo_slot_first: int,
                     n_fifo: int, budget: int, frame_len: int, memory_out: KvRing,
                     gamma: float = 0.5, kept=None, stream=None):
    """Keep the best min(n, budget) of the memory's valid slots and the FIFO block by the
    temporal-diversity rule; copy them into memory_out's slots 0 .. kept - 1.  Returns the
    kept candidate indices (device int32, ascending)."""
    import torch
    n_mem = 0 if memory is None else memory.n_valid
    m = min(n_mem + int(n_fifo), int(budget))
    if kept is None:
        kept = torch.empty((max(1, m),), dtype=torch.int32, device=fifo.k_codes.device)
    _check(lib().kv_memory_select(None if memory is None else memory.ref,
                                  None if mass_memory is None else _ptr(mass_memory), fifo.ref,
                                  None if mass_fifo is None else _ptr(mass_fifo),
                                  int(fifo_slot_first), int(n_fifo), int(budget), int(frame_len),
                                  float(gamma), memory_out.ref, _ptr(kept), _stream(stream)),
           "kv_memory_select")
    return kept[:m]
