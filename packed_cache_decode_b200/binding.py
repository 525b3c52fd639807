"""Thin ctypes binding of libbgtq (include/bgtq.h): argument marshalling only.

Every step of the path runs inside the library. If ``libbgtq.so`` is missing the
binding raises; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbgtq.so")
_lib = None

OK, ERR_INVALID, ERR_INFEASIBLE, ERR_CAPACITY, ERR_CUDA, ERR_NOMEM, ERR_WORKSPACE, ERR_DEVICE = range(8)
F32, BF16, F16 = 0, 1, 2
HEAD_DIM = 128
TILE_TOKENS = 64
STATUS_ENCODE_OVERFLOW = 1
STATUS_DECODE_CLAMPED = 2
STATUS_TIMEOUT = 4
STATUS_BAD_PAGE = 8
LAYOUT_NORM_CORRECT = 1
LAYOUT_NORM_FP16 = 2

EXPORTED = [
    "bgtq_last_error_string", "bgtq_version", "bgtq_lloyd_max", "bgtq_block_energy", "bgtq_allocate_rates",
    "bgtq_layout_create", "bgtq_layout_create_ex", "bgtq_layout_destroy", "bgtq_layout_get_info", "bgtq_layout_rotation",
    "bgtq_layout_coords", "bgtq_cache_bytes", "bgtq_layout_upload", "bgtq_encode_append",
    "bgtq_workspace_bytes", "bgtq_decode_attention", "bgtq_device_status",
    "bgtq_decode_attention_noalloc", "bgtq_noalloc_scratch_capacity", "bgtq_decode_step", "bgtq_decode_scores",
    "bgtq_paged_pool_bytes", "bgtq_encode_append_paged", "bgtq_decode_attention_paged", "bgtq_decode_step_paged",
    "bgtq_decode_attention_multi", "bgtq_decode_step_multi", "bgtq_decode_step_multi_paged",
    "bgtq_block_energy_heads", "bgtq_decode_attention_partial", "bgtq_merge_partials",
    "bgtq_layout_set_create", "bgtq_layout_set_destroy", "bgtq_layout_set_tile_bytes", "bgtq_layout_set_cache_bytes",
    "bgtq_encode_append_heads", "bgtq_decode_attention_heads", "bgtq_decode_scores_heads", "bgtq_layout_set_status",
    "bgtq_decode_step_heads", "bgtq_layout_set_paged_pool_bytes", "bgtq_encode_append_paged_heads",
    "bgtq_decode_attention_paged_heads", "bgtq_decode_attention_multi_heads", "bgtq_decode_step_multi_heads",
    "bgtq_decode_step_paged_heads",
]


class LayoutInfo(C.Structure):
    _fields_ = [("head_dim", C.c_int), ("n_blocks", C.c_int), ("n_kgroups", C.c_int),
                ("group_rate", C.c_int * 4), ("group_dim", C.c_int * 4), ("v_rate", C.c_int),
                ("k_record_bytes", C.c_int), ("v_record_bytes", C.c_int), ("bytes_per_token", C.c_int),
                ("tile_tokens", C.c_int), ("tile_bytes", C.c_int), ("seed", C.c_ulonglong),
                ("flags", C.c_uint), ("norm_bytes", C.c_int), ("n_packed", C.c_int)]


class BgtqError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: status {status}: {msg}")
        self.status = status


def load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"libbgtq.so not built ({_LIB_PATH}); run python -m packed_cache_decode_b200.build_lib")
    lib = C.CDLL(_LIB_PATH)
    P, I, LL, D, F, U = C.c_void_p, C.c_int, C.c_longlong, C.c_double, C.c_float, C.c_ulonglong
    sig = {
        "bgtq_last_error_string": (C.c_char_p, []),
        "bgtq_version": (I, []),
        "bgtq_lloyd_max": (I, [I, P, P, P]),
        "bgtq_block_energy": (I, [P, LL, I, P, LL, I, P]),
        "bgtq_block_energy_heads": (I, [P, LL, I, P, LL, I, P]),
        "bgtq_allocate_rates": (I, [P, I, I, I, LL, P, P]),
        "bgtq_layout_create": (I, [P, I, U, C.POINTER(P)]),
        "bgtq_layout_create_ex": (I, [P, I, U, C.c_uint, C.POINTER(P)]),
        "bgtq_layout_destroy": (None, [P]),
        "bgtq_layout_get_info": (I, [P, C.POINTER(LayoutInfo)]),
        "bgtq_layout_rotation": (I, [P, I, P, LL]),
        "bgtq_layout_coords": (I, [P, P]),
        "bgtq_cache_bytes": (LL, [P, I, I, LL]),
        "bgtq_layout_upload": (I, [P, I]),
        "bgtq_encode_append": (I, [P, P, P, I, I, I, I, P, P, LL, P]),
        "bgtq_workspace_bytes": (C.c_size_t, [P, I, I, I, LL]),
        "bgtq_decode_attention": (I, [P, P, I, I, I, I, P, P, LL, LL, F, P, P, C.c_size_t, P]),
        "bgtq_device_status": (I, [P, C.POINTER(C.c_uint), I]),
        "bgtq_decode_attention_partial": (I, [P, P, I, I, I, I, P, P, LL, LL, F, P, P, C.c_size_t, P]),
        "bgtq_merge_partials": (I, [P, P, I, I, I, P, P]),
        "bgtq_decode_attention_noalloc": (I, [P, P, I, I, I, I, P, P, LL, LL, F, P, P]),
        "bgtq_noalloc_scratch_capacity": (C.c_size_t, []),
        "bgtq_decode_step": (I, [P, P, P, I, I, P, I, I, I, I, P, P, LL, LL, F, P, P, C.c_size_t, P]),
        "bgtq_decode_scores": (I, [P, P, I, I, I, I, P, P, LL, LL, F, P, LL, P, C.c_size_t, P]),
        "bgtq_paged_pool_bytes": (LL, [P, I, LL]),
        "bgtq_encode_append_paged": (I, [P, P, P, I, I, I, I, P, P, LL, P, LL, P]),
        "bgtq_decode_attention_paged": (I, [P, P, I, I, I, I, P, LL, P, LL, P, LL, F, P, P, C.c_size_t, P]),
        "bgtq_decode_step_paged": (I, [P, P, P, I, I, P, I, I, I, I, P, LL, P, LL, P, LL, F, P, P, C.c_size_t, P]),
        "bgtq_decode_attention_multi": (I, [P, P, I, I, I, I, I, P, P, LL, LL, F, P, P, C.c_size_t, P]),
        "bgtq_decode_step_multi": (I, [P, P, P, I, I, P, I, I, I, I, P, P, LL, LL, F, P, P, C.c_size_t, P]),
        "bgtq_decode_step_multi_paged": (I, [P, P, P, I, I, P, I, I, I, I, P, LL, P, LL, P, LL, F, P, P, C.c_size_t,
                                             P]),
        "bgtq_layout_set_create": (I, [P, I, C.POINTER(P)]),
        "bgtq_layout_set_destroy": (None, [P]),
        "bgtq_layout_set_tile_bytes": (I, [P]),
        "bgtq_layout_set_cache_bytes": (C.c_size_t, [P, I, LL]),
        "bgtq_encode_append_heads": (I, [P, P, P, I, I, I, P, P, LL, P]),
        "bgtq_decode_attention_heads": (I, [P, P, I, I, I, P, P, LL, LL, F, P, P, C.c_size_t, P]),
        "bgtq_decode_scores_heads": (I, [P, P, I, I, I, P, P, LL, LL, F, P, LL, P, C.c_size_t, P]),
        "bgtq_layout_set_status": (I, [P, C.POINTER(C.c_uint), I]),
        "bgtq_decode_step_heads": (I, [P, P, P, I, I, P, I, I, I, P, P, LL, LL, F, P, P, C.c_size_t, P]),
        "bgtq_layout_set_paged_pool_bytes": (LL, [P, LL]),
        "bgtq_encode_append_paged_heads": (I, [P, P, P, I, I, I, P, P, LL, P, LL, P]),
        "bgtq_decode_attention_paged_heads": (I, [P, P, I, I, I, P, LL, P, LL, P, LL, F, P, P, C.c_size_t, P]),
        "bgtq_decode_attention_multi_heads": (I, [P, P, I, I, I, I, P, P, LL, LL, F, P, P, C.c_size_t, P]),
        "bgtq_decode_step_multi_heads": (I, [P, P, P, I, I, P, I, I, I, P, P, LL, LL, F, P, P, C.c_size_t, P]),
        "bgtq_decode_step_paged_heads": (I, [P, P, P, I, I, P, I, I, I, P, LL, P, LL, P, LL, F, P, P, C.c_size_t,
                                             P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != OK:
        raise BgtqError(status, where, load().bgtq_last_error_string().decode())


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


# ---------------------------------------------------------------- host planning
def lloyd_max(bits: int):
    c = np.zeros(1 << bits)
    t = np.zeros((1 << bits) - 1)
    m = np.zeros(1)
    _check(load().bgtq_lloyd_max(bits, _ptr(c), _ptr(t), _ptr(m)), "lloyd_max")
    return c, t, float(m[0])


def block_energy(q_cal, k_cal) -> np.ndarray:
    q = np.ascontiguousarray(q_cal, dtype=np.float32)
    k = np.ascontiguousarray(k_cal, dtype=np.float32)
    s = np.zeros(64)
    _check(load().bgtq_block_energy(_ptr(q), q.shape[0], q.shape[1], _ptr(k), k.shape[0], k.shape[1], _ptr(s)),
           "block_energy")
    return s


def block_energy_heads(q_cal, k_cal) -> np.ndarray:
    """Energy score per KV head, [h_kv, 64] (their sum is block_energy)."""
    q = np.ascontiguousarray(q_cal, dtype=np.float32)
    k = np.ascontiguousarray(k_cal, dtype=np.float32)
    s = np.zeros((k.shape[1], 64))
    _check(load().bgtq_block_energy_heads(_ptr(q), q.shape[0], q.shape[1], _ptr(k), k.shape[0], k.shape[1], _ptr(s)),
           "block_energy_heads")
    return s


def allocate_rates(score, min_rate: int, max_rate: int, total_bits: int, distortion=None) -> np.ndarray:
    s = np.ascontiguousarray(score, dtype=np.float64)
    out = np.zeros(len(s), dtype=np.int32)
    dptr = None
    if distortion is not None:
        d = np.zeros(6)
        for r, v in dict(distortion).items():
            d[r] = v
        dptr = _ptr(d)
    _check(load().bgtq_allocate_rates(_ptr(s), len(s), min_rate, max_rate, total_bits, dptr, _ptr(out)),
           "allocate_rates")
    return out


class Layout:
    """A layer's packing layout (owns the C handle)."""

    def __init__(self, k_rates, v_rate: int, seed: int, norm_correct: bool = False, norm_fp16: bool = False):
        lib = load()
        r = np.ascontiguousarray(k_rates, dtype=np.int32)
        if r.shape != (64,):
            raise ValueError("64 block rates expected")
        h = C.c_void_p()
        flags = (LAYOUT_NORM_CORRECT if norm_correct else 0) | (LAYOUT_NORM_FP16 if norm_fp16 else 0)
        _check(lib.bgtq_layout_create_ex(_ptr(r), int(v_rate), C.c_ulonglong(seed), flags, C.byref(h)),
               "layout_create")
        self._h = h
        self.k_rates = r.copy()
        self.v_rate = int(v_rate)
        self.seed = int(seed)
        self.norm_correct = bool(norm_correct)
        self.norm_fp16 = bool(norm_fp16)
        info = LayoutInfo()
        _check(lib.bgtq_layout_get_info(h, C.byref(info)), "layout_get_info")
        self.info = info
        self.device = None

    @property
    def handle(self):
        return self._h

    @property
    def n_kgroups(self):
        return self.info.n_kgroups

    @property
    def bytes_per_token(self):
        return self.info.bytes_per_token

    @property
    def tile_bytes(self):
        return self.info.tile_bytes

    def rotation(self, group: int) -> np.ndarray:
        d = self.info.group_dim[group] if group < self.n_kgroups else HEAD_DIM
        out = np.zeros((d, d))
        _check(load().bgtq_layout_rotation(self._h, group, _ptr(out), out.size), "layout_rotation")
        return out

    def coords(self) -> np.ndarray:
        out = np.zeros(128, dtype=np.int32)
        _check(load().bgtq_layout_coords(self._h, _ptr(out)), "layout_coords")
        return out

    def cache_bytes(self, batch: int, h_kv: int, tokens: int) -> int:
        n = load().bgtq_cache_bytes(self._h, batch, h_kv, tokens)
        if n < 0:
            _check(ERR_INVALID, "cache_bytes")
        return int(n)

    def upload(self, device: int = 0):
        _check(load().bgtq_layout_upload(self._h, device), "layout_upload")
        self.device = device
        return self

    def status(self, clear: bool = True) -> int:
        f = C.c_uint(0)
        _check(load().bgtq_device_status(self._h, C.byref(f), int(clear)), "device_status")
        return int(f.value)

    def close(self):
        if self._h:
            load().bgtq_layout_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class LayoutSet:
    """The uploaded layouts of the KV heads of one layer, in head order (owns the C handle;
    keeps the layouts alive)."""

    def __init__(self, layouts):
        self.layouts = list(layouts)
        arr = (C.c_void_p * len(self.layouts))(*[lay.handle for lay in self.layouts])
        h = C.c_void_p()
        _check(load().bgtq_layout_set_create(arr, len(self.layouts), C.byref(h)), "layout_set_create")
        self._h = h

    @property
    def handle(self):
        return self._h

    @property
    def h_kv(self):
        return len(self.layouts)

    @property
    def tile_bytes(self):
        return int(load().bgtq_layout_set_tile_bytes(self._h))

    def cache_bytes(self, batch: int, capacity: int) -> int:
        n = load().bgtq_layout_set_cache_bytes(self._h, batch, capacity)
        if n == 0:
            _check(ERR_INVALID, "layout_set_cache_bytes")
        return int(n)

    def paged_pool_bytes(self, num_pages: int) -> int:
        n = load().bgtq_layout_set_paged_pool_bytes(self._h, num_pages)
        if n < 0:
            _check(ERR_INVALID, "layout_set_paged_pool_bytes")
        return int(n)

    def status(self, clear: bool = True) -> int:
        f = C.c_uint(0)
        _check(load().bgtq_layout_set_status(self._h, C.byref(f), int(clear)), "layout_set_status")
        return int(f.value)

    def close(self):
        if self._h:
            load().bgtq_layout_set_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ---------------------------------------------------------------- device calls
_DTYPES = {}


def dtype_code(t) -> int:
    import torch
    if not _DTYPES:
        _DTYPES.update({torch.float32: F32, torch.bfloat16: BF16, torch.float16: F16})
    return _DTYPES[t.dtype]


def _stream_ptr(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def encode_append(layout: Layout, k, v, seq_lens, cache, capacity: int, stream=None):
    """k, v [B, n_new, h_kv, 128] CUDA tensors; seq_lens [B] int32 CUDA; cache uint8 CUDA."""
    B, n_new, h_kv, d = k.shape
    assert d == HEAD_DIM and k.is_contiguous() and v.is_contiguous() and v.shape == k.shape and v.dtype == k.dtype
    _check(load().bgtq_encode_append(layout.handle, C.c_void_p(k.data_ptr()), C.c_void_p(v.data_ptr()),
                                     dtype_code(k), B, n_new, h_kv, C.c_void_p(seq_lens.data_ptr()),
                                     C.c_void_p(cache.data_ptr()), capacity, _stream_ptr(stream)),
           "encode_append")


def workspace_bytes(layout: Layout, batch: int, h_q: int, h_kv: int, max_seq_len: int) -> int:
    n = load().bgtq_workspace_bytes(layout.handle, batch, h_q, h_kv, max_seq_len)
    if n == 0:
        _check(ERR_INVALID, "workspace_bytes")
    return int(n)


def decode_attention(layout: Layout, q, cache, seq_lens, capacity: int, max_seq_len: int, out, workspace,
                     h_kv: int, softmax_scale: float | None = None, stream=None):
    """q [B, h_q, 128] CUDA; out [B, h_q, 128] fp32 CUDA; workspace uint8 CUDA."""
    B, h_q, d = q.shape
    assert d == HEAD_DIM and q.is_contiguous() and out.is_contiguous()
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_attention(layout.handle, C.c_void_p(q.data_ptr()), dtype_code(q), B, h_q, h_kv,
                                        C.c_void_p(cache.data_ptr()), C.c_void_p(seq_lens.data_ptr()), capacity,
                                        max_seq_len, scale, C.c_void_p(out.data_ptr()),
                                        C.c_void_p(workspace.data_ptr()), workspace.numel(), _stream_ptr(stream)),
           "decode_attention")


PARTIAL_RECORD = HEAD_DIM + 2   # (m, l, o'[128]) per query head


def decode_attention_partial(layout: Layout, q, cache, seq_lens, capacity: int, max_seq_len: int, partial,
                             workspace, h_kv: int, softmax_scale: float | None = None, stream=None):
    """Attention over this cache's part of every row's tokens, as mergeable records:
    q [B, h_q, 128] CUDA; partial [B, h_q, 130] fp32 CUDA receives (m, l, o') per head."""
    B, h_q, d = q.shape
    assert d == HEAD_DIM and q.is_contiguous() and partial.is_contiguous()
    assert tuple(partial.shape) == (B, h_q, PARTIAL_RECORD) and str(partial.dtype) == "torch.float32"
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_attention_partial(layout.handle, C.c_void_p(q.data_ptr()), dtype_code(q), B, h_q, h_kv,
                                                C.c_void_p(cache.data_ptr()), C.c_void_p(seq_lens.data_ptr()),
                                                capacity, max_seq_len, scale, C.c_void_p(partial.data_ptr()),
                                                C.c_void_p(workspace.data_ptr()), workspace.numel(),
                                                _stream_ptr(stream)),
           "decode_attention_partial")


def merge_partials(layout: Layout, partials, out, stream=None):
    """partials [n_parts, B, h_q, 130] fp32 CUDA (records over disjoint token ranges);
    out [B, h_q, 128] fp32 CUDA = attention over the union of the ranges."""
    n, B, h_q, r = partials.shape
    assert r == PARTIAL_RECORD and partials.is_contiguous() and out.is_contiguous()
    assert tuple(out.shape) == (B, h_q, HEAD_DIM)
    _check(load().bgtq_merge_partials(layout.handle, C.c_void_p(partials.data_ptr()), n, B, h_q,
                                      C.c_void_p(out.data_ptr()), _stream_ptr(stream)), "merge_partials")


def decode_step(layout: Layout, k_new, v_new, q, cache, seq_lens, capacity: int, max_seq_len: int, out, workspace,
                softmax_scale: float | None = None, stream=None):
    """Append k_new, v_new [B, n_new, h_kv, 128] at seq_lens[b] (int32 CUDA, not advanced)
    and attend q [B, h_q, 128] over seq_lens[b] + n_new tokens; out [B, h_q, 128] fp32."""
    B_, n_new, h_kv, d = k_new.shape
    assert d == HEAD_DIM and k_new.is_contiguous() and v_new.is_contiguous()
    assert v_new.shape == k_new.shape and v_new.dtype == k_new.dtype
    Bq, h_q, dq = q.shape
    assert Bq == B_ and dq == HEAD_DIM and q.is_contiguous() and out.is_contiguous()
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_step(layout.handle, C.c_void_p(k_new.data_ptr()), C.c_void_p(v_new.data_ptr()),
                                   dtype_code(k_new), n_new, C.c_void_p(q.data_ptr()), dtype_code(q), B_, h_q, h_kv,
                                   C.c_void_p(cache.data_ptr()), C.c_void_p(seq_lens.data_ptr()), capacity,
                                   max_seq_len, scale, C.c_void_p(out.data_ptr()),
                                   C.c_void_p(workspace.data_ptr()), workspace.numel(), _stream_ptr(stream)),
           "decode_step")


def decode_scores(layout: Layout, q, cache, seq_lens, capacity: int, max_seq_len: int, scores, workspace,
                  h_kv: int, softmax_scale: float | None = None, stream=None):
    """Logits softmax_scale * q . k_hat over the packed cache: scores [B, h_q, >= max_seq_len]
    fp32 CUDA (entries past each row's length are left as they are)."""
    B_, h_q, d = q.shape
    assert d == HEAD_DIM and q.is_contiguous() and scores.is_contiguous() and scores.shape[:2] == (B_, h_q)
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_scores(layout.handle, C.c_void_p(q.data_ptr()), dtype_code(q), B_, h_q, h_kv,
                                     C.c_void_p(cache.data_ptr()), C.c_void_p(seq_lens.data_ptr()), capacity,
                                     max_seq_len, scale, C.c_void_p(scores.data_ptr()), scores.shape[2],
                                     C.c_void_p(workspace.data_ptr()), workspace.numel(), _stream_ptr(stream)),
           "decode_scores")


class PagedCache:
    """A pool of pages (uint8 CUDA tensor) and a block table [batch, max_pages] (int32 CUDA):
    page p holds the h_kv tiles of one 64-token span of one row."""

    def __init__(self, pool, block_table):
        import torch
        assert pool.dtype == torch.uint8 and block_table.dtype == torch.int32
        assert block_table.is_contiguous() and block_table.dim() == 2
        self.pool, self.table = pool, block_table

    def num_pages(self, layout: "Layout", h_kv: int) -> int:
        return self.pool.numel() // (h_kv * layout.tile_bytes)

    @property
    def max_pages(self) -> int:
        return self.table.shape[1]


def paged_pool_bytes(layout: Layout, h_kv: int, num_pages: int) -> int:
    n = load().bgtq_paged_pool_bytes(layout.handle, h_kv, num_pages)
    if n < 0:
        _check(ERR_INVALID, "paged_pool_bytes")
    return int(n)


def encode_append_paged(layout: Layout, k, v, seq_lens, cache: PagedCache, stream=None):
    """k, v [B, n_new, h_kv, 128]; tokens go to the pages the block table names."""
    B_, n_new, h_kv, d = k.shape
    assert d == HEAD_DIM and k.is_contiguous() and v.is_contiguous() and v.shape == k.shape and v.dtype == k.dtype
    _check(load().bgtq_encode_append_paged(layout.handle, C.c_void_p(k.data_ptr()), C.c_void_p(v.data_ptr()),
                                           dtype_code(k), B_, n_new, h_kv, C.c_void_p(seq_lens.data_ptr()),
                                           C.c_void_p(cache.pool.data_ptr()), cache.num_pages(layout, h_kv),
                                           C.c_void_p(cache.table.data_ptr()), cache.max_pages, _stream_ptr(stream)),
           "encode_append_paged")


def decode_attention_paged(layout: Layout, q, cache: PagedCache, seq_lens, max_seq_len: int, out, workspace,
                           h_kv: int, softmax_scale: float | None = None, stream=None):
    B_, h_q, d = q.shape
    assert d == HEAD_DIM and q.is_contiguous() and out.is_contiguous()
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_attention_paged(layout.handle, C.c_void_p(q.data_ptr()), dtype_code(q), B_, h_q, h_kv,
                                              C.c_void_p(cache.pool.data_ptr()), cache.num_pages(layout, h_kv),
                                              C.c_void_p(cache.table.data_ptr()), cache.max_pages,
                                              C.c_void_p(seq_lens.data_ptr()), max_seq_len, scale,
                                              C.c_void_p(out.data_ptr()), C.c_void_p(workspace.data_ptr()),
                                              workspace.numel(), _stream_ptr(stream)),
           "decode_attention_paged")


def decode_step_paged(layout: Layout, k_new, v_new, q, cache: PagedCache, seq_lens, max_seq_len: int, out,
                      workspace, softmax_scale: float | None = None, stream=None):
    B_, n_new, h_kv, d = k_new.shape
    assert d == HEAD_DIM and k_new.is_contiguous() and v_new.is_contiguous() and v_new.shape == k_new.shape
    Bq, h_q, dq = q.shape
    assert Bq == B_ and dq == HEAD_DIM and q.is_contiguous() and out.is_contiguous()
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_step_paged(layout.handle, C.c_void_p(k_new.data_ptr()), C.c_void_p(v_new.data_ptr()),
                                         dtype_code(k_new), n_new, C.c_void_p(q.data_ptr()), dtype_code(q), B_, h_q,
                                         h_kv, C.c_void_p(cache.pool.data_ptr()), cache.num_pages(layout, h_kv),
                                         C.c_void_p(cache.table.data_ptr()), cache.max_pages,
                                         C.c_void_p(seq_lens.data_ptr()), max_seq_len, scale,
                                         C.c_void_p(out.data_ptr()), C.c_void_p(workspace.data_ptr()),
                                         workspace.numel(), _stream_ptr(stream)),
           "decode_step_paged")


def decode_attention_multi(layout: Layout, q, cache, seq_lens, capacity: int, max_seq_len: int, out, workspace,
                           h_kv: int, softmax_scale: float | None = None, stream=None):
    """n_q query tokens per row, causal among them: q [B, n_q, h_q, 128] CUDA (the last n_q
    of each row's seq_lens[b] cached tokens); out [B, n_q, h_q, 128] fp32. The workspace is
    sized by workspace_bytes(layout, B, h_q * n_q, h_kv, max_seq_len)."""
    B_, n_q, h_q, d = q.shape
    assert d == HEAD_DIM and q.is_contiguous() and out.is_contiguous()
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_attention_multi(layout.handle, C.c_void_p(q.data_ptr()), dtype_code(q), B_, n_q, h_q,
                                              h_kv, C.c_void_p(cache.data_ptr()), C.c_void_p(seq_lens.data_ptr()),
                                              capacity, max_seq_len, scale, C.c_void_p(out.data_ptr()),
                                              C.c_void_p(workspace.data_ptr()), workspace.numel(), _stream_ptr(stream)),
           "decode_attention_multi")


def decode_step_multi(layout: Layout, k_new, v_new, q, cache, seq_lens, capacity: int, max_seq_len: int, out,
                      workspace, softmax_scale: float | None = None, stream=None):
    """Append k_new, v_new [B, n_new, h_kv, 128] at seq_lens[b] (not advanced) and attend with
    the new tokens' queries q [B, n_new, h_q, 128], causal among them; out [B, n_new, h_q, 128]."""
    B_, n_new, h_kv, d = k_new.shape
    assert d == HEAD_DIM and k_new.is_contiguous() and v_new.is_contiguous() and v_new.shape == k_new.shape
    Bq, nq, h_q, dq = q.shape
    assert Bq == B_ and nq == n_new and dq == HEAD_DIM and q.is_contiguous() and out.is_contiguous()
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_step_multi(layout.handle, C.c_void_p(k_new.data_ptr()), C.c_void_p(v_new.data_ptr()),
                                         dtype_code(k_new), n_new, C.c_void_p(q.data_ptr()), dtype_code(q), B_, h_q,
                                         h_kv, C.c_void_p(cache.data_ptr()), C.c_void_p(seq_lens.data_ptr()), capacity,
                                         max_seq_len, scale, C.c_void_p(out.data_ptr()),
                                         C.c_void_p(workspace.data_ptr()), workspace.numel(), _stream_ptr(stream)),
           "decode_step_multi")


def decode_step_multi_paged(layout: Layout, k_new, v_new, q, cache: PagedCache, seq_lens, max_seq_len: int, out,
                            workspace, softmax_scale: float | None = None, stream=None):
    B_, n_new, h_kv, d = k_new.shape
    assert d == HEAD_DIM and k_new.is_contiguous() and v_new.is_contiguous() and v_new.shape == k_new.shape
    Bq, nq, h_q, dq = q.shape
    assert Bq == B_ and nq == n_new and dq == HEAD_DIM and q.is_contiguous() and out.is_contiguous()
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_step_multi_paged(layout.handle, C.c_void_p(k_new.data_ptr()),
                                               C.c_void_p(v_new.data_ptr()), dtype_code(k_new), n_new,
                                               C.c_void_p(q.data_ptr()), dtype_code(q), B_, h_q, h_kv,
                                               C.c_void_p(cache.pool.data_ptr()), cache.num_pages(layout, h_kv),
                                               C.c_void_p(cache.table.data_ptr()), cache.max_pages,
                                               C.c_void_p(seq_lens.data_ptr()), max_seq_len, scale,
                                               C.c_void_p(out.data_ptr()), C.c_void_p(workspace.data_ptr()),
                                               workspace.numel(), _stream_ptr(stream)),
           "decode_step_multi_paged")


def decode_attention_noalloc(layout: Layout, q, cache, seq_lens, capacity: int, max_seq_len: int, out,
                             h_kv: int, softmax_scale: float | None = None, stream=None):
    """decode_attention for callers that cannot allocate device memory: the split-K
    scratch is the library's fixed device array, not a caller workspace. Calls that
    overlap on the GPU race on that array, so keep them on one stream."""
    B_, h_q, d = q.shape
    assert d == HEAD_DIM and q.is_contiguous() and out.is_contiguous()
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_attention_noalloc(layout.handle, C.c_void_p(q.data_ptr()), dtype_code(q), B_, h_q,
                                                h_kv, C.c_void_p(cache.data_ptr()), C.c_void_p(seq_lens.data_ptr()),
                                                capacity, max_seq_len, scale, C.c_void_p(out.data_ptr()),
                                                _stream_ptr(stream)),
           "decode_attention_noalloc")


def plan_layer_rates(q_cal, k_cal, avg_bits: int, min_rate: int = 1, max_rate: int = 4) -> np.ndarray:
    """Energy score + largest-marginal-gain allocation for one layer (library calls)."""
    s = block_energy(q_cal, k_cal)
    return allocate_rates(s, min_rate, max_rate, 64 * avg_bits)


def plan_head_rates(q_cal, k_cal, avg_bits: int, min_rate: int = 1, max_rate: int = 4) -> np.ndarray:
    """Rates per KV head, [h_kv, 64]: each head's own energy score and allocation (each row
    is the rate vector of that head's own layout)."""
    s = block_energy_heads(q_cal, k_cal)
    return np.stack([allocate_rates(s[h], min_rate, max_rate, 64 * avg_bits) for h in range(s.shape[0])])


# ---------------------------------------------------------------- one layout per KV head
def encode_append_heads(layouts: LayoutSet, k, v, seq_lens, cache, capacity: int, stream=None):
    """k, v [B, n_new, h_kv, 128] CUDA (h_kv = the set's size); KV head h coded with layout h."""
    B, n_new, h_kv, d = k.shape
    assert d == HEAD_DIM and h_kv == layouts.h_kv and k.is_contiguous() and v.is_contiguous()
    assert v.shape == k.shape and v.dtype == k.dtype
    _check(load().bgtq_encode_append_heads(layouts.handle, C.c_void_p(k.data_ptr()), C.c_void_p(v.data_ptr()),
                                           dtype_code(k), B, n_new, C.c_void_p(seq_lens.data_ptr()),
                                           C.c_void_p(cache.data_ptr()), capacity, _stream_ptr(stream)),
           "encode_append_heads")


def decode_attention_heads(layouts: LayoutSet, q, cache, seq_lens, capacity: int, max_seq_len: int, out, workspace,
                           softmax_scale: float | None = None, stream=None):
    """One decode-attention call over every KV head of a cache written by encode_append_heads."""
    B, h_q, d = q.shape
    assert d == HEAD_DIM and q.is_contiguous() and out.is_contiguous()
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_attention_heads(layouts.handle, C.c_void_p(q.data_ptr()), dtype_code(q), B, h_q,
                                              C.c_void_p(cache.data_ptr()), C.c_void_p(seq_lens.data_ptr()), capacity,
                                              max_seq_len, scale, C.c_void_p(out.data_ptr()),
                                              C.c_void_p(workspace.data_ptr()), workspace.numel(), _stream_ptr(stream)),
           "decode_attention_heads")


def decode_scores_heads(layouts: LayoutSet, q, cache, seq_lens, capacity: int, max_seq_len: int, scores, workspace,
                        softmax_scale: float | None = None, stream=None):
    """Logits of every KV head of a cache written by encode_append_heads: scores [B, h_q, ld]."""
    B, h_q, d = q.shape
    assert d == HEAD_DIM and q.is_contiguous() and scores.is_contiguous()
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_scores_heads(layouts.handle, C.c_void_p(q.data_ptr()), dtype_code(q), B, h_q,
                                           C.c_void_p(cache.data_ptr()), C.c_void_p(seq_lens.data_ptr()), capacity,
                                           max_seq_len, scale, C.c_void_p(scores.data_ptr()), scores.shape[-1],
                                           C.c_void_p(workspace.data_ptr()), workspace.numel(), _stream_ptr(stream)),
           "decode_scores_heads")


def decode_step_heads(layouts: LayoutSet, k_new, v_new, q, cache, seq_lens, capacity: int, max_seq_len: int, out,
                      workspace, softmax_scale: float | None = None, stream=None):
    """Append k_new, v_new [B, n_new, h_kv, 128] (KV head h with layout h of the set) at
    seq_lens[b] and attend q [B, h_q, 128] over seq_lens[b] + n_new tokens, one chain."""
    B_, n_new, h_kv, d = k_new.shape
    assert d == HEAD_DIM and h_kv == layouts.h_kv and k_new.is_contiguous() and v_new.is_contiguous()
    assert q.is_contiguous() and out.is_contiguous()
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_step_heads(layouts.handle, C.c_void_p(k_new.data_ptr()), C.c_void_p(v_new.data_ptr()),
                                         dtype_code(k_new), n_new, C.c_void_p(q.data_ptr()), dtype_code(q), B_,
                                         q.shape[1], C.c_void_p(cache.data_ptr()), C.c_void_p(seq_lens.data_ptr()),
                                         capacity, max_seq_len, scale, C.c_void_p(out.data_ptr()),
                                         C.c_void_p(workspace.data_ptr()), workspace.numel(), _stream_ptr(stream)),
           "decode_step_heads")


def encode_append_paged_heads(layouts: LayoutSet, k, v, seq_lens, pc, stream=None):
    """encode_append_heads into a paged cache pc (a PagedCache over a pool of the set's pages)."""
    B_, n_new, h_kv, d = k.shape
    assert d == HEAD_DIM and h_kv == layouts.h_kv and k.is_contiguous() and v.is_contiguous()
    _check(load().bgtq_encode_append_paged_heads(layouts.handle, C.c_void_p(k.data_ptr()), C.c_void_p(v.data_ptr()),
                                                 dtype_code(k), B_, n_new, C.c_void_p(seq_lens.data_ptr()),
                                                 C.c_void_p(pc.pool.data_ptr()),
                                                 pc.pool.numel() // (layouts.h_kv * layouts.tile_bytes),
                                                 C.c_void_p(pc.table.data_ptr()), pc.max_pages, _stream_ptr(stream)),
           "encode_append_paged_heads")


def decode_attention_paged_heads(layouts: LayoutSet, q, pc, seq_lens, max_seq_len: int, out, workspace,
                                 softmax_scale: float | None = None, stream=None):
    """decode_attention_heads over a paged cache pc."""
    B_, h_q, d = q.shape
    assert d == HEAD_DIM and q.is_contiguous() and out.is_contiguous()
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_attention_paged_heads(layouts.handle, C.c_void_p(q.data_ptr()), dtype_code(q), B_, h_q,
                                                    C.c_void_p(pc.pool.data_ptr()),
                                                    pc.pool.numel() // (layouts.h_kv * layouts.tile_bytes),
                                                    C.c_void_p(pc.table.data_ptr()), pc.max_pages,
                                                    C.c_void_p(seq_lens.data_ptr()), max_seq_len, scale,
                                                    C.c_void_p(out.data_ptr()), C.c_void_p(workspace.data_ptr()),
                                                    workspace.numel(), _stream_ptr(stream)),
           "decode_attention_paged_heads")


def decode_attention_multi_heads(layouts: LayoutSet, q, cache, seq_lens, capacity: int, max_seq_len: int, out,
                                 workspace, softmax_scale: float | None = None, stream=None):
    """decode_attention_multi over a layout set's cache: q [B, n_q, h_q, 128] CUDA (the last
    n_q of each row's cached tokens), out [B, n_q, h_q, 128] fp32."""
    B_, n_q, h_q, d = q.shape
    assert d == HEAD_DIM and q.is_contiguous() and out.is_contiguous()
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_attention_multi_heads(layouts.handle, C.c_void_p(q.data_ptr()), dtype_code(q), B_, n_q,
                                                    h_q, C.c_void_p(cache.data_ptr()),
                                                    C.c_void_p(seq_lens.data_ptr()), capacity, max_seq_len, scale,
                                                    C.c_void_p(out.data_ptr()), C.c_void_p(workspace.data_ptr()),
                                                    workspace.numel(), _stream_ptr(stream)),
           "decode_attention_multi_heads")


def decode_step_multi_heads(layouts: LayoutSet, k_new, v_new, q, cache, seq_lens, capacity: int, max_seq_len: int,
                            out, workspace, softmax_scale: float | None = None, stream=None):
    """decode_step_multi over a layout set's cache: append k_new, v_new [B, n_new, h_kv, 128]
    at seq_lens[b] and attend q [B, n_new, h_q, 128] (the new tokens' queries, causal among
    them); out [B, n_new, h_q, 128] fp32."""
    B_, n_new, h_kv, d = k_new.shape
    assert d == HEAD_DIM and h_kv == layouts.h_kv and k_new.is_contiguous() and v_new.is_contiguous()
    assert q.shape[:2] == (B_, n_new) and q.is_contiguous() and out.is_contiguous()
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_step_multi_heads(layouts.handle, C.c_void_p(k_new.data_ptr()),
                                               C.c_void_p(v_new.data_ptr()), dtype_code(k_new), n_new,
                                               C.c_void_p(q.data_ptr()), dtype_code(q), B_, q.shape[2],
                                               C.c_void_p(cache.data_ptr()), C.c_void_p(seq_lens.data_ptr()),
                                               capacity, max_seq_len, scale, C.c_void_p(out.data_ptr()),
                                               C.c_void_p(workspace.data_ptr()), workspace.numel(),
                                               _stream_ptr(stream)),
           "decode_step_multi_heads")


def decode_step_paged_heads(layouts: LayoutSet, k_new, v_new, q, pc, seq_lens, max_seq_len: int, out, workspace,
                            softmax_scale: float | None = None, stream=None):
    """decode_step_heads over a paged cache pc (a PagedCache over a pool of the set's pages)."""
    B_, n_new, h_kv, d = k_new.shape
    assert d == HEAD_DIM and h_kv == layouts.h_kv and k_new.is_contiguous() and v_new.is_contiguous()
    assert q.is_contiguous() and out.is_contiguous()
    scale = 1.0 / HEAD_DIM ** 0.5 if softmax_scale is None else float(softmax_scale)
    _check(load().bgtq_decode_step_paged_heads(layouts.handle, C.c_void_p(k_new.data_ptr()),
                                               C.c_void_p(v_new.data_ptr()), dtype_code(k_new), n_new,
                                               C.c_void_p(q.data_ptr()), dtype_code(q), B_, q.shape[1],
                                               C.c_void_p(pc.pool.data_ptr()),
                                               pc.pool.numel() // (layouts.h_kv * layouts.tile_bytes),
                                               C.c_void_p(pc.table.data_ptr()), pc.max_pages,
                                               C.c_void_p(seq_lens.data_ptr()), max_seq_len, scale,
                                               C.c_void_p(out.data_ptr()), C.c_void_p(workspace.data_ptr()),
                                               workspace.numel(), _stream_ptr(stream)),
           "decode_step_paged_heads")
