"""Thin ctypes binding of libpkv (``include/pkv.h``): the same function names,
argument marshalling only.  Every step of the decode step runs in the CUDA
kernels of ``libpkv.so``; this module never computes any of it.

The library is loaded at import.  If it has not been built the import fails
with an ImportError (build it with ``python -m paged_kv_flight_b200.build``);
there is no fallback path.

Tensors may be passed as torch tensors or as raw integer device pointers.
A tensor must be a contiguous CUDA tensor of the element type the call reads
it as: bf16 activations and weights, bf16 or uint8 / float8_e4m3fn pools,
float32 scales, int32 block tables, lengths and offsets.  Anything else
raises before the library is called; raw pointers pass through unchecked.  ``stream`` may be a
``torch.cuda.Stream``, a raw ``cudaStream_t`` integer, or None for torch's
current stream.  Each call returns its ``pkv_status``; with ``check=True``
(the default) a non-OK status raises :class:`PkvError` instead.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

# PKV_LIBRARY may point at another build of the same library (e.g. a tuning
# variant); by default the in-tree build is loaded.
_LIB_PATH = os.environ.get("PKV_LIBRARY") or os.path.join(os.path.dirname(os.path.abspath(__file__)),
                                                           "libpkv.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libpkv.so is not built ({_LIB_PATH}); run `python -m paged_kv_flight_b200.build`")
lib = C.CDLL(_LIB_PATH)

PKV_OK = 0
PKV_ERR_INVALID_ARG = 1
PKV_ERR_UNSUPPORTED = 2
PKV_ERR_CUDA = 3
PKV_ERR_OOM = 4
PKV_ERR_DEVICE_BOUNDS = 5
PKV_ERR_DEVICE_TIMEOUT = 6

PKV_KV_BF16 = 0
PKV_KV_FP8_E4M3 = 1

# names of every symbol include/pkv.h declares
EXPORTS = ("pkv_create", "pkv_rope_append", "pkv_decode_attn", "pkv_destroy", "pkv_status_str",
           "pkv_check_device_error", "pkv_set_workers", "pkv_workspace_bytes", "pkv_decode_attn_noalloc",
           "pkv_set_tail_chunks", "pkv_set_prefill_rows", "pkv_rope_append_tokens", "pkv_decode_attn_tokens",
           "pkv_pages_create", "pkv_pages_destroy", "pkv_pages_admit", "pkv_pages_reserve", "pkv_pages_advance",
           "pkv_pages_release", "pkv_pages_block_table", "pkv_pages_seq_lens", "pkv_pages_active",
           "pkv_pages_refcount", "pkv_pages_free_count", "pkv_pages_take_changes", "pkv_qkv_rope_append",
           "pkv_qkv_pack_weight", "pkv_set_qkv_split", "pkv_qkv_launch_shape",
           "pkv_table_sync", "pkv_rope_append_varlen", "pkv_decode_attn_varlen", "pkv_decode_step")


class pkv_config(C.Structure):
    _fields_ = [("num_q_heads", C.c_int), ("num_kv_heads", C.c_int), ("head_dim", C.c_int),
                ("page_size", C.c_int), ("kv_dtype", C.c_int), ("rope_base", C.c_double),
                ("max_batch", C.c_int), ("max_blocks_per_seq", C.c_int), ("num_pages", C.c_int)]


_V = C.c_void_p
lib.pkv_create.argtypes = [C.POINTER(pkv_config), C.POINTER(_V)]
lib.pkv_create.restype = C.c_int
lib.pkv_rope_append.argtypes = [_V, _V, _V, _V, _V, _V, _V, _V, _V, C.c_int, _V, C.c_int, _V]
lib.pkv_rope_append.restype = C.c_int
lib.pkv_decode_attn.argtypes = [_V, _V, _V, _V, _V, _V, _V, C.c_int, _V, C.c_int, _V, _V]
lib.pkv_decode_attn.restype = C.c_int
lib.pkv_destroy.argtypes = [_V]
lib.pkv_destroy.restype = C.c_int
lib.pkv_status_str.argtypes = [C.c_int]
lib.pkv_status_str.restype = C.c_char_p
lib.pkv_check_device_error.argtypes = [_V, _V, C.POINTER(C.c_int)]
lib.pkv_check_device_error.restype = C.c_int
lib.pkv_set_workers.argtypes = [_V, C.c_int]
lib.pkv_set_workers.restype = C.c_int
lib.pkv_rope_append_tokens.argtypes = [_V, _V, _V, _V, _V, _V, _V, _V, _V, C.c_int, _V, C.c_int, C.c_int, _V]
lib.pkv_rope_append_tokens.restype = C.c_int
lib.pkv_decode_attn_tokens.argtypes = [_V, _V, _V, _V, _V, _V, _V, C.c_int, _V, C.c_int, C.c_int, _V, _V]
lib.pkv_decode_attn_tokens.restype = C.c_int
lib.pkv_pages_create.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, C.POINTER(_V)]
lib.pkv_pages_create.restype = C.c_int
lib.pkv_pages_destroy.argtypes = [_V]
lib.pkv_pages_destroy.restype = C.c_int
lib.pkv_pages_admit.argtypes = [_V, C.c_int, C.c_int, C.c_int, C.c_int]
lib.pkv_pages_admit.restype = C.c_int
for _f in (lib.pkv_pages_reserve, lib.pkv_pages_advance, lib.pkv_pages_release):
    _f.argtypes = [_V, C.c_int]
    _f.restype = C.c_int
for _f in (lib.pkv_pages_block_table, lib.pkv_pages_seq_lens, lib.pkv_pages_active, lib.pkv_pages_refcount):
    _f.argtypes = [_V]
    _f.restype = C.POINTER(C.c_int32)
lib.pkv_pages_free_count.argtypes = [_V]
lib.pkv_pages_free_count.restype = C.c_int
lib.pkv_pages_take_changes.argtypes = [_V, _V, C.c_int]
lib.pkv_pages_take_changes.restype = C.c_int
lib.pkv_qkv_rope_append.argtypes = [_V, _V, _V, C.c_int, C.c_int, _V, _V, _V, _V, _V, _V, C.c_int, _V, C.c_int,
                                    _V]
lib.pkv_qkv_rope_append.restype = C.c_int
lib.pkv_qkv_pack_weight.argtypes = [_V, _V, C.c_int, _V, _V]
lib.pkv_qkv_pack_weight.restype = C.c_int
lib.pkv_set_qkv_split.argtypes = [_V, C.c_int]
lib.pkv_set_qkv_split.restype = C.c_int
lib.pkv_qkv_launch_shape.argtypes = [_V, C.c_int, C.c_int, _V]
lib.pkv_qkv_launch_shape.restype = C.c_int
lib.pkv_table_sync.argtypes = [_V, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, _V, _V, _V, _V]
lib.pkv_table_sync.restype = C.c_int
lib.pkv_rope_append_varlen.argtypes = [_V, _V, _V, _V, _V, _V, _V, _V, _V, C.c_int, _V, _V, C.c_int, C.c_int, _V]
lib.pkv_rope_append_varlen.restype = C.c_int
lib.pkv_decode_attn_varlen.argtypes = [_V, _V, _V, _V, _V, _V, _V, C.c_int, _V, _V, C.c_int, C.c_int, _V, _V]
lib.pkv_decode_attn_varlen.restype = C.c_int
lib.pkv_set_tail_chunks.argtypes = [_V, C.c_int]
lib.pkv_set_tail_chunks.restype = C.c_int
lib.pkv_set_prefill_rows.argtypes = [_V, C.c_int]
lib.pkv_set_prefill_rows.restype = C.c_int
lib.pkv_workspace_bytes.argtypes = [_V]
lib.pkv_workspace_bytes.restype = C.c_size_t
lib.pkv_decode_attn_noalloc.argtypes = [C.POINTER(pkv_config), _V, _V, _V, _V, _V, _V, C.c_int, _V, C.c_int,
                                        _V, _V]
lib.pkv_decode_attn_noalloc.restype = C.c_int
lib.pkv_decode_step.argtypes = [_V, _V, _V, _V, _V, _V, _V, _V, _V, C.c_int, _V, C.c_int, C.c_int, _V, _V]
lib.pkv_decode_step.restype = C.c_int


class PkvError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {pkv_status_str(status)} (status {status})")
        self.status = status


def pkv_status_str(status: int) -> str:
    return lib.pkv_status_str(int(status)).decode()


# element types the library reads each kind of device argument as
_ACT = (torch.bfloat16,)                                      # q, k_new, v_new, out, x, weights
_POOL = (torch.bfloat16, torch.uint8, torch.float8_e4m3fn)    # KV pools: bf16, or E4M3 codes
_F32 = (torch.float32,)                                       # E4M3 scales
_I32 = (torch.int32,)                                         # block tables, lengths, offsets


def _ptr(x, kinds=None, name="argument"):
    """Device pointer of a device-memory argument: None; a raw integer device
    pointer (passed through unchecked); or a contiguous CUDA tensor whose
    dtype is one of `kinds`.  A host tensor or another element type would
    make the kernels read or write memory the caller did not mean, so it
    raises here, before the library is called."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, torch.Tensor):
        if not x.is_cuda:
            raise ValueError(f"{name}: libpkv takes device tensors, got one on {x.device}")
        if kinds is not None and x.dtype not in kinds:
            raise TypeError(f"{name}: expected {' or '.join(str(k) for k in kinds)}, got {x.dtype}")
        if not x.is_contiguous():
            raise ValueError(f"{name}: libpkv takes contiguous tensors")
        return x.data_ptr()
    raise TypeError(f"{name}: expected a tensor or a device pointer, got {type(x)}")


def _kv(k_pool, v_pool, k_scale, v_scale):
    """The pools and their scales, in the order every call takes them."""
    return (_ptr(k_pool, _POOL, "k_pool"), _ptr(v_pool, _POOL, "v_pool"),
            _ptr(k_scale, _F32, "k_scale"), _ptr(v_scale, _F32, "v_scale"))


def _hptr(x, name="argument"):
    """Host pointer of an int32 host buffer: a contiguous CPU tensor or a raw
    integer host pointer."""
    if isinstance(x, int):
        return x
    if isinstance(x, torch.Tensor):
        if x.is_cuda or x.dtype != torch.int32 or not x.is_contiguous():
            raise ValueError(f"{name}: expected a contiguous int32 host tensor")
        return x.data_ptr()
    raise TypeError(f"{name}: expected a tensor or a host pointer, got {type(x)}")


# The current CUDA stream of the current device as a raw cudaStream_t: the
# query PyTorch's own generated code uses (no Stream object is built, which
# is most of the host cost of torch.cuda.current_stream()), else the public
# API.
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)
_cur_device = getattr(torch._C, "_cuda_getDevice", None)


def _stream(s):
    if s is None:
        if _raw_stream is not None and _cur_device is not None:
            return _raw_stream(_cur_device())
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, torch.cuda.Stream):
        return s.cuda_stream
    return int(s)


def _done(status: int, where: str, check: bool) -> int:
    if check and status != PKV_OK:
        raise PkvError(status, where)
    return status


def make_config(num_q_heads, num_kv_heads, head_dim, page_size, kv_dtype, rope_base, max_batch,
                max_blocks_per_seq, num_pages) -> pkv_config:
    kv = kv_dtype if isinstance(kv_dtype, int) else (PKV_KV_FP8_E4M3 if kv_dtype in ("fp8", "e4m3") else PKV_KV_BF16)
    return pkv_config(num_q_heads, num_kv_heads, head_dim, page_size, kv, float(rope_base), max_batch,
                      max_blocks_per_seq, num_pages)


def pkv_create(cfg: pkv_config, check: bool = True):
    """Returns the context handle (an int), or (status, None) with check=False."""
    h = _V()
    st = lib.pkv_create(C.byref(cfg), C.byref(h))
    if not check:
        return st, (h.value if st == PKV_OK else None)
    _done(st, "pkv_create", True)
    return h.value


def pkv_rope_append(ctx, q, k_new, v_new, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens,
                    batch: int | None = None, bt_stride: int | None = None, stream=None,
                    check: bool = True) -> int:
    if batch is None:
        batch = int(seq_lens.shape[0])
    if bt_stride is None:
        bt_stride = int(block_tables.shape[1])
    st = lib.pkv_rope_append(ctx, _ptr(q, _ACT, "q"), _ptr(k_new, _ACT, "k_new"), _ptr(v_new, _ACT, "v_new"),
                             *_kv(k_pool, v_pool, k_scale, v_scale),
                             _ptr(block_tables, _I32, "block_tables"), int(bt_stride),
                             _ptr(seq_lens, _I32, "seq_lens"), int(batch), _stream(stream))
    return _done(st, "pkv_rope_append", check)


def pkv_decode_attn(ctx, q, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens, out,
                    batch: int | None = None, bt_stride: int | None = None, stream=None,
                    check: bool = True) -> int:
    if batch is None:
        batch = int(seq_lens.shape[0])
    if bt_stride is None:
        bt_stride = int(block_tables.shape[1])
    st = lib.pkv_decode_attn(ctx, _ptr(q, _ACT, "q"), *_kv(k_pool, v_pool, k_scale, v_scale),
                             _ptr(block_tables, _I32, "block_tables"), int(bt_stride),
                             _ptr(seq_lens, _I32, "seq_lens"), int(batch), _ptr(out, _ACT, "out"),
                             _stream(stream))
    return _done(st, "pkv_decode_attn", check)


def pkv_destroy(ctx, check: bool = True) -> int:
    return _done(lib.pkv_destroy(ctx), "pkv_destroy", check)


def pkv_check_device_error(ctx, stream=None):
    """(status, raw error bits); synchronises the stream."""
    bits = C.c_int(0)
    st = lib.pkv_check_device_error(ctx, _stream(stream), C.byref(bits))
    return st, bits.value


def pkv_set_workers(ctx, workers: int, check: bool = True) -> int:
    return _done(lib.pkv_set_workers(ctx, int(workers)), "pkv_set_workers", check)


def pkv_set_tail_chunks(ctx, max_chunks: int, check: bool = True) -> int:
    return _done(lib.pkv_set_tail_chunks(ctx, int(max_chunks)), "pkv_set_tail_chunks", check)


def pkv_set_prefill_rows(ctx, rows: int, check: bool = True) -> int:
    return _done(lib.pkv_set_prefill_rows(ctx, int(rows)), "pkv_set_prefill_rows", check)


def pkv_workspace_bytes(ctx) -> int:
    return int(lib.pkv_workspace_bytes(ctx))


def pkv_decode_attn_noalloc(cfg: pkv_config, q, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens, out,
                            batch: int | None = None, bt_stride: int | None = None, stream=None,
                            check: bool = True) -> int:
    """pkv_decode_attn without a context, for callers that may not allocate
    device memory: its scratch is a fixed 16 MiB array inside the library,
    shared by every call (calls that overlap on the GPU race)."""
    if batch is None:
        batch = int(seq_lens.shape[0])
    if bt_stride is None:
        bt_stride = int(block_tables.shape[1])
    st = lib.pkv_decode_attn_noalloc(C.byref(cfg), _ptr(q, _ACT, "q"), *_kv(k_pool, v_pool, k_scale, v_scale),
                                     _ptr(block_tables, _I32, "block_tables"), int(bt_stride),
                                     _ptr(seq_lens, _I32, "seq_lens"), int(batch), _ptr(out, _ACT, "out"),
                                     _stream(stream))
    return _done(st, "pkv_decode_attn_noalloc", check)


def pkv_rope_append_tokens(ctx, q, k_new, v_new, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens,
                           batch: int | None = None, q_len: int | None = None, bt_stride: int | None = None,
                           stream=None, check: bool = True) -> int:
    """q [batch, q_len, Hq, d], k_new / v_new [batch, q_len, Hkv, d]."""
    if batch is None:
        batch = int(seq_lens.shape[0])
    if q_len is None:
        q_len = int(q.shape[1])
    if bt_stride is None:
        bt_stride = int(block_tables.shape[1])
    st = lib.pkv_rope_append_tokens(ctx, _ptr(q, _ACT, "q"), _ptr(k_new, _ACT, "k_new"), _ptr(v_new, _ACT, "v_new"),
                                    *_kv(k_pool, v_pool, k_scale, v_scale),
                                    _ptr(block_tables, _I32, "block_tables"), int(bt_stride),
                                    _ptr(seq_lens, _I32, "seq_lens"), int(batch), int(q_len), _stream(stream))
    return _done(st, "pkv_rope_append_tokens", check)


def pkv_decode_attn_tokens(ctx, q, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens, out,
                           batch: int | None = None, q_len: int | None = None, bt_stride: int | None = None,
                           stream=None, check: bool = True) -> int:
    """q and out [batch, q_len, Hq, d]."""
    if batch is None:
        batch = int(seq_lens.shape[0])
    if q_len is None:
        q_len = int(q.shape[1])
    if bt_stride is None:
        bt_stride = int(block_tables.shape[1])
    st = lib.pkv_decode_attn_tokens(ctx, _ptr(q, _ACT, "q"), *_kv(k_pool, v_pool, k_scale, v_scale),
                                    _ptr(block_tables, _I32, "block_tables"), int(bt_stride),
                                    _ptr(seq_lens, _I32, "seq_lens"), int(batch), int(q_len),
                                    _ptr(out, _ACT, "out"), _stream(stream))
    return _done(st, "pkv_decode_attn_tokens", check)


def pkv_decode_step(ctx, q, k_new, v_new, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens, out,
                    batch: int | None = None, q_len: int = 1, bt_stride: int | None = None, stream=None,
                    check: bool = True) -> int:
    """The whole step in one call: pkv_rope_append(_tokens) then
    pkv_decode_attn(_tokens), the attention overlapping the RoPE kernel's end.
    q / out [batch, (q_len,) Hq, d], k_new / v_new [batch, (q_len,) Hkv, d]."""
    if batch is None:
        batch = int(seq_lens.shape[0])
    if bt_stride is None:
        bt_stride = int(block_tables.shape[1])
    st = lib.pkv_decode_step(ctx, _ptr(q, _ACT, "q"), _ptr(k_new, _ACT, "k_new"), _ptr(v_new, _ACT, "v_new"),
                             *_kv(k_pool, v_pool, k_scale, v_scale),
                             _ptr(block_tables, _I32, "block_tables"), int(bt_stride),
                             _ptr(seq_lens, _I32, "seq_lens"), int(batch), int(q_len), _ptr(out, _ACT, "out"),
                             _stream(stream))
    return _done(st, "pkv_decode_step", check)


class Pages:
    """The host page allocator (include/pkv_pages.h): marshalling only.  The
    views (block_table, seq_lens, active, refcount) are numpy arrays over the
    library's own memory, valid while the object lives."""

    def __init__(self, num_pages: int, page_size: int, max_batch: int, max_blocks_per_seq: int):
        h = _V()
        _done(lib.pkv_pages_create(num_pages, page_size, max_batch, max_blocks_per_seq, C.byref(h)),
              "pkv_pages_create", True)
        self.h = h.value
        self.num_pages, self.P, self.max_batch, self.max_blocks = num_pages, page_size, max_batch, max_blocks_per_seq
        import numpy as np
        self.block_table = np.ctypeslib.as_array(lib.pkv_pages_block_table(self.h),
                                                 shape=(max_batch, max_blocks_per_seq))
        self.seq_lens = np.ctypeslib.as_array(lib.pkv_pages_seq_lens(self.h), shape=(max_batch,))
        self.active = np.ctypeslib.as_array(lib.pkv_pages_active(self.h), shape=(max_batch,))
        self.refcount = np.ctypeslib.as_array(lib.pkv_pages_refcount(self.h), shape=(num_pages,))

    def admit(self, slot: int, length: int, share_slot: int = -1, share_tokens: int = 0, check: bool = True) -> int:
        return _done(lib.pkv_pages_admit(self.h, slot, length, share_slot, share_tokens), "pkv_pages_admit", check)

    def reserve(self, q_len: int = 1, check: bool = True) -> int:
        return _done(lib.pkv_pages_reserve(self.h, q_len), "pkv_pages_reserve", check)

    def advance(self, q_len: int = 1, check: bool = True) -> int:
        return _done(lib.pkv_pages_advance(self.h, q_len), "pkv_pages_advance", check)

    def release(self, slot: int, check: bool = True) -> int:
        return _done(lib.pkv_pages_release(self.h, slot), "pkv_pages_release", check)

    @property
    def free_count(self) -> int:
        return lib.pkv_pages_free_count(self.h)

    def take_changes(self, out) -> int:
        """Block-table writes since the last call into `out` (int32, at least
        3 * max entries, a numpy array or a host pointer): their count, or -1
        when a full copy of the table is due."""
        import numpy as np
        if isinstance(out, np.ndarray):
            return lib.pkv_pages_take_changes(self.h, out.ctypes.data, out.size // 3)
        return lib.pkv_pages_take_changes(self.h, _hptr(out, "out"), int(out.numel()) // 3)

    def close(self):
        if self.h:
            lib.pkv_pages_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


PKV_W_ROWS, PKV_W_TILED = 0, 1


def pkv_set_qkv_split(ctx, split: int, check: bool = True) -> int:
    """CTAs (a cluster) per head over the hidden dimension: 1 .. 4, 0 = automatic."""
    return _done(lib.pkv_set_qkv_split(ctx, int(split)), "pkv_set_qkv_split", check)


def pkv_rope_append_varlen(ctx, q, k_new, v_new, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens,
                           cu_q, batch: int | None = None, bt_stride: int | None = None, stream=None,
                           check: bool = True) -> int:
    """q [n_tokens, Hq, d] (rotated in place), k_new / v_new [n_tokens, Hkv, d];
    cu_q [batch + 1] int32: request b's new tokens are rows cu_q[b] .. cu_q[b+1]-1."""
    if batch is None:
        batch = int(seq_lens.shape[0])
    if bt_stride is None:
        bt_stride = int(block_tables.shape[1])
    st = lib.pkv_rope_append_varlen(ctx, _ptr(q, _ACT, "q"), _ptr(k_new, _ACT, "k_new"), _ptr(v_new, _ACT, "v_new"),
                                    *_kv(k_pool, v_pool, k_scale, v_scale),
                                    _ptr(block_tables, _I32, "block_tables"), int(bt_stride),
                                    _ptr(seq_lens, _I32, "seq_lens"), _ptr(cu_q, _I32, "cu_q"), int(batch),
                                    int(q.shape[0]), _stream(stream))
    return _done(st, "pkv_rope_append_varlen", check)


def pkv_decode_attn_varlen(ctx, q, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens, cu_q, out,
                           batch: int | None = None, bt_stride: int | None = None, stream=None,
                           check: bool = True) -> int:
    """q / out [n_tokens, Hq, d]; token i of request b attends its cache up to
    position L_b + i - cu_q[b] (E4M3 pools take their scales, else None)."""
    if batch is None:
        batch = int(seq_lens.shape[0])
    if bt_stride is None:
        bt_stride = int(block_tables.shape[1])
    st = lib.pkv_decode_attn_varlen(ctx, _ptr(q, _ACT, "q"), *_kv(k_pool, v_pool, k_scale, v_scale),
                                    _ptr(block_tables, _I32, "block_tables"), int(bt_stride),
                                    _ptr(seq_lens, _I32, "seq_lens"), _ptr(cu_q, _I32, "cu_q"), int(batch),
                                    int(q.shape[0]), _ptr(out, _ACT, "out"),
                                    _stream(stream))
    return _done(st, "pkv_decode_attn_varlen", check)


def pkv_table_sync(upload, n_changes: int, batch: int, table, bt_out, lens_out, page_size: int, stream=None,
                   check: bool = True) -> int:
    """upload: device int32 [3 n_changes + 2 batch] (changes, slots, lengths);
    table [max_batch, max_blocks] updated in place; bt_out [>= batch,
    max_blocks] and lens_out [>= batch] receive the batch's rows and lengths."""
    st = lib.pkv_table_sync(_ptr(upload, _I32, "upload"), int(n_changes), int(batch), int(table.shape[0]),
                            int(table.shape[1]), int(page_size), _ptr(table, _I32, "table"),
                            _ptr(bt_out, _I32, "bt_out"), _ptr(lens_out, _I32, "lens_out"), _stream(stream))
    return _done(st, "pkv_table_sync", check)


def pkv_qkv_launch_shape(ctx, batch: int, hidden: int) -> dict:
    """The projection's launch shape: split (CTAs per cluster), ring stages,
    shared memory bytes per CTA, clusters the GPU holds at once."""
    out = (C.c_int * 4)()
    _done(lib.pkv_qkv_launch_shape(ctx, int(batch), int(hidden), out), "pkv_qkv_launch_shape", True)
    return {"split": out[0], "stages": out[1], "smem_bytes": out[2], "max_clusters": out[3]}


def pkv_qkv_pack_weight(ctx, w_qkv, w_tiled, stream=None, check: bool = True) -> int:
    """w_qkv [(Hq + 2 Hkv) d, hidden] -> w_tiled (same size) in the tiled layout."""
    st = lib.pkv_qkv_pack_weight(ctx, _ptr(w_qkv, _ACT, "w_qkv"), int(w_qkv.shape[-1]),
                                 _ptr(w_tiled, _ACT, "w_tiled"), _stream(stream))
    return _done(st, "pkv_qkv_pack_weight", check)


def pkv_qkv_rope_append(ctx, x, w_qkv, q_out, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens,
                        batch: int | None = None, bt_stride: int | None = None, stream=None,
                        check: bool = True, w_layout: int = PKV_W_ROWS) -> int:
    """x [batch, hidden], w_qkv [(Hq + 2 Hkv) d, hidden] (PKV_W_ROWS) or as
    pkv_qkv_pack_weight wrote it (PKV_W_TILED), q_out [batch, Hq, d]."""
    if batch is None:
        batch = int(seq_lens.shape[0])
    if bt_stride is None:
        bt_stride = int(block_tables.shape[1])
    hidden = int(x.shape[-1])
    st = lib.pkv_qkv_rope_append(ctx, _ptr(x, _ACT, "x"), _ptr(w_qkv, _ACT, "w_qkv"), hidden, int(w_layout),
                                 _ptr(q_out, _ACT, "q_out"), *_kv(k_pool, v_pool, k_scale, v_scale),
                                 _ptr(block_tables, _I32, "block_tables"), int(bt_stride),
                                 _ptr(seq_lens, _I32, "seq_lens"), int(batch), _stream(stream))
    return _done(st, "pkv_qkv_rope_append", check)
