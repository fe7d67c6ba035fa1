"""Python binding of libkvq (include/kvq.h): argument marshalling only.

PyTorch provides device memory and the current CUDA stream; every step of
the computation runs in the library's CUDA kernels.  If the library cannot
be loaded this module raises -- there is no CPU or PyTorch fallback.

Typical use, with the names of the operations on the KIVI page ("LLM系列：
KVCache量化1 KIVI ...", section 1)::

    cache = prefill_quantize(X_K, X_V, G=32, R=128, bits=2, q_heads=32)
    append(cache, t_K, t_V)
    t_O = decode_attention(cache, t_Q)
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

_lock = threading.Lock()
_lib = None

(KVQ_OK, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED, KVQ_ERR_CAPACITY, KVQ_ERR_STATE, KVQ_ERR_CUDA,
 KVQ_ERR_DEVICE_CHECK) = range(7)
KVQ_FP16, KVQ_BF16 = 0, 1
# decode kernels (kvq_set_decode_kernel)
KVQ_DECODE_AUTO, KVQ_DECODE_CUDA_CORES, KVQ_DECODE_INT8_MMA, KVQ_DECODE_BF16_MMA = range(4)

EXPORTED = ("kvq_get_sizes", "kvq_create", "kvq_destroy", "kvq_reset", "kvq_prefill_quantize",
            "kvq_append", "kvq_decode_attention", "kvq_cache_state", "kvq_set_split_limit",
            "kvq_decode_splits", "kvq_kernel_launches", "kvq_decode_attention_noalloc",
            "kvq_last_error", "kvq_layout_version", "kvq_check_device", "kvq_append_decode_attention",
            "kvq_decode_attention_partial", "kvq_merge_partials", "kvq_paged_get_sizes",
            "kvq_paged_create", "kvq_paged_destroy", "kvq_paged_prefill", "kvq_paged_append",
            "kvq_paged_decode_attention", "kvq_paged_release", "kvq_paged_seq_len",
            "kvq_paged_decode_splits", "kvq_paged_check_device", "kvq_logquant_get_sizes",
            "kvq_logquant_create", "kvq_logquant_retained", "kvq_set_key_outliers", "kvq_plan_decode",
            "kvq_binary_arch", "kvq_set_decode_kernel")


class KVQError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"kvq status {status}: {message}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("q_heads", ctypes.c_int32),
                ("kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("group_k", ctypes.c_int32), ("group_v", ctypes.c_int32),
                ("residual", ctypes.c_int32), ("bits", ctypes.c_int32),
                ("symmetric", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("capacity", ctypes.c_int64)]


class Sizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("k_codes", "k_scales", "k_zeros", "v_codes", "v_scales", "v_zeros",
                 "k_residual", "v_residual", "workspace", "state")]


class Buffers(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("k_codes", "k_scales", "k_zeros", "v_codes", "v_scales", "v_zeros",
                 "k_residual", "v_residual", "state")]


class PagedConfig(ctypes.Structure):
    _fields_ = [("geom", Config), ("page_tokens", ctypes.c_int32), ("num_pages", ctypes.c_int32)]


class PagedSizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("k_codes", "k_scales", "k_zeros", "v_codes", "v_scales", "v_zeros",
                 "k_residual", "v_residual", "page_table", "workspace", "state")]


def check_build() -> bool:
    """True when KVQ_LIBRARY=check selects the bounds-check build (libkvq_check.so)."""
    return os.environ.get("KVQ_LIBRARY", "") == "check"


def library_path() -> str:
    return _build.LIB_CHECK if check_build() else _build.LIB


def load() -> ctypes.CDLL:
    """Load libkvq.so -- or, with KVQ_LIBRARY=check, its bounds-check build libkvq_check.so --
    building it in-tree first if it is missing or stale."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = _build.build(check=check_build())
        if not os.path.exists(path):
            raise ImportError(f"{os.path.basename(path)} not found at {path}")
        lib = ctypes.CDLL(path)
        P, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        lib.kvq_get_sizes.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(Sizes)]
        lib.kvq_create.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(Buffers),
                                   ctypes.POINTER(P)]
        lib.kvq_destroy.argtypes = [P]
        lib.kvq_destroy.restype = None
        lib.kvq_reset.argtypes = [P]
        lib.kvq_prefill_quantize.argtypes = [P, P, P, i64, P]
        lib.kvq_append.argtypes = [P, P, P, P]
        lib.kvq_decode_attention.argtypes = [P, P, P, P, sz, P]
        lib.kvq_append_decode_attention.argtypes = [P, P, P, P, P, P, sz, P]
        lib.kvq_append_decode_attention.restype = ctypes.c_int
        lib.kvq_decode_attention_partial.argtypes = [P, P, P, P, P, P, sz, P]
        lib.kvq_decode_attention_partial.restype = ctypes.c_int
        lib.kvq_merge_partials.argtypes = [P, P, P, i32, i64, i32, P, P]
        lib.kvq_merge_partials.restype = ctypes.c_int
        lib.kvq_decode_attention_noalloc.argtypes = [P, P, P, P]
        lib.kvq_decode_attention_noalloc.restype = ctypes.c_int
        lib.kvq_cache_state.argtypes = [P, ctypes.POINTER(i64), ctypes.POINTER(i32)]
        lib.kvq_set_split_limit.argtypes = [P, i32]
        lib.kvq_set_decode_kernel.argtypes = [P, i32]
        lib.kvq_set_decode_kernel.restype = ctypes.c_int
        lib.kvq_decode_splits.argtypes = [P]
        lib.kvq_decode_splits.restype = i32
        lib.kvq_kernel_launches.argtypes = []
        lib.kvq_kernel_launches.restype = ctypes.c_uint64
        lib.kvq_last_error.argtypes = []
        lib.kvq_last_error.restype = ctypes.c_char_p
        lib.kvq_layout_version.argtypes = []
        lib.kvq_layout_version.restype = i32
        lib.kvq_binary_arch.argtypes = []
        lib.kvq_binary_arch.restype = i32
        if check_build():
            lib.kvq_debug_set_stall.argtypes = [P, i32]
            lib.kvq_debug_set_stall.restype = ctypes.c_int
            lib.kvq_debug_gather_rows.argtypes = [P, P, i64, P, i32, P, P]
            lib.kvq_debug_gather_rows.restype = ctypes.c_int
        lib.kvq_check_device.argtypes = [P]
        lib.kvq_paged_get_sizes.argtypes = [ctypes.POINTER(PagedConfig), ctypes.POINTER(PagedSizes)]
        lib.kvq_paged_create.argtypes = [ctypes.POINTER(PagedConfig), ctypes.POINTER(Buffers), P,
                                         ctypes.POINTER(P)]
        lib.kvq_paged_destroy.argtypes = [P]
        lib.kvq_paged_destroy.restype = None
        lib.kvq_paged_prefill.argtypes = [P, i32, P, P, i64, P]
        lib.kvq_paged_append.argtypes = [P, P, P, P]
        lib.kvq_paged_decode_attention.argtypes = [P, P, P, P, sz, P]
        lib.kvq_paged_release.argtypes = [P, i32, P]
        lib.kvq_paged_seq_len.argtypes = [P, i32, ctypes.POINTER(i64)]
        lib.kvq_paged_decode_splits.argtypes = [P]
        lib.kvq_paged_decode_splits.restype = i32
        lib.kvq_paged_check_device.argtypes = [P]
        lib.kvq_logquant_get_sizes.argtypes = [ctypes.POINTER(Config), i32, ctypes.POINTER(Sizes)]
        lib.kvq_logquant_create.argtypes = [ctypes.POINTER(Config), i32, ctypes.POINTER(Buffers),
                                            ctypes.POINTER(P)]
        lib.kvq_logquant_retained.argtypes = [P, ctypes.POINTER(i64), i32, ctypes.POINTER(i32)]
        lib.kvq_set_key_outliers.argtypes = [P, i32, P, sz]
        lib.kvq_plan_decode.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(i64), i32, i32,
                                        ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(i32)]
        lib.kvq_plan_decode.restype = ctypes.c_int
        for name in ("kvq_logquant_get_sizes", "kvq_logquant_create", "kvq_logquant_retained",
                     "kvq_set_key_outliers"):
            getattr(lib, name).restype = ctypes.c_int
        for name in ("kvq_paged_get_sizes", "kvq_paged_create", "kvq_paged_prefill", "kvq_paged_append",
                     "kvq_paged_decode_attention", "kvq_paged_release", "kvq_paged_seq_len",
                     "kvq_paged_check_device"):
            getattr(lib, name).restype = ctypes.c_int
        for name in ("kvq_get_sizes", "kvq_create", "kvq_reset", "kvq_prefill_quantize",
                     "kvq_append", "kvq_decode_attention", "kvq_cache_state", "kvq_set_split_limit",
                     "kvq_check_device"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
        return lib


def _check(status: int):
    if status != KVQ_OK:
        msg = load().kvq_last_error().decode(errors="replace")
        raise KVQError(status, msg)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float16:
        return KVQ_FP16
    if dt == torch.bfloat16:
        return KVQ_BF16
    raise TypeError(f"element type must be float16 or bfloat16, got {dt}")


def make_config(batch, q_heads, kv_heads, head_dim, group_k, group_v, residual, bits,
                symmetric, dtype, capacity) -> Config:
    return Config(batch, q_heads, kv_heads, head_dim, group_k, group_v, residual, bits,
                  int(bool(symmetric)), dtype if isinstance(dtype, int) else _dtype_code(dtype),
                  capacity)


def get_sizes(cfg: Config) -> Sizes:
    s = Sizes()
    _check(load().kvq_get_sizes(ctypes.byref(cfg), ctypes.byref(s)))
    return s


def _stream_ptr(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


class KVQCache:
    """A quantized KV cache whose device buffers are torch tensors.

    Shapes (e = fp16 or bf16): prompt X_K, X_V [B, Hkv, T, d]; new token
    t_K, t_V [B, Hkv, d]; query t_Q [B, Hq, d]; output t_O float32 [B, Hq, d].
    Inputs on the host are copied to the device first (plumbing only).
    """

    def __init__(self, batch, q_heads, kv_heads, head_dim, group_k, group_v, residual, bits,
                 symmetric=False, dtype=torch.bfloat16, capacity=None, device=None, window=None,
                 key_outliers=0):
        """window: LogQuant retention with window W instead of KIVI's residual (`residual` is
        then ignored: the full-precision store holds up to 3W tokens).  key_outliers: keep that
        many largest-magnitude entries of each token's key as sparse full-precision outliers
        (dense-and-sparse keys; 1 or 2)."""
        if capacity is None:
            raise ValueError("capacity (quantized tokens per sequence) is required")
        self.window = window
        if window:
            residual = 3 * window
        capacity = -(-capacity // residual) * residual
        dev = torch.device(device if device is not None else "cuda")
        if dev.type != "cuda":
            raise ValueError("the cache lives on a CUDA device")
        self.device = dev if dev.index is not None else torch.device("cuda", torch.cuda.current_device())
        self.dtype = dtype
        self.cfg = make_config(batch, q_heads, kv_heads, head_dim, group_k, group_v, residual,
                               bits, symmetric, dtype, capacity)
        if window:
            self.sizes = Sizes()
            _check(load().kvq_logquant_get_sizes(ctypes.byref(self.cfg), window, ctypes.byref(self.sizes)))
        else:
            self.sizes = get_sizes(self.cfg)
        BH = batch * kv_heads
        dev = self.device
        words = capacity * head_dim * bits // 32
        self.k_codes = torch.empty((BH, words), dtype=torch.int32, device=dev)
        self.v_codes = torch.empty((BH, words), dtype=torch.int32, device=dev)
        self.k_scales = torch.empty((BH, capacity // group_k, head_dim), dtype=torch.float32, device=dev)
        self.v_scales = torch.empty((BH, capacity, head_dim // group_v), dtype=torch.float32, device=dev)
        if symmetric:
            self.k_zeros = self.v_zeros = None
        else:
            self.k_zeros = torch.empty((BH, capacity // group_k, head_dim), dtype=torch.int16, device=dev)
            self.v_zeros = torch.empty((BH, capacity, head_dim // group_v), dtype=torch.int16, device=dev)
        self.k_residual = torch.zeros((BH, residual, head_dim), dtype=dtype, device=dev)
        self.v_residual = torch.zeros((BH, residual, head_dim), dtype=dtype, device=dev)
        self.workspace = torch.empty(self.sizes.workspace // 4, dtype=torch.float32, device=dev)
        self.state_buf = torch.zeros(-(-self.sizes.state // 16) * 4, dtype=torch.int32, device=dev)
        bufs = Buffers(self.k_codes.data_ptr(), self.k_scales.data_ptr(),
                       self.k_zeros.data_ptr() if self.k_zeros is not None else None,
                       self.v_codes.data_ptr(), self.v_scales.data_ptr(),
                       self.v_zeros.data_ptr() if self.v_zeros is not None else None,
                       self.k_residual.data_ptr(), self.v_residual.data_ptr(), self.state_buf.data_ptr())
        self._lib = load()
        h = ctypes.c_void_p()
        with torch.cuda.device(dev):
            if window:
                _check(self._lib.kvq_logquant_create(ctypes.byref(self.cfg), window, ctypes.byref(bufs),
                                                     ctypes.byref(h)))
            else:
                _check(self._lib.kvq_create(ctypes.byref(self.cfg), ctypes.byref(bufs), ctypes.byref(h)))
        self._h = h
        self.key_outliers = key_outliers
        self.k_outliers = None
        if key_outliers:
            self.k_outliers = torch.empty((BH, capacity, key_outliers), dtype=torch.int32, device=dev)
            _check(self._lib.kvq_set_key_outliers(h, key_outliers, self.k_outliers.data_ptr(),
                                                  self.k_outliers.numel() * 4))

    # ------------------------------------------------------------------
    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._lib.kvq_destroy(h)
            self._h = None

    def _dev(self, t: torch.Tensor) -> torch.Tensor:
        if t.dtype != self.dtype:
            raise TypeError(f"expected {self.dtype}, got {t.dtype}")
        if t.device != self.device:
            t = t.to(self.device, non_blocking=True)
        return t.contiguous()

    def state(self):
        tq = ctypes.c_int64()
        r = ctypes.c_int32()
        _check(self._lib.kvq_cache_state(self._h, ctypes.byref(tq), ctypes.byref(r)))
        return int(tq.value), int(r.value)

    def retained(self) -> list[int]:
        """LogQuant cache: token positions of the full-precision store's rows (ascending)."""
        n = ctypes.c_int32()
        _check(self._lib.kvq_logquant_retained(self._h, None, 0, ctypes.byref(n)))
        arr = (ctypes.c_int64 * max(1, n.value))()
        _check(self._lib.kvq_logquant_retained(self._h, arr, n.value, ctypes.byref(n)))
        return list(arr[:n.value])

    def set_split_limit(self, max_splits: int):
        _check(self._lib.kvq_set_split_limit(self._h, max_splits))

    def set_decode_kernel(self, kernel: int):
        """KVQ_DECODE_AUTO, _CUDA_CORES, _INT8_MMA or _BF16_MMA (kvq_set_decode_kernel)."""
        _check(self._lib.kvq_set_decode_kernel(self._h, kernel))

    def splits(self) -> int:
        return int(self._lib.kvq_decode_splits(self._h))

    def reset(self):
        _check(self._lib.kvq_reset(self._h))

    def check_device(self):
        """Raise KVQError if a decode kernel of this cache gave up one of its bounded waits."""
        _check(self._lib.kvq_check_device(self._h))

    def prefill_quantize(self, X_K: torch.Tensor, X_V: torch.Tensor, stream=None):
        X_K, X_V = self._dev(X_K), self._dev(X_V)
        c = self.cfg
        if X_K.shape != X_V.shape or X_K.dim() != 4 or X_K.shape[0] != c.batch or \
                X_K.shape[1] != c.kv_heads or X_K.shape[3] != c.head_dim:
            raise ValueError(f"X_K/X_V must be [B={c.batch}, Hkv={c.kv_heads}, T, d={c.head_dim}]")
        _check(self._lib.kvq_prefill_quantize(self._h, X_K.data_ptr(), X_V.data_ptr(),
                                              X_K.shape[2], _stream_ptr(stream)))
        self._keep = (X_K, X_V)
        return self

    def append(self, t_K: torch.Tensor, t_V: torch.Tensor, stream=None):
        t_K, t_V = self._dev(t_K), self._dev(t_V)
        c = self.cfg
        want = (c.batch, c.kv_heads, c.head_dim)
        if tuple(t_K.shape) != want or tuple(t_V.shape) != want:
            raise ValueError(f"t_K/t_V must be {list(want)}")
        _check(self._lib.kvq_append(self._h, t_K.data_ptr(), t_V.data_ptr(), _stream_ptr(stream)))
        self._keep = (t_K, t_V)
        return self

    def decode_attention(self, t_Q: torch.Tensor, out: torch.Tensor | None = None, stream=None):
        t_Q = self._dev(t_Q)
        c = self.cfg
        if tuple(t_Q.shape) != (c.batch, c.q_heads, c.head_dim):
            raise ValueError(f"t_Q must be [{c.batch}, {c.q_heads}, {c.head_dim}]")
        host_out = out is not None and not out.is_cuda
        dev_out = torch.empty((c.batch, c.q_heads, c.head_dim), dtype=torch.float32,
                              device=self.device) if (out is None or host_out) else out
        _check(self._lib.kvq_decode_attention(self._h, t_Q.data_ptr(), dev_out.data_ptr(),
                                              self.workspace.data_ptr(),
                                              self.workspace.numel() * 4, _stream_ptr(stream)))
        if host_out:
            out.copy_(dev_out, non_blocking=True)
            return out
        return dev_out

    def decode_attention_partial(self, t_Q: torch.Tensor, stream=None):
        """This cache's unnormalised partial (o [B, Hq, d], m [B, Hq], l [B, Hq]; base-2
        logits) for a token-split decode; merge with merge_partials."""
        t_Q = self._dev(t_Q)
        c = self.cfg
        if tuple(t_Q.shape) != (c.batch, c.q_heads, c.head_dim):
            raise ValueError(f"t_Q must be [{c.batch}, {c.q_heads}, {c.head_dim}]")
        o = torch.empty((c.batch, c.q_heads, c.head_dim), dtype=torch.float32, device=self.device)
        m = torch.empty((c.batch, c.q_heads), dtype=torch.float32, device=self.device)
        l = torch.empty((c.batch, c.q_heads), dtype=torch.float32, device=self.device)
        _check(self._lib.kvq_decode_attention_partial(self._h, t_Q.data_ptr(), o.data_ptr(), m.data_ptr(),
                                                      l.data_ptr(), self.workspace.data_ptr(),
                                                      self.workspace.numel() * 4, _stream_ptr(stream)))
        return o, m, l

    def append_decode(self, t_K: torch.Tensor, t_V: torch.Tensor, t_Q: torch.Tensor,
                      out: torch.Tensor | None = None, stream=None):
        """append(t_K, t_V) then decode_attention(t_Q), in one call (one kernel when possible)."""
        t_K, t_V, t_Q = self._dev(t_K), self._dev(t_V), self._dev(t_Q)
        c = self.cfg
        want = (c.batch, c.kv_heads, c.head_dim)
        if tuple(t_K.shape) != want or tuple(t_V.shape) != want:
            raise ValueError(f"t_K/t_V must be {list(want)}")
        if tuple(t_Q.shape) != (c.batch, c.q_heads, c.head_dim):
            raise ValueError(f"t_Q must be [{c.batch}, {c.q_heads}, {c.head_dim}]")
        host_out = out is not None and not out.is_cuda
        dev_out = torch.empty((c.batch, c.q_heads, c.head_dim), dtype=torch.float32,
                              device=self.device) if (out is None or host_out) else out
        _check(self._lib.kvq_append_decode_attention(self._h, t_K.data_ptr(), t_V.data_ptr(),
                                                     t_Q.data_ptr(), dev_out.data_ptr(),
                                                     self.workspace.data_ptr(),
                                                     self.workspace.numel() * 4, _stream_ptr(stream)))
        self._keep = (t_K, t_V)
        if host_out:
            out.copy_(dev_out, non_blocking=True)
            return out
        return dev_out


class PagedKVQCache:
    """A paged, ragged cache: `slots` sequences of their own lengths whose quantized tokens
    live in pages of `page_tokens` tokens of one pool (torch tensors), with a page table
    per sequence.

    Pages are handed out from a host free list when a prefill or a flush needs them and
    returned by release(); the page table (int32 [slots, capacity / page_tokens], -1 where
    unassigned) is written on the stream of the call that needs it.  Shapes: prompt
    X_K, X_V [Hkv, T, d] of one sequence; new tokens t_K, t_V [slots, Hkv, d]; queries
    t_Q [slots, Hq, d]; output float32 [slots, Hq, d] (zeros for inactive slots).
    """

    def __init__(self, slots, q_heads, kv_heads, head_dim, group_k, group_v, residual, bits,
                 symmetric=False, dtype=torch.bfloat16, capacity=None, page_tokens=None,
                 num_pages=None, device=None):
        if capacity is None:
            raise ValueError("capacity (quantized tokens per sequence) is required")
        if page_tokens is None:
            page_tokens = residual * 64 // _gcd(residual, 64)
        capacity = -(-capacity // page_tokens) * page_tokens
        max_pages = capacity // page_tokens
        if num_pages is None:
            num_pages = slots * max_pages
        dev = torch.device(device if device is not None else "cuda")
        if dev.type != "cuda":
            raise ValueError("the cache lives on a CUDA device")
        self.device = dev if dev.index is not None else torch.device("cuda", torch.cuda.current_device())
        self.dtype = dtype
        self.geom = make_config(slots, q_heads, kv_heads, head_dim, group_k, group_v, residual,
                                bits, symmetric, dtype, capacity)
        self.cfg = PagedConfig(self.geom, page_tokens, num_pages)
        self.sizes = PagedSizes()
        self._lib = load()
        _check(self._lib.kvq_paged_get_sizes(ctypes.byref(self.cfg), ctypes.byref(self.sizes)))
        self.page_tokens, self.num_pages, self.max_pages = page_tokens, num_pages, max_pages
        dev = self.device
        NP = num_pages * kv_heads
        words = page_tokens * head_dim * bits // 32
        self.k_codes = torch.empty((NP, words), dtype=torch.int32, device=dev)
        self.v_codes = torch.empty((NP, words), dtype=torch.int32, device=dev)
        self.k_scales = torch.empty((NP, page_tokens // group_k, head_dim), dtype=torch.float32, device=dev)
        self.v_scales = torch.empty((NP, page_tokens, head_dim // group_v), dtype=torch.float32, device=dev)
        if symmetric:
            self.k_zeros = self.v_zeros = None
        else:
            self.k_zeros = torch.empty((NP, page_tokens // group_k, head_dim), dtype=torch.int16, device=dev)
            self.v_zeros = torch.empty((NP, page_tokens, head_dim // group_v), dtype=torch.int16, device=dev)
        BH = slots * kv_heads
        self.k_residual = torch.zeros((BH, residual, head_dim), dtype=dtype, device=dev)
        self.v_residual = torch.zeros((BH, residual, head_dim), dtype=dtype, device=dev)
        self.page_table = torch.full((slots, max_pages), -1, dtype=torch.int32, device=dev)
        self.workspace = torch.empty(self.sizes.workspace // 4, dtype=torch.float32, device=dev)
        self.state_buf = torch.zeros(-(-self.sizes.state // 16) * 4, dtype=torch.int32, device=dev)
        bufs = Buffers(self.k_codes.data_ptr(), self.k_scales.data_ptr(),
                       self.k_zeros.data_ptr() if self.k_zeros is not None else None,
                       self.v_codes.data_ptr(), self.v_scales.data_ptr(),
                       self.v_zeros.data_ptr() if self.v_zeros is not None else None,
                       self.k_residual.data_ptr(), self.v_residual.data_ptr(), self.state_buf.data_ptr())
        h = ctypes.c_void_p()
        with torch.cuda.device(dev):
            _check(self._lib.kvq_paged_create(ctypes.byref(self.cfg), ctypes.byref(bufs),
                                              self.page_table.data_ptr(), ctypes.byref(h)))
        self._h = h
        self.free_pages = list(range(num_pages - 1, -1, -1))   # pop() hands out 0, 1, 2, ...
        self.pages = [[] for _ in range(slots)]
        self.lens = [-1] * slots

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            self._lib.kvq_paged_destroy(h)
            self._h = None

    def _dev(self, t: torch.Tensor) -> torch.Tensor:
        if t.dtype != self.dtype:
            raise TypeError(f"expected {self.dtype}, got {t.dtype}")
        if t.device != self.device:
            t = t.to(self.device, non_blocking=True)
        return t.contiguous()

    def _grow(self, need: dict, stream):
        """Give each slot b in `need` pages up to need[b] pages; write the new table entries."""
        rows, cols, vals = [], [], []
        for b, n in need.items():
            while len(self.pages[b]) < n:
                if not self.free_pages:
                    raise KVQError(KVQ_ERR_CAPACITY, "the page pool is exhausted")
                pg = self.free_pages.pop()
                rows.append(b)
                cols.append(len(self.pages[b]))
                vals.append(pg)
                self.pages[b].append(pg)
        if vals:
            s = torch.cuda.current_stream(self.device) if stream is None else stream
            with torch.cuda.stream(s):
                self.page_table[torch.tensor(rows, device=self.device), torch.tensor(cols, device=self.device)] = \
                    torch.tensor(vals, dtype=torch.int32, device=self.device)

    def seq_len(self, seq: int) -> int:
        n = ctypes.c_int64()
        _check(self._lib.kvq_paged_seq_len(self._h, seq, ctypes.byref(n)))
        return int(n.value)

    def splits(self) -> int:
        return int(self._lib.kvq_paged_decode_splits(self._h))

    def check_device(self):
        """Raise KVQError if a kernel gave up a bounded wait or met a page outside the pool."""
        _check(self._lib.kvq_paged_check_device(self._h))

    def prefill(self, seq: int, X_K: torch.Tensor, X_V: torch.Tensor, stream=None):
        X_K, X_V = self._dev(X_K), self._dev(X_V)
        g = self.geom
        if X_K.shape != X_V.shape or X_K.dim() != 3 or X_K.shape[0] != g.kv_heads or \
                X_K.shape[2] != g.head_dim:
            raise ValueError(f"X_K/X_V must be [Hkv={g.kv_heads}, T, d={g.head_dim}]")
        T = X_K.shape[1]
        Tq = T // g.residual * g.residual
        if self.lens[seq] >= 0:
            raise KVQError(KVQ_ERR_STATE, f"slot {seq} is active; release it first")
        if Tq > g.capacity:
            raise KVQError(KVQ_ERR_CAPACITY, f"prefill of {T} tokens exceeds capacity {g.capacity}")
        self._grow({seq: -(-Tq // self.page_tokens)}, stream)
        _check(self._lib.kvq_paged_prefill(self._h, seq, X_K.data_ptr(), X_V.data_ptr(), T,
                                           _stream_ptr(stream)))
        self.lens[seq] = T
        self._keep = (X_K, X_V)
        return self

    def append(self, t_K: torch.Tensor, t_V: torch.Tensor, stream=None):
        t_K, t_V = self._dev(t_K), self._dev(t_V)
        g = self.geom
        want = (g.batch, g.kv_heads, g.head_dim)
        if tuple(t_K.shape) != want or tuple(t_V.shape) != want:
            raise ValueError(f"t_K/t_V must be {list(want)}")
        need = {}
        for b, n in enumerate(self.lens):
            if n >= 0 and (n + 1) % g.residual == 0 and n + 1 <= g.capacity:
                need[b] = -(-(n + 1) // self.page_tokens)
        self._grow(need, stream)
        _check(self._lib.kvq_paged_append(self._h, t_K.data_ptr(), t_V.data_ptr(), _stream_ptr(stream)))
        self.lens = [n + 1 if n >= 0 else n for n in self.lens]
        self._keep = (t_K, t_V)
        return self

    def decode_attention(self, t_Q: torch.Tensor, out: torch.Tensor | None = None, stream=None):
        t_Q = self._dev(t_Q)
        g = self.geom
        if tuple(t_Q.shape) != (g.batch, g.q_heads, g.head_dim):
            raise ValueError(f"t_Q must be [{g.batch}, {g.q_heads}, {g.head_dim}]")
        if out is None:
            out = torch.empty((g.batch, g.q_heads, g.head_dim), dtype=torch.float32, device=self.device)
        _check(self._lib.kvq_paged_decode_attention(self._h, t_Q.data_ptr(), out.data_ptr(),
                                                    self.workspace.data_ptr(), self.workspace.numel() * 4,
                                                    _stream_ptr(stream)))
        return out

    def release(self, seq: int, stream=None):
        """End slot `seq`: it becomes inactive and its pages return to the free list (reused by
        later calls, which run after this one on the same stream)."""
        _check(self._lib.kvq_paged_release(self._h, seq, _stream_ptr(stream)))
        self.free_pages.extend(reversed(self.pages[seq]))
        self.pages[seq] = []
        self.lens[seq] = -1
        return self


def _gcd(a: int, b: int) -> int:
    while b:
        a, b = b, a % b
    return a


# ----------------------------------------------------------------------------
# function-style API with the operation names of the method
# ----------------------------------------------------------------------------

def prefill_quantize(X_K: torch.Tensor, X_V: torch.Tensor, G: int, R: int, bits: int, *,
                     q_heads: int | None = None, group_v: int | None = None,
                     symmetric: bool = False, capacity: int | None = None,
                     device=None) -> KVQCache:
    """Create a cache sized for the prompt (plus `capacity`) and quantize X_K, X_V [B, Hkv, T, d]."""
    B, Hkv, T, d = X_K.shape
    cap = capacity if capacity is not None else max(T, 1) + R
    dev = device if device is not None else (X_K.device if X_K.is_cuda else "cuda")
    gv = group_v if group_v is not None else min(G, d)
    cache = KVQCache(B, q_heads or Hkv, Hkv, d, G, gv, R, bits, symmetric, X_K.dtype, cap, dev)
    return cache.prefill_quantize(X_K, X_V)


def append(cache: KVQCache, t_K: torch.Tensor, t_V: torch.Tensor) -> KVQCache:
    return cache.append(t_K, t_V)


def decode_attention(cache: KVQCache, t_Q: torch.Tensor, out=None) -> torch.Tensor:
    return cache.decode_attention(t_Q, out)


def merge_partials(o_all: torch.Tensor, m_all: torch.Tensor, l_all: torch.Tensor,
                   out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Merge n partials (o [n, *rows, d], m and l [n, *rows], float32, one CUDA device) of caches
    holding disjoint tokens into the output [*rows, d]."""
    if not (o_all.is_cuda and m_all.is_cuda and l_all.is_cuda):
        raise ValueError("partials must be CUDA tensors")
    n, d = o_all.shape[0], o_all.shape[-1]
    rows = m_all[0].numel()
    o_all, m_all, l_all = o_all.contiguous(), m_all.contiguous(), l_all.contiguous()
    if out is None:
        out = torch.empty(o_all.shape[1:], dtype=torch.float32, device=o_all.device)
    _check(load().kvq_merge_partials(o_all.data_ptr(), m_all.data_ptr(), l_all.data_ptr(), n, rows, d,
                                     out.data_ptr(), _stream_ptr(stream)))
    return out


def plan_decode(cfg: Config, lengths, num_sms: int = 148, ctas_per_sm: int = 4):
    """(splits over the quantized tokens, 16-token tiles per split, total splits) that a decode
    over sequences of these lengths would use; host only."""
    n = len(lengths)
    arr = (ctypes.c_int64 * max(1, n))(*lengths)
    nq, per, S = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(load().kvq_plan_decode(ctypes.byref(cfg), arr, num_sms, ctas_per_sm, ctypes.byref(nq),
                                  ctypes.byref(per), ctypes.byref(S)))
    return int(nq.value), int(per.value), int(S.value)


def kernel_launches() -> int:
    """Kernels libkvq has launched in this process so far."""
    return int(load().kvq_kernel_launches())
