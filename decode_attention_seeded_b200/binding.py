"""Thin ctypes binding of libtq (C ABI in include/tq.h).

Argument marshalling only: every step of the quantize and decode path runs in
the library's CUDA kernels. Torch tensors supply device pointers and the
current CUDA stream. If libtq.so is missing this module raises on first use;
there is no fallback implementation.
"""

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

TQ_OK = 0
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "workspace", 4: "cuda error",
          5: "device error", 6: "not initialised"}
DTYPES = {"fp32": 0, "bf16": 1, "fp16": 2}
DEV_BAD_SLOT, DEV_BAD_PAGE, DEV_TIMEOUT, DEV_BAD_LENGTH = 0x1, 0x2, 0x4, 0x8
TEST_WAIT_RUNS_OUT = 0x1

_lib = None

_c = ctypes
_SIGS = {
    "tq_version": (_c.c_int, []),
    "tq_status_string": (_c.c_char_p, [_c.c_int]),
    "tq_create": (_c.c_int, [_c.POINTER(_c.c_void_p), _c.c_int, _c.c_int, _c.c_int, _c.c_int]),
    "tq_destroy": (None, [_c.c_void_p]),
    "tq_init_rotation": (_c.c_int, [_c.c_void_p, _c.c_uint64, _c.c_uint64, _c.c_uint64, _c.c_void_p]),
    "tq_init_codebooks": (_c.c_int, [_c.c_void_p, _c.c_int, _c.c_int, _c.c_void_p]),
    "tq_block_bytes": (_c.c_size_t, [_c.c_void_p]),
    "tq_page_bytes": (_c.c_size_t, [_c.c_void_p, _c.c_int]),
    "tq_quantize_append": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int, _c.c_int, _c.c_int,
                                      _c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_void_p]),
    "tq_quantize_prefill": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int, _c.c_int, _c.c_int,
                                       _c.c_void_p, _c.c_int, _c.c_void_p, _c.c_int64, _c.c_void_p]),
    "tq_decode_workspace_bytes": (_c.c_size_t, [_c.c_void_p, _c.c_int, _c.c_int, _c.c_int, _c.c_int]),
    "tq_decode_attention": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int, _c.c_void_p, _c.c_int64,
                                       _c.c_void_p, _c.c_int, _c.c_void_p, _c.c_int, _c.c_int, _c.c_int,
                                       _c.c_int, _c.c_float, _c.c_void_p, _c.c_void_p, _c.c_size_t,
                                       _c.c_void_p]),
    "tq_decode_step": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int, _c.c_void_p, _c.c_int,
                                  _c.c_void_p, _c.c_int64, _c.c_void_p, _c.c_int, _c.c_void_p, _c.c_int, _c.c_int,
                                  _c.c_int, _c.c_int, _c.c_float, _c.c_void_p, _c.c_void_p, _c.c_size_t,
                                  _c.c_void_p]),
    "tq_decode_attention_noalloc": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int, _c.c_void_p, _c.c_int64,
                                               _c.c_void_p, _c.c_int, _c.c_void_p, _c.c_int, _c.c_int, _c.c_int,
                                               _c.c_int, _c.c_float, _c.c_void_p, _c.c_void_p]),
    "tq_set_sparse_v": (_c.c_int, [_c.c_void_p, _c.c_float]),
    "tq_set_test_flags": (_c.c_int, [_c.c_void_p, _c.c_uint]),
    "tq_decode_logits": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int, _c.c_void_p, _c.c_int64, _c.c_void_p,
                                    _c.c_int, _c.c_void_p, _c.c_int, _c.c_int, _c.c_int, _c.c_int, _c.c_float,
                                    _c.c_void_p, _c.c_int64, _c.c_void_p]),
    "tq_get_device_error": (_c.c_int, [_c.c_void_p, _c.POINTER(_c.c_uint32), _c.c_void_p]),
    "tq_host_sign_vector": (_c.c_int, [_c.c_uint64, _c.c_int, _c.c_void_p]),
    "tq_host_gaussian_sketch": (_c.c_int, [_c.c_uint64, _c.c_int, _c.c_int, _c.c_void_p]),
    "tq_host_codebook": (_c.c_int, [_c.c_int, _c.c_int, _c.c_void_p, _c.c_void_p]),
}


class TQError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({code})")
        self.code = code


def lib():
    """Load libtq.so (once). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libtq.so not found at {LIB_PATH}; build it with "
                               "`python -m decode_attention_seeded_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


def _check(fn, code):
    if code != TQ_OK:
        raise TQError(fn, code)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return ctypes.c_void_p(stream)


def _dtype_code(t):
    import torch
    return {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}[t.dtype]


# ------------------------------------------------------------ host-only tables
def host_sign_vector(seed: int, d: int = 128) -> np.ndarray:
    out = np.zeros(d, dtype=np.int8)
    _check("tq_host_sign_vector", lib().tq_host_sign_vector(seed, d, out.ctypes.data))
    return out


def host_gaussian_sketch(seed: int, m: int = 128, d: int = 128) -> np.ndarray:
    out = np.zeros(m * d, dtype=np.uint16)
    _check("tq_host_gaussian_sketch", lib().tq_host_gaussian_sketch(seed, m, d, out.ctypes.data))
    return out.view(np.float16).reshape(m, d)


def host_codebook(bits: int, d: int = 128):
    c = np.zeros(2 ** bits, dtype=np.uint16)
    t = np.zeros(2 ** bits - 1, dtype=np.float32)
    _check("tq_host_codebook", lib().tq_host_codebook(bits, d, c.ctypes.data, t.ctypes.data))
    return c.view(np.float16), t


# --------------------------------------------------------------------- context
class Context:
    """A libtq context on one CUDA device (head_dim 128, m = 128, 16-token pages)."""

    def __init__(self, key_bits: int, value_bits: int, seeds, device: int = 0, stream=None):
        self._h = ctypes.c_void_p()
        L = lib()
        _check("tq_create", L.tq_create(ctypes.byref(self._h), 128, 128, 16, device))
        self.device = device
        s = _stream(stream)
        _check("tq_init_rotation", L.tq_init_rotation(self._h, int(seeds[0]), int(seeds[1]), int(seeds[2]), s))
        _check("tq_init_codebooks", L.tq_init_codebooks(self._h, key_bits, value_bits, s))
        self.key_bits, self.value_bits = key_bits, value_bits

    def close(self):
        if self._h:
            lib().tq_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def block_bytes(self) -> int:
        return int(lib().tq_block_bytes(self._h))

    def page_bytes(self, n_kv_heads: int) -> int:
        return int(lib().tq_page_bytes(self._h, n_kv_heads))

    def quantize_append(self, k, v, slot_mapping, cache, n_cache_pages: int, stream=None):
        """k, v: [T, n_kv, 128] CUDA tensors; slot_mapping int64 [T]; cache uint8 CUDA tensor."""
        n_tokens, n_kv = k.shape[0], k.shape[1]
        _check("tq_quantize_append", lib().tq_quantize_append(
            self._h, _ptr(k), _ptr(v), _dtype_code(k), n_tokens, n_kv, _ptr(slot_mapping), _ptr(cache),
            n_cache_pages, _stream(stream)))

    def quantize_prefill(self, k, v, block_table, start_pos: int, cache, n_cache_pages: int, stream=None):
        n_tokens, n_kv = k.shape[0], k.shape[1]
        _check("tq_quantize_prefill", lib().tq_quantize_prefill(
            self._h, _ptr(k), _ptr(v), _dtype_code(k), n_tokens, n_kv, _ptr(block_table), start_pos,
            _ptr(cache), n_cache_pages, _stream(stream)))

    def decode_workspace_bytes(self, batch: int, n_q_heads: int, n_kv_heads: int, max_seq_len: int) -> int:
        return int(lib().tq_decode_workspace_bytes(self._h, batch, n_q_heads, n_kv_heads, max_seq_len))

    def decode_attention(self, q, cache, n_cache_pages: int, block_tables, seq_lens, n_kv_heads: int,
                         max_seq_len: int, out, workspace, scale: float = 0.0, stream=None):
        batch, n_q = q.shape[0], q.shape[1]
        _check("tq_decode_attention", lib().tq_decode_attention(
            self._h, _ptr(q), _dtype_code(q), _ptr(cache), n_cache_pages, _ptr(block_tables),
            block_tables.shape[1], _ptr(seq_lens), batch, n_q, n_kv_heads, max_seq_len, scale, _ptr(out),
            _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))

    def decode_step(self, k_new, v_new, q, cache, n_cache_pages: int, block_tables, seq_lens, n_kv_heads: int,
                    max_seq_len: int, out, workspace, scale: float = 0.0, stream=None):
        """Append one token per sequence (at position seq_lens[b] - 1) and attend."""
        batch, n_q = q.shape[0], q.shape[1]
        _check("tq_decode_step", lib().tq_decode_step(
            self._h, _ptr(k_new), _ptr(v_new), _dtype_code(k_new), _ptr(q), _dtype_code(q), _ptr(cache),
            n_cache_pages, _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens), batch, n_q, n_kv_heads,
            max_seq_len, scale, _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
            _stream(stream)))

    def decode_attention_noalloc(self, q, cache, n_cache_pages: int, block_tables, seq_lens, n_kv_heads: int,
                                 max_seq_len: int, out, scale: float = 0.0, stream=None):
        """decode_attention with the library's fixed per-device scratch instead of a workspace."""
        batch, n_q = q.shape[0], q.shape[1]
        _check("tq_decode_attention_noalloc", lib().tq_decode_attention_noalloc(
            self._h, _ptr(q), _dtype_code(q), _ptr(cache), n_cache_pages, _ptr(block_tables),
            block_tables.shape[1], _ptr(seq_lens), batch, n_q, n_kv_heads, max_seq_len, scale, _ptr(out),
            _stream(stream)))

    def decode_logits(self, q, cache, n_cache_pages: int, block_tables, seq_lens, n_kv_heads: int,
                      max_seq_len: int, logits, scale: float = 0.0, stream=None):
        """logits: float32 [batch, n_q_heads, stride >= max_seq_len] CUDA tensor."""
        batch, n_q = q.shape[0], q.shape[1]
        _check("tq_decode_logits", lib().tq_decode_logits(
            self._h, _ptr(q), _dtype_code(q), _ptr(cache), n_cache_pages, _ptr(block_tables), block_tables.shape[1],
            _ptr(seq_lens), batch, n_q, n_kv_heads, max_seq_len, scale, _ptr(logits), logits.shape[-1],
            _stream(stream)))

    def set_sparse_v(self, tau: float):
        """Sparse V threshold of later decode calls (0: dense attention)."""
        _check("tq_set_sparse_v", lib().tq_set_sparse_v(self._h, tau))

    def set_test_flags(self, flags: int):
        """Test hook bits (TEST_WAIT_RUNS_OUT) of later decode calls; 0 turns them off."""
        _check("tq_set_test_flags", lib().tq_set_test_flags(self._h, flags))

    def device_error(self, stream=None) -> int:
        code = ctypes.c_uint32(0)
        _check("tq_get_device_error", lib().tq_get_device_error(self._h, ctypes.byref(code), _stream(stream)))
        return int(code.value)
