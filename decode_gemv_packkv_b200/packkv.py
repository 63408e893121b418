"""Python binding of the PackKV C ABI (libpackkv.so): argument marshalling only.

Every function here has the name of the C entry point it calls and forwards
torch tensors as raw device pointers on the current CUDA stream.  No step of
the encoder or of the GEMVs runs in Python or PyTorch: importing this module
raises if the CUDA library is missing, and there is no fallback.

`PackKVCache` owns the device buffers of one cache (allocated with torch) and
the `packkv_cache` struct that points into them.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("PACKKV_LIB") or os.path.join(_HERE, "libpackkv.so")

BLOCK_TOKENS = 128
HEAD_DIM = 128
FORMAT_VERSION = 1

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CAPACITY, ERR_CUDA, ERR_DEVICE = range(6)
DEV_CAPACITY, DEV_NONFINITE, DEV_BAD_RECORD, DEV_TIMEOUT = 0x1, 0x2, 0x4, 0x8
KEY_IDENTITY, KEY_K_SUM, KEY_KV_SUM = 0, 1, 2
UNITS_FOR, UNITS_WIDTH_ONLY = 0, 1      # how the encoder sizes a unit (base = min, or 0)

EXPORTED = [
    "packkv_abi_version", "packkv_cache_struct_size", "packkv_status_string", "packkv_record_bytes_max",
    "packkv_workspace_bytes", "packkv_cache_check", "packkv_cache_reset", "packkv_encode_block",
    "packkv_append_token", "packkv_qk_gemv", "packkv_pv_gemv", "packkv_get_status",
    "packkv_pv_gemv_noalloc", "packkv_attention_workspace_bytes",
    "packkv_attention_decode", "packkv_append_token_masked",
]

RAGGED_MAX_BATCH = 2048


class PackKVError(RuntimeError):
    def __init__(self, call: str, status: int, msg: str):
        super().__init__(f"{call}: {msg} (status {status})")
        self.status = status


class Format(ctypes.Structure):
    _fields_ = [("version", ctypes.c_uint32), ("bits", ctypes.c_uint32), ("block_tokens", ctypes.c_uint32),
                ("group_tokens", ctypes.c_uint32), ("head_dim", ctypes.c_uint32), ("reorder_key", ctypes.c_uint32),
                ("unit_mode", ctypes.c_uint32)]


class CacheStruct(ctypes.Structure):
    _fields_ = [("fmt", Format), ("batch", ctypes.c_int32), ("kv_heads", ctypes.c_int32),
                ("max_blocks", ctypes.c_int32), ("n_blocks", ctypes.c_int32), ("tail_len", ctypes.c_int32),
                ("reserved0", ctypes.c_int32), ("k_arena", ctypes.c_void_p), ("v_arena", ctypes.c_void_p),
                ("arena_bytes", ctypes.c_uint64), ("k_index", ctypes.c_void_p), ("v_index", ctypes.c_void_p),
                ("k_tail", ctypes.c_void_p), ("v_tail", ctypes.c_void_p), ("ctrl", ctypes.c_void_p),
                ("perm", ctypes.c_void_p), ("seq_blocks", ctypes.POINTER(ctypes.c_int32)),
                ("seq_tail", ctypes.POINTER(ctypes.c_int32)), ("block_table", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m decode_gemv_packkv_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(CacheStruct)
    vp, i32, i64, u32, sz, f32 = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32,
                                  ctypes.c_size_t, ctypes.c_float)
    sig = {
        "packkv_abi_version": (u32, []),
        "packkv_cache_struct_size": (sz, []),
        "packkv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "packkv_record_bytes_max": (sz, [u32]),
        "packkv_workspace_bytes": (sz, [P, i32]),
        "packkv_cache_check": (ctypes.c_int, [P]),
        "packkv_cache_reset": (ctypes.c_int, [P, vp]),
        "packkv_encode_block": (ctypes.c_int, [P, vp, vp, i32, vp]),
        "packkv_append_token": (ctypes.c_int, [P, vp, vp, vp]),
        "packkv_qk_gemv": (ctypes.c_int, [P, vp, i32, f32, vp, i64, vp, sz, vp]),
        "packkv_pv_gemv": (ctypes.c_int, [P, vp, i64, i32, vp, vp, sz, vp]),
        "packkv_get_status": (ctypes.c_int, [P, vp, ctypes.POINTER(u32)]),
        "packkv_pv_gemv_noalloc": (ctypes.c_int, [P, vp, i64, i32, vp, vp]),
        "packkv_attention_workspace_bytes": (sz, [P, i32]),
        "packkv_attention_decode": (ctypes.c_int, [P, vp, i32, f32, vp, vp, sz, vp]),
        "packkv_append_token_masked": (ctypes.c_int, [P, vp, vp, ctypes.POINTER(ctypes.c_uint8), vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if lib.packkv_cache_struct_size() != ctypes.sizeof(CacheStruct):
        raise ImportError("packkv_cache layout mismatch between libpackkv.so and the binding")
    return lib


_lib = _load()


def _check(call: str, status: int):
    if status != OK:
        raise PackKVError(call, status, _lib.packkv_status_string(status).decode())


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def record_bytes_max(bits: int) -> int:
    return int(_lib.packkv_record_bytes_max(bits))


class PackKVCache:
    """Device buffers + the packkv_cache struct of one layer's packed cache.

    ragged=True gives every sequence its own length (host counters seq_blocks /
    seq_tail in the struct); block_table (int32 [batch, max_blocks], on the device)
    maps each sequence's logical blocks to physical blocks of the index."""

    def __init__(self, batch: int, kv_heads: int, max_blocks: int, bits: int, reorder_key: int = KEY_K_SUM,
                 arena_bytes: int | None = None, keep_perm: bool = False, device="cuda", ragged: bool = False,
                 block_table: torch.Tensor | None = None, unit_mode: int = 0):
        dev = torch.device(device)
        if arena_bytes is None:
            arena_bytes = batch * kv_heads * max_blocks * record_bytes_max(bits)
        arena_bytes = (int(arena_bytes) + 15) // 16 * 16
        self.k_arena = torch.empty(arena_bytes, dtype=torch.uint8, device=dev)
        self.v_arena = torch.empty(arena_bytes, dtype=torch.uint8, device=dev)
        self.k_index = torch.zeros((batch, kv_heads, max_blocks, 2), dtype=torch.int32, device=dev)
        self.v_index = torch.zeros_like(self.k_index)
        self.k_tail = torch.zeros((batch, kv_heads, BLOCK_TOKENS, HEAD_DIM), dtype=torch.float16, device=dev)
        self.v_tail = torch.zeros_like(self.k_tail)
        self.ctrl = torch.zeros(4, dtype=torch.int64, device=dev)
        self.perm = (torch.zeros((batch, kv_heads, max_blocks, BLOCK_TOKENS), dtype=torch.uint8, device=dev)
                     if keep_perm else None)
        self.s = CacheStruct()
        self.s.fmt = Format(FORMAT_VERSION, bits, BLOCK_TOKENS, 32, HEAD_DIM, reorder_key, unit_mode)
        self.s.batch, self.s.kv_heads, self.s.max_blocks = batch, kv_heads, max_blocks
        self.s.n_blocks = self.s.tail_len = 0
        self.s.k_arena, self.s.v_arena = self.k_arena.data_ptr(), self.v_arena.data_ptr()
        self.s.arena_bytes = arena_bytes
        self.s.k_index, self.s.v_index = self.k_index.data_ptr(), self.v_index.data_ptr()
        self.s.k_tail, self.s.v_tail = self.k_tail.data_ptr(), self.v_tail.data_ptr()
        self.s.ctrl = self.ctrl.data_ptr()
        self.s.perm = self.perm.data_ptr() if self.perm is not None else None
        self.ragged = ragged
        if ragged:
            self._seq_blocks = (ctypes.c_int32 * batch)()
            self._seq_tail = (ctypes.c_int32 * batch)()
            self.s.seq_blocks = ctypes.cast(self._seq_blocks, ctypes.POINTER(ctypes.c_int32))
            self.s.seq_tail = ctypes.cast(self._seq_tail, ctypes.POINTER(ctypes.c_int32))
        self.block_table = None
        if block_table is not None:
            bt = block_table.to(device=dev, dtype=torch.int32).contiguous()
            if tuple(bt.shape) != (batch, max_blocks):
                raise ValueError("block_table must be int32 [batch, max_blocks]")
            self.block_table = bt
            self.s.block_table = bt.data_ptr()
        _check("packkv_cache_check", _lib.packkv_cache_check(ctypes.byref(self.s)))
        self._ws = {}

    # host counters live in the struct
    @property
    def n_blocks(self) -> int:
        return self.s.n_blocks

    @property
    def tail_len(self) -> int:
        return self.s.tail_len

    @property
    def tokens(self) -> int:
        """Tokens of the longest sequence (every sequence, for a uniform batch)."""
        if self.ragged:
            return max((self.seq_tokens(b) for b in range(self.batch)), default=0)
        return self.s.n_blocks * BLOCK_TOKENS + self.s.tail_len

    def seq_tokens(self, b: int) -> int:
        if not self.ragged:
            return self.tokens
        return self._seq_blocks[b] * BLOCK_TOKENS + self._seq_tail[b]

    @property
    def seq_blocks(self):
        return list(self._seq_blocks) if self.ragged else [self.s.n_blocks] * self.batch

    @property
    def seq_tail(self):
        return list(self._seq_tail) if self.ragged else [self.s.tail_len] * self.batch

    @property
    def bits(self) -> int:
        return self.s.fmt.bits

    @property
    def batch(self) -> int:
        return self.s.batch

    @property
    def kv_heads(self) -> int:
        return self.s.kv_heads

    def workspace(self, q_heads: int) -> torch.Tensor:
        """p·V workspace for q_heads (allocated once, reused by every call)."""
        if q_heads not in self._ws:
            n = packkv_workspace_bytes(self, q_heads)
            self._ws[q_heads] = torch.zeros(max(n, 16), dtype=torch.uint8, device=self.k_arena.device)
        return self._ws[q_heads]

    def attention_workspace(self, q_heads: int) -> torch.Tensor:
        """Fused-attention workspace for q_heads (allocated once, reused by every call)."""
        key = ("attn", q_heads)
        if key not in self._ws:
            n = int(_lib.packkv_attention_workspace_bytes(ctypes.byref(self.s), q_heads))
            self._ws[key] = torch.zeros(max(n, 16), dtype=torch.uint8, device=self.k_arena.device)
        return self._ws[key]

    def arena_used(self):
        """(K bytes, V bytes) in use; synchronises."""
        ends = self.ctrl[:2].cpu()
        return int(ends[0]) * 16, int(ends[1]) * 16


# --- the C entry points, same names --------------------------------------------------------
def packkv_workspace_bytes(cache: PackKVCache, q_heads: int) -> int:
    return int(_lib.packkv_workspace_bytes(ctypes.byref(cache.s), q_heads))


def packkv_cache_reset(cache: PackKVCache, stream=None):
    _check("packkv_cache_reset", _lib.packkv_cache_reset(ctypes.byref(cache.s), _stream(stream)))


def packkv_encode_block(cache: PackKVCache, k: torch.Tensor, v: torch.Tensor, n_blocks: int, stream=None):
    """k, v: fp16 [batch, kv_heads, n_blocks*128, 128]."""
    _check_kv(cache, k, v, n_blocks * BLOCK_TOKENS)
    _check("packkv_encode_block", _lib.packkv_encode_block(ctypes.byref(cache.s), _ptr(k), _ptr(v), n_blocks,
                                                           _stream(stream)))


def packkv_append_token(cache: PackKVCache, k: torch.Tensor, v: torch.Tensor, stream=None):
    """k, v: fp16 [batch, kv_heads, 128]."""
    if k.dtype != torch.float16 or v.dtype != torch.float16 or tuple(k.shape) != (cache.batch, cache.kv_heads,
                                                                                   HEAD_DIM) or k.shape != v.shape:
        raise ValueError("k, v must be fp16 [batch, kv_heads, 128]")
    _check("packkv_append_token", _lib.packkv_append_token(ctypes.byref(cache.s), _ptr(k), _ptr(v),
                                                           _stream(stream)))


def packkv_append_token_masked(cache: PackKVCache, k: torch.Tensor, v: torch.Tensor, active, stream=None):
    """Ragged caches: one token for the sequences with active[b] (k, v fp16 [batch, kv_heads, 128])."""
    if k.dtype != torch.float16 or v.dtype != torch.float16 or tuple(k.shape) != (cache.batch, cache.kv_heads,
                                                                                   HEAD_DIM) or k.shape != v.shape:
        raise ValueError("k, v must be fp16 [batch, kv_heads, 128]")
    act = (ctypes.c_uint8 * cache.batch)(*[1 if a else 0 for a in active])
    _check("packkv_append_token_masked", _lib.packkv_append_token_masked(ctypes.byref(cache.s), _ptr(k), _ptr(v),
                                                                         act, _stream(stream)))


def packkv_qk_gemv(cache: PackKVCache, q: torch.Tensor, scale: float, scores: torch.Tensor, stream=None):
    """q: fp16 [batch, q_heads, 128]; scores: fp32 [batch, q_heads, ld] with ld >= tokens, ld % 4 == 0."""
    if q.dtype != torch.float16 or q.dim() != 3 or scores.dtype != torch.float32 or scores.dim() != 3:
        raise ValueError("q must be fp16 [B, Hq, 128] and scores fp32 [B, Hq, ld]")
    _check("packkv_qk_gemv", _lib.packkv_qk_gemv(ctypes.byref(cache.s), _ptr(q), q.shape[1], float(scale),
                                                 _ptr(scores), scores.shape[2], None, 0, _stream(stream)))


def packkv_pv_gemv(cache: PackKVCache, p: torch.Tensor, out: torch.Tensor, ws: torch.Tensor | None = None,
                   stream=None):
    """p: fp32 [batch, q_heads, ld] (storage order); out: fp32 [batch, q_heads, 128]."""
    if p.dtype != torch.float32 or p.dim() != 3 or out.dtype != torch.float32:
        raise ValueError("p must be fp32 [B, Hq, ld], out fp32 [B, Hq, 128]")
    if ws is None:
        ws = cache.workspace(p.shape[1])
    _check("packkv_pv_gemv", _lib.packkv_pv_gemv(ctypes.byref(cache.s), _ptr(p), p.shape[2], p.shape[1],
                                                 _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))


def packkv_pv_gemv_noalloc(cache: PackKVCache, p: torch.Tensor, out: torch.Tensor, stream=None):
    """p·V with the library's own fixed scratch instead of a workspace, for callers that
    cannot allocate device memory.  Raises PackKVError (capacity) if the call needs more
    scratch than PV_NOALLOC_SCRATCH_BYTES; overlapping calls share the scratch."""
    if p.dtype != torch.float32 or p.dim() != 3 or out.dtype != torch.float32:
        raise ValueError("p must be fp32 [B, Hq, ld], out fp32 [B, Hq, 128]")
    _check("packkv_pv_gemv_noalloc", _lib.packkv_pv_gemv_noalloc(ctypes.byref(cache.s), _ptr(p), p.shape[2],
                                                                 p.shape[1], _ptr(out), _stream(stream)))


# size of the library's fixed p·V scratch (PACKKV_PV_NOALLOC_SCRATCH_BYTES in packkv.h)
PV_NOALLOC_SCRATCH_BYTES = 8 << 20


def packkv_attention_decode(cache: PackKVCache, q: torch.Tensor, scale: float, out: torch.Tensor,
                            ws: torch.Tensor | None = None, stream=None):
    """q: fp16 [batch, q_heads, 128]; out: fp32 [batch, q_heads, 128] = softmax(scale q·Kᵀ)·V."""
    if q.dtype != torch.float16 or q.dim() != 3 or out.dtype != torch.float32:
        raise ValueError("q must be fp16 [B, Hq, 128], out fp32 [B, Hq, 128]")
    if ws is None:
        ws = cache.attention_workspace(q.shape[1])
    _check("packkv_attention_decode", _lib.packkv_attention_decode(ctypes.byref(cache.s), _ptr(q), q.shape[1],
                                                                   float(scale), _ptr(out), _ptr(ws), ws.numel(),
                                                                   _stream(stream)))


def packkv_get_status(cache: PackKVCache, stream=None) -> int:
    """Synchronises the stream; returns the device status bits (and clears them)."""
    bits = ctypes.c_uint32(0)
    _lib.packkv_get_status(ctypes.byref(cache.s), _stream(stream), ctypes.byref(bits))
    return int(bits.value)


def _check_kv(cache, k, v, tokens):
    want = (cache.batch, cache.kv_heads, tokens, HEAD_DIM)
    if k.dtype != torch.float16 or v.dtype != torch.float16 or tuple(k.shape) != want or tuple(v.shape) != want:
        raise ValueError(f"k, v must be fp16 {want}")


def prefill(cache: PackKVCache, k: torch.Tensor, v: torch.Tensor, stream=None):
    """Encodes the full blocks of k, v [B, H, T, 128] and appends the remaining T % 128 tokens."""
    t = k.shape[2]
    nb = t // BLOCK_TOKENS
    if nb:
        packkv_encode_block(cache, k[:, :, :nb * BLOCK_TOKENS].contiguous(), v[:, :, :nb * BLOCK_TOKENS].contiguous(),
                            nb, stream)
    for i in range(nb * BLOCK_TOKENS, t):
        packkv_append_token(cache, k[:, :, i].contiguous(), v[:, :, i].contiguous(), stream)
