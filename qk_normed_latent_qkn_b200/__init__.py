"""Python binding of libqkn (QK-Normed MLA absorbed latent decode for B200).

Argument marshalling only: every call forwards device pointers, sizes and the
current CUDA stream to the C ABI declared in ``include/qkn.h``; all
arithmetic runs in the library's kernels.  PyTorch is used for device memory
and streams.  There is no fallback: if ``libqkn.so`` is missing or a call
fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqkn.so")

# ----------------------------------------------------------------- enums
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_BOUNDS = range(6)
F32, BF16 = 0, 1
AK_CACHE, AK_ONE = 0, 1
KERNEL_AUTO, KERNEL_SIMT, KERNEL_TCGEN05 = 0, 1, 2

EXPORTED = ["qkn_append", "qkn_absorb_query", "qkn_decode_workspace_size", "qkn_workspace_init",
            "qkn_decode", "qkn_read_device_status", "qkn_decode_kernel_for", "qkn_status_string",
            "qkn_version", "qkn_decode_noalloc", "qkn_append_absorb", "qkn_key_gram", "qkn_decode_up",
            "qkn_merge_partials", "qkn_gqa_append", "qkn_gqa_workspace_size", "qkn_gqa_decode"]
NOALLOC_SCRATCH_BYTES = 32 << 20


class QknError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


class _Dims(ctypes.Structure):
    _fields_ = [("num_heads", ctypes.c_int32), ("num_groups", ctypes.c_int32), ("r_kv", ctypes.c_int32),
                ("d_h", ctypes.c_int32), ("d_rope", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("eps", ctypes.c_float), ("softmax_scale", ctypes.c_float), ("rope_theta", ctypes.c_float),
                ("dtype", ctypes.c_int32)]


class _Cache(ctypes.Structure):
    _fields_ = [("latent", ctypes.c_void_p), ("k_rope", ctypes.c_void_p), ("a_k", ctypes.c_void_p),
                ("num_blocks", ctypes.c_int32), ("ak_scratch", ctypes.c_void_p)]


class _GqaCache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("k_rope", ctypes.c_void_p),
                ("num_blocks", ctypes.c_int32), ("d_v", ctypes.c_int32)]


class _Opts(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int32), ("max_ctas", ctypes.c_int32), ("head_tile", ctypes.c_int32),
                ("wait_limit", ctypes.c_int64), ("split_event", ctypes.c_void_p),
                ("step_writes_only", ctypes.c_int32), ("test_withhold_ak", ctypes.c_int32),
                ("vis_end", ctypes.c_void_p)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with `python -m qk_normed_latent_qkn_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    PD, PC, PO = ctypes.POINTER(_Dims), ctypes.POINTER(_Cache), ctypes.POINTER(_Opts)
    PG = ctypes.POINTER(_GqaCache)
    sig = {
        "qkn_append": (I32, [PD, PC, P, P, P, P, I32, P, P, P, P]),
        "qkn_key_gram": (I32, [PD, P, P, P]),
        "qkn_absorb_query": (I32, [PD, P, P, P, I32, P, P, P, P, P, P, P, P]),
        "qkn_decode_workspace_size": (I32, [PD, I32, I32, I32, ctypes.POINTER(SZ)]),
        "qkn_workspace_init": (I32, [P, SZ, P]),
        "qkn_decode": (I32, [PD, PC, I32, P, P, P, P, I32, P, I32, I32, P, SZ, P, P, PO, P]),
        "qkn_decode_up": (I32, [PD, PC, I32, P, P, P, P, I32, P, I32, I32, P, I32, P, SZ, P, P, PO, P]),
        "qkn_read_device_status": (I32, [P, P, ctypes.POINTER(I32)]),
        "qkn_merge_partials": (I32, [PD, I32, I64, P, P, P, P, P]),
        "qkn_decode_kernel_for": (I32, [PD, I32, PO]),
        "qkn_status_string": (ctypes.c_char_p, [I32]),
        "qkn_version": (I32, []),
        "qkn_decode_noalloc": (I32, [PD, PC, I32, P, P, P, P, I32, P, I32, I32, P, P, P, PO, P]),
        "qkn_append_absorb": (I32, [PD, PC, P, P, P, P, I32, P, P, P, I32, P, P, P, P, P, P, P, P, P, P]),
        "qkn_gqa_append": (I32, [PD, PG, P, P, P, P, I32, P, P, P, P, P]),
        "qkn_gqa_workspace_size": (I32, [PD, I32, I32, I32, I32, ctypes.POINTER(SZ)]),
        "qkn_gqa_decode": (I32, [PD, PG, P, P, P, P, P, I32, P, I32, I32, P, I32, P, SZ, P, P, I32, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


_lib = _load()


def status_string(status: int) -> str:
    return _lib.qkn_status_string(int(status)).decode()


def version() -> int:
    return int(_lib.qkn_version())


def _check(status: int, what: str) -> None:
    if status != OK:
        raise QknError(status, what)


# ----------------------------------------------------------------- dims / cache
@dataclasses.dataclass(frozen=True)
class Dims:
    num_heads: int
    num_groups: int
    r_kv: int
    d_h: int
    d_rope: int
    eps: float = 1e-6
    softmax_scale: Optional[float] = None     # None: the library's default, 1/sqrt(d_h + d_rope)
    rope_theta: float = 10000.0
    dtype: int = BF16
    block_size: int = 64

    def c(self) -> _Dims:
        scale = self.softmax_scale if self.softmax_scale is not None else 0.0
        return _Dims(self.num_heads, self.num_groups, self.r_kv, self.d_h, self.d_rope, self.block_size,
                     self.eps, scale, self.rope_theta, self.dtype)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == BF16 else torch.float32


class Cache:
    """Paged decode cache: latent, normalised+rotated RoPE key, and the a_k scalar cache."""

    def __init__(self, dims: Dims, num_blocks: int, device="cuda"):
        bs = dims.block_size
        self.dims = dims
        self.num_blocks = num_blocks
        self.latent = torch.empty((num_blocks, bs, dims.r_kv), dtype=dims.torch_dtype, device=device)
        self.k_rope = torch.empty((num_blocks, bs, dims.d_rope), dtype=dims.torch_dtype, device=device)
        self.a_k = torch.empty((num_blocks, bs, dims.num_groups), dtype=torch.float32, device=device)
        # append's per-slot accumulator and arrival count; zero now, left zero by every append
        self.ak_scratch = torch.zeros((num_blocks, bs, dims.num_groups, 2), dtype=torch.int32, device=device)

    def c(self) -> _Cache:
        return _Cache(self.latent.data_ptr(), self.k_rope.data_ptr(), self.a_k.data_ptr(), self.num_blocks,
                      None if self.ak_scratch is None else self.ak_scratch.data_ptr())


class GqaCache:
    """The GQA route's paged cache: per-group normalised keys and values, and the shared RoPE key."""

    def __init__(self, dims: Dims, num_blocks: int, d_v: int, device="cuda"):
        bs = dims.block_size
        self.dims = dims
        self.num_blocks = num_blocks
        self.d_v = d_v
        self.k = torch.empty((num_blocks, dims.num_groups, bs, dims.d_h), dtype=dims.torch_dtype, device=device)
        self.v = torch.empty((num_blocks, dims.num_groups, bs, d_v), dtype=dims.torch_dtype, device=device)
        self.k_rope = torch.empty((num_blocks, bs, dims.d_rope), dtype=dims.torch_dtype, device=device)

    def c(self) -> _GqaCache:
        return _GqaCache(self.k.data_ptr(), self.v.data_ptr(), self.k_rope.data_ptr(), self.num_blocks, self.d_v)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _opts(kernel=KERNEL_AUTO, max_ctas=0, head_tile=0, wait_limit=0, split_event=None, step_writes_only=0,
          test_withhold_ak=0, vis_end=None) -> _Opts:
    return _Opts(kernel, max_ctas, head_tile, wait_limit, split_event, step_writes_only, test_withhold_ak,
                 vis_end)


# ----------------------------------------------------------------- calls
def key_gram(dims: Dims, w_k, out, stream=None) -> None:
    """out[g] = W^K_g (W^K_g)^T, fp32 [num_groups, r_kv, r_kv] (see qkn_key_gram)."""
    _check(_lib.qkn_key_gram(ctypes.byref(dims.c()), _ptr(w_k), _ptr(out), _stream(stream)), "qkn_key_gram")


def append(dims: Dims, cache: Cache, c_new, k_rope_raw, slot, pos, w_k, key_gram, gamma_kr, stream=None) -> None:
    """Write tokens into the cache and compute their a_k (see qkn_append); key_gram may be None."""
    n_tok = int(c_new.shape[0]) if c_new is not None else 0
    _check(_lib.qkn_append(ctypes.byref(dims.c()), ctypes.byref(cache.c()), _ptr(c_new), _ptr(k_rope_raw),
                           _ptr(slot), _ptr(pos), n_tok, _ptr(w_k), _ptr(key_gram), _ptr(gamma_kr),
                           _stream(stream)),
           "qkn_append")


def absorb_query(dims: Dims, q, q_rope, pos, w_k, gamma_q, gamma_k, gamma_qr, q_tilde, a_q, q_rope_hat,
                 stream=None) -> None:
    """q~, a_q and the rotated RoPE query from q and q^R (see qkn_absorb_query)."""
    n_q = int(q.shape[0])
    _check(_lib.qkn_absorb_query(ctypes.byref(dims.c()), _ptr(q), _ptr(q_rope), _ptr(pos), n_q, _ptr(w_k),
                                 _ptr(gamma_q), _ptr(gamma_k), _ptr(gamma_qr), _ptr(q_tilde), _ptr(a_q),
                                 _ptr(q_rope_hat), _stream(stream)), "qkn_absorb_query")


def append_absorb(dims: Dims, cache: Cache, c_new, k_rope_raw, slot, pos, q, q_rope, qpos, w_k, key_gram, gamma_q,
                  gamma_k, gamma_qr, gamma_kr, q_tilde, a_q, q_rope_hat, stream=None) -> None:
    """qkn_append followed by qkn_absorb_query, in one launch where possible (see qkn_append_absorb)."""
    _check(_lib.qkn_append_absorb(ctypes.byref(dims.c()), ctypes.byref(cache.c()), _ptr(c_new), _ptr(k_rope_raw),
                                  _ptr(slot), _ptr(pos), int(c_new.shape[0]), _ptr(q), _ptr(q_rope), _ptr(qpos),
                                  int(q.shape[0]), _ptr(w_k), _ptr(key_gram), _ptr(gamma_q), _ptr(gamma_k),
                                  _ptr(gamma_qr),
                                  _ptr(gamma_kr), _ptr(q_tilde), _ptr(a_q), _ptr(q_rope_hat), _stream(stream)),
           "qkn_append_absorb")


def decode_workspace_size(dims: Dims, batch: int, s_q: int, num_sms: int = 0) -> int:
    out = ctypes.c_size_t(0)
    _check(_lib.qkn_decode_workspace_size(ctypes.byref(dims.c()), batch, s_q, num_sms, ctypes.byref(out)),
           "qkn_decode_workspace_size")
    return int(out.value)


def workspace_init(workspace: torch.Tensor, stream=None) -> None:
    _check(_lib.qkn_workspace_init(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream(stream)), "qkn_workspace_init")


def decode_kernel_for(dims: Dims, s_q: int, kernel=KERNEL_AUTO, head_tile=0) -> int:
    return int(_lib.qkn_decode_kernel_for(ctypes.byref(dims.c()), s_q,
                                          ctypes.byref(_opts(kernel, 0, head_tile, 0))))


def decode(dims: Dims, cache: Cache, q_tilde, a_q, q_rope_hat, block_table, seq_lens, s_q: int,
           workspace: torch.Tensor, out, lse, ak_mode: int = AK_CACHE, kernel: int = KERNEL_AUTO,
           max_ctas: int = 0, head_tile: int = 0, wait_limit: int = 0, split_event=None, step_writes_only=False,
           test_withhold_ak=False, vis_end=None, stream=None) -> None:
    """One decode step over the cache (see qkn_decode).  ``split_event`` is a raw cudaEvent_t handle;
    ``step_writes_only``, ``test_withhold_ak`` and ``vis_end`` (a device int32 tensor [batch] or None)
    are the qkn_decode_opts fields of those names."""
    batch = int(block_table.shape[0])
    max_blocks = int(block_table.shape[1])
    opts = _opts(kernel, max_ctas, head_tile, wait_limit, split_event, int(bool(step_writes_only)),
                 int(bool(test_withhold_ak)), _ptr(vis_end))
    _check(_lib.qkn_decode(ctypes.byref(dims.c()), ctypes.byref(cache.c()), ak_mode, _ptr(q_tilde), _ptr(a_q),
                           _ptr(q_rope_hat), _ptr(block_table), max_blocks, _ptr(seq_lens), batch, s_q,
                           _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(out), _ptr(lse),
                           ctypes.byref(opts), _stream(stream)), "qkn_decode")


def decode_up(dims: Dims, cache: Cache, q_tilde, a_q, q_rope_hat, block_table, seq_lens, s_q: int, w_uv,
              workspace: torch.Tensor, out_v, lse, ak_mode: int = AK_CACHE, kernel: int = KERNEL_AUTO,
              max_ctas: int = 0, head_tile: int = 0, wait_limit: int = 0, split_event=None, step_writes_only=False,
              stream=None) -> None:
    """The decode step with each head's value up-projection fused into the merge (see qkn_decode_up):
    ``w_uv`` is [H, r_kv, d_v] in the storage dtype, ``out_v`` [batch, s_q, H, d_v]."""
    batch = int(block_table.shape[0])
    max_blocks = int(block_table.shape[1])
    opts = _opts(kernel, max_ctas, head_tile, wait_limit, split_event, int(bool(step_writes_only)))
    _check(_lib.qkn_decode_up(ctypes.byref(dims.c()), ctypes.byref(cache.c()), ak_mode, _ptr(q_tilde), _ptr(a_q),
                              _ptr(q_rope_hat), _ptr(block_table), max_blocks, _ptr(seq_lens), batch, s_q,
                              _ptr(w_uv), int(w_uv.shape[-1]), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _ptr(out_v), _ptr(lse),
                              ctypes.byref(opts), _stream(stream)), "qkn_decode_up")


def decode_noalloc(dims: Dims, cache: Cache, q_tilde, a_q, q_rope_hat, block_table, seq_lens, s_q: int, out, lse,
                   device_status=None, ak_mode: int = AK_CACHE, kernel: int = KERNEL_AUTO, stream=None) -> None:
    """qkn_decode_noalloc: the decode step without a workspace, for callers that cannot allocate
    device memory; its scratch is a fixed array inside the library (see include/qkn.h)."""
    batch = int(block_table.shape[0])
    max_blocks = int(block_table.shape[1])
    opts = _opts(kernel)
    _check(_lib.qkn_decode_noalloc(ctypes.byref(dims.c()), ctypes.byref(cache.c()), ak_mode, _ptr(q_tilde),
                                   _ptr(a_q), _ptr(q_rope_hat), _ptr(block_table), max_blocks, _ptr(seq_lens),
                                   batch, s_q, _ptr(out), _ptr(lse), _ptr(device_status), ctypes.byref(opts),
                                   _stream(stream)), "qkn_decode_noalloc")


def merge_partials(dims: Dims, parts, lse_parts, out, lse, stream=None) -> None:
    """Merge partial results of the same rows (see qkn_merge_partials): ``parts`` [n_parts, ..., r_kv] in the
    storage dtype, ``lse_parts`` [n_parts, ...] fp32; ``out`` / ``lse`` take the row shape."""
    n_parts = int(parts.shape[0])
    rows = int(lse_parts[0].numel())
    _check(_lib.qkn_merge_partials(ctypes.byref(dims.c()), n_parts, rows, _ptr(parts), _ptr(lse_parts), _ptr(out),
                                   _ptr(lse), _stream(stream)), "qkn_merge_partials")


def gqa_append(dims: Dims, cache: GqaCache, c_new, k_rope_raw, slot, pos, w_uk, gamma_k, w_uv, gamma_kr,
               stream=None) -> None:
    """qkn_gqa_append: expand tokens into the GQA route's cache (per-group keys and values, RoPE key)."""
    n_tok = int(c_new.shape[0])
    _check(_lib.qkn_gqa_append(ctypes.byref(dims.c()), ctypes.byref(cache.c()), _ptr(c_new), _ptr(k_rope_raw),
                               _ptr(slot), _ptr(pos), n_tok, _ptr(w_uk), _ptr(gamma_k), _ptr(w_uv), _ptr(gamma_kr),
                               _stream(stream)), "qkn_gqa_append")


def gqa_workspace_size(dims: Dims, d_v: int, batch: int, s_q: int, num_sms: int = 0) -> int:
    out = ctypes.c_size_t(0)
    _check(_lib.qkn_gqa_workspace_size(ctypes.byref(dims.c()), d_v, batch, s_q, num_sms, ctypes.byref(out)),
           "qkn_gqa_workspace_size")
    return int(out.value)


def gqa_decode(dims: Dims, cache: GqaCache, q, q_rope, gamma_q, gamma_qr, block_table, seq_lens, s_q: int,
               workspace, out_v, lse, selection=None, max_ctas: int = 0, stream=None) -> None:
    """qkn_gqa_decode: grouped-query attention over the GQA route's cache (dense), or over each query token's
    listed tokens per group (``selection`` [batch, s_q, groups, k] int32, sparse)."""
    batch = int(block_table.shape[0])
    max_blocks = int(block_table.shape[1])
    sel_k = 0 if selection is None else int(selection.shape[-1])
    _check(_lib.qkn_gqa_decode(ctypes.byref(dims.c()), ctypes.byref(cache.c()), _ptr(q), _ptr(q_rope), _ptr(gamma_q),
                               _ptr(gamma_qr), _ptr(block_table), max_blocks, _ptr(seq_lens), batch, s_q,
                               _ptr(selection), sel_k, _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _ptr(out_v), _ptr(lse), max_ctas, _stream(stream)), "qkn_gqa_decode")


def read_device_status(workspace: torch.Tensor, stream=None) -> int:
    out = ctypes.c_int32(0)
    _check(_lib.qkn_read_device_status(_ptr(workspace), _stream(stream), ctypes.byref(out)),
           "qkn_read_device_status")
    return int(out.value)


def raw_library() -> ctypes.CDLL:
    """The loaded C library (for ABI-level tests)."""
    return _lib
