"""Python binding of libmlra.so, the B200 decode path for Multi-Head Low-Rank Attention.

Argument marshalling only: every step of the decode runs in the library's CUDA kernels.
PyTorch supplies device memory and streams. The functions carry the C ABI's names
(include/mlra.h) and raise ``MlraError`` on a non-zero status.

There is no CPU fallback: importing works without a GPU (so the library's exports can be
checked), but any compute call needs the built library and a B200.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmlra.so")

MLRA_F32, MLRA_BF16 = 0, 1

STATUS = {
    0: "MLRA_OK",
    -1: "MLRA_ERR_INVALID_ARG",
    -2: "MLRA_ERR_UNSUPPORTED",
    -3: "MLRA_ERR_CUDA",
    -4: "MLRA_ERR_PAGE_OOB",
    -5: "MLRA_ERR_TIMEOUT",
    -6: "MLRA_ERR_WORKSPACE",
    -7: "MLRA_ERR_SEQ_LEN",
    -8: "MLRA_ERR_SCRATCH_LIMIT",
    -9: "MLRA_ERR_DRAIN",
}

EXPORTED = [
    "mlra_create", "mlra_destroy", "mlra_workspace_size", "mlra_decode", "mlra_decode_latent",
    "mlra_append_cache", "mlra_plan", "mlra_get_info", "mlra_get_status", "mlra_status_string",
    "mlra_decode_profiled", "mlra_decode_noalloc", "mlra_project_workspace_size", "mlra_project_append",
]


class MlraError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}")


class mlra_config(ctypes.Structure):
    _fields_ = [("h", ctypes.c_int), ("d_h", ctypes.c_int), ("d_c", ctypes.c_int),
                ("d_rope", ctypes.c_int), ("k", ctypes.c_int), ("page_size", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("blocks_summed", ctypes.c_int),
                ("attn_scale", ctypes.c_float), ("cache_fp8", ctypes.c_int),
                ("latent_scale", ctypes.c_float), ("rope_scale", ctypes.c_float)]


class mlra_info(ctypes.Structure):
    _fields_ = [("num_sms", ctypes.c_int), ("groups", ctypes.c_int),
                ("ctas_per_group", ctypes.c_int), ("heads_per_cta", ctypes.c_int),
                ("tile_tokens", ctypes.c_int), ("stages", ctypes.c_int),
                ("softmax_scale", ctypes.c_float)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libmlra.so; raises if it has not been built (no fallback exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: run `python -m rank_latent_kv_mlra_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.mlra_create.argtypes = [ctypes.POINTER(mlra_config), P, P, ctypes.POINTER(P)]
    lib.mlra_destroy.argtypes = [P]
    lib.mlra_destroy.restype = None
    lib.mlra_workspace_size.argtypes = [P, I, ctypes.POINTER(S)]
    lib.mlra_decode.argtypes = [P, P, I, P, I, P, I, P, I, P, I, P, P, S, P]
    lib.mlra_decode_noalloc.argtypes = [P, P, I, P, I, P, I, P, I, P, I, P, P, P]
    lib.mlra_decode_latent.argtypes = [P, P, I, P, I, P, I, P, I, P, P, P, S, P]
    lib.mlra_decode_profiled.argtypes = [P, P, I, P, I, P, I, P, I, P, I, P, P, S, P, P]
    lib.mlra_append_cache.argtypes = [P, P, I, P, I, I, P, P, P, P, I, I, P, P]
    lib.mlra_project_workspace_size.argtypes = [P, I, I, ctypes.POINTER(S)]
    lib.mlra_project_append.argtypes = [P, P, I, P, ctypes.c_float, P, P, I, P, I, I, P, S, P]
    lib.mlra_plan.argtypes = [P, P, I, I, P, I, P, P]
    lib.mlra_get_info.argtypes = [P, ctypes.POINTER(mlra_info)]
    lib.mlra_get_status.argtypes = [P, ctypes.POINTER(I)]
    lib.mlra_status_string.argtypes = [I]
    lib.mlra_status_string.restype = ctypes.c_char_p
    lib.mlra_test_decode_stalled.argtypes = [P, P, I, P, I, P, I, P, I, P, P, S, ctypes.c_ulonglong, I, P]
    _lib = lib
    return lib


def _check(code: int, where: str):
    if code != 0:
        raise MlraError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return MLRA_F32
    if t.dtype == torch.bfloat16:
        return MLRA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _require(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}")


class Handle:
    """Owns an mlra_handle and keeps the borrowed weight tensors alive."""

    def __init__(self, ptr: ctypes.c_void_p, cfg: mlra_config, w_uk, w_uv):
        self.ptr = ptr
        self.cfg = cfg
        self._weights = (w_uk, w_uv)

    def __del__(self):
        if self.ptr and _lib is not None:
            _lib.mlra_destroy(self.ptr)
            self.ptr = None


def mlra_create(h: int, d_h: int, d_c: int, d_rope: int, k: int, w_uk: torch.Tensor,
                w_uv: torch.Tensor, softmax_scale: float = 0.0, page_size: int = 64,
                blocks_summed: bool = False, attn_scale: float = 0.0, cache_fp8: bool = False,
                latent_scale: float = 1.0, rope_scale: float = 1.0) -> Handle:
    """blocks_summed: every head attends to every block with weights [k][h][d_c/k][d_h] and the
    per-block outputs are summed times attn_scale (<= 0: 1/sqrt(k)); lse is then [batch][k*h].
    cache_fp8: the pool holds E4M3 bytes (uint8), a latent byte e meaning latent_scale *
    e4m3(e) and a RoPE-key byte rope_scale * e4m3(e)."""
    lib = load_library()
    shape = (k, h, d_c // k, d_h) if blocks_summed else (h, d_c // k, d_h)
    for t, n in ((w_uk, "w_uk"), (w_uv, "w_uv")):
        _require(t, n, torch.bfloat16)
        if tuple(t.shape) != shape:
            raise ValueError(f"{n} must be {'[k][h]' if blocks_summed else '[h]'}[d_c/k][d_h]")
    cfg = mlra_config(h, d_h, d_c, d_rope, k, page_size, softmax_scale, int(blocks_summed), attn_scale,
                      int(cache_fp8), latent_scale, rope_scale)
    out = ctypes.c_void_p()
    _check(lib.mlra_create(ctypes.byref(cfg), _ptr(w_uk), _ptr(w_uv), ctypes.byref(out)), "mlra_create")
    return Handle(out, cfg, w_uk, w_uv)


def mlra_workspace_size(handle: Handle, batch: int) -> int:
    n = ctypes.c_size_t()
    _check(load_library().mlra_workspace_size(handle.ptr, batch, ctypes.byref(n)), "mlra_workspace_size")
    return n.value


def alloc_workspace(handle: Handle, batch: int, device=None) -> torch.Tensor:
    """Workspace for `batch` sequences (a uint8 CUDA tensor; torch allocations are 256-aligned)."""
    return torch.empty(mlra_workspace_size(handle, batch), dtype=torch.uint8, device=device or "cuda")


def mlra_get_info(handle: Handle) -> dict:
    info = mlra_info()
    _check(load_library().mlra_get_info(handle.ptr, ctypes.byref(info)), "mlra_get_info")
    return {f: getattr(info, f) for f, _ in mlra_info._fields_}


def _pool_dtype(handle):
    return torch.uint8 if handle.cfg.cache_fp8 else torch.bfloat16


def _decode_common(handle, q, pool, page_table, seq_lens, workspace):
    _require(q, "q")
    _require(pool, "pool", _pool_dtype(handle))
    _require(page_table, "page_table", torch.int32)
    _require(seq_lens, "seq_lens", torch.int32)
    _require(workspace, "workspace")
    cfg = handle.cfg
    B = q.shape[0]
    if tuple(q.shape) != (B, cfg.h, cfg.d_h + cfg.d_rope):
        raise ValueError("q must be [batch][h][d_h + d_rope]")
    if pool.dim() != 3 or pool.shape[1] != cfg.page_size or pool.shape[2] != cfg.d_c + cfg.d_rope:
        raise ValueError("pool must be [num_pages][page_size][d_c + d_rope]")
    if page_table.dim() != 2 or page_table.shape[0] != B or seq_lens.shape != (B,):
        raise ValueError("page_table must be [batch][pt_stride], seq_lens [batch]")
    return B


def mlra_decode(handle: Handle, q, pool, page_table, seq_lens, out, lse=None, workspace=None,
                stream=None):
    """One decode step; `out` [batch][h][d_h] (fp32 or bf16), `lse` fp32 [batch][h] or None."""
    if workspace is None:
        workspace = alloc_workspace(handle, q.shape[0], q.device)
    B = _decode_common(handle, q, pool, page_table, seq_lens, workspace)
    _require(out, "out")
    if lse is not None:
        _require(lse, "lse", torch.float32)
    _check(load_library().mlra_decode(
        handle.ptr, _ptr(q), _dtype(q), _ptr(pool), pool.shape[0], _ptr(page_table),
        page_table.shape[1], _ptr(seq_lens), B, _ptr(out), _dtype(out), _ptr(lse), _ptr(workspace),
        workspace.numel(), _stream(stream)), "mlra_decode")
    return workspace


def mlra_decode_noalloc(handle: Handle, q, pool, page_table, seq_lens, out, lse=None, status=None,
                        stream=None):
    """mlra_decode without a workspace: the scratch is the library's fixed 16 MiB device array,
    shared by every call on the device, so calls must not overlap on the GPU. For callers that
    cannot allocate device memory while decoding. `status` is an optional device int32 tensor
    that receives the call's device status. Raises MlraError(MLRA_ERR_SCRATCH_LIMIT) for a
    batch the array cannot hold."""
    _require(q, "q")
    _require(pool, "pool", _pool_dtype(handle))
    _require(page_table, "page_table", torch.int32)
    _require(seq_lens, "seq_lens", torch.int32)
    _require(out, "out")
    if lse is not None:
        _require(lse, "lse", torch.float32)
    if status is not None:
        _require(status, "status", torch.int32)
    cfg = handle.cfg
    B = q.shape[0]
    if tuple(q.shape) != (B, cfg.h, cfg.d_h + cfg.d_rope):
        raise ValueError("q must be [batch][h][d_h + d_rope]")
    if pool.dim() != 3 or pool.shape[1] != cfg.page_size or pool.shape[2] != cfg.d_c + cfg.d_rope:
        raise ValueError("pool must be [num_pages][page_size][d_c + d_rope]")
    if page_table.dim() != 2 or page_table.shape[0] != B or seq_lens.shape != (B,):
        raise ValueError("page_table must be [batch][pt_stride], seq_lens [batch]")
    _check(load_library().mlra_decode_noalloc(
        handle.ptr, _ptr(q), _dtype(q), _ptr(pool), pool.shape[0], _ptr(page_table),
        page_table.shape[1], _ptr(seq_lens), B, _ptr(out), _dtype(out), _ptr(lse), _ptr(status),
        _stream(stream)), "mlra_decode_noalloc")


def mlra_decode_profiled(handle: Handle, q, pool, page_table, seq_lens, out, events, lse=None,
                         workspace=None, stream=None):
    """mlra_decode that records four torch.cuda.Event objects around its three kernels."""
    if workspace is None:
        workspace = alloc_workspace(handle, q.shape[0], q.device)
    B = _decode_common(handle, q, pool, page_table, seq_lens, workspace)
    for e in events:
        if e.cuda_event == 0:  # torch creates the CUDA event on its first record
            e.record(stream or torch.cuda.current_stream())
    ev = (ctypes.c_void_p * 4)(*[e.cuda_event for e in events])
    _check(load_library().mlra_decode_profiled(
        handle.ptr, _ptr(q), _dtype(q), _ptr(pool), pool.shape[0], _ptr(page_table),
        page_table.shape[1], _ptr(seq_lens), B, _ptr(out), _dtype(out), _ptr(lse), _ptr(workspace),
        workspace.numel(), ev, _stream(stream)), "mlra_decode_profiled")
    return workspace


def mlra_decode_latent(handle: Handle, q, pool, page_table, seq_lens, latent_out, lse=None,
                       workspace=None, stream=None):
    """Decode without the up-projection: `latent_out` fp32 [batch][h][d_c/k]."""
    if workspace is None:
        workspace = alloc_workspace(handle, q.shape[0], q.device)
    B = _decode_common(handle, q, pool, page_table, seq_lens, workspace)
    _require(latent_out, "latent_out", torch.float32)
    if lse is not None:
        _require(lse, "lse", torch.float32)
    _check(load_library().mlra_decode_latent(
        handle.ptr, _ptr(q), _dtype(q), _ptr(pool), pool.shape[0], _ptr(page_table),
        page_table.shape[1], _ptr(seq_lens), B, _ptr(latent_out), _ptr(lse), _ptr(workspace),
        workspace.numel(), _stream(stream)), "mlra_decode_latent")
    return workspace


def mlra_append_cache(handle: Handle, pool, page_table, seq_ids, positions, c_new, kr_new,
                      status=None, stream=None):
    _require(pool, "pool", _pool_dtype(handle))
    for t, n in ((page_table, "page_table"), (seq_ids, "seq_ids"), (positions, "positions")):
        _require(t, n, torch.int32)
    _require(c_new, "c_new")
    _require(kr_new, "kr_new")
    if c_new.dtype != kr_new.dtype:
        raise TypeError("c_new and kr_new must share a dtype")
    _check(load_library().mlra_append_cache(
        handle.ptr, _ptr(pool), pool.shape[0], _ptr(page_table), page_table.shape[1],
        page_table.shape[0], _ptr(seq_ids), _ptr(positions), _ptr(c_new), _ptr(kr_new),
        _dtype(c_new), seq_ids.numel(), _ptr(status), _stream(stream)), "mlra_append_cache")


def mlra_project_workspace_size(handle: Handle, batch: int, d_model: int) -> int:
    n = ctypes.c_size_t()
    _check(load_library().mlra_project_workspace_size(handle.ptr, batch, d_model, ctypes.byref(n)),
           "mlra_project_workspace_size")
    return n.value


def mlra_project_append(handle: Handle, x, w_down, positions, pool, page_table, rope_base=10000.0,
                        workspace=None, stream=None):
    """The new token's cache row [x W^DKV | RoPE(x W^KR)] of each sequence, stored at its
    position. x bf16 [batch][d_model]; w_down bf16 [d_c + d_rope][d_model]; positions int32
    [batch]. Returns the workspace, whose first int32 is the call's status word."""
    _require(x, "x", torch.bfloat16)
    _require(w_down, "w_down", torch.bfloat16)
    _require(positions, "positions", torch.int32)
    _require(pool, "pool", _pool_dtype(handle))
    _require(page_table, "page_table", torch.int32)
    cfg = handle.cfg
    B, d_model = x.shape
    if tuple(w_down.shape) != (cfg.d_c + cfg.d_rope, d_model):
        raise ValueError("w_down must be [d_c + d_rope][d_model]")
    if positions.shape != (B,) or page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("positions must be [batch], page_table [batch][pt_stride]")
    if workspace is None:
        workspace = torch.empty(mlra_project_workspace_size(handle, B, d_model), dtype=torch.uint8,
                                device=x.device)
    _require(workspace, "workspace")
    _check(load_library().mlra_project_append(
        handle.ptr, _ptr(x), d_model, _ptr(w_down), float(rope_base), _ptr(positions), _ptr(pool),
        pool.shape[0], _ptr(page_table), page_table.shape[1], B, _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)), "mlra_project_append")
    return workspace


def mlra_plan(handle: Handle, seq_lens, pt_stride: int, max_segments: int = 4096, stream=None):
    """Device split plan as a list of (b, group, tile_begin, tile_end, slot) tuples."""
    _require(seq_lens, "seq_lens", torch.int32)
    segs = torch.zeros((max_segments, 5), dtype=torch.int32, device=seq_lens.device)
    count = torch.zeros(1, dtype=torch.int32, device=seq_lens.device)
    _check(load_library().mlra_plan(handle.ptr, _ptr(seq_lens), seq_lens.numel(), pt_stride,
                                    _ptr(segs), max_segments, _ptr(count), _stream(stream)),
           "mlra_plan")
    n = int(count.item())
    return [tuple(r) for r in segs[:min(n, max_segments)].tolist()], n


def mlra_get_status(status_word: torch.Tensor) -> int:
    """Device status word (first int32 of a decode workspace, or an append status tensor)."""
    v = ctypes.c_int()
    _check(load_library().mlra_get_status(_ptr(status_word), ctypes.byref(v)), "mlra_get_status")
    return v.value


def mlra_status_string(code: int) -> str:
    return load_library().mlra_status_string(code).decode()


def mlra_test_decode_stalled(handle: Handle, q, pool, page_table, seq_lens, out, workspace,
                             wait_limit_ns: int, where: int = 1, stream=None):
    """Test hook: a decode with one wait made to run out (where = 1: the decode kernel's
    producer withholds its first tile; 2: one absorb CTA never issues its MMA)."""
    B = _decode_common(handle, q, pool, page_table, seq_lens, workspace)
    _check(load_library().mlra_test_decode_stalled(
        handle.ptr, _ptr(q), _dtype(q), _ptr(pool), pool.shape[0], _ptr(page_table),
        page_table.shape[1], _ptr(seq_lens), B, _ptr(out), _ptr(workspace), workspace.numel(),
        wait_limit_ns, where, _stream(stream)), "mlra_test_decode_stalled")
