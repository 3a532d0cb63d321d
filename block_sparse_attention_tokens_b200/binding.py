"""Thin Python binding of libbsa.so (argument marshalling only).

Every function here has the name of the C entry point it wraps (see
``include/bsa.h``), takes torch tensors where the C ABI takes device pointers,
passes the current torch CUDA stream, and raises ``BsaError`` on a non-OK
status.  All arithmetic happens in the library's CUDA kernels; when the shared
library is missing the import fails loudly -- there is no other code path.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbsa.so")

STATUS = {0: "BSA_OK", 1: "BSA_ERR_INVALID_ARG", 2: "BSA_ERR_UNSUPPORTED", 3: "BSA_ERR_WORKSPACE",
          4: "BSA_ERR_CUDA", 5: "BSA_ERR_TIMEOUT"}

EXPORTS = [
    "bsa_status_string", "bsa_last_error_message", "bsa_version", "bsa_tile_permute",
    "bsa_tile_untile", "bsa_sta_mask", "bsa_radial_mask", "bsa_nabla_workspace_size",
    "bsa_nabla_mask", "bsa_mask_compact", "bsa_attn_workspace_size", "bsa_attn_fwd",
    "bsa_attn_fwd_noalloc", "bsa_read_status", "bsa_tile_permute_pool", "bsa_nabla_select",
    "bsa_wait_selftest", "bsa_attn_bwd_workspace_size", "bsa_attn_bwd", "bsa_sics_blocks",
    "bsa_sics_workspace_size", "bsa_sics_scheme", "bsa_kv_write", "bsa_block_pool",
    "bsa_kv_resident_blocks", "bsa_kv_page_scores", "bsa_kv_keep_pages", "bsa_attn_fwd_paged",
    "bsa_scheme_permute", "bsa_scheme_untile",
]


class BsaError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str = ""):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)}" + (f" ({detail})" if detail else ""))


_lib = None


def load_library(path: str = _LIB_PATH) -> ctypes.CDLL:
    """Loads libbsa.so once.  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libbsa.so not found at {path}; build it with "
                          f"`python -m block_sparse_attention_tokens_b200.build`")
    lib = ctypes.CDLL(path)
    c_int, c_void, c_size, c_float = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float
    sig = {
        "bsa_status_string": (ctypes.c_char_p, [c_int]),
        "bsa_last_error_message": (ctypes.c_char_p, []),
        "bsa_version": (c_int, []),
        "bsa_tile_permute": (c_int, [c_void, c_void] + [c_int] * 11 + [c_void]),
        "bsa_tile_untile": (c_int, [c_void, c_void] + [c_int] * 11 + [c_void]),
        "bsa_sta_mask": (c_int, [c_int] * 7 + [c_void, c_void]),
        "bsa_radial_mask": (c_int, [c_int] * 3 + [c_void, c_void]),
        "bsa_nabla_workspace_size": (c_size, [c_int] * 6),
        "bsa_nabla_mask": (c_int, [c_void, c_void] + [c_int] * 7 + [c_float, c_float] + [c_int] * 3
                           + [c_void, c_void, c_void, c_size, c_void]),
        "bsa_mask_compact": (c_int, [c_void, c_int, c_int, c_void, c_void, c_void]),
        "bsa_attn_workspace_size": (c_size, [c_int] * 7),
        "bsa_attn_fwd": (c_int, [c_void, c_void, c_void] + [c_int] * 9 + [c_void, c_void, c_int,
                                                                           c_float, c_void, c_void,
                                                                           c_void, c_size, c_void]),
        "bsa_attn_fwd_noalloc": (c_int, [c_void, c_void, c_void] + [c_int] * 7
                                 + [c_void, c_void, c_int, c_float, c_void, c_void, c_void,
                                    c_void]),
        "bsa_attn_bwd_workspace_size": (c_size, [c_int] * 7),
        "bsa_attn_bwd": (c_int, [c_void] * 6 + [c_int] * 9 + [c_void, c_void, c_int, c_float]
                         + [c_void] * 4 + [c_size, c_void]),
        "bsa_sics_blocks": (c_int, [c_void] + [c_int] * 10 + [c_void, c_void]),
        "bsa_sics_workspace_size": (c_size, [c_int] * 5 + [c_void, c_int]),
        "bsa_sics_scheme": (c_int, [c_void, c_void] + [c_int] * 7 + [c_void, c_int]
                            + [c_void] * 3 + [c_size, c_void]),
        "bsa_read_status": (c_int, [c_void, ctypes.POINTER(c_int), c_void]),
        "bsa_wait_selftest": (c_int, [c_void, ctypes.c_ulonglong, c_void]),
        "bsa_tile_permute_pool": (c_int, [c_void, c_void] + [c_int] * 11 + [c_void, c_int, c_int,
                                                                             c_void]),
        "bsa_scheme_permute": (c_int, [c_void, c_void] + [c_int] * 4 + [c_void, c_int, c_void]
                               + [c_int] * 4 + [c_void, c_int, c_int, c_void, c_void]),
        "bsa_scheme_untile": (c_int, [c_void, c_void] + [c_int] * 4 + [c_void, c_int, c_void]
                              + [c_int] * 5 + [c_void, c_void]),
        "bsa_nabla_select": (c_int, [c_void, c_void] + [c_int] * 5 + [c_float, c_float]
                             + [c_int] * 3 + [c_void] * 5),
        "bsa_kv_write": (c_int, [c_void] + [c_int] * 5 + [c_void, c_int, c_void, c_int, c_void,
                                                           c_void]),
        "bsa_block_pool": (c_int, [c_void, c_void] + [c_int] * 8 + [c_void, c_int, c_void]),
        "bsa_kv_resident_blocks": (c_int, [c_void] + [c_int] * 4 + [c_void, c_void]),
        "bsa_kv_page_scores": (c_int, [c_void, c_void] + [c_int] * 5 + [c_float, c_int, c_int]
                               + [c_void, c_int, c_int, c_void, c_void]),
        "bsa_kv_keep_pages": (c_int, [c_void] + [c_int] * 5 + [c_void, c_int] + [c_void] * 3),
        "bsa_attn_fwd_paged": (c_int, [c_void] * 3 + [c_int, c_void] + [c_int] * 8
                               + [c_void, c_void, c_int, c_float] + [c_void] * 3
                               + [c_size, c_void]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check(code: int, where: str):
    if code != 0:
        detail = load_library().bsa_last_error_message().decode() if code in (3, 4) else ""
        raise BsaError(code, where, detail)


def _cuda(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _token_problem(shape, dtype, batch: int, n: int, heads: int, head_dim: int):
    """Why a tensor of this shape and dtype cannot serve as n token rows of the C ABI's
    [batch, n, heads, head_dim] bf16 layout (None if it can).  The library derives
    the batch stride from n, so with batch > 1 the tensor must hold exactly n rows;
    with batch == 1 extra rows (e.g. a zero-padded tail) are allowed and ignored."""
    if dtype != torch.bfloat16:
        return f"must be bfloat16, got {dtype}"
    if len(shape) != 4 or shape[0] != batch or tuple(shape[2:]) != (heads, head_dim):
        return f"must be [{batch}, n, {heads}, {head_dim}], got {tuple(shape)}"
    if shape[1] < n:
        return f"has {shape[1]} rows for {n} tokens"
    if batch > 1 and shape[1] != n:
        return f"has {shape[1]} rows per batch for {n} tokens (batch > 1 needs exactly {n})"
    return None


def _tokens(t: torch.Tensor, name: str, batch: int, n: int, heads: int, head_dim: int):
    _cuda(t, name)
    problem = _token_problem(tuple(t.shape), t.dtype, batch, n, heads, head_dim)
    if problem:
        raise ValueError(f"{name} {problem}")


def _stride_problem(shape, strides, n: int, dense_row: int, align_elems: int):
    """Why token rows of this shape and strides (elements) cannot be described by
    one row stride: every row contiguous, rows row_stride = strides[1] apart (at
    least a whole row, a multiple of align_elems), batches n rows apart (None if
    they can)."""
    inner = 1
    for size, st in zip(reversed(shape[2:]), reversed(strides[2:])):
        if size > 1 and st != inner:
            return "rows must be contiguous (only the token-row stride may differ)"
        inner *= size
    rs = strides[1] if shape[1] > 1 else dense_row
    if rs < dense_row or rs % align_elems:
        return f"row stride {rs} must be >= {dense_row} and a multiple of {align_elems}"
    if shape[0] > 1 and strides[0] != n * rs:
        return f"batch stride {strides[0]} must be {n} rows of {rs}"
    return None


def _strided_tokens(t: torch.Tensor, name: str, batch: int, n: int, heads: int,
                    head_dim: int) -> int:
    """Checks a [batch, >= n, heads, head_dim] bf16 CUDA tensor whose token rows may
    be a slice of wider rows (a range of heads, or Q / K / V of a fused projection)
    and returns its row stride in elements."""
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    problem = _token_problem(tuple(t.shape), t.dtype, batch, n, heads, head_dim)
    if problem and "rows per batch" not in problem:
        raise ValueError(f"{name} {problem}")
    problem = _stride_problem(tuple(t.shape), tuple(t.stride()), n, heads * head_dim, 8)
    if problem:
        raise ValueError(f"{name}: {problem}")
    if t.data_ptr() % 16:
        raise ValueError(f"{name} must start on a 16-byte boundary")
    return t.stride(1) if t.shape[1] > 1 else heads * head_dim


def _shared_stride(pairs) -> int:
    """The one row stride of several token tensors [(tensor, name, stride)]."""
    strides = {st for _, _, st in pairs}
    if len(strides) != 1:
        raise ValueError(", ".join(n for _, n, _ in pairs) + " must share one token-row stride, got "
                         + str(sorted(strides)))
    return strides.pop()


def _buffer(t: torch.Tensor, name: str, dtype, numel: int):
    _cuda(t, name)
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements, {numel} needed")


def _lists(row_ptr: torch.Tensor, col_idx: torch.Tensor, list_heads: int, nq: int, block_q: int,
           nk: int, block_k: int):
    """Kept lists: row_ptr has one entry per (list head, query block) plus one;
    col_idx has room for every (list head, query block, key block), the worst case
    bsa_mask_compact writes, because the library trusts row_ptr up to that bound
    (checking the actual count would need a device synchronisation)."""
    QB, KB = -(-nq // block_q), -(-nk // block_k)
    _buffer(row_ptr, "row_ptr", torch.int32, list_heads * QB + 1)
    _buffer(col_idx, "col_idx", torch.int32, list_heads * QB * KB)


def _means(t: torch.Tensor, name: str, batch: int, heads: int, head_dim: int):
    """Pooled block means [batch, heads, blocks, head_dim] float32."""
    _cuda(t, name)
    if t.dtype != torch.float32 or t.dim() != 4 or tuple(t.shape[:2]) != (batch, heads) \
            or t.shape[3] != head_dim:
        raise ValueError(f"{name} must be float32 [{batch}, {heads}, blocks, {head_dim}], "
                         f"got {t.dtype} {tuple(t.shape)}")


def _pool(t: torch.Tensor, name: str, heads: int, head_dim: int):
    """A paged K or V pool [pages, KV_PAGE, heads, head_dim] bf16."""
    _cuda(t, name)
    if t.dtype != torch.bfloat16 or t.dim() != 4 or tuple(t.shape[1:]) != (KV_PAGE, heads, head_dim):
        raise ValueError(f"{name} must be bfloat16 [pages, {KV_PAGE}, {heads}, {head_dim}], "
                         f"got {t.dtype} {tuple(t.shape)}")


def _table(t: torch.Tensor, name: str, batch: int, pages: int = 0):
    """A page table [>= batch, >= pages] int32 (physical page or -1)."""
    _cuda(t, name)
    if t.dtype != torch.int32 or t.dim() != 2 or t.shape[0] < batch or t.shape[1] < pages:
        raise ValueError(f"{name} must be int32 [{batch}, >= {pages} pages], "
                         f"got {t.dtype} {tuple(t.shape)}")


def _nbytes(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


def _row_problem(shape, elem_bytes: int, batch: int, n: int, row_bytes: int):
    """Why a tensor cannot serve as n rows of row_bytes each per batch ([batch, n, ...]
    with the batch stride n rows; extra rows allowed only for one batch)."""
    if len(shape) < 2 or shape[0] != batch:
        return f"must be [{batch}, rows, ...], got {tuple(shape)}"
    if math.prod(shape[2:]) * elem_bytes != row_bytes:
        return f"rows of {math.prod(shape[2:]) * elem_bytes} bytes, {row_bytes} expected"
    if shape[1] < n:
        return f"has {shape[1]} rows for {n}"
    if batch > 1 and shape[1] != n:
        return f"has {shape[1]} rows per batch for {n} (batch > 1 needs exactly {n})"
    return None


def _rows(t: torch.Tensor, name: str, batch: int, n: int, row_bytes: int):
    _cuda(t, name)
    problem = _row_problem(tuple(t.shape), t.element_size(), batch, n, row_bytes)
    if problem:
        raise ValueError(f"{name} {problem}")


def _strided_rows(t: torch.Tensor, name: str, batch: int, n: int) -> Tuple[int, int]:
    """A [batch, >= n, ...] CUDA tensor whose rows (the trailing dims) are contiguous
    but may lie further apart than their size: returns (row bytes, row stride in
    bytes)."""
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    es = t.element_size()
    row_bytes = math.prod(t.shape[2:]) * es
    if t.dim() < 2 or t.shape[0] != batch or t.shape[1] < n:
        raise ValueError(f"{name} must be [{batch}, >= {n}, ...], got {tuple(t.shape)}")
    problem = _stride_problem(tuple(t.shape), tuple(t.stride()), n, row_bytes // es,
                              max(1, 16 // es))
    if problem:
        raise ValueError(f"{name}: {problem}")
    if t.data_ptr() % 16:
        raise ValueError(f"{name} must start on a 16-byte boundary")
    return row_bytes, (t.stride(1) if t.shape[1] > 1 else row_bytes // es) * es


def _bytes(t: torch.Tensor, name: str, numel: int):
    """A byte mask / flag buffer (uint8 or bool) of at least numel entries."""
    _cuda(t, name)
    if t.dtype not in (torch.uint8, torch.bool):
        raise ValueError(f"{name} must be uint8 (or bool), got {t.dtype}")
    if t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} entries, {numel} needed")


# --------------------------------------------------------------------------- (a)

def bsa_tile_permute(x: torch.Tensor, grid: Tuple[int, int, int], tile: Tuple[int, int, int],
                     n_pad: int, y: Optional[torch.Tensor] = None) -> torch.Tensor:
    """x [B, N, ...] raster order -> y [B, n_pad, ...] tile order with a zero tail.
    x and y may be slices of wider rows (e.g. x[:, :, h0:h1] of a [B, N, H, D]
    tensor): only the row stride may differ from a dense layout."""
    B = x.shape[0]
    N = grid[0] * grid[1] * grid[2]
    row_bytes, xs = _strided_rows(x, "x", B, N)
    if y is None:
        y = torch.empty((B, n_pad) + tuple(x.shape[2:]), dtype=x.dtype, device=x.device)
    y_bytes, ys = _strided_rows(y, "y", B, n_pad)
    if y_bytes != row_bytes:
        raise ValueError(f"y rows of {y_bytes} bytes, {row_bytes} expected")
    _check(load_library().bsa_tile_permute(_ptr(x), _ptr(y), B, *grid, *tile, row_bytes, n_pad,
                                           xs, ys, _stream()), "bsa_tile_permute")
    return y


def bsa_tile_untile(y: torch.Tensor, grid: Tuple[int, int, int], tile: Tuple[int, int, int],
                    x: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y [B, n_pad, ...] tile order -> x [B, N, ...] raster order (either may be a
    slice of wider rows)."""
    B, n_pad = y.shape[0], y.shape[1]
    N = grid[0] * grid[1] * grid[2]
    row_bytes, ys = _strided_rows(y, "y", B, n_pad)
    if x is None:
        x = torch.empty((B, N) + tuple(y.shape[2:]), dtype=y.dtype, device=y.device)
    x_bytes, xs = _strided_rows(x, "x", B, N)
    if x_bytes != row_bytes:
        raise ValueError(f"x rows of {x_bytes} bytes, {row_bytes} expected")
    _check(load_library().bsa_tile_untile(_ptr(y), _ptr(x), B, *grid, *tile, row_bytes, n_pad,
                                          ys, xs, _stream()), "bsa_tile_untile")
    return x


def bsa_tile_permute_pool(x: torch.Tensor, grid: Tuple[int, int, int],
                          tile: Tuple[int, int, int], n_pad: int, block: int,
                          y: Optional[torch.Tensor] = None,
                          pooled: Optional[torch.Tensor] = None):
    """x [B, N, H, D] bf16 raster -> (y [B, n_pad, H, D] tile order,
    pooled [B, H, n_pad / block, D] fp32 block means).  x and y may be head
    slices of wider tensors."""
    B, _, H, D = x.shape
    xs = _strided_tokens(x, "x", B, grid[0] * grid[1] * grid[2], H, D)
    if y is None:
        y = torch.empty((B, n_pad, H, D), dtype=x.dtype, device=x.device)
    ys = _strided_tokens(y, "y", B, n_pad, H, D)
    if pooled is None:
        pooled = torch.empty((B, H, n_pad // block, D), dtype=torch.float32, device=x.device)
    _buffer(pooled, "pooled", torch.float32, B * H * (n_pad // max(block, 1)) * D)
    _check(load_library().bsa_tile_permute_pool(_ptr(x), _ptr(y), B, *grid, *tile, H, D, n_pad,
                                                block, _ptr(pooled), xs, ys, _stream()),
           "bsa_tile_permute_pool")
    return y, pooled


def _status(device_status: Optional[torch.Tensor]):
    """The optional one-word error status a kernel writes on the device."""
    if device_status is not None:
        _buffer(device_status, "device_status", torch.int32, 1)


def _choice(choice: torch.Tensor, batch: int, heads: int):
    _cuda(choice, "choice")
    if choice.dtype != torch.int32 or choice.numel() != batch * heads or not choice.is_contiguous():
        raise ValueError(f"choice: expected contiguous int32 [{batch}, {heads}], got "
                         f"{choice.dtype} {tuple(choice.shape)}")


def bsa_scheme_permute(x: torch.Tensor, grid: Tuple[int, int, int], shapes, choice: torch.Tensor,
                       n_pad: int, block: int = 0, y: Optional[torch.Tensor] = None,
                       pooled: Optional[torch.Tensor] = None, pool: bool = False,
                       device_status: Optional[torch.Tensor] = None):
    """Tile permute with the slice shape shapes[choice[b, h]] per (batch, head).
    x [B, N, H, D] bf16 raster -> y [B, n_pad, H, D] (per-head tile order, zero
    tail); with ``pool`` (or a ``pooled`` buffer) also the per-block means
    [B, H, n_pad / block, D] fp32.  x and y may be head slices of wider tensors.
    Returns (y, pooled or None)."""
    _status(device_status)
    B, _, H, D = x.shape
    xs = _strided_tokens(x, "x", B, grid[0] * grid[1] * grid[2], H, D)
    _choice(choice, B, H)
    if y is None:
        y = torch.empty((B, n_pad, H, D), dtype=x.dtype, device=x.device)
    ys = _strided_tokens(y, "y", B, n_pad, H, D)
    if pooled is None and pool:
        pooled = torch.empty((B, H, n_pad // max(block, 1), D), dtype=torch.float32,
                             device=x.device)
    if pooled is not None:
        _buffer(pooled, "pooled", torch.float32, B * H * (n_pad // max(block, 1)) * D)
    arr, n = _shape_array(shapes)
    _check(load_library().bsa_scheme_permute(_ptr(x), _ptr(y), B, *grid, arr, n, _ptr(choice),
                                             H, D, n_pad, block, _ptr(pooled), xs, ys,
                                             _ptr(device_status), _stream()),
           "bsa_scheme_permute")
    return y, pooled


def bsa_scheme_untile(y: torch.Tensor, grid: Tuple[int, int, int], shapes, choice: torch.Tensor,
                      x: Optional[torch.Tensor] = None,
                      device_status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Inverse of bsa_scheme_permute: y [B, n_pad, H, D] -> x [B, N, H, D] raster (either
    may be a head slice of a wider tensor)."""
    _status(device_status)
    B, n_pad, H, D = y.shape
    N = grid[0] * grid[1] * grid[2]
    ys = _strided_tokens(y, "y", B, n_pad, H, D)
    _choice(choice, B, H)
    if x is None:
        x = torch.empty((B, N, H, D), dtype=y.dtype, device=y.device)
    xs = _strided_tokens(x, "x", B, N, H, D)
    arr, n = _shape_array(shapes)
    _check(load_library().bsa_scheme_untile(_ptr(y), _ptr(x), B, *grid, arr, n, _ptr(choice), H,
                                            D, n_pad, ys, xs, _ptr(device_status), _stream()),
           "bsa_scheme_untile")
    return x


# --------------------------------------------------------------------------- (b)

def bsa_sta_mask(tile_grid: Tuple[int, int, int], window: Tuple[int, int, int], shift: int = 0,
                 mask: Optional[torch.Tensor] = None, device="cuda") -> torch.Tensor:
    n = tile_grid[0] * tile_grid[1] * tile_grid[2]
    if mask is None:
        mask = torch.empty((n, n), dtype=torch.uint8, device=device)
    _bytes(mask, "mask", n * n)
    _check(load_library().bsa_sta_mask(*tile_grid, *window, int(shift), _ptr(mask), _stream()),
           "bsa_sta_mask")
    return mask


def bsa_radial_mask(n_tokens: int, tokens_per_frame: int, block: int,
                    mask: Optional[torch.Tensor] = None, device="cuda") -> torch.Tensor:
    nb = -(-n_tokens // block)
    if mask is None:
        mask = torch.empty((nb, nb), dtype=torch.uint8, device=device)
    _bytes(mask, "mask", nb * nb)
    _check(load_library().bsa_radial_mask(n_tokens, tokens_per_frame, block, _ptr(mask),
                                          _stream()), "bsa_radial_mask")
    return mask


def bsa_nabla_workspace_size(batch, heads, nq, nk, head_dim, block) -> int:
    return int(load_library().bsa_nabla_workspace_size(batch, heads, nq, nk, head_dim, block))


def bsa_nabla_mask(q: torch.Tensor, k: torch.Tensor, block: int, p: float, scale: float = 0.0,
                   kb_begin: int = 0, kb_end: Optional[int] = None, force_outside: int = 0,
                   nq: Optional[int] = None, nk: Optional[int] = None,
                   mask: Optional[torch.Tensor] = None, near_count: Optional[torch.Tensor] = None,
                   ws: Optional[torch.Tensor] = None):
    """NABLA block mask [B, H, QB, KB] (uint8) from q, k [B, N, H, D] (bf16).

    nq / nk: number of valid tokens (default: the tensors' lengths).
    Returns (mask, near_count tensor).
    """
    B, _, H, D = q.shape
    nq = q.shape[1] if nq is None else nq
    nk = k.shape[1] if nk is None else nk
    rs = _shared_stride([(q, "q", _strided_tokens(q, "q", B, nq, H, D)),
                         (k, "k", _strided_tokens(k, "k", B, nk, H, D))])
    QB, KB = -(-nq // block), -(-nk // block)
    kb_end = KB if kb_end is None else kb_end
    if mask is None:
        mask = torch.empty((B, H, QB, KB), dtype=torch.uint8, device=q.device)
    _buffer(mask, "mask", torch.uint8, B * H * QB * KB)
    if near_count is None:
        near_count = torch.zeros(1, dtype=torch.int32, device=q.device)
    _buffer(near_count, "near_count", torch.int32, 1)
    if ws is None:
        ws = torch.empty(bsa_nabla_workspace_size(B, H, nq, nk, D, block), dtype=torch.uint8,
                         device=q.device)
    _cuda(ws, "ws")
    _check(load_library().bsa_nabla_mask(_ptr(q), _ptr(k), B, H, nq, nk, D, rs, block, float(p),
                                         float(scale), kb_begin, kb_end, int(force_outside),
                                         _ptr(mask), _ptr(near_count), _ptr(ws), _nbytes(ws),
                                         _stream()), "bsa_nabla_mask")
    return mask, near_count


def bsa_nabla_select(qbar: torch.Tensor, kbar: torch.Tensor, p: float, scale: float = 0.0,
                     kb_begin: int = 0, kb_end: Optional[int] = None, force_outside: int = 0,
                     base_mask: Optional[torch.Tensor] = None,
                     mask: Optional[torch.Tensor] = None,
                     near_count: Optional[torch.Tensor] = None,
                     key_allowed: Optional[torch.Tensor] = None):
    """NABLA selection from pooled means qbar [B, H, QB, D], kbar [B, H, KB, D] (fp32),
    optionally OR-ed with a head-shared base mask [QB, KB] and restricted to the key
    blocks with key_allowed [B, KB] != 0.  Returns (mask, near_count)."""
    _cuda(qbar, "qbar")
    _cuda(kbar, "kbar")
    B, H, QB, D = qbar.shape
    KB = kbar.shape[2]
    _means(qbar, "qbar", B, H, D)
    _means(kbar, "kbar", B, H, D)
    kb_end = KB if kb_end is None else kb_end
    if mask is None:
        mask = torch.empty((B, H, QB, KB), dtype=torch.uint8, device=qbar.device)
    _bytes(mask, "mask", B * H * QB * KB)
    if base_mask is not None:
        _bytes(base_mask, "base_mask", QB * KB)
    if key_allowed is not None:
        _bytes(key_allowed, "key_allowed", B * KB)
    if near_count is None:
        near_count = torch.zeros(1, dtype=torch.int32, device=qbar.device)
    _buffer(near_count, "near_count", torch.int32, 1)
    _check(load_library().bsa_nabla_select(_ptr(qbar), _ptr(kbar), B, H, QB, KB, D, float(p),
                                           float(scale), kb_begin, kb_end, int(force_outside),
                                           _ptr(base_mask), _ptr(key_allowed), _ptr(mask),
                                           _ptr(near_count), _stream()), "bsa_nabla_select")
    return mask, near_count


# --------------------------------------------------------------------------- (c)

def bsa_mask_compact(mask: torch.Tensor, row_ptr: Optional[torch.Tensor] = None,
                     col_idx: Optional[torch.Tensor] = None):
    """uint8 mask [..., KB] (rows = product of leading dims) -> (row_ptr, col_idx) int32."""
    _cuda(mask, "mask")
    KB = mask.shape[-1]
    rows = mask.numel() // KB
    _bytes(mask, "mask", rows * KB)
    if row_ptr is None:
        row_ptr = torch.empty(rows + 1, dtype=torch.int32, device=mask.device)
    if col_idx is None:
        col_idx = torch.empty(rows * KB, dtype=torch.int32, device=mask.device)
    _buffer(row_ptr, "row_ptr", torch.int32, rows + 1)
    _buffer(col_idx, "col_idx", torch.int32, rows * KB)
    _check(load_library().bsa_mask_compact(_ptr(mask), rows, KB, _ptr(row_ptr), _ptr(col_idx),
                                           _stream()), "bsa_mask_compact")
    return row_ptr, col_idx


# --------------------------------------------------------------------------- (d)

def bsa_attn_workspace_size(batch, heads, nq, nk, block_q, block_k, list_heads) -> int:
    return int(load_library().bsa_attn_workspace_size(batch, heads, nq, nk, block_q, block_k,
                                                      list_heads))


def bsa_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, row_ptr: torch.Tensor,
                 col_idx: torch.Tensor, block_q: int, block_k: int, list_heads: int,
                 nq: Optional[int] = None, nk: Optional[int] = None, scale: float = 0.0,
                 o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                 ws: Optional[torch.Tensor] = None):
    """Block-sparse attention forward.  Returns (o [B, nq_rows, H, D] bf16, lse [B, H, nq], ws).

    q, k, v (and o) may be head slices of wider [B, N, H_total, D] tensors or the Q,
    K, V views of a fused projection: q, k and v must share one token-row stride,
    o may have its own."""
    B, _, H, D = q.shape
    nq = q.shape[1] if nq is None else nq
    nk = k.shape[1] if nk is None else nk
    qkv_rs = _shared_stride([(q, "q", _strided_tokens(q, "q", B, nq, H, D)),
                             (k, "k", _strided_tokens(k, "k", B, nk, H, D)),
                             (v, "v", _strided_tokens(v, "v", B, nk, H, D))])
    _lists(row_ptr, col_idx, list_heads, nq, block_q, nk, block_k)
    if o is None:
        o = torch.empty((B, q.shape[1], H, D), dtype=q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B, H, nq), dtype=torch.float32, device=q.device)
    o_rs = _strided_tokens(o, "o", B, nq, H, D)
    _buffer(lse, "lse", torch.float32, B * H * nq)
    if ws is None:
        ws = torch.empty(bsa_attn_workspace_size(B, H, nq, nk, block_q, block_k, list_heads),
                         dtype=torch.uint8, device=q.device)
    _cuda(ws, "ws")
    _check(load_library().bsa_attn_fwd(_ptr(q), _ptr(k), _ptr(v), B, H, nq, nk, D, qkv_rs, o_rs,
                                       block_q, block_k, _ptr(row_ptr), _ptr(col_idx), list_heads,
                                       float(scale), _ptr(o), _ptr(lse), _ptr(ws), _nbytes(ws),
                                       _stream()), "bsa_attn_fwd")
    return o, lse, ws


def bsa_attn_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                         row_ptr: torch.Tensor, col_idx: torch.Tensor, block_q: int, block_k: int,
                         list_heads: int, nq: Optional[int] = None, nk: Optional[int] = None,
                         scale: float = 0.0, o: Optional[torch.Tensor] = None,
                         lse: Optional[torch.Tensor] = None,
                         device_status: Optional[torch.Tensor] = None):
    """bsa_attn_fwd without a workspace argument: the library's fixed per-device
    scratch array is used instead (for callers that may not allocate device
    memory; see include/bsa.h).  Outputs are passed in or created here by the
    caller-side wrapper.  Returns (o, lse)."""
    _cuda(q, "q")
    B, _, H, D = q.shape
    nq = q.shape[1] if nq is None else nq
    nk = k.shape[1] if nk is None else nk
    _tokens(q, "q", B, nq, H, D)
    _tokens(k, "k", B, nk, H, D)
    _tokens(v, "v", B, nk, H, D)
    _lists(row_ptr, col_idx, list_heads, nq, block_q, nk, block_k)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, nq), dtype=torch.float32, device=q.device)
    _tokens(o, "o", B, nq, H, D)
    _buffer(lse, "lse", torch.float32, B * H * nq)
    _status(device_status)
    _check(load_library().bsa_attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), B, H, nq, nk, D,
                                               block_q, block_k, _ptr(row_ptr), _ptr(col_idx),
                                               list_heads, float(scale), _ptr(o), _ptr(lse),
                                               _ptr(device_status), _stream()),
           "bsa_attn_fwd_noalloc")
    return o, lse


def bsa_attn_bwd_workspace_size(batch, heads, nq, nk, block_q, block_k, list_heads) -> int:
    return int(load_library().bsa_attn_bwd_workspace_size(batch, heads, nq, nk, block_q, block_k,
                                                          list_heads))


def bsa_attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                 dout: torch.Tensor, lse: torch.Tensor, row_ptr: torch.Tensor,
                 col_idx: torch.Tensor, block_q: int, block_k: int, list_heads: int,
                 nq: Optional[int] = None, nk: Optional[int] = None, scale: float = 0.0,
                 dq: Optional[torch.Tensor] = None, dk: Optional[torch.Tensor] = None,
                 dv: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None):
    """Block-sparse attention backward.  Returns (dq, dk, dv, ws).

    q, k, v, dq, dk, dv share one token-row stride, o and dout another (each may be
    a head slice of a wider tensor; see bsa_attn_fwd)."""
    B, _, H, D = q.shape
    nq = q.shape[1] if nq is None else nq
    nk = k.shape[1] if nk is None else nk
    _buffer(lse, "lse", torch.float32, B * H * nq)
    _lists(row_ptr, col_idx, list_heads, nq, block_q, nk, block_k)
    dq = torch.empty((B, q.shape[1], H, D), dtype=q.dtype, device=q.device) if dq is None else dq
    dk = torch.empty((B, k.shape[1], H, D), dtype=k.dtype, device=k.device) if dk is None else dk
    dv = torch.empty((B, v.shape[1], H, D), dtype=v.dtype, device=v.device) if dv is None else dv
    qkv_rs = _shared_stride([(t, n, _strided_tokens(t, n, B, rows, H, D)) for t, n, rows in
                             ((q, "q", nq), (k, "k", nk), (v, "v", nk), (dq, "dq", nq),
                              (dk, "dk", nk), (dv, "dv", nk))])
    o_rs = _shared_stride([(t, n, _strided_tokens(t, n, B, nq, H, D)) for t, n in
                           ((o, "o"), (dout, "dout"))])
    if ws is None:
        ws = torch.empty(bsa_attn_bwd_workspace_size(B, H, nq, nk, block_q, block_k, list_heads),
                         dtype=torch.uint8, device=q.device)
    _cuda(ws, "ws")
    _check(load_library().bsa_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                                       B, H, nq, nk, D, qkv_rs, o_rs, block_q, block_k, _ptr(row_ptr),
                                       _ptr(col_idx), list_heads, float(scale), _ptr(dq),
                                       _ptr(dk), _ptr(dv), _ptr(ws), _nbytes(ws), _stream()),
           "bsa_attn_bwd")
    return dq, dk, dv, ws


def _n_tiles(grid, tile) -> int:
    return (-(-grid[0] // tile[0])) * (-(-grid[1] // tile[1])) * (-(-grid[2] // tile[2]))


def bsa_sics_blocks(x: torch.Tensor, grid, tile, out: Optional[torch.Tensor] = None):
    """SICS of every tile of shape `tile` per head.  x: [B, T*H*W, heads, D] bf16 in
    raster order (may be a head slice of a wider tensor).  Returns out [B, heads, n_tiles]
    float32."""
    B, _, Hh, D = x.shape
    xs = _strided_tokens(x, "x", B, grid[0] * grid[1] * grid[2], Hh, D)
    if out is None:
        out = torch.empty((B, Hh, _n_tiles(grid, tile)), dtype=torch.float32, device=x.device)
    _buffer(out, "out", torch.float32, B * Hh * _n_tiles(grid, tile))
    _check(load_library().bsa_sics_blocks(_ptr(x), B, *grid, *tile, Hh, D, xs, _ptr(out),
                                          _stream()), "bsa_sics_blocks")
    return out


def _shape_array(shapes):
    flat = [int(v) for s in shapes for v in s]
    return (ctypes.c_int * len(flat))(*flat), len(shapes)


def bsa_sics_workspace_size(batch, heads, grid, shapes) -> int:
    arr, n = _shape_array(shapes)
    return int(load_library().bsa_sics_workspace_size(batch, heads, *grid, arr, n))


def bsa_sics_scheme(q: torch.Tensor, k: torch.Tensor, grid, shapes,
                    scores: Optional[torch.Tensor] = None, choice: Optional[torch.Tensor] = None,
                    ws: Optional[torch.Tensor] = None):
    """Per-head slicing choice from a shape menu.  Returns (scores [B, H, n_shapes]
    float32, choice [B, H] int32, ws)."""
    B, _, Hh, D = q.shape
    N = grid[0] * grid[1] * grid[2]
    rs = _shared_stride([(q, "q", _strided_tokens(q, "q", B, N, Hh, D)),
                         (k, "k", _strided_tokens(k, "k", B, N, Hh, D))])
    arr, n = _shape_array(shapes)
    if scores is None:
        scores = torch.empty((B, Hh, n), dtype=torch.float32, device=q.device)
    if choice is None:
        choice = torch.empty((B, Hh), dtype=torch.int32, device=q.device)
    _buffer(scores, "scores", torch.float32, B * Hh * n)
    _buffer(choice, "choice", torch.int32, B * Hh)
    if ws is None:
        ws = torch.empty(max(1, bsa_sics_workspace_size(B, Hh, grid, shapes)), dtype=torch.uint8,
                         device=q.device)
    _cuda(ws, "ws")
    _check(load_library().bsa_sics_scheme(_ptr(q), _ptr(k), B, *grid, Hh, D, rs, arr, n,
                                          _ptr(scores), _ptr(choice), _ptr(ws), _nbytes(ws),
                                          _stream()), "bsa_sics_scheme")
    return scores, choice, ws


# --------------------------------------------------------------------------- (g)
# Paged KV cache: pages of KV_PAGE tokens, page tables [B, pages_per_batch] int32.

KV_PAGE = 128


def bsa_kv_write(src: torch.Tensor, first_token: int, page_table: torch.Tensor,
                 pool: torch.Tensor, device_status: Optional[torch.Tensor] = None):
    """Rows src [B, n_new, H, D] -> logical tokens first_token.. of each batch in the
    pool [P, KV_PAGE, H, D] through page_table [B, pages_per_batch]."""
    _cuda(src, "src")
    B, n_new, H, D = src.shape
    _tokens(src, "src", B, n_new, H, D)
    _table(page_table, "page_table", B)
    _pool(pool, "pool", H, D)
    _status(device_status)
    _check(load_library().bsa_kv_write(_ptr(src), B, n_new, H, D, int(first_token),
                                       _ptr(page_table), page_table.shape[1], _ptr(pool),
                                       pool.shape[0], _ptr(device_status), _stream()),
           "bsa_kv_write")


def bsa_block_pool(x: torch.Tensor, n_tokens: int, block: int, first_block: int, n_blocks: int,
                   out: torch.Tensor, page_table: Optional[torch.Tensor] = None, batch: int = 0):
    """Block means of x ([B, n, H, D], or a paged pool [P, KV_PAGE, H, D] with its
    page_table) into out [B, H, out_blocks, D] float32 at blocks first_block.."""
    _cuda(x, "x")
    B = batch if page_table is not None else x.shape[0]
    H, D = x.shape[2], x.shape[3]
    if page_table is not None:
        _pool(x, "x", H, D)
        _table(page_table, "page_table", B)
    else:
        _tokens(x, "x", B, int(n_tokens), H, D)
    _cuda(out, "out")
    if out.dtype != torch.float32 or out.dim() != 4 or out.shape[0] < B or out.shape[1] != H \
            or out.shape[3] != D:
        raise ValueError(f"out must be float32 [{B}, {H}, blocks, {D}], got {out.dtype} "
                         f"{tuple(out.shape)}")
    ppb = page_table.shape[1] if page_table is not None else 0
    _check(load_library().bsa_block_pool(_ptr(x), _ptr(page_table), ppb, B, int(n_tokens), H, D,
                                         int(block), int(first_block), int(n_blocks), _ptr(out),
                                         out.shape[2], _stream()), "bsa_block_pool")
    return out


def bsa_kv_resident_blocks(page_table: torch.Tensor, block: int, KB: int,
                           allowed: Optional[torch.Tensor] = None):
    _table(page_table, "page_table", 1)
    B, ppb = page_table.shape
    if allowed is None:
        allowed = torch.empty((B, KB), dtype=torch.uint8, device=page_table.device)
    _bytes(allowed, "allowed", B * KB)
    _check(load_library().bsa_kv_resident_blocks(_ptr(page_table), B, ppb, int(block), int(KB),
                                                 _ptr(allowed), _stream()),
           "bsa_kv_resident_blocks")
    return allowed


def bsa_kv_page_scores(qbar: torch.Tensor, kbar: torch.Tensor, kb_begin: int, kb_end: int,
                       block: int, n_pages: int, scale: float = 0.0,
                       key_allowed: Optional[torch.Tensor] = None,
                       scores: Optional[torch.Tensor] = None):
    """Page importance [B, n_pages] float32 from pooled means (see include/bsa.h)."""
    _cuda(qbar, "qbar")
    B, H, QB, D = qbar.shape
    _means(qbar, "qbar", B, H, D)
    _means(kbar, "kbar", B, H, D)
    KB = kbar.shape[2]
    if key_allowed is not None:
        _bytes(key_allowed, "key_allowed", B * KB)
    if scale <= 0:
        scale = 1.0 / math.sqrt(D)
    if scores is None:
        scores = torch.empty((B, n_pages), dtype=torch.float32, device=qbar.device)
    _buffer(scores, "scores", torch.float32, B * n_pages)
    _check(load_library().bsa_kv_page_scores(_ptr(qbar), _ptr(kbar), B, H, QB, KB, D, float(scale),
                                             int(kb_begin), int(kb_end), _ptr(key_allowed),
                                             int(block), int(n_pages), _ptr(scores), _stream()),
           "bsa_kv_page_scores")
    return scores


def bsa_kv_keep_pages(scores: torch.Tensor, anchor_pages: int, recent_begin: int, budget: int,
                      page_table: torch.Tensor, freed: torch.Tensor, freed_count: torch.Tensor):
    """Evicts middle pages beyond the budget in place (page_table entries -> -1); the
    freed physical pages are appended to freed at atomic index freed_count."""
    _cuda(scores, "scores")
    if scores.dtype != torch.float32 or scores.dim() != 2:
        raise ValueError(f"scores must be float32 [batch, pages], got {scores.dtype} "
                         f"{tuple(scores.shape)}")
    B, n_pages = scores.shape
    _table(page_table, "page_table", B, n_pages)
    # at most (middle pages - budget) pages per batch are evicted and appended
    _buffer(freed, "freed", torch.int32, B * max(0, recent_begin - anchor_pages - max(budget, 0)))
    _buffer(freed_count, "freed_count", torch.int32, 1)
    _check(load_library().bsa_kv_keep_pages(_ptr(scores), B, n_pages, int(anchor_pages),
                                            int(recent_begin), int(budget), _ptr(page_table),
                                            page_table.shape[1], _ptr(freed), _ptr(freed_count),
                                            _stream()),
           "bsa_kv_keep_pages")


def bsa_attn_fwd_paged(q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor,
                       page_table: torch.Tensor, nk: int, row_ptr: torch.Tensor,
                       col_idx: torch.Tensor, block_q: int, block_k: int, list_heads: int,
                       nq: Optional[int] = None, scale: float = 0.0,
                       o: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                       ws: Optional[torch.Tensor] = None):
    """Block-sparse attention with K/V in paged pools [P, KV_PAGE, H, D]."""
    _cuda(q, "q")
    B, _, H, D = q.shape
    nq = q.shape[1] if nq is None else nq
    _tokens(q, "q", B, nq, H, D)
    _pool(k_pool, "k_pool", H, D)
    _pool(v_pool, "v_pool", H, D)
    if v_pool.shape[0] != k_pool.shape[0]:
        raise ValueError("k_pool and v_pool must hold the same number of pages")
    _table(page_table, "page_table", B)
    _lists(row_ptr, col_idx, list_heads, nq, block_q, nk, block_k)
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, nq), dtype=torch.float32, device=q.device)
    _tokens(o, "o", B, nq, H, D)
    _buffer(lse, "lse", torch.float32, B * H * nq)
    if ws is None:
        ws = torch.empty(bsa_attn_workspace_size(B, H, nq, nk, block_q, block_k, list_heads),
                         dtype=torch.uint8, device=q.device)
    _cuda(ws, "ws")
    _check(load_library().bsa_attn_fwd_paged(_ptr(q), _ptr(k_pool), _ptr(v_pool), k_pool.shape[0],
                                             _ptr(page_table), page_table.shape[1], B, H, nq,
                                             int(nk), D, block_q, block_k, _ptr(row_ptr),
                                             _ptr(col_idx), list_heads, float(scale), _ptr(o),
                                             _ptr(lse), _ptr(ws), _nbytes(ws), _stream()),
           "bsa_attn_fwd_paged")
    return o, lse, ws


def bsa_read_status(ws: torch.Tensor) -> int:
    out = ctypes.c_int(0)
    _check(load_library().bsa_read_status(_ptr(ws), ctypes.byref(out), _stream()),
           "bsa_read_status")
    return out.value


def bsa_wait_selftest(timeout_ns: int, device_status: Optional[torch.Tensor] = None) -> int:
    """Runs the bounded-wait self-test and returns the status it recorded
    (BSA_ERR_TIMEOUT = 5 when the wait gave up as designed)."""
    if device_status is None:
        device_status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(load_library().bsa_wait_selftest(_ptr(device_status), int(timeout_ns), _stream()),
           "bsa_wait_selftest")
    torch.cuda.synchronize()
    return int(device_status.item())


def bsa_status_string(code: int) -> str:
    return load_library().bsa_status_string(code).decode()


def bsa_version() -> int:
    return int(load_library().bsa_version())
