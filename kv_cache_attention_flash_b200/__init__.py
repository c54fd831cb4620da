"""Flash-dLLM per-layer hot path on NVIDIA B200 (sm_100a).

Python binding over the C ABI of libfdllm.so (include/fdllm.h). Functions
carry the C names; they only marshal torch tensors (device memory and the
current CUDA stream) into pointers. The layer step itself, the attention
mass and the top-k selection all run in the library's CUDA kernels; if the
library is missing or no GPU is present the calls raise.

Sources: "Flash-dLLM: I/O-Aware KV Caching and Parallel Decoding for Fast,
Memory-Efficient Diffusion LLMs" (ai4snews summary of the full text),
paragraphs 1-3 (Flash-Cache fusion, scheduled attention with a block table,
tracking budget, Flash-Verify two-view mask).
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import numpy as np
import torch

from . import _lib
from ._lib import (FDLLM_BF16, FDLLM_F32, FDLLM_OK, CacheConfig, FdllmError, Step,  # noqa: F401
                   check_status, load)

__all__ = [
    "fdllm_cache_create", "fdllm_cache_destroy", "fdllm_layer_step", "fdllm_layer_step_noalloc",
    "fdllm_select_tracked", "fdllm_verify_accept", "fdllm_plan_tile_schedule", "fdllm_oproj",
    "fdllm_check", "fdllm_inject_fault", "fdllm_last_launch_count", "FlashCache", "FdllmError",
    "load",
]


def _stream_ptr(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev_ptr(t: Optional[torch.Tensor], dtype=None, name="tensor") -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _out_bf16(out: Optional[torch.Tensor]) -> int:
    """1 for a bf16 `out`, 0 for fp32; anything else is refused."""
    if out is None or out.dtype == torch.float32:
        return 0
    if out.dtype == torch.bfloat16:
        return 1
    raise ValueError(f"out must be float32 or bfloat16, got {out.dtype}")


def _host_i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def fdllm_cache_create(n_layers: int, n_heads: int, head_dim: int, page_size: int,
                       num_pages: int, max_position: int, rope_theta: float, dtype: str,
                       k_pool: torch.Tensor, v_pool: torch.Tensor, max_batch: int,
                       max_slots_per_seq: int, stream=None) -> int:
    """Returns an opaque handle (int) over the caller's K/V pools."""
    lib = load()
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    cfg = CacheConfig(n_layers, n_heads, head_dim, page_size, num_pages, max_position, max_batch,
                      max_slots_per_seq, float(rope_theta),
                      FDLLM_BF16 if dtype == "bf16" else FDLLM_F32)
    shape = (n_layers, num_pages, n_heads, page_size, head_dim)
    for nm, p in (("k_pool", k_pool), ("v_pool", v_pool)):
        if tuple(p.shape) != shape:
            raise ValueError(f"{nm} must have shape {shape}, got {tuple(p.shape)}")
    out = ctypes.c_void_p()
    check_status(lib.fdllm_cache_create(ctypes.byref(cfg), _dev_ptr(k_pool, tdt, "k_pool"),
                                        _dev_ptr(v_pool, tdt, "v_pool"), _stream_ptr(stream),
                                        ctypes.byref(out)))
    return out.value


def fdllm_cache_destroy(handle: int) -> None:
    if handle:
        load().fdllm_cache_destroy(handle)


def fdllm_layer_step(handle: int, layer: int, cu_rows: Sequence[int], seq_lens: Sequence[int],
                     max_blocks_per_seq: int, x: torch.Tensor, wqkv: torch.Tensor,
                     positions: torch.Tensor, block_table: torch.Tensor,
                     view_mask: Optional[torch.Tensor], out: torch.Tensor,
                     attn_mass: Optional[torch.Tensor], slots: Optional[torch.Tensor] = None,
                     validate: bool = False, stream=None) -> None:
    """One Flash-Cache + scheduled-attention layer step (see include/fdllm.h).

    cu_rows, seq_lens: host integer sequences; all tensors on the device."""
    lib = load()
    cu = _host_i32(cu_rows)
    sl = _host_i32(seq_lens)
    st = Step(len(sl), int(cu[-1]), int(max_blocks_per_seq),
              cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
              sl.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
              _dev_ptr(slots, torch.int32, "slots"), 1 if validate else 0, _out_bf16(out))
    check_status(lib.fdllm_layer_step(
        handle, int(layer), ctypes.byref(st), _dev_ptr(x, None, "x"), _dev_ptr(wqkv, None, "wqkv"),
        _dev_ptr(positions, torch.int32, "positions"), _dev_ptr(block_table, torch.int32, "block_table"),
        _dev_ptr(view_mask, torch.int8, "view_mask"), _dev_ptr(out, None, "out"),
        _dev_ptr(attn_mass, torch.float32, "attn_mass"), _stream_ptr(stream)))


def fdllm_layer_step_noalloc(n_layers: int, n_heads: int, head_dim: int, page_size: int,
                             num_pages: int, max_position: int, rope_theta: float, dtype: str,
                             max_batch: int, max_slots_per_seq: int, k_pool: torch.Tensor,
                             v_pool: torch.Tensor, rope_cos: torch.Tensor, rope_sin: torch.Tensor,
                             layer: int, cu_rows: Sequence[int], seq_lens: Sequence[int],
                             max_blocks_per_seq: int, x: torch.Tensor, wqkv: torch.Tensor,
                             positions: torch.Tensor, block_table: torch.Tensor,
                             view_mask: Optional[torch.Tensor], out: torch.Tensor,
                             attn_mass: Optional[torch.Tensor],
                             slots: Optional[torch.Tensor] = None, validate: bool = False,
                             stream=None) -> None:
    """The layer step without a handle or any device allocation, for callers
    that cannot call cudaMalloc when they step (their HBM is already handed
    to a KV pool or to their own allocator). The library keeps its scratch
    in a fixed per-device array; overlapping calls on one GPU race on it.
    rope_cos / rope_sin: caller-owned fp64 [max_position][head_dim / 2]
    tables (see include/fdllm.h)."""
    lib = load()
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    cfg = CacheConfig(n_layers, n_heads, head_dim, page_size, num_pages, max_position, max_batch,
                      max_slots_per_seq, float(rope_theta),
                      FDLLM_BF16 if dtype == "bf16" else FDLLM_F32)
    half = head_dim // 2
    for nm, t in (("rope_cos", rope_cos), ("rope_sin", rope_sin)):
        if tuple(t.shape) != (max_position, half):
            raise ValueError(f"{nm} must have shape {(max_position, half)}, got {tuple(t.shape)}")
    cu = _host_i32(cu_rows)
    sl = _host_i32(seq_lens)
    st = Step(len(sl), int(cu[-1]), int(max_blocks_per_seq),
              cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
              sl.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
              _dev_ptr(slots, torch.int32, "slots"), 1 if validate else 0, _out_bf16(out))
    check_status(lib.fdllm_layer_step_noalloc(
        ctypes.byref(cfg), _dev_ptr(k_pool, tdt, "k_pool"), _dev_ptr(v_pool, tdt, "v_pool"),
        _dev_ptr(rope_cos, torch.float64, "rope_cos"), _dev_ptr(rope_sin, torch.float64, "rope_sin"),
        int(layer), ctypes.byref(st), _dev_ptr(x, None, "x"), _dev_ptr(wqkv, None, "wqkv"),
        _dev_ptr(positions, torch.int32, "positions"), _dev_ptr(block_table, torch.int32, "block_table"),
        _dev_ptr(view_mask, torch.int8, "view_mask"), _dev_ptr(out, None, "out"),
        _dev_ptr(attn_mass, torch.float32, "attn_mass"), _stream_ptr(stream)))


def fdllm_select_tracked(attn_mass: torch.Tensor, seq_lens: torch.Tensor, k: int,
                         exclude_cu: Optional[torch.Tensor] = None,
                         exclude_slots: Optional[torch.Tensor] = None,
                         tracked: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Top-k most attended slots per sequence (see include/fdllm.h)."""
    lib = load()
    B, stride = attn_mass.shape
    if tracked is None:
        tracked = torch.empty(B, k, dtype=torch.int32, device=attn_mass.device)
    check_status(lib.fdllm_select_tracked(
        _dev_ptr(attn_mass, torch.float32, "attn_mass"), _dev_ptr(seq_lens, torch.int32, "seq_lens"),
        int(B), int(stride), int(k), _dev_ptr(exclude_cu, torch.int32, "exclude_cu"),
        _dev_ptr(exclude_slots, torch.int32, "exclude_slots"), _dev_ptr(tracked, torch.int32, "tracked"),
        _stream_ptr(stream)))
    return tracked


def fdllm_verify_accept(mask_logits: torch.Tensor, cu_rows: torch.Tensor,
                        draft_tokens: torch.Tensor, tau: float, pred: Optional[torch.Tensor] = None,
                        conf: Optional[torch.Tensor] = None,
                        n_accepted: Optional[torch.Tensor] = None, stream=None):
    """Flash-Verify acceptance (see include/fdllm.h): returns (pred, conf,
    n_accepted) for mask-view logits [rows, vocab] (bf16 or fp32)."""
    lib = load()
    if mask_logits.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("mask_logits must be bf16 or fp32")
    rows, vocab = mask_logits.shape
    batch = int(cu_rows.numel()) - 1
    dev = mask_logits.device
    if pred is None:
        pred = torch.empty(rows, dtype=torch.int32, device=dev)
    if conf is None:
        conf = torch.empty(rows, dtype=torch.float32, device=dev)
    if n_accepted is None:
        n_accepted = torch.empty(batch, dtype=torch.int32, device=dev)
    check_status(lib.fdllm_verify_accept(
        _dev_ptr(mask_logits, None, "mask_logits"),
        FDLLM_BF16 if mask_logits.dtype == torch.bfloat16 else FDLLM_F32, int(rows), int(vocab),
        _dev_ptr(cu_rows, torch.int32, "cu_rows"), batch,
        _dev_ptr(draft_tokens, torch.int32, "draft_tokens"), float(tau),
        _dev_ptr(pred, torch.int32, "pred"), _dev_ptr(conf, torch.float32, "conf"),
        _dev_ptr(n_accepted, torch.int32, "n_accepted"), _stream_ptr(stream)))
    return pred, conf, n_accepted


def fdllm_plan_tile_schedule(group_cost: Sequence[float], n_heads: int, n_bins: int):
    """The bf16 step's static tile schedule (see include/fdllm.h): returns
    (bin_start [n_bins + 1], tiles [n_groups * n_heads]) as int32 arrays;
    tile t is group t // n_heads, head t % n_heads. Host only."""
    lib = load()
    cost = np.ascontiguousarray(np.asarray(group_cost, dtype=np.float64))
    n_groups = int(cost.size)
    bin_start = np.zeros(max(int(n_bins), 0) + 1, np.int32)
    tiles = np.zeros(max(n_groups * int(n_heads), 0), np.int32)
    check_status(lib.fdllm_plan_tile_schedule(
        cost.ctypes.data if n_groups else None, n_groups, int(n_heads), int(n_bins),
        bin_start.ctypes.data, tiles.ctypes.data if tiles.size else None))
    return bin_start, tiles


def fdllm_oproj(attn_out: torch.Tensor, w_o: torch.Tensor, y: Optional[torch.Tensor] = None,
                status: Optional[torch.Tensor] = None, stream=None,
                residual: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Output projection y = residual + attn_out W_o (see include/fdllm.h):
    bf16 [rows, hidden] times bf16 [hidden, hidden], bf16 result; residual
    is optional and may be y itself."""
    lib = load()
    rows, hidden = attn_out.shape
    if tuple(w_o.shape) != (hidden, hidden):
        raise ValueError(f"w_o must be [{hidden}, {hidden}], got {tuple(w_o.shape)}")
    if residual is not None and tuple(residual.shape) != (rows, hidden):
        raise ValueError(f"residual must be [{rows}, {hidden}], got {tuple(residual.shape)}")
    if y is None:
        y = torch.empty(rows, hidden, dtype=torch.bfloat16, device=attn_out.device)
    check_status(lib.fdllm_oproj(
        _dev_ptr(attn_out, torch.bfloat16, "attn_out"), _dev_ptr(w_o, torch.bfloat16, "w_o"),
        _dev_ptr(residual, torch.bfloat16, "residual"), _dev_ptr(y, torch.bfloat16, "y"),
        int(rows), int(hidden), _dev_ptr(status, torch.int32, "status"), _stream_ptr(stream)))
    return y


def fdllm_check(handle: int, stream=None) -> None:
    """Synchronises the stream and raises FdllmError on a device-side error."""
    check_status(load().fdllm_check(handle, _stream_ptr(stream)))


def fdllm_inject_fault(handle: int, kind: int, wait_ns: int = 0) -> None:
    """Arms a host-made failure for the handle's next split-tile step (see
    include/fdllm.h: the attending CTAs' bounded flag wait runs out after
    wait_ns and the step records FDLLM_ERR_TIMEOUT)."""
    check_status(load().fdllm_inject_fault(handle, int(kind), int(wait_ns)))


def fdllm_last_launch_count() -> int:
    return int(load().fdllm_last_launch_count())


class FlashCache:
    """Owns K/V pools (torch device memory) and the library handle."""

    def __init__(self, n_layers: int, n_heads: int, head_dim: int, page_size: int,
                 num_pages: int, max_position: int, rope_theta: float, dtype: str,
                 max_batch: int, max_slots_per_seq: int, k_pool: Optional[torch.Tensor] = None,
                 v_pool: Optional[torch.Tensor] = None, device="cuda"):
        tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
        shape = (n_layers, num_pages, n_heads, page_size, head_dim)
        self.k_pool = k_pool if k_pool is not None else torch.zeros(shape, dtype=tdt, device=device)
        self.v_pool = v_pool if v_pool is not None else torch.zeros(shape, dtype=tdt, device=device)
        self.page_size = page_size
        self.n_heads = n_heads
        self.head_dim = head_dim
        self.handle = fdllm_cache_create(n_layers, n_heads, head_dim, page_size, num_pages,
                                         max_position, rope_theta, dtype, self.k_pool, self.v_pool,
                                         max_batch, max_slots_per_seq)

    def step(self, layer, cu_rows, seq_lens, x, wqkv, positions, block_table, view_mask=None,
             slots=None, with_mass=True, out=None, attn_mass=None, validate=False, stream=None):
        R = int(cu_rows[-1])
        B = len(seq_lens)
        mb = int(block_table.shape[1])
        if out is None:
            out = torch.empty(R, self.n_heads * self.head_dim, dtype=torch.float32, device=x.device)
        if with_mass and attn_mass is None:
            attn_mass = torch.empty(B, mb * self.page_size, dtype=torch.float32, device=x.device)
        fdllm_layer_step(self.handle, layer, cu_rows, seq_lens, mb, x, wqkv, positions, block_table,
                         view_mask, out, attn_mass if with_mass else None, slots, validate, stream)
        return out, (attn_mass if with_mass else None)

    def check(self, stream=None):
        fdllm_check(self.handle, stream)

    def close(self):
        if self.handle:
            fdllm_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
