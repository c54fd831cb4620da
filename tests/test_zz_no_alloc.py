"""fdllm_layer_step_noalloc: the layer step for callers that cannot allocate.

A serving engine that has already reserved nearly all free HBM for its paged
KV pool, or a framework whose own allocator must account for every device
byte, cannot let a library call cudaMalloc when a step runs. The no-alloc
entry point serves them: it takes the pools and RoPE tables the caller owns,
and keeps its only scratch (per-head attention-mass partials and an error
word) in a fixed array inside the library's device image.

These tests call it through the C ABI twice in a row (the second call runs
on the cache the first one wrote, and on whatever the first call left in the
shared scratch). Each call is compared with fdllm_layer_step on the same
inputs and with the CPU oracle, within the parity tests' tolerances. This file sorts last so that a run
stopping at the first failure has run every other test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

import kv_cache_attention_flash_b200 as fd
from kv_cache_attention_flash_b200 import _lib
from kv_cache_attention_flash_b200 import workloads as W
from oracle import oracle as O

from gpu_case import GpuResult, compare

# Capacity of the library's fixed mass scratch, in floats (8 MiB less a
# 256-byte header for the error word).
SCRATCH_FLOATS = ((8 << 20) - 256) // 4


def rope_tables(max_position, head_dim, theta, device):
    """cos / sin of p * theta^(-2i/head_dim), float64 (the caller's tables)."""
    half = head_dim // 2
    inv = np.power(np.float64(np.float32(theta)), -2.0 * np.arange(half) / head_dim)
    phi = np.arange(max_position, dtype=np.float64)[:, None] * inv[None, :]
    return (torch.from_numpy(np.cos(phi)).to(device), torch.from_numpy(np.sin(phi)).to(device))


def bf16_ulp(v):
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


@np.errstate(invalid="ignore")      # the pools hold NaN sentinels outside the written slots
def assert_close(spec, a_out, a_mass, a_k, a_v, b_out, b_mass, b_k, b_v, what):
    rms = float(np.sqrt(np.mean(a_out ** 2)))
    tol = (1e-2 if spec.shape.dtype == "bf16" else 1e-4) * rms
    err = float(np.max(np.abs(a_out - b_out))) if a_out.size else 0.0
    assert np.all(np.isfinite(b_out)), f"{what}: non-finite out"
    assert err <= tol, f"{what}: out differs by {err:.3e} > {tol:.3e}"
    d = np.abs(a_mass - b_mass)
    assert np.all(d <= 1e-3 * np.abs(a_mass) + 1e-6), f"{what}: mass differs by {d.max():.3e}"
    for name, pa, pb in (("k", a_k, b_k), ("v", a_v, b_v)):
        if spec.shape.dtype == "bf16":
            va = (pa.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            vb = (pb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        else:
            va = pa.view(np.float32).astype(np.float64)
            vb = pb.view(np.float32).astype(np.float64)
        same = pa == pb
        fin = np.isfinite(va)
        wrms = float(np.sqrt(np.mean(va[fin] ** 2))) if fin.any() else 0.0
        if spec.shape.dtype == "bf16":
            ok = same | (np.abs(va - vb) <= bf16_ulp(va) * 1.0001 + 1e-3 * wrms)
        else:
            ok = same | (np.abs(va - vb) <= 1e-5 * (np.abs(va) + wrms))
        assert np.all(ok), f"{what}: {int((~ok).sum())} {name} cache values differ"


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["small_bf16_divergent", "small_f32_divergent", "b32_divergent"])
def test_noalloc_matches_layer_step_twice(name):
    spec = W.get_spec(name)
    sh = spec.shape
    dev = "cuda"
    meta = W.make_meta(spec, 0)
    mb, ps = meta.max_blocks, sh.page_size
    assert sh.n_heads * meta.batch * mb * ps <= SCRATCH_FLOATS
    # dense inputs on the grids where the fp32 projection is exact, so that
    # the oracle comparison can hold the plain bar (fp32 workloads: plain)
    grid = sh.dtype == "bf16"
    mx = W.make_x_grid if grid else W.make_x
    xs = [mx(spec, meta, 0, device=dev), mx(spec, meta, 1, device=dev)]
    w = (W.make_w_grid if grid else W.make_w)(spec, 0, device=dev)
    kp, vp = W.make_pools(spec, meta, 0, device=dev, n_layers=1)
    pos = torch.from_numpy(meta.positions).to(dev)
    slots = torch.from_numpy(meta.slots).to(dev)
    view = torch.from_numpy(meta.view).to(dev)
    bt = torch.from_numpy(meta.block_table).to(dev)
    R, H = meta.total_rows, sh.hidden

    # existing entry point, on its own copy of the pools
    cache = fd.FlashCache(1, sh.n_heads, sh.head_dim, ps, meta.num_pages, meta.max_position,
                          sh.rope_theta, sh.dtype, max_batch=meta.batch, max_slots_per_seq=mb * ps,
                          k_pool=kp.clone(), v_pool=vp.clone())
    # no-alloc entry point, on another copy
    kb, vb = kp.clone(), vp.clone()
    cos, sin = rope_tables(meta.max_position, sh.head_dim, sh.rope_theta, dev)

    def bits(t):
        return W.bits_np(t[0])

    # the oracle's own cache state, carried from call to call
    o_kp, o_vp = W.bits_np(kp), W.bits_np(vp)
    sl_d = torch.from_numpy(meta.seq_lens).to(dev)
    ecu_d = torch.from_numpy(meta.exclude_cu).to(dev)
    esl_d = torch.from_numpy(meta.exclude_slots if len(meta.exclude_slots)
                             else np.zeros(1, np.int32)).to(dev)
    for call, x in enumerate(xs):
        out_a, mass_a = cache.step(0, meta.cu_rows, meta.seq_lens, x, w, pos, bt, view_mask=view,
                                   slots=slots, validate=True)
        cache.check()
        out_b = torch.full((R, H), float("nan"), dtype=torch.float32, device=dev)
        mass_b = torch.full((meta.batch, mb * ps), float("nan"), dtype=torch.float32, device=dev)
        fd.fdllm_layer_step_noalloc(1, sh.n_heads, sh.head_dim, ps, meta.num_pages,
                                    meta.max_position, sh.rope_theta, sh.dtype, meta.batch, mb * ps,
                                    kb, vb, cos, sin, 0, meta.cu_rows, meta.seq_lens, mb, x, w, pos,
                                    bt, view, out_b, mass_b, slots=slots, validate=True)
        assert fd.fdllm_last_launch_count() == 2
        torch.cuda.synchronize()
        assert_close(spec, out_a.cpu().numpy(), mass_a.cpu().numpy(), bits(cache.k_pool),
                     bits(cache.v_pool), out_b.cpu().numpy(), mass_b.cpu().numpy(), bits(kb),
                     bits(vb), f"{name} call {call + 1}")
        # and against the oracle directly
        orc = O.layer_step(sh, o_kp, o_vp, 0, W.bits_np(x), W.bits_np(w), meta.positions,
                           meta.slots, meta.cu_rows, meta.seq_lens, meta.block_table, meta.view)
        tracked = fd.fdllm_select_tracked(mass_b, sl_d, meta.track_k, ecu_d, esl_d).cpu().numpy()
        g = GpuResult(out_b.cpu().numpy(), mass_b.cpu().numpy(), tracked, bits(kb), bits(vb))
        compare(spec, meta, g, orc, o_kp, o_vp, mode="grid" if grid else "plain",
                label=f"{name} no-alloc call {call + 1}")
        o_kp, o_vp = orc[2], orc[3]
    cache.close()


@pytest.mark.gpu
def test_noalloc_reports_device_errors_once():
    """A bad block-table entry in a call without validation is kept in the
    shared error word, reported by the next validating call, then cleared."""
    spec = W.get_spec("small_bf16_divergent")
    sh = spec.shape
    dev = "cuda"
    meta = W.make_meta(spec, 0)
    mb, ps = meta.max_blocks, sh.page_size
    x = W.make_x(spec, meta, 0, device=dev)
    w = W.make_w(spec, 0, device=dev)
    kp, vp = W.make_pools(spec, meta, 0, device=dev, n_layers=1)
    cos, sin = rope_tables(meta.max_position, sh.head_dim, sh.rope_theta, dev)
    pos = torch.from_numpy(meta.positions).to(dev)
    slots = torch.from_numpy(meta.slots).to(dev)
    view = torch.from_numpy(meta.view).to(dev)
    bad = meta.block_table.copy()
    bad[0, 0] = meta.num_pages + 5          # outside the pool: the kernel skips and records it
    out = torch.empty(meta.total_rows, sh.hidden, dtype=torch.float32, device=dev)
    mass = torch.empty(meta.batch, mb * ps, dtype=torch.float32, device=dev)
    args = (1, sh.n_heads, sh.head_dim, ps, meta.num_pages, meta.max_position, sh.rope_theta,
            sh.dtype, meta.batch, mb * ps, kp, vp, cos, sin, 0, meta.cu_rows, meta.seq_lens, mb, x,
            w, pos)
    fd.fdllm_layer_step_noalloc(*args, torch.from_numpy(bad).to(dev), view, out, mass, slots=slots,
                                validate=False)
    torch.cuda.synchronize()
    good = torch.from_numpy(meta.block_table).to(dev)
    with pytest.raises(fd.FdllmError) as ei:
        fd.fdllm_layer_step_noalloc(*args, good, view, out, mass, slots=slots, validate=True)
    assert ei.value.status == 4
    fd.fdllm_layer_step_noalloc(*args, good, view, out, mass, slots=slots, validate=True)


def test_noalloc_rejects_oversized_mass_scratch():
    """Host check, no GPU needed: a step whose mass partials exceed the fixed
    scratch is refused before anything touches the device."""
    lib = _lib.load()
    n_heads, batch, mb, ps = 32, 64, 32, 64       # 32 * 64 * 2048 floats > capacity
    assert n_heads * batch * mb * ps > SCRATCH_FLOATS
    cfg = _lib.CacheConfig(1, n_heads, 128, ps, 4096, 4096, batch, mb * ps, 500000.0, _lib.FDLLM_BF16)
    cu = np.arange(batch + 1, dtype=np.int32)
    sl = np.full(batch, 100, dtype=np.int32)
    st = _lib.Step(batch, batch, mb, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                   sl.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), None, 0)
    fake = 1 << 20          # 16-byte aligned, never dereferenced: the call must stop first
    rc = lib.fdllm_layer_step_noalloc(ctypes.byref(cfg), fake, fake, fake, fake, 0, ctypes.byref(st),
                                      fake, fake, fake, fake, None, fake, fake, None)
    assert rc == 2, lib.fdllm_last_error()
    assert b"scratch" in lib.fdllm_last_error()
    # null tables are refused as well
    rc = lib.fdllm_layer_step_noalloc(ctypes.byref(cfg), fake, fake, None, None, 0, ctypes.byref(st),
                                      fake, fake, fake, fake, None, fake, fake, None)
    assert rc == 1
