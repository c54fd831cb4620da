"""GPU parity of the output projection y = o W_o (fdllm_oproj) against the
oracle, and of the layer step's bf16 `out`.

Tolerance for y: the kernel sums `hidden` bf16 products in fp32 and rounds
once to bf16, so each element is within half a bf16 ulp (2^-9 relative) of
the fp32 sum, and the fp32 sum is within about 1e-6 relative of the exact
one at these sizes; the test allows 2^-8 * |ref| + 1e-4 * RMS(ref)."""
import numpy as np
import pytest
import torch

import kv_cache_attention_flash_b200 as fd
from kv_cache_attention_flash_b200 import workloads as W
from oracle import oracle as O

from gpu_case import build_inputs

pytestmark = pytest.mark.gpu


def _case(rows, hidden, seed):
    g = torch.Generator().manual_seed(seed)
    o = torch.randn(rows, hidden, generator=g).to(torch.bfloat16)
    w = (torch.randn(hidden, hidden, generator=g) * 0.02).to(torch.bfloat16)
    return o, w


def _check(o_bits, w_bits, y_rows):
    ref = O.oproj(o_bits, w_bits)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    bad = np.abs(y_rows - ref) > 2.0 ** -8 * np.abs(ref) + 1e-4 * rms
    assert not bad.any(), f"{int(bad.sum())} elements off; max err {np.abs(y_rows - ref).max():.3e}"


@pytest.mark.parametrize("rows,hidden", [(1, 256), (5, 512), (128, 256), (200, 768), (300, 1024)])
def test_oproj_small(rows, hidden):
    o, w = _case(rows, hidden, rows + hidden)
    y = fd.fdllm_oproj(o.cuda(), w.cuda())
    torch.cuda.synchronize()
    assert fd.fdllm_last_launch_count() == 1
    _check(W.bits_np(o), W.bits_np(w), y.float().cpu().numpy())


def test_oproj_full_size_sampled_rows():
    """The batch-32 size (1536 rows, hidden 4096) in the bench's launch
    configuration, checked on sampled rows (every row tile and both ends of
    every column tile are covered by the rows below)."""
    rows, hidden = 1536, 4096
    o, w = _case(rows, hidden, 7)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = fd.fdllm_oproj(o.cuda(), w.cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rng = np.random.default_rng(0)
    idx = np.unique(np.concatenate([[0, 1, 127, 128, 767, 1535],
                                    np.arange(12) * 128 + 64, rng.integers(0, rows, 8)]))
    _check(W.bits_np(o)[idx], W.bits_np(w), y.float().cpu().numpy()[idx])


def test_oproj_wide_tiles_sampled_rows():
    """128 row tiles per SM at hidden 256: one wave of 256-column tiles
    beats two of 128-column ones, so this runs the 256-wide instance."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rows, hidden = 128 * sms, 256
    o, w = _case(rows, hidden, 9)
    y = fd.fdllm_oproj(o.cuda(), w.cuda())
    torch.cuda.synchronize()
    rng = np.random.default_rng(1)
    idx = np.unique(np.concatenate([[0, rows - 1], np.arange(0, rows, 997), rng.integers(0, rows, 16)]))
    _check(W.bits_np(o)[idx], W.bits_np(w), y.float().cpu().numpy()[idx])


def test_oproj_zero_rows_enqueues_nothing():
    o = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(256, 256, dtype=torch.bfloat16, device="cuda")
    y = fd.fdllm_oproj(o, w)
    assert y.shape == (0, 256)
    assert fd.fdllm_last_launch_count() == 0


def test_oproj_identity_is_exact():
    """W_o = I: every y element is one product by 1 plus exact zeros, so y
    equals o bit for bit."""
    rows, hidden = 130, 512
    o, _ = _case(rows, hidden, 3)
    w = torch.eye(hidden).to(torch.bfloat16)
    y = fd.fdllm_oproj(o.cuda(), w.cuda())
    torch.cuda.synchronize()
    assert torch.equal(y.cpu().view(torch.int16), o.view(torch.int16))


@pytest.mark.parametrize("name", ["small_bf16_divergent", "small_bf16_two_view"])
def test_layer_step_bf16_out_then_oproj(name):
    """The bf16 `out` is the fp32 `out` rounded to nearest even, bit for bit
    (the kernel computes the same fp32 values either way); the projection of
    it matches the oracle's projection of the same bf16 values."""
    spec = W.get_spec(name)
    meta, x, w, kp, vp = build_inputs(spec, 0)
    sh = spec.shape
    dev = "cuda"
    outs = []
    for dt in (torch.float32, torch.bfloat16):
        kp_d, vp_d = kp.to(dev).contiguous(), vp.to(dev).contiguous()
        cache = fd.FlashCache(1, sh.n_heads, sh.head_dim, sh.page_size, meta.num_pages,
                              meta.max_position, sh.rope_theta, sh.dtype, max_batch=meta.batch,
                              max_slots_per_seq=meta.max_blocks * sh.page_size,
                              k_pool=kp_d, v_pool=vp_d)
        out = torch.empty(meta.total_rows, sh.hidden, dtype=dt, device=dev)
        cache.step(0, meta.cu_rows, meta.seq_lens, x.to(dev), w.to(dev),
                   torch.from_numpy(meta.positions).to(dev), torch.from_numpy(meta.block_table).to(dev),
                   view_mask=torch.from_numpy(meta.view).to(dev),
                   slots=torch.from_numpy(meta.slots).to(dev), out=out, validate=True)
        cache.check()
        outs.append(out)
        cache.close()
    assert torch.equal(outs[1].view(torch.int16), outs[0].to(torch.bfloat16).view(torch.int16))
    hidden = sh.hidden
    if hidden % 256 == 0:
        g = torch.Generator().manual_seed(5)
        w_o = (torch.randn(hidden, hidden, generator=g) * 0.02).to(torch.bfloat16)
        y = fd.fdllm_oproj(outs[1], w_o.to(dev))
        torch.cuda.synchronize()
        _check(W.bits_np(outs[1].cpu()), W.bits_np(w_o), y.float().cpu().numpy())


def _check_resid(o_bits, w_bits, r_bits, y_rows):
    ref = O.oproj(o_bits, w_bits, r_bits)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    bad = np.abs(y_rows - ref) > 2.0 ** -8 * np.abs(ref) + 1e-4 * rms
    assert not bad.any(), f"{int(bad.sum())} elements off; max err {np.abs(y_rows - ref).max():.3e}"


@pytest.mark.parametrize("rows,hidden", [(3, 256), (130, 512), (1536, 4096)])
def test_oproj_with_residual_and_in_place(rows, hidden):
    """y = residual + o W_o, into a fresh buffer and in place over the
    residual (the residual stream of a chained stack)."""
    o, w = _case(rows, hidden, 11 + rows)
    g = torch.Generator().manual_seed(rows)
    r = torch.randn(rows, hidden, generator=g).to(torch.bfloat16)
    y = fd.fdllm_oproj(o.cuda(), w.cuda(), residual=r.cuda())
    rd = r.cuda()
    fd.fdllm_oproj(o.cuda(), w.cuda(), y=rd, residual=rd)
    torch.cuda.synchronize()
    idx = np.arange(rows) if rows <= 256 else np.unique(
        np.concatenate([[0, 127, 128, rows - 1], np.random.default_rng(1).integers(0, rows, 16)]))
    ob, wb, rb = W.bits_np(o), W.bits_np(w), W.bits_np(r)
    _check_resid(ob[idx], wb, rb[idx], y.float().cpu().numpy()[idx])
    assert torch.equal(y, rd)
