"""Failure detection without a GPU fault: a bounded in-kernel wait is made
to run out by a host-side injection, the step reports FDLLM_ERR_TIMEOUT
through fdllm_check, and the same handle then runs a correct step.

The injected wait is the one that the attending CTA of a split tile makes
for the two cache-writing CTAs of its cluster (small steps run each tile as
a cluster of four CTAs). The injection makes those CTAs withhold their
signal, and the wait is bounded to a few milliseconds; nothing traps,
faults or spins unbounded."""
import numpy as np
import pytest
import torch

import kv_cache_attention_flash_b200 as fd
from kv_cache_attention_flash_b200 import _lib
from kv_cache_attention_flash_b200 import workloads as W

from gpu_case import build_inputs, compare, run_gpu, run_oracle


@pytest.mark.gpu
def test_injected_flag_wait_times_out_and_the_handle_recovers():
    spec = W.get_spec("small_bf16_divergent")
    sh = spec.shape
    meta, x, w, kp, vp = build_inputs(spec, 0)
    dev = "cuda"
    cache = fd.FlashCache(1, sh.n_heads, sh.head_dim, sh.page_size, meta.num_pages,
                          meta.max_position, sh.rope_theta, sh.dtype, max_batch=meta.batch,
                          max_slots_per_seq=meta.max_blocks * sh.page_size,
                          k_pool=kp.to(dev), v_pool=vp.to(dev))
    pos = torch.from_numpy(meta.positions).to(dev)
    slots = torch.from_numpy(meta.slots).to(dev)
    view = torch.from_numpy(meta.view).to(dev)
    bt = torch.from_numpy(meta.block_table).to(dev)
    fd.fdllm_inject_fault(cache.handle, _lib.FDLLM_INJECT_SPLIT_FLAG_TIMEOUT, 2_000_000)
    cache.step(0, meta.cu_rows, meta.seq_lens, x.to(dev), w.to(dev), pos, bt, view_mask=view,
               slots=slots, validate=False)
    # this step's tiles ran as four-CTA clusters (the injection is used up)
    with pytest.raises(fd.FdllmError) as ei:
        cache.check()
    assert ei.value.status == _lib.FDLLM_ERR_TIMEOUT
    assert "timed out" in str(ei.value)
    # the word was cleared, and the next step on the same handle is correct
    cache.check()
    g = run_gpu(spec, meta, x, w, kp, vp, cache=cache)
    o = run_oracle(spec, meta, x, w, kp, vp)
    compare(spec, meta, g, o, W.bits_np(kp), W.bits_np(vp), mode="dense",
            label="small_bf16_divergent after a timeout")
    cache.close()


def test_inject_fault_rejects_bad_arguments_without_a_gpu():
    lib = _lib.load()
    assert lib.fdllm_inject_fault(None, 1, 1000) == _lib.FDLLM_ERR_INVALID_ARG
    assert b"null handle" in lib.fdllm_last_error()
