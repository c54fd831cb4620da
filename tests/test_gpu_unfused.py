"""The unfused PyTorch arm of the benchmark (the pages' prior art: separate
launches for the projection, RoPE, the cache write, the gathers and the
attention) computes the same step: compared with the oracle at the same bar
as the fused path, on grid inputs (exact projection) at small and full
size. It runs torch/cuBLAS kernels, not this library's."""
import numpy as np
import pytest
import torch

import bench
from kv_cache_attention_flash_b200 import workloads as W

from gpu_case import build_inputs, run_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["small_bf16_divergent", "small_bf16_two_view", "b32_divergent"])
def test_unfused_arm_matches_oracle(name):
    torch.backends.cuda.matmul.allow_tf32 = True
    spec = W.get_spec(name)
    sh = spec.shape
    meta, x, w, kp, vp = build_inputs(spec, 0, grid=True)
    dev = "cuda"
    u = bench.UnfusedStep(spec, meta, dev)
    kd, vd = kp.to(dev), vp.to(dev)
    out = torch.zeros(meta.total_rows, sh.hidden, dtype=torch.float32, device=dev)
    mass = torch.zeros(meta.batch, meta.max_blocks * sh.page_size, dtype=torch.float32, device=dev)
    u.step(0, kd, vd, x.to(dev), w.to(dev), torch.from_numpy(meta.positions).to(dev),
           torch.from_numpy(meta.slots).to(dev), torch.from_numpy(meta.view).to(dev),
           torch.from_numpy(meta.block_table).to(dev), out, mass)
    torch.cuda.synchronize()
    o_out, o_mass, _, _ = run_oracle(spec, meta, x, w, kp, vp)
    rms = float(np.sqrt(np.mean(o_out ** 2)))
    err = float(np.max(np.abs(out.cpu().numpy() - o_out)))
    print(f"[parity] unfused {name}: max|err|/RMS = {err / rms:.3e}")
    assert err <= 1e-2 * rms
    md = np.abs(mass.cpu().numpy() - o_mass)
    assert np.all(md <= 1e-3 * np.abs(o_mass) + 1e-6)
