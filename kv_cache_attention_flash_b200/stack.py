"""A stack of Flash-Cache layer steps chained through the residual stream.

The pages describe one layer's hot path ("Flash-dLLM: I/O-Aware KV Caching
and Parallel Decoding for Fast, Memory-Efficient Diffusion LLMs", ai4snews
summary, paragraph 1). A model runs it once per layer, and a layer's output
reaches the next layer through the attention block's output projection and
the residual stream. Per layer l this module runs

    out_l   = fused layer step on x_l          (fdllm_layer_step, bf16 out)
    x_{l+1} = x_l + out_l W_o,l                (fdllm_oproj with the residual,
                                                in place over x)

The MLP and the norms of a full transformer block are not part of the path
and are left out. Host orchestration only: every arithmetic step runs in the
library's kernels, in stream order.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import FlashCache, fdllm_last_launch_count, fdllm_layer_step, fdllm_oproj


class LayerStack:
    """Chained layers over one FlashCache (one pool slice per layer).

    wqkv[l]: bf16 [H, 3H]; w_o[l]: bf16 [H, H]. run() updates x in place
    (x_0 in, x_L out) and returns the last layer's attention mass."""

    def __init__(self, cache: FlashCache, wqkv: Sequence[torch.Tensor],
                 w_o: Sequence[torch.Tensor]):
        if len(wqkv) != len(w_o):
            raise ValueError("one W_o per layer")
        self.cache = cache
        self.wqkv = list(wqkv)
        self.w_o = list(w_o)
        self.n_layers = len(self.wqkv)
        self._out = None
        self.launches = 0

    def run(self, cu_rows, seq_lens, x: torch.Tensor, positions: torch.Tensor,
            block_table: torch.Tensor, view_mask: Optional[torch.Tensor] = None,
            slots: Optional[torch.Tensor] = None, attn_mass: Optional[torch.Tensor] = None,
            stream=None, x_out: Optional[torch.Tensor] = None, outs=None):
        """One pass through the stack. With x_out, x stays as it is: the
        first projection writes the residual stream into x_out and the later
        layers update x_out in place; without it, x is updated in place.
        `outs`, a dict, receives a copy of each layer's bf16 out when given
        (for tests). Returns (the final residual stream, attn_mass)."""
        R, H = x.shape
        if self._out is None or self._out.shape != (R, H):
            self._out = torch.empty(R, H, dtype=torch.bfloat16, device=x.device)
        mb = int(block_table.shape[1])
        n = 0
        cur = x
        dst = x if x_out is None else x_out
        for l in range(self.n_layers):
            fdllm_layer_step(self.cache.handle, l, cu_rows, seq_lens, mb, cur, self.wqkv[l],
                             positions, block_table, view_mask, self._out, attn_mass, slots,
                             False, stream)
            n += fdllm_last_launch_count()
            if outs is not None:
                outs[l] = self._out.clone()
            fdllm_oproj(self._out, self.w_o[l], y=dst, residual=cur, stream=stream)
            n += fdllm_last_launch_count()
            cur = dst
        self.launches = n
        return dst, attn_mass
