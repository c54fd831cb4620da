"""A toy masked-diffusion decode loop on random weights, driven by the
layer-step library.

The pages describe the control flow of Flash-dLLM decoding ("Flash-dLLM:
I/O-Aware KV Caching and Parallel Decoding for Fast, Memory-Efficient
Diffusion LLMs", ai4snews summary of the full text): each step's queries are
a sliding unmasking window plus a fixed budget of the most-attended tokens,
whose cache entries are refreshed (paragraph 2); the attention mass of a
step chooses the next step's tracked tokens (paragraph 2); and a drafted
token is accepted when it agrees with the model's prediction at a
confidence above a threshold, in position order, stopping at the first
disagreement (paragraph 3). This module runs that loop on random weights so
that the feedback from the attention mass to the next step's rows is
exercised end to end. It measures throughput only and claims nothing about
output quality.

Per decode step, for every unfinished sequence b:
  1. rows: the window positions [w_b, w_b + window) (clipped at L), then the
     tracked positions outside the window; x = E[token] of each row.
  2. the chained layer stack (kv_cache_attention_flash_b200.stack): fused
     layer step, output projection with the residual, per layer.
  3. fdllm_select_tracked on the last layer's attention mass, the window
     excluded: the next step's tracked positions.
  4. logits of the window rows through a random LM head of vocabulary H
     (fdllm_oproj against W_lm [H, H]).
  5. fdllm_verify_accept against the drafts (the previous step's
     predictions at the same positions; none at first): the accepted prefix.
     At least one token is unmasked per step (the first window position,
     with its prediction), so every sequence finishes.
  6. accepted tokens are committed, the window slides past them, and the
     remaining window positions keep their predictions as drafts.

The cache is filled first by a chunked prefill (at most 128 positions per
sequence per step, each chunk seeing the slots written so far). Every slot
[0, L) stays visible afterwards: masked positions attend and are attended
(bidirectional masked diffusion). Host orchestration only: all arithmetic
of the steps runs in the library's kernels; torch gathers embedding rows
and moves the small per-step metadata.
"""
from __future__ import annotations

from typing import List, Optional

import numpy as np
import torch

from . import FlashCache, fdllm_oproj, fdllm_select_tracked, fdllm_verify_accept
from .stack import LayerStack
from .workloads import ToyConfig, toy_layout, toy_weights  # noqa: F401


class ToyDecodeLoop:
    """The loop on the GPU (see the module docstring)."""

    def __init__(self, cfg: ToyConfig, device="cuda"):
        self.cfg = cfg
        self.dev = device
        H, L = cfg.hidden, cfg.prompt_len + cfg.gen_len
        if cfg.window + cfg.track_k > 128:
            raise ValueError("window + track_k rows must fit one 128-row sequence")
        if H % 256:
            raise ValueError("hidden must be a multiple of 256 (output projection and LM head)")
        self.L = L
        self.wt = toy_weights(cfg, device)
        tokens, bt, num_pages = toy_layout(cfg)
        self.tokens = tokens
        self.bt = torch.from_numpy(bt).to(device)
        self.mb = bt.shape[1]
        self.cache = FlashCache(cfg.n_layers, cfg.n_heads, cfg.head_dim, cfg.page_size, num_pages,
                                L, cfg.rope_theta, "bf16", cfg.batch, self.mb * cfg.page_size,
                                device=device)
        self.stack = LayerStack(self.cache, self.wt["wqkv"], self.wt["w_o"])
        self.w = np.full(cfg.batch, cfg.prompt_len, np.int64)      # window starts
        self.draft = np.full((cfg.batch, L), -1, np.int64)        # predictions kept as drafts
        self.tracked = np.full((cfg.batch, cfg.track_k), -1, np.int32)
        self.mass = torch.empty(cfg.batch, self.mb * cfg.page_size, dtype=torch.float32,
                                device=device)
        self.seq_lens_d = torch.full((cfg.batch,), L, dtype=torch.int32, device=device)
        self.steps = 0
        self.rows_done = 0

    def _run_stack(self, pos_lists: List[np.ndarray], seq_lens, with_mass: bool):
        cu = np.zeros(len(pos_lists) + 1, np.int32)
        cu[1:] = np.cumsum([len(p) for p in pos_lists])
        pos = np.concatenate(pos_lists).astype(np.int32) if cu[-1] else np.zeros(0, np.int32)
        ids = np.concatenate([self.tokens[b][p] for b, p in enumerate(pos_lists)]) \
            if cu[-1] else np.zeros(0, np.int64)
        x = self.wt["emb"][torch.from_numpy(ids).to(self.dev)].contiguous()
        pos_d = torch.from_numpy(pos).to(self.dev)
        xo = torch.empty_like(x)
        self.stack.run(cu, seq_lens, x, pos_d, self.bt, None, None,
                       self.mass if with_mass else None, x_out=xo)
        return cu, pos, xo

    def prefill(self):
        """Chunked prefill: chunk c holds positions [128c, 128c + 128) of
        every sequence and sees the slots [0, 128(c + 1)) written so far."""
        c = 0
        while 128 * c < self.L:
            hi = min(128 * (c + 1), self.L)
            self._run_stack([np.arange(128 * c, hi) for _ in range(self.cfg.batch)],
                            [hi] * self.cfg.batch, with_mass=False)
            c += 1
        self.cache.check()

    def done(self) -> bool:
        return bool(np.all(self.w >= self.L))

    def step(self):
        """One decode step. Returns (accepted per sequence, the next tracked
        set [B, k], the window predictions in row order)."""
        cfg = self.cfg
        B = cfg.batch
        wins, rows = [], []
        for b in range(B):
            win = np.arange(self.w[b], min(self.w[b] + cfg.window, self.L))
            trk = self.tracked[b][self.tracked[b] >= 0].astype(np.int64)
            trk = trk[~np.isin(trk, win)]
            wins.append(win)
            rows.append(np.concatenate([win, trk]))
        cu, pos, xo = self._run_stack(rows, [self.L] * B, with_mass=True)
        # next tracked set: the most attended slots outside the window
        ex_cu = np.zeros(B + 1, np.int32)
        ex_cu[1:] = np.cumsum([len(w) for w in wins])
        ex = np.concatenate(wins).astype(np.int32) if ex_cu[-1] else np.zeros(1, np.int32)
        tracked = fdllm_select_tracked(self.mass, self.seq_lens_d, cfg.track_k,
                                       torch.from_numpy(ex_cu).to(self.dev),
                                       torch.from_numpy(ex).to(self.dev))
        # window rows -> LM head -> acceptance against the drafts
        widx = np.concatenate([cu[b] + np.arange(len(wins[b])) for b in range(B)]).astype(np.int64)
        cu_w = np.zeros(B + 1, np.int32)
        cu_w[1:] = np.cumsum([len(w) for w in wins])
        accepted = np.zeros(B, np.int64)
        pred_h = np.zeros(0, np.int32)
        if len(widx):
            xw = xo[torch.from_numpy(widx).to(self.dev)].contiguous()
            logits = fdllm_oproj(xw, self.wt["w_lm"])
            draft = np.concatenate([self.draft[b][wins[b]] for b in range(B)]).astype(np.int32)
            pred, conf, nacc = fdllm_verify_accept(logits, torch.from_numpy(cu_w).to(self.dev),
                                                   torch.from_numpy(draft).to(self.dev), cfg.tau)
            pred_h = pred.cpu().numpy()
            nacc_h = nacc.cpu().numpy()
            for b in range(B):
                n = len(wins[b])
                if n == 0:
                    continue
                a = min(n, max(1, int(nacc_h[b])))
                p = pred_h[cu_w[b]:cu_w[b + 1]]
                self.tokens[b][wins[b][:a]] = p[:a]
                self.draft[b][wins[b]] = p
                self.w[b] += a
                accepted[b] = a
        self.tracked = tracked.cpu().numpy()
        self.steps += 1
        self.rows_done += int(cu[-1])
        return accepted, self.tracked.copy(), pred_h
