"""The toy decode loop (kv_cache_attention_flash_b200.decode_loop) against
the same loop driven entirely by the oracle: chunked prefill, then decode
steps whose rows are the sliding window plus the tracked tokens, with the
next tracked set chosen from the last layer's attention mass and tokens
unmasked by the Flash-Verify acceptance rule ("Flash-dLLM: I/O-Aware KV Caching and
Parallel Decoding for Fast, Memory-Efficient Diffusion LLMs", ai4snews summary,
paragraphs 2 and 3).

The oracle side restates the loop's host rules here (window, exclusions,
at least one token per step, drafts) and shares nothing with the GPU side
but the seeded generators. The two loops run independently. Per step the
accepted counts, the window predictions and the tracked sets must agree;
where they first differ, the difference must be a near-tie in the oracle's
own numbers (two logits within one bf16 ulp, or attention masses within a
relative 1e-3, or a confidence within 1e-4 of the threshold), and the
comparison ends there because the loops then legitimately diverge."""
import numpy as np
import pytest
import torch

from kv_cache_attention_flash_b200.decode_loop import ToyDecodeLoop
from kv_cache_attention_flash_b200.workloads import ToyConfig, toy_layout, toy_weights
from oracle import oracle as O

pytestmark = pytest.mark.gpu


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


class Shape:
    def __init__(self, cfg):
        self.dtype = "bf16"
        self.hidden = cfg.hidden
        self.n_heads = cfg.n_heads
        self.head_dim = cfg.head_dim
        self.page_size = cfg.page_size
        self.rope_theta = cfg.rope_theta


class OracleLoop:
    def __init__(self, cfg):
        self.cfg = cfg
        self.sh = Shape(cfg)
        wt = toy_weights(cfg, "cpu")
        self.emb = bits(wt["emb"])
        self.wqkv = [bits(w) for w in wt["wqkv"]]
        self.w_o = [bits(w) for w in wt["w_o"]]
        self.w_lm = bits(wt["w_lm"])
        self.tokens, self.bt, num_pages = toy_layout(cfg)
        self.L = cfg.prompt_len + cfg.gen_len
        shape = (cfg.n_layers, num_pages, cfg.n_heads, cfg.page_size, cfg.head_dim)
        self.kp = np.zeros(shape, np.uint16)
        self.vp = np.zeros(shape, np.uint16)
        self.w = np.full(cfg.batch, cfg.prompt_len, np.int64)
        self.draft = np.full((cfg.batch, self.L), -1, np.int64)
        self.tracked = np.full((cfg.batch, cfg.track_k), -1, np.int32)

    def stack(self, pos_lists, seq_lens):
        B = self.cfg.batch
        cu = np.zeros(B + 1, np.int32)
        cu[1:] = np.cumsum([len(p) for p in pos_lists])
        pos = np.concatenate(pos_lists).astype(np.int32)
        x = self.emb[np.concatenate([self.tokens[b][p] for b, p in enumerate(pos_lists)])]
        view = np.zeros(len(pos), np.int8)
        mass = None
        for l in range(self.cfg.n_layers):
            out, mass, self.kp, self.vp = O.layer_step(
                self.sh, self.kp, self.vp, l, x, self.wqkv[l], pos, pos, cu,
                np.asarray(seq_lens, np.int32), self.bt, view)
            x = O.f64_to_bf16_bits(O.oproj(O.f64_to_bf16_bits(out), self.w_o[l], x))
        return cu, x, mass

    def prefill(self):
        c = 0
        while 128 * c < self.L:
            hi = min(128 * (c + 1), self.L)
            self.stack([np.arange(128 * c, hi) for _ in range(self.cfg.batch)],
                       [hi] * self.cfg.batch)
            c += 1

    def step(self):
        cfg = self.cfg
        B = cfg.batch
        wins, rows = [], []
        for b in range(B):
            win = np.arange(self.w[b], min(self.w[b] + cfg.window, self.L))
            trk = self.tracked[b][self.tracked[b] >= 0].astype(np.int64)
            trk = trk[~np.isin(trk, win)]
            wins.append(win)
            rows.append(np.concatenate([win, trk]))
        cu, x, mass = self.stack(rows, [self.L] * B)
        ex_cu = np.zeros(B + 1, np.int32)
        ex_cu[1:] = np.cumsum([len(w) for w in wins])
        ex = np.concatenate(wins).astype(np.int32)
        tracked = O.select_tracked(mass, np.full(B, self.L, np.int32), cfg.track_k, ex_cu, ex)
        widx = np.concatenate([cu[b] + np.arange(len(wins[b])) for b in range(B)])
        logits = O.f64_to_bf16_bits(O.oproj(x[widx], self.w_lm))
        pred, conf = O.verify_rows(logits, "bf16")
        cu_w = ex_cu
        draft = np.concatenate([self.draft[b][wins[b]] for b in range(B)]).astype(np.int32)
        nacc = O.verify_accept(pred, conf.astype(np.float32), draft, cu_w, np.float32(cfg.tau))
        accepted = np.zeros(B, np.int64)
        for b in range(B):
            n = len(wins[b])
            a = min(n, max(1, int(nacc[b])))
            p = pred[cu_w[b]:cu_w[b + 1]]
            self.tokens[b][wins[b][:a]] = p[:a]
            self.draft[b][wins[b]] = p
            self.w[b] += a
            accepted[b] = a
        self.tracked = tracked
        return accepted, tracked, pred, O.decode(logits, "bf16"), conf, mass


def near_tie_logits(lg_row):
    top = np.sort(lg_row)[-2:]
    ulp = 2.0 ** (np.floor(np.log2(max(abs(top[1]), 2.0 ** -126))) - 7)
    return top[1] - top[0] <= ulp


def test_toy_decode_loop_matches_oracle_driven_loop():
    cfg = ToyConfig(hidden=512, n_heads=4, head_dim=128, n_layers=2, batch=2, prompt_len=64,
                    gen_len=64, window=8, track_k=8, tau=0.5, seed=3)
    gpu = ToyDecodeLoop(cfg, "cuda")
    orc = OracleLoop(cfg)
    gpu.prefill()
    orc.prefill()
    compared = 0
    for step in range(4):
        g_acc, g_trk, g_pred = gpu.step()
        o_acc, o_trk, o_pred, o_logits, o_conf, o_mass = orc.step()
        if not np.array_equal(g_pred, o_pred):
            i = int(np.flatnonzero(g_pred != o_pred)[0])
            assert near_tie_logits(o_logits[i]), f"step {step}: prediction of row {i} differs"
            break
        if not np.array_equal(g_acc, o_acc):
            assert np.any(np.abs(o_conf - cfg.tau) <= 1e-4), f"step {step}: accepted differ"
            break
        same = True
        for b in range(cfg.batch):
            a, o = set(g_trk[b][g_trk[b] >= 0].tolist()), set(o_trk[b][o_trk[b] >= 0].tolist())
            if a != o:
                kth = min(o_mass[b, j] for j in o)
                for j in a ^ o:
                    assert abs(o_mass[b, j] - kth) <= 1e-3 * kth, f"step {step}: slot {j} not a near-tie"
                same = False
        compared += 1
        print(f"[decode] step {step}: accepted {g_acc.tolist()}, tracked sets equal: {same}")
        if not same:
            break
    assert compared >= 1
    # the loop makes progress and its tracked slots are valid positions
    assert np.all(gpu.w > cfg.prompt_len)
    assert np.all((g_trk >= -1) & (g_trk < cfg.prompt_len + cfg.gen_len))


def test_toy_decode_loop_runs_to_completion():
    cfg = ToyConfig(hidden=512, n_heads=4, head_dim=128, n_layers=2, batch=3, prompt_len=64,
                    gen_len=40, window=8, track_k=8, tau=0.5, seed=4)
    gpu = ToyDecodeLoop(cfg, "cuda")
    gpu.prefill()
    steps = 0
    while not gpu.done():
        acc, trk, _ = gpu.step()
        steps += 1
        assert steps <= cfg.gen_len
        for b in range(cfg.batch):
            t = trk[b][trk[b] >= 0]
            assert len(set(t.tolist())) == len(t)
    gpu.cache.check()
    assert np.all(gpu.tokens[:, cfg.prompt_len:] < cfg.hidden)
    assert gpu.rows_done > 0
