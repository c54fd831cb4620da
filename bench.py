"""Benchmark of the Flash-dLLM per-layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

`--workload verify_b8` measures the Flash-Verify acceptance step instead
(mask-view logits of 8 x 32 block positions over the 126464-token LLaDA
vocabulary, bf16): positions/s, HBM roofline of the logits read.
`--workload oproj_b32` measures the output projection y = o W_o of the
batch-32 step's 1536 rows at hidden 4096 (bf16): rows/s, tensor roofline.

A step is one pass of the whole hot path over one batch of synthetic input:
the fused layer step (projection, RoPE, cache write, scheduled attention,
attention mass) for every layer of the workload, then the top-k tracking
selection. The default workload is the batch-32 divergent-length layer
(32 sequences, context U[256, 1024], half caching stage, half update stage,
LLaDA-8B layer shape, bf16).

Timing: W untimed warm-up steps, then exactly K steps, each bracketed by CUDA
events on the launching stream with an L2 flush (a 256 MB write) between
steps, outside the events, followed by a short device-side spin so that the
host has queued the step before its start event is reached (the events time
GPU work; the end-to-end figure keeps host planning and copies in its timed
region); barrier + synchronize on both sides; the total is the max over
ranks. Under torchrun each rank runs its own batch (independent
sequences: weak scaling, no collective on the data path).

One JSON line is printed by rank 0.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from kv_cache_attention_flash_b200 import workloads as W  # noqa: E402

METRIC = "fused layer-step query-tokens/s; achieved HBM GB/s and % of roofline (1×B200)"
UNIT = "query-tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


# ------------------------------------------------------------------ helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# DRAM traffic of the fused step kernel, per launch, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), with the code hashes of the
# sources it was captured on: the kernel, its PTX helpers and the host code
# that plans its launch. The figure is reported only while all three match.
CAPTURED_TRAFFIC = {
    "b32_divergent": {
        "bytes": 736288768.0,     # 686.40 MB read + 49.89 MB written, one launch
        "sources": ["d2c28123dd4f13676f9d438248cd6a0d8d0f8cb0abb2a46ebf2c508dbc1101a7",
                    "fe252cfc00f64efb448b0b58ddb2084b317046d35d5a39eef1fab7842009c83a",
                    "552a823d86a5e54df26e2e180d35ea47c9a07907f4669983f5435c1b5c152123"],
        "source": "ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum, one launch "
                  "(profiles/step_bf16_b32_divergent.md)",
    },
}


def captured_traffic(name: str):
    """DRAM bytes per launch of the step kernel for this workload, if a
    capture of the current kernel sources is recorded above (else None)."""
    rec = CAPTURED_TRAFFIC.get(name)
    if rec is None:
        return None
    csrc = os.path.join(ROOT, "kv_cache_attention_flash_b200", "csrc")
    have = [code_hash(os.path.join(csrc, f)) for f in ("step_bf16.cu", "ptx.cuh", "api.cu")]
    return rec["bytes"] if have == rec["sources"] else None


def code_hash(path: str) -> str:
    """sha256 of a CUDA source with // comments and blank lines removed, so
    that an edit of comments alone keeps a capture valid."""
    import hashlib
    lines = []
    for line in open(path).read().splitlines():
        code = line.split("//", 1)[0].rstrip()
        if code.strip():
            lines.append(code)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def reduce_max(value: float, device) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value: float, device) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def aggregate(total_ms_local: float, units_local: float, device):
    """Whole-job throughput of independent replicas: the slowest rank's time
    and the units of all ranks. Returns (max ms, total units, units/s)."""
    total_ms = reduce_max(total_ms_local, device)
    units_all = reduce_sum(units_local, device)
    return total_ms, units_all, units_all / (total_ms / 1000.0)


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


class ClockSampler:
    """nvidia-smi clock/throttle sampling in the background."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.thread = None
        self.window = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        rows = []
        for t, line in self.samples:
            if self.window and not (self.window[0] - 0.1 <= t <= self.window[1] + 0.1):
                continue
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            rows.append(p)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ workload
class Workload:
    """Device-resident inputs of one workload (one rank's batch)."""

    def __init__(self, name: str, seed: int, device):
        import kv_cache_attention_flash_b200 as fd
        self.fd = fd
        self.spec = W.get_spec(name)
        self.meta = W.make_meta(self.spec, seed)
        sh = self.spec.shape
        self.n_layers = sh.n_layers
        self.device = device
        m = self.meta
        self.x = [W.make_x(self.spec, m, seed, layer=l, device=device) for l in range(self.n_layers)]
        self.w = [W.make_w(self.spec, seed, layer=l, device=device) for l in range(self.n_layers)]
        kp, vp = W.make_pools(self.spec, m, seed, device=device)
        self.cache = fd.FlashCache(self.n_layers, sh.n_heads, sh.head_dim, sh.page_size, m.num_pages,
                                   m.max_position, sh.rope_theta, sh.dtype, m.batch,
                                   m.max_blocks * sh.page_size, k_pool=kp, v_pool=vp)
        self.pos = torch.from_numpy(m.positions).to(device)
        self.slots = torch.from_numpy(m.slots).to(device)
        self.view = torch.from_numpy(m.view).to(device)
        self.bt = torch.from_numpy(m.block_table).to(device)
        self.seq_lens_d = torch.from_numpy(m.seq_lens).to(device)
        self.ex_cu = torch.from_numpy(m.exclude_cu).to(device)
        ex = m.exclude_slots if len(m.exclude_slots) else np.zeros(1, np.int32)
        self.ex_sl = torch.from_numpy(ex).to(device)
        R = m.total_rows
        H = sh.hidden
        self.out = torch.empty(R, H, dtype=torch.float32, device=device)
        # a chained stack: x_0 only; layer l's x is the residual stream
        # x_{l-1} + out_{l-1} W_o,{l-1} (bf16 out, output projection with the
        # residual), kept in self.xs while x_0 stays as drawn
        self.chained = self.spec.chained
        if self.chained:
            from kv_cache_attention_flash_b200.stack import LayerStack
            self.x = self.x[:1]
            self.w_o = [W.make_w_o(self.spec, seed, layer=l, device=device)
                        for l in range(self.n_layers)]
            self.stack = LayerStack(self.cache, self.w, self.w_o)
            self.xs = torch.empty_like(self.x[0])
        self.mass = torch.empty(m.batch, m.max_blocks * sh.page_size, dtype=torch.float32, device=device)
        self.tracked = torch.empty(m.batch, m.track_k, dtype=torch.int32, device=device)
        self.launches_per_step = None

    def step(self, x_list=None, ev=None, layer_span=False):
        """One pass of the hot path; returns the number of kernels launched.
        If `ev` is given, events are recorded around the first layer step, or
        (layer_span) from the first layer step to the end of the last."""
        fd = self.fd
        m = self.meta
        n = 0
        xs = x_list if x_list is not None else self.x
        nl = self.n_layers
        if self.chained:
            if ev is not None:
                ev[0].record()
            self.stack.run(m.cu_rows, m.seq_lens, xs[0], self.pos, self.bt, self.view, self.slots,
                           self.mass, x_out=self.xs)
            n += self.stack.launches
            if ev is not None:
                ev[1].record()
            fd.fdllm_select_tracked(self.mass, self.seq_lens_d, m.track_k, self.ex_cu, self.ex_sl,
                                    self.tracked)
            return n + fd.fdllm_last_launch_count()
        for l in range(nl):
            if ev is not None and l == 0:
                ev[0].record()
            fd.fdllm_layer_step(self.cache.handle, l, m.cu_rows, m.seq_lens, m.max_blocks, xs[l],
                                self.w[l], self.pos, self.bt, self.view, self.out, self.mass,
                                self.slots)
            if ev is not None and (l == nl - 1 or not layer_span):
                ev[1].record()
                ev = None
            n += fd.fdllm_last_launch_count()
        fd.fdllm_select_tracked(self.mass, self.seq_lens_d, m.track_k, self.ex_cu, self.ex_sl,
                                self.tracked)
        n += fd.fdllm_last_launch_count()
        return n


# ------------------------------------------------------------------ unfused baseline
class UnfusedStep:
    """The pages' prior art for one layer step, as separate PyTorch launches
    whose intermediates all round-trip HBM ("Flash-dLLM: I/O-Aware KV Caching
    and Parallel Decoding for Fast, Memory-Efficient Diffusion LLMs", ai4snews
    summary, paragraph 1: before Flash-Cache the per-layer cache update was
    a chain of separate kernel launches): a cuBLAS GEMM x Wqkv, RoPE as
    elementwise ops, index_put_ of k and v into the paged pools, a gather of
    every sequence's keys and values through the block table, then scores,
    masked softmax and P V on a padded batch, and the attention mass from
    the probabilities. Same inputs, pool layout and results (within the
    parity bar) as the fused step; it exists only to measure what the fusion
    saves. The projection and the scores take bf16 operands with fp32
    results (cuBLAS); RoPE runs in double and rounds q and k to bf16 once,
    as in the fused step; P V runs in fp32 with TF32 allowed, which is exact
    for the bf16-valued v and rounds P to 11 bits.

    The padded shapes and the row / key index tensors depend only on cu_rows
    and seq_lens (host metadata, as in the fused path) and are built once;
    everything that depends on the device inputs (positions, slots, views,
    block table) is computed on the device in every step."""

    def __init__(self, spec, meta, device):
        sh = spec.shape
        self.sh, self.meta, self.dev = sh, meta, device
        D, ps = sh.head_dim, sh.page_size
        half = D // 2
        inv = np.float64(np.float32(sh.rope_theta)) ** (-2.0 * np.arange(half) / D)
        phi = np.arange(meta.max_position, dtype=np.float64)[:, None] * inv[None, :]
        self.cos = torch.from_numpy(np.cos(phi)).to(device)
        self.sin = torch.from_numpy(np.sin(phi)).to(device)
        B = meta.batch
        cu = meta.cu_rows
        n = np.diff(cu)
        self.Rmax = max(1, int(n.max()))
        kb = [max(int(meta.seq_lens[b]), int(meta.slots[cu[b]:cu[b + 1]].max()) + 1 if n[b] else 0)
              for b in range(B)]
        self.Kmax = max(1, max(kb))
        rowidx = np.full((B, self.Rmax), -1, np.int64)
        rowb = np.zeros(meta.total_rows, np.int64)
        for b in range(B):
            rowidx[b, :n[b]] = np.arange(cu[b], cu[b + 1])
            rowb[cu[b]:cu[b + 1]] = b
        kslot = np.tile(np.arange(self.Kmax, dtype=np.int64), (B, 1))
        kvalid = kslot < np.array(kb)[:, None]
        wgt = np.where(n > 0, 1.0 / np.maximum(n, 1) / sh.n_heads, 0.0)
        self.rowvalid = torch.from_numpy(rowidx >= 0).to(device)
        self.rowidx = torch.from_numpy(np.maximum(rowidx, 0)).to(device)
        self.rowb = torch.from_numpy(rowb).to(device)
        self.kslot = torch.from_numpy(kslot).to(device)
        self.kvalid = torch.from_numpy(kvalid).to(device)
        self.seq_lens = torch.from_numpy(meta.seq_lens.astype(np.int64)).to(device)
        self.wgt = torch.from_numpy(wgt.astype(np.float32)).to(device)
        self.scale = 1.0 / float(np.sqrt(D))

    def _rope(self, u, c, s):
        """Rotate-half RoPE in double from double tables, returned as bf16
        rounded once: double -> float with round-to-odd (truncate toward
        zero, set the last bit when inexact), then float -> bf16 to nearest
        even, which together round the double to the nearest bf16 (Boldo and
        Melquiond, "When double rounding is odd")."""
        half = self.sh.head_dim // 2
        u = u.double()
        a, b = u[..., :half], u[..., half:]
        d = torch.cat([a * c - b * s, b * c + a * s], dim=-1)
        f = d.float()
        away = f.double().abs() > d.abs()
        fb = f.view(torch.int32)
        fb = torch.where(away, fb - 1, fb)                 # toward zero
        f = fb.view(torch.float32)
        inexact = f.double() != d
        f = torch.where(inexact, (f.view(torch.int32) | 1).view(torch.float32), f)
        return f.to(torch.bfloat16)

    def step(self, layer, k_pool, v_pool, x, w, pos, slots, view, bt, out, mass):
        torch.cuda.nvtx.range_push("unfused_layer_step")
        self._step(layer, k_pool, v_pool, x, w, pos, slots, view, bt, out, mass)
        torch.cuda.nvtx.range_pop()

    def _step(self, layer, k_pool, v_pool, x, w, pos, slots, view, bt, out, mass):
        sh, meta = self.sh, self.meta
        H, nh, D, ps = sh.hidden, sh.n_heads, sh.head_dim, sh.page_size
        R, B = meta.total_rows, meta.batch
        bf = torch.bfloat16
        # 1. projection (cuBLAS, bf16 in, fp32 out so that q and k are rounded
        # once, after RoPE, as in the fused step), q, k, v through HBM
        qkv = torch.mm(x, w, out_dtype=torch.float32) if x.is_cuda else x.float() @ w.float()
        q = qkv[:, :H].view(R, nh, D)
        k = qkv[:, H:2 * H].view(R, nh, D)
        v = qkv[:, 2 * H:].view(R, nh, D)
        # 2. RoPE (elementwise launches)
        p = pos.long()
        c = self.cos[p][:, None, :]
        s = self.sin[p][:, None, :]
        qr = self._rope(q, c, s)
        kr = self._rope(k, c, s)
        # 3. cache write through the block table (index_put_)
        sl = slots.long()
        btl = bt.long()
        page = btl[self.rowb, sl // ps]
        off = sl % ps
        kp, vp = k_pool[layer], v_pool[layer]
        kp[page, :, off] = kr
        vp[page, :, off] = v.to(bf)
        # 4. gather every sequence's keys / values (padded batch)
        ks = self.kslot
        kpage = btl.gather(1, torch.clamp(ks // ps, max=btl.shape[1] - 1))
        kpage = torch.where(self.kvalid, kpage, torch.zeros_like(kpage))
        K = kp[kpage, :, ks % ps]                     # [B, Kmax, nh, D]
        V = vp[kpage, :, ks % ps]
        Q = qr[self.rowidx]                           # [B, Rmax, nh, D]
        # 5. visibility: context slots, plus own-view fresh slots at earlier
        # or equal positions
        rv = view.long()[self.rowidx]
        rp = p[self.rowidx]
        wv = torch.full((B, self.Kmax), -1, dtype=torch.long, device=self.dev)
        wp = torch.zeros((B, self.Kmax), dtype=torch.long, device=self.dev)
        wv[self.rowb, sl] = view.long()
        wp[self.rowb, sl] = p
        ctx = ks < self.seq_lens[:, None]
        own = (wv[:, None, :] == rv[:, :, None]) & (rv[:, :, None] != 0) & \
              (wp[:, None, :] <= rp[:, :, None])
        vis = (ctx[:, None, :] | own) & self.kvalid[:, None, :] & self.rowvalid[:, :, None]
        # 6. scores, masked softmax, P V
        Qb = Q.permute(0, 2, 1, 3).reshape(B * nh, self.Rmax, D)
        Kb = K.permute(0, 2, 3, 1).reshape(B * nh, D, self.Kmax)
        S = (torch.bmm(Qb, Kb, out_dtype=torch.float32) if Qb.is_cuda
             else torch.bmm(Qb.float(), Kb.float()))
        S = S.view(B, nh, self.Rmax, self.Kmax) * self.scale
        S = S.masked_fill(~vis[:, None], float("-inf"))
        P = torch.nan_to_num(torch.softmax(S, dim=-1), nan=0.0)
        O = torch.matmul(P, V.permute(0, 2, 1, 3).float())    # [B, nh, Rmax, D]
        o = O.permute(0, 2, 1, 3).reshape(B, self.Rmax, H)
        out[self.rowidx[self.rowvalid]] = o[self.rowvalid]
        # 7. attention mass: mean over heads and rows
        if mass is not None:
            m = P.sum(dim=(1, 2)) * self.wgt[:, None]
            mass.zero_()
            mass[:, :self.Kmax] = m


# ------------------------------------------------------------------ CPU baseline
_ORACLE_INPUTS = {}


def oracle_inputs(spec, meta, seed):
    key = (spec.name, seed)
    if key not in _ORACLE_INPUTS:
        x = W.make_x(spec, meta, seed)
        w = W.make_w(spec, seed)
        kp, vp = W.make_pools(spec, meta, seed, n_layers=1)
        _ORACLE_INPUTS[key] = (W.bits_np(x), W.bits_np(w), W.bits_np(kp), W.bits_np(vp))
    return _ORACLE_INPUTS[key]


def oracle_sample(spec, meta, seed, budget_s=12.0):
    """Times the CPU oracle on a bounded sample of the workload: the first
    sequences of layer 0 (as many as fit the time budget). Returns
    (rows/s, description, threads)."""
    sys.path.insert(0, ROOT)
    from oracle import oracle as O
    xb, wb, kb, vb = oracle_inputs(spec, meta, seed)
    total_rows = 0
    total_t = 0.0
    nseq = 0
    b = 0
    while b < meta.batch and total_t < budget_s:
        r0, r1 = int(meta.cu_rows[b]), int(meta.cu_rows[b + 1])
        cu = np.array([0, r1 - r0], np.int32)
        t0 = time.perf_counter()
        O.layer_step(spec.shape, kb, vb, 0, xb[r0:r1], wb, meta.positions[r0:r1], meta.slots[r0:r1], cu,
                     meta.seq_lens[b:b + 1], meta.block_table[b:b + 1], meta.view[r0:r1])
        total_t += time.perf_counter() - t0
        total_rows += r1 - r0
        nseq += 1
        b += 1
    try:
        from threadpoolctl import threadpool_info
        threads = max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count() or 1
    desc = (f"oracle (numpy float64) on {nseq} of {meta.batch} sequences of layer 0 "
            f"({total_rows} query rows), one sequence per call, {total_t:.1f} s")
    return total_rows / total_t, desc, threads


def e2e_measure(wl: Workload, steps: int):
    """Same metric through the public API with host buffers: per step the
    inputs (x of every layer, positions, slots, views, block table) are copied
    from pinned host memory, and out, attn_mass and the tracked set are read
    back; all inside the timed region.

    Returns (pipelined ms, serial ms, h2d bytes, d2h bytes) per step.
    Serial: copy in, compute and copy out one after another on one stream.
    Pipelined, as a serving loop runs it: uploads on one stream and
    downloads on another, with device and host buffers doubled, so that step
    i+1's inputs go up and step i-1's outputs come down while step i
    computes. Every step still moves all of its bytes inside the timed
    region."""
    fd = wl.fd
    m = wl.meta
    NB = 2
    hx = [x.cpu().pin_memory() for x in wl.x]
    dmeta0 = (wl.pos, wl.slots, wl.view, wl.bt)
    hmeta = [t.cpu().pin_memory() for t in dmeta0]
    bufs = []
    # a chained stack's result is the final residual stream (bf16)
    res_like = wl.xs if wl.chained else wl.out
    for _ in range(NB):
        bufs.append({
            "x": [torch.empty_like(x) for x in wl.x],
            "meta": [torch.empty_like(t) for t in dmeta0],
            "out": torch.empty_like(res_like), "mass": torch.empty_like(wl.mass),
            "tr": torch.empty_like(wl.tracked),
            "hout": torch.empty(res_like.shape, dtype=res_like.dtype).pin_memory(),
            "hmass": torch.empty(wl.mass.shape, dtype=wl.mass.dtype).pin_memory(),
            "htr": torch.empty(wl.tracked.shape, dtype=wl.tracked.dtype).pin_memory(),
            "ev_in": torch.cuda.Event(), "ev_comp": torch.cuda.Event(), "ev_out": torch.cuda.Event(),
        })
    h2d = sum(x.numel() * x.element_size() for x in hx) + sum(
        t.numel() * t.element_size() for t in hmeta)
    d2h = sum(t.numel() * t.element_size() for t in (bufs[0]["hout"], bufs[0]["hmass"],
                                                      bufs[0]["htr"]))
    comp = torch.cuda.current_stream()
    s_in = torch.cuda.Stream()
    s_out = torch.cuda.Stream()

    def compute(b, stream):
        pos, slots, view, bt = b["meta"]
        if wl.chained:
            wl.stack.run(m.cu_rows, m.seq_lens, b["x"][0], pos, bt, view, slots, b["mass"],
                         stream=stream, x_out=b["out"])
            fd.fdllm_select_tracked(b["mass"], wl.seq_lens_d, m.track_k, wl.ex_cu, wl.ex_sl,
                                    b["tr"], stream=stream)
            return
        for l in range(wl.n_layers):
            fd.fdllm_layer_step(wl.cache.handle, l, m.cu_rows, m.seq_lens, m.max_blocks, b["x"][l],
                                wl.w[l], pos, bt, view, b["out"], b["mass"], slots, stream=stream)
        fd.fdllm_select_tracked(b["mass"], wl.seq_lens_d, m.track_k, wl.ex_cu, wl.ex_sl, b["tr"],
                                stream=stream)

    def one_serial():
        b = bufs[0]
        for l in range(len(wl.x)):
            b["x"][l].copy_(hx[l], non_blocking=True)
        for d, h in zip(b["meta"], hmeta):
            d.copy_(h, non_blocking=True)
        compute(b, comp)
        b["hout"].copy_(b["out"], non_blocking=True)
        b["hmass"].copy_(b["mass"], non_blocking=True)
        b["htr"].copy_(b["tr"], non_blocking=True)

    def one_pipelined(i):
        b = bufs[i % NB]
        if i >= NB:   # step i-NB no longer reads these inputs
            s_in.wait_event(b["ev_comp"])
        with torch.cuda.stream(s_in):
            for l in range(len(wl.x)):
                b["x"][l].copy_(hx[l], non_blocking=True)
            for d, h in zip(b["meta"], hmeta):
                d.copy_(h, non_blocking=True)
            b["ev_in"].record(s_in)
        comp.wait_event(b["ev_in"])
        if i >= NB:   # step i-NB's outputs have come down
            comp.wait_event(b["ev_out"])
        compute(b, comp)
        b["ev_comp"].record(comp)
        s_out.wait_event(b["ev_comp"])
        with torch.cuda.stream(s_out):
            b["hout"].copy_(b["out"], non_blocking=True)
            b["hmass"].copy_(b["mass"], non_blocking=True)
            b["htr"].copy_(b["tr"], non_blocking=True)
            b["ev_out"].record(s_out)

    def timed(run):
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(steps):
            run(i)
        comp.wait_stream(s_in)
        comp.wait_stream(s_out)
        e1.record(comp)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    for _ in range(3):
        one_serial()
    serial_ms = timed(lambda i: one_serial())
    for i in range(3):
        one_pipelined(i)
    pipe_ms = timed(one_pipelined)
    return pipe_ms, serial_ms, h2d, d2h


# ------------------------------------------------------------------ main arms
def run_reference(args):
    """The reference arm: the CPU oracle as it stands, on the host cores.
    Every step is one bounded sample of the workload (the first sequences
    of layer 0, as many as fit about 20 s / (steps + warm-up) of oracle
    time, at least one), and every step is timed whole, so ms_per_step x
    steps is the time the run spent in timed steps."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from oracle import oracle as O
    spec = W.get_spec(args.workload)
    meta = W.make_meta(spec, args.seed)
    xb, wb, kb, vb = oracle_inputs(spec, meta, args.seed)
    budget = max(1.0, 20.0 / max(1, args.steps + args.warmup))

    def one_seq(b):
        r0, r1 = int(meta.cu_rows[b]), int(meta.cu_rows[b + 1])
        O.layer_step(spec.shape, kb, vb, 0, xb[r0:r1], wb, meta.positions[r0:r1],
                     meta.slots[r0:r1], np.array([0, r1 - r0], np.int32), meta.seq_lens[b:b + 1],
                     meta.block_table[b:b + 1], meta.view[r0:r1])
        return r1 - r0

    # calibrate the sample on the first warm-up step
    t0 = time.perf_counter()
    one_seq(0)
    per_seq = time.perf_counter() - t0
    n_s = int(max(1, min(meta.batch, budget // max(per_seq, 1e-6))))
    rows = int(meta.cu_rows[n_s] - meta.cu_rows[0])
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        for b in range(n_s):
            one_seq(b)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    ms = 1000.0 * float(np.mean(times))
    value = rows / (ms / 1000.0)
    desc = (f"oracle (numpy float64) per step on the first {n_s} of {meta.batch} sequences of "
            f"layer 0 ({rows} of {meta.total_rows} query rows), one sequence per call; "
            f"{ms / 1000.0:.2f} s per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_block(spec, meta, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([int(d.get("num_threads", 1)) for d in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def config_block(spec, meta, args):
    sh = spec.shape
    return {"workload": spec.name, "layers": sh.n_layers, "batch": meta.batch,
            "query_rows_per_layer": meta.total_rows,
            "context_slots": [int(meta.seq_lens.min()), int(meta.seq_lens.max())],
            "hidden": sh.hidden, "heads": sh.n_heads, "head_dim": sh.head_dim,
            "page_size": sh.page_size, "track_k": meta.track_k,
            "l2": "flushed between timed steps (256 MB write)", "parallelism": f"replicas x{args.gpus}",
            "seed": args.seed}


def roofline_of(spec, meta, kern_s, peaks, peak_src, kernel_name, traffic=None):
    """Roofline of one layer step: the slower of algorithmic bytes over the
    measured HBM copy rate and algorithmic FLOPs over the measured (burst)
    bf16 rate, against the measured time of one layer step."""
    byt, fl = W.algorithmic_bytes_flops(spec, meta)
    t_hbm = byt / (peaks["hbm_gbs"] * 1e9)
    t_tc = fl / (peaks["bf16_tflops"] * 1e12)
    bound = "tensor" if t_tc >= t_hbm else "hbm"
    if bound == "tensor":
        achieved, peak, unit = fl / kern_s / 1e12, peaks["bf16_tflops"], "TFLOP/s"
    else:
        achieved, peak, unit = byt / kern_s / 1e9, peaks["hbm_gbs"], "GB/s"
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
            "traffic": traffic, "peak_source": f"{peak_src} (burst)", "kernel": kernel_name,
            "kernel_us": kern_s * 1e6, "algorithmic_bytes": byt, "algorithmic_flops": fl,
            "hbm_gbs_achieved": byt / kern_s / 1e9,
            "roofline_us": max(t_hbm, t_tc) * 1e6, "frac_of_roofline": max(t_hbm, t_tc) / kern_s}


def hold_device(us: float = 1000.0):
    """Keeps the stream busy for about `us` microseconds (a device-side spin,
    outside the timed region) so that the host has queued the whole step
    before the start event is reached: the events then time the GPU work,
    not host planning and launch latency. The end-to-end figure keeps the
    host in its timed region."""
    sleep = getattr(torch.cuda, "_sleep", None)
    if sleep is not None:
        sleep(int(us * 2000))      # cycles at about 2 GHz


def time_steps(step_fn, steps, warmup, flush, ev_layers=True):
    """Runs `warmup` untimed steps, then `steps` steps bracketed by CUDA
    events on the current stream with an L2 flush between them (outside the
    events). step_fn(ev) runs one step and returns its kernel launches; with
    ev = (start, end) it records them around its first-layer step and last
    layer step. Returns (per-step ms list, per-step layer-span ms list,
    launches)."""
    for _ in range(warmup):
        step_fn(None)
    torch.cuda.synchronize()
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ev_ls = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ev_le = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    launches = 0
    for i in range(steps):
        flush.fill_(i & 0xFF)
        hold_device()
        ev_s[i].record()
        launches += step_fn((ev_ls[i], ev_le[i]) if ev_layers else None)
        ev_e[i].record()
    torch.cuda.synchronize()
    step_ms = [ev_s[i].elapsed_time(ev_e[i]) for i in range(steps)]
    layer_ms = [ev_ls[i].elapsed_time(ev_le[i]) for i in range(steps)] if ev_layers else step_ms
    return step_ms, layer_ms, launches


def measure_workload(name, seed, dev, steps, warmup, flush, peaks, peak_src, cpu_budget):
    """Device-timed throughput of one layer workload plus its roofline and
    an oracle CPU sample (for the per-workload table of the default run)."""
    wl = Workload(name, seed, dev)
    spec, meta = wl.spec, wl.meta
    step_ms, layer_ms, launches = time_steps(lambda ev: wl.step(ev=ev, layer_span=True), steps,
                                             warmup, flush)
    wl.cache.check()
    nl = spec.shape.n_layers
    ms = float(np.mean(step_ms))
    kern_s = float(np.mean(layer_ms)) / nl / 1000.0
    roof = roofline_of(spec, meta, kern_s, peaks, peak_src,
                       "fdllm_layer_step (fused step kernel + mass reduce), mean over layers")
    cpu = None
    if cpu_budget > 0:
        v, desc, threads = oracle_sample(spec, meta, seed, budget_s=cpu_budget)
        cpu = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc}
    res = {"value": meta.total_rows / (ms / 1000.0), "unit": UNIT,
           "layer_steps_per_s": nl / (ms / 1000.0), "ms_per_step": ms, "steps": steps,
           "dtype": spec.shape.dtype, "gpu_launches": launches,
           "config": config_block(spec, meta, argparse.Namespace(gpus=1, seed=seed)),
           "roofline": {k: roof[k] for k in ("bound", "achieved", "peak", "unit", "frac", "kernel_us",
                                              "roofline_us", "algorithmic_bytes",
                                              "algorithmic_flops")},
           "cpu_baseline": cpu}
    wl.cache.close()
    del wl
    torch.cuda.empty_cache()
    return res


PER_WORKLOAD = ("tiny_f32", "llada8b_b1", "two_view_b8", "stacked32_b4", "stacked32_b4_chained")


def run_native(args):
    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, peak_src = load_peaks()
    wl = Workload(args.workload, args.seed + rank, dev)
    spec, meta = wl.spec, wl.meta
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    for _ in range(args.warmup):
        wl.step()
    wl.cache.check()
    torch.cuda.synchronize()

    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    step_ms, layer_ms, launches = time_steps(lambda ev: wl.step(ev=ev), args.steps, 0, flush)
    barrier()
    t_wall1 = time.time()
    if sampler:
        sampler.mark(t_wall0, t_wall1)
        time.sleep(0.25)
        sampler.stop()
    wl.cache.check()
    total_ms_local = float(sum(step_ms))
    total_ms, _, value = aggregate(total_ms_local, meta.total_rows * args.steps, dev)

    # roofline of the dominant kernel (the fused layer step, layer 0)
    kern_s = float(np.mean(layer_ms)) / 1000.0
    traffic = args.traffic if args.traffic is not None else captured_traffic(spec.name)
    roof = roofline_of(spec, meta, kern_s, peaks, peak_src,
                       "fdllm_layer_step (fused step kernel + mass reduce), layer 0", traffic)
    if traffic is not None:
        roof["traffic_source"] = CAPTURED_TRAFFIC[spec.name]["source"]

    e2e_ms, serial_ms, h2d, d2h = e2e_measure(wl, max(10, min(args.steps, 200)))
    e2e_ms_max = reduce_max(e2e_ms, dev)
    serial_ms_max = reduce_max(serial_ms, dev)
    e2e_value = meta.total_rows * world / (e2e_ms_max / 1000.0)
    wl.cache.close()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, threads = oracle_sample(spec, meta, args.seed + rank)
        cpu = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc}

    # the other layer workloads, each device-timed with its own roofline and
    # oracle sample (single-GPU runs of the default workload only)
    per = None
    if world == 1 and not args.no_per_workload and args.workload == "b32_divergent":
        per = {}
        for name in PER_WORKLOAD:
            per[name] = measure_workload(name, args.seed, dev, min(args.steps, 20), 3, flush, peaks,
                                         peak_src, 0.0 if args.no_cpu_baseline else 4.0)

    clocks = sampler.summary() if sampler else None
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": spec.shape.dtype, "data": "synthetic",
        "config": config_block(spec, meta, argparse.Namespace(gpus=world, seed=args.seed)),
        "layer_steps_per_s": value / meta.total_rows * spec.shape.n_layers,
        "roofline": roof, "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms_max, "copies": "pipelined (upload, compute, download streams)",
                "serial_value": meta.total_rows * world / (serial_ms_max / 1000.0),
                "serial_ms_per_step": serial_ms_max},
        "gpu_launches": launches, "clocks": clocks,
    }
    if per is not None:
        line["per_workload"] = per
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_unfused(args):
    """The unfused PyTorch arm (the pages' prior art) on a layer workload:
    same inputs and metric; printed as one JSON line with impl "unfused"."""
    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
    dev = torch.device("cuda", torch.cuda.current_device())
    torch.backends.cuda.matmul.allow_tf32 = True
    peaks, peak_src = load_peaks()
    spec = W.get_spec(args.workload)
    if spec.shape.dtype != "bf16":
        print(json.dumps({"impl": "unfused", "unavailable": "the unfused arm serves bf16 workloads"}))
        return 0
    meta = W.make_meta(spec, args.seed + rank)
    sh = spec.shape
    nl = sh.n_layers
    xs = [W.make_x(spec, meta, args.seed + rank, layer=l, device=dev) for l in range(nl)]
    ws = [W.make_w(spec, args.seed + rank, layer=l, device=dev) for l in range(nl)]
    kp, vp = W.make_pools(spec, meta, args.seed + rank, device=dev)
    u = UnfusedStep(spec, meta, dev)
    pos = torch.from_numpy(meta.positions).to(dev)
    slots = torch.from_numpy(meta.slots).to(dev)
    view = torch.from_numpy(meta.view).to(dev)
    bt = torch.from_numpy(meta.block_table).to(dev)
    out = torch.empty(meta.total_rows, sh.hidden, dtype=torch.float32, device=dev)
    mass = torch.empty(meta.batch, meta.max_blocks * sh.page_size, dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(ev):
        for l in range(nl):
            if ev is not None and l == 0:
                ev[0].record()
            u.step(l, kp, vp, xs[l], ws[l], pos, slots, view, bt, out, mass)
            if ev is not None and l == nl - 1:
                ev[1].record()
        return 0

    # kernels per step, counted once with the torch profiler (untimed; left
    # out under an external profiler, which the torch profiler would clash with)
    step(None)
    torch.cuda.synchronize()
    per_step = None
    if not args.no_launch_count:
        from torch.profiler import ProfilerActivity, profile
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            step(None)
            torch.cuda.synchronize()
        per_step = sum(1 for e in prof.events() if e.device_type.name == "CUDA")
    step_ms, layer_ms, _ = time_steps(step, args.steps, args.warmup, flush)
    ms = float(np.mean(step_ms))
    roof = roofline_of(spec, meta, float(np.mean(layer_ms)) / nl / 1000.0, peaks, peak_src,
                       "unfused PyTorch layer step (all its kernels), mean over layers")
    line = {"impl": "unfused", "metric": METRIC, "value": meta.total_rows / (ms / 1000.0),
            "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": config_block(spec, meta, argparse.Namespace(gpus=1, seed=args.seed)),
            "layer_steps_per_s": nl / (ms / 1000.0), "roofline": roof,
            "gpu_launches": per_step * args.steps if per_step is not None else None,
            "note": "torch/cuBLAS kernels, not this library's; selection not included"}
    if rank == 0:
        print(json.dumps(line))
    return 0


# ------------------------------------------------------------------ Flash-Verify
VERIFY_METRIC = "Flash-Verify acceptance block-positions/s; achieved HBM GB/s and % of roofline (1×B200)"
VERIFY_UNIT = "positions/s"


def verify_bytes(spec):
    """Algorithmic bytes of one acceptance step: the logits once, the drafted
    tokens, predictions and confidences (4 bytes each per row), cu_rows and
    the accepted lengths."""
    s = 2 if spec.dtype == "bf16" else 4
    R = spec.batch * spec.rows
    return R * spec.vocab * s + R * 12 + (spec.batch + 1) * 4 + spec.batch * 4


def verify_oracle_sample(spec, logits_cpu, cu, draft, budget_s):
    from oracle import oracle as O
    bits = W.bits_np(logits_cpu)
    t0 = time.perf_counter()
    rows = 0
    nseq = 0
    while nseq < spec.batch and time.perf_counter() - t0 < budget_s:
        r0, r1 = int(cu[nseq]), int(cu[nseq + 1])
        pred, conf = O.verify_rows(bits[r0:r1], spec.dtype)
        O.verify_accept(pred, conf, draft[r0:r1], np.array([0, r1 - r0]), spec.tau)
        rows += r1 - r0
        nseq += 1
    dt = time.perf_counter() - t0
    desc = (f"oracle (numpy float64) on {nseq} of {spec.batch} sequences ({rows} positions x "
            f"{spec.vocab} logits), one sequence per call, {dt:.1f} s")
    return rows / dt, desc


def verify_config(spec, args, world):
    return {"workload": spec.name, "batch": spec.batch, "positions_per_sequence": spec.rows,
            "vocab": spec.vocab, "logits": spec.dtype, "tau": spec.tau,
            "l2": "flushed between timed steps (256 MB write)", "parallelism": f"replicas x{world}",
            "seed": args.seed}


def run_verify(args):
    rank, world, local = dist_env()
    spec = W.VERIFY_WORKLOADS[args.workload]
    R = spec.batch * spec.rows
    if args.impl == "reference":
        if rank != 0:
            return 0
        logits, cu, draft = W.make_verify(spec, args.seed)
        budget = max(2.0, 20.0 / max(1, args.steps + args.warmup))
        vals, desc = [], ""
        for i in range(args.warmup + args.steps):
            v, desc = verify_oracle_sample(spec, logits, cu, draft, budget)
            if i >= args.warmup:
                vals.append(v)
        value = float(np.mean(vals))
        line = {"impl": "reference", "metric": VERIFY_METRIC, "value": value, "unit": VERIFY_UNIT,
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1000.0 * R / value, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": verify_config(spec, args, args.gpus),
                "cpu_baseline": {"value": value, "unit": VERIFY_UNIT, "cores": os.cpu_count() or 1,
                                 "kind": "oracle", "sample": desc},
                "e2e": {"value": value, "unit": VERIFY_UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0
    import kv_cache_attention_flash_b200 as fd
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, peak_src = load_peaks()
    logits, cu, draft = W.make_verify(spec, args.seed + rank, device=dev)
    cu_d = torch.from_numpy(cu).to(dev)
    draft_d = torch.from_numpy(draft).to(dev)
    pred = torch.empty(R, dtype=torch.int32, device=dev)
    conf = torch.empty(R, dtype=torch.float32, device=dev)
    nacc = torch.empty(spec.batch, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        fd.fdllm_verify_accept(logits, cu_d, draft_d, spec.tau, pred, conf, nacc)
        return fd.fdllm_last_launch_count()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    launches = 0
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        hold_device()
        ev_s[i].record()
        launches += step()
        ev_e[i].record()
    torch.cuda.synchronize()
    barrier()
    t_wall1 = time.time()
    if sampler:
        sampler.mark(t_wall0, t_wall1)
        time.sleep(0.25)
        sampler.stop()
    step_ms = [ev_s[i].elapsed_time(ev_e[i]) for i in range(args.steps)]
    total_ms, _, value = aggregate(float(sum(step_ms)), R * args.steps, dev)
    byt = verify_bytes(spec)
    kern_s = float(np.mean(step_ms)) / 1000.0
    achieved = byt / kern_s / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": None, "peak_source": f"{peak_src} (burst)",
            "kernel": "fdllm_verify_accept (row reduction + acceptance scan)",
            "kernel_us": kern_s * 1e6, "algorithmic_bytes": byt}
    # end to end: logits from pinned host memory in, predictions,
    # confidences and accepted lengths out, every step
    hlog = logits.cpu().pin_memory()
    hpred = torch.empty(R, dtype=torch.int32).pin_memory()
    hconf = torch.empty(R, dtype=torch.float32).pin_memory()
    hnacc = torch.empty(spec.batch, dtype=torch.int32).pin_memory()
    dlog = torch.empty_like(logits)
    h2d = hlog.numel() * hlog.element_size()
    d2h = R * 8 + spec.batch * 4
    n_e2e = max(10, min(args.steps, 200))

    def one():
        dlog.copy_(hlog, non_blocking=True)
        fd.fdllm_verify_accept(dlog, cu_d, draft_d, spec.tau, pred, conf, nacc)
        hpred.copy_(pred, non_blocking=True)
        hconf.copy_(conf, non_blocking=True)
        hnacc.copy_(nacc, non_blocking=True)

    for _ in range(3):
        one()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n_e2e):
        one()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1) / n_e2e, dev)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc = verify_oracle_sample(spec, logits.cpu(), cu, draft, 12.0)
        cpu = {"value": v, "unit": VERIFY_UNIT, "cores": os.cpu_count() or 1, "kind": "oracle",
               "sample": desc}
    line = {
        "metric": VERIFY_METRIC, "value": value, "unit": VERIFY_UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": spec.dtype,
        "data": "synthetic", "config": verify_config(spec, args, world), "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": R * world / (e2e_ms / 1000.0), "unit": VERIFY_UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches, "clocks": sampler.summary() if sampler else None,
    }
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


OPROJ_METRIC = "output projection rows/s; achieved TFLOP/s and % of roofline (1\u00d7B200)"
OPROJ_UNIT = "rows/s"


def oproj_oracle_sample(o_cpu, w_cpu, budget_s):
    """The oracle's y = o W_o on whole row blocks of 64 until the budget."""
    from oracle import oracle as O
    ob, wb = W.bits_np(o_cpu), W.bits_np(w_cpu)
    rows = 0
    t0 = time.perf_counter()
    while rows < ob.shape[0] and time.perf_counter() - t0 < budget_s:
        O.oproj(ob[rows:rows + 64], wb)
        rows += min(64, ob.shape[0] - rows)
    dt = time.perf_counter() - t0
    desc = (f"oracle (numpy float64 matmul) on {rows} of {ob.shape[0]} rows x "
            f"{ob.shape[1]} x {wb.shape[1]}, 64 rows per call, {dt:.1f} s")
    return rows / dt, desc


def oproj_threads():
    try:
        from threadpoolctl import threadpool_info
        return max(int(i.get("num_threads", 1)) for i in threadpool_info()) or 1
    except Exception:
        return os.cpu_count() or 1


def run_oproj(args):
    """The output projection y = o W_o alone: one tcgen05 GEMM per step."""
    rank, world, local = dist_env()
    spec = W.OPROJ_WORKLOADS[args.workload]
    R, H = spec.rows, spec.hidden
    config = {"workload": spec.name, "rows": R, "hidden": H, "operands": "bf16 in, bf16 out",
              "l2": "flushed between timed steps (256 MB write)",
              "parallelism": f"replicas x{world}", "seed": args.seed}
    if args.impl == "reference":
        if rank != 0:
            return 0
        o, w = W.make_oproj(spec, args.seed)
        budget = max(2.0, 20.0 / max(1, args.steps + args.warmup))
        vals, desc = [], ""
        for i in range(args.warmup + args.steps):
            v, desc = oproj_oracle_sample(o, w, budget)
            if i >= args.warmup:
                vals.append(v)
        value = float(np.mean(vals))
        print(json.dumps({
            "impl": "reference", "metric": OPROJ_METRIC, "value": value, "unit": OPROJ_UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * R / value, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "cpu_baseline": {"value": value, "unit": OPROJ_UNIT, "cores": oproj_threads(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": OPROJ_UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}))
        return 0
    import kv_cache_attention_flash_b200 as fd
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks, peak_src = load_peaks()
    o, w = W.make_oproj(spec, args.seed + rank, device=dev)
    y = torch.empty(R, H, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        fd.fdllm_oproj(o, w, y)
        return fd.fdllm_last_launch_count()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    launches = 0
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        hold_device()
        ev_s[i].record()
        launches += step()
        ev_e[i].record()
    torch.cuda.synchronize()
    barrier()
    t_wall1 = time.time()
    if sampler:
        sampler.mark(t_wall0, t_wall1)
        time.sleep(0.25)
        sampler.stop()
    step_ms = [ev_s[i].elapsed_time(ev_e[i]) for i in range(args.steps)]
    total_ms, _, value = aggregate(float(sum(step_ms)), R * args.steps, dev)
    kern_s = float(np.mean(step_ms)) / 1000.0
    fl = 2.0 * R * H * H
    byt = 2.0 * (R * H + H * H + R * H)
    achieved = fl / kern_s / 1e12
    peak = peaks["bf16_tflops"]
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": None, "peak_source": f"{peak_src} (burst)",
            "kernel": "fdllm_oproj (tcgen05 GEMM)", "kernel_us": kern_s * 1e6,
            "algorithmic_flops": fl, "algorithmic_bytes": byt,
            "hbm_gbs_achieved": byt / kern_s / 1e9,
            "roofline_us": max(byt / (peaks["hbm_gbs"] * 1e9), fl / (peak * 1e12)) * 1e6}
    # end to end: o up from pinned host memory, y down, every step
    ho = o.cpu().pin_memory()
    hy = torch.empty(R, H, dtype=torch.bfloat16).pin_memory()
    do = torch.empty_like(o)
    n_e2e = max(10, min(args.steps, 200))

    def one():
        do.copy_(ho, non_blocking=True)
        fd.fdllm_oproj(do, w, y)
        hy.copy_(y, non_blocking=True)

    for _ in range(3):
        one()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n_e2e):
        one()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1) / n_e2e, dev)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc = oproj_oracle_sample(o.cpu(), w.cpu(), 12.0)
        cpu = {"value": v, "unit": OPROJ_UNIT, "cores": oproj_threads(), "kind": "oracle",
               "sample": desc}
    line = {
        "metric": OPROJ_METRIC, "value": value, "unit": OPROJ_UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": config, "roofline": roof, "cpu_baseline": cpu,
        "e2e": {"value": R * world / (e2e_ms / 1000.0), "unit": OPROJ_UNIT,
                "h2d_bytes_per_step": R * H * 2, "d2h_bytes_per_step": R * H * 2,
                "ms_per_step": e2e_ms},
        "gpu_launches": launches, "clocks": sampler.summary() if sampler else None,
    }
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


DECODE_METRIC = "toy decode loop: decoded tokens/s (random weights; throughput only)"
DECODE_CONFIGS = {
    # LLaDA-8B layer shape, 4 chained layers, batch 8, 256-token prompt and
    # 256-token generation, 32-token window, 32 tracked tokens
    "decode_llada8b_4l": dict(hidden=4096, n_heads=32, head_dim=128, n_layers=4, batch=8,
                              prompt_len=256, gen_len=256, window=32, track_k=32, tau=0.5),
}


def run_decode(args):
    """The toy decode loop (kv_cache_attention_flash_b200.decode_loop): a
    chunked prefill, then decode steps until `steps` steps are timed (or
    every sequence finished). Timed with CUDA events around each step; the
    host work between steps (acceptance, next rows) is inside the timed
    span, as in a serving loop."""
    from kv_cache_attention_flash_b200.decode_loop import ToyDecodeLoop
    from kv_cache_attention_flash_b200.workloads import ToyConfig
    rank, world, local = dist_env()
    if args.impl != "native":
        print(json.dumps({"impl": args.impl, "unavailable": "the toy decode loop has one arm"}))
        return 0
    if world > 1:
        torch.cuda.set_device(local)
    cfg = ToyConfig(seed=args.seed + rank, **DECODE_CONFIGS[args.workload])
    loop = ToyDecodeLoop(cfg, "cuda")
    loop.prefill()
    for _ in range(args.warmup):
        loop.step()
    torch.cuda.synchronize()
    accepted, rows, times = 0, 0, []
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    for _ in range(args.steps):
        if loop.done():
            break
        r0 = loop.rows_done
        e0.record()
        acc, _, _ = loop.step()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
        accepted += int(acc.sum())
        rows += loop.rows_done - r0
    loop.cache.check()
    ms = float(np.mean(times))
    n = len(times)
    line = {"metric": DECODE_METRIC, "value": accepted / (sum(times) / 1000.0), "unit": "tokens/s",
            "n_gpus": 1, "steps": n, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic (random weights)",
            "config": {"workload": args.workload, **DECODE_CONFIGS[args.workload]},
            "query_rows_per_s": rows / (sum(times) / 1000.0),
            "accepted_per_step": accepted / max(n, 1)}
    if rank == 0:
        print(json.dumps(line))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="b32_divergent",
                    choices=sorted(W.WORKLOADS) + sorted(W.VERIFY_WORKLOADS) +
                    sorted(W.OPROJ_WORKLOADS) + sorted(DECODE_CONFIGS))
    ap.add_argument("--impl", default="native", choices=["native", "reference", "unfused"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per launch of the step kernel, when captured for this build")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-launch-count", action="store_true",
                    help="unfused arm: skip counting its kernels with the torch profiler")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip the table of the other layer workloads in the default run")
    ap.add_argument("--layers", type=int, default=None,
                    help="run a layer workload with this many layers (same per-layer shapes and "
                         "contexts; a small case of a deep stack for profiling)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.layers is not None:
        if args.workload not in W.WORKLOADS or args.layers < 1:
            ap.error("--layers takes a positive count and a layer workload")
        # the named workload with another layer count, for this run only
        s = W.WORKLOADS[args.workload]
        W.WORKLOADS[args.workload] = dataclasses.replace(
            s, shape=dataclasses.replace(s.shape, n_layers=args.layers))
        args.no_per_workload = True
        try:
            return _dispatch(args)
        finally:
            W.WORKLOADS[args.workload] = s
    return _dispatch(args)


def _dispatch(args):
    if args.workload in W.VERIFY_WORKLOADS:
        return run_verify(args)
    if args.workload in W.OPROJ_WORKLOADS:
        return run_oproj(args)
    if args.workload in DECODE_CONFIGS:
        return run_decode(args)
    if args.impl == "reference":
        return run_reference(args)
    if args.impl == "unfused":
        return run_unfused(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
