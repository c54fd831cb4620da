"""Seeded synthetic workloads for the Flash-dLLM per-layer step.

This module only draws inputs. It holds none of the step's arithmetic: no
projection, no rotary embedding, no attention, no rounding of results. Both
the CUDA path and the CPU oracle consume what it produces, so it is the one
piece of code they share.

The five workloads mirror the settings the Flash-dLLM pages describe for
LLaDA-1.5 serving ("Flash-dLLM: I/O-Aware KV Caching and Parallel Decoding
for Fast, Memory-Efficient Diffusion LLMs", ai4snews summary of the full
text, paragraphs 1-4): a single layer at LLaDA-8B shape, a batch of 32
sequences whose lengths and stages diverge, the Flash-Verify two-view block,
and a 32-layer stack. No public benchmark data is used; every tensor is
drawn from a seeded generator.

Recipe (all seeds fixed by the caller):
  * metadata (lengths, positions, stages, page permutation) from
    ``numpy.random.default_rng(seed)``;
  * x ~ N(0, 1), Wqkv ~ N(0, 0.02^2), drawn as float32 by a seeded
    ``torch.Generator`` and cast to the workload dtype (bf16 casts round to
    nearest even);
  * the pre-existing cache holds N(0, 1.28^2) values in the visible slots
    (1.28^2 ~= H * 0.02^2, the second moment of a projected key), a NaN bit
    pattern in every slot this step writes and in every page tail past the
    sequence's last slot, and random bits in spare pages.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np
import torch

BF16_NAN_BITS = 0x7FC1      # a quiet NaN that no arithmetic produces by itself
F32_NAN_BITS = 0x7FC00011


@dataclasses.dataclass(frozen=True)
class LayerShape:
    dtype: str            # "bf16" or "f32": x, Wqkv and the cache pools
    hidden: int
    n_heads: int
    head_dim: int
    page_size: int
    rope_theta: float
    n_layers: int = 1


@dataclasses.dataclass(frozen=True)
class WorkloadSpec:
    name: str
    shape: LayerShape
    batch: int
    kind: str                     # "window", "divergent", "two_view"
    ctx_len: int = 0              # fixed visible context (window / two_view)
    prompt_len: int = 0           # window start is drawn after the prompt
    ctx_min: int = 0              # divergent: L_b ~ U[ctx_min, ctx_max]
    ctx_max: int = 0
    window: int = 32
    # stack: layer l's x is the residual stream x_l + out_{l-1} W_o,{l-1}
    # (chained), or an independent seeded draw per layer (not chained)
    chained: bool = False
    tracked: int = 32             # tracked rows per update-stage sequence
    track_k: int = 32             # k of the next step's top-k selection
    view_rows: int = 32           # two_view: rows per view
    spare_pages: int = 4


LLADA8B = LayerShape("bf16", 4096, 32, 128, 64, 500000.0)

WORKLOADS: Dict[str, WorkloadSpec] = {
    # Tiny single layer, fp32; 64 prompt + 64 generated slots, 16-slot pages.
    "tiny_f32": WorkloadSpec("tiny_f32", LayerShape("f32", 256, 4, 64, 16, 10000.0),
                             batch=1, kind="window", ctx_len=128, prompt_len=64,
                             window=8, tracked=8, track_k=8, spare_pages=3),
    # LLaDA-8B-shaped layer, batch 1, 256 prompt + 512 generated slots.
    "llada8b_b1": WorkloadSpec("llada8b_b1", LLADA8B, batch=1, kind="window",
                               ctx_len=768, prompt_len=256, window=32, tracked=32, track_k=32),
    # Batch 32, L_b ~ U[256, 1024], half caching stage (window only), half
    # update stage (window + 32 tracked), pages permuted in the pool.
    "b32_divergent": WorkloadSpec("b32_divergent", LLADA8B, batch=32, kind="divergent",
                                  ctx_min=256, ctx_max=1024, window=32, tracked=32, track_k=32,
                                  spare_pages=8),
    # Flash-Verify two views: 32 draft + 32 mask rows at the same positions.
    "two_view_b8": WorkloadSpec("two_view_b8", LLADA8B, batch=8, kind="two_view",
                                ctx_len=1024, view_rows=32, track_k=32),
    # 32 stacked layers, batch 4, 8192 context slots, 32 window + 64 tracked.
    "stacked32_b4": WorkloadSpec("stacked32_b4", dataclasses.replace(LLADA8B, n_layers=32),
                                 batch=4, kind="window", ctx_len=8192, prompt_len=0,
                                 window=32, tracked=64, track_k=64),
    # the same stack chained: each layer's bf16 out goes through its output
    # projection into the residual stream that is the next layer's x
    "stacked32_b4_chained": WorkloadSpec("stacked32_b4_chained",
                                         dataclasses.replace(LLADA8B, n_layers=32), batch=4,
                                         kind="window", ctx_len=8192, prompt_len=0, window=32,
                                         tracked=64, track_k=64, chained=True),
}

# Small variants of the same structure (same code paths, oracle-sized).
SMALL_WORKLOADS: Dict[str, WorkloadSpec] = {
    "small_bf16_divergent": WorkloadSpec(
        "small_bf16_divergent", LayerShape("bf16", 512, 4, 128, 64, 500000.0),
        batch=6, kind="divergent", ctx_min=70, ctx_max=400, window=32, tracked=32,
        track_k=16, spare_pages=3),
    "small_bf16_two_view": WorkloadSpec(
        "small_bf16_two_view", LayerShape("bf16", 512, 4, 128, 64, 10000.0),
        batch=3, kind="two_view", ctx_len=200, view_rows=24, track_k=8, spare_pages=2),
    # a short chained stack at oracle size
    "small_bf16_chained": WorkloadSpec(
        "small_bf16_chained", LayerShape("bf16", 512, 4, 128, 64, 500000.0, n_layers=4),
        batch=3, kind="window", ctx_len=300, prompt_len=64, window=16, tracked=16, track_k=8,
        chained=True, spare_pages=2),
    "small_f32_divergent": WorkloadSpec(
        "small_f32_divergent", LayerShape("f32", 128, 2, 64, 16, 10000.0),
        batch=4, kind="divergent", ctx_min=20, ctx_max=90, window=8, tracked=8,
        track_k=6, spare_pages=2),
}


def get_spec(name: str) -> WorkloadSpec:
    if name in WORKLOADS:
        return WORKLOADS[name]
    return SMALL_WORKLOADS[name]


@dataclasses.dataclass
class StepMeta:
    """Host-side description of one step (all arrays numpy)."""
    batch: int
    cu_rows: np.ndarray       # int32 [B+1]
    seq_lens: np.ndarray      # int32 [B]  visible context slots L_b
    positions: np.ndarray     # int32 [R]
    slots: np.ndarray         # int32 [R]
    view: np.ndarray          # int8  [R]  0 plain, 1 draft, 2 mask
    block_table: np.ndarray   # int32 [B, max_blocks]
    num_pages: int
    max_position: int         # exclusive bound on positions (RoPE table size)
    exclude_cu: np.ndarray    # int32 [B+1] exclusion list offsets (the window slots)
    exclude_slots: np.ndarray  # int32 [E]
    track_k: int
    stage: np.ndarray         # int8 [B] 0 caching, 1 update, 2 verify

    @property
    def total_rows(self) -> int:
        return int(self.cu_rows[-1])

    @property
    def max_blocks(self) -> int:
        return int(self.block_table.shape[1])


def _window_and_tracked(rng, L, window, tracked, lo):
    lo = max(0, min(lo, L - window))
    start = int(rng.integers(lo, L - window + 1))
    win = np.arange(start, start + window, dtype=np.int64)
    rest = np.setdiff1d(np.arange(L, dtype=np.int64), win)
    trk = np.sort(rng.choice(rest, size=tracked, replace=False)) if tracked else np.zeros(0, np.int64)
    return win, trk


def make_meta(spec: WorkloadSpec, seed: int = 0) -> StepMeta:
    rng = np.random.default_rng(seed)
    B = spec.batch
    ps = spec.shape.page_size
    rows_pos: List[np.ndarray] = []
    rows_slot: List[np.ndarray] = []
    rows_view: List[np.ndarray] = []
    seq_lens = np.zeros(B, np.int32)
    need_slots = np.zeros(B, np.int64)
    excl: List[np.ndarray] = []
    stage = np.zeros(B, np.int8)
    if spec.kind == "divergent":
        stage[:] = 0
        upd = rng.permutation(B)[: B // 2]
        stage[upd] = 1
    for b in range(B):
        if spec.kind == "two_view":
            L = spec.ctx_len
            n = spec.view_rows
            pos = np.arange(L, L + n, dtype=np.int64)
            # draft rows write their own positions, mask rows write scratch
            # slots right after them; both lie past the visible context.
            p = np.concatenate([pos, pos])
            s = np.concatenate([pos, pos + n])
            v = np.concatenate([np.full(n, 1), np.full(n, 2)])
            seq_lens[b] = L
            need_slots[b] = L + 2 * n
            stage[b] = 2
            excl.append(np.zeros(0, np.int64))
        else:
            if spec.kind == "divergent":
                L = int(rng.integers(spec.ctx_min, spec.ctx_max + 1))
                lo = L // 4
                n_trk = spec.tracked if stage[b] == 1 else 0
            else:
                L = spec.ctx_len
                lo = spec.prompt_len if spec.prompt_len else L // 4
                n_trk = spec.tracked
                stage[b] = 1
            win, trk = _window_and_tracked(rng, L, spec.window, n_trk, lo)
            p = np.concatenate([win, trk])
            s = p.copy()
            v = np.zeros(len(p), np.int64)
            seq_lens[b] = L
            need_slots[b] = L
            excl.append(win)
        rows_pos.append(p)
        rows_slot.append(s)
        rows_view.append(v)
    cu = np.zeros(B + 1, np.int32)
    cu[1:] = np.cumsum([len(p) for p in rows_pos])
    blocks_per = [(int(n) + ps - 1) // ps for n in need_slots]
    max_blocks = max(blocks_per)
    num_pages = int(sum(blocks_per)) + spec.spare_pages
    perm = rng.permutation(num_pages).astype(np.int32)
    bt = np.full((B, max_blocks), -1, np.int32)
    k = 0
    for b in range(B):
        for i in range(blocks_per[b]):
            bt[b, i] = perm[k]
            k += 1
    positions = np.concatenate(rows_pos).astype(np.int32)
    max_pos = int(positions.max()) + 1
    exclude_cu = np.zeros(B + 1, np.int32)
    exclude_cu[1:] = np.cumsum([len(e) for e in excl])
    return StepMeta(batch=B, cu_rows=cu, seq_lens=seq_lens, positions=positions,
                    slots=np.concatenate(rows_slot).astype(np.int32),
                    view=np.concatenate(rows_view).astype(np.int8), block_table=bt,
                    num_pages=num_pages, max_position=max_pos,
                    exclude_cu=exclude_cu,
                    exclude_slots=(np.concatenate(excl) if excl else np.zeros(0)).astype(np.int32),
                    track_k=spec.track_k, stage=stage)


def torch_dtype(shape: LayerShape) -> torch.dtype:
    return torch.bfloat16 if shape.dtype == "bf16" else torch.float32


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_x(spec: WorkloadSpec, meta: StepMeta, seed: int, layer: int = 0,
           device="cpu") -> torch.Tensor:
    """x [R, H]: N(0,1). In a two-view step every mask-view row carries the
    same vector (the [MASK] embedding); draft rows are independent."""
    H = spec.shape.hidden
    g = _gen(seed * 1000003 + 17 + layer * 7919, device)
    x = torch.randn(meta.total_rows, H, generator=g, device=device, dtype=torch.float32)
    if spec.kind == "two_view":
        m = torch.randn(1, H, generator=g, device=device, dtype=torch.float32)
        mask_rows = torch.from_numpy(np.nonzero(meta.view == 2)[0]).to(device)
        x[mask_rows] = m
    return x.to(torch_dtype(spec.shape))


def make_x_onehot(spec: WorkloadSpec, meta: StepMeta, seed: int, scale: float = 64.0,
                  device="cpu") -> torch.Tensor:
    """x [R, H] whose rows are scale * e_i for seeded columns i (scale a power
    of two). With it every projected value is one bf16 entry of Wqkv times a
    power of two, so fp32 and fp64 accumulation give the same number and no
    bf16 rounding decision can differ between two implementations. With
    scale 64 and Wqkv ~ N(0, 0.02^2) the projected values are N(0, 1.28^2),
    the magnitude of the dense workloads."""
    rng = np.random.default_rng(seed * 7 + 3)
    H = spec.shape.hidden
    idx = rng.integers(0, H, meta.total_rows)
    x = torch.zeros(meta.total_rows, H, dtype=torch.float32, device=device)
    x[torch.arange(meta.total_rows, device=device), torch.from_numpy(idx).to(device)] = scale
    return x.to(torch_dtype(spec.shape))


def make_x_grid(spec: WorkloadSpec, meta: StepMeta, seed: int, layer: int = 0,
                device="cpu") -> torch.Tensor:
    """x [R, H] ~ N(0, 1) snapped to multiples of 1/4 in [-4, 4] (two-view:
    mask rows share one vector, as in make_x). Together with make_w_grid
    every product x_k W_kn is a multiple of 2^-12 and every partial sum of
    4096 of them stays below 2^11 in magnitude, so each sum is exact in
    float32 whatever the order of accumulation: the projection of these
    dense, normally shaped inputs is exact in fp32 and fp64 alike."""
    x = make_x(spec, meta, seed, layer=layer, device=device).float()
    return (torch.clamp(torch.round(x * 4.0), -16, 16) / 4.0).to(torch_dtype(spec.shape))


def make_w_grid(spec: WorkloadSpec, seed: int, layer: int = 0, device="cpu") -> torch.Tensor:
    """Wqkv ~ N(0, 0.02^2) snapped to multiples of 2^-10 in [-127, 127] *
    2^-10 (see make_x_grid)."""
    w = make_w(spec, seed, layer=layer, device=device).float()
    return (torch.clamp(torch.round(w * 1024.0), -127, 127) / 1024.0).to(torch_dtype(spec.shape))


def make_w(spec: WorkloadSpec, seed: int, layer: int = 0, device="cpu") -> torch.Tensor:
    """Wqkv [H, 3H] row-major, N(0, 0.02^2); columns are [Q | K | V], each
    block head-major (head h at columns h*D .. h*D+D-1)."""
    H = spec.shape.hidden
    g = _gen(seed * 1000003 + 29 + layer * 104729, device)
    w = torch.randn(H, 3 * H, generator=g, device=device, dtype=torch.float32) * 0.02
    return w.to(torch_dtype(spec.shape))


def make_w_o(spec: WorkloadSpec, seed: int, layer: int = 0, device="cpu") -> torch.Tensor:
    """W_o [H, H] row-major, N(0, 0.02^2): the output projection of a chained
    stack's layer."""
    H = spec.shape.hidden
    g = _gen(seed * 1000003 + 67 + layer * 130363, device)
    w = torch.randn(H, H, generator=g, device=device, dtype=torch.float32) * 0.02
    return w.to(torch_dtype(spec.shape))


def make_pools(spec: WorkloadSpec, meta: StepMeta, seed: int, device="cpu",
               n_layers: Optional[int] = None):
    """K and V pools [n_layers, num_pages, n_heads, page_size, head_dim].

    Visible slots hold N(0, 1.28^2); every slot the step writes and every page
    tail past the sequence's last visible/written slot holds a NaN pattern;
    spare pages hold random bits."""
    sh = spec.shape
    nl = sh.n_layers if n_layers is None else n_layers
    shape = (nl, meta.num_pages, sh.n_heads, sh.page_size, sh.head_dim)
    g = _gen(seed * 1000003 + 41, device)
    dt = torch_dtype(sh)
    nan_bits = BF16_NAN_BITS if sh.dtype == "bf16" else F32_NAN_BITS
    int_dt = torch.int16 if sh.dtype == "bf16" else torch.int32
    pools = []
    for _ in range(2):
        # start from random bits everywhere (spare pages keep them)
        if sh.dtype == "bf16":
            bits = torch.randint(-32768, 32767, shape, generator=g, device=device, dtype=torch.int16)
        else:
            bits = torch.randint(-2**31, 2**31 - 1, shape, generator=g, device=device, dtype=torch.int32)
        pool = bits.view(dt)
        ps = sh.page_size
        for b in range(meta.batch):
            L = int(meta.seq_lens[b])
            r0, r1 = int(meta.cu_rows[b]), int(meta.cu_rows[b + 1])
            top = max([L] + [int(s) + 1 for s in meta.slots[r0:r1]])
            nblk = (top + ps - 1) // ps
            for i in range(nblk):
                pg = int(meta.block_table[b, i])
                lo = i * ps
                n_vis = max(0, min(ps, L - lo))
                if n_vis:
                    vals = torch.randn((nl, sh.n_heads, n_vis, sh.head_dim), generator=g,
                                       device=device, dtype=torch.float32) * 1.28
                    pool[:, pg, :, :n_vis, :] = vals.to(dt)
                if n_vis < ps:
                    pool.view(int_dt)[:, pg, :, n_vis:, :] = nan_bits if sh.dtype == "f32" else _i16(nan_bits)
            for s in meta.slots[r0:r1]:
                pg = int(meta.block_table[b, int(s) // ps])
                pool.view(int_dt)[:, pg, :, int(s) % ps, :] = nan_bits if sh.dtype == "f32" else _i16(nan_bits)
        pools.append(pool)
    return pools[0], pools[1]


def _i16(u: int) -> int:
    return u - 65536 if u >= 32768 else u


def bits_np(t: torch.Tensor) -> np.ndarray:
    """Raw bits of a bf16/f32 tensor as uint16/uint32 numpy (host copy)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy().view(np.uint32)
    raise TypeError(t.dtype)


def algorithmic_bytes_flops(spec: WorkloadSpec, meta: StepMeta, with_mass: bool = True):
    """Byte and FLOP model of one layer step (per layer).

    bytes = Wqkv + x + cache reads of visible non-fresh slots + cache writes
            + out (fp32) + attn_mass (fp32);
    flops = 2*R*H*3H (projection) + 4*D*n_h*sum_r |K(r)| (QK^T and PV).
    The second key pass, padding rows and RoPE/softmax arithmetic are not
    counted. A chained stack's layer adds its output projection with the
    residual: W_o read, x_{l+1} written in place of the fp32 out, and
    2*R*H*H flops (the bf16 out that feeds the projection is an
    intermediate, not counted)."""
    sh = spec.shape
    s = 2 if sh.dtype == "bf16" else 4
    H = sh.hidden
    R = meta.total_rows
    byt = H * 3 * H * s + R * H * s + R * 2 * H * s
    fl = 2 * R * H * 3 * H
    if spec.chained:
        byt += H * H * s + R * H * s
        fl += 2 * R * H * H
    else:
        byt += R * H * 4
    keys = 0
    for b in range(meta.batch):
        L = int(meta.seq_lens[b])
        r0, r1 = int(meta.cu_rows[b]), int(meta.cu_rows[b + 1])
        sl = meta.slots[r0:r1]
        vw = meta.view[r0:r1]
        ps_ = meta.positions[r0:r1]
        fresh_vis = int(np.sum((sl < L) & (vw == 0)))
        byt += (L - fresh_vis) * 2 * H * s
        if with_mass:
            byt += 4 * L
        for i in range(r1 - r0):
            k = L
            if vw[i] != 0:
                k += int(np.sum((vw == vw[i]) & (ps_ <= ps_[i])))
            keys += k
    fl += 4 * sh.head_dim * sh.n_heads * keys
    return byt, fl


# ------------------------------------------------------------------ Flash-Verify
@dataclasses.dataclass(frozen=True)
class VerifySpec:
    """Mask-view logits of a Flash-Verify block for every sequence."""
    name: str
    batch: int
    rows: int            # block positions per sequence (the mask view's rows)
    vocab: int
    dtype: str           # "bf16" or "f32"
    tau: float           # confidence threshold


VERIFY_WORKLOADS: Dict[str, VerifySpec] = {
    # the two-view workload's mask view: batch 8 x 32 positions, LLaDA
    # vocabulary (126464 tokens), bf16 logits
    "verify_b8": VerifySpec("verify_b8", batch=8, rows=32, vocab=126464, dtype="bf16", tau=0.9),
    "verify_small": VerifySpec("verify_small", batch=5, rows=12, vocab=1000, dtype="bf16", tau=0.6),
}


def make_verify(spec: VerifySpec, seed: int, device="cpu"):
    """(logits [R, V], cu_rows [B+1] int32, draft [R] int32).

    Logits are N(0, 2^2). Each sequence gets a seeded prefix length a in
    [0, rows]; the drafted token of a position before a is given a raised
    logit (+9 to +14, so that it is usually the most likely token with a
    high softmax probability), the position at a gets a draft token with no
    raised logit (or a smaller raise), and later positions get random
    drafts, half of them raised. The step's own rule then decides what is
    accepted."""
    rng = np.random.default_rng(seed)
    B, n, V = spec.batch, spec.rows, spec.vocab
    R = B * n
    g = _gen(seed * 1000003 + 57, device)
    logits = torch.randn(R, V, generator=g, device=device, dtype=torch.float32) * 2.0
    draft = rng.integers(0, V, R).astype(np.int64)
    boost = np.zeros(R)
    for b in range(B):
        a = int(rng.integers(0, n + 1))
        for i in range(n):
            r = b * n + i
            if i < a:
                boost[r] = rng.uniform(9.0, 14.0)
            elif i == a:
                boost[r] = 0.0 if rng.random() < 0.5 else rng.uniform(1.0, 4.0)
            else:
                boost[r] = rng.uniform(9.0, 14.0) if rng.random() < 0.5 else 0.0
    rows_t = torch.arange(R, device=device)
    d_t = torch.from_numpy(draft).to(device)
    logits[rows_t, d_t] += torch.from_numpy(boost).to(device=device, dtype=torch.float32)
    dt = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
    cu = (np.arange(B + 1) * n).astype(np.int32)
    return logits.to(dt), cu, draft.astype(np.int32)


# ------------------------------------------------------------------ output projection
@dataclasses.dataclass(frozen=True)
class OprojSpec:
    """Attention output rows of one layer step and the layer's W_o."""
    name: str
    rows: int
    hidden: int


OPROJ_WORKLOADS: Dict[str, OprojSpec] = {
    # the batch-32 layer step's 1536 query rows at LLaDA-8B width
    "oproj_b32": OprojSpec("oproj_b32", rows=1536, hidden=4096),
}


def make_oproj(spec: OprojSpec, seed: int, device="cpu"):
    """(o [rows, hidden] bf16 ~ N(0, 1), W_o [hidden, hidden] bf16 ~
    N(0, 0.02^2)), drawn by a seeded torch generator as float32 and cast
    (round to nearest even)."""
    g = _gen(seed * 1000003 + 91, device)
    o = torch.randn(spec.rows, spec.hidden, generator=g, device=device, dtype=torch.float32)
    w = torch.randn(spec.hidden, spec.hidden, generator=g, device=device, dtype=torch.float32) * 0.02
    return o.to(torch.bfloat16), w.to(torch.bfloat16)


# ------------------------------------------------------------------ toy decode loop
@dataclasses.dataclass(frozen=True)
class ToyConfig:
    hidden: int = 512
    n_heads: int = 4
    head_dim: int = 128
    n_layers: int = 2
    page_size: int = 64
    rope_theta: float = 500000.0
    batch: int = 2
    prompt_len: int = 64
    gen_len: int = 64
    window: int = 8
    track_k: int = 8
    tau: float = 0.5
    seed: int = 0


def toy_weights(cfg: ToyConfig, device="cpu"):
    """Random bf16 weights of the toy model, from seeded generators:
    E [V, H] ~ N(0, 1) (V = H, the last id is [MASK]); per layer Wqkv
    [H, 3H] and W_o [H, H] ~ N(0, 0.02^2); the LM head W_lm [H, V] ~
    N(0, 0.02^2) scaled by 8 so that some predictions are confident."""
    H = cfg.hidden
    g = torch.Generator(device="cpu").manual_seed(cfg.seed * 7919 + 5)
    bf = torch.bfloat16
    emb = torch.randn(H, H, generator=g).to(bf)
    wqkv = [(torch.randn(H, 3 * H, generator=g) * 0.02).to(bf) for _ in range(cfg.n_layers)]
    w_o = [(torch.randn(H, H, generator=g) * 0.02).to(bf) for _ in range(cfg.n_layers)]
    w_lm = (torch.randn(H, H, generator=g) * 0.16).to(bf)
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else [t.to(device) for t in v])
            for k, v in dict(emb=emb, wqkv=wqkv, w_o=w_o, w_lm=w_lm).items()}


def toy_layout(cfg: ToyConfig):
    """Seeded host state: prompt tokens, the [MASK]ed generation region and
    a permuted block table. Returns (tokens [B, L] int64, block_table
    [B, blocks] int32, num_pages)."""
    rng = np.random.default_rng(cfg.seed)
    B, L, ps = cfg.batch, cfg.prompt_len + cfg.gen_len, cfg.page_size
    V = cfg.hidden
    tokens = np.full((B, L), V - 1, np.int64)
    tokens[:, :cfg.prompt_len] = rng.integers(0, V - 1, (B, cfg.prompt_len))
    nblk = (L + ps - 1) // ps
    num_pages = B * nblk + 2
    perm = rng.permutation(num_pages).astype(np.int32)
    bt = perm[:B * nblk].reshape(B, nblk)
    return tokens, bt, num_pages
