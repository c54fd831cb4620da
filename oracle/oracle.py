"""CPU oracle for the Flash-dLLM per-layer decoding step.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports this module:
only the tests, the smoke check and the benchmark's CPU-baseline leg call it.
It shares no code with the CUDA path; the only common code is the seeded
input generator, which holds none of the step's arithmetic.

What it computes is the plain definition of one layer step, in float64, one
sequence and one head at a time, with no blocking and no fusion. Fusion in
Flash-Cache changes where data lives, not the mathematics, so the plain
definition is the exact target up to rounding order.

Citations name the page they follow:
  [FD] "Flash-dLLM: I/O-Aware KV Caching and Parallel Decoding for Fast,
       Memory-Efficient Diffusion LLMs" (ai4snews summary of the full text);
       paragraph numbers count that page's body paragraphs.
  [AB] "Flash-dLLM: IO-Aware KV Caching and Parallel Decoding for Fast,
       Memory-Efficient Diffusion LLMs" (arXiv abstract page), Abstract.

Readings where the pages are silent (each is listed in the design notes):
  * Wqkv is [H, 3H] row-major, y = x W, column blocks Q | K | V, head-major
    inside each block; no bias.
  * RoPE is the rotate-half form: pair (i, i + D/2), angle
    p * theta^(-2i/D), computed here in float64.
  * Attention is bidirectional with scale 1/sqrt(D); rows in a Flash-Verify
    view also see earlier-or-equal positions of their own view.
  * Attention reads the cache after all of this step's writes.
  * The per-key attention mass is the mean over heads and over the
    sequence's query rows of the softmax probabilities, so it sums to 1.
  * Top-k ties go to the lower slot.
  * Flash-Verify: the views agree when the mask view's most likely token
    (lowest id among equal logits) is the drafted token; the confidence is
    that token's softmax probability; the threshold is a parameter.

Every function here has a pin in tests/test_oracle_pins.py,
tests/test_oracle_verify_pins.py or tests/test_oracle_oproj_pins.py (brute
force, closed forms, library special cases or invariants); none is "parity
unpinned".
"""
from __future__ import annotations

import numpy as np

# --------------------------------------------------------------------------
# Number formats
# --------------------------------------------------------------------------

_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bfloat16 bit patterns (the top half of a binary32)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def f32_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint32).view(np.float32).astype(np.float64)


def round_to_bf16(v: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16, ties to even.

    bfloat16 has 8 significant bits and binary32's exponent range, so a
    value in [2^(e-1), 2^e) has spacing 2^(e-8), with the subnormal spacing
    2^-133 as the floor. Dividing by that spacing, rounding to the nearest
    integer (half to even) and scaling back is exact in float64. Magnitudes
    that round past the largest finite bfloat16 become infinite.
    Returns float64 values (each exactly representable in bfloat16)."""
    v = np.asarray(v, dtype=np.float64)
    _, e = np.frexp(v)
    q = np.maximum(e - 8, -133)
    r = np.ldexp(np.rint(np.ldexp(v, -q)), q)
    return np.where(np.abs(r) > _BF16_MAX, np.copysign(np.inf, v), r)


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    r = round_to_bf16(v)
    return (r.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def f64_to_f32_bits(v: np.ndarray) -> np.ndarray:
    # numpy's float64 -> float32 conversion rounds to nearest even (IEEE 754)
    return np.asarray(v, dtype=np.float64).astype(np.float32).view(np.uint32)


def decode(bits: np.ndarray, dtype: str) -> np.ndarray:
    return bf16_bits_to_f64(bits) if dtype == "bf16" else f32_bits_to_f64(bits)


def encode(v: np.ndarray, dtype: str) -> np.ndarray:
    return f64_to_bf16_bits(v) if dtype == "bf16" else f64_to_f32_bits(v)


# --------------------------------------------------------------------------
# Rotary position embedding  [FD ¶1: RoPE is fused with the projection]
# --------------------------------------------------------------------------

def rope(u: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotate-half RoPE. u: [R, n_heads, D] float64; positions: [R].

    For i < D/2 the pair (u_i, u_{i+D/2}) turns by the angle
    p * theta^(-2i/D)."""
    R, nh, D = u.shape
    half = D // 2
    i = np.arange(half, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / D)
    phi = np.asarray(positions, dtype=np.float64)[:, None] * inv_freq[None, :]
    c = np.cos(phi)[:, None, :]
    s = np.sin(phi)[:, None, :]
    a = u[..., :half]
    b = u[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


# --------------------------------------------------------------------------
# Key visibility  [FD ¶1 block table; ¶3 Flash-Verify two-view mask]
# --------------------------------------------------------------------------

def visible_keys(L: int, view: np.ndarray, positions: np.ndarray, slots: np.ndarray):
    """Key slots of one sequence and the [rows, keys] visibility matrix.

    Every row sees the context slots [0, L). A row in view 1 (draft) or 2
    (mask) also sees the slots written this step by rows of the same view
    whose position is at most its own; the two views never see each other's
    fresh slots. Plain rows (view 0) see only [0, L)."""
    R = len(view)
    extra_idx = [t for t in range(R) if view[t] != 0]
    keys = np.concatenate([np.arange(L, dtype=np.int64),
                           np.asarray([slots[t] for t in extra_idx], dtype=np.int64)])
    vis = np.zeros((R, len(keys)), dtype=bool)
    vis[:, :L] = True
    for r in range(R):
        if view[r] == 0:
            continue
        for j, t in enumerate(extra_idx):
            if view[t] == view[r] and positions[t] <= positions[r]:
                vis[r, L + j] = True
    return keys, vis


# --------------------------------------------------------------------------
# One layer step
# --------------------------------------------------------------------------

def layer_step(shape, k_pool, v_pool, layer, x_bits, w_bits, positions, slots,
               cu_rows, seq_lens, block_table, view, probs=None, accumulate="f64"):
    """One Flash-Cache + scheduled-attention layer step.

    shape: object with dtype ("bf16"/"f32"), hidden, n_heads, head_dim,
      page_size, rope_theta.
    k_pool, v_pool: raw bits [n_layers, num_pages, n_heads, page_size, D]
      (uint16 for bf16, uint32 for f32). Copies are returned, the inputs are
      not modified.
    x_bits [R, H], w_bits [H, 3H]: raw bits.
    positions, slots, view: [R]; cu_rows [B+1]; seq_lens [B];
      block_table [B, max_blocks].

    Returns (out [R, H] float64, mass [B, max_blocks * page_size] float64,
             k_pool', v_pool').
    If `probs` is a dict, probs[(b, h)] = (key slots, P [R_b, keys]) is
    recorded for the tests' error analysis (no effect on the results).

    Steps [FD ¶1]: project the selected rows, rotate q and k, write k and v
    into the paged cache, then attend over each sequence's pages through its
    block table. [FD ¶2]: the step's rows are the unmasking window plus the
    tracked tokens; the per-key attention mass feeds the next tracked set.
    [FD ¶3]: the draft and mask views share positions (hence RoPE) and are
    isolated from each other.

    accumulate: "f64" (default) takes the projection exactly (float64 sums
    of exact products); "f32" takes it from a float32 matrix product of the
    same bf16/fp32 inputs (project_f32acc): the bf16-in / fp32-accumulate
    reading of the step, whose fresh k and v can land on the other side of a
    bf16 rounding midpoint. Everything after the projection is the same."""
    if accumulate == "f64":
        a = project(shape, x_bits, w_bits)
    elif accumulate == "f32":
        a = project_f32acc(shape, x_bits, w_bits)
    else:
        raise ValueError(f"accumulate must be 'f64' or 'f32', got {accumulate!r}")
    return layer_step_from_projection(shape, k_pool, v_pool, layer, a, positions, slots,
                                      cu_rows, seq_lens, block_table, view, probs)


def project(shape, x_bits, w_bits):
    """Step 1, the QKV projection: a = x Wqkv in float64 (library matmul on
    the exact values of the bf16/fp32 inputs). [R, 3H]."""
    return decode(x_bits, shape.dtype) @ decode(w_bits, shape.dtype)


def project_f32acc(shape, x_bits, w_bits):
    """Step 1 with float32 accumulation: the library's float32 matrix
    product of the same inputs (each bf16/fp32 input is exact in float32),
    returned as float64. It differs from `project` only by float32 rounding
    of the sums (at most about K * 2^-24 * sum |x_k w_k| per entry)."""
    xf = decode(x_bits, shape.dtype).astype(np.float32)
    wf = decode(w_bits, shape.dtype).astype(np.float32)
    return (xf @ wf).astype(np.float64)


def layer_step_from_projection(shape, k_pool, v_pool, layer, a, positions, slots, cu_rows,
                               seq_lens, block_table, view, probs=None):
    """Steps 2-6 of layer_step from a given projection result a [R, 3H]."""
    dt = shape.dtype
    H, nh, D, ps = shape.hidden, shape.n_heads, shape.head_dim, shape.page_size
    k_pool = k_pool.copy()
    v_pool = v_pool.copy()
    B = len(seq_lens)
    R = a.shape[0]
    row_stride = block_table.shape[1] * ps

    q = a[:, 0:H].reshape(R, nh, D)
    k = a[:, H:2 * H].reshape(R, nh, D)
    v = a[:, 2 * H:3 * H].reshape(R, nh, D)
    # 2. rotary embedding on q and k
    q = rope(q, positions, shape.rope_theta)
    k = rope(k, positions, shape.rope_theta)
    # 3. the query is held in the compute dtype (bf16 in bf16 configs)
    if dt == "bf16":
        q = round_to_bf16(q)
    # 4. write k, v into the paged cache, in the cache dtype
    for r in range(R):
        b = int(np.searchsorted(cu_rows, r, side="right") - 1)
        s = int(slots[r])
        pg = int(block_table[b, s // ps])
        k_pool[layer, pg, :, s % ps, :] = encode(k[r], dt)
        v_pool[layer, pg, :, s % ps, :] = encode(v[r], dt)

    # 5. attention over the cache as it stands after every write of the step
    out = np.zeros((R, H), dtype=np.float64)
    mass = np.zeros((B, row_stride), dtype=np.float64)
    for b in range(B):
        r0, r1 = int(cu_rows[b]), int(cu_rows[b + 1])
        if r1 == r0:
            continue
        L = int(seq_lens[b])
        keys, vis = visible_keys(L, view[r0:r1], positions[r0:r1], slots[r0:r1])
        pages = block_table[b, keys // ps]
        offs = keys % ps
        Kc = decode(k_pool[layer, pages, :, offs, :], dt)   # [nk, nh, D]
        Vc = decode(v_pool[layer, pages, :, offs, :], dt)
        for h in range(nh):
            S = (q[r0:r1, h, :] @ Kc[:, h, :].T) / np.sqrt(D)
            P = softmax_rows(S, vis)
            out[r0:r1, h * D:(h + 1) * D] = P @ Vc[:, h, :]
            if probs is not None:
                probs[(b, h)] = (keys, P)
            # 6. attention mass: mean over heads and rows  [FD ¶2]
            np.add.at(mass[b], keys, P.sum(axis=0) * mass_weight(r1 - r0, nh))
    return out, mass, k_pool, v_pool


def mass_weight(n_rows: int, n_heads: int) -> float:
    """Weight of one probability in the attention mass: the mass is the
    mean over the sequence's rows and over the heads [FD ¶2], so each of the
    n_rows * n_heads probability rows counts 1 / (n_rows * n_heads)."""
    return 1.0 / (n_rows * n_heads)


def softmax_rows(S: np.ndarray, vis: np.ndarray) -> np.ndarray:
    """Row softmax of S restricted to the visible entries; invisible entries
    get probability 0, and a row with no visible key gets all zeros (its
    output is 0 and it adds no mass)."""
    has = vis.any(axis=1, keepdims=True)
    Sm = np.where(vis, S, -np.inf)
    m = np.where(has, Sm.max(axis=1, keepdims=True, initial=-np.inf), 0.0)
    E = np.where(vis, np.exp(np.where(vis, S, 0.0) - m), 0.0)
    den = E.sum(axis=1, keepdims=True)
    return np.where(has, E / np.where(has, den, 1.0), 0.0)


# --------------------------------------------------------------------------
# Next step's tracked set  [FD ¶2: a fixed budget of most-attended tokens]
# --------------------------------------------------------------------------

def select_tracked(mass: np.ndarray, seq_lens, k: int, exclude_cu=None, exclude_slots=None):
    """Per sequence, the k slots in [0, L_b) (minus the exclusion list) with
    the largest mass; ties go to the lower slot; descending mass order;
    padded with -1. The comparison is made on the values as given (fp32
    mass from the kernel is compared in fp32)."""
    B = len(seq_lens)
    out = np.full((B, k), -1, dtype=np.int32)
    for b in range(B):
        L = int(seq_lens[b])
        cand = np.arange(L, dtype=np.int64)
        if exclude_cu is not None:
            ex = set(int(s) for s in exclude_slots[exclude_cu[b]:exclude_cu[b + 1]])
            cand = np.asarray([j for j in cand if j not in ex], dtype=np.int64)
        if len(cand) == 0:
            continue
        vals = mass[b, cand]
        order = np.lexsort((cand, -vals))      # by -mass, then by slot
        take = cand[order[:k]]
        out[b, :len(take)] = take
    return out


# --------------------------------------------------------------------------
# Flash-Verify acceptance  [FD ¶3]
# --------------------------------------------------------------------------

def verify_rows(logits_bits: np.ndarray, dtype: str):
    """Mask-view prediction and confidence of every row of logits [R, V]:
    the prediction is the token with the largest logit (the lowest token id
    among equal largest logits) and the confidence is that token's softmax
    probability, 1 / sum_v exp(logit_v - max). Computed in float64 from the
    exactly decoded logits. Returns (pred int32 [R], conf float64 [R])."""
    lg = decode(logits_bits, dtype)
    R = lg.shape[0]
    pred = np.zeros(R, dtype=np.int32)
    conf = np.zeros(R, dtype=np.float64)
    for r in range(R):
        row = lg[r]
        mx = row.max()
        pred[r] = int(np.flatnonzero(row == mx)[0])
        conf[r] = 1.0 / np.sum(np.exp(row - mx))
    return pred, conf


def verify_accept(pred, conf, draft_tokens, cu_rows, tau: float):
    """Accepted prefix length of every sequence [FD ¶3]: the rows of sequence
    b are its block positions in causal order; position i is accepted when
    the mask view's prediction equals the drafted token and its confidence
    exceeds tau, and acceptance stops at the first position that is not.
    The confidences are compared as given (a kernel's fp32 values are
    compared in fp32), so the decision is taken in the kernel's precision.
    Returns int32 [B]."""
    B = len(cu_rows) - 1
    out = np.zeros(B, dtype=np.int32)
    for b in range(B):
        n = 0
        for i in range(int(cu_rows[b]), int(cu_rows[b + 1])):
            if int(pred[i]) == int(draft_tokens[i]) and conf[i] > tau:
                n += 1
            else:
                break
        out[b] = n
    return out


# --------------------------------------------------------------------------
# Output projection of the attention block (a "next" step after the layer)
# --------------------------------------------------------------------------

def oproj(out_bits: np.ndarray, w_bits: np.ndarray, residual_bits=None) -> np.ndarray:
    """The attention block's output projection y = o W_o, float64.

    o [R, H] holds each row's attention output with the heads side by side
    (head h in columns h*D .. h*D + D - 1, the layout of the layer step's
    `out`), given as bf16 bits; W_o [H, H] is row-major bf16 bits, no bias.
    The pages stop at the attention output ([FD ¶1]: QKV projection, RoPE,
    cache write, scheduled attention) and say nothing of W_o; this is the
    plain linear map that follows attention in a transformer layer, read
    with the same conventions as Wqkv (y = x W, row-major, no bias).
    With residual_bits (bf16 [R, H]) it returns residual + o W_o: the
    residual stream of a transformer layer, which is how one layer's output
    becomes the next layer's input when layers are chained.
    Returns float64 [R, H]; rounding y to bf16 is the caller's business."""
    o = bf16_bits_to_f64(out_bits)
    w = bf16_bits_to_f64(w_bits)
    y = o @ w
    if residual_bits is not None:
        y = y + bf16_bits_to_f64(residual_bits)
    return y
