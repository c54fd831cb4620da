"""Pins for the CPU oracle, checked against things other than the oracle.

Each pin uses an independent route: a library routine (torch's bf16 cast,
torch's scaled_dot_product_attention in float64), a closed form (the complex
exponential form of rotary embedding, exact rounding cases), brute force
over the whole sequence, or an invariant the method must keep (softmax rows
sum to one, the two Flash-Verify views are isolated, the block table is a
pure indirection, untouched cache bytes stay untouched).
"""
import dataclasses

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import oracle as O

# --------------------------------------------------------------------------
# independent helpers (written from the definitions, not from the oracle)
# --------------------------------------------------------------------------


@dataclasses.dataclass
class Shape:
    dtype: str
    hidden: int
    n_heads: int
    head_dim: int
    page_size: int
    rope_theta: float


def bf16_round_to_odd(v64: np.ndarray) -> np.ndarray:
    """float64 -> bf16 bits through a round-to-odd float32 intermediate and
    torch's float32 -> bf16 cast. Round-to-odd at 24 bits followed by
    round-to-nearest-even at 8 bits equals direct round-to-nearest-even
    (Boldo & Melquiond, 'When double rounding is odd')."""
    v64 = np.asarray(v64, np.float64)
    f = v64.astype(np.float32)
    bits = f.view(np.uint32).copy()
    back = f.astype(np.float64)
    away = np.abs(back) > np.abs(v64)           # RNE went away from zero
    bits = np.where(away, bits - 1, bits)       # truncate toward zero
    inexact = back != v64
    bits = np.where(inexact, bits | 1, bits)    # ... then make it odd
    t = torch.from_numpy(bits.view(np.float32).copy()).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def torch_bf16_value(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    return t.to(torch.float64)


def rope_complex(u: torch.Tensor, pos: torch.Tensor, theta: float) -> torch.Tensor:
    """RoPE as multiplication of (u_i + j u_{i+D/2}) by exp(j p theta^(-2i/D))."""
    D = u.shape[-1]
    half = D // 2
    i = torch.arange(half, dtype=torch.float64)
    ang = pos.to(torch.float64)[:, None] * torch.pow(torch.tensor(theta, dtype=torch.float64), -2.0 * i / D)
    z = torch.complex(u[..., :half], u[..., half:])
    rot = torch.polar(torch.ones_like(ang), ang)[:, None, :]
    z = z * rot
    return torch.cat([z.real, z.imag], dim=-1)


def round_cache(v: torch.Tensor, dtype: str):
    """Cache-dtype bits of float64 values, by an independent route."""
    if dtype == "bf16":
        return bf16_round_to_odd(v.numpy())
    return v.to(torch.float32).numpy().view(np.uint32)


def cache_value(bits, dtype) -> torch.Tensor:
    if dtype == "bf16":
        return torch_bf16_value(np.asarray(bits))
    return torch.from_numpy(np.asarray(bits).view(np.float32).copy()).to(torch.float64)


def rand_bits(rng, shape, dtype, scale=1.0):
    v = rng.standard_normal(shape) * scale
    if dtype == "bf16":
        return torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return v.astype(np.float32).view(np.uint32)


def make_case(rng, shape, lens, rows_per_seq, extra_pages=2, views=None, nan_fill=True):
    """A small step: per sequence L_b context slots and rows at distinct
    positions inside the context (or the given views past it)."""
    B = len(lens)
    ps = shape.page_size
    pos_l, slot_l, view_l = [], [], []
    need = []
    for b in range(B):
        L = lens[b]
        if views is not None and views[b] is not None:
            n = views[b]
            p = np.arange(L, L + n)
            pos_l.append(np.concatenate([p, p]))
            slot_l.append(np.concatenate([p, p + n]))
            view_l.append(np.concatenate([np.ones(n, np.int8), np.full(n, 2, np.int8)]))
            need.append(L + 2 * n)
        else:
            p = np.sort(rng.choice(L, size=rows_per_seq[b], replace=False))
            pos_l.append(p)
            slot_l.append(p)
            view_l.append(np.zeros(len(p), np.int8))
            need.append(L)
    nblk = [(n + ps - 1) // ps for n in need]
    mb = max(nblk)
    npg = sum(nblk) + extra_pages
    perm = rng.permutation(npg)
    bt = np.full((B, mb), -1, np.int32)
    k = 0
    for b in range(B):
        for i in range(nblk[b]):
            bt[b, i] = perm[k]
            k += 1
    cu = np.zeros(B + 1, np.int32)
    cu[1:] = np.cumsum([len(p) for p in pos_l])
    R = int(cu[-1])
    H = shape.hidden
    x = rand_bits(rng, (R, H), shape.dtype)
    w = rand_bits(rng, (H, 3 * H), shape.dtype, 0.02 * np.sqrt(4096 / H))
    pshape = (1, npg, shape.n_heads, ps, shape.head_dim)
    kp = rand_bits(rng, pshape, shape.dtype, 1.28)
    vp = rand_bits(rng, pshape, shape.dtype, 1.28)
    return dict(x=x, w=w, kp=kp, vp=vp, positions=np.concatenate(pos_l).astype(np.int32),
                slots=np.concatenate(slot_l).astype(np.int32), view=np.concatenate(view_l).astype(np.int8),
                cu=cu, lens=np.asarray(lens, np.int32), bt=bt)


def run_oracle(shape, c, **over):
    d = dict(c)
    d.update(over)
    return O.layer_step(shape, d["kp"], d["vp"], 0, d["x"], d["w"], d["positions"], d["slots"],
                        d["cu"], d["lens"], d["bt"], d["view"],
                        accumulate=d.get("accumulate", "f64"))


def brute_force(shape, c):
    """Whole-step brute force with torch float64: project, rotate (complex
    form), round k/v to the cache dtype, assemble each sequence's full K/V
    (fresh rows replace the cached ones, the rest is read from the pre-state
    cache), then scaled_dot_product_attention per head with an explicit
    boolean mask."""
    dt = shape.dtype
    H, nh, D, ps = shape.hidden, shape.n_heads, shape.head_dim, shape.page_size
    x = cache_value(c["x"], dt)
    w = cache_value(c["w"], dt)
    a = x @ w
    R = x.shape[0]
    pos = torch.from_numpy(c["positions"].astype(np.int64))
    q = rope_complex(a[:, :H].reshape(R, nh, D), pos, shape.rope_theta)
    k = rope_complex(a[:, H:2 * H].reshape(R, nh, D), pos, shape.rope_theta)
    v = a[:, 2 * H:].reshape(R, nh, D)
    if dt == "bf16":
        q = torch_bf16_value(bf16_round_to_odd(q.numpy()))
    kq = cache_value(round_cache(k, dt), dt)
    vq = cache_value(round_cache(v, dt), dt)
    out = torch.zeros(R, H, dtype=torch.float64)
    B = len(c["lens"])
    mass = torch.zeros(B, c["bt"].shape[1] * ps, dtype=torch.float64)
    for b in range(B):
        r0, r1 = int(c["cu"][b]), int(c["cu"][b + 1])
        L = int(c["lens"][b])
        slots = c["slots"][r0:r1]
        vw = c["view"][r0:r1]
        ps_ = c["positions"][r0:r1]
        # key list: context [0, L) then the view rows' slots
        key_slots = list(range(L)) + [int(slots[t]) for t in range(r1 - r0) if vw[t] != 0]
        Kb = torch.zeros(len(key_slots), nh, D, dtype=torch.float64)
        Vb = torch.zeros(len(key_slots), nh, D, dtype=torch.float64)
        fresh = {int(slots[t]): t for t in range(r1 - r0)}
        for j, s in enumerate(key_slots):
            if s in fresh:
                Kb[j] = kq[r0 + fresh[s]]
                Vb[j] = vq[r0 + fresh[s]]
            else:
                pg = int(c["bt"][b, s // ps])
                Kb[j] = cache_value(c["kp"][0, pg, :, s % ps, :], dt)
                Vb[j] = cache_value(c["vp"][0, pg, :, s % ps, :], dt)
        mask = torch.zeros(r1 - r0, len(key_slots), dtype=torch.bool)
        mask[:, :L] = True
        ex = [t for t in range(r1 - r0) if vw[t] != 0]
        for r in range(r1 - r0):
            for jj, t in enumerate(ex):
                if vw[r] != 0 and vw[t] == vw[r] and ps_[t] <= ps_[r]:
                    mask[r, L + jj] = True
        Q = q[r0:r1].permute(1, 0, 2)            # [nh, Rb, D]
        Kt = Kb.permute(1, 0, 2)
        Vt = Vb.permute(1, 0, 2)
        o = F.scaled_dot_product_attention(Q, Kt, Vt, attn_mask=mask)
        out[r0:r1] = o.permute(1, 0, 2).reshape(r1 - r0, H)
        P = torch.softmax((Q @ Kt.transpose(1, 2)) / np.sqrt(D) + torch.where(mask, 0.0, -torch.inf), dim=-1)
        m = P.sum(dim=(0, 1)) / ((r1 - r0) * nh)
        for j, s in enumerate(key_slots):
            mass[b, s] += m[j]
    return out.numpy(), mass.numpy(), round_cache(k, dt), round_cache(v, dt)


SHAPES = {
    "f32": Shape("f32", 64, 2, 32, 8, 10000.0),
    "bf16": Shape("bf16", 128, 2, 64, 16, 500000.0),
}

# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------


def test_bf16_rounding_matches_torch_cast_of_float32():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),      # subnormal range
        (rng.standard_normal(2000) * 1e38).astype(np.float32),       # near the top
        # exact ties: low 16 bits 0x8000 on odd and even bf16 mantissas
        (rng.integers(0, 2**15, 2000).astype(np.uint32) << 16 | 0x8000).view(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.3895314e38], np.float32),
    ])
    vals = vals[np.isfinite(vals)]
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = O.f64_to_bf16_bits(vals.astype(np.float64))
    assert np.array_equal(got, ref)


def test_bf16_rounding_is_single_rounding_from_float64():
    # 1 + 2^-8 + 2^-40 lies just above the midpoint of 1 and 1 + 2^-7: the
    # nearest bfloat16 is 1 + 2^-7. Rounding to float32 first lands exactly on
    # the midpoint and ties-to-even would then give 1.0.
    v = np.array([1 + 2.0**-8 + 2.0**-40, -(1 + 2.0**-8 + 2.0**-40), 1 + 2.0**-8, 1 + 3 * 2.0**-8])
    got = O.round_to_bf16(v)
    assert list(got) == [1 + 2.0**-7, -(1 + 2.0**-7), 1.0, 1 + 2.0**-6]
    # overflow to infinity and the largest finite value
    assert np.isinf(O.round_to_bf16(np.array([3.4e38]))[0])
    assert O.round_to_bf16(np.array([(2 - 2.0**-7) * 2.0**127]))[0] == (2 - 2.0**-7) * 2.0**127
    # round-to-odd route agrees on random float64
    rng = np.random.default_rng(2)
    r = rng.standard_normal(50000) * np.exp(rng.uniform(-20, 20, 50000))
    assert np.array_equal(O.f64_to_bf16_bits(r), bf16_round_to_odd(r))


# --------------------------------------------------------------------------
# rotary embedding
# --------------------------------------------------------------------------


@pytest.mark.parametrize("D,theta", [(64, 10000.0), (128, 500000.0), (8, 10.0)])
def test_rope_equals_complex_exponential_form(D, theta):
    rng = np.random.default_rng(3)
    u = rng.standard_normal((9, 3, D))
    pos = np.array([0, 1, 2, 7, 100, 1023, 4096, 8191, 12345])
    got = O.rope(u, pos, theta)
    ref = rope_complex(torch.from_numpy(u), torch.from_numpy(pos), theta).numpy()
    # the two routes round the angle p * theta^(-2i/D) differently: the
    # difference grows with p (about 1 ulp of the angle)
    tol = 1e-15 * (pos + 1.0)[:, None, None] * 4
    assert np.all(np.abs(got - ref) <= tol)


def test_rope_invariants():
    rng = np.random.default_rng(4)
    D = 128
    u = rng.standard_normal((5, 2, D))
    pos = np.array([0, 3, 77, 900, 8000])
    r = O.rope(u, pos, 500000.0)
    assert np.allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(u, axis=-1), rtol=1e-12, atol=0)
    assert np.array_equal(r[0], u[0])                    # position 0 is the identity
    # <R_m q, R_n k> depends only on m - n
    q = rng.standard_normal((1, 1, D))
    k = rng.standard_normal((1, 1, D))
    for m, n, t in [(5, 2, 100), (40, 90, 7), (1000, 0, 3000)]:
        a = (O.rope(q, np.array([m]), 1e4) * O.rope(k, np.array([n]), 1e4)).sum()
        b = (O.rope(q, np.array([m + t]), 1e4) * O.rope(k, np.array([n + t]), 1e4)).sum()
        assert abs(a - b) < 1e-9 * (1 + abs(a))


# --------------------------------------------------------------------------
# softmax
# --------------------------------------------------------------------------


def test_softmax_rows_sum_to_one_and_match_library():
    rng = np.random.default_rng(5)
    S = rng.standard_normal((7, 40)) * 5
    vis = rng.random((7, 40)) < 0.6
    vis[0] = False            # a row with no visible key
    P = O.softmax_rows(S, vis)
    assert np.all(P[0] == 0)
    assert np.allclose(P[1:].sum(1), 1.0, rtol=0, atol=1e-12)
    assert np.all(P[~vis] == 0)
    ref = torch.softmax(torch.from_numpy(np.where(vis, S, -np.inf)[1:]), dim=-1).numpy()
    assert np.allclose(P[1:], ref, rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# the float32-accumulation reading of the projection
# --------------------------------------------------------------------------


def test_f32_accumulated_projection_is_within_the_float32_bound():
    """project_f32acc differs from the exact projection by no more than the
    standard bound for a float32 sum of K exact products, K * 2^-24 *
    sum_k |x_k w_k| (any summation order), and it does differ somewhere."""
    sh = Shape("bf16", 512, 4, 128, 64, 1e4)
    rng = np.random.default_rng(21)
    x = (rng.standard_normal((40, 512))).astype(np.float32)
    w = (rng.standard_normal((512, 1536)) * 0.02).astype(np.float32)
    xb = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    wb = torch.from_numpy(w).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    xv = torch_bf16_value(xb).numpy()
    wv = torch_bf16_value(wb).numpy()
    exact = xv @ wv                                # products of 8-bit significands are exact
    a32 = O.project_f32acc(sh, xb, wb)
    bound = 512 * 2.0 ** -24 * (np.abs(xv) @ np.abs(wv))
    assert np.all(np.abs(a32 - exact) <= bound)
    assert np.any(a32 != exact)
    assert np.allclose(O.project(sh, xb, wb), exact, rtol=0, atol=1e-12)


def test_f32_reading_equals_exact_reading_for_one_hot_rows():
    """With one-hot x (a power of two times one weight row) every projected
    value is exact in float32 too, so both readings give identical steps."""
    sh = SHAPES["bf16"]
    rng = np.random.default_rng(22)
    c = make_case(rng, sh, lens=[30, 41], rows_per_seq=[6, 9])
    R = c["x"].shape[0]
    onehot = np.zeros((R, sh.hidden), np.float32)
    onehot[np.arange(R), rng.integers(0, sh.hidden, R)] = 64.0
    c["x"] = torch.from_numpy(onehot).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    o64 = run_oracle(sh, c)
    o32 = run_oracle(sh, c, accumulate="f32")
    for a, b in zip(o64, o32):
        assert np.array_equal(a, b)
    # dense rows: the readings stay close
    c2 = make_case(rng, sh, lens=[30, 41], rows_per_seq=[6, 9])
    d64 = run_oracle(sh, c2)[0]
    d32 = run_oracle(sh, c2, accumulate="f32")[0]
    assert np.max(np.abs(d64 - d32)) <= 1e-2 * np.sqrt(np.mean(d64 ** 2))


# --------------------------------------------------------------------------
# whole step against brute force
# --------------------------------------------------------------------------


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_step_matches_brute_force_stale_cache(dt):
    """General case: pre-existing cache holds unrelated values (the stale
    keys of the caching approximation); fresh rows replace theirs."""
    sh = SHAPES[dt]
    rng = np.random.default_rng(6)
    c = make_case(rng, sh, lens=[37, 16, 50], rows_per_seq=[5, 16, 9])
    out, mass, kp, vp = run_oracle(sh, c)
    bo, bm, bk, bv = brute_force(sh, c)
    rms = np.sqrt(np.mean(bo ** 2))
    assert np.max(np.abs(out - bo)) <= 1e-11 * rms
    assert np.max(np.abs(mass - bm)) <= 1e-13
    # written slots hold the brute-force k/v bits (same value up to float64
    # summation order; equality is expected on these sizes)
    ps = sh.page_size
    for b in range(3):
        for r in range(c["cu"][b], c["cu"][b + 1]):
            s = c["slots"][r]
            pg = c["bt"][b, s // ps]
            assert np.array_equal(kp[0, pg, :, s % ps, :], bk[r])
            assert np.array_equal(vp[0, pg, :, s % ps, :], bv[r])


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_step_with_prefilled_cache_equals_dense_bidirectional_sdpa(dt):
    """Prefill: a step whose rows are the whole sequence writes its K/V. A
    later step over any subset of those rows then reproduces dense
    bidirectional attention over the full sequence (torch SDPA, float64)."""
    sh = SHAPES[dt]
    rng = np.random.default_rng(7)
    L = 29
    c = make_case(rng, sh, lens=[L], rows_per_seq=[L], extra_pages=1)
    x_full = rand_bits(rng, (L, sh.hidden), dt)
    pre = dict(c, x=x_full, positions=np.arange(L, dtype=np.int32), slots=np.arange(L, dtype=np.int32),
               view=np.zeros(L, np.int8), cu=np.array([0, L], np.int32))
    _, _, kp, vp = run_oracle(sh, pre)
    sub = np.array([2, 3, 11, 28], dtype=np.int32)
    step = dict(pre, kp=kp, vp=vp, x=x_full[sub], positions=sub, slots=sub,
                view=np.zeros(len(sub), np.int8), cu=np.array([0, len(sub)], np.int32))
    out, _, _, _ = run_oracle(sh, step)
    # dense reference straight from x_full
    H, nh, D = sh.hidden, sh.n_heads, sh.head_dim
    a = cache_value(x_full, dt) @ cache_value(c["w"], dt)
    pos = torch.arange(L)
    q = rope_complex(a[:, :H].reshape(L, nh, D), pos, sh.rope_theta)
    k = rope_complex(a[:, H:2 * H].reshape(L, nh, D), pos, sh.rope_theta)
    v = a[:, 2 * H:].reshape(L, nh, D)
    if dt == "bf16":
        q = torch_bf16_value(bf16_round_to_odd(q.numpy()))
    k = cache_value(round_cache(k, dt), dt)
    v = cache_value(round_cache(v, dt), dt)
    o = F.scaled_dot_product_attention(q.permute(1, 0, 2), k.permute(1, 0, 2), v.permute(1, 0, 2))
    ref = o.permute(1, 0, 2).reshape(L, H).numpy()[sub]
    assert np.max(np.abs(out - ref)) <= 1e-11 * np.sqrt(np.mean(ref ** 2))


def test_cache_bytes_outside_written_slots_unchanged():
    sh = SHAPES["bf16"]
    rng = np.random.default_rng(8)
    c = make_case(rng, sh, lens=[40, 70], rows_per_seq=[6, 10], extra_pages=3)
    kp0 = c["kp"].copy()
    vp0 = c["vp"].copy()
    # poison the slots to be written
    ps = sh.page_size
    written = np.zeros(kp0.shape[:2] + (ps,), bool)
    for b in range(2):
        for r in range(c["cu"][b], c["cu"][b + 1]):
            s = c["slots"][r]
            written[0, c["bt"][b, s // ps], s % ps] = True
    kp0.transpose(0, 1, 3, 2, 4)[written] = 0x7FC1
    kp0_in, vp0_in = kp0.copy(), vp0.copy()
    _, _, kp, vp = run_oracle(sh, c, kp=kp0, vp=vp0)
    mask = np.broadcast_to(written[:, :, None, :, None], kp0.shape)
    assert np.array_equal(kp[~mask], kp0[~mask])
    assert np.array_equal(vp[~mask], vp0[~mask])
    assert not np.any(kp[mask] == 0x7FC1)
    # the oracle returns new pools; the arrays it was given are not modified
    assert np.array_equal(kp0, kp0_in)
    assert np.array_equal(vp0, vp0_in)


def test_block_table_permutation_is_pure_indirection():
    sh = SHAPES["bf16"]
    rng = np.random.default_rng(9)
    c = make_case(rng, sh, lens=[33, 60, 18], rows_per_seq=[4, 8, 3], extra_pages=4)
    out, mass, kp, vp = run_oracle(sh, c)
    npg = c["kp"].shape[1]
    perm = rng.permutation(npg)                 # new physical page of old page p
    kp2 = np.empty_like(c["kp"])
    vp2 = np.empty_like(c["vp"])
    kp2[:, perm] = c["kp"]
    vp2[:, perm] = c["vp"]
    bt2 = np.where(c["bt"] >= 0, perm[np.maximum(c["bt"], 0)], -1).astype(np.int32)
    out2, mass2, kq, vq = run_oracle(sh, c, kp=kp2, vp=vp2, bt=bt2)
    assert np.array_equal(out, out2)
    assert np.array_equal(mass, mass2)
    assert np.array_equal(kq[:, perm], kp)


# --------------------------------------------------------------------------
# Flash-Verify two views
# --------------------------------------------------------------------------


def test_two_views_without_context_are_causal_sdpa_each():
    sh = SHAPES["bf16"]
    rng = np.random.default_rng(10)
    n = 6
    c = make_case(rng, sh, lens=[0], rows_per_seq=[0], views=[n], extra_pages=1)
    out, mass, _, _ = run_oracle(sh, c)
    bo, bm, _, _ = brute_force(sh, c)
    assert np.max(np.abs(out - bo)) <= 1e-11 * np.sqrt(np.mean(bo ** 2))
    # each view alone: plain causal attention over its own rows
    H, nh, D = sh.hidden, sh.n_heads, sh.head_dim
    a = cache_value(c["x"], "bf16") @ cache_value(c["w"], "bf16")
    pos = torch.from_numpy(c["positions"].astype(np.int64))
    q = torch_bf16_value(bf16_round_to_odd(rope_complex(a[:, :H].reshape(-1, nh, D), pos, sh.rope_theta).numpy()))
    k = cache_value(round_cache(rope_complex(a[:, H:2 * H].reshape(-1, nh, D), pos, sh.rope_theta), "bf16"), "bf16")
    v = cache_value(round_cache(a[:, 2 * H:].reshape(-1, nh, D), "bf16"), "bf16")
    for lo in (0, n):
        sl = slice(lo, lo + n)
        o = F.scaled_dot_product_attention(q[sl].permute(1, 0, 2), k[sl].permute(1, 0, 2),
                                           v[sl].permute(1, 0, 2), is_causal=True)
        ref = o.permute(1, 0, 2).reshape(n, H).numpy()
        assert np.max(np.abs(out[sl] - ref)) <= 1e-11 * np.sqrt(np.mean(ref ** 2))


def test_two_views_are_isolated():
    sh = SHAPES["bf16"]
    rng = np.random.default_rng(11)
    n = 5
    c = make_case(rng, sh, lens=[21, 40], rows_per_seq=[0, 0], views=[n, n], extra_pages=2)
    out, mass, _, _ = run_oracle(sh, c)
    for b in range(2):
        r0 = c["cu"][b]
        draft = slice(r0, r0 + n)
        maskv = slice(r0 + n, r0 + 2 * n)
        x2 = c["x"].copy()
        x2[maskv] = rand_bits(rng, x2[maskv].shape, "bf16")
        out2, _, _, _ = run_oracle(sh, c, x=x2)
        assert np.array_equal(out2[draft], out[draft])
        assert not np.array_equal(out2[maskv], out[maskv])
        x3 = c["x"].copy()
        x3[draft] = rand_bits(rng, x3[draft].shape, "bf16")
        out3, _, _, _ = run_oracle(sh, c, x=x3)
        assert np.array_equal(out3[maskv], out[maskv])
    bo, bm, _, _ = brute_force(sh, c)
    assert np.max(np.abs(out - bo)) <= 1e-11 * np.sqrt(np.mean(bo ** 2))
    assert np.max(np.abs(mass - bm)) <= 1e-13


# --------------------------------------------------------------------------
# attention mass and top-k
# --------------------------------------------------------------------------


def test_mass_sums_to_one_per_sequence():
    sh = SHAPES["f32"]
    rng = np.random.default_rng(12)
    c = make_case(rng, sh, lens=[17, 64, 30], rows_per_seq=[3, 12, 30])
    _, mass, _, _ = run_oracle(sh, c)
    assert np.allclose(mass.sum(1), 1.0, rtol=0, atol=1e-12)
    assert np.all(mass >= 0)
    for b, L in enumerate(c["lens"]):
        assert np.all(mass[b, L:] == 0)


def test_uniform_keys_give_uniform_probabilities():
    """With every key vector equal, every score ties: P is uniform, out is
    the mean of the visible values, the mass is 1/L per slot, and the top-k
    set is the k lowest slots."""
    sh = SHAPES["f32"]
    rng = np.random.default_rng(13)
    L = 40
    c = make_case(rng, sh, lens=[L], rows_per_seq=[1], extra_pages=0)
    # one row; W's K block zero so its fresh key is 0; cache keys all 0 too
    w = c["w"].view(np.float32).copy()
    w[:, sh.hidden:2 * sh.hidden] = 0
    kp = np.zeros_like(c["kp"])
    out, mass, kq, vq = run_oracle(sh, c, w=w.view(np.uint32), kp=kp)
    ps = sh.page_size
    vals = np.stack([O.decode(vq[0, c["bt"][0, s // ps], :, s % ps, :], "f32") for s in range(L)])
    assert np.allclose(out[0], vals.mean(0).reshape(-1), rtol=0, atol=1e-12)
    assert np.allclose(mass[0, :L], 1.0 / L, rtol=0, atol=1e-15)
    top = O.select_tracked(mass.astype(np.float32), c["lens"], 5)
    assert list(top[0]) == [0, 1, 2, 3, 4]


def test_select_tracked_brute_force():
    rng = np.random.default_rng(14)
    for trial in range(30):
        B = 4
        stride = 50
        lens = rng.integers(0, stride + 1, B)
        # few distinct values so ties are common
        mass = rng.integers(0, 6, (B, stride)).astype(np.float32) / 7
        k = int(rng.integers(1, 60))
        ex_cu = np.zeros(B + 1, np.int32)
        ex = []
        for b in range(B):
            e = rng.choice(max(int(lens[b]), 1), size=min(3, int(lens[b])), replace=False) if lens[b] else []
            ex.append(np.asarray(e, np.int32))
            ex_cu[b + 1] = ex_cu[b] + len(e)
        ex_s = np.concatenate(ex).astype(np.int32) if ex else np.zeros(0, np.int32)
        got = O.select_tracked(mass, lens, k, ex_cu, ex_s)
        for b in range(B):
            cands = [j for j in range(int(lens[b])) if j not in set(ex[b].tolist())]
            ref = sorted(cands, key=lambda j: (-float(mass[b, j]), j))[:k]
            ref = ref + [-1] * (k - len(ref))
            assert list(got[b]) == ref


# --------------------------------------------------------------------------
# planted mistakes: each must be caught by one of the pins above
# --------------------------------------------------------------------------


def _rope_wrong_sign(u, positions, theta):
    R, nh, D = u.shape
    half = D // 2
    inv = theta ** (-2.0 * np.arange(half) / D)
    phi = np.asarray(positions, np.float64)[:, None] * inv[None, :]
    c, s = np.cos(phi)[:, None, :], np.sin(phi)[:, None, :]
    a, b = u[..., :half], u[..., half:]
    return np.concatenate([a * c + b * s, b * c - a * s], axis=-1)


def _rope_interleaved(u, positions, theta):
    R, nh, D = u.shape
    inv = theta ** (-2.0 * np.arange(D // 2) / D)
    phi = np.asarray(positions, np.float64)[:, None] * inv[None, :]
    c, s = np.cos(phi)[:, None, :], np.sin(phi)[:, None, :]
    a, b = u[..., 0::2], u[..., 1::2]
    outp = np.empty_like(u)
    outp[..., 0::2] = a * c - b * s
    outp[..., 1::2] = b * c + a * s
    return outp


@pytest.mark.parametrize("mutant", ["rope_sign", "rope_interleaved", "q_not_rotated",
                                    "no_view_isolation", "mass_no_head_mean",
                                    "softmax_ignores_mask", "scale_missing"])
def test_planted_oracle_mistakes_are_caught(monkeypatch, mutant):
    sh = SHAPES["bf16"]
    rng = np.random.default_rng(15)
    c = make_case(rng, sh, lens=[25, 30], rows_per_seq=[4, 0], views=[None, 4], extra_pages=1)
    bo, bm, _, _ = brute_force(sh, c)
    if mutant == "rope_sign":
        monkeypatch.setattr(O, "rope", _rope_wrong_sign)
    elif mutant == "rope_interleaved":
        monkeypatch.setattr(O, "rope", _rope_interleaved)
    elif mutant == "no_view_isolation":
        orig = O.visible_keys

        def leaky(L, view, positions, slots):
            keys, vis = orig(L, view, positions, slots)
            vis[:, L:] = True
            return keys, vis
        monkeypatch.setattr(O, "visible_keys", leaky)
    elif mutant == "mass_no_head_mean":
        # the oracle's own normalisation forgets the heads: a mean over rows only
        monkeypatch.setattr(O, "mass_weight", lambda n_rows, n_heads: 1.0 / n_rows)
    elif mutant == "q_not_rotated":
        orig_rope = O.rope
        calls = []

        def rope_k_only(u, positions, theta):
            calls.append(1)
            return u if len(calls) % 2 == 1 else orig_rope(u, positions, theta)
        monkeypatch.setattr(O, "rope", rope_k_only)
    elif mutant == "softmax_ignores_mask":
        orig_sm = O.softmax_rows
        monkeypatch.setattr(O, "softmax_rows", lambda S, vis: orig_sm(S, np.ones_like(vis)))
    elif mutant == "scale_missing":
        orig_sm = O.softmax_rows
        monkeypatch.setattr(O, "softmax_rows", lambda S, vis: orig_sm(S * np.sqrt(sh.head_dim), vis))
    out, mass, _, _ = O.layer_step(sh, c["kp"], c["vp"], 0, c["x"], c["w"], c["positions"], c["slots"],
                                   c["cu"], c["lens"], c["bt"], c["view"])
    err_out = np.max(np.abs(out - bo)) / np.sqrt(np.mean(bo ** 2))
    err_mass = np.max(np.abs(mass - bm))
    assert err_out > 1e-9 or err_mass > 1e-12
