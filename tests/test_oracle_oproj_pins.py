"""Pins of the oracle's output projection y = o W_o, checked against things
other than itself: special matrices with a known product, a brute-force
triple loop on tiny sizes, and the head-block structure of o.
Each planted mistake at the end must break at least one pin.
"""
import numpy as np
import pytest

from oracle import oracle as O


def _bits(v):
    return O.f64_to_bf16_bits(np.asarray(v, np.float64))


def _rand_bf16(rng, shape, scale=1.0):
    return _bits(rng.standard_normal(shape) * scale)


def pin_identity() -> bool:
    rng = np.random.default_rng(1)
    o = _rand_bf16(rng, (5, 16))
    y = O.oproj(o, _bits(np.eye(16)))
    return bool(np.array_equal(y, O.bf16_bits_to_f64(o)))


def pin_permutation() -> bool:
    # W_o with W[i, perm[i]] = 1 sends column i of o to column perm[i] of y
    rng = np.random.default_rng(2)
    H = 24
    perm = rng.permutation(H)
    w = np.zeros((H, H))
    w[np.arange(H), perm] = 1.0
    o = _rand_bf16(rng, (7, H))
    y = O.oproj(o, _bits(w))
    ov = O.bf16_bits_to_f64(o)
    want = np.empty_like(ov)
    want[:, perm] = ov
    return bool(np.array_equal(y, want))


def pin_brute_force() -> bool:
    rng = np.random.default_rng(3)
    R, H = 3, 8
    o = _rand_bf16(rng, (R, H))
    w = _rand_bf16(rng, (H, H), 0.02)
    ov, wv = O.bf16_bits_to_f64(o), O.bf16_bits_to_f64(w)
    y = O.oproj(o, w)
    ok = True
    for r in range(R):
        for n in range(H):
            acc = 0.0
            for k in range(H):
                acc += ov[r, k] * wv[k, n]
            ok &= abs(y[r, n] - acc) <= 1e-12 * max(1.0, abs(acc))
    return bool(ok)


def pin_head_blocks() -> bool:
    # W_o block diagonal over heads: y's head h depends on o's head h only
    rng = np.random.default_rng(4)
    nh, D = 4, 8
    H = nh * D
    w = np.zeros((H, H))
    blocks = [rng.standard_normal((D, D)) * 0.1 for _ in range(nh)]
    for h in range(nh):
        w[h * D:(h + 1) * D, h * D:(h + 1) * D] = blocks[h]
    wb = _bits(w)
    o = _rand_bf16(rng, (6, H))
    y = O.oproj(o, wb)
    ov, wv = O.bf16_bits_to_f64(o), O.bf16_bits_to_f64(wb)
    ok = True
    for h in range(nh):
        sl = slice(h * D, (h + 1) * D)
        ok &= bool(np.allclose(y[:, sl], ov[:, sl] @ wv[sl, sl], rtol=1e-12, atol=1e-14))
    return ok


def pin_residual_zero_weight() -> bool:
    # W_o = 0: y is the residual row exactly
    rng = np.random.default_rng(5)
    r = _rand_bf16(rng, (4, 16))
    o = _rand_bf16(rng, (4, 16))
    y = O.oproj(o, _bits(np.zeros((16, 16))), r)
    return bool(np.array_equal(y, O.bf16_bits_to_f64(r)))


def pin_residual_brute_force() -> bool:
    # residual + o W_o by a triple loop, each residual element added once
    rng = np.random.default_rng(6)
    R, H = 3, 8
    o = _rand_bf16(rng, (R, H))
    w = _rand_bf16(rng, (H, H), 0.02)
    r = _rand_bf16(rng, (R, H))
    ov, wv, rv = O.bf16_bits_to_f64(o), O.bf16_bits_to_f64(w), O.bf16_bits_to_f64(r)
    y = O.oproj(o, w, r)
    ok = True
    for i in range(R):
        for n in range(H):
            acc = rv[i, n]
            for k in range(H):
                acc += ov[i, k] * wv[k, n]
            ok &= abs(y[i, n] - acc) <= 1e-12 * max(1.0, abs(acc))
    return bool(ok)


PINS = [pin_identity, pin_permutation, pin_brute_force, pin_head_blocks, pin_residual_zero_weight,
        pin_residual_brute_force]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oproj_pin(pin):
    assert pin()


def _with_residual(y, residual_bits):
    return y if residual_bits is None else y + O.bf16_bits_to_f64(residual_bits)


def _transposed(out_bits, w_bits, residual_bits=None):
    return _with_residual(O.bf16_bits_to_f64(out_bits) @ O.bf16_bits_to_f64(w_bits).T,
                          residual_bits)


def _dropped_k(out_bits, w_bits, residual_bits=None):
    o, w = O.bf16_bits_to_f64(out_bits), O.bf16_bits_to_f64(w_bits)
    return _with_residual(o[:, :-1] @ w[:-1, :], residual_bits)


def _bf16_rounded(out_bits, w_bits, residual_bits=None):
    return _with_residual(O.round_to_bf16(O.bf16_bits_to_f64(out_bits) @ O.bf16_bits_to_f64(w_bits)),
                          residual_bits)


def _residual_dropped(out_bits, w_bits, residual_bits=None):
    return O.bf16_bits_to_f64(out_bits) @ O.bf16_bits_to_f64(w_bits)


def _residual_twice(out_bits, w_bits, residual_bits=None):
    y = O.bf16_bits_to_f64(out_bits) @ O.bf16_bits_to_f64(w_bits)
    return _with_residual(_with_residual(y, residual_bits), residual_bits)


@pytest.mark.parametrize("mutant", [_transposed, _dropped_k, _bf16_rounded, _residual_dropped,
                                    _residual_twice],
                         ids=lambda f: f.__name__)
def test_planted_oproj_mistakes_are_caught(monkeypatch, mutant):
    monkeypatch.setattr(O, "oproj", mutant)
    assert not all(p() for p in PINS)
