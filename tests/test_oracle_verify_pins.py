"""Pins of the oracle's Flash-Verify acceptance, checked against things
other than itself.

"Flash-dLLM: I/O-Aware KV Caching and Parallel Decoding for Fast,
Memory-Efficient Diffusion LLMs" (ai4snews summary of the full text),
paragraph 3: a block position is accepted only when the draft view and the
mask view agree and the mask view's confidence exceeds a threshold;
acceptance runs in causal order and stops at the first position that fails.

Pins:
  * prediction and confidence against torch's argmax (first maximal index)
    and float64 softmax, on logits with many exact ties;
  * closed forms: uniform logits give token 0 with confidence 1/V; one
    raised logit x gives e^x / (e^x + V - 1);
  * the accepted length against an independent formulation (the length of
    the all-true prefix, via a cumulative product) over every pass/fail
    pattern of short blocks;
  * the threshold is strict: a confidence equal to it is rejected.
Each planted mistake at the end must break at least one pin.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O


def _bf16_bits(v: np.ndarray) -> np.ndarray:
    return O.f64_to_bf16_bits(np.asarray(v, np.float64))


def pin_rows_vs_torch() -> bool:
    rng = np.random.default_rng(3)
    ok = True
    for dtype in ("bf16", "f32"):
        R, V = 24, 57
        vals = rng.integers(-6, 7, (R, V)) * 0.5     # coarse grid: many exact ties
        vals[3] = 1.25                                # a row of all-equal logits
        bits = _bf16_bits(vals) if dtype == "bf16" else O.f64_to_f32_bits(vals)
        pred, conf = O.verify_rows(bits, dtype)
        t = torch.from_numpy(O.decode(bits, dtype))
        ok &= bool(np.array_equal(pred, torch.argmax(t, dim=1).numpy()))
        ref = torch.softmax(t, dim=1).max(dim=1).values.numpy()
        ok &= bool(np.allclose(conf, ref, rtol=1e-12, atol=0))
    return ok


def pin_closed_forms() -> bool:
    V = 100
    ok = True
    pred, conf = O.verify_rows(_bf16_bits(np.zeros((1, V))), "bf16")
    ok &= int(pred[0]) == 0 and abs(conf[0] - 1.0 / V) < 1e-15
    for j, x in ((0, 3.0), (57, 0.5), (99, 8.0)):
        row = np.zeros((1, V))
        row[0, j] = x
        pred, conf = O.verify_rows(_bf16_bits(row), "bf16")
        want = math.exp(x) / (math.exp(x) + V - 1)
        ok &= int(pred[0]) == j and abs(conf[0] - want) < 1e-14
    return ok


def pin_prefix_formulation() -> bool:
    ok = True
    for n in range(0, 6):
        for agree in itertools.product([0, 1], repeat=n):
            for high in itertools.product([0, 1], repeat=n):
                pred = np.arange(n, dtype=np.int32)
                draft = np.where(np.asarray(agree, bool), pred, pred + 1).astype(np.int32)
                conf = np.where(np.asarray(high, bool), 0.9, 0.1)
                got = O.verify_accept(pred, conf, draft, np.array([0, n]), 0.5)[0]
                passes = (np.asarray(agree, int) * np.asarray(high, int)) if n else np.zeros(0, int)
                want = int(np.cumprod(passes).sum()) if n else 0
                ok &= int(got) == want
    # several sequences at once: the same rule per sequence
    rng = np.random.default_rng(5)
    cu = np.array([0, 4, 4, 9, 16])
    pred = rng.integers(0, 3, 16).astype(np.int32)
    draft = rng.integers(0, 3, 16).astype(np.int32)
    conf = rng.random(16)
    got = O.verify_accept(pred, conf, draft, cu, 0.3)
    for b in range(4):
        p = ((pred == draft) & (conf > 0.3))[cu[b]:cu[b + 1]].astype(int)
        ok &= int(got[b]) == int(np.cumprod(p).sum())
    return ok


def pin_strict_threshold() -> bool:
    pred = np.array([2, 2], np.int32)
    draft = np.array([2, 2], np.int32)
    conf = np.array([0.75, 0.5])
    return (int(O.verify_accept(pred, conf, draft, np.array([0, 2]), 0.5)[0]) == 1 and
            int(O.verify_accept(pred, conf, draft, np.array([0, 2]), 0.4)[0]) == 2)


PINS = [pin_rows_vs_torch, pin_closed_forms, pin_prefix_formulation, pin_strict_threshold]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_verify_pin(pin):
    assert pin()


# --------------------------------------------------------------------------
# planted mistakes
# --------------------------------------------------------------------------

def _rows_last_max(logits_bits, dtype):
    lg = O.decode(logits_bits, dtype)
    pred = np.array([int(np.flatnonzero(r == r.max())[-1]) for r in lg], np.int32)
    conf = np.array([1.0 / np.sum(np.exp(r - r.max())) for r in lg])
    return pred, conf


def _rows_unnormalised(logits_bits, dtype):
    lg = O.decode(logits_bits, dtype)
    pred = np.array([int(np.flatnonzero(r == r.max())[0]) for r in lg], np.int32)
    return pred, np.exp(lg.max(axis=1))


def _accept_no_stop(pred, conf, draft, cu_rows, tau):
    B = len(cu_rows) - 1
    return np.array([int(((pred == draft) & (conf > tau))[cu_rows[b]:cu_rows[b + 1]].sum())
                     for b in range(B)], np.int32)


def _accept_ge(pred, conf, draft, cu_rows, tau):
    B = len(cu_rows) - 1
    out = np.zeros(B, np.int32)
    for b in range(B):
        for i in range(int(cu_rows[b]), int(cu_rows[b + 1])):
            if pred[i] == draft[i] and conf[i] >= tau:
                out[b] += 1
            else:
                break
    return out


@pytest.mark.parametrize("mutant", ["argmax_last", "conf_unnormalised", "no_stop", "ge_threshold"])
def test_planted_verify_mistakes_are_caught(monkeypatch, mutant):
    if mutant == "argmax_last":
        monkeypatch.setattr(O, "verify_rows", _rows_last_max)
    elif mutant == "conf_unnormalised":
        monkeypatch.setattr(O, "verify_rows", _rows_unnormalised)
    elif mutant == "no_stop":
        monkeypatch.setattr(O, "verify_accept", _accept_no_stop)
    elif mutant == "ge_threshold":
        monkeypatch.setattr(O, "verify_accept", _accept_ge)
    assert not all(p() for p in PINS)
