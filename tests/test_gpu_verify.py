"""GPU parity of the Flash-Verify acceptance step against the oracle.

Predictions must match exactly (the argmax is decided on the stored logit
values on both sides, ties to the lowest token id). Confidences must be
within 1e-5 relative of the float64 oracle (fp32 accumulation of up to
~1e5 exponentials). The accepted length must equal the oracle's scan over
the kernel's own fp32 confidences (the threshold decision taken in the
kernel's precision), and also the oracle's float64 decision wherever no
confidence lies within 1e-5 of the threshold.
"""
import numpy as np
import pytest
import torch

import kv_cache_attention_flash_b200 as fd
from kv_cache_attention_flash_b200 import workloads as W
from oracle import oracle as O

pytestmark = pytest.mark.gpu


def _check(logits, cu, draft, tau):
    dev = "cuda"
    lg = logits.to(dev)
    pred, conf, nacc = fd.fdllm_verify_accept(lg, torch.from_numpy(cu).to(dev),
                                              torch.from_numpy(draft).to(dev), tau)
    torch.cuda.synchronize()
    pred, conf, nacc = pred.cpu().numpy(), conf.cpu().numpy(), nacc.cpu().numpy()
    dtype = "bf16" if logits.dtype == torch.bfloat16 else "f32"
    o_pred, o_conf = O.verify_rows(W.bits_np(logits), dtype)
    assert np.array_equal(pred, o_pred), "prediction differs"
    assert np.all(np.abs(conf - o_conf) <= 1e-5 * o_conf), f"conf off by {np.max(np.abs(conf - o_conf) / o_conf):.2e}"
    same_prec = O.verify_accept(o_pred, conf, draft, cu, np.float32(tau))
    assert np.array_equal(nacc, same_prec), "accepted length differs (kernel precision)"
    if not np.any(np.abs(o_conf - tau) <= 1e-5):
        assert np.array_equal(nacc, O.verify_accept(o_pred, o_conf, draft, cu, tau))
    return nacc


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_verify_small(seed):
    spec = W.VERIFY_WORKLOADS["verify_small"]
    logits, cu, draft = W.make_verify(spec, seed)
    nacc = _check(logits, cu, draft, spec.tau)
    assert 0 <= nacc.min() and nacc.max() <= spec.rows


def test_verify_full_size_sampled():
    """The LLaDA-vocabulary workload (8 x 32 rows, 126464 tokens, bf16)."""
    spec = W.VERIFY_WORKLOADS["verify_b8"]
    logits, cu, draft = W.make_verify(spec, 0, device="cuda")
    nacc = _check(logits.cpu(), cu, draft, spec.tau)
    assert nacc.sum() > 0


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("vocab", [1, 7, 333, 2050])
def test_verify_odd_vocab_and_ties(dtype, vocab):
    """Vocabulary sizes that are not a multiple of the 16-byte load (scalar
    path), logits on a coarse grid (many exact ties), fp32 and bf16."""
    rng = np.random.default_rng(vocab)
    R = 10
    vals = (rng.integers(-4, 5, (R, vocab)) * 0.5).astype(np.float32)
    logits = torch.from_numpy(vals).to(torch.bfloat16 if dtype == "bf16" else torch.float32)
    cu = np.array([0, 3, 3, 10], np.int32)
    pred, _ = O.verify_rows(W.bits_np(logits), dtype)
    draft = np.where(rng.random(R) < 0.7, pred, (pred + 1) % vocab).astype(np.int32)
    _check(logits, cu, draft, 0.0)
    _check(logits, cu, draft, 0.3)


def test_verify_neg_inf_and_thresholds():
    """Rows with -inf logits, a threshold of 0 (agreement alone decides) and
    1 (nothing is accepted)."""
    rng = np.random.default_rng(9)
    R, V = 8, 640
    vals = rng.normal(0, 1, (R, V)).astype(np.float32)
    vals[:, ::3] = -np.inf
    vals[np.arange(R), 1 + 3 * np.arange(R)] += 6.0
    logits = torch.from_numpy(vals).to(torch.bfloat16)
    cu = np.array([0, 8], np.int32)
    pred, _ = O.verify_rows(W.bits_np(logits), "bf16")
    draft = pred.copy()
    draft[5] = (draft[5] + 1) % V
    assert _check(logits, cu, draft, 0.0)[0] == 5
    assert _check(logits, cu, draft, 1.0)[0] == 0


def test_verify_empty_batch_rows():
    logits = torch.zeros(0, 16, dtype=torch.bfloat16)
    dev = "cuda"
    cu = torch.zeros(3, dtype=torch.int32, device=dev)
    pred = torch.zeros(1, dtype=torch.int32, device=dev)
    conf = torch.zeros(1, dtype=torch.float32, device=dev)
    _, _, nacc = fd.fdllm_verify_accept(logits.to(dev), cu, torch.zeros(1, dtype=torch.int32, device=dev),
                                        0.5, pred=pred, conf=conf)
    torch.cuda.synchronize()
    assert nacc.cpu().tolist() == [0, 0]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("vocab", [50000, 50003, 126464])
def test_verify_large_vocab_ties_far_apart(dtype, vocab):
    """Few rows over a large vocabulary, logits on a coarse grid with three
    equal largest logits far apart in each row (the lowest id must win
    across the threads and warps that saw them); an odd vocabulary takes
    the scalar path."""
    rng = np.random.default_rng(vocab + (dtype == "f32"))
    R = 6
    vals = (rng.integers(-6, 7, (R, vocab)) * 0.5).astype(np.float32)
    # equal largest logits in different slices: the lowest id must win
    top = float(vals.max()) + 1.0
    for r in range(R):
        cols = np.sort(rng.choice(vocab, size=3, replace=False))
        vals[r, cols] = top
    logits = torch.from_numpy(vals).to(torch.bfloat16 if dtype == "bf16" else torch.float32)
    cu = np.array([0, 2, 6], np.int32)
    pred, _ = O.verify_rows(W.bits_np(logits), dtype)
    draft = np.where(rng.random(R) < 0.8, pred, (pred + 1) % vocab).astype(np.int32)
    _check(logits, cu, draft, 0.0)
