"""GPU parity of a chained stack (kv_cache_attention_flash_b200.stack):
per layer the fused step with bf16 out, then x_{l+1} = x_l + out_l W_o,l,
against the same chain run entirely in the oracle (layer_step, bf16
rounding of out, oproj with the residual, bf16 rounding of x).

Inputs: x_0 and every Wqkv on the grids on which the fp32 projection is
exact (workloads.make_x_grid), so layer 0 has one correct result; the
residual stream of later layers is off the grid.

Tolerances: layer 0's out (bf16) meets the plain 1e-2 x RMS bar plus half
a bf16 ulp of the value (its own rounding) against the oracle's. A later
layer meets the same bar, or, where its input already carries earlier
layers' one-ulp rounding differences, the bar plus twice the spread that
the oracle's own chain shows at that layer when every out is rounded
toward zero instead of to nearest (every code off by at most one ulp). The
final residual stream x_L is compared as its change over the stack,
x_L - x_0, within 1e-2 x RMS of that change plus one bf16 ulp of x_L per
layer, plus, where that is exceeded, twice the one-ulp chain's movement of
the stream (each layer rounds the stream to bf16 once; the two chains may
round a value on opposite sides of a midpoint)."""
import numpy as np
import pytest
import torch

import kv_cache_attention_flash_b200 as fd
from kv_cache_attention_flash_b200 import workloads as W
from kv_cache_attention_flash_b200.stack import LayerStack
from oracle import oracle as O

pytestmark = pytest.mark.gpu


def bf16_ulp(v):
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def bf16_bits_toward_zero(v):
    """bf16 bits of float64 values rounded toward zero (test helper)."""
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(a, 2.0 ** -126))) - 7)
    t = np.copysign(np.floor(a / ulp) * ulp, v)
    return (t.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def run_chain(name, n_layers, seed=0):
    spec = W.get_spec(name)
    sh = spec.shape
    meta = W.make_meta(spec, seed)
    dev = "cuda"
    kp, vp = W.make_pools(spec, meta, seed, n_layers=n_layers)
    # x_0 and Wqkv on the grids where the fp32 projection is exact (layer 0
    # then has one correct bf16 code per fresh value); later layers' x is
    # the residual stream and leaves the grid
    x0 = W.make_x_grid(spec, meta, seed)
    ws = [W.make_w_grid(spec, seed, layer=l) for l in range(n_layers)]
    wos = [W.make_w_o(spec, seed, layer=l) for l in range(n_layers)]
    ps = sh.page_size
    cache = fd.FlashCache(n_layers, sh.n_heads, sh.head_dim, ps, meta.num_pages,
                          meta.max_position, sh.rope_theta, sh.dtype, max_batch=meta.batch,
                          max_slots_per_seq=meta.max_blocks * ps, k_pool=kp.to(dev),
                          v_pool=vp.to(dev))
    stack = LayerStack(cache, [w.to(dev) for w in ws], [w.to(dev) for w in wos])
    mass = torch.empty(meta.batch, meta.max_blocks * ps, dtype=torch.float32, device=dev)
    outs = {}
    x0d = x0.to(dev)
    xl, _ = stack.run(meta.cu_rows, meta.seq_lens, x0d, torch.from_numpy(meta.positions).to(dev),
                      torch.from_numpy(meta.block_table).to(dev),
                      torch.from_numpy(meta.view).to(dev), torch.from_numpy(meta.slots).to(dev),
                      mass, x_out=torch.empty_like(x0d), outs=outs)
    cache.check()
    torch.cuda.synchronize()
    assert stack.launches == 3 * n_layers
    assert torch.equal(x0d.cpu(), x0)          # x_0 is left as it was
    g_outs = {l: o.float().cpu().numpy() for l, o in outs.items()}
    g_x = xl.float().cpu().numpy()
    g_mass = mass.cpu().numpy()
    cache.close()

    # the oracle's chain
    def oracle_chain(round_out):
        kb, vb = W.bits_np(kp), W.bits_np(vp)
        xb = W.bits_np(x0)
        outs = {}
        for l in range(n_layers):
            o_out, o_mass, kb, vb = O.layer_step(sh, kb, vb, l, xb, W.bits_np(ws[l]),
                                                 meta.positions, meta.slots, meta.cu_rows,
                                                 meta.seq_lens, meta.block_table, meta.view)
            outs[l] = o_out
            ob = round_out(o_out)
            xb = O.f64_to_bf16_bits(O.oproj(ob, W.bits_np(wos[l]), xb))
        return outs, O.bf16_bits_to_f64(xb), o_mass

    o_outs, o_x, o_mass = oracle_chain(O.f64_to_bf16_bits)
    # The GPU rounds an fp32 out to bf16, the oracle an fp64 one: where the
    # two lie on either side of a midpoint their codes differ by one ulp, and
    # the next layer's input moves with them. The same chain with every out
    # rounded toward zero (each code off by at most one ulp) shows how far
    # such one-ulp changes carry to the next layer.
    alt = {}

    def o_alt(l):
        """layer l's out in the one-ulp chain (l = "x": its final stream)."""
        if not alt:
            outs_t, x_t, _ = oracle_chain(bf16_bits_toward_zero)
            alt.update(outs_t)
            alt["x"] = x_t
        return alt[l]
    return spec, g_outs, g_x, g_mass, o_outs, o_alt, o_x, x0, o_mass


def check_chain(spec, g_outs, g_x, g_mass, o_outs, o_alt, o_x, x0, o_mass, n_layers):
    for l in range(n_layers):
        ref = o_outs[l]
        rms = float(np.sqrt(np.mean(ref ** 2)))
        diff = np.abs(g_outs[l] - ref)
        # out is bf16 here: half a bf16 ulp of its own rounding on top of the bar
        excess = float(np.max(diff - 0.5001 * bf16_ulp(ref)))
        print(f"[parity] {spec.name} layer {l}: out max(|err| - ulp/2)/RMS = {excess / rms:.3e}")
        if excess > 1e-2 * rms:
            # after the first layer: the input already carries the previous
            # layers' one-ulp rounding differences
            assert l > 0, f"layer 0: out off by {excess / rms:.3e} x RMS"
            spread = float(np.max(np.abs(o_alt(l) - ref)))
            print(f"[parity] {spec.name} layer {l}: one-ulp chain spread {spread / rms:.3e} x RMS")
            assert excess <= 1e-2 * rms + 2.0 * spread, f"layer {l}: out off by {excess / rms:.3e}"
    x0v = x0.double().numpy()
    d_ref = o_x - x0v
    d_rms = float(np.sqrt(np.mean(d_ref ** 2)))
    diff = np.abs(g_x - o_x)
    bound = 1e-2 * d_rms + n_layers * bf16_ulp(o_x)
    print(f"[parity] {spec.name}: residual stream max|err| = {diff.max():.3e}, change RMS "
          f"{d_rms:.3e}")
    if np.any(diff > bound):
        # the stream carries the layers' one-ulp rounding differences: the
        # one-ulp chain's distance from the oracle's shows how far they go
        spread = float(np.max(np.abs(o_alt("x") - o_x)))
        print(f"[parity] {spec.name}: one-ulp chain moves the stream by up to {spread:.3e}")
        bound = bound + 2.0 * spread
    assert np.all(diff <= bound), f"{int((diff > bound).sum())} elements of x_L off"
    md = np.abs(g_mass - o_mass)
    assert np.all(md <= 1e-3 * np.abs(o_mass) + 1e-6), f"last-layer mass off by {md.max():.3e}"


def test_chained_stack_small():
    r = run_chain("small_bf16_chained", 4)
    check_chain(*r, 4)


def test_chained_stack_full_size_first_layers():
    """The 32-layer, batch-4, 8192-slot stack at full size, chained: its
    first two layers against the oracle's chain."""
    r = run_chain("stacked32_b4_chained", 2)
    check_chain(*r, 2)
