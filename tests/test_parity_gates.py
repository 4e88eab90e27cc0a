"""The gradient gates of tests/parity.py on the CPU: a model of the backward
kernel's arithmetic (P and dS rounded to bf16 before their products, every
product summed in fp32, D from the bf16-rounded O) stays inside the
componentwise bound 2u A and the norm-wise gates against the fp64 oracle, and
plausible mistakes (a gradient scaled by 1.02, a term dropped, D left out)
fail them."""
import numpy as np
import pytest

import oracle
import parity
import synth


def _bf16(x):
    """Round float32 values to bf16 (nearest even), returned as float32."""
    b = np.asarray(x, np.float32).view(np.uint32)
    r = ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)) << np.uint32(16)
    return r.astype(np.uint32).view(np.float32)


def _model_grads(w, inp, dout, drop_D=False):
    """The kernel's rounding steps, per head, on causal attention over all
    visible keys (lambda = 0)."""
    f32 = lambda a: (a.astype(np.uint32) << 16).view(np.float32)
    B, Hq, Lq, d = inp.q.shape
    g = w.Hq // w.Hkv
    scale = np.float32(1.0 / np.sqrt(d))
    dq = np.zeros((B, Hq, Lq, d), np.float64)
    dk = np.zeros((B, w.Hkv, w.Lkv, d), np.float64)
    dv = np.zeros_like(dk)
    keys = np.arange(w.Lkv)
    rows = np.arange(Lq)
    for b in range(B):
        for h in range(Hq):
            q, k, v, do = (f32(t) for t in (inp.q[b, h], inp.k[b, h // g], inp.v[b, h // g], dout[b, h]))
            s = (q @ k.T).astype(np.float32) * scale
            keep = keys[None, :] <= rows[:, None] + (w.Lkv - w.Lq)
            s = np.where(keep, s, -np.inf).astype(np.float32)
            lse = (np.log(np.exp((s - s.max(1, keepdims=True)).astype(np.float64)).sum(1))
                   + s.max(1)).astype(np.float32)
            p32 = np.exp(s - lse[:, None]).astype(np.float32)
            o = _bf16((_bf16(p32) @ v).astype(np.float32))
            D = np.float32(0.0) if drop_D else np.sum(do * o, axis=1, keepdims=True, dtype=np.float32)
            dp = (do @ v.T).astype(np.float32)
            ds = _bf16((p32 * (dp - D)).astype(np.float32))
            dv[b, h // g] += (_bf16(p32).T @ do).astype(np.float32)
            dk[b, h // g] += (scale * (ds.T @ q)).astype(np.float32)
            dq[b, h] = (scale * (ds @ k)).astype(np.float32)
    return dq, dk, dv


W = synth.CONFIGS["prefill_32k"].replace(name="gate_model", Hq=4, Hkv=2, Lq=384, Lkv=384,
                                         window=128, n_needles=1)


@pytest.fixture(scope="module")
def case():
    inp = synth.generate(W)
    dout = synth.grad_output(W)
    ref = oracle.backward(inp.q, inp.k, inp.v, dout, causal=True, Br=W.Br, Bc=W.Bc)
    scales = parity.grad_abs_scales(inp.q, inp.k, inp.v, dout, causal=True,
                                    scale=1.0 / np.sqrt(W.d), tile_mask=None, Br=W.Br, Bc=W.Bc)
    return inp, dout, ref, scales


def test_rounding_model_fits_the_gates(case):
    inp, dout, ref, scales = case
    model = _model_grads(W, inp, dout)
    for name, g, r, a in zip(("dq", "dk", "dv"), model, ref, scales):
        e = parity.assert_grad_within(g, r, name, abs_scale=a)
        assert e["abs_excess"] < 0.6, (name, e)  # well inside the bound


def test_gates_reject_plausible_mistakes(case):
    inp, dout, ref, scales = case
    dq, dk, dv = _model_grads(W, inp, dout)
    with pytest.raises(AssertionError):
        parity.assert_grad_within(dk * 1.02, ref[1], "dk x 1.02", abs_scale=scales[1])
    with pytest.raises(AssertionError):
        parity.assert_grad_within(dv * 1.02, ref[2], "dv x 1.02", abs_scale=scales[2])
    bad = _model_grads(W, inp, dout, drop_D=True)
    with pytest.raises(AssertionError):
        parity.assert_grad_within(bad[0], ref[0], "dq without D", abs_scale=scales[0])


def test_sampled_scales_equal_the_full_ones(case):
    inp, dout, _, (aq, ak, av) = case
    rows = np.array([5, 383, 384 + 17, 3 * 384 + 200])
    sq, sk, sv = parity.grad_abs_scales(inp.q, inp.k, inp.v, dout, causal=True,
                                        scale=1.0 / np.sqrt(W.d), tile_mask=None, Br=W.Br, Bc=W.Bc,
                                        rows=rows, key_range=(0, 1, 256, 384))
    np.testing.assert_allclose(sq, aq.reshape(-1, W.d)[rows], rtol=1e-12)
    np.testing.assert_allclose(sk, ak[0, 1, 256:384], rtol=1e-12)
    np.testing.assert_allclose(sv, av[0, 1, 256:384], rtol=1e-12)
