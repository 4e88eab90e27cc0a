"""The pipelined end-to-end loop the benchmark times (uploads, prefill and
readbacks on three streams over two device buffer sets): every step's
read-back result must equal one direct call on the same inputs, bit for bit
(the prefill kernel is deterministic), so no step reads or overwrites a
buffer another step still uses."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


def test_pipelined_steps_match_a_direct_call():
    import torch
    from dynamic_block_sparse_tiled_b200 import build
    build.build()
    import dynamic_block_sparse_tiled_b200 as bl
    import bench

    w = synth.CONFIGS["prefill_32k"].replace(name="e2e_small", Hq=8, Hkv=2, Lq=4096, Lkv=4096,
                                             amp=12.0, window=512, n_needles=2)
    lam = float(np.float32(1e-3))
    stream = torch.cuda.Stream()
    pipe = bench.E2EPipeline(w, lam, torch.device("cuda", 0), stream)
    q = pipe.hq.to("cuda").view(torch.bfloat16)
    k = pipe.hk.to("cuda").view(torch.bfloat16)
    v = pipe.hv.to("cuda").view(torch.bfloat16)
    o_ref, lse_ref, _ = bl.attention_prefill(q, k, v, causal=True, lam=lam, Br=w.Br, Bc=w.Bc)
    assert bl.blasst_check() == 0
    o_ref = o_ref.view(torch.int16).cpu().numpy()
    lse_ref = lse_ref.cpu().numpy()
    for n in (1, 2, 5):
        for h in pipe.host_out:  # stale results must not pass
            h["o"].fill_(-1)
            h["lse"].fill_(float("nan"))
        pipe.run(n)
        stream.synchronize()
        assert bl.blasst_check(stream) == 0
        for i in range(max(0, n - 2), n):  # the last one or two steps' buffer sets
            h = pipe.host_out[i % 2]
            assert np.array_equal(h["o"].numpy(), o_ref), (n, i)
            assert np.array_equal(h["lse"].numpy(), lse_ref), (n, i)
