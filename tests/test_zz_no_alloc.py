"""kie_decode_static, the decode call that allocates nothing, against kie_decode.

Some callers must not allocate device memory while they decode: a serving loop
with a latency budget cannot afford to stall on the driver's allocator
(cudaMalloc may synchronise the whole device), and a component embedded in
another framework may find all device memory owned by that framework's pool.
kie_decode_static serves them: it runs the same persistent kernel with its
scratch in a fixed array inside the library's device image. Its tokens must be
the ones kie_decode produces from the same state, call after call.

(This file is named to be collected last.)
"""
import numpy as np
import pytest

import synthetic as S
from transformer_decode_persistent_b200 import Engine, KieError

pytestmark = pytest.mark.gpu


def test_static_scratch_decode_equals_decode_on_two_calls():
    import torch
    s = S.TINY
    w = S.make_weights(s, seed=0)
    prompt = S.make_prompt(s, seed=0)
    e = Engine(s)
    e.load_weights(w)

    # reference: kie_decode, two calls in a row
    e.prefill(prompt)
    r1 = e.decode(11, out=torch.empty(11, dtype=torch.int32, device="cuda"))["tokens"].cpu().numpy()
    r2 = e.decode(17, out=torch.empty(17, dtype=torch.int32, device="cuda"))["tokens"].cpu().numpy()
    ref_pos, ref_pending = e.position, e.pending

    # the no-allocation call, two calls in a row from the same state
    e.reset()
    e.prefill(prompt)
    a1 = e.decode_static(11, torch.empty(11, dtype=torch.int32, device="cuda")).cpu().numpy()
    a2 = e.decode_static(17, torch.empty(17, dtype=torch.int32, device="cuda")).cpu().numpy()
    # greedy token ids are exact integers: the tolerance is equality
    assert np.array_equal(a1, r1)
    assert np.array_equal(a2, r2)
    assert e.position == ref_pos and e.pending == ref_pending

    # the KV cache it wrote is the same: a regular call continues identically
    nxt = e.decode(5)["tokens"]
    e.reset()
    e.prefill(prompt)
    e.decode(28)
    assert np.array_equal(nxt, e.decode(5)["tokens"])
    e.close()


def test_static_scratch_rejects_models_that_do_not_fit():
    # 32 query heads of 128 dims over 8 KV heads at up to 4480 positions keep
    # 20 attention chunk records per head: about 0.75 MB of scratch
    s = S.Shape("wide-heads", n_layers=1, d_model=256, n_heads=32, n_kv_heads=8, head_dim=128,
                ffn=256, vocab=100, max_ctx=4480)
    e = Engine(s)
    e.load_weights(S.make_weights(s, seed=1, cache=False))
    import torch
    with pytest.raises(KieError) as ei:
        e.decode_static(1, torch.empty(1, dtype=torch.int32, device="cuda"))
    assert ei.value.status == -1 and "scratch" in str(ei.value)
    e.close()
