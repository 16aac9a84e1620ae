"""C-ABI behaviour on the GPU: call order, errors, state, determinism, and the
bounded device-side waits (a fault is injected by a CTA that skips one grid
barrier arrival; the waits run out and the call returns KIE_ERR_TIMEOUT
without hanging the GPU)."""
import ctypes

import numpy as np
import pytest

import synthetic as S
from transformer_decode_persistent_b200 import Engine, KieError
from transformer_decode_persistent_b200 import kie as K

pytestmark = pytest.mark.gpu

SH = S.TINY


@pytest.fixture(scope="module")
def weights():
    return S.make_weights(SH, seed=0)


@pytest.fixture()
def eng(weights):
    e = Engine(SH)
    e.load_weights(weights)
    yield e
    e.close()


def test_decode_before_prefill_and_before_load(weights):
    e = Engine(SH)
    with pytest.raises(KieError) as ei:
        e.decode(1)
    assert ei.value.status == -2
    with pytest.raises(KieError) as ei:
        e.prefill([1, 2, 3])
    assert ei.value.status == -2
    e.load_weights(weights)
    with pytest.raises(KieError) as ei:
        e.decode(1)
    assert ei.value.status == -2  # no pending token yet
    e.close()


def test_bad_weights_rejected(weights):
    e = Engine(SH)
    w = dict(weights)
    w.pop("lm_head")
    with pytest.raises(KieError) as ei:
        e.load_weights(w)
    assert ei.value.status == -1 and "lm_head" in str(ei.value)
    w = dict(weights)
    w["layers.0.wq"] = w["layers.0.wq"][:, :128]
    with pytest.raises(KieError) as ei:
        e.load_weights(w)
    assert ei.value.status == -1
    w = dict(weights)
    w["bogus"] = w["final_norm"]
    with pytest.raises(KieError):
        e.load_weights(w)
    e.close()


def test_token_range_and_context_full(eng):
    with pytest.raises(KieError) as ei:
        eng.prefill([0, SH.vocab])
    assert ei.value.status == -1
    with pytest.raises(KieError) as ei:
        eng.prefill([-1])
    assert ei.value.status == -1
    eng.prefill(S.make_prompt(SH, 0))          # 15 committed, 1 pending
    with pytest.raises(KieError) as ei:
        eng.decode(50)                           # 15 + 50 > 64: nothing done
    assert ei.value.status == -3
    assert eng.position == 15
    with pytest.raises(KieError) as ei:
        eng.decode(2, forced=[3, SH.vocab])
    assert ei.value.status == -1
    eng.decode(49)
    assert eng.position == 64
    with pytest.raises(KieError) as ei:
        eng.decode(1)
    assert ei.value.status == -3


def test_split_calls_equal_one_call(eng):
    p = S.make_prompt(SH, 0)
    eng.prefill(p)
    one = eng.decode(30, logits=True)
    eng.reset()
    eng.prefill(p[:5])
    eng.prefill(p[5:11])
    eng.prefill(p[11:])
    a = eng.decode(7, logits=True)
    b = eng.decode(23, logits=True)
    assert np.array_equal(np.concatenate([a["tokens"], b["tokens"]]), one["tokens"])
    # deterministic kernel: the same logits bit for bit
    lg = np.concatenate([a["logits"].cpu().numpy(), b["logits"].cpu().numpy()])
    assert np.array_equal(lg, one["logits"].cpu().numpy())


def test_reset_equals_fresh_context(weights, eng):
    p = S.make_prompt(SH, 0)
    eng.prefill(p)
    first = eng.decode(20)["tokens"]
    eng.reset()
    assert eng.position == 0 and eng.pending == -1
    eng.prefill(S.make_tokens(SH, 9, seed=5))
    eng.decode(5)
    eng.reset()
    eng.prefill(p)
    again = eng.decode(20)["tokens"]
    e2 = Engine(SH)
    e2.load_weights(weights)
    e2.prefill(p)
    fresh = e2.decode(20)["tokens"]
    e2.close()
    assert np.array_equal(first, again) and np.array_equal(first, fresh)


def test_outputs_to_device_and_pinned_memory(eng):
    import torch
    p = S.make_prompt(SH, 0)
    eng.prefill(p)
    ref = eng.decode(10)["tokens"]
    eng.reset()
    eng.prefill(p)
    dev = torch.empty(10, dtype=torch.int32, device="cuda")
    eng.decode(10, out=dev)
    eng.reset()
    eng.prefill(p)
    pin = torch.empty(10, dtype=torch.int32).pin_memory()
    eng.decode(10, out=pin)
    assert np.array_equal(dev.cpu().numpy(), ref) and np.array_equal(pin.numpy(), ref)


def test_rewind_regenerates_from_a_prefix(eng):
    p = S.make_prompt(SH, 0)
    eng.prefill(p)
    a = eng.decode(12, logits=True)
    eng.rewind(len(p) - 1, int(p[-1]))
    b = eng.decode(12, logits=True)
    assert np.array_equal(a["tokens"], b["tokens"])
    assert np.array_equal(a["logits"].cpu().numpy(), b["logits"].cpu().numpy())
    with pytest.raises(KieError) as ei:
        eng.rewind(eng.position + 1, 0)
    assert ei.value.status == -1
    with pytest.raises(KieError) as ei:
        eng.rewind(0, SH.vocab)
    assert ei.value.status == -1


def test_pending_token_and_forced_feedback(eng):
    p = S.make_prompt(SH, 0)
    eng.prefill(p)
    assert eng.pending == int(p[-1]) and eng.position == len(p) - 1
    r = eng.decode(3, forced=[-1, 7, -1])
    assert eng.pending == int(r["tokens"][2])
    r = eng.decode(1, forced=[11])
    assert eng.pending == 11


def test_weights_from_device_tensors(weights):
    import torch
    p = S.make_prompt(SH, 0)
    e1 = Engine(SH)
    e1.load_weights(weights)
    e1.prefill(p)
    a = e1.decode(12, logits=True)
    e1.close()
    e2 = Engine(SH)
    e2.load_weights({k: torch.from_numpy(v).cuda() for k, v in weights.items()})
    e2.prefill(p)
    b = e2.decode(12, logits=True)
    e2.close()
    assert np.array_equal(a["tokens"], b["tokens"])
    assert torch.equal(a["logits"], b["logits"])


def test_injected_barrier_fault_times_out_and_recovers(eng):
    p = S.make_prompt(SH, 0)
    eng.prefill(p)
    with pytest.raises(KieError) as ei:
        # CTA 3 never arrives at grid barrier 2 (the end of step 2): every
        # other CTA's wait runs out
        eng.decode(4, timeout_ms=200, fault=(3, 2))
    assert ei.value.status == -5 and "timeout" in str(ei.value)
    with pytest.raises(KieError) as ei:
        eng.decode(1)
    assert ei.value.status == -2  # poisoned until reset
    eng.reset()
    eng.prefill(p)
    r = eng.decode(8)
    eng.reset()
    eng.prefill(p)
    assert np.array_equal(eng.decode(8)["tokens"], r["tokens"])


def test_barrier_trace(eng):
    import torch
    info = eng.info()
    eng.prefill(S.make_prompt(SH, 0))
    n = 4
    cap = n * info["barriers_per_token"]
    tr = torch.zeros((info["grid"], cap, 2), dtype=torch.int64, device="cuda")
    eng.decode(n, trace=tr)
    t = tr.cpu().numpy()
    assert (t[:, :, 0] > 0).all() and (t[:, :, 1] >= t[:, :, 0]).all()
    # every CTA is released from barrier k only after the last arrival at k
    last_arrival = t[:, :, 0].max(axis=0)
    assert (t[:, :, 1].min(axis=0) >= last_arrival - 2000).all()


def test_info_counts(eng):
    info = eng.info()
    d, L, V, ff = SH.d_model, SH.n_layers, SH.vocab, SH.ffn
    mats = L * (4 * d * d + 3 * ff * d) * 2 + V * d * 2
    assert info["stream_bytes"] == mats + (2 * L + 1) * d * 2 + d * 2
    assert info["kv_bytes_per_pos"] == 2 * L * SH.n_kv_heads * SH.head_dim * 2
    assert info["grid"] >= 100 and info["threads"] == 256
    assert info["resident_bytes"] == mats
