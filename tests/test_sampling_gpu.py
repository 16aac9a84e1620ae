"""In-kernel sampling (temperature, top-k, top-p, Philox uniforms) against the
sampling oracle, through the C ABI.

The engine decodes free-running with sampling; the oracle recomputes every
step's logits on the engine's own history (one full-sequence forward) and
applies its definition with the same uniform (Philox4x32-10 keyed by the seed,
counter = the position of the step's forward). Where the uniform lies more than
1e-3 (in probability) from a CDF bucket edge or the top-p cut, the engine's
token must be the oracle's: fp32 against fp64 logits move the edges by far
less than that."""
import numpy as np
import pytest

import oracle as O
import synthetic as S
from oracle import sampling as SM
from parity import check_step_logits, make_engine

pytestmark = pytest.mark.gpu

EDGE = 1e-3


def _run(shape, seed_w, n, T, k, p, seed, engine=None, weights=None):
    w = weights if weights is not None else S.make_weights(shape, seed_w, cache=False)
    prompt = S.make_prompt(shape, seed_w)
    P = len(prompt)
    eng = engine or make_engine(shape, w, max_ctx=P + n)
    eng.reset()
    eng.prefill(prompt)
    r = eng.decode(n, logits=True, temperature=T, top_k=k, top_p=p, seed=seed)
    toks = np.asarray(r["tokens"]).astype(np.int64)
    ol = O.Decoder(shape, w).forward_sequence(np.concatenate([prompt, toks[:n - 1]]))[P - 1:P - 1 + n]
    return r["logits"].cpu().numpy(), ol, toks, P, eng, w


@pytest.mark.parametrize("T,k,p,seed", [(0.8, 40, 0.9, 1234), (1.3, 64, 1.0, 7), (0.6, 5, 0.5, 2 ** 40 + 3),
                                        (1.0, 33, 0.95, 99)])
def test_sampled_tokens_match_the_oracle(T, k, p, seed):
    s = S.TINY
    n = 40
    gl, ol, toks, P, eng, _ = _run(s, 11, n, T, k, p, seed)
    eng.close()
    check_step_logits(gl, ol, "sampling run")
    compared = 0
    for i in range(n):
        u = SM.step_uniform(seed, P - 1 + i)
        if SM.sample_margin(ol[i], T, k, p, u) > EDGE:
            assert toks[i] == SM.sample_token(ol[i], T, k, p, u), f"step {i}"
            compared += 1
    assert compared >= 0.8 * n
    # the run really samples: it is not the greedy sequence
    assert any(toks[i] != O.argmax_lowest(ol[i]) for i in range(n))


def test_sampling_on_the_0_5b_model():
    s = S.SMALL
    n = 24
    gl, ol, toks, P, eng, _ = _run(s, 0, n, 0.7, 17, 0.8, 4242)
    eng.close()
    check_step_logits(gl, ol, "0.5B sampling")
    for i in range(n):
        u = SM.step_uniform(4242, P - 1 + i)
        if SM.sample_margin(ol[i], 0.7, 17, 0.8, u) > EDGE:
            assert toks[i] == SM.sample_token(ol[i], 0.7, 17, 0.8, u), f"step {i}"


def test_sampling_special_cases_and_split_calls():
    s = S.TINY
    w = S.make_weights(s, seed=12, cache=False)
    prompt = S.make_prompt(s, 12)
    eng = make_engine(s, w)
    eng.prefill(prompt)
    greedy = eng.decode(20)["tokens"]
    # top-k 1 is greedy whatever the temperature and seed
    eng.reset(); eng.prefill(prompt)
    assert np.array_equal(eng.decode(20, temperature=2.0, top_k=1, seed=5)["tokens"], greedy)
    # the uniform is keyed by position: one call of 20 = calls of 7 and 13
    eng.reset(); eng.prefill(prompt)
    one = eng.decode(20, temperature=1.1, top_k=50, top_p=0.9, seed=77)["tokens"]
    eng.reset(); eng.prefill(prompt)
    a = eng.decode(7, temperature=1.1, top_k=50, top_p=0.9, seed=77)["tokens"]
    b = eng.decode(13, temperature=1.1, top_k=50, top_p=0.9, seed=77)["tokens"]
    assert np.array_equal(np.concatenate([a, b]), one)
    # another seed gives another sequence
    eng.reset(); eng.prefill(prompt)
    assert not np.array_equal(eng.decode(20, temperature=1.1, top_k=50, top_p=0.9, seed=78)["tokens"], one)
    # invalid arguments are rejected before launch
    from transformer_decode_persistent_b200 import KieError
    for kw in (dict(temperature=1.0, top_k=0), dict(temperature=1.0, top_k=65),
               dict(temperature=1.0, top_k=5, top_p=0.0), dict(temperature=-1.0)):
        with pytest.raises(KieError) as ei:
            eng.decode(1, **kw)
        assert ei.value.status == -1
    eng.close()
