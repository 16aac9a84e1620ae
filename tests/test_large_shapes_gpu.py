"""Shapes past the per-CTA partial-sum buffer and larger MoE routing, against
the oracle through the C ABI: a 128,000-token vocabulary and a gate/up
projection of 2 x 24,576 rows over 2,048 inputs (both run in row chunks; 3,460
and 1,336 partial sums per CTA against 1,280), greedy and sampled; and 128
routed experts with top-8; and 64 routed experts with top-8 and no shared
expert (the layer of Mixtral- and OLMoE-class models)."""
import numpy as np
import pytest

import oracle as O
import synthetic as S
from oracle import sampling as SM
from parity import check_step_logits, check_tokens, forced_sequence_case, logit_errors, make_engine

pytestmark = pytest.mark.gpu

WIDE = S.Shape("wide-vocab-ffn", n_layers=1, d_model=2048, n_heads=16, n_kv_heads=8, head_dim=128,
               ffn=24576, vocab=128000, prompt_len=16, decode_len=12, max_ctx=48)
MOE_NOSHARED = S.Shape("moe-64x-top8-noshared", n_layers=2, d_model=512, n_heads=8, n_kv_heads=2, head_dim=64,
                       ffn=0, vocab=3000, n_experts=64, top_k=8, ffn_expert=128, ffn_shared=0,
                       prompt_len=20, decode_len=24, max_ctx=48)
MOE_WIDE = S.Shape("moe-128x-top8", n_layers=2, d_model=512, n_heads=8, n_kv_heads=2, head_dim=64,
                   ffn=0, vocab=3000, n_experts=128, top_k=8, ffn_expert=64, ffn_shared=256,
                   prompt_len=20, decode_len=24, max_ctx=48)


@pytest.fixture(scope="module")
def wide():
    w = S.make_weights(WIDE, seed=31)
    e = make_engine(WIDE, w)
    yield w, e
    e.close()


def test_chunked_lm_head_and_gate_up(wide):
    w, eng = wide
    gl, ol, gt, gm = forced_sequence_case(WIDE, 31, WIDE.decode_len, weights=w, engine=eng)
    check_step_logits(gl, ol, "128K vocabulary, chunked gate/up")
    check_tokens(gt, ol, "128K vocabulary, chunked gate/up")
    srt = np.sort(gl, axis=-1)
    assert np.array_equal(gm, srt[:, -1] - srt[:, -2])


def test_sampling_over_a_chunked_lm_head(wide):
    w, eng = wide
    prompt = S.make_prompt(WIDE, 31)
    P, n, T, k, p, seed = len(prompt), 16, 0.9, 64, 0.95, 555
    eng.reset()
    eng.prefill(prompt)
    r = eng.decode(n, logits=True, temperature=T, top_k=k, top_p=p, seed=seed)
    toks = np.asarray(r["tokens"]).astype(np.int64)
    ol = O.Decoder(WIDE, w).forward_sequence(np.concatenate([prompt, toks[:n - 1]]))[P - 1:]
    check_step_logits(r["logits"].cpu().numpy(), ol, "sampling, 128K vocabulary")
    compared = 0
    for i in range(n):
        u = SM.step_uniform(seed, P - 1 + i)
        if SM.sample_margin(ol[i], T, k, p, u) > 1e-3:
            assert toks[i] == SM.sample_token(ol[i], T, k, p, u), f"step {i}"
            compared += 1
    assert compared >= 0.75 * n


@pytest.mark.parametrize("s", [MOE_WIDE, MOE_NOSHARED], ids=lambda s: s.name)
def test_moe_many_experts_top8(s):
    # router weights scaled up so that the routing decisions are far from ties
    w = S.make_weights(s, seed=32, cache=False)
    for l in range(s.n_layers):
        w[f"layers.{l}.router"] = (w[f"layers.{l}.router"].astype(np.float32) * 8).astype(np.float16)
    ref = O.Decoder(s, w)
    prompt = S.make_prompt(s, 32)
    ot, ol, om = ref.greedy(prompt, s.decode_len)
    eng = make_engine(s, w)
    eng.prefill(prompt)
    r = eng.decode(s.decode_len, forced=ot.astype(np.int32), logits=True)
    gl = r["logits"].cpu().numpy()
    # a step whose routing came within 2e-3 (router logits) of a tie may
    # diverge; only such steps, and few of them
    gaps = np.asarray(ref.route_gaps).reshape(-1, s.n_layers)[s.prompt_len - 1:]
    near = gaps.min(axis=1) < 2e-3
    max_abs, rel = logit_errors(gl, ol)
    bad = (max_abs > 2e-2) | (rel > 1e-3)
    assert not (bad & ~near).any(), np.flatnonzero(bad & ~near)
    assert bad.sum() <= 2
    check_tokens(np.asarray(r["tokens"])[~bad], ol[~bad], s.name)
