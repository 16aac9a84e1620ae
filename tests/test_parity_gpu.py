"""GPU engine vs the fp64 oracle on seeded synthetic weights and prompts.

Every test runs the persistent kernel through the C ABI (libkie.so) and
compares with the oracle element by element (logits) and exactly (token ids
where the oracle's margin is above 0.05)."""
import numpy as np
import pytest

import synthetic as S
import oracle as O
from parity import (check_free_run, check_step_logits, check_tokens, forced_sequence_case,
                    free_run_case, greedy_case, make_engine)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    w = S.make_weights(S.TINY, seed=0)
    return w, make_engine(S.TINY, w)


def test_tiny_full_greedy_teacher_forced_and_free(tiny):
    # workload 1 in full: 2 layers, d 256, prompt 16, 32 greedy tokens, max ctx 64
    w, eng = tiny
    r = greedy_case(S.TINY, 0, S.TINY.decode_len, weights=w, engine=eng)
    check_step_logits(r["forced_logits"], r["oracle_logits"], "tiny forced")
    check_tokens(r["forced_tokens"], r["oracle_logits"], "tiny forced")
    check_free_run(r["free_tokens"], r["oracle_tokens"], r["oracle_margins"])
    # in-kernel margins equal the margins of the kernel's own logits
    gl = r["forced_logits"]
    srt = np.sort(gl, axis=-1)
    assert np.allclose(r["forced_margins"], srt[:, -1] - srt[:, -2], atol=0, rtol=0)


def test_tiny_seeded_continuation_to_max_ctx(tiny):
    # prompt 16 (15 committed + 1 pending) + 49 forced steps fills all 64 positions
    w, eng = tiny
    gl, ol, gt, _ = forced_sequence_case(S.TINY, 0, 49, weights=w, engine=eng)
    check_step_logits(gl, ol, "tiny continuation")
    check_tokens(gt, ol, "tiny continuation")
    assert eng.position == 64


@pytest.mark.parametrize("seed", [1, 2])
def test_tiny_other_seeds(seed):
    w = S.make_weights(S.TINY, seed=seed)
    gl, ol, gt, _ = forced_sequence_case(S.TINY, seed, 24, weights=w)
    check_step_logits(gl, ol, f"tiny seed {seed}")
    check_tokens(gt, ol, f"tiny seed {seed}")


GQA = S.Shape("gqa-5:2", n_layers=3, d_model=320, n_heads=5, n_kv_heads=2, head_dim=64,
              ffn=640, vocab=3000, prompt_len=37, decode_len=40, max_ctx=80)
RAGGED = S.Shape("ragged", n_layers=2, d_model=136, n_heads=2, n_kv_heads=1, head_dim=64,
                 ffn=200, vocab=1001, prompt_len=1, decode_len=70, max_ctx=71)


@pytest.mark.parametrize("shape", [GQA, RAGGED], ids=lambda s: s.name)
def test_odd_shapes(shape):
    # non-integer GQA groups (5 query heads over 2 KV heads: 3 + 2), widths that are
    # not multiples of the tile, a one-token prompt, rows fewer than CTAs
    w = S.make_weights(shape, seed=3, cache=False)
    r = greedy_case(shape, 3, shape.decode_len, weights=w)
    check_step_logits(r["forced_logits"], r["oracle_logits"], shape.name)
    check_tokens(r["forced_tokens"], r["oracle_logits"], shape.name)
    check_free_run(r["free_tokens"], r["oracle_tokens"], r["oracle_margins"])


def test_small_prefix():
    # workload 2 (16 layers, d 1536, V 32000): prompt 128 and 24 forced steps
    s = S.SMALL
    w = S.make_weights(s, seed=0)
    gl, ol, gt, _ = forced_sequence_case(s, 0, 24, weights=w)
    check_step_logits(gl, ol, "0.5B")
    check_tokens(gt, ol, "0.5B")


def test_dense_2b_prefix():
    # the 2.2B workload at its full size and launch shape: prompt 256, 6 forced steps
    s = S.DENSE_2B
    w = S.make_weights(s, seed=0)
    gl, ol, gt, _ = forced_sequence_case(s, 0, 6, weights=w)
    check_step_logits(gl, ol, "2.2B")
    check_tokens(gt, ol, "2.2B")


MOE_SMALL = S.Shape("moe-small", n_layers=3, d_model=256, n_heads=4, n_kv_heads=2, head_dim=64,
                    ffn=0, vocab=2000, n_experts=8, top_k=2, ffn_expert=128, ffn_shared=256,
                    prompt_len=20, decode_len=40, max_ctx=60)


def test_moe_small_greedy():
    # routed top-2 of 8 experts + shared expert, GQA 4:2. The oracle records how
    # close each routing decision came to a tie; decisions the fp32 engine could
    # take the other way (gap < 1e-4) would make the comparison meaningless.
    import oracle as O
    s = MOE_SMALL
    w = S.make_weights(s, seed=4, cache=False)
    ref = O.Decoder(s, w)
    prompt = S.make_prompt(s, 4)
    ot, ol, om = ref.greedy(prompt, s.decode_len)
    assert min(ref.route_gaps) > 1e-4, "a routing decision is within 1e-4 of a tie"
    eng = make_engine(s, w)
    eng.prefill(prompt)
    forced = eng.decode(s.decode_len, forced=ot.astype(np.int32), logits=True)
    check_step_logits(forced["logits"].cpu().numpy(), ol, "moe-small")
    check_tokens(forced["tokens"], ol, "moe-small")
    eng.reset()
    eng.prefill(prompt)
    check_free_run(eng.decode(s.decode_len)["tokens"], ot, om)


def test_moe_full_size_prefix():
    # the MoE workload at its full size: prompt 128 and 6 forced steps
    s = S.MOE
    w = S.make_weights(s, seed=0)
    gl, ol, gt, _ = forced_sequence_case(s, 0, 6, weights=w)
    check_step_logits(gl, ol, "moe")
    check_tokens(gt, ol, "moe")


GQA_LONG = S.Shape("gqa-10:8-long", n_layers=3, d_model=512, n_heads=10, n_kv_heads=8,
                   head_dim=128, ffn=1024, vocab=3000, prompt_len=5000, decode_len=8,
                   max_ctx=5008)


def test_gqa_long_context_multi_round_attention():
    # ~5000 positions x 8 KV heads: attention units span several CTAs per head
    # and several 32-position rounds per warp; 10:8 groups are 1 or 2 heads
    s = GQA_LONG
    w = S.make_weights(s, seed=5, cache=False)
    gl, ol, gt, _ = forced_sequence_case(s, 5, s.decode_len, prompt_len=s.prompt_len, weights=w)
    check_step_logits(gl, ol, "gqa-long")
    check_tokens(gt, ol, "gqa-long")


GQA_WIDE_SHORT = S.Shape("gqa-16:2", n_layers=2, d_model=1024, n_heads=16, n_kv_heads=2, head_dim=64,
                         ffn=2048, vocab=4000, prompt_len=37, decode_len=40, max_ctx=80)
GQA_WIDE_LONG = S.Shape("gqa-14:2-long", n_layers=2, d_model=896, n_heads=14, n_kv_heads=2, head_dim=64,
                        ffn=1024, vocab=3000, prompt_len=2400, decode_len=24, max_ctx=2424)


@pytest.mark.parametrize("s", [GQA_WIDE_SHORT, GQA_WIDE_LONG], ids=lambda s: s.name)
def test_gqa_groups_wider_than_one_unit(s):
    # more query heads per KV head than one attention unit holds (8:1 and 7:1):
    # at short context every query head is its own unit; at ~2400 positions
    # (11 chunks per head) each group runs as sub-units of 4 and 3 query heads
    # over the same K/V rows, with cross-CTA chunk merges
    w = S.make_weights(s, seed=9, cache=False)
    gl, ol, gt, _ = forced_sequence_case(s, 9, s.decode_len, prompt_len=s.prompt_len, weights=w)
    check_step_logits(gl, ol, s.name)
    check_tokens(gt, ol, s.name)


GRID_SMALL = S.Shape("gqa-367:40-d112", n_layers=2, d_model=112, n_heads=367, n_kv_heads=40, head_dim=64,
                     ffn=224, vocab=1000, prompt_len=600, decode_len=12, max_ctx=612)


def test_more_attention_units_than_ctas():
    # d_model 112 gives 112 CTAs, fewer than one chunk's attention units (40
    # KV heads in groups of 9 and 10 query heads, each group as sub-units of
    # 4, 4 and 1 or 2: 120 units per chunk), so the chunks cannot be fitted
    # into one wave: at 600+ positions (3 chunks per head) every CTA runs 3 or
    # 4 units in a row and publishes their chunk records before it merges the
    # heads whose chunk 0 it holds
    s = GRID_SMALL
    w = S.make_weights(s, seed=12, cache=False)
    gl, ol, gt, _ = forced_sequence_case(s, 12, s.decode_len, prompt_len=s.prompt_len, weights=w)
    check_step_logits(gl, ol, s.name)
    check_tokens(gt, ol, s.name)


ZERO_DENSE = S.Shape("zero-dense", n_layers=2, d_model=512, n_heads=8, n_kv_heads=2, head_dim=64,
                     ffn=1024, vocab=3000, prompt_len=9, decode_len=12, max_ctx=24)
ZERO_MOE = S.Shape("zero-moe", n_layers=2, d_model=512, n_heads=8, n_kv_heads=2, head_dim=64, ffn=0,
                   vocab=3000, n_experts=8, top_k=2, ffn_expert=128, ffn_shared=256, prompt_len=9,
                   decode_len=12, max_ctx=24)


@pytest.mark.parametrize("case", ["Z1-dense", "Z2-dense", "Z2-moe"])
def test_zero_weight_closed_forms_on_the_gpu(case):
    # Z1: every layer matrix zero; Z2: only the output and down projections
    # (MoE: every expert's and the shared expert's) zero. Either way each
    # block adds nothing to the residual stream, whatever attention and the
    # FFN compute, so the logits of every step are lm_head . RMSNorm(E[t]; g_f)
    # of the step's input token t: a closed form written out here in numpy,
    # independent of the oracle. Isolates GEMV / LM-head errors from
    # attention and routing.
    s = ZERO_MOE if case.endswith("moe") else ZERO_DENSE
    w = S.make_weights(s, seed=13, cache=False)
    for n in list(w):
        if not n.startswith("layers.") or w[n].ndim != 2:
            continue
        if case.startswith("Z1") or n.endswith(".wo") or n.endswith(".w_down"):
            w[n] = np.zeros_like(w[n])
    prompt = S.make_prompt(s, 13)
    cont = S.make_tokens(s, s.decode_len, 13)
    inputs = np.concatenate([prompt[-1:], cont[:-1]])  # the token each step forwards
    e = w["embed"][inputs].astype(np.float64)
    xn = e / np.sqrt((e * e).mean(axis=1, keepdims=True) + s.rms_eps) * w["final_norm"].astype(np.float64)
    closed = xn @ w["lm_head"].astype(np.float64).T
    eng = make_engine(s, w)
    eng.prefill(prompt)
    r = eng.decode(s.decode_len, forced=cont.astype(np.int32), logits=True)
    check_step_logits(r["logits"].cpu().numpy(), closed, case)
    check_tokens(np.asarray(r["tokens"]), closed, case)


def test_long_context_full_size_self_consistency():
    # The long-context workload at full size (32768-token prompt, GQA 20:8, fp16
    # KV cache of 3.5 GB). The oracle cannot run a 32K-token 2.2B prefix, so the
    # checks are properties. (a) Re-forwarding the last prompt tokens through
    # the prompt path after a rewind rewrites the same cache entries, so the
    # following logits and tokens are bit-identical (the prompt path's results
    # do not depend on how the prompt is cut into calls or chunks). (b)
    # Re-forwarding them through the decode kernel instead (teacher-forced)
    # gives logits within the parity tolerance of the prompt path's.
    s = S.LONG_2B
    w = S.make_weights(s, seed=0)
    prompt = S.make_prompt(s, 0)
    eng = make_engine(s, w, max_ctx=s.prompt_len + 32)
    eng.prefill(prompt)
    P = len(prompt)
    a = eng.decode(16, logits=True)
    k = 8
    eng.rewind(P - 1 - k, int(prompt[P - 1 - k]))
    eng.prefill(prompt[P - k:])
    assert eng.position == P - 1 and eng.pending == int(prompt[-1])
    b = eng.decode(16, logits=True)
    assert np.array_equal(a["tokens"], b["tokens"])
    assert np.array_equal(a["logits"].cpu().numpy(), b["logits"].cpu().numpy())
    eng.rewind(P - 1 - k, int(prompt[P - 1 - k]))
    eng.decode(k, forced=prompt[P - k:].astype(np.int32))
    assert eng.position == P - 1 and eng.pending == int(prompt[-1])
    c = eng.decode(16, logits=True)
    check_step_logits(c["logits"].cpu().numpy(), a["logits"].cpu().numpy().astype(np.float64),
                      "decode-path re-forward vs prompt path")
    lg = a["logits"].cpu().numpy()
    assert np.isfinite(lg).all() and (np.std(lg, axis=1) > 0.1).all()


MOE_PROMPT = S.Shape("moe-prompt", n_layers=3, d_model=1024, n_heads=8, n_kv_heads=2, head_dim=128, ffn=0,
                     vocab=8000, n_experts=16, top_k=2, ffn_expert=512, ffn_shared=1024, prompt_len=300,
                     decode_len=16, max_ctx=316)
MOE_PROMPT_NS = S.Shape("moe-prompt-64x-top8-noshared", n_layers=2, d_model=512, n_heads=8, n_kv_heads=2,
                        head_dim=64, ffn=0, vocab=3000, n_experts=64, top_k=8, ffn_expert=128, ffn_shared=0,
                        prompt_len=300, decode_len=16, max_ctx=316)


MOE_PROMPT_2CHUNK = MOE_PROMPT_NS.with_(name="moe-prompt-2-chunks", prompt_len=1100, max_ctx=1116)


@pytest.mark.parametrize("s", [S.SMALL, MOE_PROMPT, MOE_PROMPT_NS, MOE_PROMPT_2CHUNK], ids=lambda s: s.name)
def test_prompt_path_matches_decode_path_and_oracle(s):
    # The tensor-core prompt path and the decode kernel run teacher-forced over
    # the same prompt fill caches whose next 16 steps agree with each other and
    # with the oracle under the parity criteria. MoE: the prompt path routes
    # each chunk (router GEMM, top-k, experts over their own sorted rows); the
    # router weights are scaled up so that no routing decision is near a tie.
    w = S.make_weights(s, seed=0, cache=not s.n_experts)
    for l in range(s.n_layers if s.n_experts else 0):
        w[f"layers.{l}.router"] = (w[f"layers.{l}.router"].astype(np.float32) * 8).astype(np.float16)
    prompt = S.make_prompt(s, 0)
    P = len(prompt)
    eng = make_engine(s, w, max_ctx=P + 16)
    eng.prefill(prompt)
    a = eng.decode(16, logits=True, forced=S.make_tokens(s, 16, 9))
    eng.reset()
    eng.prefill(prompt[:1])
    eng.decode(P - 1, forced=prompt[1:].astype(np.int32))
    assert eng.position == P - 1 and eng.pending == int(prompt[-1])
    b = eng.decode(16, logits=True, forced=S.make_tokens(s, 16, 9))
    ga, gb = a["logits"].cpu().numpy(), b["logits"].cpu().numpy()
    check_step_logits(ga, gb.astype(np.float64), "prompt path vs decode path")
    cont = S.make_tokens(s, 16, 9)
    ol = O.Decoder(s, w).forward_sequence(np.concatenate([prompt, cont[:15]]))[P - 1:]
    check_step_logits(ga, ol, "prompt path vs oracle")
    check_tokens(a["tokens"], ol, "prompt path vs oracle")


RAGGED_LONG = S.Shape("ragged-long", n_layers=2, d_model=136, n_heads=2, n_kv_heads=1, head_dim=64,
                      ffn=200, vocab=1001, prompt_len=300, decode_len=12, max_ctx=312)


def test_prompt_path_ragged_tiles():
    # widths that fill no tensor-core tile (d 136, q/k/v rows 256, gate/up rows
    # 400, K 136 and 200) and a 300-token prompt over three 128-token tiles
    s = RAGGED_LONG
    w = S.make_weights(s, seed=6, cache=False)
    gl, ol, gt, _ = forced_sequence_case(s, 6, s.decode_len, weights=w)
    check_step_logits(gl, ol, "ragged prompt path")
    check_tokens(gt, ol, "ragged prompt path")


def test_dense_2b_benchmarked_run():
    # The run the benchmark times, in full: the 2.2B workload, prompt 256, 1024
    # greedy tokens in one launch (positions 255-1278, attention split over up
    # to 6 chunks per head). Every step's logits against the oracle on the
    # same history; tokens exact at every confident step, so the free run is
    # the oracle's greedy run up to its first step with margin <= 0.05.
    s = S.DENSE_2B
    gl, ol, gt, gm, _ = free_run_case(s, 0, s.decode_len)
    check_step_logits(gl, ol, "2.2B 1024 steps")
    check_tokens(gt, ol, "2.2B 1024 steps")
    # the in-kernel margins are those of the kernel's own logits
    srt = np.sort(gl, axis=-1)
    assert np.array_equal(gm, srt[:, -1] - srt[:, -2])


def test_long_context_32k_one_layer_oracle_parity():
    # The long-context head layout (GQA 20:8, d 2560, head_dim 128) at the full
    # 32768-token prompt, on one layer so that the oracle can follow: its
    # cache comes from the prompt's projections (layer 0 needs no attention
    # output for them), then 8 teacher-forced steps at positions 32767..32774
    # compare logits with the engine's (tensor-core prompt path, then decode
    # attention over ~32K positions in 17 chunks per head: 136 units on 148 CTAs).
    s = S.LONG_2B.with_(name="gqa20:8-32k-1L", n_layers=1, decode_len=8, max_ctx=32768 + 8)
    w = S.make_weights(s, seed=4, cache=False)
    prompt = S.make_prompt(s, 4)
    cont = S.make_tokens(s, s.decode_len, 4)
    P = len(prompt)
    ref = O.Decoder(s, w)
    cache = ref.new_cache(P + s.decode_len)
    ref.fill_cache_one_layer(prompt[:-1], cache)
    ol, cur = [], int(prompt[-1])
    for i in range(s.decode_len):
        ol.append(ref.step(cur, cache))
        cur = int(cont[i])
    ol = np.stack(ol)
    eng = make_engine(s, w, max_ctx=P + s.decode_len)
    eng.prefill(prompt)
    r = eng.decode(s.decode_len, forced=cont.astype(np.int32), logits=True)
    check_step_logits(r["logits"].cpu().numpy(), ol, "GQA 20:8, 32K context, one layer")
    check_tokens(np.asarray(r["tokens"]), ol, "GQA 20:8, 32K context, one layer")


def test_long_context_reduced_oracle_parity():
    # The long-context workload's weights and head layout (GQA 20:8 at d 2560)
    # with the prompt cut to 2048 tokens and 32 greedy steps, as far as the
    # oracle can follow.
    s = S.LONG_2B_REDUCED
    gl, ol, gt, _, _ = free_run_case(s, 0, s.decode_len)
    check_step_logits(gl, ol, "2.2B GQA 20:8, 2K context")
    check_tokens(gt, ol, "2.2B GQA 20:8, 2K context")


# A routing decision whose k-th and (k+1)-th router logits are closer than
# this may go either way between the kernel (fp32 activations, whose error
# against fp64 reaches ~1e-4 relative in the deep layers) and the oracle. Like
# a token tie, such a step may then differ beyond the logit tolerance, and
# decoding goes on teacher-forced (the engine's tokens are the history of both
# sides). Only such steps may fail, and only a few of them.
ROUTE_TIE = 2e-3


def test_moe_full_size_64_steps():
    # The MoE workload at full size: prompt 128, 64 greedy steps.
    from parity import logit_errors, TOL_MAX_ABS, TOL_REL_L2
    s = S.MOE
    n = 64
    gl, ol, gt, _, ref = free_run_case(s, 0, n)
    T = s.prompt_len - 1 + n
    gaps = np.asarray(ref.route_gaps).reshape(s.n_layers, T)[:, s.prompt_len - 1:]
    near = gaps.min(axis=0) < ROUTE_TIE
    max_abs, rel = logit_errors(gl, ol)
    bad = (max_abs > TOL_MAX_ABS) | (rel > TOL_REL_L2)
    assert not (bad & ~near).any(), f"steps {np.flatnonzero(bad & ~near)} fail without a routing near-tie"
    assert bad.sum() <= 3, f"{bad.sum()} near-tie steps diverge"
    keep = ~bad
    check_step_logits(gl[keep], ol[keep], "moe 64 steps")
    check_tokens(np.asarray(gt)[keep], ol[keep], "moe 64 steps")


@pytest.mark.parametrize("pair", [(7, 4001), (1200, 1201), (3000, 3)], ids=str)
def test_planted_lm_head_tie_takes_the_lower_index(pair):
    # Two identical LM-head rows that win every step: the kernel must report
    # both logits bit-identical, choose the lower row index and a margin of
    # exactly 0. The rows have one non-zero weight, so their logit is one
    # rounded product whatever the summation order. Output and down
    # projections are zero, so the final hidden state is the embedding of the
    # (forced, constant) input token and the winning column is known.
    s = S.TINY
    w = S.make_weights(s, seed=21, cache=False)
    for l in range(s.n_layers):
        w[f"layers.{l}.wo"][:] = 0
        w[f"layers.{l}.w_down"][:] = 0
    t0 = 123
    e = w["embed"][t0].astype(np.float64)
    xn = e / np.sqrt(np.mean(e * e) + s.rms_eps) * w["final_norm"].astype(np.float64)
    k = int(np.argmax(np.abs(xn)))
    row = np.zeros(s.d_model, dtype=np.float16)
    row[k] = np.float16(64.0 * np.sign(xn[k]))
    for i in pair:
        w["lm_head"][i] = row
    eng = make_engine(s, w)
    prompt = np.array([t0], dtype=np.int32)
    n = 12
    eng.prefill(prompt)
    r = eng.decode(n, forced=np.full(n, t0, dtype=np.int32), logits=True, margins=True)
    g = r["logits"].cpu().numpy()
    lo, hi = min(pair), max(pair)
    assert np.array_equal(g[:, lo], g[:, hi])
    assert (np.argmax(g, axis=1) == lo).all()          # numpy also takes the first maximum
    assert (np.asarray(r["tokens"]) == lo).all()
    assert (r["margins"].cpu().numpy() == 0.0).all()
    ol = O.Decoder(s, w).forward_sequence(np.full(n, t0))
    check_step_logits(g, ol, "planted tie")
    assert all(O.argmax_lowest(x) == lo for x in ol)


def test_planted_router_tie_takes_the_lower_expert():
    # Router rows: expert 6 = 2r, experts 2 and 5 = r (an exact tie), all
    # others = -r, in every layer. With s = r . xn > 0 the top-2 are {6, 2}: the
    # tie between 2 and 5 for the second slot goes to 2; with s < 0 the five
    # others tie at the top and the two lowest, {0, 1}, win. Identical,
    # negated and doubled rows give bit-identical, negated and doubled logits
    # in any fixed summation order, so the kernel meets an exact tie; the
    # experts' own weights differ, so taking the wrong one changes the logits.
    s = MOE_SMALL
    w = S.make_weights(s, seed=22, cache=False)
    for l in range(s.n_layers):
        R = w[f"layers.{l}.router"]
        r = R[0].copy()
        for e in range(s.n_experts):
            R[e] = -r
        R[2] = r
        R[5] = r
        R[6] = (2 * r.astype(np.float32)).astype(np.float16)
    prompt = S.make_prompt(s, 22)
    ref = O.Decoder(s, w)
    ot, ol, om = ref.greedy(prompt, s.decode_len)
    assert min(ref.route_gaps) == 0.0       # the ties really are met
    eng = make_engine(s, w)
    eng.prefill(prompt)
    forced = eng.decode(s.decode_len, forced=ot.astype(np.int32), logits=True)
    check_step_logits(forced["logits"].cpu().numpy(), ol, "router tie")
    check_tokens(forced["tokens"], ol, "router tie")


@pytest.mark.parametrize("which", ["small", "dense2b"])
def test_fp16_cache_error_against_unrounded_definition(which):
    # The kernel keeps K and V in fp16 (the workloads' cache); the oracle by
    # default rounds them the same way. This measures the cache's own error
    # against the unrounded fp64 definition. The 0.5B model meets the stated
    # tolerances; at 26 layers the fp16 cache alone moves the logits by a
    # relative L2 of 1.2e-3 to 1.5e-3 (max-abs ~6e-3, within 2e-2), so the
    # relative bound is 2e-3 there. Against the fp16-cache definition the
    # kernel's logits are within ~1e-5.
    from parity import logit_errors
    s = S.SMALL if which == "small" else S.DENSE_2B
    w = S.make_weights(s, seed=0)
    n = 24 if which == "small" else 6
    ref = O.Decoder(s, w, kv_fp16=False)
    gl, ol, gt, _ = forced_sequence_case(s, 0, n, weights=w, oracle=ref)
    max_abs, rel = logit_errors(gl, ol)
    assert max_abs.max() <= 2e-2, max_abs
    assert rel.max() <= (1e-3 if which == "small" else 2e-3), rel
    check_tokens(gt, ol, f"{which} vs unrounded cache")
