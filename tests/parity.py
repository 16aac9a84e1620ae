"""Shared helpers of the GPU parity tests: run the engine and the oracle on the
same seeded inputs and compare them under the stated criteria.

Criteria (the parity bar of the decode path):
  * logits of every compared step within max-abs 2e-2 and relative L2 1e-3;
  * greedy token ids identical wherever the oracle's top-1/top-2 margin > 0.05;
  * a free-running decode reproduces the oracle's greedy tokens up to the first
    step whose margin is <= 0.05.
"""
from __future__ import annotations

import numpy as np

import oracle as O
import synthetic as S

TOL_MAX_ABS = 2e-2
TOL_REL_L2 = 1e-3
MARGIN = 0.05


def logit_errors(g: np.ndarray, o: np.ndarray):
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    d = g - o
    max_abs = np.max(np.abs(d), axis=-1)
    rel = np.linalg.norm(d, axis=-1) / np.linalg.norm(o, axis=-1)
    return max_abs, rel


def check_step_logits(g, o, what=""):
    max_abs, rel = logit_errors(g, o)
    bad = np.flatnonzero((max_abs > TOL_MAX_ABS) | (rel > TOL_REL_L2))
    assert bad.size == 0, (f"{what}: {bad.size} steps out of tolerance; first {bad[:5]}: "
                           f"max_abs={max_abs[bad[:5]]}, rel={rel[bad[:5]]}")
    return float(max_abs.max()), float(rel.max())


def check_tokens(gpu_tokens, oracle_logits, what=""):
    ot = np.array([O.argmax_lowest(r) for r in oracle_logits])
    om = np.array([O.top2_margin(r) for r in oracle_logits])
    sure = om > MARGIN
    mism = np.flatnonzero(sure & (np.asarray(gpu_tokens) != ot))
    assert mism.size == 0, f"{what}: argmax differs at confident steps {mism[:10]}"
    return int(sure.sum())


def make_engine(shape, weights, max_ctx=None, device=0):
    from transformer_decode_persistent_b200 import Engine
    e = Engine(shape, device=device, max_ctx=max_ctx)
    e.load_weights(weights)
    return e


def forced_sequence_case(shape, seed: int, n: int, prompt_len: int | None = None,
                         weights=None, engine=None, oracle=None):
    """Teacher forcing with a seeded continuation: the oracle computes every
    position in one full-sequence forward; the engine decodes n steps with the
    continuation forced. Returns (gpu_logits, oracle_logits, gpu_tokens)."""
    w = weights if weights is not None else S.make_weights(shape, seed)
    prompt = S.make_prompt(shape, seed, prompt_len)
    cont = S.make_tokens(shape, n, seed)
    P = len(prompt)
    ref = oracle or O.Decoder(shape, w)
    ol = ref.forward_sequence(np.concatenate([prompt, cont[:n - 1]]))[P - 1:P - 1 + n]
    eng = engine or make_engine(shape, w, max_ctx=P + n)
    eng.reset()
    eng.prefill(prompt)
    r = eng.decode(n, forced=cont, logits=True, margins=True)
    return r["logits"].cpu().numpy(), ol, r["tokens"], r["margins"].cpu().numpy()


def greedy_case(shape, seed: int, n: int, prompt_len: int | None = None, weights=None,
                engine=None):
    """Oracle greedy decode (incremental); engine teacher-forced on the oracle's
    tokens and then free-running. Returns a dict of arrays."""
    w = weights if weights is not None else S.make_weights(shape, seed)
    prompt = S.make_prompt(shape, seed, prompt_len)
    P = len(prompt)
    ref = O.Decoder(shape, w)
    ot, ol, om = ref.greedy(prompt, n)
    eng = engine or make_engine(shape, w, max_ctx=P + n)
    eng.reset()
    eng.prefill(prompt)
    forced = eng.decode(n, forced=ot.astype(np.int32), logits=True, margins=True)
    eng.reset()
    eng.prefill(prompt)
    free = eng.decode(n)
    return dict(oracle_tokens=ot, oracle_logits=ol, oracle_margins=om,
                forced_tokens=forced["tokens"], forced_logits=forced["logits"].cpu().numpy(),
                forced_margins=forced["margins"].cpu().numpy(), free_tokens=free["tokens"])


def check_free_run(free_tokens, oracle_tokens, oracle_margins):
    # steps before the first low-margin step must agree; that step may differ
    low = np.flatnonzero(oracle_margins <= MARGIN)
    k = int(low[0]) if low.size else len(oracle_tokens)
    assert np.array_equal(np.asarray(free_tokens[:k]), oracle_tokens[:k]), \
        f"free run diverges before step {k}"
    return k


def free_run_case(shape, seed: int, n: int, prompt_len: int | None = None, weights=None,
                  engine=None, oracle=None):
    """The engine decodes n tokens free-running (greedy, one launch, logits
    kept); the oracle then computes every step's logits from the same history
    (prompt + the engine's own tokens) in one full-sequence forward. If the
    engine's token equals the oracle's argmax at every step whose oracle margin
    exceeds 0.05, the engine's free run is, by induction, the oracle's own
    greedy run up to the first step with a smaller margin. Returns
    (gpu_logits, oracle_logits, gpu_tokens, gpu_margins, oracle)."""
    w = weights if weights is not None else S.make_weights(shape, seed)
    prompt = S.make_prompt(shape, seed, prompt_len)
    P = len(prompt)
    eng = engine or make_engine(shape, w, max_ctx=P + n)
    eng.reset()
    eng.prefill(prompt)
    r = eng.decode(n, logits=True, margins=True)
    toks = np.asarray(r["tokens"]).astype(np.int64)
    ref = oracle or O.Decoder(shape, w)
    ol = ref.forward_sequence(np.concatenate([prompt, toks[:n - 1]]))[P - 1:P - 1 + n]
    return r["logits"].cpu().numpy(), ol, toks, r["margins"].cpu().numpy(), ref
