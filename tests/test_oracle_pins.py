"""Pins for the fp64 oracle: closed forms, invariants and brute force.

Each test fixes one part of the oracle against something other than the
oracle itself, chosen so that a plausible slip (eps outside the root, the wrong
RoPE pairing or sign, a missing 1/sqrt(dh), a transposed weight, a dropped
residual, non-causal attention, the wrong GQA map, a wrong MoE weight) fails.
"""
import math

import numpy as np
import pytest

import oracle as O
import synthetic as S


# ------------------------------------------------------------------ RMSNorm

def test_rmsnorm_constant_vector_closed_form():
    # x = c * 1  =>  y = g * c / sqrt(c^2 + eps); with c = 1e-3, eps = 1e-5 the
    # value (0.30151) is far from what eps outside the root would give (0.990).
    c, eps = 1e-3, 1e-5
    g = np.array([1.0, 2.0, -0.5, 3.0])
    y = O.rmsnorm(np.full(4, c), g, eps)
    want = g * c / math.sqrt(c * c + eps)
    assert np.allclose(y, want, rtol=0, atol=1e-15)
    assert abs(y[0] - 0.30151134457776363) < 1e-12


def test_rmsnorm_hand_value_and_unit_rms():
    # [3, 4]: mean square 12.5, root 3.5355...
    y = O.rmsnorm(np.array([3.0, 4.0]), np.ones(2), 0.0)
    assert np.allclose(y, [3 / math.sqrt(12.5), 4 / math.sqrt(12.5)], atol=1e-15)
    rng = np.random.default_rng(0)
    x = rng.normal(size=257) * 7.0
    g = 1.0 + 0.1 * rng.normal(size=257)
    y = O.rmsnorm(x, g, 0.0) / g
    assert abs(math.sqrt(np.mean(y * y)) - 1.0) < 1e-13
    # scale invariance (eps = 0) and the row-wise form on [T, d]
    assert np.allclose(O.rmsnorm(5.0 * x, g, 0.0), O.rmsnorm(x, g, 0.0), atol=1e-13)
    X = rng.normal(size=(3, 257))
    Y = O.rmsnorm(X, g, 1e-5)
    for t in range(3):
        ms = sum(v * v for v in X[t]) / 257
        assert np.allclose(Y[t], [X[t, i] / math.sqrt(ms + 1e-5) * g[i] for i in range(257)],
                           atol=1e-13)


# ------------------------------------------------------------------ RoPE

def test_rope_identity_at_zero_and_norm_preserving():
    rng = np.random.default_rng(1)
    u = rng.normal(size=(3, 16))
    assert np.array_equal(O.rope(u, 0, 10000.0), u)
    for p in (1, 7, 1279, 33000):
        r = O.rope(u, p, 10000.0)
        assert np.allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(u, axis=-1), atol=1e-12)


def test_rope_half_split_pairing_and_frequency():
    # dh = 4: pairs (0, 2) at frequency 1 and (1, 3) at 10000^(-1/2) = 0.01.
    e1 = np.array([[0.0, 1.0, 0.0, 0.0]])
    r = O.rope(e1, 1, 10000.0)[0]
    assert np.allclose(r, [0.0, math.cos(0.01), 0.0, math.sin(0.01)], atol=1e-15)
    e0 = np.array([[1.0, 0.0, 0.0, 0.0]])
    r = O.rope(e0, 2, 10000.0)[0]
    assert np.allclose(r, [math.cos(2.0), 0.0, math.sin(2.0), 0.0], atol=1e-15)
    # the second member of a pair rotates to (-sin, cos)
    e2 = np.array([[0.0, 0.0, 1.0, 0.0]])
    r = O.rope(e2, 2, 10000.0)[0]
    assert np.allclose(r, [-math.sin(2.0), 0.0, math.cos(2.0), 0.0], atol=1e-15)


def test_rope_relative_position_property():
    rng = np.random.default_rng(2)
    q, k = rng.normal(size=(1, 8)), rng.normal(size=(1, 8))
    for m in range(0, 17, 3):
        for n in range(0, 17, 5):
            a = float(O.rope(q, m, 100.0)[0] @ O.rope(k, n, 100.0)[0])
            b = float(O.rope(q, m - n + 20, 100.0)[0] @ O.rope(k, 20, 100.0)[0])
            assert abs(a - b) < 1e-12


def test_rope_sequence_form_matches_scalar_form():
    rng = np.random.default_rng(3)
    u = rng.normal(size=(5, 3, 8))
    r = O.rope(u, np.arange(5), 10000.0)
    for t in range(5):
        assert np.allclose(r[t], O.rope(u[t], t, 10000.0), atol=0)


# ------------------------------------------------------------------ softmax

def test_softmax_known_value_sum_and_shift():
    assert np.allclose(O.softmax([0.0, math.log(3.0)]), [0.25, 0.75], atol=1e-15)
    rng = np.random.default_rng(4)
    s = rng.normal(size=(4, 50)) * 30
    p = O.softmax(s)
    assert np.all(np.abs(p.sum(-1) - 1) < 1e-12)
    assert np.allclose(O.softmax(s + 1234.5), p, atol=1e-14)
    m = np.array([1.0, -np.inf, 2.0])
    assert O.softmax(m)[1] == 0.0


# ------------------------------------------------------------------ attention

def _attention_brute(q, K, V, hq, hk):
    dh = q.shape[1]
    o = np.zeros((hq, dh))
    for h in range(hq):
        g = (h * hk) // hq
        T = K.shape[1]
        sc = [sum(q[h, i] * K[g, j, i] for i in range(dh)) / math.sqrt(dh) for j in range(T)]
        m = max(sc)
        w = [math.exp(v - m) for v in sc]
        z = sum(w)
        for i in range(dh):
            o[h, i] = sum(w[j] * V[g, j, i] for j in range(T)) / z
    return o


@pytest.mark.parametrize("hq,hk,T", [(2, 2, 1), (3, 3, 5), (5, 2, 7), (4, 1, 6)])
def test_attention_brute_force(hq, hk, T):
    rng = np.random.default_rng(hq * 100 + T)
    dh = 4
    q = rng.normal(size=(hq, dh))
    K, V = rng.normal(size=(hk, T, dh)), rng.normal(size=(hk, T, dh))
    assert np.allclose(O.attend_one(q, K, V), _attention_brute(q, K, V, hq, hk), atol=1e-13)


def test_attention_single_position_returns_v0_and_scale():
    rng = np.random.default_rng(5)
    q = rng.normal(size=(2, 8)) * 100
    K, V = rng.normal(size=(2, 1, 8)), rng.normal(size=(2, 1, 8))
    assert np.array_equal(O.attend_one(q, K, V), V[:, 0, :])
    # two keys: s0 = a*b/sqrt(dh), s1 = 0 => weight sigma(s0) on v0
    dh, a, b = 16, 2.0, 3.0
    q = np.zeros((1, dh)); q[0, 0] = a
    K = np.zeros((1, 2, dh)); K[0, 0, 0] = b
    V = np.zeros((1, 2, dh)); V[0, 0, 1] = 1.0; V[0, 1, 2] = 1.0
    w0 = 1.0 / (1.0 + math.exp(-a * b / 4.0))
    o = O.attend_one(q, K, V)[0]
    assert abs(o[1] - w0) < 1e-15 and abs(o[2] - (1 - w0)) < 1e-15


def test_gqa_head_map_non_integer_groups():
    # hq = 5, hk = 2: floor(h*2/5) = 0, 0, 0, 1, 1 ; 20:8 gives groups 3,2,3,2,...
    assert [O.kv_head_of(h, 5, 2) for h in range(5)] == [0, 0, 0, 1, 1]
    m = [O.kv_head_of(h, 20, 8) for h in range(20)]
    assert m == [0, 0, 0, 1, 1, 2, 2, 2, 3, 3, 4, 4, 4, 5, 5, 6, 6, 6, 7, 7]
    assert [O.kv_head_of(h, 16, 4) for h in range(16)] == [h // 4 for h in range(16)]
    q = np.ones((5, 4))
    K = np.zeros((2, 3, 4))
    V = np.zeros((2, 3, 4)); V[0] = 1.0
    o = O.attend_one(q, K, V)
    assert np.array_equal(o[:3], np.ones((3, 4))) and np.array_equal(o[3:], np.zeros((2, 4)))


def test_causal_attention_equals_one_query_at_a_time():
    rng = np.random.default_rng(6)
    T, hq, hk, dh = 6, 5, 2, 4
    q, k, v = rng.normal(size=(T, hq, dh)), rng.normal(size=(T, hk, dh)), rng.normal(size=(T, hk, dh))
    full = O.causal_attention(q, k, v)
    for t in range(T):
        Kc = np.transpose(k[:t + 1], (1, 0, 2))
        Vc = np.transpose(v[:t + 1], (1, 0, 2))
        assert np.allclose(full[t], O.attend_one(q[t], Kc, Vc), atol=1e-13)
    # causality: changing a later position does not change earlier rows
    k2 = k.copy(); k2[4:] += 10
    assert np.array_equal(O.causal_attention(q, k2, v)[:4], full[:4])


# ------------------------------------------------------------------ MLP / GEMV

def test_silu_special_values():
    assert O.silu(0.0) == 0.0
    assert abs(O.silu(1.0) - 0.7310585786300049) < 1e-15
    assert abs(O.silu(30.0) - 30.0) < 1e-10
    assert abs(O.silu(-40.0)) < 1e-15
    assert abs(O.silu(-1.0) - (-0.2689414213699951)) < 1e-15


def test_swiglu_identity_weights():
    x = np.array([0.5, -2.0])
    I = np.eye(2)
    y = O.swiglu_ffn(x, I, I, I)
    assert np.allclose(y, [0.5 * 0.5 / (1 + math.exp(-0.5)), -2.0 * -2.0 / (1 + math.exp(2.0))], atol=1e-15)
    # gate and up are not interchangeable: silu(g) * u
    Wg = np.array([[1.0, 0.0]]); Wu = np.array([[0.0, 1.0]]); Wd = np.array([[1.0]])
    y = O.swiglu_ffn(np.array([1.0, 3.0]), Wg, Wu, Wd)
    assert abs(y[0] - 3.0 / (1 + math.exp(-1.0))) < 1e-15


def test_gemv_orientation_brute_force():
    # y_i = sum_j W_ij x_j with W [out, in] row-major (non-square)
    rng = np.random.default_rng(7)
    W, x = rng.normal(size=(3, 5)), rng.normal(size=5)
    Wd = np.zeros((2, 3)); Wd[1, 2] = 1.0
    y = O.swiglu_ffn(x, W, W, Wd)
    h = [sum(W[i, j] * x[j] for j in range(5)) for i in range(3)]
    assert abs(y[1] - h[2] * h[2] / (1 + math.exp(-h[2]))) < 1e-12 and y[0] == 0.0


# ------------------------------------------------------------------ sampling

def test_argmax_lowest_index_on_ties_and_margin():
    v = np.array([0.1, 3.0, -1.0, 3.0, 2.5])
    assert O.argmax_lowest(v) == 1
    assert O.top2_margin(v) == 0.0
    w = np.array([0.1, 3.0, -1.0, 2.0, 2.5])
    assert O.argmax_lowest(w) == 1 and abs(O.top2_margin(w) - 0.5) < 1e-15
    rng = np.random.default_rng(8)
    for _ in range(20):
        z = rng.integers(-3, 4, size=9).astype(float)
        best = max(range(9), key=lambda i: (z[i], -i))
        assert O.argmax_lowest(z) == best
    assert O.topk_lowest([1.0, 5.0, 5.0, 2.0, 5.0], 2) == [1, 2]
    assert O.topk_lowest([1.0, 5.0, 3.0, 3.0], 2) == [1, 2]


# ------------------------------------------------------------------ MoE

def test_moe_router_renormalisation_and_expert_identity():
    rng = np.random.default_rng(9)
    d, f, E = 6, 5, 8
    xn = rng.normal(size=d)
    G, U, D = rng.normal(size=(f, d)), rng.normal(size=(f, d)), rng.normal(size=(d, f))
    base = O.swiglu_ffn(xn, G, U, D)
    # experts differ only by a scale c_e on w_down; router rows planted so that
    # experts 3 and 6 lead with logits r3 = 2 and r6 = 1 (the others < 0).
    c = np.arange(1, E + 1, dtype=float)
    experts = [(G, U, c[e] * D) for e in range(E)]
    router = np.zeros((E, d))
    logit = np.array([-1.0, -2.0, -3.0, 2.0, -1.5, -0.5, 1.0, -4.0])
    u = xn / (xn @ xn)
    for e in range(E):
        router[e] = logit[e] * u
    zero = (np.zeros((f, d)), np.zeros((f, d)), np.zeros((d, f)))
    y = O.moe_ffn(xn, router, experts, zero, 2)
    w3 = 1.0 / (1.0 + math.exp(-(2.0 - 1.0)))      # 2-way softmax of the chosen logits
    assert np.allclose(y, (w3 * c[3] + (1 - w3) * c[6]) * base, atol=1e-12)
    # identical experts: the routed part is exactly one expert; shared added at weight 1
    same = [(G, U, D)] * E
    y = O.moe_ffn(xn, router, same, (G, U, 2 * D), 2)
    assert np.allclose(y, 3 * base, atol=1e-12)


# ------------------------------------------------------------------ whole model

def _tiny(kind):
    if kind == "mha":
        return S.Shape("t-mha", n_layers=2, d_model=32, n_heads=4, n_kv_heads=4, head_dim=8,
                       ffn=48, vocab=61, max_ctx=24)
    if kind == "gqa":
        return S.Shape("t-gqa", n_layers=2, d_model=40, n_heads=5, n_kv_heads=2, head_dim=8,
                       ffn=24, vocab=53, max_ctx=24)
    if kind == "moe-noshared":
        return S.Shape("t-moe-ns", n_layers=2, d_model=32, n_heads=4, n_kv_heads=2, head_dim=8,
                       ffn=0, vocab=47, n_experts=8, top_k=3, ffn_expert=16, ffn_shared=0,
                       max_ctx=24)
    return S.Shape("t-moe", n_layers=2, d_model=32, n_heads=4, n_kv_heads=2, head_dim=8,
                   ffn=0, vocab=47, n_experts=6, top_k=2, ffn_expert=16, ffn_shared=24,
                   max_ctx=24)


def _scaled(w, k=10.0):
    # larger weights so attention is far from uniform and errors would show
    return {n: (a * k).astype(np.float16) if a.ndim == 2 else a for n, a in w.items()}


@pytest.mark.parametrize("kind", ["mha", "gqa", "moe", "moe-noshared"])
def test_incremental_decode_equals_full_recompute(kind):
    s = _tiny(kind)
    w = _scaled(S.make_weights(s, seed=3, cache=False))
    m = O.Decoder(s, w)
    toks = S.make_tokens(s, 20, seed=4)
    full = m.forward_sequence(toks)
    cache = m.new_cache(20)
    for t in range(20):
        lg = m.step(toks[t], cache)
        assert np.allclose(lg, full[t], rtol=0, atol=1e-12 * max(1.0, np.abs(full[t]).max()))
    # teacher-forced greedy = full recompute on the forced sequence
    prompt, forced = toks[:6], toks[6:]
    tk, lg, mg = m.greedy(prompt, len(forced), forced=forced)
    assert np.allclose(lg, full[5:5 + len(forced)], rtol=0, atol=1e-10)
    assert list(tk) == [O.argmax_lowest(r) for r in full[5:5 + len(forced)]]
    assert np.all(mg >= 0)


def test_greedy_protocol_first_token_from_last_prompt_position():
    s = _tiny("mha")
    w = _scaled(S.make_weights(s, seed=5, cache=False))
    m = O.Decoder(s, w)
    prompt = S.make_prompt(s, seed=5, length=7)
    tk, lg, _ = m.greedy(prompt, 4)
    full = m.forward_sequence(np.concatenate([prompt, tk[:3]]))
    assert tk[0] == O.argmax_lowest(full[6])
    for i in range(4):
        assert tk[i] == O.argmax_lowest(full[6 + i])


def _closed_form_logits(w, s, t):
    e = w["embed"][t].astype(np.float64)
    ms = sum(v * v for v in e) / len(e)
    xn = [e[i] / math.sqrt(ms + s.rms_eps) * float(w["final_norm"][i]) for i in range(len(e))]
    L = w["lm_head"].astype(np.float64)
    return np.array([sum(L[r, i] * xn[i] for i in range(len(e))) for r in range(L.shape[0])])


@pytest.mark.parametrize("which", ["Z1", "Z2"])
def test_zero_weight_closed_forms(which):
    s = _tiny("gqa")
    w = _scaled(S.make_weights(s, seed=6, cache=False), 3.0)
    for n in list(w):
        if not n.startswith("layers."):
            continue
        if which == "Z1" and w[n].ndim == 2:
            w[n] = np.zeros_like(w[n])
        if which == "Z2" and (n.endswith(".wo") or n.endswith(".w_down")):
            w[n] = np.zeros_like(w[n])
    m = O.Decoder(s, w)
    toks = S.make_tokens(s, 5, seed=7)
    full = m.forward_sequence(toks)
    for t in range(5):
        assert np.allclose(full[t], _closed_form_logits(w, s, toks[t]), atol=1e-12)


def test_uniform_attention_layer_closed_form():
    # One layer, Wq = Wk = 0 (uniform weights over j <= p), Wv = Wo = I, FFN = 0:
    # x_p' = x_p + mean_{j<=p} fp16(RMSNorm(x_j; g1)) (V is cached in fp16). Pins
    # causal masking, the V and O paths and the residual add.
    s = S.Shape("t-u", n_layers=1, d_model=8, n_heads=2, n_kv_heads=2, head_dim=4, ffn=4,
                vocab=11, max_ctx=8)
    w = S.make_weights(s, seed=8, cache=False)
    w["layers.0.wq"][:] = 0
    w["layers.0.wk"][:] = 0
    w["layers.0.wv"][:] = np.eye(8, dtype=np.float16)
    w["layers.0.wo"][:] = np.eye(8, dtype=np.float16)
    w["layers.0.w_down"][:] = 0
    w["final_norm"][:] = 1
    w["lm_head"] = np.eye(11, 8, dtype=np.float16)
    m = O.Decoder(s, w)
    toks = [3, 9, 1, 4, 7]
    full = m.forward_sequence(toks)
    xs = [w["embed"][t].astype(np.float64) for t in toks]
    g1 = w["layers.0.attn_norm"].astype(np.float64)

    def nrm(v, g):
        r = math.sqrt(sum(a * a for a in v) / len(v) + s.rms_eps)
        return np.array([v[i] / r * g[i] for i in range(len(v))])

    for p in range(5):
        mean = sum(nrm(xs[j], g1).astype(np.float16).astype(np.float64) for j in range(p + 1)) / (p + 1)
        xp = xs[p] + mean
        want = np.zeros(11); want[:8] = nrm(xp, np.ones(8))
        assert np.allclose(full[p], want, atol=1e-12)


def test_long_context_weights_are_prefix_of_dense():
    # the reading "same weights with 8 KV heads": Wk/Wv are the first rows
    s3 = S.DENSE_2B.with_(n_layers=1, vocab=64)
    s4 = S.LONG_2B.with_(n_layers=1, vocab=64)
    w3 = S.make_weights(s3, seed=0, cache=False)
    w4 = S.make_weights(s4, seed=0, cache=False)
    assert np.array_equal(w4["layers.0.wk"], w3["layers.0.wk"][:1024])
    assert np.array_equal(w4["layers.0.wv"], w3["layers.0.wv"][:1024])
    assert np.array_equal(w4["layers.0.wq"], w3["layers.0.wq"])


def test_kv_cache_holds_fp16_rounded_values():
    # The cache keeps K (after RoPE) and V rounded to fp16; queries are not rounded.
    s = _tiny("gqa")
    w = _scaled(S.make_weights(s, seed=11, cache=False), 10.0)
    m = O.Decoder(s, w)
    cache = m.new_cache(4)
    toks = S.make_tokens(s, 3, seed=12)
    for t in toks:
        m.step(t, cache)
    K, V = cache["K"][:, :, :3, :], cache["V"][:, :, :3, :]
    assert np.array_equal(K.astype(np.float16).astype(np.float64), K)
    assert np.array_equal(V.astype(np.float16).astype(np.float64), V)
    # layer 0, position 0: v = Wv . RMSNorm(E[t0]) rounded to fp16 (elementwise, brute force)
    e = w["embed"][toks[0]].astype(np.float64)
    r = math.sqrt(sum(x * x for x in e) / len(e) + s.rms_eps)
    g = w["layers.0.attn_norm"].astype(np.float64)
    xn = [e[i] / r * g[i] for i in range(len(e))]
    Wv = w["layers.0.wv"].astype(np.float64)
    for row in range(Wv.shape[0]):
        val = sum(Wv[row, j] * xn[j] for j in range(len(xn)))
        assert V[0, row // s.head_dim, 0, row % s.head_dim] == float(np.float16(val))
    # the unrounded variant differs (the rounding is really applied)
    m2 = O.Decoder(s, w, kv_fp16=False)
    c2 = m2.new_cache(4)
    for t in toks:
        m2.step(t, c2)
    assert not np.array_equal(c2["V"][:, :, :3, :], V)


@pytest.mark.parametrize("hk", [2, 1], ids=["mha", "gqa2:1"])
def test_rope_wiring_in_the_model_brute_force(hk):
    # One layer whose q, k and v are known multiples of the normalised input:
    # Wq = Wk = 3 I (per head), Wv = Wo = I, FFN output 0, lm_head = I, final
    # gain 1. The expected logits are built with scalar loops: q and k of the
    # token at position p are rotated by the angles of position p (pairs i,
    # i + dh/2, angle p * theta^(-2i/dh)); v is not rotated; K (after the
    # rotation) and V enter the cache rounded to fp16; causal softmax over
    # j <= p with max subtraction. Large scores make the attention weights, and
    # so the logits, depend on every rotation angle; the cache check fixes the
    # absolute position at which k is rotated. A model that leaves k unrotated,
    # rotates v, or rotates at position p + 1 fails here.
    d, hq, dh, theta = 8, 2, 4, 10.0
    s = S.Shape("t-rope", n_layers=1, d_model=d, n_heads=hq, n_kv_heads=hk, head_dim=dh, ffn=4,
                vocab=11, max_ctx=8, rope_theta=theta)
    w = S.make_weights(s, seed=13, cache=False)
    w["layers.0.wq"][:] = 3 * np.eye(hq * dh, d, dtype=np.float16)
    w["layers.0.wk"][:] = 3 * np.eye(hk * dh, d, dtype=np.float16)
    w["layers.0.wv"][:] = np.eye(hk * dh, d, dtype=np.float16)
    w["layers.0.wo"][:] = np.eye(d, hq * dh, dtype=np.float16)
    w["layers.0.w_down"][:] = 0
    w["final_norm"][:] = 1
    w["lm_head"] = np.eye(11, d, dtype=np.float16)
    toks = [5, 2, 9, 2, 7, 0]
    T = len(toks)
    g1 = [float(v) for v in w["layers.0.attn_norm"]]

    def nrm(v, g):
        r = math.sqrt(sum(a * a for a in v) / len(v) + s.rms_eps)
        return [v[i] / r * g[i] for i in range(len(v))]

    def rot(u, pos):  # one head's dh values
        out = list(u)
        for i in range(dh // 2):
            phi = pos * theta ** (-2.0 * i / dh)
            a, b = u[i], u[i + dh // 2]
            out[i] = a * math.cos(phi) - b * math.sin(phi)
            out[i + dh // 2] = a * math.sin(phi) + b * math.cos(phi)
        return out

    f16 = lambda v: float(np.float16(v))
    xs = [[float(v) for v in w["embed"][t]] for t in toks]
    xn = [nrm(x, g1) for x in xs]
    # per position and KV head: cached K (rotated, fp16) and V (fp16)
    Kc = [[[f16(v) for v in rot([3 * xn[j][g * dh + e] for e in range(dh)], j)] for g in range(hk)]
          for j in range(T)]
    Vc = [[[f16(xn[j][g * dh + e]) for e in range(dh)] for g in range(hk)] for j in range(T)]
    want = []
    for p in range(T):
        o = []
        for h in range(hq):
            g = (h * hk) // hq
            qh = rot([3 * xn[p][h * dh + e] for e in range(dh)], p)
            sc = [sum(qh[e] * Kc[j][g][e] for e in range(dh)) / math.sqrt(dh) for j in range(p + 1)]
            m = max(sc)
            ex = [math.exp(v - m) for v in sc]
            z = sum(ex)
            o += [sum(ex[j] / z * Vc[j][g][e] for j in range(p + 1)) for e in range(dh)]
        x2 = [xs[p][i] + o[i] for i in range(d)]
        lg = nrm(x2, [1.0] * d) + [0.0] * 3
        want.append(lg)
    want = np.array(want)
    # the attention weights are far from uniform, so the rotations matter
    assert np.ptp(want[:, :d]) > 1.0

    m = O.Decoder(s, w)
    full = m.forward_sequence(toks)
    assert np.allclose(full, want, rtol=0, atol=1e-12)
    cache = m.new_cache(T)
    for p in range(T):
        assert np.allclose(m.step(toks[p], cache), want[p], rtol=0, atol=1e-12)
    for j in range(T):
        for g in range(hk):
            assert list(cache["K"][0, g, j]) == Kc[j][g]
            assert list(cache["V"][0, g, j]) == Vc[j][g]


def test_moe_without_shared_expert_equals_a_zero_shared_expert():
    """A MoE layer with no shared expert (ffn_shared = 0, no shared tensors)
    is the same function as one whose shared expert has all-zero weights:
    SwiGLU of zero weights is zero, whatever the input."""
    ns = _tiny("moe-noshared")
    zs = ns.with_(name="t-moe-zero-shared", ffn_shared=8)
    w = _scaled(S.make_weights(ns, seed=11, cache=False))
    assert not any(".shared." in n for n in w)
    wz = dict(w)
    for l in range(zs.n_layers):
        wz[f"layers.{l}.shared.w_gate"] = np.zeros((8, zs.d_model), np.float16)
        wz[f"layers.{l}.shared.w_up"] = np.zeros((8, zs.d_model), np.float16)
        wz[f"layers.{l}.shared.w_down"] = np.zeros((zs.d_model, 8), np.float16)
    toks = S.make_tokens(ns, 12, seed=12)
    a = O.Decoder(ns, w).forward_sequence(toks)
    b = O.Decoder(zs, wz).forward_sequence(toks)
    assert np.array_equal(a, b)


def test_one_layer_cache_fill_equals_stepping_the_prompt():
    """The one-layer cache fill (projections of the embedded prompt, for long
    contexts) gives the same cache and the same following logits as
    forwarding the prompt one token at a time."""
    s = S.Shape("t-1l", n_layers=1, d_model=40, n_heads=5, n_kv_heads=2, head_dim=8,
                ffn=24, vocab=53, max_ctx=40)
    w = _scaled(S.make_weights(s, seed=21, cache=False))
    toks = S.make_tokens(s, 30, seed=22)
    a, b = O.Decoder(s, w), O.Decoder(s, w)
    ca, cb = a.new_cache(40), b.new_cache(40)
    for t in toks[:25]:
        a.step(t, ca, want_logits=False)
    b.fill_cache_one_layer(toks[:25], cb)
    assert ca["pos"] == cb["pos"] == 25
    assert np.allclose(ca["K"], cb["K"], rtol=0, atol=1e-12) and np.allclose(ca["V"], cb["V"], rtol=0, atol=1e-12)
    for t in toks[25:]:
        la, lb = a.step(t, ca), b.step(t, cb)
        assert np.allclose(la, lb, rtol=0, atol=1e-10 * np.abs(la).max())
