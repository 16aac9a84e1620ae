"""fp64 CPU oracle for batch-1 greedy decode of a dense (or MoE) decoder.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. The GPU engine never calls it and shares no code with it; the two meet
only in the seeded inputs of the ``synthetic`` module.

What it computes. The pages describe one persistent GPU program that performs
the whole per-token decode step (the matrix products, attention, normalisations
and the token choice) and emits output tokens one by one without returning to
the host
("メモリの壁を打破する：標準的なGPUで3,000 tokens/sの推論を実現する", section
"1. The Monokernel Runtime"; "Kog、より深いGPU最適化でAI推論を高速化できると賭ける",
section "KogがGPU推論の最適化をさらに深める理由"). Batch-1 decode with a KV cache
reaches exactly the full-sequence causal forward, only faster, so this oracle
is that plain definition written out: a pre-norm decoder with RMSNorm, RoPE,
causal softmax attention, a SwiGLU MLP (or a top-k routed MoE with a shared
expert), an untied LM head and greedy argmax. The pages do not fix the layer
math; the readings taken (all listed in the design notes) are:

* RMSNorm: y = x / sqrt(mean(x^2) + eps) * g (eps inside the root, gain after).
* RoPE: half-split pairs (i, i + dh/2), angle p * theta^(-2i/dh), 0-based p,
  applied to q and k only.
* Attention: scores q.k / sqrt(dh) over positions 0..p, max-subtracted
  softmax; query head h reads KV head floor(h * hk / hq).
* SwiGLU: down(silu(gate(xn)) * up(xn)), silu(z) = z / (1 + exp(-z)).
* MoE: softmax over all router logits, the top-k (lowest index on ties),
  weights renormalised over the chosen k, plus the shared expert at weight 1.
* Greedy: argmax with the lowest index on exact ties; the margin is the top
  value minus the second-largest value (0 on a tie).
* No biases, no QK-norm, no logit scaling. Weights are fp16 and widened to
  fp64 at use.
* The KV cache is fp16: the workload descriptions fix it (the cache, and the
  prompt prefilled into it, are fp16) and the method's attention reads an
  fp16 cache. So K (after RoPE) and V are rounded to fp16 (round to nearest even)
  when they enter the cache, in both the incremental and the full-sequence
  form; every other step stays in fp64. ``kv_fp16=False`` keeps them
  unrounded (for diagnosis).

Everything is float64, single process; numpy's matrix product is used as the
plain library primitive for y = W x (and X W^T in the full-sequence form).
"""
from __future__ import annotations

import numpy as np


# ---------------------------------------------------------------- primitives

def f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def rmsnorm(x, g, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * g.

    The "normalization" step of the monokernel ("1. The Monokernel Runtime");
    its type (RMS, eps inside the root, gain after) is the workload's reading.
    """
    x = f64(x)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * f64(g)


def rope(u, pos, theta: float) -> np.ndarray:
    """Rotary position embedding, half-split pairing.

    ``u`` has shape [..., H, dh]; ``pos`` is a scalar position or an array of
    positions matching the leading axes of ``u`` without the head axis. Pair
    (u_i, u_{i+dh/2}) is rotated by phi = pos * theta^(-2 i / dh):
    (a, b) -> (a cos phi - b sin phi, a sin phi + b cos phi).
    """
    u = f64(u)
    dh = u.shape[-1]
    half = dh // 2
    i = np.arange(half, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / dh)
    p = np.asarray(pos, dtype=np.float64)
    phi = p[..., None] * inv_freq                 # [..., half]
    phi = phi[..., None, :]                        # broadcast over heads
    c, s = np.cos(phi), np.sin(phi)
    a, b = u[..., :half], u[..., half:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def softmax(s) -> np.ndarray:
    """Max-subtracted softmax over the last axis (masked entries = -inf)."""
    s = f64(s)
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def kv_head_of(h: int, n_heads: int, n_kv_heads: int) -> int:
    """KV head read by query head h: floor(h * hk / hq)."""
    return (h * n_kv_heads) // n_heads


def attend_one(q, K, V) -> np.ndarray:
    """Attention of one query position over cached positions 0..p.

    q: [hq, dh]; K, V: [hk, p+1, dh]. Returns o: [hq, dh] with
    o_h = sum_j softmax_j(q_h . k_{g,j} / sqrt(dh)) v_{g,j}, g = kv_head_of(h).
    The "attention" step of the monokernel ("1. The Monokernel Runtime").
    """
    q, K, V = f64(q), f64(K), f64(V)
    hq, dh = q.shape
    hk = K.shape[0]
    o = np.empty((hq, dh))
    for h in range(hq):
        g = kv_head_of(h, hq, hk)
        s = K[g] @ q[h] / np.sqrt(dh)
        o[h] = softmax(s) @ V[g]
    return o


def causal_attention(q, k, v) -> np.ndarray:
    """Full-sequence causal attention. q: [T, hq, dh]; k, v: [T, hk, dh].

    Row t attends to positions j <= t only. Returns [T, hq, dh].
    """
    q, k, v = f64(q), f64(k), f64(v)
    T, hq, dh = q.shape
    hk = k.shape[1]
    mask = np.triu(np.ones((T, T), dtype=bool), k=1)   # j > t is masked
    o = np.empty_like(q)
    for h in range(hq):
        g = kv_head_of(h, hq, hk)
        S = q[:, h, :] @ k[:, g, :].T / np.sqrt(dh)     # [T, T]
        S[mask] = -np.inf
        o[:, h, :] = softmax(S) @ v[:, g, :]
    return o


def silu(z) -> np.ndarray:
    z = f64(z)
    return z / (1.0 + np.exp(-z))


def swiglu_ffn(xn, w_gate, w_up, w_down) -> np.ndarray:
    """down(silu(gate . xn) * (up . xn)); works on [d] or [T, d] inputs."""
    xn = f64(xn)
    g = xn @ f64(w_gate).T
    u = xn @ f64(w_up).T
    return (silu(g) * u) @ f64(w_down).T


def argmax_lowest(v) -> int:
    """Index of the largest value; the lowest such index on exact ties."""
    v = f64(v)
    return int(np.flatnonzero(v == np.max(v))[0])


def top2_margin(v) -> float:
    """Largest value minus the second-largest value (0 when the top is tied)."""
    v = f64(v)
    i = argmax_lowest(v)
    rest = np.delete(v, i)
    return float(v[i] - np.max(rest))


def topk_lowest(v, k: int) -> list[int]:
    """The k largest entries, ordered by value, ties broken by lower index."""
    v = f64(v)
    order = sorted(range(len(v)), key=lambda i: (-v[i], i))
    return order[:k]


def moe_ffn(xn, router, experts, shared, top_k: int) -> np.ndarray:
    """Routed SwiGLU experts plus an always-on shared expert, for one token.

    router: [E, d]; experts: list of (w_gate, w_up, w_down); shared: the same
    triple, or None for a model without one (Qwen-class layers). r =
    softmax(router . xn) over all E; the top-k experts (lowest index on ties)
    are weighted by r_e / sum of the chosen r; the shared expert is added with
    weight 1. Active-parameter streaming is what the pages say
    bounds MoE decode ("スケーリングをFrontier MoEモデルへ").
    """
    xn = f64(xn)
    r = softmax(xn @ f64(router).T)
    chosen = topk_lowest(r, top_k)
    wsum = sum(r[e] for e in chosen)
    y = swiglu_ffn(xn, *shared) if shared is not None else np.zeros_like(xn)
    for e in chosen:
        y = y + (r[e] / wsum) * swiglu_ffn(xn, *experts[e])
    return y


# ---------------------------------------------------------------- the model

def fp16_round(a) -> np.ndarray:
    """Round to the nearest fp16 value (ties to even), returned as float64."""
    return np.asarray(a, dtype=np.float64).astype(np.float16).astype(np.float64)


class Decoder:
    """The whole decoder over fp16 weights from ``synthetic.make_weights``.

    ``cache_f64`` keeps a widened copy of each matrix after its first use
    (memory for speed; the values are the same either way). ``kv_fp16``
    rounds cached K and V to fp16 (the workloads' fp16 KV cache).
    """

    def __init__(self, shape, weights: dict, cache_f64: bool = True, kv_fp16: bool = True):
        self.s = shape
        self.w16 = weights
        self._w64 = {} if cache_f64 else None
        self.kv = fp16_round if kv_fp16 else f64
        # gap between the k-th and (k+1)-th largest router logit of every MoE
        # decision taken (how close each routing was to a tie; diagnostic
        # only). ``step`` appends one per layer; ``forward_sequence`` one per
        # row for each layer in turn (layer-major).
        self.route_gaps: list[float] = []

    def W(self, name: str) -> np.ndarray:
        if self._w64 is None:
            return f64(self.w16[name])
        a = self._w64.get(name)
        if a is None:
            a = f64(self.w16[name])
            self._w64[name] = a
        return a

    def _ffn(self, l: int, xn):
        s, p = self.s, f"layers.{l}."
        if not s.is_moe:
            return swiglu_ffn(xn, self.W(p + "w_gate"), self.W(p + "w_up"),
                              self.W(p + "w_down"))
        experts = [(self.W(p + f"experts.{e}.w_gate"),
                    self.W(p + f"experts.{e}.w_up"),
                    self.W(p + f"experts.{e}.w_down")) for e in range(s.n_experts)]
        shared = (self.W(p + "shared.w_gate"), self.W(p + "shared.w_up"),
                  self.W(p + "shared.w_down")) if s.ffn_shared else None
        if np.ndim(xn) == 1:
            return moe_ffn(xn, self.W(p + "router"), experts, shared, s.top_k)
        # diagnostic only: how close each row's routing came to a tie
        for r in xn @ self.W(p + "router").T:
            srt = np.sort(r)[::-1]
            self.route_gaps.append(float(srt[s.top_k - 1] - srt[s.top_k]))
        return np.stack([moe_ffn(r, self.W(p + "router"), experts, shared, s.top_k)
                         for r in xn])

    def _moe_ffn_lazy(self, l: int, xn):
        """One token's MoE FFN, widening only the experts it chooses."""
        s, p = self.s, f"layers.{l}."
        logit = xn @ self.W(p + "router").T
        r = softmax(logit)
        chosen = topk_lowest(r, s.top_k)
        srt = np.sort(logit)[::-1]
        self.route_gaps.append(float(srt[s.top_k - 1] - srt[s.top_k]))
        wsum = sum(r[e] for e in chosen)
        y = (swiglu_ffn(xn, self.W(p + "shared.w_gate"), self.W(p + "shared.w_up"),
                        self.W(p + "shared.w_down")) if s.ffn_shared else np.zeros_like(xn))
        for e in chosen:
            q = p + f"experts.{e}."
            y = y + (r[e] / wsum) * swiglu_ffn(xn, self.W(q + "w_gate"),
                                                self.W(q + "w_up"), self.W(q + "w_down"))
        return y

    # ---- full-sequence recompute (the plain definition)
    def forward_sequence(self, tokens) -> np.ndarray:
        """Logits [T, V] of the causal forward over ``tokens`` (positions 0..T-1)."""
        s = self.s
        tokens = np.asarray(tokens)
        T, dh = len(tokens), s.head_dim
        pos = np.arange(T)
        x = f64(self.w16["embed"][tokens])                  # [T, d]
        for l in range(s.n_layers):
            p = f"layers.{l}."
            xn = rmsnorm(x, self.w16[p + "attn_norm"], s.rms_eps)
            q = (xn @ self.W(p + "wq").T).reshape(T, s.n_heads, dh)
            k = (xn @ self.W(p + "wk").T).reshape(T, s.n_kv_heads, dh)
            v = (xn @ self.W(p + "wv").T).reshape(T, s.n_kv_heads, dh)
            q, k = rope(q, pos, s.rope_theta), rope(k, pos, s.rope_theta)
            k, v = self.kv(k), self.kv(v)
            o = causal_attention(q, k, v).reshape(T, s.n_heads * dh)
            x = x + o @ self.W(p + "wo").T
            xn = rmsnorm(x, self.w16[p + "mlp_norm"], s.rms_eps)
            x = x + self._ffn(l, xn)
        xn = rmsnorm(x, self.w16["final_norm"], s.rms_eps)
        return xn @ self.W("lm_head").T

    # ---- incremental decode with a KV cache
    def new_cache(self, max_ctx: int | None = None):
        s = self.s
        n = max_ctx or s.max_ctx
        return {"pos": 0,
                "K": np.zeros((s.n_layers, s.n_kv_heads, n, s.head_dim)),
                "V": np.zeros((s.n_layers, s.n_kv_heads, n, s.head_dim))}

    def step(self, token: int, cache, want_logits: bool = True):
        """Forward ``token`` at position cache['pos'], append its K/V, advance.

        Returns the logits [V] (None when ``want_logits`` is False).
        """
        s = self.s
        p, dh = cache["pos"], s.head_dim
        x = f64(self.w16["embed"][int(token)])
        for l in range(s.n_layers):
            w = f"layers.{l}."
            xn = rmsnorm(x, self.w16[w + "attn_norm"], s.rms_eps)
            q = (self.W(w + "wq") @ xn).reshape(s.n_heads, dh)
            k = (self.W(w + "wk") @ xn).reshape(s.n_kv_heads, dh)
            v = (self.W(w + "wv") @ xn).reshape(s.n_kv_heads, dh)
            q, k = rope(q, p, s.rope_theta), rope(k, p, s.rope_theta)
            cache["K"][l, :, p, :] = self.kv(k)
            cache["V"][l, :, p, :] = self.kv(v)
            o = attend_one(q, cache["K"][l, :, :p + 1, :], cache["V"][l, :, :p + 1, :])
            x = x + self.W(w + "wo") @ o.reshape(-1)
            xn = rmsnorm(x, self.w16[w + "mlp_norm"], s.rms_eps)
            x = x + (self._moe_ffn_lazy(l, xn) if s.is_moe else self._ffn(l, xn))
        cache["pos"] = p + 1
        if not want_logits:
            return None
        xn = rmsnorm(x, self.w16["final_norm"], s.rms_eps)
        return self.W("lm_head") @ xn

    def fill_cache_one_layer(self, tokens, cache):
        """For a one-layer model: the K/V cache of positions 0..T-1 straight
        from ``tokens``, so a long prompt can be followed without T attention
        steps. Layer 0's key and value at position p are the projections of the
        normalised embedding of token p, rotated (the key) and rounded exactly
        as ``step`` does; they need no attention output, and a one-layer model
        caches nothing else. Advances the cache to position T."""
        s = self.s
        assert s.n_layers == 1 and cache["pos"] == 0
        tokens = np.asarray(tokens)
        T, dh = len(tokens), s.head_dim
        xn = rmsnorm(f64(self.w16["embed"][tokens]), self.w16["layers.0.attn_norm"], s.rms_eps)
        k = (xn @ self.W("layers.0.wk").T).reshape(T, s.n_kv_heads, dh)
        v = (xn @ self.W("layers.0.wv").T).reshape(T, s.n_kv_heads, dh)
        k = rope(k, np.arange(T), s.rope_theta)
        cache["K"][0, :, :T, :] = self.kv(k).transpose(1, 0, 2)
        cache["V"][0, :, :T, :] = self.kv(v).transpose(1, 0, 2)
        cache["pos"] = T

    def greedy(self, prompt, n: int, forced=None, cache=None):
        """Greedy decode of ``n`` tokens after ``prompt``.

        Protocol: positions 0..P-2 are forwarded without logits; the forward
        at P-1 gives the first generated token; each generated token is then
        forwarded in turn (n forwards in all, the first at position P-1).
        ``forced[i] >= 0`` replaces the token fed back after step i (teacher
        forcing); the argmax is still reported. Returns (tokens, logits, margins)
        with tokens the argmax of each step.
        """
        prompt = [int(t) for t in prompt]
        cache = cache or self.new_cache(len(prompt) + n)
        for t in prompt[:-1]:
            self.step(t, cache, want_logits=False)
        cur = prompt[-1]
        toks, logits, margins = [], [], []
        for i in range(n):
            lg = self.step(cur, cache)
            t = argmax_lowest(lg)
            toks.append(t)
            logits.append(lg)
            margins.append(top2_margin(lg))
            cur = t if forced is None or forced[i] < 0 else int(forced[i])
        return np.array(toks, dtype=np.int64), np.stack(logits), np.array(margins)
