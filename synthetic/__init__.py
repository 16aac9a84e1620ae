"""Seeded synthetic inputs shared by the oracle and the CUDA path.

This module holds the model shapes of the five decoder workloads and the seeded
draws of their weights and prompts. It holds none of the decode arithmetic: no
normalisation, attention, projection or sampling lives here, so that the oracle
and the GPU engine, which both read these inputs, share no computation.

Conventions (a reading of the workload descriptions; the pages give no
architecture, only that the matrix products, attention, normalisations and
token choice all run inside the persistent kernel: "メモリの壁を打破する：
標準的なGPUで3,000 tokens/sの推論を実現する", section "1. The Monokernel Runtime"):

* "N(0, s)" is a normal distribution with standard deviation s.
* Each tensor has its own torch CPU generator seeded with
  ``seed * 1000003 + crc32(name)``; values are drawn row-major in fp32 and then
  rounded to fp16 (round to nearest even).
* Matrices and the embedding / LM head are N(0, 0.02); norm gains are
  1 + 0.01 * N(0, 1); the MoE router is N(0, 0.02).
* The long-context workload uses "the same weights" as the 2.2B workload with
  fewer KV heads: the per-tensor streams are the same, so its Wk and Wv are the
  first n_kv_heads * head_dim rows of the 2.2B workload's matrices (torch fills
  row-major, so a shorter draw is a prefix of a longer one; a test checks it).
* Prompt tokens are ``torch.randint(0, vocab, (P,))`` from a generator seeded
  with ``seed + 1``.

Tensor names and shapes ([rows, cols], row-major, W[out, in] so y = W x):

    embed                 [V, d]
    layers.{l}.attn_norm  [d]
    layers.{l}.wq         [hq*dh, d]
    layers.{l}.wk         [hk*dh, d]
    layers.{l}.wv         [hk*dh, d]
    layers.{l}.wo         [d, hq*dh]
    layers.{l}.mlp_norm   [d]
    dense FFN:  layers.{l}.w_gate [ff, d], layers.{l}.w_up [ff, d], layers.{l}.w_down [d, ff]
    MoE FFN:    layers.{l}.router [E, d]
                layers.{l}.experts.{e}.w_gate / w_up [ffe, d], .w_down [d, ffe]
                layers.{l}.shared.w_gate / w_up [ffs, d], .w_down [d, ffs]
    final_norm            [d]
    lm_head               [V, d]
"""
from __future__ import annotations

import dataclasses
import os
import zlib
from concurrent.futures import ThreadPoolExecutor

import numpy as np


@dataclasses.dataclass(frozen=True)
class Shape:
    """Shape of one decoder workload (no arithmetic, sizes only)."""

    name: str
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int            # dense SwiGLU width (0 for MoE)
    vocab: int
    n_experts: int = 0  # routed experts (0 = dense)
    top_k: int = 0
    ffn_expert: int = 0
    ffn_shared: int = 0
    prompt_len: int = 16
    decode_len: int = 32
    max_ctx: int = 64
    rms_eps: float = 1e-5
    rope_theta: float = 10000.0

    @property
    def is_moe(self) -> bool:
        return self.n_experts > 0

    def with_(self, **kw) -> "Shape":
        return dataclasses.replace(self, **kw)


# The five workloads (sizes as the workload descriptions state them).
TINY = Shape("tiny-2L-d256", n_layers=2, d_model=256, n_heads=4, n_kv_heads=4,
             head_dim=64, ffn=1024, vocab=4096, prompt_len=16, decode_len=32,
             max_ctx=64)
SMALL = Shape("0.5B-16L-d1536", n_layers=16, d_model=1536, n_heads=12,
              n_kv_heads=12, head_dim=128, ffn=4096, vocab=32000,
              prompt_len=128, decode_len=512, max_ctx=640)
DENSE_2B = Shape("2.2B-26L-d2560", n_layers=26, d_model=2560, n_heads=20,
                 n_kv_heads=20, head_dim=128, ffn=6912, vocab=32000,
                 prompt_len=256, decode_len=1024, max_ctx=1280)
LONG_2B = DENSE_2B.with_(name="2.2B-26L-d2560-gqa20:8-32k", n_kv_heads=8,
                         prompt_len=32768, decode_len=256, max_ctx=33024)
MOE = Shape("moe-24L-d2048-16x1408-top2", n_layers=24, d_model=2048,
            n_heads=16, n_kv_heads=4, head_dim=128, ffn=0, vocab=32000,
            n_experts=16, top_k=2, ffn_expert=1408, ffn_shared=2816,
            prompt_len=128, decode_len=512, max_ctx=640)

CONFIGS = {1: TINY, 2: SMALL, 3: DENSE_2B, 4: LONG_2B, 5: MOE}

# Reduced long-context case that the oracle can finish: same weights,
# a 2048-token prompt and 32 decode steps.
LONG_2B_REDUCED = LONG_2B.with_(name="2.2B-26L-d2560-gqa20:8-2k",
                                prompt_len=2048, decode_len=32, max_ctx=2080)


def tensor_specs(s: Shape):
    """(name, shape, kind) for every tensor; kind is 'w' (N(0,0.02)) or 'g' (gain)."""
    d, dh = s.d_model, s.head_dim
    out = [("embed", (s.vocab, d), "w")]
    for l in range(s.n_layers):
        p = f"layers.{l}."
        out += [(p + "attn_norm", (d,), "g"),
                (p + "wq", (s.n_heads * dh, d), "w"),
                (p + "wk", (s.n_kv_heads * dh, d), "w"),
                (p + "wv", (s.n_kv_heads * dh, d), "w"),
                (p + "wo", (d, s.n_heads * dh), "w"),
                (p + "mlp_norm", (d,), "g")]
        if s.is_moe:
            out.append((p + "router", (s.n_experts, d), "w"))
            for e in range(s.n_experts):
                q = p + f"experts.{e}."
                out += [(q + "w_gate", (s.ffn_expert, d), "w"),
                        (q + "w_up", (s.ffn_expert, d), "w"),
                        (q + "w_down", (d, s.ffn_expert), "w")]
            if s.ffn_shared:  # Qwen-class MoE layers have no shared expert
                q = p + "shared."
                out += [(q + "w_gate", (s.ffn_shared, d), "w"),
                        (q + "w_up", (s.ffn_shared, d), "w"),
                        (q + "w_down", (d, s.ffn_shared), "w")]
        else:
            out += [(p + "w_gate", (s.ffn, d), "w"),
                    (p + "w_up", (s.ffn, d), "w"),
                    (p + "w_down", (d, s.ffn), "w")]
    out += [("final_norm", (d,), "g"), ("lm_head", (s.vocab, d), "w")]
    return out


def _draw(name: str, shape, kind: str, seed: int) -> np.ndarray:
    import torch

    g = torch.Generator().manual_seed(seed * 1000003 + zlib.crc32(name.encode()))
    z = torch.randn(shape, generator=g, dtype=torch.float32)
    if kind == "g":
        z = 1.0 + 0.01 * z
    else:
        z = 0.02 * z
    return z.to(torch.float16).numpy()


def _cache_dir() -> str | None:
    d = os.environ.get("KIE_SYNTH_CACHE")
    if d == "":
        return None
    return d or os.path.join(os.environ.get("TMPDIR", "/tmp"), "kie_synth_cache")


def make_weights(s: Shape, seed: int = 0, threads: int | None = None,
                 cache: bool = True) -> dict[str, np.ndarray]:
    """All weights of workload ``s`` as fp16 numpy arrays (seeded, deterministic).

    Large workloads are cached as .npy files (per tensor name and seed) under
    $KIE_SYNTH_CACHE (default $TMPDIR/kie_synth_cache); set it to "" to disable.
    """
    specs = tensor_specs(s)
    cdir = _cache_dir() if cache else None

    def one(spec):
        name, shape, kind = spec
        path = None
        if cdir is not None and int(np.prod(shape)) >= (1 << 20):
            path = os.path.join(cdir, f"s{seed}", f"{name}.{'x'.join(map(str, shape))}.npy")
            if os.path.exists(path):
                try:
                    return name, np.load(path, mmap_mode=None)
                except Exception:
                    pass
        a = _draw(name, shape, kind, seed)
        if path is not None:
            os.makedirs(os.path.dirname(path), exist_ok=True)
            tmp = f"{path}.{os.getpid()}.tmp.npy"
            np.save(tmp, a)
            os.replace(tmp, path)
        return name, a

    n = threads or min(16, os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=n) as ex:
        return dict(ex.map(one, specs))


def make_prompt(s: Shape, seed: int = 0, length: int | None = None) -> np.ndarray:
    """Prompt token ids, uniform over the vocabulary (int32)."""
    import torch

    g = torch.Generator().manual_seed(seed + 1)
    P = s.prompt_len if length is None else length
    return torch.randint(0, s.vocab, (P,), generator=g).to(torch.int32).numpy()


def make_tokens(s: Shape, n: int, seed: int) -> np.ndarray:
    """Extra uniform token ids (for teacher forcing with a seeded continuation)."""
    import torch

    g = torch.Generator().manual_seed(seed * 7919 + 17)
    return torch.randint(0, s.vocab, (n,), generator=g).to(torch.int32).numpy()


def weight_bytes(s: Shape) -> int:
    return sum(int(np.prod(sh)) * 2 for _, sh, _ in tensor_specs(s))
