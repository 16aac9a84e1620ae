"""The weight-tape plan (kie_plan) on the host, no GPU: every matrix row is
owned by exactly one CTA, the tape is each CTA's ranges back to back in
execution order, tiles fit the ring stages, and the residual rows a CTA
owns are the same in every layer (the kernel keeps them in shared memory)."""
import ctypes

import numpy as np
import pytest

import synthetic as S
from transformer_decode_persistent_b200 import build as B
from transformer_decode_persistent_b200 import kie as K

GQA_ODD = S.Shape("gqa-odd", n_layers=3, d_model=512, n_heads=10, n_kv_heads=8, head_dim=64, ffn=1376,
                  vocab=5000, max_ctx=64)
MOE_SMALL = S.Shape("moe-small", n_layers=2, d_model=512, n_heads=8, n_kv_heads=2, head_dim=64, ffn=0,
                    vocab=3000, n_experts=6, top_k=2, ffn_expert=352, ffn_shared=704, max_ctx=64)
MOE_NOSHARED = S.Shape("moe-noshared", n_layers=2, d_model=512, n_heads=8, n_kv_heads=2, head_dim=64, ffn=0,
                       vocab=3000, n_experts=64, top_k=8, ffn_expert=128, ffn_shared=0, max_ctx=64)
SHAPES = [S.TINY, S.SMALL, S.DENSE_2B, S.LONG_2B, S.MOE, GQA_ODD, MOE_SMALL, MOE_NOSHARED]
GEOMETRY = [(148, 13312), (132, 16384), (148, 9088), (148, 8192)]
PART_FLOATS = 1280  # per-CTA partial sums the kernel holds for one phase


@pytest.fixture(scope="module", autouse=True)
def _built():
    B.build()


def rows_of(shape, kind):
    hq, hk, dh, d = shape.n_heads, shape.n_kv_heads, shape.head_dim, shape.d_model
    return {"qkv": (hq + 2 * hk) * dh, "o": d, "gate_up": 2 * shape.ffn, "down": d,
            "shared_gate_up": 2 * shape.ffn_shared, "expert_gate_up": 2 * shape.ffn_expert,
            "shared_down": d, "expert_down": d, "lm_head": shape.vocab}[kind]


def slot_kinds(shape):
    E = shape.n_experts
    if not E:
        return ["qkv", "o", "gate_up", "down"]
    return ["qkv", "o", "shared_gate_up", "shared_down"] + ["expert_gate_up"] * E + ["expert_down"] * E


@pytest.mark.parametrize("grid,stage", GEOMETRY)
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
def test_plan_invariants(shape, grid, stage):
    info, r = K.plan(shape, grid, stage)
    L, slots = shape.n_layers, info["slots"]
    kinds = slot_kinds(shape)
    assert slots == len(kinds) and info["ranges_per_cta"] == L * slots + 1
    assert r.shape == (grid, L * slots + 1)
    sh = info["shapes"]

    # tile shapes: K split exactly into column blocks of 8-half chunks; tiles fit a stage
    for kind in set(kinds) | {"lm_head"}:
        s = sh[kind]
        assert s["nk"] * s["kc"] == s["K"] and s["kc"] % 8 == 0
        assert 1 <= s["g"] <= (13 if s["kc"] == 512 else 8)
        assert s["g"] * s["kc"] * 2 <= stage

    # every row of every matrix owned by exactly one CTA; pair units stay whole
    def check_partition(col, kind):
        rr = r[:, col]
        if rows_of(shape, kind) == 0:  # e.g. the shared expert of a model without one
            assert (rr["nrows"] == 0).all()
            return
        order = np.argsort(rr["row0"], kind="stable")
        row0, n = rr["row0"][order], rr["nrows"][order]
        keep = n > 0
        row0, n = row0[keep], n[keep]
        assert row0[0] == 0 and (row0[1:] == (row0 + n)[:-1]).all()
        assert int(n.sum()) == rows_of(shape, kind)
        unit = 2 if kind in ("qkv", "gate_up", "shared_gate_up", "expert_gate_up") else 1
        if unit == 2:
            assert (rr["row0"] % 2 == 0).all() and (rr["nrows"] % 2 == 0).all()
        # near-equal split: CTAs differ by at most one unit
        assert int(rr["nrows"].max()) - int(rr["nrows"].min()) <= unit

    for l in range(L):
        for s_, kind in enumerate(kinds):
            check_partition(l * slots + s_, kind)
    check_partition(L * slots, "lm_head")

    # the residual rows a CTA owns: the same for o and down, in every layer
    res_cols = [l * slots + s_ for l in range(L) for s_, k in enumerate(kinds)
                if k in ("o", "down", "shared_down", "expert_down")]
    ref = r[:, res_cols[0]]
    for c in res_cols[1:]:
        assert (r[:, c]["row0"] == ref["row0"]).all() and (r[:, c]["nrows"] == ref["nrows"]).all()

    # the tape: each CTA's ranges back to back in execution order, CTAs in order
    K_of = [sh[k]["K"] for k in kinds]
    off = 0
    for c in range(grid):
        for l in range(L):
            for s_ in range(slots):
                e = r[c, l * slots + s_]
                assert e["off"] == off
                off += int(e["nrows"]) * K_of[s_] * 2
        e = r[c, L * slots]
        assert e["off"] == off
        off += int(e["nrows"]) * sh["lm_head"]["K"] * 2
    assert off == info["tape_bytes"]

    # partial sums per phase fit the kernel's buffer (dense phases); gate/up
    # and the LM head run in row chunks, so one tile group has to fit
    if not shape.n_experts:
        for l in range(L):
            for s_, kind in enumerate(kinds):
                n = r[:, l * slots + s_]["nrows"]
                if kind == "gate_up":
                    n = np.minimum(n, sh[kind]["g"])
                assert (n * sh[kind]["nk"] <= PART_FLOATS).all()
        n = np.minimum(r[:, L * slots]["nrows"], sh["lm_head"]["g"])
        assert (n * sh["lm_head"]["nk"] <= PART_FLOATS).all()


def test_plan_tape_is_the_weight_bytes():
    """The tape holds every matrix exactly once: its size is the sum of the
    matrices' fp16 bytes (experts included), independent of the geometry."""
    for shape in SHAPES:
        hq, hk, dh, d, L = shape.n_heads, shape.n_kv_heads, shape.head_dim, shape.d_model, shape.n_layers
        per_layer = ((hq + 2 * hk) * dh * d + d * hq * dh) * 2
        if shape.n_experts:
            per_layer += 3 * d * (shape.ffn_shared + shape.n_experts * shape.ffn_expert) * 2
        else:
            per_layer += 3 * d * shape.ffn * 2
        want = L * per_layer + shape.vocab * d * 2
        for grid, stage in GEOMETRY:
            assert K.plan(shape, grid, stage)[0]["tape_bytes"] == want


@pytest.mark.parametrize("grid,stage,cap", [(0, 13312, None), (148, 4000, None), (148, 13320, None),
                                            (148, 13312, 10)])
def test_plan_rejects_bad_arguments(grid, stage, cap):
    L = K.lib()
    cfg = K.config_from(S.TINY)
    info = K.kie_plan_info()
    buf = (K.kie_seg_range * 16)() if cap else None
    st = L.kie_plan(ctypes.byref(cfg), grid, stage, ctypes.byref(info), buf, cap or 0)
    assert st == -1 and L.kie_last_error(None)


def test_plan_stage_holds_an_attention_sub_block():
    """A ring stage also carries 32 K or V rows of one head: 8 KiB at head_dim
    128, 4 KiB at 64. Smaller stages are rejected before anything could copy
    past one."""
    K.plan(S.TINY, 148, 4096)  # head_dim 64
    with pytest.raises(K.KieError) as ei:
        K.plan(S.DENSE_2B, 148, 6144)  # head_dim 128
    assert ei.value.status == -1 and "attention sub-block" in str(ei.value)
    K.plan(S.DENSE_2B, 148, 8192)


def test_plan_rejects_shapes_like_create():
    L = K.lib()
    info = K.kie_plan_info()
    for bad in (dict(head_dim=96), dict(n_kv_heads=8), dict(d_model=100)):
        base = {f: getattr(K.config_from(S.TINY), f) for f, _ in K.kie_config._fields_}
        base.update(bad)
        cfg = K.kie_config(**base)
        assert L.kie_plan(ctypes.byref(cfg), 148, 13312, ctypes.byref(info), None, 0) == -1
    assert L.kie_plan(None, 148, 13312, ctypes.byref(info), None, 0) == -1


def test_plan_rejects_more_partial_sums_than_the_kernel_holds():
    """The LM head runs in row chunks, so 32000 rows over 16 CTAs (2000 rows
    per CTA) plan fine; a down projection is not chunked, and 64 rows per CTA
    of a 30720-wide one (40 column blocks of 768) are more partial sums than
    one CTA holds."""
    info, _ = K.plan(S.SMALL, 16, 13312)
    assert info["shapes"]["lm_head"]["g"] * info["shapes"]["lm_head"]["nk"] <= 1280
    wide = S.Shape("wide-down", n_layers=1, d_model=1024, n_heads=8, n_kv_heads=8, head_dim=128,
                   ffn=30720, vocab=1000, max_ctx=16)
    with pytest.raises(K.KieError) as ei:
        K.plan(wide, 16, 13312)
    assert ei.value.status == -1 and "partial sums" in str(ei.value)


@pytest.mark.parametrize("shape", [S.SMALL, S.DENSE_2B, S.LONG_2B, S.MOE], ids=lambda s: s.name)
def test_plan_balances_the_tape_over_ctas(shape):
    """Every SM streams about the same number of weight bytes: the per-CTA
    tape regions are within 3 % of their mean (148 CTAs, 13 KB stages)."""
    info, r = K.plan(shape, 148, 13312)
    starts = r["off"][:, 0].astype(np.int64)
    sizes = np.append(starts[1:], info["tape_bytes"]) - starts
    assert sizes.max() <= 1.03 * sizes.mean() and sizes.min() >= 0.97 * sizes.mean()


def test_plan_accepts_wide_gqa_groups_and_rejects_what_the_attention_cannot_split():
    """Up to 16 query heads per KV head are attended in equal sub-units of at
    most 4 (8:1 Llama-3-70B-like, 7:1 Qwen-like layouts plan); more than 16, or
    uneven groups that would leave a sub-unit without a head (25 query heads
    over 2 KV heads: groups of 13 and 12 in sub-units of 4), are rejected."""
    for hq, hk in ((32, 4), (64, 8), (28, 4), (14, 2)):
        s = S.Shape(f"gqa-{hq}:{hk}", n_layers=1, d_model=hq * 64, n_heads=hq, n_kv_heads=hk, head_dim=64,
                    ffn=1024, vocab=1000, max_ctx=64)
        K.plan(s, 148, 13312)
    # uneven groups of 9 and 10 query heads (sub-units of 4, 4 and 1 or 2) on a
    # grid of 112 CTAs, fewer than one chunk's 120 attention units
    s = S.Shape("gqa-367:40-d112", n_layers=1, d_model=112, n_heads=367, n_kv_heads=40, head_dim=64,
                ffn=224, vocab=1000, max_ctx=612)
    K.plan(s, 112, 13312)
    for hq, hk in ((34, 2), (25, 2)):
        s = S.Shape(f"gqa-{hq}:{hk}", n_layers=1, d_model=hq * 64, n_heads=hq, n_kv_heads=hk, head_dim=64,
                    ffn=1024, vocab=1000, max_ctx=64)
        with pytest.raises(K.KieError) as ei:
            K.plan(s, 148, 13312)
        assert ei.value.status == -1 and "query heads" in str(ei.value)


def test_plan_moe_without_shared_expert():
    """ffn_shared = 0 is a valid MoE shape; a negative or unaligned width is not."""
    K.plan(MOE_NOSHARED, 148, 13312)
    for bad in (-8, 12):
        with pytest.raises(K.KieError):
            K.plan(MOE_NOSHARED.with_(ffn_shared=bad), 148, 13312)
