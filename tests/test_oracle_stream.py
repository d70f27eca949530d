"""Pins for the oracle's stream format, byte accounting and the end-to-end codec (CPU only)."""
import numpy as np
import pytest

import synth
from oracle import jolt, stream


@pytest.fixture(scope="module")
def c0_stream():
    cfg = synth.config(0)
    K, _ = synth.gen_cache_numpy(cfg)
    plan = jolt.Plan(L=1, H=8, T=256, D=128, has_v=False, budget=synth.kv.budget_bytes(cfg, 2.0),
                     num_groups=1, encoder="exact", out_f32=True)
    st, dbg = jolt.encode(plan, K, None, seed=42)
    return cfg, K, plan, st, dbg


def small_kv(seed=3, L=4):
    cfg = synth.config(1, layers=L, tokens=128, seed=seed)
    K, V = synth.gen_cache_numpy(cfg)
    return cfg, K, V


def test_serialize_parse_roundtrip(c0_stream):
    _, K, plan, st, _ = c0_stream
    buf = stream.serialize(st)
    st2 = stream.parse(buf)
    assert np.array_equal(st2.alloc, st.alloc)
    for lt, c in st.lts.items():
        c2 = st2.lts[lt]
        for f in ("U_T", "U_D", "G", "scales", "codes"):
            assert np.array_equal(getattr(c, f), getattr(c2, f))
    assert stream.serialize(st2) == buf


def test_crc_and_header_checks(c0_stream):
    buf = bytearray(stream.serialize(c0_stream[3]))
    bad = bytearray(buf)
    bad[len(bad) // 2] ^= 0x10
    with pytest.raises(stream.CorruptStream):
        stream.parse(bytes(bad))
    with pytest.raises(stream.CorruptStream):
        stream.parse(b"JOLX" + bytes(buf[4:]))
    with pytest.raises(stream.CorruptStream):
        stream.parse(bytes(buf[:-1]))


def test_byte_accounting_matches_stream_arrays_and_budget(c0_stream):
    _, K, plan, st, _ = c0_stream
    layout, _ = stream.body_layout(st.L, st.H, st.T, st.D, st.has_v, st.num_groups, st.alloc)
    total = 0
    for lt, parts in layout.items():
        c = st.lts[lt]
        assert sum(s for _, s in parts) == jolt.layer_bytes(st.H, st.T, st.D, c.rt, c.rd, c.b)
        assert all(o % stream.ALIGN == 0 for o, _ in parts)
        total += sum(s for _, s in parts)
    assert total <= plan.budget


def test_c0_end_to_end_quality(c0_stream):
    _, K, plan, st, _ = c0_stream
    Kh, _ = jolt.decode(st)
    e = jolt.rel_frob(K, Kh)
    assert e < 0.02
    Kh2, _ = jolt.decode(stream.parse(stream.serialize(st)))
    assert np.array_equal(Kh, Kh2)


def test_split_pools_each_meet_their_budget_and_error_falls_with_budget():
    cfg, K, V = small_kv()
    full = synth.bf16_bytes(cfg)
    errs = []
    for ratio in (4.0, 3.0, 2.0):
        plan = jolt.Plan(L=cfg.layers, H=cfg.heads, T=cfg.tokens, D=cfg.head_dim, has_v=True,
                         budget=int(full / ratio), num_groups=2, encoder="sketch", split_kv=True)
        st, dbg = jolt.encode(plan, K, V, seed=42)
        for kinds, bud in plan.pools():
            used = sum(jolt.layer_bytes(st.H, st.T, st.D, *st.alloc[g, k]) * len(lay)
                       for g, lay in enumerate(jolt.group_ranges(st.L, st.num_groups)) for k in kinds)
            assert used <= bud
        Kh, Vh = jolt.decode(st)
        errs.append((jolt.rel_frob(K, Kh), jolt.rel_frob(V, Vh)))
    for (k1, v1), (k2, v2) in zip(errs, errs[1:]):
        assert k2 < k1 and v2 < v1


def test_sketch_close_to_exact_quality():
    """FlashJoLT's 'matched quality': sketch error within 5% of exact on a small GQA cache."""
    cfg, K, V = small_kv(5)
    out = {}
    for enc in ("exact", "sketch"):
        plan = jolt.Plan(L=cfg.layers, H=cfg.heads, T=cfg.tokens, D=cfg.head_dim, has_v=True,
                         budget=synth.bf16_bytes(cfg) // 2, num_groups=2, encoder=enc, split_kv=True)
        st, _ = jolt.encode(plan, K, V, seed=42)
        Kh, Vh = jolt.decode(st)
        out[enc] = (jolt.rel_frob(K, Kh), jolt.rel_frob(V, Vh))
    for i in range(2):
        assert out["sketch"][i] <= 1.05 * out["exact"][i]


def test_stored_values_are_on_their_grids(c0_stream):
    from oracle import numerics as nm
    st = c0_stream[3]
    for c in st.lts.values():
        for a in (c.U_T, c.U_D, c.G):
            assert np.array_equal(nm.round_bf16(a), a)
        assert np.array_equal(nm.round_fp16_sat(c.scales), c.scales)
