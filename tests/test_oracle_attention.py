"""Pins for the oracle's attention over the compressed cache (CPU only).

The plain definition is pinned by closed forms (uniform weights, a dominant key, the grouped-query
head mapping); the factored form, which never rebuilds the cache, is pinned against the plain
definition on encoded streams, and the whole chain against attention over the original cache when
the codec is lossless (full ranks, no residual, float64 storage).
"""
import math

import numpy as np
import pytest

from oracle import attention as oa
from oracle import jolt


def test_uniform_scores_average_the_values():
    """Identical keys (or scale 0) give every token the weight 1/T: the output is the mean value."""
    rng = np.random.default_rng(0)
    H, T, D = 2, 9, 8
    K = np.repeat(rng.standard_normal((H, 1, D)), T, axis=1)
    V = rng.standard_normal((H, T, D))
    Q = rng.standard_normal((H, 3, D))
    out = oa.attention_dense(Q, K, V, 0.7)
    assert np.abs(out - V.mean(axis=1, keepdims=True)).max() < 1e-14
    out0 = oa.attention_dense(Q, rng.standard_normal((H, T, D)), V, 0.0)
    assert np.abs(out0 - V.mean(axis=1, keepdims=True)).max() < 1e-14


def test_dominant_key_selects_its_value():
    """One key aligned with the query and 40 units above the rest: weight 1 - O(T e^-40)."""
    H, T, D = 1, 6, 4
    K = np.zeros((H, T, D))
    K[0, 4, 0] = 40.0
    V = np.arange(H * T * D, dtype=np.float64).reshape(H, T, D)
    Q = np.zeros((1, 1, D))
    Q[0, 0, 0] = 1.0
    out = oa.attention_dense(Q, K, V, 1.0)
    assert np.abs(out[0, 0] - V[0, 4]).max() < 1e-12 * np.abs(V).max() * T


def test_grouped_query_heads_read_their_kv_head():
    """Hq = 6 query heads over H = 2 KV heads: heads 0-2 read KV head 0, heads 3-5 KV head 1."""
    H, T, D, Hq = 2, 5, 4, 6
    K = np.zeros((H, T, D))
    V = np.zeros((H, T, D))
    V[0] += 1.0
    V[1] += 2.0
    Q = np.ones((Hq, 2, D))
    out = oa.attention_dense(Q, K, V, 1.0)
    assert [oa.kv_head_of(j, Hq, H) for j in range(Hq)] == [0, 0, 0, 1, 1, 1]
    assert np.allclose(out[:3], 1.0, atol=0, rtol=0) and np.allclose(out[3:], 2.0, atol=0, rtol=0)


def _stream(L=2, H=2, T=24, D=16, budget_div=2, seed=5, spec=True, bits=(0, 2, 3, 4, 5)):
    """Noise plus a rank-3 token x feature component: at half the bf16 size every layer-tensor
    takes Tucker ranks and a residual (both parts of the factored form are exercised)."""
    rng = np.random.default_rng(11)
    K = rng.standard_normal((L, H, T, D))
    V = rng.standard_normal((L, H, T, D))
    U, W = rng.standard_normal((T, 3)), rng.standard_normal((D, 3))
    K += 10.0 * (U @ W.T)[None, None]
    V += 10.0 * (U[::-1] @ W.T)[None, None]
    plan = jolt.Plan(L=L, H=H, T=T, D=D, has_v=True, budget=L * H * T * D * 2 * 2 // budget_div, num_groups=L,
                     encoder="exact", rank_step=4, bits=bits)
    st, _ = jolt.encode(plan, K, V, seed, spec=spec)
    return st, K, V


@pytest.mark.parametrize("Hq,n", [(2, 1), (8, 3)])
def test_factored_form_equals_the_definition(Hq, n):
    st, _, _ = _stream()
    assert all(st.lts[lt].rt > 0 and st.lts[lt].b > 0 for lt in st.lts), st.alloc
    rng = np.random.default_rng(3)
    for layer in range(st.L):
        Q = rng.standard_normal((Hq, n, st.D))
        a = oa.attention_over_stream(st, layer, Q, 1.0 / math.sqrt(st.D))
        b = oa.attention_factored(st, layer, Q, 1.0 / math.sqrt(st.D))
        assert np.abs(a - b).max() <= 1e-12 * np.abs(a).max()


def test_lossless_codec_gives_attention_over_the_original_cache():
    """Full ranks and b = 0 in float64 storage reproduce K and V, so attention is unchanged."""
    rng = np.random.default_rng(12)
    L, H, T, D = 1, 2, 8, 8
    K = rng.standard_normal((L, H, T, D))
    V = rng.standard_normal((L, H, T, D))
    plan = jolt.Plan(L=L, H=H, T=T, D=D, has_v=True, budget=10 ** 9, num_groups=1, encoder="exact",
                     rank_step=1, rt_cap=T, bits=(0,))
    alloc = np.zeros((1, 2, 3), dtype=np.int64)
    alloc[0, 0] = alloc[0, 1] = (T, D, 0)
    st, _ = jolt.encode(plan, K, V, 1, spec=False, alloc=alloc)
    Q = rng.standard_normal((4, 2, D))
    ref = oa.attention_dense(Q, K[0], V[0], 0.5)
    assert np.abs(oa.attention_factored(st, 0, Q, 0.5) - ref).max() <= 1e-10 * np.abs(ref).max()
