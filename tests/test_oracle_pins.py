"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test checks the oracle against one of:
  * a textbook routine it reduces to in a special case (full causal or
    sliding-window softmax attention, computed here with
    ``torch.nn.functional.scaled_dot_product_attention`` in float64);
  * a closed form (constant streams: EWMA c(1 - gamma^m), ring mean
    c min(t+1,16)/16, basis-vector slots);
  * an unrolled formulation of the whole path on tiny inputs (sums over the
    history instead of recurrences, the pool as library attention);
  * constants and worked numbers the pages print (``tests/golden/``).

Sources (web pages):
  [P1] "Signal Field Attention (SFA)：8KB代码实现4.16倍推理加速与248倍内存压缩"
  [P2] "Signal Field Attention (SFA)" (project README page)
  [P3] "Dalin Soma SFA基于信号场注意力机制的神经网络推理加速框架"
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import OracleParams, OracleState

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TOL = 1e-10


def _rng(seed):
    return np.random.default_rng(seed)


def _run(p, alpha_base, decay, slots, q, k, v, n_layers=None, state=None):
    """Oracle on [L,B,n,...] inputs; returns out [L,B,n,H]."""
    L, B = q.shape[0], q.shape[1]
    st = state if state is not None else OracleState(p, L * B)
    out, _ = oracle.run_layers(p, alpha_base, decay, slots.astype(np.float32),
                               q.astype(np.float32), k.astype(np.float32),
                               v.astype(np.float32), st, n_layers=n_layers)
    return out


def _sdpa_window(q, k, v, window):
    """Softmax attention of one stream with a causal band of ``window`` keys.

    q [n, nq, d]; k, v [n, nkv, d].  KV head of query head h is h // (nq/nkv).
    window=None gives full causal attention.  float64, library routine.
    """
    n, nq, d = q.shape
    nkv = k.shape[1]
    qt = torch.from_numpy(np.asarray(q, np.float64)).permute(1, 0, 2)  # [nq, n, d]
    kt = torch.from_numpy(np.asarray(k, np.float64)).permute(1, 0, 2)
    vt = torch.from_numpy(np.asarray(v, np.float64)).permute(1, 0, 2)
    kt = kt.repeat_interleave(nq // nkv, dim=0)
    vt = vt.repeat_interleave(nq // nkv, dim=0)
    i = torch.arange(n).view(n, 1)
    j = torch.arange(n).view(1, n)
    mask = j <= i
    if window is not None:
        mask = mask & (j > i - window)
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)
    return o.permute(1, 0, 2).reshape(n, nq * d).numpy()


def _pool_library(x, slots, T):
    """Semantic pool as library attention: query x/|x|, keys slot/|slot|,
    values the raw slots, scale 1/T.  x [n, H], slots [P, H]."""
    xt = torch.from_numpy(np.asarray(x, np.float64))
    st = torch.from_numpy(np.asarray(slots, np.float64))
    qn = xt / xt.norm(dim=-1, keepdim=True)
    kn = st / st.norm(dim=-1, keepdim=True)
    o = F.scaled_dot_product_attention(qn.unsqueeze(0), kn.unsqueeze(0), st.unsqueeze(0),
                                       scale=1.0 / T)
    return o.squeeze(0).numpy()


def _inputs(seed, L, B, n, nq, nkv, d, P=64, scale=1.0):
    r = _rng(seed)
    H = nq * d
    q = (r.standard_normal((L, B, n, nq, d)) * scale).astype(np.float32)
    k = (r.standard_normal((L, B, n, nkv, d)) * scale).astype(np.float32)
    v = (r.standard_normal((L, B, n, nkv, d)) * scale).astype(np.float32)
    slots = r.standard_normal((L, P, H)).astype(np.float32)
    return q, k, v, slots


# ---------------------------------------------------------------- near field

@pytest.mark.parametrize("nq,nkv", [(2, 2), (4, 2), (6, 1)])
def test_near_field_is_full_causal_attention_when_n_le_k(nq, nkv):
    """[P1 §2.1 eq. O_near]: while n <= k the window holds every token, so with
    alpha_far = alpha_base = 0 the output is plain causal attention."""
    d, K, n = 8, 12, 12
    q, k, v, slots = _inputs(1, 1, 1, n, nq, nkv, d)
    p = OracleParams(nq, nkv, d, K, gamma_far=0.9, alpha_far=0.0)
    out = _run(p, 0.0, 0.8, slots, q, k, v)[0, 0]
    ref = _sdpa_window(q[0, 0], k[0, 0], v[0, 0], window=None)
    np.testing.assert_allclose(out, ref, rtol=TOL, atol=TOL)


@pytest.mark.parametrize("K", [1, 3, 5])
def test_near_field_is_sliding_window_attention(K):
    """[P1 §2.1 eq. O_near] over the last k tokens, inclusive of token t."""
    nq, nkv, d, n = 4, 2, 8, 23
    q, k, v, slots = _inputs(2, 1, 1, n, nq, nkv, d)
    p = OracleParams(nq, nkv, d, K, gamma_far=0.5, alpha_far=0.0)
    out = _run(p, 0.0, 0.8, slots, q, k, v)[0, 0]
    ref = _sdpa_window(q[0, 0], k[0, 0], v[0, 0], window=K)
    np.testing.assert_allclose(out, ref, rtol=TOL, atol=TOL)


# ----------------------------------------------------------------- far field

def test_far_field_gamma_zero_is_the_evicted_key():
    """[P1 §2.1 eq. S_t] with gamma = 0: S_t is the key leaving the window,
    K_{t-k}, and nothing before the first eviction."""
    nq, nkv, d, K, n = 4, 2, 8, 5, 19
    alpha_far = 0.75
    q, k, v, slots = _inputs(3, 1, 1, n, nq, nkv, d)
    p = OracleParams(nq, nkv, d, K, gamma_far=0.0, alpha_far=alpha_far)
    out = _run(p, 0.0, 0.8, slots, q, k, v)[0, 0]
    near = _sdpa_window(q[0, 0], k[0, 0], v[0, 0], window=K)
    far = (out - near).reshape(n, nq, d) / alpha_far
    for t in range(n):
        for h in range(nq):
            g = h // (nq // nkv)
            want = k[0, 0, t - K, g] if t >= K else np.zeros(d)
            np.testing.assert_allclose(far[t, h], want, rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("gamma", [0.9, 0.98])
def test_far_field_constant_key_stream_closed_form(gamma):
    """Constant keys K == c: after m = t - k + 1 evictions S = c (1 - gamma^m).
    V == 0 makes the near field vanish, so out = alpha_far * S exactly."""
    nq, nkv, d, K, n = 4, 2, 8, 4, 40
    r = _rng(4)
    c = r.standard_normal((nkv, d))
    k = np.broadcast_to(c, (1, 1, n, nkv, d)).astype(np.float32)
    v = np.zeros((1, 1, n, nkv, d), np.float32)
    q = r.standard_normal((1, 1, n, nq, d)).astype(np.float32)
    slots = r.standard_normal((1, 64, nq * d)).astype(np.float32)
    p = OracleParams(nq, nkv, d, K, gamma_far=gamma, alpha_far=1.0)
    out = _run(p, 0.0, 0.8, slots, q, k, v)[0, 0].reshape(n, nq, d)
    c32 = c.astype(np.float32).astype(np.float64)
    for t in range(n):
        m = max(0, t - K + 1)
        for h in range(nq):
            np.testing.assert_allclose(out[t, h], c32[h // 2] * (1 - gamma ** m),
                                       rtol=1e-12, atol=1e-14)


# ------------------------------------------------- ring, field, fusion, clip

def _constant_stream(n, nq, nkv, d, v0, P, slot_vec):
    q = _rng(5).standard_normal((1, 1, n, nq, d)).astype(np.float32)
    k = _rng(6).standard_normal((1, 1, n, nkv, d)).astype(np.float32)
    v = np.broadcast_to(v0, (1, 1, n, nkv, d)).astype(np.float32)
    slots = np.broadcast_to(slot_vec, (1, P, nq * d)).astype(np.float32)
    return q, k, v, slots


def test_ring_field_and_fusion_constant_stream_closed_form():
    """V == v0 and alpha_far = 0 give x_t == v0 (weights sum to one); equal
    slots give sem == slot.  Then, with the [P3 §2.4] /RING_SIZE mean, the
    [P3 §2.1] field recursion and the [P3 §2.2] fusion:
      out_t = x + a * clip(x*min(t+1,16)/16 + 0.5*x*(1-0.98^(t+1)) + 0.5*s)."""
    nq, nkv, d, K, n, P = 4, 2, 8, 4, 40, 64
    r = _rng(7)
    v0 = (0.2 * r.standard_normal((nkv, d))).astype(np.float32)
    s0 = (0.3 * r.standard_normal(nq * d)).astype(np.float32)
    q, k, v, slots = _constant_stream(n, nq, nkv, d, v0, P, s0)
    alpha_base = 0.1
    p = OracleParams(nq, nkv, d, K, gamma_far=0.9, alpha_far=0.0)
    out = _run(p, alpha_base, 0.8, slots, q, k, v)[0, 0]
    x = np.repeat(v0.astype(np.float64), nq // nkv, axis=0).reshape(-1)
    a0 = 0.3 * alpha_base  # layer 0 of a single-layer model
    for t in range(n):
        u = x * min(t + 1, 16) / 16 + 0.5 * x * (1 - 0.98 ** (t + 1)) + 0.5 * s0.astype(np.float64)
        want = x + a0 * np.clip(u, -0.5, 0.5)
        np.testing.assert_allclose(out[t], want, rtol=1e-12, atol=1e-14)


def test_clip_bound_and_saturation():
    """[P3 §2.2]: clip to [-eps, eps] first, then scale by alpha_layer, so
    |out - x| <= eps * alpha_layer, with equality where u saturates."""
    nq, nkv, d, K, n = 4, 2, 8, 4, 30
    q, k, v, slots = _inputs(8, 1, 1, n, nq, nkv, d, scale=3.0)
    p = OracleParams(nq, nkv, d, K, gamma_far=0.9, alpha_far=0.3, clip_eps=0.25)
    x = _run(p, 0.0, 0.8, slots, q, k, v)[0, 0]          # alpha_base = 0 gives out = x
    alpha_base = 7.0
    out = _run(p, alpha_base, 0.8, slots, q, k, v)[0, 0]
    a0 = 0.3 * alpha_base
    dev = np.abs(out - x)
    assert np.all(dev <= 0.25 * a0 * (1 + 1e-12))
    sat = np.isclose(dev, 0.25 * a0, rtol=1e-12)
    assert sat.mean() > 0.2  # inputs of scale 3 saturate many elements
    assert (~sat).mean() > 0.05


# --------------------------------------------------------------- semantic pool

def test_pool_basis_slots_closed_form():
    """Slots beta_j e_j (scaled unit vectors): cos(x, slot_j) = x_j/|x|, so the
    weights are softmax(x_j / (|x| T)) and sem_j = w_j beta_j (raw slots)."""
    nq, nkv, d, K, n, P = 4, 2, 16, 4, 6, 64
    H = nq * d
    r = _rng(9)
    v0 = (0.2 * r.standard_normal((nkv, d))).astype(np.float32)
    beta = (0.5 + r.random(P)).astype(np.float32)
    slots = np.zeros((1, P, H), np.float32)
    slots[0, np.arange(P), np.arange(P)] = beta
    q = r.standard_normal((1, 1, n, nq, d)).astype(np.float32)
    k = r.standard_normal((1, 1, n, nkv, d)).astype(np.float32)
    v = np.broadcast_to(v0, (1, 1, n, nkv, d)).astype(np.float32)
    p = OracleParams(nq, nkv, d, K, gamma_far=0.9, alpha_far=0.0, clip_eps=1e9)
    alpha_base = 1.0
    out = _run(p, alpha_base, 0.8, slots, q, k, v)[0, 0]
    x = np.repeat(v0.astype(np.float64), nq // nkv, axis=0).reshape(-1)
    logits = x[:P] / (np.linalg.norm(x) * 0.07)
    w = np.exp(logits - logits.max())
    w /= w.sum()
    sem = np.zeros(H)
    sem[:P] = w * beta.astype(np.float64)
    a0 = 0.3 * alpha_base
    for t in range(n):
        u = x * min(t + 1, 16) / 16 + 0.5 * x * (1 - 0.98 ** (t + 1)) + 0.5 * sem
        np.testing.assert_allclose(out[t], x + a0 * u, rtol=1e-11, atol=1e-13)


def test_pool_equal_slots_gives_the_slot_for_any_x():
    nq, nkv, d, K, n, P = 4, 2, 8, 4, 9, 64
    q, k, v, _ = _inputs(10, 1, 1, n, nq, nkv, d)
    s0 = _rng(11).standard_normal(nq * d).astype(np.float32) * 0.1
    slots = np.broadcast_to(s0, (1, P, nq * d)).astype(np.float32)
    p = OracleParams(nq, nkv, d, K, gamma_far=0.9, alpha_far=0.2, clip_eps=1e9)
    x = _run(p, 0.0, 0.8, slots, q, k, v)[0, 0]
    out = _run(p, 1.0, 0.8, slots, q, k, v)[0, 0]
    # Ring and field of x are checked elsewhere; here remove them via the
    # unrolled forms and compare what is left with 0.5 * slot.
    rm = np.stack([x[max(0, t - 15):t + 1].sum(0) / 16 for t in range(n)])
    fld = np.stack([sum(0.02 * 0.98 ** (t - j) * x[j] for j in range(t + 1)) for t in range(n)])
    sem = ((out - x) / 0.3 - rm - 0.5 * fld) / 0.5
    np.testing.assert_allclose(sem, np.broadcast_to(s0.astype(np.float64), sem.shape),
                               rtol=1e-9, atol=1e-12)


# ------------------------------------------------- whole path, unrolled form

def _unrolled_reference(q, k, v, slots, p, a_l, S0=None):
    """The operator on one stream from its definition in closed, unrolled form:
    S_t = sum over evicted keys of (1-g) g^(age); F_t = sum_j (1-ge) ge^(t-j) x_j;
    ring mean = (1/16) sum of the last 16 x; pool = library attention."""
    n, nq, d = q.shape
    nkv = k.shape[1]
    K, gf, ge = p.window_k, p.gamma_far, p.ema_gamma
    near = _sdpa_window(q, k, v, window=K)
    kd = k.astype(np.float64)
    S = np.zeros((n, nkv, d))
    for t in range(n):
        for e in range(0, t - K + 1):           # keys evicted at steps K..t
            S[t] += (1 - gf) * gf ** ((t - K) - e) * kd[e]
    grp = nq // nkv
    x = near + p.alpha_far * np.repeat(S, grp, axis=1).reshape(n, nq * d)
    ring = np.stack([x[max(0, t - p.ring_size + 1):t + 1].sum(0) / p.ring_size
                     for t in range(n)])
    fld = np.stack([sum((1 - ge) * ge ** (t - j) * x[j] for j in range(t + 1))
                    for t in range(n)])
    sem = _pool_library(x, slots, p.temperature)
    u = ring + 0.5 * fld + 0.5 * sem
    return x + a_l * np.clip(u, -p.clip_eps, p.clip_eps)


@pytest.mark.parametrize("nq,nkv,d,K,gf", [(4, 2, 8, 5, 0.9), (6, 3, 4, 3, 0.98),
                                           (2, 2, 16, 1, 0.5), (4, 1, 8, 8, 0.7)])
def test_whole_path_matches_unrolled_definition(nq, nkv, d, K, gf):
    """Every channel at once, generic values, two layers (both alpha_layer
    endpoints), two sequences.  Inputs at scale 0.5 keep most u inside the
    clip so the channel values matter, while some elements saturate."""
    L, B, n = 2, 2, 37
    q, k, v, slots = _inputs(12 + nq + K, L, B, n, nq, nkv, d, scale=1.0)
    p = OracleParams(nq, nkv, d, K, gamma_far=gf, alpha_far=0.4, clip_eps=0.5)
    alpha_base, decay = 0.7, 0.9
    out = _run(p, alpha_base, decay, slots, q, k, v)
    a = [0.3 * alpha_base, alpha_base * decay]  # endpoints, layer 0 and L-1 = 1
    for l in range(L):
        for b in range(B):
            ref = _unrolled_reference(q[l, b], k[l, b], v[l, b], slots[l], p, a[l])
            np.testing.assert_allclose(out[l, b], ref, rtol=1e-9, atol=1e-11)


try:
    from hypothesis import HealthCheck, given, settings, strategies as st
except ImportError:  # pragma: no cover
    given = None

if given is not None:
    @settings(max_examples=30, deadline=None, derandomize=True,
              suppress_health_check=[HealthCheck.too_slow])
    @given(grp=st.sampled_from([(1, 1), (2, 1), (2, 2), (4, 2), (3, 1)]),
           d=st.sampled_from([2, 4, 8]), K=st.integers(1, 6), n=st.integers(1, 21),
           gf=st.floats(0.0, 0.99), af=st.floats(0.0, 1.0), ab=st.floats(0.0, 3.0),
           eps=st.floats(0.05, 2.0), seed=st.integers(0, 2**16))
    def test_whole_path_matches_unrolled_definition_on_random_shapes(grp, d, K, n, gf, af, ab,
                                                                     eps, seed):
        """The unrolled pin above, drawn over small shapes, GQA groupings,
        windows longer and shorter than the sequence, and the scalar ranges."""
        nq, nkv = grp
        f32 = lambda x: float(np.float32(x))
        gf, af, ab, eps = f32(gf), f32(af), f32(ab), f32(eps)
        q, k, v, slots = _inputs(seed, 1, 1, n, nq, nkv, d)
        p = OracleParams(nq, nkv, d, K, gamma_far=gf, alpha_far=af, clip_eps=eps)
        out = _run(p, ab, 0.9, slots, q, k, v)[0, 0]
        ref = _unrolled_reference(q[0, 0], k[0, 0], v[0, 0], slots[0], p, 0.3 * ab)
        np.testing.assert_allclose(out, ref, rtol=1e-9, atol=1e-11)


# ------------------------------------------------------------- alpha_layer

def test_alpha_layer_endpoints_and_worked_values():
    """[P3 §2.2], [P2 cross-layer decay formula]: 0.3*alpha_base at layer 0,
    alpha_base*decay^(L-1) at layer L-1, ratio 0 when L = 1."""
    for ab, dec, L in [(0.1, 0.8, 24), (1.0, 0.95, 28), (10.0, 0.98, 28), (0.04, 0.9, 2)]:
        assert oracle.alpha_layer(ab, dec, 0, L) == pytest.approx(0.3 * ab, rel=1e-15)
        assert oracle.alpha_layer(ab, dec, L - 1, L) == pytest.approx(ab * dec ** (L - 1), rel=1e-13)
    assert oracle.alpha_layer(0.1, 0.8, 0, 1) == pytest.approx(0.03, rel=1e-15)
    # worked by hand: alpha_base 1, decay 0.5, L 3, layer 1 -> (0.3 + 0.35) * 0.5
    assert oracle.alpha_layer(1.0, 0.5, 1, 3) == pytest.approx(0.325, rel=1e-15)
    # alpha_base 2, decay 0.5, L 5, layer 2 -> 2 * (0.3 + 0.35) * 0.25 = 0.325
    assert oracle.alpha_layer(2.0, 0.5, 2, 5) == pytest.approx(0.325, rel=1e-15)


def test_alpha_layer_reaches_the_output():
    """Saturated enhancement exposes alpha_layer per layer: out - x = eps*a_l."""
    nq, nkv, d, K, n, L = 2, 2, 8, 4, 3, 4
    q, k, v, slots = _inputs(13, L, 1, n, nq, nkv, d)
    v[:] = 50.0  # x == 50 everywhere (alpha_far = 0): u is far above eps
    p = OracleParams(nq, nkv, d, K, gamma_far=0.9, alpha_far=0.0, clip_eps=0.5)
    ab, dec = 2.0, 0.5
    out = _run(p, ab, dec, slots, q, k, v)
    got = (out[:, 0] - 50.0) / 0.5
    np.testing.assert_allclose(got[0], 0.3 * ab, rtol=1e-12)            # layer 0
    np.testing.assert_allclose(got[L - 1], ab * dec ** (L - 1), rtol=1e-12)  # layer L-1
    # worked by hand: layer 1 of 4 -> 2 * (0.3 + 0.7/3) * 0.5 = 0.53333...
    np.testing.assert_allclose(got[1], 0.5333333333333333, rtol=1e-12)


# ------------------------------------------------------- oracle consistency

def test_prefill_equals_token_by_token_and_chunks():
    nq, nkv, d, K, n = 4, 2, 8, 5, 29
    q, k, v, slots = _inputs(14, 2, 2, n, nq, nkv, d)
    p = OracleParams(nq, nkv, d, K, gamma_far=0.9, alpha_far=0.2)
    whole = _run(p, 0.5, 0.9, slots, q, k, v)
    st = OracleState(p, 4)
    parts = []
    for a, b in [(0, 1), (1, 7), (7, 8), (8, 29)]:
        parts.append(_run(p, 0.5, 0.9, slots, q[:, :, a:b], k[:, :, a:b], v[:, :, a:b],
                          state=st))
    np.testing.assert_array_equal(np.concatenate(parts, axis=2), whole)
    assert list(st.pos) == [n] * 4


def test_streams_are_independent():
    nq, nkv, d, K, n = 4, 2, 8, 5, 12
    q, k, v, slots = _inputs(15, 2, 3, n, nq, nkv, d)
    p = OracleParams(nq, nkv, d, K, gamma_far=0.9, alpha_far=0.2)
    base = _run(p, 0.5, 0.9, slots, q, k, v)
    perm = [2, 0, 1]
    permuted = _run(p, 0.5, 0.9, slots, q[:, perm], k[:, perm], v[:, perm])
    np.testing.assert_array_equal(permuted, base[:, perm])
    q2 = q.copy()
    q2[1] += 1.0  # change layer 1 only
    other = _run(p, 0.5, 0.9, slots, q2, k, v)
    np.testing.assert_array_equal(other[0], base[0])


def test_zero_x_gives_uniform_pool_weights():
    """Norm floor: x = 0 gives cos = 0 for every slot, so uniform weights."""
    nq, nkv, d, K, n, P = 2, 2, 8, 4, 2, 64
    q, k, _, slots = _inputs(16, 1, 1, n, nq, nkv, d)
    v = np.zeros((1, 1, n, nkv, d), np.float32)
    p = OracleParams(nq, nkv, d, K, gamma_far=0.9, alpha_far=0.0, clip_eps=1e9)
    out = _run(p, 1.0, 0.8, slots, q, k, v)[0, 0]
    sem = slots[0].astype(np.float64).mean(0)
    np.testing.assert_allclose(out, np.broadcast_to(0.3 * 0.5 * sem, out.shape), rtol=1e-12)


# ------------------------------------------------------------------ golden

def _golden_kv(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("--")[0].split("#")[0].strip()
            if "=" in line:
                a, b = line.split("=")
                vals[a.strip()] = float(b)
    return vals


def test_oracle_defaults_match_the_printed_constants():
    g = _golden_kv("sfa_config_defaults.txt")
    p = OracleParams(2, 2, 8, 16, gamma_far=0.9, alpha_far=0.1)
    assert p.ema_gamma == g["ema_gamma"]
    assert p.ring_size == g["ring_size"]
    assert p.n_slots == g["n_slots"]
    assert p.clip_eps == g["enhancement_clip"]
    assert p.temperature == g["temperature"]
    assert p.window_k == g["window_k"]
    from workloads import SfaConfigValues
    c = SfaConfigValues()
    assert (c.alpha_base, c.cross_decay, c.ema_gamma, c.ring_size, c.n_slots, c.clip_eps,
            c.temperature) == (g["alpha_base"], g["cross_decay"], g["ema_gamma"],
                               g["ring_size"], g["n_slots"], g["enhancement_clip"],
                               g["temperature"])


def test_fusion_weights_match_the_printed_formula():
    """Recover the three fusion weights from the oracle with constant channels:
    ring mean, field and sem are each set apart by a linear solve."""
    g = _golden_kv("sfa_config_defaults.txt")
    nq, nkv, d, K, P = 2, 2, 8, 4, 64
    H = nq * d
    r = _rng(17)
    v0 = (0.01 * r.standard_normal((nkv, d))).astype(np.float32)
    s0 = (0.01 * r.standard_normal(H)).astype(np.float32)
    n = 3
    q, k, v, slots = _constant_stream(n, nq, nkv, d, v0, P, s0)
    p = OracleParams(nq, nkv, d, K, gamma_far=0.9, alpha_far=0.0, clip_eps=1e9)
    out = _run(p, 1.0 / 0.3, 0.8, slots, q, k, v)[0, 0]   # layer 0: a = 1
    x = np.repeat(v0.astype(np.float64), 1, axis=0).reshape(-1)
    # columns: ring mean, field, sem at t = 0, 1, 2 for element 0..H-1
    A, y = [], []
    for t in range(n):
        for i in range(H):
            A.append([x[i] * min(t + 1, 16) / 16, x[i] * (1 - 0.98 ** (t + 1)), s0[i]])
            y.append(out[t, i] - x[i])
    wts = np.linalg.lstsq(np.array(A), np.array(y), rcond=None)[0]
    np.testing.assert_allclose(wts, [g["fuse_ring"], g["fuse_field"], g["fuse_semantic"]],
                               rtol=1e-8)


def test_alpha_calibration_presets_are_the_printed_table():
    from workloads import ALPHA_PRESETS
    rows = []
    with open(os.path.join(GOLDEN, "alpha_calibration.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append(tuple(float(t) for t in line.split()))
    assert [(a, b) for a, b, _ in rows] == list(ALPHA_PRESETS)
