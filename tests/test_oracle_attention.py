"""Pins for the fp64 patch-attention oracle (CPU only).

Each test checks the oracle against something other than itself: hand-derived
fixtures, closed forms, pure-Python brute force, or a reduction of the schedule to
ordinary full attention.  A plausible slip in the oracle (a wrong fresh/stale index, an
off-by-one patch boundary, a transposed operand, a missing scale) fails at least one.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from patch_attention_b200 import synth
from tests._oracle_util import bits, f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(rng, *shape):
    return rng.standard_normal(shape)


# ---------------------------------------------------------------- closed forms


def test_golden_two_keys():
    g = json.load(open(os.path.join(GOLDEN, "attention_two_keys.json")))
    q = np.array(g["q"])[:, None, :]
    k = np.array(g["k"])[:, None, :]
    v = np.array(g["v"])[:, None, :]
    w = oracle.softmax_probs(q, k, g["scale"])[0, 0]
    np.testing.assert_allclose(w, g["weights"], rtol=0, atol=1e-15)
    o = oracle.attend(q, k, v, g["scale"])[:, 0, :]
    np.testing.assert_allclose(o, g["o"], rtol=0, atol=1e-14)


def test_single_key_returns_its_value():
    rng = np.random.default_rng(0)
    q, k, v = _rand(rng, 5, 3, 8), _rand(rng, 1, 3, 8), _rand(rng, 1, 3, 8)
    o = oracle.attend(q, k, v, 0.7)
    np.testing.assert_allclose(o, np.broadcast_to(v, o.shape), rtol=0, atol=1e-15)


def test_zero_query_is_mean_of_values():
    rng = np.random.default_rng(1)
    k, v = _rand(rng, 37, 2, 16), _rand(rng, 37, 2, 16)
    q = np.zeros((4, 2, 16))
    o = oracle.attend(q, k, v, 0.25)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(0), o.shape), rtol=1e-13, atol=1e-15)


def test_equal_keys_is_mean_of_values():
    rng = np.random.default_rng(2)
    k = np.broadcast_to(_rand(rng, 1, 2, 8), (19, 2, 8)).copy()
    v = _rand(rng, 19, 2, 8)
    q = _rand(rng, 3, 2, 8)
    o = oracle.attend(q, k, v, 1.3)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(0), o.shape), rtol=1e-13, atol=1e-15)


def test_unit_values_give_unit_output():
    rng = np.random.default_rng(3)
    q, k = _rand(rng, 6, 3, 8), _rand(rng, 50, 3, 8)
    o = oracle.attend(q, k, np.ones((50, 3, 8)), 0.5)
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-14)


def test_dominant_logit_selects_its_value():
    rng = np.random.default_rng(4)
    d = 4
    k = _rand(rng, 10, 1, d) * 0.1
    v = _rand(rng, 10, 1, d)
    q = np.zeros((1, 1, d))
    q[0, 0, 0] = 1.0
    k[7, 0, 0] = 40.0  # logit gap >= ~39: other weights <= 10 * e^-39
    o = oracle.attend(q, k, v, 1.0)
    np.testing.assert_allclose(o[0, 0], v[7, 0], rtol=0, atol=1e-15 + 10 * math.exp(-39) * 10)


def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(5)
    w = oracle.softmax_probs(_rand(rng, 33, 4, 16) * 3, _rand(rng, 71, 4, 16) * 3, 0.25)
    assert np.max(np.abs(w.sum(-1) - 1.0)) <= 1e-12
    assert np.all(w >= 0)


def test_scale_enters_logits():
    # doubling the scale equals doubling the query
    rng = np.random.default_rng(6)
    q, k, v = _rand(rng, 3, 2, 8), _rand(rng, 9, 2, 8), _rand(rng, 9, 2, 8)
    np.testing.assert_allclose(oracle.attend(q, k, v, 0.5), oracle.attend(2 * q, k, v, 0.25),
                               rtol=1e-13, atol=1e-14)


def test_not_transposed_heads():
    # heads are independent: zeroing head 1's keys must leave head 0 untouched
    rng = np.random.default_rng(7)
    q, k, v = _rand(rng, 3, 2, 8), _rand(rng, 9, 2, 8), _rand(rng, 9, 2, 8)
    o1 = oracle.attend(q, k, v, 0.3)
    k2 = k.copy()
    k2[:, 1] = 0
    o2 = oracle.attend(q, k2, v, 0.3)
    np.testing.assert_array_equal(o1[:, 0], o2[:, 0])
    assert not np.allclose(o1[:, 1], o2[:, 1])


def test_pure_python_brute_force():
    """Random tiny case vs explicit loops with math.exp (no numpy in the reference)."""
    rng = np.random.default_rng(8)
    n_img, M, T, H, d = 6, 3, 2, 2, 3
    plen = n_img // M
    scale = 0.6
    kprev, vprev = _rand(rng, n_img, H, d), _rand(rng, n_img, H, d)
    qn, kn, vn = _rand(rng, n_img, H, d), _rand(rng, n_img, H, d), _rand(rng, n_img, H, d)
    kt, vt = _rand(rng, T, H, d), _rand(rng, T, H, d)
    for p in range(M):
        got = oracle.patch_attention(qn, kn, vn, kprev, vprev, kt, vt, p, M, scale)
        for i in range(plen):
            row = p * plen + i
            for h in range(H):
                keys, vals = [], []
                for r in range(n_img):
                    src_k, src_v = (kn, vn) if r // plen <= p else (kprev, vprev)
                    keys.append([float(x) for x in src_k[r, h]])
                    vals.append([float(x) for x in src_v[r, h]])
                for t in range(T):
                    keys.append([float(x) for x in kt[t, h]])
                    vals.append([float(x) for x in vt[t, h]])
                logits = [scale * sum(float(qn[row, h, c]) * kk[c] for c in range(d)) for kk in keys]
                mx = max(logits)
                ws = [math.exp(z - mx) for z in logits]
                tot = sum(ws)
                for c in range(d):
                    ref = sum(w * vv[c] for w, vv in zip(ws, vals)) / tot
                    assert abs(got[i, h, c] - ref) <= 1e-13


# ---------------------------------------------------------------- schedule


def test_schedule_fixture_plain_and_stateful():
    g = json.load(open(os.path.join(GOLDEN, "schedule_case.json")))
    n_img, M = g["n_img"], g["n_patches"]
    plen = n_img // M
    steps = g["steps"]

    def arr(xs):
        return np.array(xs, dtype=np.float64).reshape(-1, 1, 1)

    K = [np.log(arr(s["k_int"])) for s in steps]
    V = [arr(s["v"]) for s in steps]
    Q = [arr(s["q"]) for s in steps]
    KT = [np.log(arr([s["ktxt_int"]])) for s in steps]
    VT = [arr([s["vtxt"]]) for s in steps]
    exp = {(e["step"], e["patch"], e["row"]): Fraction(e["o_num"], e["o_den"]) for e in g["expected"]}
    walk = oracle.KVBufferWalk(n_img, M, g["scale"])
    walk.init(K[0], V[0])
    for s in range(len(steps)):
        kp, vp = (K[s - 1], V[s - 1]) if s > 0 else (K[0], V[0])
        for p in range(M):
            plain = oracle.patch_attention(Q[s], K[s], V[s], kp, vp, KT[s], VT[s], p, M, g["scale"])
            sl = slice(p * plen, (p + 1) * plen)
            stateful = walk.step(p, Q[s][sl], K[s][sl], V[s][sl], KT[s], VT[s])
            for i in range(plen):
                want = float(exp[(s, p, i)])
                assert abs(plain[i, 0, 0] - want) <= 1e-12 * abs(want)
                assert abs(stateful[i, 0, 0] - want) <= 1e-12 * abs(want)


def _gen_steps(wl, n_steps, seed=11, a=None, b=None):
    gen = synth.AttnInputs(wl, seed=seed, a=a, b=b)
    return [{k: v[0] for k, v in gen.step_tensors(0).items()} for _ in range(n_steps)]


def _small_wl(**kw):
    base = dict(name="tiny", batch=1, heads=2, head_dim=8, grid_h=4, grid_w=6, n_patches=3,
                n_txt=5, n_layers=1, n_steps=3, ar_a=0.95, ar_b=0.3)
    base.update(kw)
    return synth.AttnWorkload(**base)


def test_single_patch_is_full_attention():
    wl = _small_wl(n_patches=1)
    steps = _gen_steps(wl, 3)
    for s in range(1, 3):
        cur, prev = steps[s], steps[s - 1]
        got = oracle.patch_attention(f64(cur["q"]), f64(cur["k"]), f64(cur["v"]), f64(prev["k"]),
                                     f64(prev["v"]), f64(cur["k_txt"]), f64(cur["v_txt"]), 0, 1,
                                     wl.softmax_scale)
        ref = oracle.attend(f64(cur["q"]), np.concatenate([f64(cur["k"]), f64(cur["k_txt"])]),
                            np.concatenate([f64(cur["v"]), f64(cur["v_txt"])]), wl.softmax_scale)
        np.testing.assert_array_equal(got, ref)


def test_stale_equal_fresh_is_full_attention():
    # a = 1, b = 0: every step repeats step 0, so stale == fresh
    wl = _small_wl()
    steps = _gen_steps(wl, 3, a=1.0, b=0.0)
    assert torch.equal(steps[0]["k"], steps[2]["k"])
    cur, prev = steps[2], steps[1]
    full = oracle.attend(f64(cur["q"]), np.concatenate([f64(cur["k"]), f64(cur["k_txt"])]),
                         np.concatenate([f64(cur["v"]), f64(cur["v_txt"])]), wl.softmax_scale)
    for p in range(wl.n_patches):
        got = oracle.patch_attention(f64(cur["q"]), f64(cur["k"]), f64(cur["v"]), f64(prev["k"]),
                                     f64(prev["v"]), f64(cur["k_txt"]), f64(cur["v_txt"]), p,
                                     wl.n_patches, wl.softmax_scale)
        np.testing.assert_array_equal(got, full[p * wl.patch_len:(p + 1) * wl.patch_len])


def test_first_step_is_full_attention():
    wl = _small_wl()
    cur = _gen_steps(wl, 1)[0]
    full = oracle.attend(f64(cur["q"]), np.concatenate([f64(cur["k"]), f64(cur["k_txt"])]),
                         np.concatenate([f64(cur["v"]), f64(cur["v_txt"])]), wl.softmax_scale)
    for p in range(wl.n_patches):
        got = oracle.patch_attention(f64(cur["q"]), f64(cur["k"]), f64(cur["v"]), f64(cur["k"]),
                                     f64(cur["v"]), f64(cur["k_txt"]), f64(cur["v_txt"]), p,
                                     wl.n_patches, wl.softmax_scale)
        np.testing.assert_array_equal(got, full[p * wl.patch_len:(p + 1) * wl.patch_len])


def test_context_uses_fresh_rows_up_to_p_and_stale_after():
    wl = _small_wl(n_patches=4, grid_h=4, grid_w=4)
    steps = _gen_steps(wl, 2)
    cur, prev = steps[1], steps[0]
    args = [f64(cur["q"]), f64(cur["k"]), f64(cur["v"]), f64(prev["k"]), f64(prev["v"]),
            f64(cur["k_txt"]), f64(cur["v_txt"])]
    plen = wl.patch_len
    for p in range(wl.n_patches):
        base = oracle.patch_attention(*args, p, wl.n_patches, wl.softmax_scale)
        for r_patch in range(wl.n_patches):
            rows = slice(r_patch * plen, (r_patch + 1) * plen)
            # perturb the stale (previous-step) rows of patch r_patch
            a2 = [x.copy() for x in args]
            a2[3][rows] += 1.0
            a2[4][rows] += 1.0
            changed = not np.array_equal(base, oracle.patch_attention(*a2, p, wl.n_patches, wl.softmax_scale))
            assert changed == (r_patch > p), (p, r_patch, "stale")
            # perturb this step's rows of patch r_patch (keys and values only)
            a3 = [x.copy() for x in args]
            a3[1][rows] += 1.0
            a3[2][rows] += 1.0
            changed = not np.array_equal(base, oracle.patch_attention(*a3, p, wl.n_patches, wl.softmax_scale))
            assert changed == (r_patch <= p), (p, r_patch, "fresh")
        # text keys always count
        a4 = [x.copy() for x in args]
        a4[5] += 1.0
        assert not np.array_equal(base, oracle.patch_attention(*a4, p, wl.n_patches, wl.softmax_scale))


def test_stateful_walk_equals_plain_definition_bitwise():
    wl = _small_wl()
    steps = _gen_steps(wl, 3)
    walk = oracle.KVBufferWalk(wl.n_img, wl.n_patches, wl.softmax_scale)
    walk.init(f64(steps[0]["k"]), f64(steps[0]["v"]))
    plen = wl.patch_len
    for s, cur in enumerate(steps):
        prev = steps[s - 1] if s else cur
        for p in range(wl.n_patches):
            sl = slice(p * plen, (p + 1) * plen)
            got = walk.step(p, f64(cur["q"])[sl], f64(cur["k"])[sl], f64(cur["v"])[sl],
                            f64(cur["k_txt"]), f64(cur["v_txt"]))
            ref = oracle.patch_attention(f64(cur["q"]), f64(cur["k"]), f64(cur["v"]), f64(prev["k"]),
                                         f64(prev["v"]), f64(cur["k_txt"]), f64(cur["v_txt"]), p,
                                         wl.n_patches, wl.softmax_scale)
            np.testing.assert_array_equal(got, ref)
            np.testing.assert_array_equal(walk.k, oracle.expected_buffer(f64(cur["k"]), f64(prev["k"]), p, wl.n_patches))
        # after the last patch of a step the buffer holds exactly that step's K/V
        np.testing.assert_array_equal(walk.k, f64(cur["k"]))
        np.testing.assert_array_equal(walk.v, f64(cur["v"]))


def test_expected_buffer_on_bit_patterns():
    wl = _small_wl()
    steps = _gen_steps(wl, 2)
    cur, prev = bits(steps[1]["k"]), bits(steps[0]["k"])
    plen = wl.patch_len
    for p in range(wl.n_patches):
        e = oracle.expected_buffer(cur, prev, p, wl.n_patches)
        np.testing.assert_array_equal(e[: (p + 1) * plen], cur[: (p + 1) * plen])
        np.testing.assert_array_equal(e[(p + 1) * plen:], prev[(p + 1) * plen:])
    np.testing.assert_array_equal(oracle.expected_buffer(cur, prev, wl.n_patches - 1, wl.n_patches), cur)


def test_walk_rejects_out_of_order():
    walk = oracle.KVBufferWalk(8, 4, 1.0)
    z = np.zeros((2, 1, 1))
    with pytest.raises(RuntimeError):
        walk.step(0, z, z, z, np.zeros((0, 1, 1)), np.zeros((0, 1, 1)))
    walk.init(np.zeros((8, 1, 1)), np.zeros((8, 1, 1)))
    with pytest.raises(RuntimeError):
        walk.step(1, z, z, z, np.zeros((0, 1, 1)), np.zeros((0, 1, 1)))


def test_key_order_does_not_matter():
    rng = np.random.default_rng(9)
    q, k, v = _rand(rng, 4, 2, 8), _rand(rng, 30, 2, 8), _rand(rng, 30, 2, 8)
    perm = rng.permutation(30)
    np.testing.assert_allclose(oracle.attend(q, k, v, 0.4), oracle.attend(q, k[perm], v[perm], 0.4),
                               rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- DistriFusion schedule


def _df_args(steps, s):
    cur, prev = steps[s], steps[s - 1]
    return [f64(cur["q"]), f64(cur["k"]), f64(cur["v"]), f64(prev["k"]), f64(prev["v"]),
            f64(cur["k_txt"]), f64(cur["v_txt"])]


def test_distrifusion_single_patch_and_stale_equal_fresh_are_full_attention():
    wl = _small_wl(n_patches=1)
    steps = _gen_steps(wl, 2)
    args = _df_args(steps, 1)
    full = oracle.attend(args[0], np.concatenate([args[1], args[5]]), np.concatenate([args[2], args[6]]),
                         wl.softmax_scale)
    np.testing.assert_array_equal(oracle.distrifusion_attention(*args, 0, 1, wl.softmax_scale), full)
    wl = _small_wl()
    steps = _gen_steps(wl, 2, a=1.0, b=0.0)
    args = _df_args(steps, 1)
    full = oracle.attend(args[0], np.concatenate([args[1], args[5]]), np.concatenate([args[2], args[6]]),
                         wl.softmax_scale)
    for p in range(wl.n_patches):
        np.testing.assert_array_equal(oracle.distrifusion_attention(*args, p, wl.n_patches, wl.softmax_scale),
                                      full[p * wl.patch_len:(p + 1) * wl.patch_len])


def test_distrifusion_sees_only_its_own_fresh_rows():
    wl = _small_wl(n_patches=4, grid_h=4, grid_w=4)
    args = _df_args(_gen_steps(wl, 2), 1)
    plen = wl.patch_len
    for p in range(wl.n_patches):
        base = oracle.distrifusion_attention(*args, p, wl.n_patches, wl.softmax_scale)
        for r in range(wl.n_patches):
            rows = slice(r * plen, (r + 1) * plen)
            a2 = [x.copy() for x in args]
            a2[1][rows] += 1.0
            a2[2][rows] += 1.0
            fresh_changed = not np.array_equal(base, oracle.distrifusion_attention(*a2, p, wl.n_patches, wl.softmax_scale))
            a3 = [x.copy() for x in args]
            a3[3][rows] += 1.0
            a3[4][rows] += 1.0
            stale_changed = not np.array_equal(base, oracle.distrifusion_attention(*a3, p, wl.n_patches, wl.softmax_scale))
            assert fresh_changed == (r == p) and stale_changed == (r != p), (p, r)


def test_distrifusion_matches_pipefusion_on_last_patch_only_at_first_patch():
    # patch 0: both schedules see stale rows for every other patch -> identical
    wl = _small_wl()
    args = _df_args(_gen_steps(wl, 2), 1)
    np.testing.assert_array_equal(oracle.distrifusion_attention(*args, 0, wl.n_patches, wl.softmax_scale),
                                  oracle.patch_attention(*args, 0, wl.n_patches, wl.softmax_scale))


def test_pipefusion_stays_closer_to_fresh_attention_than_distrifusion():
    """The pages' quality claim ("기술 요약: PipeFusion", 주요 기여 / 품질 보존: PipeFusion uses
    fresh activations over a wider area than DistriFusion), on AR(1) synthetic activations:
    the error against all-fresh attention, over a whole step, is smaller for PipeFusion."""
    wl = _small_wl(n_patches=4, grid_h=8, grid_w=8, n_txt=4, heads=2, head_dim=16)
    steps = _gen_steps(wl, 3)
    for s in (1, 2):
        args = _df_args(steps, s)
        fresh = oracle.attend(args[0], np.concatenate([args[1], args[5]]), np.concatenate([args[2], args[6]]),
                              wl.softmax_scale)
        e_pf = e_df = 0.0
        for p in range(wl.n_patches):
            sl = slice(p * wl.patch_len, (p + 1) * wl.patch_len)
            e_pf += np.sum((oracle.patch_attention(*args, p, wl.n_patches, wl.softmax_scale) - fresh[sl]) ** 2)
            e_df += np.sum((oracle.distrifusion_attention(*args, p, wl.n_patches, wl.softmax_scale) - fresh[sl]) ** 2)
        assert e_pf < e_df, (s, e_pf, e_df)
