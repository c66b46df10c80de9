"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Every check here compares the oracle with something other than itself: the
worked example printed on the pages (tests/golden/running_example.json), a
special case with a textbook closed form, an invariant the pages state, or a
different algorithm of the oracle computing the same mathematical object.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import msr as omsr
from retention_inputs import gamma_schedule


def ex(golden):
    Q = np.array(golden["Q"], float)[None, :, None, :]
    K = np.array(golden["K"], float)[None, :, None, :]
    V = np.array(golden["V"], float)[None, :, None, :]
    return Q, K, V, np.array([golden["gamma"]])


# ------------------------------------------------ the page's running example

def test_recurrent_running_example_outputs(golden):
    Q, K, V, g = ex(golden)
    out, S4 = oracle.retention_recurrent(Q, K, V, g)
    np.testing.assert_allclose(out[0, :, 0, :], golden["O"], atol=1e-12)
    np.testing.assert_allclose(S4[0, 0], golden["S"][3], atol=1e-12)


def test_recurrent_running_example_states_and_norms(golden):
    Q, K, V, g = ex(golden)
    for n in range(1, 5):
        _, Sn = oracle.retention_recurrent(Q[:, :n], K[:, :n], V[:, :n], g)
        np.testing.assert_allclose(Sn[0, 0], golden["S"][n - 1], atol=1e-12)
        assert round(float(np.linalg.norm(Sn[0, 0])), 2) == pytest.approx(golden["state_norms_2dp"][n - 1])


def test_parallel_running_example(golden):
    Q, K, V, g = ex(golden)
    out = oracle.retention_parallel(Q, K, V, g)
    np.testing.assert_allclose(out[0, :, 0, :], golden["O"], atol=1e-12)
    # the page's intermediates: (Q K^T (.) D) V with its printed Q K^T (.) D
    np.testing.assert_allclose(np.array(golden["QKt_D"]) @ np.array(golden["V"]), golden["O"], atol=1e-12)
    # D from the oracle's gamma power helper
    D = np.array([[oracle.gamma_pow(0.9, n - m) if n >= m else 0.0 for m in range(4)] for n in range(4)])
    np.testing.assert_allclose(D, golden["D"], atol=1e-12)


def test_chunkwise_running_example(golden):
    Q, K, V, g = ex(golden)
    c = golden["chunk2"]
    out, R2 = oracle.retention_chunkwise(Q, K, V, g, chunk=2)
    np.testing.assert_allclose(out[0, :, 0, :], golden["O"], atol=1e-12)
    np.testing.assert_allclose(R2[0, 0], c["R_2"], atol=1e-12)
    # R_1: the state after the first chunk
    out1, R1 = oracle.retention_chunkwise(Q[:, :2], K[:, :2], V[:, :2], g, chunk=2)
    np.testing.assert_allclose(R1[0, 0], c["R_1"], atol=1e-12)
    np.testing.assert_allclose(out1[0, :, 0, :], c["inner_1"], atol=1e-12)
    # Inner_2: chunk 2 on its own (zero incoming state) is the inner term only
    inner2, _ = oracle.retention_chunkwise(Q[:, 2:], K[:, 2:], V[:, 2:], g, chunk=2)
    np.testing.assert_allclose(inner2[0, :, 0, :], c["inner_2"], atol=1e-12)
    # Cross_2 = output of chunk 2 minus Inner_2, equal to (Q_[2] R_1) (.) xi
    np.testing.assert_allclose(out[0, 2:, 0, :] - inner2[0, :, 0, :], c["cross_2"], atol=1e-12)
    np.testing.assert_allclose(np.array(c["Q2_R1"]) * np.array(c["xi"])[:, None], c["cross_2"], atol=1e-12)
    # zeta and xi from the gamma power helper, 0-based rows, B = 2
    assert [oracle.gamma_pow(0.9, 2 - 1 - j) for j in range(2)] == pytest.approx(c["zeta"], abs=1e-15)
    assert [oracle.gamma_pow(0.9, j + 1) for j in range(2)] == pytest.approx(c["xi"], abs=1e-15)


def test_linear_attention_special_case(golden):
    """gamma = 1 with phi(x) = elu(x) + 1 keys is the linear-attention state
    of the page's section 1.1 (exact integers)."""
    Q, K, V, _ = ex(golden)
    phiK = np.where(K > 0, K, np.expm1(np.minimum(K, 0))) + 1.0
    la = golden["linear_attention"]
    for n in range(1, 5):
        _, Sn = oracle.retention_recurrent(Q[:, :n], phiK[:, :n], V[:, :n], np.array([1.0]))
        np.testing.assert_array_equal(Sn[0, 0], la["S"][n - 1])
        assert round(float(np.linalg.norm(Sn[0, 0])), 2) == pytest.approx(la["norms_2dp"][n - 1])


def test_decay_table(golden):
    t = golden["decay_table"]
    for e, val in t["powers"].items():
        got = oracle.gamma_pow(t["gamma"], int(e))
        # printed to 3 significant figures (2 for 0.0052): round to match
        sig = 2 if val == 0.0052 else 3
        assert float(f"{got:.{sig - 1}e}") == pytest.approx(val, rel=1e-12)
    assert oracle.gamma_pow(0.0, 0) == 1.0 and oracle.gamma_pow(0.0, 3) == 0.0
    assert oracle.gamma_pow(1.0, 10 ** 6) == 1.0


def test_rotation_table(golden):
    """A query at n = 4 against keys at m = 1..4 with theta = pi/4: the rotated
    dot product gives cos((n-m) theta) for q = k = e_0 and sin((n-m) theta)
    for q = e_0, k = e_1."""
    t = golden["rotation_table"]
    # d = 4 and theta_base = (4/pi)^2 make the pair p = 1 turn by pi/4 per step
    base = (4.0 / math.pi) ** 2
    assert base ** (-2 * 1 / 4) == pytest.approx(t["theta"], rel=1e-15)
    N = 5
    e0 = np.zeros((1, N, 1, 4)); e0[..., 2] = 1.0
    e1 = np.zeros((1, N, 1, 4)); e1[..., 3] = 1.0
    r0 = oracle.xpos_rotate(e0, 0, base)
    r1 = oracle.xpos_rotate(e1, 0, base)
    n = t["n"]
    cos = [float(r0[0, n, 0] @ r0[0, m, 0]) for m in t["m"]]
    sin = [float(r0[0, n, 0] @ r1[0, m, 0]) for m in t["m"]]
    np.testing.assert_allclose(cos, t["cos"], atol=1e-3)
    np.testing.assert_allclose(sin, t["sin"], atol=1e-3)


def test_gamma_schedule(golden):
    t = golden["gamma_schedule"]
    np.testing.assert_array_equal(gamma_schedule(8), t["gamma"])
    win = np.log(0.01) / np.log(np.array(t["gamma"]))
    # the first four are printed from the exact formula; the rest are within 0.2%
    np.testing.assert_allclose(np.round(win[:4]), t["window"][:4], atol=1.0)
    np.testing.assert_allclose(win, t["window"], rtol=2e-3)


def test_scaled_gamma_schedule():
    """1 - gamma runs from 1/32 to 1/512 with a constant ratio between heads
    (log spacing): for 5 heads the ratio is (1/16)^(1/4) = 1/2 exactly."""
    from retention_inputs import gamma_schedule_scaled
    g = gamma_schedule_scaled(5)
    np.testing.assert_allclose(1 - g, [1 / 32, 1 / 64, 1 / 128, 1 / 256, 1 / 512], rtol=1e-13)
    g16 = gamma_schedule_scaled(16)
    r = (1 - g16[1:]) / (1 - g16[:-1])
    np.testing.assert_allclose(r, (1 / 16) ** (1 / 15), rtol=1e-12)
    assert g16[0] == pytest.approx(1 - 1 / 32) and g16[-1] == pytest.approx(1 - 1 / 512)


# --------------------------------------------- forms agree, special cases

def rand_qkv(rng, B, N, H, dk, dv):
    return (rng.standard_normal((B, N, H, dk)), rng.standard_normal((B, N, H, dk)),
            rng.standard_normal((B, N, H, dv)))


@pytest.mark.parametrize("N", [1, 2, 5, 17, 33])
def test_three_forms_agree(N):
    rng = np.random.default_rng(100 + N)
    B, H, dk, dv = 2, 3, 4, 6
    q, k, v = rand_qkv(rng, B, N, H, dk, dv)
    g = np.array([0.5, 0.9, 0.999])
    rec, S = oracle.retention_recurrent(q, k, v, g)
    par = oracle.retention_parallel(q, k, v, g)
    scale = np.abs(rec).max() + 1.0
    np.testing.assert_allclose(par, rec, atol=1e-12 * scale, rtol=0)
    for c in sorted({1, 2, 3, 4, 8, N, N + 3}):
        chk, R = oracle.retention_chunkwise(q, k, v, g, chunk=c)
        np.testing.assert_allclose(chk, rec, atol=1e-12 * scale, rtol=0)
        np.testing.assert_allclose(R, S, atol=1e-12 * (np.abs(S).max() + 1), rtol=0)


def test_gamma_zero_closed_form():
    """gamma = 0 (0^0 = 1): o_n = (q_n . k_n) v_n; gamma = 1e-30 is within
    rounding of it."""
    rng = np.random.default_rng(7)
    q, k, v = rand_qkv(rng, 1, 9, 2, 5, 3)
    expect = np.einsum("bnhd,bnhd->bnh", q, k)[..., None] * v
    for g in (0.0, 1e-30):
        gam = np.array([g, g])
        rec, S = oracle.retention_recurrent(q, k, v, gam)
        np.testing.assert_allclose(rec, expect, atol=1e-12)
        np.testing.assert_allclose(oracle.retention_parallel(q, k, v, gam), expect, atol=1e-12)
        np.testing.assert_allclose(oracle.retention_chunkwise(q, k, v, gam, 4)[0], expect, atol=1e-12)
        np.testing.assert_allclose(S[0, :, :, :], np.einsum("hd,he->hde", k[0, -1], v[0, -1]), atol=1e-12)


def test_gamma_one_is_causal_linear_attention():
    """gamma = 1: un-normalised causal linear attention, tril(Q K^T) V."""
    rng = np.random.default_rng(8)
    q, k, v = rand_qkv(rng, 1, 12, 1, 4, 5)
    expect = np.tril(q[0, :, 0] @ k[0, :, 0].T) @ v[0, :, 0]
    rec, _ = oracle.retention_recurrent(q, k, v, np.array([1.0]))
    np.testing.assert_allclose(rec[0, :, 0], expect, atol=1e-12)


def test_relative_position_invariance():
    """A common position offset on Q and K leaves retention unchanged
    (the score depends only on n - m)."""
    rng = np.random.default_rng(9)
    q, k, v = rand_qkv(rng, 1, 11, 2, 8, 3)
    g = np.array([0.9, 0.97])
    outs = []
    for off in (0, 5, 1000):
        outs.append(oracle.retention_recurrent(oracle.xpos_rotate(q, off), oracle.xpos_rotate(k, off), v, g)[0])
    np.testing.assert_allclose(outs[1], outs[0], atol=1e-9)
    np.testing.assert_allclose(outs[2], outs[0], atol=1e-9)
    # and the rotation does change the result against no rotation
    plain = oracle.retention_recurrent(q, k, v, g)[0]
    assert np.abs(plain - outs[0]).max() > 1e-3


def test_rotation_preserves_pair_norms_and_position_zero():
    rng = np.random.default_rng(10)
    x = rng.standard_normal((2, 7, 3, 8))
    y = oracle.xpos_rotate(x, 3)
    np.testing.assert_allclose(np.hypot(y[..., 0::2], y[..., 1::2]), np.hypot(x[..., 0::2], x[..., 1::2]), atol=1e-12)
    z = oracle.xpos_rotate(x, 0)
    np.testing.assert_array_equal(z[:, 0], x[:, 0])   # angle 0 at position 0
    # pair 0 turns by exactly one radian per position
    np.testing.assert_allclose(z[0, 1, 0, 0], x[0, 1, 0, 0] * math.cos(1) - x[0, 1, 0, 1] * math.sin(1), atol=1e-14)


def test_bounded_state():
    rng = np.random.default_rng(11)
    N = 400
    q, k, v = rand_qkv(rng, 1, N, 2, 3, 3)
    k = np.clip(k, -1, 1); v = np.clip(v, -1, 1)
    g = np.array([0.9, 0.99])
    c = 1.0
    for n in (1, 10, 100, 400):
        _, S = oracle.retention_recurrent(q[:, :n], k[:, :n], v[:, :n], g)
        for h in range(2):
            bound = c * (1 - g[h] ** n) / (1 - g[h])
            assert np.abs(S[0, h]).max() <= bound + 1e-12


def test_decode_continues_the_recurrence():
    """prefill then decode steps == the recurrence over the concatenation."""
    rng = np.random.default_rng(12)
    B, N, H, dk, dv, T = 2, 9, 2, 4, 5, 4
    q, k, v = rand_qkv(rng, B, N + T, H, dk, dv)
    g = np.array([0.8, 0.95])
    full, Sfull = oracle.retention_recurrent(q, k, v, g)
    _, S = oracle.retention_recurrent(q[:, :N], k[:, :N], v[:, :N], g)
    for t in range(T):
        o, S = oracle.decode_step(q[:, N + t], k[:, N + t], v[:, N + t], g, S)
        np.testing.assert_allclose(o, full[:, N + t], atol=1e-12)
    np.testing.assert_allclose(S, Sfull, atol=1e-12)
    # and init_state of the recurrent form agrees with it
    out2, S2 = oracle.retention_recurrent(q[:, N:], k[:, N:], v[:, N:], g,
                                          init_state=oracle.retention_recurrent(q[:, :N], k[:, :N], v[:, :N], g)[1])
    np.testing.assert_allclose(out2, full[:, N:], atol=1e-12)


def test_threads_do_not_change_results():
    rng = np.random.default_rng(13)
    q, k, v = rand_qkv(rng, 2, 20, 3, 4, 4)
    g = np.array([0.5, 0.9, 0.99])
    a = oracle.retention_recurrent(q, k, v, g, nthreads=1)[0]
    b = oracle.retention_recurrent(q, k, v, g, nthreads=4)[0]
    np.testing.assert_array_equal(a, b)


# ------------------------------------------------------- MSR layer pieces

def test_swish_closed_form():
    x = np.array([-30.0, -2.0, -0.5, 0.0, 0.5, 2.0, 30.0])
    s = omsr.swish(x)
    assert s[3] == 0.0
    np.testing.assert_allclose(s[-1], 30.0, rtol=1e-12)
    np.testing.assert_allclose(s[0], 0.0, atol=1e-11)
    # swish(-x) = swish(x) - x  (since sigma(-x) = 1 - sigma(x))
    np.testing.assert_allclose(omsr.swish(-x), s - x, atol=1e-12)
    np.testing.assert_allclose(omsr.swish(np.array([1.0])), [1.0 / (1.0 + math.exp(-1.0))], rtol=1e-15)


def test_group_norm_invariants():
    rng = np.random.default_rng(14)
    y = rng.standard_normal((2, 5, 3, 16)) * np.array([0.1, 1.0, 30.0])[None, None, :, None] + 2.0
    z = omsr.group_norm_heads(y, 1e-5)
    np.testing.assert_allclose(z.mean(-1), 0.0, atol=1e-12)
    var = (z ** 2).mean(-1)
    expect = (y.var(-1)) / (y.var(-1) + 1e-5)
    np.testing.assert_allclose(var, expect, rtol=1e-12)
    # scale invariance (exact when eps = 0), per head
    z0 = omsr.group_norm_heads(y, 0.0)
    z1 = omsr.group_norm_heads(y * np.array([3.0, 0.5, 7.0])[None, None, :, None], 0.0)
    np.testing.assert_allclose(z1, z0, atol=1e-12)


def test_project_brute_force():
    rng = np.random.default_rng(15)
    x = rng.standard_normal((2, 3, 4)); w = rng.standard_normal((4, 5))
    got = omsr.project(x, w)
    for a in range(2):
        for b in range(3):
            for j in range(5):
                assert got[a, b, j] == pytest.approx(sum(x[a, b, i] * w[i, j] for i in range(4)), abs=1e-12)


def _tiny_msr(rng, B=1, N=10, dm=8, H=2, dk=4, dv=6):
    x = rng.standard_normal((B, N, dm))
    W = dict(wq=rng.standard_normal((dm, H * dk)), wk=rng.standard_normal((dm, H * dk)),
             wv=rng.standard_normal((dm, H * dv)), wg=rng.standard_normal((dm, H * dv)),
             wo=rng.standard_normal((H * dv, dm)))
    return x, W, np.array([0.9, 0.99])


def test_msr_layer_invariants():
    rng = np.random.default_rng(16)
    x, W, g = _tiny_msr(rng)
    H, dv = 2, 6
    out = omsr.msr_forward(x, **W, gammas=g, H=H, k_scale=0.5, eps=0.0)
    # scaling one head's value projection does not change the output: the
    # normalisation is per head (a layer-wide norm would change it)
    W2 = dict(W); W2["wv"] = W["wv"].copy(); W2["wv"][:, :dv] *= 5.0
    np.testing.assert_allclose(omsr.msr_forward(x, **W2, gammas=g, H=H, k_scale=0.5, eps=0.0), out, atol=1e-9)
    # causality: a change at token t leaves earlier outputs unchanged
    x2 = x.copy(); x2[:, 6] += 1.0
    out2 = omsr.msr_forward(x2, **W, gammas=g, H=H, k_scale=0.5, eps=0.0)
    np.testing.assert_allclose(out2[:, :6], out[:, :6], atol=1e-12)
    assert np.abs(out2[:, 6:] - out[:, 6:]).max() > 1e-6
    # the sampled-heads form agrees with the full layer's gated heads
    _, z, y, ret = omsr.msr_forward(x, **W, gammas=g, H=H, k_scale=0.5, eps=0.0, return_parts=True)
    z1 = omsr.msr_forward(x, **W, gammas=g, H=H, k_scale=0.5, eps=0.0, heads=[1])
    np.testing.assert_allclose(z1[:, :, 0], z[:, :, 1], atol=1e-12)
    # output = Z W_O
    np.testing.assert_allclose(out, z.reshape(1, 10, H * dv) @ W["wo"], atol=1e-12)


def test_msr_layer_brute_force_tiny():
    """The MSR layer written out step by step with loops on a tiny case,
    without calling msr_forward (P1 section 9.1, section 8.4 and the summary's
    "Gated Multi-Scale Retention"): projections as explicit sums, the xPos
    rotation of each consecutive pair by n theta_p with its own cos / sin
    (P1 sections 6.6-6.8), retention through the pinned recurrent definition,
    GroupNorm per (token, head) over d_v, then swish(G) times it, then W_O."""
    rng = np.random.default_rng(17)
    B, N, dm, H, dk, dv = 1, 7, 6, 2, 4, 3
    x = rng.standard_normal((B, N, dm))
    W = dict(wq=rng.standard_normal((dm, H * dk)), wk=rng.standard_normal((dm, H * dk)),
             wv=rng.standard_normal((dm, H * dv)), wg=rng.standard_normal((dm, H * dv)),
             wo=rng.standard_normal((H * dv, dm)))
    g = np.array([0.8, 0.95])
    k_scale, eps, base = 0.5, 1e-5, 10000.0

    def proj(w, n, j):
        return sum(x[0, n, i] * w[i, j] for i in range(dm))

    def rotated(vec, n):
        out = list(vec)
        for p in range(dk // 2):
            ang = n * base ** (-2.0 * p / dk)
            c, s = math.cos(ang), math.sin(ang)
            x0, x1 = vec[2 * p], vec[2 * p + 1]
            out[2 * p], out[2 * p + 1] = x0 * c - x1 * s, x0 * s + x1 * c
        return out

    q = np.zeros((1, N, H, dk)); k = np.zeros((1, N, H, dk))
    v = np.zeros((1, N, H, dv)); gate = np.zeros((N, H, dv))
    for n in range(N):
        for h in range(H):
            q[0, n, h] = rotated([proj(W["wq"], n, h * dk + i) for i in range(dk)], n)
            k[0, n, h] = rotated([k_scale * proj(W["wk"], n, h * dk + i) for i in range(dk)], n)
            for j in range(dv):
                v[0, n, h, j] = proj(W["wv"], n, h * dv + j)
                gj = proj(W["wg"], n, h * dv + j)
                gate[n, h, j] = gj / (1.0 + math.exp(-gj))
    ret, _ = oracle.retention_recurrent(q, k, v, g)
    z = np.zeros((N, H * dv))
    for n in range(N):
        for h in range(H):
            row = ret[0, n, h]
            mu = sum(row) / dv
            var = sum((r - mu) ** 2 for r in row) / dv
            for j in range(dv):
                z[n, h * dv + j] = gate[n, h, j] * (row[j] - mu) / math.sqrt(var + eps)
    want = np.array([[sum(z[n, c] * W["wo"][c, o] for c in range(H * dv)) for o in range(dm)] for n in range(N)])
    got = omsr.msr_forward(x, **W, gammas=g, H=H, k_scale=k_scale, eps=eps, theta_base=base)
    np.testing.assert_allclose(got[0], want, rtol=1e-10, atol=1e-10)


# ---- gradients of the definition (oracle.retention_backward)

def _loss(q, k, v, dout, g, xpos, off):
    if xpos:
        q, k = oracle.xpos_rotate(q, off), oracle.xpos_rotate(k, off)
    out, _ = oracle.retention_recurrent(q, k, v, g)
    return float((out * dout).sum())


@pytest.mark.parametrize("xpos", [False, True])
def test_backward_matches_finite_differences(xpos):
    """<grad, d> equals the central difference of sum(out * dout) along a
    random direction d, for each of q, k, v (the loss is cubic in the inputs,
    so the difference is exact up to eps^2 and rounding)."""
    rng = np.random.default_rng(11 + xpos)
    B, N, H, dk, dv, off = 2, 7, 2, 6, 5, 3
    q, k = rng.standard_normal((B, N, H, dk)), rng.standard_normal((B, N, H, dk))
    v, dout = rng.standard_normal((B, N, H, dv)), rng.standard_normal((B, N, H, dv))
    g = np.array([0.9, 0.55])
    grads = oracle.retention_backward(q, k, v, dout, g, xpos=xpos, pos_offset=off)
    eps = 1e-6
    for idx, base in enumerate((q, k, v)):
        d = rng.standard_normal(base.shape)
        args_p = [q, k, v]
        args_m = [q, k, v]
        args_p[idx] = base + eps * d
        args_m[idx] = base - eps * d
        fd = (_loss(*args_p, dout, g, xpos, off) - _loss(*args_m, dout, g, xpos, off)) / (2 * eps)
        an = float((grads[idx] * d).sum())
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (idx, fd, an)


def test_backward_single_entries_match_finite_differences():
    """Entry by entry on a tiny case: every element of every gradient."""
    rng = np.random.default_rng(5)
    B, N, H, dk, dv = 1, 4, 1, 2, 3
    q, k = rng.standard_normal((B, N, H, dk)), rng.standard_normal((B, N, H, dk))
    v, dout = rng.standard_normal((B, N, H, dv)), rng.standard_normal((B, N, H, dv))
    g = np.array([0.8])
    grads = oracle.retention_backward(q, k, v, dout, g)
    eps = 1e-6
    for idx, base in enumerate((q, k, v)):
        for pos in np.ndindex(base.shape):
            d = np.zeros_like(base)
            d[pos] = 1.0
            a_p, a_m = [q, k, v], [q, k, v]
            a_p[idx], a_m[idx] = base + eps * d, base - eps * d
            fd = (_loss(*a_p, dout, g, False, 0) - _loss(*a_m, dout, g, False, 0)) / (2 * eps)
            assert abs(fd - grads[idx][pos]) <= 1e-7 * max(1.0, abs(fd)), (idx, pos)


def test_backward_gamma_zero_closed_form():
    """gamma = 0: o_n = (q_n . k_n) v_n, so dq_n = (dout_n . v_n) k_n,
    dk_n = (dout_n . v_n) q_n and dv_n = (q_n . k_n) dout_n."""
    rng = np.random.default_rng(8)
    q, k = rng.standard_normal((1, 5, 1, 3)), rng.standard_normal((1, 5, 1, 3))
    v, dout = rng.standard_normal((1, 5, 1, 4)), rng.standard_normal((1, 5, 1, 4))
    dq, dk, dv = oracle.retention_backward(q, k, v, dout, np.array([0.0]))
    gv = (dout * v).sum(-1, keepdims=True)
    qk = (q * k).sum(-1, keepdims=True)
    assert np.allclose(dq, gv * k, rtol=0, atol=1e-14)
    assert np.allclose(dk, gv * q, rtol=0, atol=1e-14)
    assert np.allclose(dv, qk * dout, rtol=0, atol=1e-14)


def test_unrotate_inverts_rotate():
    x = np.random.default_rng(9).standard_normal((2, 6, 3, 8))
    assert np.allclose(oracle.xpos_unrotate(oracle.xpos_rotate(x, 4), 4), x, rtol=0, atol=1e-14)
    assert np.allclose(oracle.xpos_rotate(oracle.xpos_unrotate(x, 4), 4), x, rtol=0, atol=1e-14)


# ------------------------------------------------ score normalizations 2 and 3

def test_normalized_hand_example():
    """Two tokens, d = 1, gamma = 0.5, worked by hand from the definitions
    (P1 section 8.5): D = [[1, 0], [0.5, 1]], row sums of D 1 and 1.5, so
    Dt = [[1, 0], [0.5, 1] / sqrt(1.5)]; Q K^T = [[2, .], [3, 6]], so
    R = [[2, 0], [1.5, 6] / sqrt(1.5)] with row sums 2 and 7.5 / sqrt(1.5);
    Rt = [[1, 0], [0.2, 0.8]] and with v = (1, 10): out = (1, 8.2)."""
    q = np.array([2.0, 3.0]).reshape(1, 2, 1, 1)
    k = np.array([1.0, 2.0]).reshape(1, 2, 1, 1)
    v = np.array([1.0, 10.0]).reshape(1, 2, 1, 1)
    out = oracle.retention_normalized(q, k, v, [0.5])
    np.testing.assert_allclose(out.ravel(), [1.0, 8.2], rtol=1e-14)
    # normalization 2 alone: row 1 is (1.5 + 60) / sqrt(1.5)
    out2 = oracle.retention_normalized(q, k, v, [0.5], flags=oracle.NORM_DECAY)
    np.testing.assert_allclose(out2.ravel(), [2.0, 61.5 / math.sqrt(1.5)], rtol=1e-14)
    # normalization 3 alone: row 1 scores (1.5, 6) over 7.5
    out3 = oracle.retention_normalized(q, k, v, [0.5], flags=oracle.NORM_SCORE)
    np.testing.assert_allclose(out3.ravel(), [1.0, 8.2], rtol=1e-14)


@pytest.mark.parametrize("gamma", [0.5, 0.9, 1 - 2.0 ** -5, 1.0])
def test_decay_normalization_closed_form(gamma):
    """Unit scores (q = k = e_1) and v = 1 make out_n the row sum of Dt, i.e.
    sum_i D_ni / sqrt(sum_i D_ni) = sqrt of the geometric series
    (1 - gamma^(n+1)) / (1 - gamma)  (n + 1 at gamma = 1)."""
    N = 40
    q = np.zeros((1, N, 1, 3))
    q[..., 0] = 1.0
    v = np.ones((1, N, 1, 2))
    out = oracle.retention_normalized(q, q, v, [gamma], flags=oracle.NORM_DECAY)
    n = np.arange(N)
    geo = n + 1.0 if gamma == 1.0 else (1 - gamma ** (n + 1)) / (1 - gamma)
    np.testing.assert_allclose(out[0, :, 0, 0] ** 2, geo, rtol=1e-12)
    np.testing.assert_allclose(out[0, :, 0, 1], out[0, :, 0, 0], rtol=0)


@pytest.mark.parametrize("flags", [oracle.NORM_SCORE, oracle.NORM_DECAY | oracle.NORM_SCORE])
def test_score_normalization_row_sums(flags):
    """With v = 1 the output is the row sum of Rt: sum_m R_nm divided by
    max(|sum_m R_nm|, 1), i.e. sign(s) where |s| >= 1 and s itself where
    |s| < 1.  s comes from the plain oracle (pinned above) with v = 1,
    times 1 / sqrt(sum_i D_ni) when normalization 2 is on."""
    rng = np.random.default_rng(31)
    B, N, H, d = 2, 37, 3, 5
    q = rng.standard_normal((B, N, H, d)) * 0.6
    k = rng.standard_normal((B, N, H, d)) * 0.6
    g = np.array([0.5, 0.9, 0.99])
    ones = np.ones((B, N, H, 1))
    s, _ = oracle.retention_recurrent(q, k, ones, g)
    s = s[..., 0]
    if flags & oracle.NORM_DECAY:
        n = np.arange(N)[None, :, None]
        s = s / np.sqrt((1 - g[None, None, :] ** (n + 1)) / (1 - g[None, None, :]))
    expect = s / np.maximum(np.abs(s), 1.0)
    out = oracle.retention_normalized(q, k, ones, g, flags=flags)[..., 0]
    np.testing.assert_allclose(out, expect, rtol=1e-12, atol=1e-14)
    # both branches of the max occur in this sample
    assert (np.abs(s) < 1).any() and (np.abs(s) > 1).any()


def test_normalizations_vanish_under_group_norm():
    """GroupNorm per head is scale-invariant (P1 section 8.4), and both
    normalizations scale each (token, head) output row by a positive scalar,
    so GroupNorm of the normalized output equals GroupNorm of the plain one
    (P1 section 8.5: they do not change the model's output)."""
    rng = np.random.default_rng(32)
    B, N, H, dk, dv = 1, 29, 2, 6, 8
    q = rng.standard_normal((B, N, H, dk))
    k = rng.standard_normal((B, N, H, dk))
    v = rng.standard_normal((B, N, H, dv))
    g = np.array([0.8, 0.97])
    plain = oracle.retention_parallel(q, k, v, g)
    for flags in (oracle.NORM_DECAY, oracle.NORM_SCORE, oracle.NORM_DECAY | oracle.NORM_SCORE):
        out = oracle.retention_normalized(q, k, v, g, flags=flags)
        np.testing.assert_allclose(omsr.group_norm_heads(out, 0.0), omsr.group_norm_heads(plain, 0.0), atol=1e-9)
        # and the scale is a per-row positive scalar, not the identity
        alpha = (out * plain).sum(-1) / (plain * plain).sum(-1)
        np.testing.assert_allclose(out, alpha[..., None] * plain, rtol=0,
                                   atol=1e-12 * np.abs(plain).max())
        assert (alpha > 0).all() and not np.allclose(alpha, 1.0)


def test_normalized_without_flags_is_the_parallel_form():
    rng = np.random.default_rng(33)
    q, k, v = (rng.standard_normal((1, 11, 2, 4)) for _ in range(3))
    g = [0.7, 0.95]
    np.testing.assert_allclose(oracle.retention_normalized(q, k, v, g, flags=0),
                               oracle.retention_parallel(q, k, v, g), rtol=1e-13, atol=1e-13)


# ------------------------------------------------ RetNet block pieces

def test_layer_norm_invariants():
    rng = np.random.default_rng(41)
    x = rng.standard_normal((3, 7, 32)) * 5.0 + 2.0
    y = omsr.layer_norm(x, eps=1e-5)
    np.testing.assert_allclose(y.mean(-1), 0.0, atol=1e-12)
    np.testing.assert_allclose((y ** 2).mean(-1), x.var(-1) / (x.var(-1) + 1e-5), rtol=1e-12)
    # invariant to a per-row shift and positive scale (eps = 0)
    np.testing.assert_allclose(omsr.layer_norm(x * 3.5 - 7.0, eps=0.0), omsr.layer_norm(x, eps=0.0), atol=1e-12)
    # gain and bias act per feature
    g, b = rng.standard_normal(32), rng.standard_normal(32)
    np.testing.assert_allclose(omsr.layer_norm(x, g, b, 1e-5), y * g + b, atol=1e-12)
    # a row of two values +-a normalises to +-1 (eps = 0)
    np.testing.assert_allclose(omsr.layer_norm(np.array([[5.0, -1.0]]), eps=0.0), [[1.0, -1.0]], atol=1e-15)


def test_gelu_values():
    """gelu(x) = x Phi(x): textbook values of the standard normal CDF,
    Phi(1) = 0.8413447460685429, Phi(2) = 0.9772498680518208, Phi(0) = 1/2,
    and the identity gelu(x) - gelu(-x) = x (Phi(x) + Phi(-x) = 1)."""
    np.testing.assert_allclose(omsr.gelu(np.array([1.0, 2.0, -1.0, 0.0])),
                               [0.8413447460685429, 2 * 0.9772498680518208, -(1 - 0.8413447460685429), 0.0],
                               rtol=1e-14, atol=1e-16)
    x = np.linspace(-6, 6, 101)
    np.testing.assert_allclose(omsr.gelu(x) - omsr.gelu(-x), x, atol=1e-14)
    from scipy.stats import norm
    np.testing.assert_allclose(omsr.gelu(x), x * norm.cdf(x), rtol=1e-13, atol=1e-15)


def _block_case(seed, B=1, N=5, dm=8, H=2, dk=2, dv=4, dff=16):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, N, dm))
    W = dict(wq=rng.standard_normal((dm, H * dk)) * 0.3, wk=rng.standard_normal((dm, H * dk)) * 0.3,
             wv=rng.standard_normal((dm, H * dv)) * 0.3, wg=rng.standard_normal((dm, H * dv)) * 0.3,
             wo=rng.standard_normal((H * dv, dm)) * 0.3, w1=rng.standard_normal((dm, dff)) * 0.3,
             w2=rng.standard_normal((dff, dm)) * 0.3)
    return x, W


def test_block_with_zero_branches_is_the_identity():
    x, W = _block_case(42)
    W["wo"][:] = 0.0
    W["w2"][:] = 0.0
    out = omsr.retnet_block(x, *(W[n] for n in ("wq", "wk", "wv", "wg", "wo", "w1", "w2")), gammas=[0.9, 0.5],
                            H=2, k_scale=0.5)
    np.testing.assert_array_equal(out, x)


def test_block_brute_force_tiny():
    """Every step of the block written out with loops on a tiny case (LayerNorm
    per token, the MSR through the oracle's pinned retention, the FFN with
    math.erf), in the pre-norm residual order of P1 section 9.2."""
    import math
    x, W = _block_case(43)
    B, N, dm = x.shape
    H, dk, dv, g = 2, 2, 4, [0.9, 0.5]
    ln1 = (np.linspace(0.5, 1.5, dm), np.linspace(-0.2, 0.3, dm))
    ln2 = (np.linspace(1.2, 0.8, dm), np.linspace(0.1, -0.1, dm))
    eps = 1e-5

    def ln(row, gb):
        mu = sum(row) / len(row)
        var = sum((r - mu) ** 2 for r in row) / len(row)
        return [(r - mu) / math.sqrt(var + eps) * gb[0][i] + gb[1][i] for i, r in enumerate(row)]

    def mm(rows, w):
        return [[sum(r[i] * w[i][j] for i in range(len(r))) for j in range(w.shape[1])] for r in rows]

    xn = np.array([[ln(list(x[0, n]), ln1) for n in range(N)]])
    msr = omsr.msr_forward(xn, *(W[n] for n in ("wq", "wk", "wv", "wg", "wo")), gammas=g, H=H, k_scale=0.5, eps=1e-5)
    y = msr + x
    yn = [ln(list(y[0, n]), ln2) for n in range(N)]
    hid = [[0.5 * v * (1 + math.erf(v / math.sqrt(2))) for v in r] for r in mm(yn, W["w1"])]
    out = np.array(mm(hid, W["w2"])) + y[0]
    got = omsr.retnet_block(x, *(W[n] for n in ("wq", "wk", "wv", "wg", "wo", "w1", "w2")), gammas=g, H=H,
                            k_scale=0.5, ln1=ln1, ln2=ln2)
    np.testing.assert_allclose(got[0], out, rtol=1e-12, atol=1e-12)
