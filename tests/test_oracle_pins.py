"""Pins of the fp64 oracle against facts that do not come from the oracle itself:
a hand-worked example, closed forms of special cases, invariants of the
transition, a finite-difference gradient, brute-force transition products on
d = 4, a library matrix inverse, and chunkwise == recurrent.

Citations name the page and section each fact comes from:
  * Gated DeltaNet / KDA definitions: FG2-GDN paper, section 1 "Introduction"
    (scalar alpha_t, then Diag(alpha_t) as a tied diagonal-plus-rank-1
    transition) and section 5 (unified view S_t = A_t S_{t-1} + k v^T,
    o_t = S_t^T q_t).
  * The delta rule is one SGD step on ||S^T k - v||^2: FG2-GDN section 5,
    "Delta Rule and Online Learning".
  * Chunkwise WY/UT algorithm identical in form to the recurrence: FG2-GDN
    section 3.6.
  * A state impulse is forgotten within hundreds of steps: the NVFP4 (Minima)
    abstract on the DeltaNet papers page.
  * FG2-GDN's channel-wise writing rate keeps KDA's tied transition through
    square-root-scaled keys (FG2-GDN sections 3.2, 3.4, 3.6): uniform rates give
    KDA; the update is KDA's with unit rate on the scaled keys and values, so
    KDA's chunkwise form computes it.
"""
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.txt")


def _rand_problem(rng, B=1, T=37, H=2, dk=8, dv=6, channel=False, s0=True, beta_range=(0, 1),
                  la_scale=1.0):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    beta = rng.uniform(*beta_range, size=(B, T, H))
    la_shape = (B, T, H, dk) if channel else (B, T, H)
    la = -la_scale * np.log1p(np.exp(rng.standard_normal(la_shape) + 1.0))
    S0 = rng.standard_normal((B, H, dv, dk)) * 0.3 if s0 else None
    return q, k, v, la, beta, S0


# --------------------------------------------------------------------------- #
# hand-worked example (tests/golden/hand_worked.txt)                           #
# --------------------------------------------------------------------------- #
def _golden():
    cases = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        case, field, vals = (x.strip() for x in line.split("|"))
        cases.setdefault(case, {})[field] = np.array([float(x) for x in vals.split(",")])
    return cases


@pytest.mark.parametrize("case", ["gdn", "kda"])
def test_hand_worked_example(case):
    g = _golden()[case]
    T = len(g["beta"])
    d = 2
    q = g["q"].reshape(1, T, 1, d)
    k = g["k"].reshape(1, T, 1, d)
    v = g["v"].reshape(1, T, 1, d)
    beta = g["beta"].reshape(1, T, 1)
    if case == "gdn":
        la = np.log(g["alpha"]).reshape(1, T, 1)
    else:
        la = np.log(g["alpha"]).reshape(1, T, 1, d)
    S0 = g["S0"].reshape(1, 1, d, d)
    o, sf = oracle.recurrent(q, k, v, la, beta, S0)
    np.testing.assert_allclose(o.reshape(-1), g["o"], atol=1e-13)
    np.testing.assert_allclose(sf.reshape(-1), g["S_final"], atol=1e-13)
    oc, sfc = oracle.chunkwise(q, k, v, la, beta, S0, chunk=2)
    np.testing.assert_allclose(oc.reshape(-1), g["o"], atol=1e-13)
    np.testing.assert_allclose(sfc.reshape(-1), g["S_final"], atol=1e-13)


# --------------------------------------------------------------------------- #
# closed forms of special cases                                               #
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("channel", [False, True])
def test_beta_zero_is_pure_decay(channel):
    """beta = 0: nothing is erased or written, S_t = S_0 Diag(gamma_t)."""
    rng = np.random.default_rng(1)
    q, k, v, la, beta, S0 = _rand_problem(rng, T=23, channel=channel)
    beta[:] = 0.0
    o, sf = oracle.recurrent(q, k, v, la, beta, S0)
    g = np.cumsum(la, axis=1)  # [B,T,H] or [B,T,H,dk]
    for t in range(q.shape[1]):
        for h in range(q.shape[2]):
            dec = np.exp(g[0, t, h])  # scalar or per key channel
            St = S0[0, h] * dec       # broadcasts over the key axis
            np.testing.assert_allclose(o[0, t, h], St @ q[0, t, h], rtol=1e-12, atol=1e-14)
    dec = np.exp(g[0, -1])
    exp_sf = S0[0] * (dec[:, None, None] if not channel else dec[:, None, :])
    np.testing.assert_allclose(sf[0], exp_sf, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("channel", [False, True])
def test_delta_rule_is_one_sgd_step(channel):
    """One token: S_1 = S~ - beta * grad_S (1/2)||S k - v||^2 at S~ = decayed S_0,
    with the gradient taken by central finite differences (alpha = 1 is DeltaNet)."""
    rng = np.random.default_rng(2)
    for alpha_one in (True, False):
        q, k, v, la, beta, S0 = _rand_problem(rng, T=1, H=1, dk=5, dv=4, channel=channel)
        if alpha_one:
            la[:] = 0.0
        o, sf = oracle.recurrent(q, k, v, la, beta, S0)
        kk, vv, b = k[0, 0, 0], v[0, 0, 0], beta[0, 0, 0]
        Sd = S0[0, 0] * np.exp(la[0, 0, 0])  # scalar or per key column
        loss = lambda S: 0.5 * np.sum((S @ kk - vv) ** 2)
        grad = np.zeros_like(Sd)
        eps = 1e-6
        for i in range(Sd.shape[0]):
            for j in range(Sd.shape[1]):
                E = np.zeros_like(Sd)
                E[i, j] = eps
                grad[i, j] = (loss(Sd + E) - loss(Sd - E)) / (2 * eps)
        expect = Sd - b * grad
        np.testing.assert_allclose(sf[0, 0], expect, atol=1e-8)
        np.testing.assert_allclose(o[0, 0, 0], expect @ q[0, 0, 0], atol=1e-8)


def test_retrieval_with_orthonormal_keys():
    """alpha = 1, beta = 1, orthonormal keys: after the writes S k_i = v_i exactly,
    whatever the initial state, and the read-out of key k_i returns v_i."""
    rng = np.random.default_rng(3)
    dk, dv, n = 8, 5, 6
    Q, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Q[:, :n].T.reshape(1, n, 1, dk)
    v = rng.standard_normal((1, n, 1, dv))
    q = k.copy()
    la = np.zeros((1, n, 1))
    beta = np.ones((1, n, 1))
    S0 = rng.standard_normal((1, 1, dv, dk))
    o, sf = oracle.recurrent(q, k, v, la, beta, S0)
    for i in range(n):
        np.testing.assert_allclose(sf[0, 0] @ k[0, i, 0], v[0, i, 0], atol=1e-12)
        np.testing.assert_allclose(o[0, i, 0], v[0, i, 0], atol=1e-12)


def test_householder_reflection_preserves_norm():
    """alpha = 1, beta = 2, v = 0: each step multiplies S by I - 2 k k^T (a
    reflection), so ||S||_F is preserved; with beta in (0,1) it cannot grow."""
    rng = np.random.default_rng(4)
    q, k, v, la, beta, S0 = _rand_problem(rng, T=50, H=1)
    v[:] = 0.0
    la[:] = 0.0
    beta[:] = 2.0
    _, sf = oracle.recurrent(q, k, v, la, beta, S0)
    assert abs(np.linalg.norm(sf) - np.linalg.norm(S0)) < 1e-12 * np.linalg.norm(S0)
    beta[:] = rng.uniform(0.05, 0.95, size=beta.shape)
    _, sf2 = oracle.recurrent(q, k, v, la, beta, S0)
    assert np.linalg.norm(sf2) < np.linalg.norm(S0)


def test_orthogonal_keys_reduce_to_decayed_linear_attention():
    """Mutually orthogonal keys and S_0 = 0: the erase term reads nothing, so
    o_t = sum_{s<=t} e^{g_t - g_s} beta_s (k_s . q_t) v_s (scalar-gated linear
    attention, the RetNet/Mamba-2 row of the unified view)."""
    rng = np.random.default_rng(5)
    dk, dv, T = 16, 7, 12
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm[:, :T].T.reshape(1, T, 1, dk)
    q = rng.standard_normal((1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    la = -rng.uniform(0.0, 0.7, size=(1, T, 1))
    beta = rng.uniform(0.1, 0.9, size=(1, T, 1))
    o, _ = oracle.recurrent(q, k, v, la, beta)
    g = np.cumsum(la[0, :, 0])
    for t in range(T):
        ref = sum(np.exp(g[t] - g[s]) * beta[0, s, 0] * (k[0, s, 0] @ q[0, t, 0]) * v[0, s, 0]
                  for s in range(t + 1))
        np.testing.assert_allclose(o[0, t, 0], ref, rtol=1e-11, atol=1e-13)


def test_channel_decay_with_disjoint_keys():
    """KDA with keys on distinct basis vectors and S_0 = 0: the erase reads
    nothing and each key channel decays on its own,
    o_t = sum_{s<=t} beta_s v_s q_{t,c_s} e^{g_{t,c_s} - g_{s,c_s}}."""
    rng = np.random.default_rng(6)
    dk, dv, T = 10, 3, 8
    chans = rng.permutation(dk)[:T]
    k = np.zeros((1, T, 1, dk))
    for s, c in enumerate(chans):
        k[0, s, 0, c] = 1.0
    q = rng.standard_normal((1, T, 1, dk))
    v = rng.standard_normal((1, T, 1, dv))
    la = -rng.uniform(0.0, 1.0, size=(1, T, 1, dk))
    beta = rng.uniform(0.1, 0.9, size=(1, T, 1))
    o, _ = oracle.recurrent(q, k, v, la, beta)
    g = np.cumsum(la[0, :, 0], axis=0)
    for t in range(T):
        ref = sum(beta[0, s, 0] * v[0, s, 0] * q[0, t, 0, c] * np.exp(g[t, c] - g[s, c])
                  for s, c in enumerate(chans[: t + 1]))
        np.testing.assert_allclose(o[0, t, 0], ref, rtol=1e-11, atol=1e-13)


def test_scalar_channel_decay_equals_gdn():
    """KDA with the same decay in every channel is Gated DeltaNet."""
    rng = np.random.default_rng(7)
    q, k, v, la, beta, S0 = _rand_problem(rng, B=2, T=40, H=3)
    la_c = np.repeat(la[..., None], q.shape[-1], axis=-1)
    o1, s1 = oracle.recurrent(q, k, v, la, beta, S0)
    o2, s2 = oracle.recurrent(q, k, v, la_c, beta, S0)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s1, s2, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("channel", [False, True])
def test_brute_force_transition_products(channel):
    """d = 4: the state after T tokens is the affine map
    S_T = S_0 M_1...M_T + sum_t beta_t v_t k_t^T M_{t+1}...M_T with
    M_t = Diag(alpha_t)(I - beta_t k_t k_t^T) (scalar alpha for GDN); the read-out
    uses the same expansion for each prefix."""
    rng = np.random.default_rng(8)
    d, T = 4, 9
    q, k, v, la, beta, S0 = _rand_problem(rng, T=T, H=1, dk=d, dv=d, channel=channel)
    o, sf = oracle.recurrent(q, k, v, la, beta, S0)
    I = np.eye(d)
    M = []
    for t in range(T):
        a = np.exp(la[0, t, 0])
        D = np.diag(a) if channel else a * I
        kk = k[0, t, 0][:, None]
        M.append(D @ (I - beta[0, t, 0] * kk @ kk.T))
    for t_end in range(1, T + 1):
        P = np.eye(d)
        for t in range(t_end):
            P = P @ M[t]
        S = S0[0, 0] @ P
        for t in range(t_end):
            tail = np.eye(d)
            for u in range(t + 1, t_end):
                tail = tail @ M[u]
            S = S + beta[0, t, 0] * np.outer(v[0, t, 0], k[0, t, 0]) @ tail
        np.testing.assert_allclose(o[0, t_end - 1, 0], S @ q[0, t_end - 1, 0], atol=1e-12)
    np.testing.assert_allclose(sf[0, 0], S, atol=1e-12)


# --------------------------------------------------------------------------- #
# the chunkwise form                                                          #
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("channel", [False, True])
@pytest.mark.parametrize("chunk", [1, 3, 16, 64])
def test_chunkwise_equals_recurrent(channel, chunk):
    rng = np.random.default_rng(9 + chunk)
    q, k, v, la, beta, S0 = _rand_problem(rng, B=2, T=101, H=2, dk=12, dv=10, channel=channel)
    o1, s1 = oracle.recurrent(q, k, v, la, beta, S0)
    o2, s2 = oracle.chunkwise(q, k, v, la, beta, S0, chunk=chunk)
    scale = max(np.abs(o1).max(), 1.0)
    np.testing.assert_allclose(o2, o1, atol=1e-12 * scale)
    np.testing.assert_allclose(s2, s1, atol=1e-12 * max(np.abs(s1).max(), 1.0))


@pytest.mark.parametrize("channel", [False, True])
def test_chunk_stage_ut_factor(channel):
    """T = (I + A)^{-1}: A strictly lower, T unit lower, equal to a LAPACK inverse."""
    rng = np.random.default_rng(10)
    L, dk, dv = 24, 16, 8
    q, k, v, la, beta, S0 = _rand_problem(rng, T=L, H=1, dk=dk, dv=dv, channel=channel)
    st = oracle.chunk_stage(q[0, :, 0], k[0, :, 0], v[0, :, 0], la[0, :, 0], beta[0, :, 0],
                            S0[0, 0])
    A, T = st["A"], st["T"]
    assert np.all(np.triu(A) == 0.0)
    np.testing.assert_allclose(np.diag(T), 1.0)
    assert np.all(np.triu(T, 1) == 0.0)
    np.testing.assert_allclose(T, np.linalg.inv(np.eye(L) + A), atol=1e-12)
    np.testing.assert_allclose((np.eye(L) + A) @ T, np.eye(L), atol=1e-12)
    # g is the running sum of the log decay
    la2 = la[0, :, 0] if channel else np.repeat(la[0, :, 0][:, None], dk, axis=1)
    np.testing.assert_allclose(st["G"], np.cumsum(la2, axis=0), atol=1e-13)


@pytest.mark.parametrize("channel", [False, True])
def test_chunk_stage_pseudo_values_are_the_recurrence_writes(channel):
    """Row r of V' = U - W S^T is the vector the recurrence writes at token r,
    u_r = beta_r (v_r - S_{r-1} Diag(alpha_r) k_r), recovered here from
    consecutive recurrent states as (S_r - S_{r-1} Diag(alpha_r)) k_r / |k_r|^2.
    The chunk output and end state equal the recurrence's."""
    rng = np.random.default_rng(11)
    L, dk, dv = 10, 6, 5
    q, k, v, la, beta, S0 = _rand_problem(rng, T=L, H=1, dk=dk, dv=dv, channel=channel)
    st = oracle.chunk_stage(q[0, :, 0], k[0, :, 0], v[0, :, 0], la[0, :, 0], beta[0, :, 0],
                            S0[0, 0])
    S_prev = S0[0, 0]
    o_all, _ = oracle.recurrent(q, k, v, la, beta, S0)
    for r in range(L):
        sl = slice(0, r + 1)
        _, S_r = oracle.recurrent(q[:, sl], k[:, sl], v[:, sl], la[:, sl], beta[:, sl], S0)
        S_r = S_r[0, 0]
        decayed = S_prev * np.exp(la[0, r, 0])
        kr = k[0, r, 0]
        u = (S_r - decayed) @ kr / (kr @ kr)
        np.testing.assert_allclose(st["Vp"][r], u, atol=1e-12)
        S_prev = S_r
    np.testing.assert_allclose(st["O"], o_all[0, :, 0], atol=1e-12)
    np.testing.assert_allclose(st["S_out"], S_prev, atol=1e-12)


# --------------------------------------------------------------------------- #
# state plumbing: chaining, varlen, empty sequences, forgetting               #
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("channel", [False, True])
def test_segment_chaining(channel):
    rng = np.random.default_rng(12)
    q, k, v, la, beta, S0 = _rand_problem(rng, T=90, H=2, channel=channel)
    o, sf = oracle.recurrent(q, k, v, la, beta, S0)
    a, b = slice(0, 33), slice(33, 90)
    oa, sa = oracle.chunkwise(q[:, a], k[:, a], v[:, a], la[:, a], beta[:, a], S0, chunk=16)
    ob, sb = oracle.chunkwise(q[:, b], k[:, b], v[:, b], la[:, b], beta[:, b], sa, chunk=16)
    np.testing.assert_allclose(np.concatenate([oa, ob], axis=1), o, atol=1e-12)
    np.testing.assert_allclose(sb, sf, atol=1e-12)


def test_varlen_equals_separate_runs_and_empty_sequence():
    rng = np.random.default_rng(13)
    lens = [17, 0, 64, 5, 130]
    T = sum(lens)
    q, k, v, la, beta, _ = _rand_problem(rng, T=T, H=2, dk=8, dv=8)
    S0 = rng.standard_normal((len(lens), 2, 8, 8)) * 0.2
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o, sf = oracle.recurrent(q, k, v, la, beta, S0, cu_seqlens=cu)
    oc, sfc = oracle.chunkwise(q, k, v, la, beta, S0, cu_seqlens=cu, chunk=16)
    np.testing.assert_allclose(oc, o, atol=1e-12)
    np.testing.assert_allclose(sfc, sf, atol=1e-12)
    for n, (s, e) in enumerate(zip(cu[:-1], cu[1:])):
        sl = slice(int(s), int(e))
        if e == s:
            np.testing.assert_array_equal(sf[n], S0[n])  # empty: final = initial
            continue
        on, sn = oracle.recurrent(q[:, sl], k[:, sl], v[:, sl], la[:, sl], beta[:, sl],
                                  S0[n:n + 1])
        np.testing.assert_allclose(o[:, sl], on, atol=1e-13)
        np.testing.assert_allclose(sf[n], sn[0], atol=1e-13)


def test_state_perturbation_is_forgotten():
    """The map S_0 -> S_t is affine with linear part Delta -> Delta M_1...M_t;
    with unit keys and beta in (0,1) each I - beta k k^T is a contraction, so
    ||Delta S_t||_F <= gamma_t ||Delta||_F, and an impulse is forgotten within a
    few hundred steps at the workloads' decay rates."""
    torch.manual_seed(0)
    from gated_delta_rule_140_b200.inputs import prefill_inputs
    x = prefill_inputs(1, 300, 1, 16, 16, dtype=torch.float64, seed=14)
    rng = np.random.default_rng(14)
    S0 = rng.standard_normal((1, 1, 16, 16))
    D = rng.standard_normal((1, 1, 16, 16))
    args = [x[n].numpy() for n in ("q", "k", "v", "log_alpha", "beta")]
    _, s1 = oracle.recurrent(*args, S0)
    _, s2 = oracle.recurrent(*args, S0 + D)
    gamma = np.exp(x["log_alpha"].numpy().sum())
    diff = np.linalg.norm(s2 - s1)
    assert diff <= gamma * np.linalg.norm(D) * (1 + 1e-9)
    assert diff < 1e-3 * np.linalg.norm(D)
    # linearity in the initial state: S(S0 + D) - S(S0) == S(D) - S(0)
    _, sD = oracle.recurrent(*args, D)
    _, sZ = oracle.recurrent(*args, np.zeros_like(D))
    np.testing.assert_allclose(s2 - s1, sD - sZ, atol=1e-12)


def test_threads_do_not_change_results():
    rng = np.random.default_rng(15)
    q, k, v, la, beta, S0 = _rand_problem(rng, B=3, T=50, H=4)
    o1, s1 = oracle.recurrent(q, k, v, la, beta, S0, nthreads=1)
    o2, s2 = oracle.recurrent(q, k, v, la, beta, S0, nthreads=8)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)


# --------------------------------------------------------------------------- #
# the fused entry point's input prologue (FG2-GDN section 3.5, "Gate           #
# Parameterization": L2-normalised queries and keys, beta from a sigmoid, the   #
# decay from a negative softplus)                                               #
# --------------------------------------------------------------------------- #
def _prologue_gates(a, b, bias=None, H=None):
    a = np.asarray(a, dtype=np.float64).reshape(-1, H or 1)
    b = np.asarray(b, dtype=np.float64).reshape(-1, H or 1)
    H = a.shape[1]
    z = np.ones((a.shape[0], H, 4))
    _, _, la, be = oracle.prologue(z, z, a, b, bias)
    return la, be


def test_prologue_gate_closed_forms():
    """Points where sigmoid and softplus have exact values: sigmoid(0) = 1/2,
    sigmoid(ln 3) = 3/4, softplus(0) = ln 2, softplus(ln(e^2 - 1)) = 2; the
    identities sigmoid(x) + sigmoid(-x) = 1 and softplus(x) - softplus(-x) = x;
    and the tails softplus(40) = 40 + e^-40, softplus(-40) = e^-40 (up to
    rounding), where a naive log(1 + e^x) would overflow or lose all digits."""
    x = np.array([0.0, np.log(3.0), np.log(np.e ** 2 - 1.0), 40.0, -40.0, 1.7, -0.3])
    la, be = _prologue_gates(x, x)
    la_m, be_m = _prologue_gates(-x, -x)
    sp, sig = -la[:, 0], be[:, 0]
    assert sig[0] == 0.5 and abs(sig[1] - 0.75) < 1e-15
    assert abs(sp[0] - np.log(2.0)) < 1e-15 and abs(sp[1] - np.log(4.0)) < 1e-15
    assert abs(sp[2] - 2.0) < 1e-14
    assert abs(sp[3] - 40.0) < 1e-13 and abs(sp[4] - np.exp(-40.0)) < 1e-30
    assert np.all(np.abs(sig + be_m[:, 0] - 1.0) < 1e-15)
    assert np.all(np.abs(sp - (-la_m[:, 0]) - x) < 1e-13)
    assert np.all(la < 0) and np.all((be > 0) & (be <= 1))  # sigmoid(40) rounds to 1


def test_prologue_decay_bias_per_head_and_channel():
    """The bias is added to the decay logit before the softplus, per head
    (scalar decay) or per head and key channel (channel decay): a bias equal
    to c gives exactly the unbiased result at logit + c."""
    rng = np.random.default_rng(80)
    a = rng.standard_normal((5, 3))
    bias = np.array([0.5, -1.0, 2.0])
    la_b, _ = _prologue_gates(a, a, bias, H=3)
    la_s, _ = _prologue_gates(a + bias[None, :], a, None, H=3)
    assert np.array_equal(la_b, la_s)
    z = np.ones((5, 3, 4))
    ac = rng.standard_normal((5, 3, 4))
    bc = rng.standard_normal((3, 4))
    _, _, la1, _ = oracle.prologue(z, z, ac, a, bc)
    _, _, la2, _ = oracle.prologue(z, z, ac + bc[None], a, None)
    assert np.array_equal(la1, la2)


def test_prologue_unit_norm_scale_invariance_and_direction():
    """Each (token, head) query and key vector comes out with unit norm, in the
    direction of the raw vector, unchanged by a positive scale of the raw
    vector; a zero vector stays zero; heads do not mix."""
    rng = np.random.default_rng(81)
    q = rng.standard_normal((7, 3, 16)) * rng.uniform(0.01, 100, (7, 3, 1))
    k = rng.standard_normal((7, 3, 16))
    k[2, 1] = 0.0
    a, b = np.zeros((7, 3)), np.zeros((7, 3))
    qn, kn, _, _ = oracle.prologue(q, k, a, b)
    assert np.all(np.abs(np.linalg.norm(qn, axis=-1) - 1) < 1e-14)
    nz = np.linalg.norm(k, axis=-1) > 0
    assert np.all(np.abs(np.linalg.norm(kn, axis=-1)[nz] - 1) < 1e-14)
    assert np.all(kn[2, 1] == 0)
    # collinear with the raw vector and pointing the same way
    dots = np.einsum("thd,thd->th", qn, q)
    assert np.all(dots > 0)
    assert np.max(np.abs(q - dots[..., None] * qn)) < 1e-12 * np.abs(q).max()
    qn2, _, _, _ = oracle.prologue(3.5 * q, k, a, b)
    assert np.max(np.abs(qn2 - qn)) < 1e-15
    q3 = q.copy()
    q3[:, 0] *= -7.0
    qn3, _, _, _ = oracle.prologue(q3, k, a, b)
    assert np.array_equal(qn3[:, 1:], qn[:, 1:])


# --------------------------------------------------------------------------- #
# FG2-GDN: channel-wise writing rate through square-root-scaled keys          #
# --------------------------------------------------------------------------- #
def _fg2_problem(rng, B=1, T=41, H=2, dk=8, dv=6):
    q, k, v, la, _, S0 = _rand_problem(rng, B=B, T=T, H=H, dk=dk, dv=dv, channel=True)
    bk = rng.uniform(0.05, 1.0, size=(B, T, H, dk))
    bv = rng.uniform(0.05, 1.0, size=(B, T, H, dv))
    return q, k, v, la, bk, bv, S0


def test_fg2_uniform_rates_equal_kda():
    """beta^k = beta^v = b on every channel: FG2-GDN+ is KDA with beta = b (the
    page's claim that FG2-GDN extends KDA's scalar rate to a vector)."""
    rng = np.random.default_rng(91)
    q, k, v, la, _, _, S0 = _fg2_problem(rng)
    b = rng.uniform(0.05, 1.0, size=q.shape[:3])
    bk = np.repeat(b[..., None], q.shape[-1], axis=-1)
    bv = np.repeat(b[..., None], v.shape[-1], axis=-1)
    o1, s1 = oracle.fg2_recurrent(q, k, v, la, bk, bv, S0)
    o2, s2 = oracle.recurrent(q, k, v, la, b, S0)
    assert np.allclose(o1, o2, rtol=0, atol=1e-12) and np.allclose(s1, s2, rtol=0, atol=1e-12)
    # FG2-GDN (no value gate) is FG2-GDN+ with a unit value rate, exactly
    o3, s3 = oracle.fg2_recurrent(q, k, v, la, bk)
    o4, s4 = oracle.fg2_recurrent(q, k, v, la, bk, np.ones_like(bv))
    assert np.array_equal(o3, o4) and np.array_equal(s3, s4)


def test_fg2_is_kda_on_scaled_keys_and_values_chunkwise_too():
    """The update is KDA's with unit rate on k~ = sqrt(beta^k) k, v~ = sqrt(beta^v) v
    (the page's 'identical in form'): the KDA recurrence and KDA's chunkwise WY/UT
    form (chunks of 16 over 41 tokens, packed sequences) fed the scaled keys and
    values give FG2's result."""
    rng = np.random.default_rng(92)
    q, k, v, la, bk, bv, _ = _fg2_problem(rng, T=41)
    cu = np.array([0, 7, 7, 41])
    S0 = rng.standard_normal((3, 2, 6, 8)) * 0.3
    kt, vt = np.sqrt(bk) * k, np.sqrt(bv) * v
    ones = np.ones(q.shape[:3])
    o1, s1 = oracle.fg2_recurrent(q, k, v, la, bk, bv, S0, cu)
    o2, s2 = oracle.recurrent(q, kt, vt, la, ones, S0, cu)
    o3, s3 = oracle.chunkwise(q, kt, vt, la, ones, S0, cu, chunk=16)
    for o, st in ((o2, s2), (o3, s3)):
        assert np.allclose(o1, o, rtol=0, atol=1e-11) and np.allclose(s1, st, rtol=0, atol=1e-11)


def test_fg2_erase_is_exact_along_a_unit_scaled_key():
    """No decay, one token whose scaled key k~ = sqrt(beta^k) . k has unit norm:
    the delta rule overwrites the memory along k~, S_1 k~ = v~ exactly, and leaves
    every direction orthogonal to k~ as it was."""
    rng = np.random.default_rng(93)
    dk, dv = 8, 5
    u = rng.standard_normal(dk)
    u /= np.linalg.norm(u)
    bk = rng.uniform(0.1, 1.0, size=dk)
    k = u / np.sqrt(bk)                   # so that sqrt(bk) * k = u
    v = rng.standard_normal(dv)
    bv = rng.uniform(0.1, 1.0, size=dv)
    S0 = rng.standard_normal((1, 1, dv, dk))
    q = rng.standard_normal(dk)
    sh = lambda x: x.reshape(1, 1, 1, -1)
    _, s1 = oracle.fg2_recurrent(sh(q), sh(k), sh(v), np.zeros((1, 1, 1, dk)), sh(bk), sh(bv), S0)
    S1 = s1[0, 0]
    assert np.allclose(S1 @ u, np.sqrt(bv) * v, rtol=0, atol=1e-13)
    w = rng.standard_normal(dk)
    w -= (w @ u) * u
    assert np.allclose(S1 @ w, S0[0, 0] @ w, rtol=0, atol=1e-13)
