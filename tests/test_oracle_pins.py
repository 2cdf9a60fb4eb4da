"""Pins for the fp64 oracle: closed forms, invariants and brute force that do
not reuse the oracle's own loop.  CPU only.

The recurrence is the gated delta rule replayed by Tail-Replay ("Tail-Replay:
Escaping the Curse of Linear Attention in Prefix Caching for Hybrid LLMs",
section "Mecanismos Principais", item "Reconstrucao de Estado Independente"):
    S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,  o_t = S_t^T q_t.
"""
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(seed, n, dk, dv, a_lo=0.9, a_hi=0.999, unit_keys=True):
    r = np.random.default_rng(seed)
    k = r.standard_normal((n, dk))
    if unit_keys:
        k /= np.linalg.norm(k, axis=1, keepdims=True)
    q = r.standard_normal((n, dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    v = r.standard_normal((n, dv))
    a = r.uniform(a_lo, a_hi, n)
    b = 1.0 / (1.0 + np.exp(-r.standard_normal(n)))
    return q, k, v, a, b


def load_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *nums = line.split()
            vals[key] = np.array([float(x) for x in nums])
    return vals


def test_hand_worked_example():
    g = load_golden("hand_worked_d2.txt")
    k, v, q = g["k"].reshape(3, 2), g["v"].reshape(3, 2), g["q"].reshape(3, 2)
    S, o = oracle.recurrence(k, v, g["alpha"], g["beta"], q=q)
    np.testing.assert_allclose(o, g["o"].reshape(3, 2), rtol=0, atol=1e-12)
    np.testing.assert_allclose(S, g["S"].reshape(2, 2), rtol=0, atol=1e-12)


def test_identity_transition_keeps_state():
    """alpha = 1, beta = 0: S is unchanged and o_t = S_in^T q_t."""
    q, k, v, _, _ = rnd(1, 7, 8, 5)
    S0 = np.random.default_rng(2).standard_normal((8, 5))
    S, o = oracle.recurrence(k, v, np.ones(7), np.zeros(7), q=q, S0=S0)
    np.testing.assert_array_equal(S, S0)
    np.testing.assert_allclose(o, q @ S0, rtol=0, atol=1e-13)


def test_zero_gate_resets_to_last_write():
    """alpha_t = 0 at the last token: S = beta_t k_t v_t^T whatever came before."""
    q, k, v, a, b = rnd(3, 9, 6, 4)
    a[-1] = 0.0
    S0 = np.random.default_rng(4).standard_normal((6, 4))
    S, _ = oracle.recurrence(k, v, a, b, S0=S0)
    np.testing.assert_allclose(S, b[-1] * np.outer(k[-1], v[-1]), rtol=0, atol=1e-15)


def test_orthonormal_keys_overwrite_closed_form():
    """Orthonormal keys, beta = 1, alpha = 1 from zero: S = sum_i k_i v_i^T and
    o_t = sum_{i<=t} (q_t . k_i) v_i."""
    n, dk, dv = 6, 8, 5
    Qm, _ = np.linalg.qr(np.random.default_rng(5).standard_normal((dk, dk)))
    k = Qm[:n]
    r = np.random.default_rng(6)
    v = r.standard_normal((n, dv))
    q = r.standard_normal((n, dk))
    S, o = oracle.recurrence(k, v, np.ones(n), np.ones(n), q=q)
    np.testing.assert_allclose(S, k.T @ v, rtol=0, atol=1e-13)
    o_ref = np.stack([sum((q[t] @ k[i]) * v[i] for i in range(t + 1)) for t in range(n)])
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-13)


def test_single_token_and_pure_decay():
    q, k, v, a, b = rnd(7, 1, 5, 3)
    S, _ = oracle.recurrence(k, v, a, b)
    np.testing.assert_allclose(S, b[0] * np.outer(k[0], v[0]), rtol=0, atol=1e-15)
    q, k, v, a, b = rnd(8, 11, 5, 3)
    S0 = np.random.default_rng(9).standard_normal((5, 3))
    S, _ = oracle.recurrence(k, v, a, np.zeros(11), S0=S0)
    np.testing.assert_allclose(S, np.prod(a) * S0, rtol=1e-14, atol=0)


def unrolled_product(k, v, a, b):
    """S_L = sum_j [prod_{i>j} alpha_i (I - beta_i k_i k_i^T)] beta_j k_j v_j^T with
    explicit d_k x d_k transition matrices."""
    n, dk = k.shape
    S = np.zeros((dk, v.shape[1]))
    for j in range(n):
        M = np.eye(dk)
        for i in range(j + 1, n):
            M = a[i] * (np.eye(dk) - b[i] * np.outer(k[i], k[i])) @ M
        S += M @ (b[j] * np.outer(k[j], v[j]))
    return S


@pytest.mark.parametrize("n", [1, 5, 16])
def test_unrolled_product_brute_force(n):
    q, k, v, a, b = rnd(10 + n, n, 6, 4, a_lo=0.5, a_hi=1.0)
    S, _ = oracle.recurrence(k, v, a, b)
    np.testing.assert_allclose(S, unrolled_product(k, v, a, b), rtol=0, atol=1e-12)


def chunked_bruteforce(q, k, v, a, b, C, S0):
    """Chunkwise form of the gated delta rule with an explicit matrix inverse.

    Within a chunk with start state S0 and gamma_i = prod_{m<=i} alpha_m:
      A_ij = beta_i (gamma_i / gamma_j) k_i.k_j for i > j,  T = (I + A)^-1,
      U = T (diag(beta) V - diag(beta gamma) K S0),
      S_C = gamma_C S0 + K^T diag(gamma_C / gamma) U,
      O = diag(gamma) Q S0 + (tril(Q K^T) * gamma_i / gamma_j) U.
    """
    n = k.shape[0]
    S = S0.copy()
    outs = []
    for s in range(0, n, C):
        e = min(s + C, n)
        K, V, Q = k[s:e], v[s:e], q[s:e]
        al, be = a[s:e], b[s:e]
        g = np.cumprod(al)
        c = e - s
        A = np.zeros((c, c))
        for i in range(c):
            for j in range(i):
                A[i, j] = be[i] * (g[i] / g[j]) * (K[i] @ K[j])
        T = np.linalg.inv(np.eye(c) + A)
        U = T @ (be[:, None] * V - (be * g)[:, None] * (K @ S))
        Gm = np.tril(np.outer(g, 1.0 / g))
        outs.append(g[:, None] * (Q @ S) + (np.tril(Q @ K.T) * Gm) @ U)
        S = g[-1] * S + K.T @ ((g[-1] / g)[:, None] * U)
    return S, np.concatenate(outs)


@pytest.mark.parametrize("C", [1, 3, 4, 16, 64])
def test_chunked_form_matches_recurrence(C):
    n, dk, dv = 37, 16, 12
    q, k, v, a, b = rnd(20 + C, n, dk, dv, a_lo=0.8, a_hi=1.0)
    S0 = np.random.default_rng(21).standard_normal((dk, dv)) * 0.3
    S_r, o_r = oracle.recurrence(k, v, a, b, q=q, S0=S0)
    S_c, o_c = chunked_bruteforce(q, k, v, a, b, C, S0)
    np.testing.assert_allclose(S_r, S_c, rtol=0, atol=1e-12)
    np.testing.assert_allclose(o_r, o_c, rtol=0, atol=1e-12)


def to_bits(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def packed_case(seed, H, dk, dv, cached, dtype="f32"):
    r = np.random.default_rng(seed)
    rows = int(sum(cached))
    k = r.standard_normal((rows, H, dk)).astype(np.float32)
    k /= np.linalg.norm(k, axis=2, keepdims=True)
    q = r.standard_normal((rows, H, dk)).astype(np.float32)
    v = r.standard_normal((rows, H, dv)).astype(np.float32)
    a = r.uniform(0.9, 0.999, (rows, H)).astype(np.float32)
    b = (1 / (1 + np.exp(-r.standard_normal((rows, H))))).astype(np.float32)
    if dtype == "bf16":
        q, k, v = to_bits(q), to_bits(k), to_bits(v)
    return q, k, v, a, b


def test_replay_full_length_equals_full_prefill_state():
    """R = L reproduces the state of a full prefill from zero (bit-exact)."""
    cached = [40, 70, 33]
    q, k, v, a, b = packed_case(30, 2, 8, 6, cached)
    so = np.concatenate([[0], np.cumsum(cached)]).astype(np.int32)
    ml = np.array([40, 65, 20], np.int32)
    st = oracle.replay_state(k, v, a, b, so, ml, ml)
    # the same rows [offset, offset + L) as a prefill from zero
    rows = np.concatenate([np.arange(so[i], so[i] + ml[i]) for i in range(3)])
    cu = np.concatenate([[0], np.cumsum(ml)]).astype(np.int32)
    _, st2 = oracle.prefill(q[rows], k[rows], v[rows], a[rows], b[rows], cu)
    np.testing.assert_array_equal(st, st2)


def test_replay_window_indexing():
    """Orthonormal cycling keys, alpha = beta = 1, v_t = row index: each state row
    records exactly which cached row was replayed into it."""
    H, dk, dv = 1, 64, 2
    cached = [100, 37, 300, 5]
    rows = sum(cached)
    k = np.zeros((rows, H, dk), np.float32)
    k[np.arange(rows), 0, np.arange(rows) % dk] = 1.0
    v = np.zeros((rows, H, dv), np.float32)
    v[:, 0, 0] = np.arange(rows)
    v[:, 0, 1] = 1.0
    a = np.ones((rows, H), np.float32)
    b = np.ones((rows, H), np.float32)
    so = np.concatenate([[0], np.cumsum(cached)]).astype(np.int32)
    ml = np.array([90, 37, 250, 5], np.int32)
    R = np.array([20, 64, 0, 9], np.int32)   # 64 > 37 and 9 > 5 clamp; 0 = Zero-Only
    st = oracle.replay_state(k, v, a, b, so, ml, R)
    for i in range(4):
        reff = min(R[i], ml[i])
        want = np.zeros((dk, dv))
        for t in range(so[i] + ml[i] - reff, so[i] + ml[i]):
            want[t % dk] = [t, 1.0]
        np.testing.assert_array_equal(st[i, 0], want)
        assert oracle.replay_window(so, ml, R, i) == (so[i] + ml[i] - reff, reff)


def test_invalid_windows_rejected():
    so = np.array([0, 10, 20], np.int32)
    assert oracle.replay_window(so, [11, 5], [3, 3], 0) is None      # match beyond cache
    assert oracle.replay_window(so, [5, 5], [-1, 3], 0) is None      # negative budget
    k = np.zeros((20, 1, 4), np.float32)
    with pytest.raises(ValueError):
        oracle.replay_state(k, k, np.ones((20, 1), np.float32), np.ones((20, 1), np.float32),
                            so, np.array([11, 5], np.int32), np.array([3, 3], np.int32))


def test_affine_decomposition():
    """S_full(L) = S_replay(R) + Phi S_full(L - R), Phi = the window's transitions
    applied with v = 0."""
    n, R, dk, dv = 50, 12, 8, 6
    q, k, v, a, b = rnd(40, n, dk, dv)
    S_full, _ = oracle.recurrence(k, v, a, b)
    S_head, _ = oracle.recurrence(k[: n - R], v[: n - R], a[: n - R], b[: n - R])
    S_tail, _ = oracle.recurrence(k[n - R:], v[n - R:], a[n - R:], b[n - R:])
    Phi_head, _ = oracle.recurrence(k[n - R:], np.zeros((R, dv)), a[n - R:], b[n - R:], S0=S_head)
    np.testing.assert_allclose(S_full, S_tail + Phi_head, rtol=0, atol=1e-13)


@pytest.mark.parametrize("R", [1, 4, 16, 40])
def test_replay_error_bound(R):
    """Unit keys and beta in [0, 1] make every transition a contraction, so
    ||S_full - S_replay||_F <= (prod of the window's alpha) ||S_full(L - R)||_F."""
    n, dk, dv = 60, 8, 8
    q, k, v, a, b = rnd(50 + R, n, dk, dv, a_lo=0.85, a_hi=0.99)
    S_full, _ = oracle.recurrence(k, v, a, b)
    S_head, _ = oracle.recurrence(k[: n - R], v[: n - R], a[: n - R], b[: n - R])
    S_tail, _ = oracle.recurrence(k[n - R:], v[n - R:], a[n - R:], b[n - R:])
    err = np.linalg.norm(S_full - S_tail)
    bound = np.prod(a[n - R:]) * np.linalg.norm(S_head)
    assert err <= bound * (1 + 1e-12)
    assert err > 0


def test_replay_then_suffix_equals_one_prefill():
    """Replay(R) then prefill(suffix) = one prefill from zero over tail ++ suffix (bit-exact)."""
    H, dk, dv = 3, 8, 8
    L, R, N = 80, 24, 17
    q, k, v, a, b = packed_case(60, H, dk, dv, [L + N])
    so = np.array([0, L], np.int32)
    st = oracle.replay_state(k[:L], v[:L], a[:L], b[:L], so, np.array([L], np.int32), np.array([R], np.int32))
    o_suf, st_suf = oracle.prefill(q[L:], k[L:], v[L:], a[L:], b[L:], np.array([0, N], np.int32), state_in=st)
    sl = slice(L - R, L + N)
    o_all, st_all = oracle.prefill(q[sl], k[sl], v[sl], a[sl], b[sl], np.array([0, R + N], np.int32))
    np.testing.assert_array_equal(st_suf, st_all)
    np.testing.assert_array_equal(o_suf, o_all[R:])


def test_bf16_inputs_widen_exactly():
    """bf16 bit patterns are widened exactly: same result as the fp32 values torch decodes."""
    cached = [30]
    qf, kf, vf, a, b = packed_case(70, 2, 8, 8, cached)
    kb, vb = to_bits(kf), to_bits(vf)
    kd = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).float().numpy()
    vd = torch.from_numpy(vb.view(np.int16)).view(torch.bfloat16).float().numpy()
    so = np.array([0, 30], np.int32)
    ml = np.array([30], np.int32)
    R = np.array([25], np.int32)
    np.testing.assert_array_equal(oracle.replay_state(kb, vb, a, b, so, ml, R),
                                  oracle.replay_state(kd, vd, a, b, so, ml, R))


def test_packed_prefill_matches_single_head_loop():
    """The varlen packing (row = token, then head, then feature) is read correctly."""
    cached = [9, 14]
    H, dk, dv = 3, 4, 5
    q, k, v, a, b = packed_case(80, H, dk, dv, cached)
    cu = np.array([0, 9, 23], np.int32)
    S_in = np.random.default_rng(81).standard_normal((2, H, dk, dv))
    o, st = oracle.prefill(q, k, v, a, b, cu, state_in=S_in)
    for bi in range(2):
        for h in range(H):
            rows = slice(cu[bi], cu[bi + 1])
            S, oo = oracle.recurrence(k[rows, h], v[rows, h], a[rows, h], b[rows, h], q=q[rows, h], S0=S_in[bi, h])
            np.testing.assert_array_equal(st[bi, h], S)
            np.testing.assert_array_equal(o[rows, h], oo)
