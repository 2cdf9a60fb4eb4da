"""The chunk algebra the tensor-core kernels use, written out in fp64 numpy and
checked against the oracle's token-by-token recurrence.

The kernels do not evaluate the textbook chunkwise form directly; per 64-token
chunk they
  * clamp log2(alpha) at -115 and form G = cumulative log2 decay;
  * factorise 2^(G_i - G_j) = 2^G_i * 2^-G_j when the chunk's total decay is at
    least 2^-100, and take the exponent per element below that;
  * scale the rows of T diag(beta) and T diag(beta gamma) by E = diag(2^(G_C - G)),
    so the products come out as E U' and E W;
  * keep the state as S / sigma with a running scalar sigma, multiply the state
    product by -sigma, and fold sigma back into the state when sigma * gamma_C
    falls below 2^-40.
The prefill keeps U unscaled for its outputs, O = M U + diag(sigma gamma)
(Q (S / sigma)) (the state term formed from Q itself and scaled per row after),
and applies E and 1 / sigma_new to U for the state update only.
This test restates those steps (not the kernels' code) and shows that they
reproduce the recurrence (states and outputs) to fp64 rounding, including under
strong and zero gates, so the kernels' parity rests on an exact reformulation."""
import numpy as np
import pytest

import oracle

C = 64
LOG2_FLOOR = -115.0
FAST_FLOOR = -100.0
RENORM_BELOW = 2.0 ** -40


def chunk_algebra_state(k, v, alpha, beta, S0=None):
    n, dk = k.shape
    dv = v.shape[1]
    St = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)   # S / sigma
    sigma = 1.0
    for c0 in range(0, n, C):
        kc = np.zeros((C, dk))
        vc = np.zeros((C, dv))
        ac = np.ones(C)
        bc = np.zeros(C)
        m = min(C, n - c0)
        kc[:m], vc[:m], ac[:m], bc[:m] = k[c0:c0 + m], v[c0:c0 + m], alpha[c0:c0 + m], beta[c0:c0 + m]
        lg = np.array([max(np.log2(a), LOG2_FLOOR) if a > 0 else LOG2_FLOOR for a in ac])
        g2 = np.cumsum(lg)
        gam = np.exp2(g2)
        e = np.exp2(g2[-1] - g2)
        kk = kc @ kc.T
        if g2[-1] >= FAST_FLOOR:
            decay = (bc * gam)[:, None] * np.exp2(-g2)[None, :]
        else:
            decay = bc[:, None] * np.exp2(g2[:, None] - g2[None, :])
        A = np.tril(decay * kk, -1)
        T = np.linalg.inv(np.eye(C) + A)
        tb = e[:, None] * T * bc[None, :]              # E T diag(beta)
        tbg = tb * gam[None, :]                        # E T diag(beta gamma)
        EU = tb @ vc - sigma * (tbg @ kc) @ St         # E (U' - W S0), S0 = sigma * St
        snew = sigma * gam[-1]
        if snew < RENORM_BELOW:
            St = St * snew
            snew = 1.0
        St = St + kc.T @ (EU / snew)
        sigma = snew
    return sigma * St


def chunk_algebra_state_grouped(k, v, alpha, beta):
    """The replay kernel's grouping of the state term: P = K_c (S / sigma) is formed
    right after the previous chunk's state update, from the chunk's own keys (rows past
    the window as zeros), and E U = E T diag(beta) V + (-sigma E T diag(beta gamma)) P,
    both products into one accumulator.  From a zero state (the replay), so the first
    chunk has no P term."""
    n, dk = k.shape
    dv = v.shape[1]
    St = np.zeros((dk, dv))
    sigma = 1.0
    chunks = []
    for c0 in range(0, n, C):
        m = min(C, n - c0)
        kc = np.zeros((C, dk))
        vc = np.zeros((C, dv))
        ac = np.ones(C)
        bc = np.zeros(C)
        kc[:m], vc[:m], ac[:m], bc[:m] = k[c0:c0 + m], v[c0:c0 + m], alpha[c0:c0 + m], beta[c0:c0 + m]
        chunks.append((kc, vc, ac, bc))
    P = None
    for ci, (kc, vc, ac, bc) in enumerate(chunks):
        lg = np.array([max(np.log2(a), LOG2_FLOOR) if a > 0 else LOG2_FLOOR for a in ac])
        g2 = np.cumsum(lg)
        gam = np.exp2(g2)
        e = np.exp2(g2[-1] - g2)
        if g2[-1] >= FAST_FLOOR:
            decay = (bc * gam)[:, None] * np.exp2(-g2)[None, :]
        else:
            decay = bc[:, None] * np.exp2(g2[:, None] - g2[None, :])
        T = np.linalg.inv(np.eye(C) + np.tril(decay * (kc @ kc.T), -1))
        tb = e[:, None] * T * bc[None, :]                      # E T diag(beta), bf16 operand
        b2 = -sigma * tb * gam[None, :]                        # -sigma E T diag(beta gamma), fp32 operand
        EU = tb @ vc
        if P is not None:
            EU = EU + b2 @ P
        snew = sigma * gam[-1]
        if snew < RENORM_BELOW:
            St = St * snew
            snew = 1.0
        St = St + kc.T @ (EU / snew)
        sigma = snew
        if ci + 1 < len(chunks):
            P = chunks[ci + 1][0] @ St                         # next chunk's keys times S / sigma
    return sigma * St


def chunk_algebra_state_prescaled(k, v, alpha, beta, zero_fold_is_none=False):
    """The warp-specialised replay's form: the running sigma and the fold decision come
    from the gates alone (before any state arithmetic), and both T operands carry the
    scales, so U~ = E U / sigma' leaves the product ready for the state update:
        U~ = (E T diag(beta) / sigma') V + (-(sigma / sigma') E T diag(beta gamma)) P,
        S~ <- fold * S~ (when sigma gamma_C < 2^-40; then sigma' = 1),  S~ += K^T U~.
    zero_fold_is_none plants a mistake (a fold factor of exactly 0 read as 'no fold')."""
    n, dk = k.shape
    dv = v.shape[1]
    chunks = []
    for c0 in range(0, n, C):
        m = min(C, n - c0)
        kc = np.zeros((C, dk))
        vc = np.zeros((C, dv))
        ac = np.ones(C)
        bc = np.zeros(C)
        kc[:m], vc[:m], ac[:m], bc[:m] = k[c0:c0 + m], v[c0:c0 + m], alpha[c0:c0 + m], beta[c0:c0 + m]
        chunks.append((kc, vc, ac, bc))
    # the gate side: per chunk (sigma, sigma', fold factor or None)
    scales, sigma = [], 1.0
    for kc, vc, ac, bc in chunks:
        g2C = sum(max(np.log2(a), LOG2_FLOOR) if a > 0 else LOG2_FLOOR for a in ac)
        snew, fold = sigma * np.exp2(g2C), None
        if snew < RENORM_BELOW:
            fold, snew = snew, 1.0
        if zero_fold_is_none and fold == 0.0:
            fold = None
        scales.append((sigma, snew, fold))
        sigma = snew
    St = np.zeros((dk, dv))
    P = None
    for ci, (kc, vc, ac, bc) in enumerate(chunks):
        lg = np.array([max(np.log2(a), LOG2_FLOOR) if a > 0 else LOG2_FLOOR for a in ac])
        g2 = np.cumsum(lg)
        gam = np.exp2(g2)
        e = np.exp2(g2[-1] - g2)
        if g2[-1] >= FAST_FLOOR:
            decay = (bc * gam)[:, None] * np.exp2(-g2)[None, :]
        else:
            # only i > j is used (G is non-increasing there); the upper triangle is clamped
            decay = bc[:, None] * np.exp2(np.minimum(g2[:, None] - g2[None, :], 0.0))
        T = np.linalg.inv(np.eye(C) + np.tril(decay * (kc @ kc.T), -1))
        sg, snew, fold = scales[ci]
        tbv = T * bc[None, :]
        tb = (e / snew)[:, None] * tbv                          # bf16 operand
        tbg = (-(sg / snew) * e)[:, None] * tbv * gam[None, :]  # fp32 operand
        Ut = tb @ vc
        if P is not None:
            Ut = Ut + tbg @ P
        if fold is not None:
            St = St * fold
        St = St + kc.T @ Ut
        if ci + 1 < len(chunks):
            P = chunks[ci + 1][0] @ St
    return (scales[-1][1] if scales else 1.0) * St


def _inputs(n, dk, dv, case, seed):
    g = np.random.default_rng(seed)
    k = g.standard_normal((n, dk))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = g.standard_normal((n, dv))
    b = 1.0 / (1.0 + np.exp(-g.standard_normal(n)))
    a = g.uniform(0.9, 0.999, n)
    if case == "strong_decay":
        a = g.uniform(0.0, 0.3, n)
    elif case == "zero_gates":
        a[::29] = 0.0
        a[-1] = 0.0
    elif case == "slow_decay":
        a = g.uniform(0.999, 1.0, n)
    return k, v, a, b


@pytest.mark.parametrize("case", ["normal", "strong_decay", "zero_gates", "slow_decay"])
@pytest.mark.parametrize("n", [1, 63, 64, 200])
def test_chunk_algebra_matches_recurrence(case, n):
    dk, dv = 16, 8
    k, v, a, b = _inputs(n, dk, dv, case, seed=n)
    S_ref, _ = oracle.recurrence(k, v, a, b)
    S = chunk_algebra_state(k, v, a, b)
    scale = max(np.abs(S_ref).max(), 1e-300)
    assert np.abs(S - S_ref).max() / scale <= 1e-10


@pytest.mark.parametrize("case", ["normal", "strong_decay", "zero_gates", "slow_decay"])
@pytest.mark.parametrize("n", [1, 63, 64, 65, 200])
def test_grouped_state_term_matches_recurrence(case, n):
    dk, dv = 16, 8
    k, v, a, b = _inputs(n, dk, dv, case, seed=300 + n)
    S_ref, _ = oracle.recurrence(k, v, a, b)
    S = chunk_algebra_state_grouped(k, v, a, b)
    scale = max(np.abs(S_ref).max(), 1e-300)
    assert np.abs(S - S_ref).max() / scale <= 1e-10


@pytest.mark.parametrize("case", ["normal", "strong_decay", "zero_gates", "slow_decay"])
@pytest.mark.parametrize("n", [1, 63, 64, 65, 200])
def test_prescaled_operands_match_recurrence(case, n):
    dk, dv = 16, 8
    k, v, a, b = _inputs(n, dk, dv, case, seed=600 + n)
    S_ref, _ = oracle.recurrence(k, v, a, b)
    S = chunk_algebra_state_prescaled(k, v, a, b)
    scale = max(np.abs(S_ref).max(), 1e-300)
    assert np.abs(S - S_ref).max() / scale <= 1e-10


def test_prescaled_fold_of_zero_is_still_a_fold():
    """Planted mistake: a chunk of zero gates makes the fold factor exactly 0 (the kernel's
    fp32 arithmetic already reaches 0 for chunks whose decay is below about 2^-150);
    reading that as 'no fold' keeps the old state and fails against the recurrence."""
    dk, dv, n = 16, 8, 200
    k, v, a, b = _inputs(n, dk, dv, "normal", seed=11)
    a[64:128] = 0.0
    S_ref, _ = oracle.recurrence(k, v, a, b)
    good = chunk_algebra_state_prescaled(k, v, a, b)
    bad = chunk_algebra_state_prescaled(k, v, a, b, zero_fold_is_none=True)
    scale = np.abs(S_ref).max()
    assert np.abs(good - S_ref).max() / scale <= 1e-10
    assert np.abs(bad - S_ref).max() / scale > 1e-3


def test_grouped_state_term_needs_the_updated_state():
    """Planted mistake: P taken from the state before the previous chunk's update."""
    dk, dv, n = 16, 8, 200
    k, v, a, b = _inputs(n, dk, dv, "normal", seed=7)
    S_ref, _ = oracle.recurrence(k, v, a, b)
    # restate with the stale state: the P of chunk c + 1 from S before chunk c's update
    St = np.zeros((dk, dv))
    sigma, P, prev = 1.0, None, np.zeros((dk, dv))
    for c0 in range(0, n, C):
        m = min(C, n - c0)
        kc = np.zeros((C, dk)); vc = np.zeros((C, dv)); ac = np.ones(C); bc = np.zeros(C)
        kc[:m], vc[:m], ac[:m], bc[:m] = k[c0:c0 + m], v[c0:c0 + m], a[c0:c0 + m], b[c0:c0 + m]
        g2 = np.cumsum(np.log2(ac))
        gam = np.exp2(g2)
        e = np.exp2(g2[-1] - g2)
        T = np.linalg.inv(np.eye(C) + np.tril(bc[:, None] * np.exp2(g2[:, None] - g2[None, :]) * (kc @ kc.T), -1))
        tb = e[:, None] * T * bc[None, :]
        EU = tb @ vc + (0 if c0 == 0 else (-sigma * tb * gam[None, :]) @ (kc @ prev))
        prev = St.copy()
        snew = sigma * gam[-1]
        St = St + kc.T @ (EU / snew)
        sigma = snew
    assert np.abs(sigma * St - S_ref).max() / np.abs(S_ref).max() > 1e-3


def test_chunk_algebra_from_a_nonzero_state():
    dk, dv, n = 16, 8, 150
    k, v, a, b = _inputs(n, dk, dv, "normal", seed=5)
    S0 = np.random.default_rng(6).standard_normal((dk, dv))
    S_ref, _ = oracle.recurrence(k, v, a, b, S0=S0)
    S = chunk_algebra_state(k, v, a, b, S0=S0)
    assert np.abs(S - S_ref).max() / np.abs(S_ref).max() <= 1e-10


def test_renormalisation_is_exercised():
    """Strong decay drives sigma * gamma_C below 2^-40 in every chunk, so the fold path
    runs; the factorised path runs for ordinary gates.  Both are covered above."""
    _, _, a, _ = _inputs(64, 4, 4, "strong_decay", seed=1)
    assert np.prod(a) < RENORM_BELOW
    _, _, a, _ = _inputs(64, 4, 4, "normal", seed=1)
    assert np.sum(np.log2(a)) >= FAST_FLOOR


def chunk_algebra_prefill(q, k, v, alpha, beta, S0=None, unscaled_output_state_term=False):
    """The prefill's grouping (the P-form): P = K (S / sigma) from the state entering
    the chunk, U = T diag(beta) V + (-sigma T diag(beta gamma)) P, unscaled (the
    outputs use it); E and 1/sigma_new are applied to U only for the state update.
    Per chunk the outputs are O = M U + diag(sigma gamma) (Q (S / sigma)) with
    M_ij = (q_i . k_j) 2^(G_i - G_j), j <= i: the state term is formed from Q itself
    and its rows are scaled afterwards.  A zero entering state skips chunk 0's state
    terms (P and the outputs' state term), as the kernel does."""
    n, dk = k.shape
    dv = v.shape[1]
    St = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    sigma = 1.0
    o = np.zeros((n, dv))
    for c0 in range(0, n, C):
        qc = np.zeros((C, dk))
        kc = np.zeros((C, dk))
        vc = np.zeros((C, dv))
        ac = np.ones(C)
        bc = np.zeros(C)
        m = min(C, n - c0)
        qc[:m], kc[:m], vc[:m] = q[c0:c0 + m], k[c0:c0 + m], v[c0:c0 + m]
        ac[:m], bc[:m] = alpha[c0:c0 + m], beta[c0:c0 + m]
        lg = np.array([max(np.log2(a), LOG2_FLOOR) if a > 0 else LOG2_FLOOR for a in ac])
        g2 = np.cumsum(lg)
        gam = np.exp2(g2)
        e = np.exp2(g2[-1] - g2)
        if g2[-1] >= FAST_FLOOR:
            ratio = gam[:, None] * np.exp2(-g2)[None, :]
        else:
            ratio = np.exp2(g2[:, None] - g2[None, :])
        A = np.tril(bc[:, None] * ratio * (kc @ kc.T), -1)
        Mq = np.tril(ratio * (qc @ kc.T))
        T = np.linalg.inv(np.eye(C) + A)
        U = (T * bc[None, :]) @ vc
        O = Mq @ U
        if c0 > 0 or S0 is not None:
            P = kc @ St
            Tg = -sigma * (T * (bc * gam)[None, :])
            U = U + Tg @ P
            qs = gam if unscaled_output_state_term else sigma * gam
            O = Mq @ U + qs[:, None] * (qc @ St)
        o[c0:c0 + m] = O[:m]
        snew = sigma * gam[-1]
        if snew < RENORM_BELOW:
            St = St * snew
            snew = 1.0
        St = St + kc.T @ ((e[:, None] * U) / snew)
        sigma = snew
    return sigma * St, o


@pytest.mark.parametrize("case", ["normal", "strong_decay", "zero_gates"])
@pytest.mark.parametrize("n", [1, 64, 150])
def test_prefill_chunk_algebra_matches_recurrence(case, n):
    dk, dv = 16, 8
    k, v, a, b = _inputs(n, dk, dv, case, seed=100 + n)
    g = np.random.default_rng(200 + n)
    q = g.standard_normal((n, dk))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    S0 = g.standard_normal((dk, dv))
    for s0 in (S0, None):
        S_ref, o_ref = oracle.recurrence(k, v, a, b, q=q, S0=s0)
        S, o = chunk_algebra_prefill(q, k, v, a, b, S0=s0)
        assert np.abs(S - S_ref).max() / np.abs(S_ref).max() <= 1e-10
        assert np.abs(o - o_ref).max() / np.abs(o_ref).max() <= 1e-10


def test_prefill_output_state_term_needs_sigma():
    """Planted mistake: the outputs' state term built from gamma Q instead of sigma gamma Q
    (the bf16 copy holds S / sigma, so sigma must come with Q)."""
    dk, dv, n = 16, 8, 150
    k, v, a, b = _inputs(n, dk, dv, "normal", seed=9)
    g = np.random.default_rng(10)
    q = g.standard_normal((n, dk))
    S0 = g.standard_normal((dk, dv))
    _, o_ref = oracle.recurrence(k, v, a, b, q=q, S0=S0)
    _, good = chunk_algebra_prefill(q, k, v, a, b, S0=S0)
    _, bad = chunk_algebra_prefill(q, k, v, a, b, S0=S0, unscaled_output_state_term=True)
    scale = np.abs(o_ref).max()
    assert np.abs(good - o_ref).max() / scale <= 1e-10
    assert np.abs(bad - o_ref).max() / scale > 1e-3


def blocked_unit_lower_inverse(A):
    """(I + A)^-1 for strictly lower triangular 64 x 64 A by the kernels' block scheme:
    16 x 16 diagonal inverses D_b, then T_10 = -D_1 A_10 D_0 and T_32 = -D_3 A_32 D_2,
    X = A_21 T_11 by block rows (X_r0 = A_r0 D_0 + A_r1 T_10, X_r1 = A_r1 D_1), and
    the lower-left 32 x 32 block T_21 = -T_22 X."""
    B = 16
    blk = lambda M, r, c: M[B * r:B * (r + 1), B * c:B * (c + 1)]
    D = [np.linalg.inv(np.eye(B) + np.tril(blk(A, b, b), -1)) for b in range(4)]
    T10 = -D[1] @ blk(A, 1, 0) @ D[0]
    T32 = -D[3] @ blk(A, 3, 2) @ D[2]
    X = {}
    for r in (2, 3):
        X[r, 0] = blk(A, r, 0) @ D[0] + blk(A, r, 1) @ T10
        X[r, 1] = blk(A, r, 1) @ D[1]
    T = np.zeros_like(A)
    for b in range(4):
        T[B * b:B * (b + 1), B * b:B * (b + 1)] = D[b]
    T[B:2 * B, 0:B] = T10
    T[3 * B:4 * B, 2 * B:3 * B] = T32
    for c in (0, 1):
        T[2 * B:3 * B, B * c:B * (c + 1)] = -D[2] @ X[2, c]
        T[3 * B:4 * B, B * c:B * (c + 1)] = -(T32 @ X[2, c] + D[3] @ X[3, c])
    return T


@pytest.mark.parametrize("case", ["normal", "strong_decay"])
def test_blocked_inverse_matches_dense_inverse(case):
    g = np.random.default_rng(9)
    for _ in range(5):
        k, _, a, b = _inputs(C, 128, 1, case, seed=int(g.integers(1 << 30)))
        g2 = np.cumsum(np.maximum(np.log2(np.maximum(a, 1e-300)), LOG2_FLOOR))
        A = np.tril(b[:, None] * np.exp2(g2[:, None] - g2[None, :]) * (k @ k.T), -1)
        ref = np.linalg.inv(np.eye(C) + A)
        got = blocked_unit_lower_inverse(A)
        assert np.abs(got - ref).max() / np.abs(ref).max() <= 1e-12
