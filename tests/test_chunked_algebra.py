"""The chunked (WY / UT) prefill's algebra, the form the tensor-core kernels evaluate,
written out in fp64 with numpy and checked against the oracle's token-serial scan.

Per chunk of C tokens with S0 the state at the chunk start, gamma_t the product of the
chunk's gates a up to t, b_t the write strength (beta for the delta rules):
  L = strictly-lower(b_t gamma_t / gamma_s k_t . k_s)  (zero for the linear / gated rules)
  T = (I + L)^-1,  W = T diag(b gamma) K,  U~ = T diag(b) V,  U = U~ - W S0
  O = scale (diag(gamma) Q S0 + (Q K^T . M) U),  M_ts = gamma_t / gamma_s for s <= t
  S = gamma_C S0 + K^T diag(gamma_C / gamma) U
This is the "Kimi Linear" section's chunkwise-parallel evaluation and the "Gated
DeltaNet-2" section's chunkwise WY algorithm ("Seven Architectures Replacing KV Cache With
Bounded Mutable State") for the recurrence u = b (v - c S^T k), S <- a S + k u^T with
c = a (prediction from the decayed state).  The two are the same result up to rounding,
so a dropped term, a transposed operand or a gate ratio taken the wrong way round fails
at 1e-9.  The 32 x 32 block form of T used by the prep launch is checked as well."""
import numpy as np
import pytest

from oracle import oracle

RULE_ABC = {
    "linear": lambda g, b: (np.ones_like(g), np.ones_like(b), False),
    "gated": lambda g, b: (g, np.ones_like(b), False),
    "delta": lambda g, b: (np.ones_like(g), b, True),
    "gated_delta": lambda g, b: (g, b, True),
}


def chunked_head(rule, S0, Q, K, V, G, B, scale, C):
    """One (sequence, head) by chunks; returns (final state, outputs)."""
    T_len = Q.shape[0]
    S = S0.copy()
    O = np.zeros((T_len, V.shape[1]))
    for c0 in range(0, T_len, C):
        q, k, v = Q[c0:c0 + C], K[c0:c0 + C], V[c0:c0 + C]
        a, b, delta = RULE_ABC[rule](G[c0:c0 + C], B[c0:c0 + C])
        n = q.shape[0]
        gam = np.cumprod(a)
        ratio = np.tril(gam[:, None] / gam[None, :])          # gamma_t / gamma_s, s <= t
        if delta:
            L = np.tril(b[:, None] * ratio * (k @ k.T), -1)
            Tm = np.linalg.inv(np.eye(n) + L)
        else:
            Tm = np.eye(n)
        W = Tm @ ((b * gam)[:, None] * k)
        U = Tm @ (b[:, None] * v) - (W @ S if delta else 0.0)
        O[c0:c0 + n] = scale * (gam[:, None] * (q @ S) + ((q @ k.T) * ratio) @ U)
        S = gam[-1] * S + k.T @ ((gam[-1] / gam)[:, None] * U)
    return S, O


@pytest.mark.parametrize("rule", list(RULE_ABC))
@pytest.mark.parametrize("C", [16, 64])
def test_chunked_algebra_matches_the_recurrence(rule, C):
    rng = np.random.default_rng(7)
    lens = [130, 64, 1, 0, 77]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    Tt, H, dk, dv = int(cu[-1]), 2, 16, 12
    q = rng.standard_normal((Tt, H, dk))
    k = rng.standard_normal((Tt, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((Tt, H, dv))
    g = rng.uniform(-1.0, 1.0, (Tt, H))          # either sign ("Complex KDA" ranges)
    beta = rng.uniform(0.0, 2.0, (Tt, H))
    S0 = rng.standard_normal((len(lens), H, dk, dv)) * 0.3
    S_ref, o_ref, err = oracle.scan(rule, H, cu, q, k, v, g, beta, 0.7, src_pool=S0,
                                    read_slot=np.arange(len(lens), dtype=np.int32))
    assert err == 0
    for s in range(len(lens)):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        for h in range(H):
            S, O = chunked_head(rule, S0[s, h], q[t0:t1, h], k[t0:t1, h], v[t0:t1, h], g[t0:t1, h],
                                beta[t0:t1, h], 0.7, C)
            sc = max(1.0, np.abs(S_ref[s, h]).max())
            assert np.abs(S - S_ref[s, h]).max() <= 1e-9 * sc, (rule, s, h)
            if t1 > t0:
                assert np.abs(O - o_ref[t0:t1, h]).max() <= 1e-9 * max(1.0, np.abs(o_ref[t0:t1, h]).max())


def test_block_inverse_form():
    """T = (I + L)^-1 by 32 x 32 blocks, as the prep launch forms it: the diagonal blocks by
    forward substitution and the off-diagonal block as -D (L10 A)."""
    rng = np.random.default_rng(3)
    L = np.tril(rng.standard_normal((64, 64)) * 0.4, -1)

    def subst(Lb):
        n = Lb.shape[0]
        X = np.zeros((n, n))
        for c in range(n):
            x = np.zeros(n)
            x[c] = 1.0
            for r in range(1, n):
                x[r] -= Lb[r, :r] @ x[:r]
            X[:, c] = x
        return X
    A, D = subst(L[:32, :32]), subst(L[32:, 32:])
    Tb = np.block([[A, np.zeros((32, 32))], [-D @ (L[32:, :32] @ A), D]])
    assert np.abs(Tb - np.linalg.inv(np.eye(64) + L)).max() < 1e-10


# ---- the channel-wise gate (rule kda) ---------------------------------------------------
# With alpha_t in R^{d_k} ("Kimi Linear": S_t = (I - beta k k^T) Diag(alpha_t) S_{t-1} +
# beta k v^T, prediction from the decayed state) the chunk's decay products Gamma_t =
# prod_{s <= t} alpha_s are vectors, and the ratios Gamma_t / Gamma_s sit inside the sums
# over d_k, so they are absorbed into the operands:
#   K+ = K (.) Gamma,  Q+ = Q (.) Gamma,  K^ = K (.) Gamma_C / Gamma
#   L_ts = beta_t sum_i k_ti k_si Gamma_ti / Gamma_si (s < t),  P_ts = the same with q_t (s <= t)
#   T = (I + L)^-1,  Tw = T diag(beta),  W = Tw K+,  U = Tw V - W S0
#   O = scale (Q+ S0 + P U),  S = Diag(Gamma_C) S0 + K^^T U
# The ratio products are factored per 16-token block b of the row token t around a
# reference m_b (the mean of the log-magnitudes at the block's two ends):
#   Gamma_ti / Gamma_si = [sigma_ti e^{l_ti - m_bi}] e^{m_bi - m_ji} [sigma_si e^{m_ji - l_si}]
# (j the block of s), so every factor stays within e^{+-64} once each token's log-magnitude
# is held to [-8, 8]: magnitudes below e^-8 (zero included) act as e^-8.

KDA_CLAMP = 8.0


def kda_chunk_operands(alpha, C=64, blk=16):
    """The per-chunk factors of the factored form for one chunk of n <= C tokens (rows
    beyond n take alpha = 1): E_t = sigma_t e^{l_t - m_b}, R_t = sigma_t e^{m_b - l_t},
    F[b, j] = e^{m_b - m_j}, Gamma_t, Gamma_C and Gamma_C / Gamma_t."""
    n, dk = alpha.shape
    a = np.ones((C, dk))
    a[:n] = alpha
    lg = np.clip(np.log(np.maximum(np.abs(a), 1e-300)), -KDA_CLAMP, KDA_CLAMP)
    sg = np.where(a < 0, -1.0, 1.0)
    lam = np.cumsum(lg, axis=0)
    sig = np.cumprod(sg, axis=0)
    nb = C // blk
    ends = np.vstack([np.zeros((1, dk)), lam[blk - 1::blk]])       # l before each block, then each block's end
    m = 0.5 * (ends[:-1] + ends[1:])                                 # [nb, dk]
    mb = np.repeat(m, blk, axis=0)                                   # m of each token's block
    E = sig * np.exp(lam - mb)
    R = sig * np.exp(mb - lam)
    F = np.exp(m[:, None, :] - m[None, :, :])                        # F[b, j]
    gam = E * np.exp(mb)                                             # Gamma_t
    gam_c = sig[-1] * np.exp(lam[-1])                                # Gamma_C
    kh = R * (sig[-1] * np.exp(lam[-1] - mb))                        # Gamma_C / Gamma_t
    return E, R, F, gam, gam_c, kh


def chunked_head_kda(S0, Q, K, V, A, Bt, scale, C=64, blk=16):
    T_len = Q.shape[0]
    S = S0.copy()
    O = np.zeros((T_len, V.shape[1]))
    for c0 in range(0, T_len, C):
        n = min(C, T_len - c0)
        q = np.zeros((C, Q.shape[1]))
        k = np.zeros((C, K.shape[1]))
        v = np.zeros((C, V.shape[1]))
        b = np.zeros(C)
        q[:n], k[:n], v[:n], b[:n] = Q[c0:c0 + n], K[c0:c0 + n], V[c0:c0 + n], Bt[c0:c0 + n]
        E, R, F, gam, gam_c, kh = kda_chunk_operands(A[c0:c0 + n], C, blk)
        aq, ak, bm = q * E, k * E, k * R
        blkof = np.arange(C) // blk
        GQ = np.zeros((C, C))
        GK = np.zeros((C, C))
        for t in range(C):
            for s in range(t + 1):
                f = F[blkof[t], blkof[s]]
                GQ[t, s] = np.sum(aq[t] * bm[s] * f)
                GK[t, s] = np.sum(ak[t] * bm[s] * f)
        P = np.tril(GQ)
        L = b[:, None] * np.tril(GK, -1)
        Tw = np.linalg.inv(np.eye(C) + L) * b[None, :]
        W = Tw @ (k * gam)
        U = Tw @ v - W @ S
        O[c0:c0 + n] = (scale * ((q * gam) @ S + P @ U))[:n]
        S = gam_c[:, None] * S + (k * kh).T @ U
    return S, O


def _kda_case(seed, alpha_fn, lens=(130, 64, 1, 0, 77), H=2, dk=16, dv=12):
    rng = np.random.default_rng(seed)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    Tt = int(cu[-1])
    q = rng.standard_normal((Tt, H, dk))
    k = rng.standard_normal((Tt, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((Tt, H, dv))
    alpha = alpha_fn(rng, (Tt, H, dk))
    beta = rng.uniform(0.0, 2.0, (Tt, H))
    S0 = rng.standard_normal((len(lens), H, dk, dv)) * 0.3
    return cu, q, k, v, alpha, beta, S0


def _check_kda(cu, q, k, v, alpha, beta, S0, alpha_ref, tol):
    H = q.shape[1]
    n_seqs = len(cu) - 1
    S_ref, o_ref, err = oracle.scan("kda", H, cu, q, k, v, alpha_ref, beta, 0.7, src_pool=S0,
                                    read_slot=np.arange(n_seqs, dtype=np.int32))
    assert err == 0
    for s in range(n_seqs):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        for h in range(H):
            S, O = chunked_head_kda(S0[s, h], q[t0:t1, h], k[t0:t1, h], v[t0:t1, h], alpha[t0:t1, h],
                                    beta[t0:t1, h], 0.7)
            sc = max(1.0, np.abs(S_ref[s, h]).max())
            assert np.abs(S - S_ref[s, h]).max() <= tol * sc, (s, h)
            if t1 > t0:
                assert np.abs(O - o_ref[t0:t1, h]).max() <= tol * max(1.0, np.abs(o_ref[t0:t1, h]).max())


def test_kda_chunked_algebra_matches_the_recurrence():
    """Decays of either sign with magnitudes in [e^-6, 1] (no clamping), beta in [0, 2]: the
    factored chunk form equals the token recurrence to rounding."""
    def alpha_fn(rng, shape):
        return rng.choice([-1.0, 1.0], shape) * np.exp(-rng.uniform(0.0, 6.0, shape))
    case = _kda_case(11, alpha_fn)
    _check_kda(*case, alpha_ref=case[4], tol=1e-9)


def test_kda_chunked_algebra_steep_decays():
    """Every channel decaying by up to e^-8 per token (spans of 512 over a chunk): the
    factors stay finite and the result is still the recurrence's."""
    def alpha_fn(rng, shape):
        return np.exp(-rng.uniform(4.0, 8.0, shape))
    case = _kda_case(12, alpha_fn, lens=(200, 70))
    _check_kda(*case, alpha_ref=case[4], tol=1e-9)


def test_kda_chunked_algebra_clamps_tiny_decays():
    """Decays of magnitude below e^-8 (zero included) act as e^-8 with their sign: the
    factored form equals the recurrence on the clamped decays, and stays within e^-8 of the
    unclamped recurrence's largest value."""
    def alpha_fn(rng, shape):
        a = rng.uniform(-1.0, 1.0, shape)
        pick = rng.random(shape)
        a[pick < 0.05] = 0.0
        a[(pick >= 0.05) & (pick < 0.1)] *= 1e-6
        return a
    case = _kda_case(13, alpha_fn)
    alpha = case[4]
    clamped = np.where(alpha < 0, -1.0, 1.0) * np.maximum(np.abs(alpha), np.exp(-KDA_CLAMP))
    _check_kda(*case, alpha_ref=clamped, tol=1e-9)
    _check_kda(*case, alpha_ref=alpha, tol=2.0 * np.exp(-KDA_CLAMP))
