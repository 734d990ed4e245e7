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
