"""Pins of the CPU oracle against facts fixed by the pages and by the algebra.

Each pin is a function taking the oracle module and raising AssertionError when the
oracle disagrees.  tests/test_oracle_pins.py runs them on the oracle as built;
tests/test_oracle_mutants.py runs them on copies of the oracle with a planted mistake
and checks that every mistake is caught.

What the pins rest on (none of them re-types the oracle's recurrence):
  * the matrix (transition) form of each rule: gated_delta as
    S_t = g (I - beta k k^T) S_{t-1} + beta k v^T  ("Seven Architectures ...", section
    "Gated DeltaNet-2": b = w = beta with a scalar decay recovers Gated DeltaNet), delta
    without the decay, gated as g S + k v^T and linear as S + k v^T (ONNX section), and
    kda as the diagonal-plus-low-rank transition (I - beta k k^T) Diag(alpha) S_{t-1} +
    beta k v^T (section "Kimi Linear": a rank-one correction of the decayed state),
    evaluated as explicit products of d_k x d_k transition matrices in extended
    precision, and in exact rational arithmetic on the smallest shapes;
  * closed forms of the linear and gated rules (sums of outer products);
  * invariants: beta = 0 with g = 1 leaves S unchanged; delta with beta = 1 and a unit
    key stores v exactly under k; transitions with g in [-1, 1], beta in [0, 2] are
    non-expansive ("Complex KDA" section);
  * IEEE round-to-nearest-even to bfloat16 as implemented by torch's conversion;
  * plain numpy indexing for whole-slot copies.
"""
from fractions import Fraction

import numpy as np
import torch

from gated_deltanet_recurrent_la_b200 import workloads as W

LD = np.longdouble


def close(a, b, tol, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    ref = float(np.max(np.abs(b))) if b.size else 0.0
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol * max(ref, 1e-300), f"{what}: max|err| {err:.3e} > {tol:.1e} * max|ref| {ref:.3e}"


def np64(t):
    return None if t is None else t.double().numpy()


def transition(rule, k, v, g, beta, dtype=LD):
    """(A, W) of one token: S_t = A S_{t-1} + W, written from each rule's matrix form."""
    cast = (lambda x: x) if dtype is object else dtype
    k = np.asarray(k, dtype=dtype)
    v = np.asarray(v, dtype=dtype)
    I = np.eye(k.shape[0], dtype=dtype)
    kkT = np.outer(k, k)
    if rule == "linear":
        return I, np.outer(k, v)
    if rule == "gated":
        return cast(g) * I, np.outer(k, v)
    if rule == "delta":
        return I - cast(beta) * kkT, cast(beta) * np.outer(k, v)
    if rule == "gated_delta":
        return cast(g) * (I - cast(beta) * kkT), cast(beta) * np.outer(k, v)
    if rule == "kda":
        D = np.diag(np.asarray([cast(x) for x in g], dtype=dtype))
        return (I - cast(beta) * kkT).dot(D), cast(beta) * np.outer(k, v)
    raise ValueError(rule)


def brute_force_head(rule, S0, Q, K, V, G, Beta, scale=1.0, dtype=LD):
    """States S_1..S_T and outputs o_1..o_T of one head from products of transition
    matrices: S_t = (A_t ... A_1) S_0 + sum_s (A_t ... A_{s+1}) W_s, o_t = scale S_t^T q_t."""
    T = K.shape[0]
    AW = [transition(rule, K[t], V[t], None if G is None else G[t], None if Beta is None else Beta[t], dtype)
          for t in range(T)]
    S0 = np.asarray(S0, dtype=dtype)
    states, outs = [], []
    for t in range(T):
        P = np.eye(S0.shape[0], dtype=dtype)
        acc = AW[t][1].copy()
        for s in range(t - 1, -1, -1):
            P = P @ AW[s + 1][0]
            acc = acc + P @ AW[s][1]
        P = P @ AW[0][0]
        acc = acc + P @ S0
        states.append(acc)
        outs.append(dtype(scale) * (acc.T @ np.asarray(Q[t], dtype=dtype)))
    return states, outs


# ---------------------------------------------------------------------------------
# bfloat16 rounding


def pin_bf16_rounding(orc):
    rng = np.random.default_rng(0)
    x = rng.standard_normal(20000).astype(np.float32) * np.float32(3.0) ** rng.integers(-40, 40, 20000).astype(np.float32)
    # exact ties: a bf16 value plus half its quantum, both neighbours' parities
    base = torch.tensor(rng.standard_normal(4000).astype(np.float32)).to(torch.bfloat16).float().numpy()
    bits = base.view(np.uint32)
    ties = (bits | np.uint32(0x8000)).view(np.float32)
    special = np.array([0.0, -0.0, 1.0, -1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 3.3895313e38, 3.3961e38,
                        3.4e38, 1e-38, 1e-40, -1e-41, 2.0 ** -133, 2.0 ** -134, 3 * 2.0 ** -135,
                        np.inf, -np.inf], dtype=np.float32)
    xs = np.concatenate([x, ties, special]).astype(np.float32)
    ref = torch.tensor(xs).to(torch.bfloat16).double().numpy()
    got = orc.round_bf16(xs.astype(np.float64))
    bad = np.flatnonzero(~((got == ref) & (np.signbit(got) == np.signbit(ref))))
    assert bad.size == 0, f"bf16 rounding differs at {xs[bad[:5]]}: {got[bad[:5]]} vs {ref[bad[:5]]}"
    assert np.isnan(orc.round_bf16(np.array([np.nan]))[0])


# ---------------------------------------------------------------------------------
# helpers running the oracle on one workload


def run_scan_f64(orc, inp, init=None):
    """Oracle scan in pure f64 (no storage rounding); init [n_seqs, H, dk, dv] or None."""
    n_seqs = inp.cu_seqlens.numel() - 1
    kw = {}
    if init is not None:
        kw = dict(src_pool=init, read_slot=np.arange(n_seqs, dtype=np.int32))
    return orc.scan(inp.rule, inp.n_qk_heads, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k), np64(inp.v),
                    np64(inp.g), np64(inp.beta), inp.scale, **kw)


def run_steps_f64(orc, inp, init=None):
    """The same tokens fed as one decode step per token position (sequences of equal length)."""
    cu = inp.cu_seqlens.numpy()
    n_seqs = len(cu) - 1
    L = int(cu[1] - cu[0])
    assert all(cu[s + 1] - cu[s] == L for s in range(n_seqs))
    H, dk, dv = inp.n_v_heads, inp.d_k, inp.d_v
    pool = np.zeros((n_seqs, H, dk, dv)) if init is None else np.array(init, dtype=np.float64)
    outs = np.zeros((int(cu[-1]), H, dv))
    q, k, v = np64(inp.q), np64(inp.k), np64(inp.v)
    g, b = np64(inp.g), np64(inp.beta)
    for t in range(L):
        rows = cu[:-1] + t
        pool, o, err = orc.step(inp.rule, inp.n_qk_heads, pool, q[rows], k[rows], v[rows],
                                None if g is None else g[rows], None if b is None else b[rows], inp.scale)
        assert err == 0
        outs[rows] = o
    return pool, outs


def brute_force_all(inp, init=None, dtype=LD):
    cu = inp.cu_seqlens.numpy()
    H, dk, dv = inp.n_v_heads, inp.d_k, inp.d_v
    ratio = H // inp.n_qk_heads
    n_seqs = len(cu) - 1
    states = np.zeros((n_seqs, H, dk, dv))
    outs = np.zeros((int(cu[-1]), H, dv))
    q, k, v = np64(inp.q), np64(inp.k), np64(inp.v)
    g, b = np64(inp.g), np64(inp.beta)
    for s in range(n_seqs):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        for h in range(H):
            hq = h // ratio
            S0 = np.zeros((dk, dv)) if init is None else init[s, h]
            st, ou = brute_force_head(inp.rule, S0, q[t0:t1, hq], k[t0:t1, hq], v[t0:t1, h],
                                      None if g is None else g[t0:t1, h], None if b is None else b[t0:t1, h],
                                      inp.scale, dtype)
            states[s, h] = st[-1] if st else S0
            for i, o in enumerate(ou):
                outs[t0 + i, h] = o
    return states, outs


# ---------------------------------------------------------------------------------
# pins


def pin_brute_force_all_rules(orc):
    """All five rules on the tiny workload shapes (2 x 64 tokens, 2 heads, 16 x 16) with
    a random initial state: oracle scan and oracle decode steps vs transition products."""
    for rule in W.ALL_RULES:
        inp = W.tiny(rule, seed=3)
        init = np.random.default_rng(1).standard_normal((2, 2, 16, 16)) * 0.3
        S_ref, o_ref = brute_force_all(inp, init)
        S_scan, o_scan, err = run_scan_f64(orc, inp, init)
        assert err == 0
        close(S_scan, S_ref, 1e-9, f"{rule} scan state")
        close(o_scan, o_ref, 1e-9, f"{rule} scan output")
        S_step, o_step = run_steps_f64(orc, inp, init)
        close(S_step, S_ref, 1e-9, f"{rule} step state")
        close(o_step, o_ref, 1e-9, f"{rule} step output")


def pin_gqa_grouping(orc):
    """4 state heads over 2 q/k heads: heads 0, 1 read q/k head 0 and heads 2, 3 read
    q/k head 1 (contiguous groups).  Checked head by head against transition products."""
    inp = W.scan_inputs(lengths=[9, 14], n_qk_heads=2, n_v_heads=4, d_k=16, d_v=16, rule="gated_delta",
                        state_dtype=torch.float32, io_dtype=torch.float32, seed=5)
    S_ref, o_ref = brute_force_all(inp)
    S, o, err = run_scan_f64(orc, inp)
    assert err == 0
    close(S, S_ref, 1e-9, "gqa state")
    close(o, o_ref, 1e-9, "gqa output")


def pin_exact_rational(orc):
    """Exact rational arithmetic on the smallest shapes: dyadic inputs, d_k = 3, d_v = 2,
    5 tokens, every rule.  The oracle's double result must agree to ~1e-15."""
    rng = np.random.default_rng(7)
    dk, dv, T = 3, 2, 5

    def dy(shape, den=8):
        return rng.integers(-8, 9, size=shape) / den

    for rule in W.ALL_RULES:
        K, Q, V = dy((T, dk)), dy((T, dk)), dy((T, dv))
        G = rng.integers(1, 8, size=(T, dk) if rule == "kda" else T) / 8.0
        Bt = rng.integers(0, 9, size=T) / 8.0
        S0 = dy((dk, dv), 4)
        F = lambda a: np.vectorize(Fraction)(a).astype(object)  # noqa: E731
        S = F(S0)
        outs = []
        for t in range(T):
            Gt = list(F(G[t])) if rule == "kda" else Fraction(G[t])
            A, Wm = transition(rule, F(K[t]), F(V[t]), Gt, Fraction(Bt[t]), dtype=object)
            S = A.dot(S) + Wm
            outs.append(S.T.dot(F(Q[t])))
        inp = W.Inputs("scan", rule, 1, 1, dk, dv, torch.float64, torch.float64,
                       torch.tensor(Q[:, None, :]), torch.tensor(K[:, None, :]), torch.tensor(V[:, None, :]),
                       torch.tensor(G[:, None]), torch.tensor(Bt[:, None]), 1.0, None, None, None,
                       torch.tensor([0, T], dtype=torch.int32))
        Sg, og, err = run_scan_f64(orc, inp, S0[None, None])
        assert err == 0
        close(Sg[0, 0], np.array(S, dtype=np.float64), 1e-14, f"{rule} exact state")
        close(og[:, 0], np.array(outs, dtype=np.float64), 1e-14, f"{rule} exact output")


def pin_linear_closed_form(orc):
    """linear: S_T = S_0 + sum_t k_t v_t^T and o_t = (S_0 + sum_{s<=t} k_s v_s^T)^T q_t."""
    inp = W.tiny("linear", seed=11)
    init = np.random.default_rng(2).standard_normal((2, 2, 16, 16))
    S, o, err = run_scan_f64(orc, inp, init)
    assert err == 0
    cu = inp.cu_seqlens.numpy()
    q, k, v = np64(inp.q), np64(inp.k), np64(inp.v)
    for s in range(2):
        t0, t1 = cu[s], cu[s + 1]
        for h in range(2):
            outer = np.einsum("ti,tj->tij", k[t0:t1, h], v[t0:t1, h])
            cum = init[s, h][None] + np.cumsum(outer, axis=0)
            close(S[s, h], cum[-1], 1e-12, "linear closed-form state")
            close(o[t0:t1, h], np.einsum("tij,ti->tj", cum, q[t0:t1, h]), 1e-12, "linear closed-form output")


def pin_gated_closed_form(orc):
    """gated: S_T = (prod_t g_t) S_0 + sum_t (prod_{s>t} g_s) k_t v_t^T."""
    inp = W.tiny("gated", seed=12)
    init = np.random.default_rng(3).standard_normal((2, 2, 16, 16))
    S, o, err = run_scan_f64(orc, inp, init)
    assert err == 0
    cu = inp.cu_seqlens.numpy()
    k, v, g = np64(inp.k), np64(inp.v), np64(inp.g)
    for s in range(2):
        t0, t1 = cu[s], cu[s + 1]
        for h in range(2):
            gs = g[t0:t1, h]
            tail = np.array([np.prod(gs[t + 1:]) for t in range(len(gs))])
            ref = np.prod(gs) * init[s, h] + np.einsum("t,ti,tj->ij", tail, k[t0:t1, h], v[t0:t1, h])
            close(S[s, h], ref, 1e-12, "gated closed-form state")


def pin_beta0_g1_identity(orc):
    """beta = 0 with g = 1 leaves the state unchanged, bit for bit, at every storage type."""
    for rule in ("delta", "gated_delta"):
        for dt in ("f32", "bf16"):
            inp = W.step_inputs(B=3, n_qk_heads=1, n_v_heads=2, d_k=16, d_v=16, rule=rule, slot_map="dense",
                                state_dtype=torch.float32 if dt == "f32" else torch.bfloat16,
                                io_dtype=torch.float32, g_mode="one", beta_mode="zero", seed=4)
            pool = np64(inp.pool)
            new, o, err = orc.step(rule, 1, pool, np64(inp.q), np64(inp.k), np64(inp.v), np64(inp.g),
                                   np64(inp.beta), dst_dtype=dt)
            assert err == 0
            assert np.array_equal(new, pool), f"{rule}/{dt}: state changed"
            ref = np.einsum("bhij,bi->bhj", pool, np64(inp.q)[:, 0])
            close(o, ref, 1e-12, "readout of the unchanged state")


def pin_delta_stores_value(orc):
    """delta, beta = 1, unit key: S_new^T k = v (the association is stored exactly), and
    reading with q = k returns v."""
    inp = W.step_inputs(B=4, n_qk_heads=2, n_v_heads=2, d_k=16, d_v=16, rule="delta", slot_map="dense",
                        state_dtype=torch.float64, io_dtype=torch.float64, beta_mode="one", seed=6, pool_std=1.0)
    k = np64(inp.k)
    k = k / np.linalg.norm(k, axis=-1, keepdims=True)  # unit to double precision
    new, o, err = orc.step("delta", 2, np64(inp.pool), k, k, np64(inp.v), None, np64(inp.beta))
    assert err == 0
    close(np.einsum("bhij,bhi->bhj", new, k), np64(inp.v), 1e-12, "S^T k = v")
    close(o, np64(inp.v), 1e-12, "o = v for q = k")


def pin_rearranged_readout(orc):
    """o from the updated state equals the rearranged form a S_old^T q + (k.q) u (checked
    against the direct readout of the brute-force state)."""
    for rule in W.ALL_RULES:
        inp = W.step_inputs(B=3, n_qk_heads=1, n_v_heads=2, d_k=16, d_v=16, rule=rule, slot_map="dense",
                            state_dtype=torch.float64, io_dtype=torch.float64, seed=8, pool_std=0.5, scale=0.7)
        pool = np64(inp.pool)
        args = (np64(inp.q), np64(inp.k), np64(inp.v), np64(inp.g), np64(inp.beta), 0.7)
        _, o_direct, err = orc.step(rule, 1, pool, *args)
        assert err == 0
        o_re = orc.readout_rearranged(rule, 1, pool, *args)
        close(o_re, o_direct, 1e-12, f"{rule} rearranged readout")
        q, k, v = np64(inp.q), np64(inp.k), np64(inp.v)
        for b in range(3):
            for h in range(2):
                gb = inp.g[b, h].tolist() if rule == "kda" else inp.g[b, h].item()
                A, Wm = transition(rule, k[b, 0], v[b, h], gb, inp.beta[b, h].item(), np.float64)
                S1 = A @ pool[b, h] + Wm
                close(o_direct[b, h], 0.7 * S1.T @ q[b, 0], 1e-12, f"{rule} direct readout")


def pin_scan_structure(orc):
    """A scan over cu_seqlens equals separate scans of each sequence; a one-token scan
    equals one decode step; an empty sequence stores its initial state unchanged."""
    inp = W.scan_inputs(lengths=[5, 0, 17, 1], n_qk_heads=1, n_v_heads=2, d_k=16, d_v=16, rule="gated_delta",
                        state_dtype=torch.float32, io_dtype=torch.float32, seed=9, init="slots")
    init = np64(inp.pool)[inp.read_slot.numpy()]
    S, o, err = run_scan_f64(orc, inp, init)
    assert err == 0
    cu = inp.cu_seqlens.numpy()
    for s in range(4):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        sub = W.Inputs("scan", inp.rule, 1, 2, 16, 16, inp.state_dtype, inp.io_dtype, inp.q[t0:t1],
                       inp.k[t0:t1], inp.v[t0:t1], inp.g[t0:t1], inp.beta[t0:t1], 1.0, None, None, None,
                       torch.tensor([0, t1 - t0], dtype=torch.int32))
        Ss, os_, err = run_scan_f64(orc, sub, init[s:s + 1])
        assert err == 0
        assert np.array_equal(Ss[0], S[s]) and np.array_equal(os_, o[t0:t1]), f"sequence {s}"
    assert np.array_equal(S[1], init[1]), "empty sequence must keep its initial state"
    one = W.scan_inputs(lengths=[1, 1, 1], n_qk_heads=1, n_v_heads=2, d_k=16, d_v=16, rule="delta",
                        state_dtype=torch.float32, io_dtype=torch.float32, seed=10)
    pool0 = np.random.default_rng(4).standard_normal((3, 2, 16, 16))
    S1, o1, _ = run_scan_f64(orc, one, pool0)
    S2, o2, _ = orc.step("delta", 1, pool0, np64(one.q), np64(one.k), np64(one.v), np64(one.g), np64(one.beta))
    assert np.array_equal(S1, S2) and np.array_equal(o1, o2)


def pin_wide_ranges_non_expansive(orc):
    """g ~ U[-1, 1], beta ~ U[0, 2], unit keys: the oracle follows the transition products
    (nothing is clamped), and since |g| max(1, |1 - beta|) <= 1 the state norm obeys
    ||S_t||_F <= ||S_{t-1}||_F + beta ||k|| ||v|| at every step."""
    inp = W.scan_inputs(lengths=[48], n_qk_heads=1, n_v_heads=2, d_k=16, d_v=16, rule="gated_delta",
                        state_dtype=torch.float32, io_dtype=torch.float32, seed=13, g_mode="uniform_pm1",
                        beta_mode="uniform_0_2")
    init = np.random.default_rng(5).standard_normal((1, 2, 16, 16))
    S_ref, o_ref = brute_force_all(inp, init)
    S, o, err = run_scan_f64(orc, inp, init)
    assert err == 0
    close(S, S_ref, 1e-9, "wide-range state")
    close(o, o_ref, 1e-9, "wide-range output")
    pool = init.copy()
    q, k, v, g, b = np64(inp.q), np64(inp.k), np64(inp.v), np64(inp.g), np64(inp.beta)
    for t in range(48):
        prev = np.linalg.norm(pool.reshape(2, -1), axis=1)
        pool, _, _ = orc.step("gated_delta", 1, pool, q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1], b[t:t + 1])
        now = np.linalg.norm(pool.reshape(2, -1), axis=1)
        bound = prev + b[t] * np.linalg.norm(v[t], axis=1) + 1e-12
        assert np.all(now <= bound), (t, now, bound)


def pin_long_sequence_bounded(orc):
    """gated_delta with unit keys, beta in (0, 1), g < 1 over a prefill-length sequence:
    the state stays bounded by the recursion ||S_t|| <= g_t ||S_{t-1}|| + beta_t ||v_t||."""
    inp = W.scan_inputs(lengths=[8192], n_qk_heads=1, n_v_heads=1, d_k=16, d_v=16, rule="gated_delta",
                        state_dtype=torch.float32, io_dtype=torch.float32, seed=14)
    S, o, err = run_scan_f64(orc, inp)
    assert err == 0 and np.all(np.isfinite(S)) and np.all(np.isfinite(o))
    g, b, v = np64(inp.g)[:, 0], np64(inp.beta)[:, 0], np64(inp.v)[:, 0]
    bound = 0.0
    for t in range(8192):
        bound = g[t] * bound + b[t] * np.linalg.norm(v[t])
    assert np.linalg.norm(S) <= bound * (1 + 1e-9)


def pin_storage_rounding_points(orc):
    """Decode rounds the state to the storage type after each step; the scan keeps it
    unrounded across tokens and rounds once at the end; outputs round to the io type."""
    inp = W.tiny("gated_delta", seed=15)
    cu = inp.cu_seqlens.numpy()
    S64, o64, _ = run_scan_f64(orc, inp)
    Sbf, obf, _ = orc.scan("gated_delta", 2, cu, np64(inp.q), np64(inp.k), np64(inp.v), np64(inp.g),
                           np64(inp.beta), dst_dtype="bf16", io_dtype="bf16")
    ref_S = torch.tensor(S64).to(torch.bfloat16).double().numpy()
    ref_o = torch.tensor(o64).to(torch.bfloat16).double().numpy()
    assert np.array_equal(Sbf, ref_S) and np.array_equal(obf, ref_o)
    pool = np.zeros((2, 2, 16, 16))
    q, k, v, g, b = np64(inp.q), np64(inp.k), np64(inp.v), np64(inp.g), np64(inp.beta)
    for t in range(3):
        rows = cu[:-1] + t
        new64, _, _ = orc.step("gated_delta", 2, pool, q[rows], k[rows], v[rows], g[rows], b[rows])
        newbf, _, _ = orc.step("gated_delta", 2, pool, q[rows], k[rows], v[rows], g[rows], b[rows], dst_dtype="bf16")
        assert np.array_equal(newbf, torch.tensor(new64).to(torch.bfloat16).double().numpy())
        pool = newbf


def pin_slots(orc):
    """Slots: a request that reads a checkpoint slot and writes a live slot leaves the
    checkpoint untouched; untouched slots stay unchanged; reading and writing through a
    permutation gives the same states as the dense step on the gathered states."""
    inp = W.step_inputs(B=6, n_qk_heads=1, n_v_heads=2, d_k=16, d_v=16, n_slots=12, rule="gated_delta",
                        slot_map="checkpoint", state_dtype=torch.float32, io_dtype=torch.float32, seed=16)
    pool = np64(inp.pool)
    rs, ws = inp.read_slot.numpy(), inp.write_slot.numpy()
    args = (np64(inp.q), np64(inp.k), np64(inp.v), np64(inp.g), np64(inp.beta))
    new, o, err = orc.step("gated_delta", 1, pool, *args, read_slot=rs, write_slot=ws)
    assert err == 0
    dense_new, dense_o, _ = orc.step("gated_delta", 1, pool[rs], *args)
    assert np.array_equal(new[ws], dense_new) and np.array_equal(o, dense_o)
    untouched = np.setdiff1d(np.arange(12), ws)
    assert np.array_equal(new[untouched], pool[untouched])
    assert set(rs) - set(ws), "the workload must contain checkpoint reads"
    bad = rs.copy()
    bad[2] = 12
    new2, o2, err = orc.step("gated_delta", 1, pool, *args, read_slot=bad, write_slot=ws)
    assert err == 1 and np.array_equal(new2[ws[2]], pool[ws[2]]) and not o2[2].any()


def pin_pool_ops(orc):
    """Whole-slot copy / gather / scatter / zero equal numpy indexing, bit for bit."""
    rng = np.random.default_rng(17)
    pool = torch.randn(10, 2, 16, 16).to(torch.bfloat16).view(torch.int16).numpy().copy()
    slots = np.array([7, 2, 2, 9], dtype=np.int32)
    dense, err = orc.pool_gather(pool, slots)
    assert err == 0 and np.array_equal(dense, pool[slots])
    p2 = pool.copy()
    src, dst = np.array([1, 3], dtype=np.int32), np.array([5, 0], dtype=np.int32)
    assert orc.pool_copy(p2, src, dst) == 0
    ref = pool.copy()
    ref[dst] = pool[src]
    assert np.array_equal(p2, ref)
    p3 = pool.copy()
    new = rng.integers(-30000, 30000, size=(2, 2, 16, 16)).astype(np.int16)
    assert orc.pool_scatter(p3, np.array([4, 8], dtype=np.int32), new) == 0
    ref = pool.copy()
    ref[[4, 8]] = new
    assert np.array_equal(p3, ref)
    p4 = pool.copy()
    assert orc.pool_zero(p4, np.array([6], dtype=np.int32)) == 0
    ref = pool.copy()
    ref[6] = 0
    assert np.array_equal(p4, ref)
    assert orc.pool_zero(p4, np.array([10], dtype=np.int32)) == 2


def pin_scan_checkpoints(orc):
    """Checkpoint j of a sequence is the state after its first (j + 1) * every tokens:
    checked against the transition-product states at those positions, for every rule,
    with a random initial state; a checkpoint beyond the sequence is reported (bit 4)."""
    every = 4
    for rule in W.ALL_RULES:
        inp = W.scan_inputs(lengths=[21, 7, 0, 12], n_qk_heads=1, n_v_heads=2, d_k=16, d_v=16, rule=rule,
                            state_dtype=torch.float32, io_dtype=torch.float32, seed=17)
        init = np.random.default_rng(6).standard_normal((4, 2, 16, 16)) * 0.5
        cu = inp.cu_seqlens.numpy()
        lens = cu[1:] - cu[:-1]
        n_ck = lens // every
        ckpt_cu = np.concatenate([[0], np.cumsum(n_ck)]).astype(np.int32)
        ckpt_slots = (4 + np.arange(ckpt_cu[-1])).astype(np.int32)
        dst = np.zeros((4 + ckpt_cu[-1], 2, 16, 16))
        S, o, err = orc.scan(rule, 1, cu, np64(inp.q), np64(inp.k), np64(inp.v), np64(inp.g), np64(inp.beta),
                             src_pool=init, read_slot=np.arange(4, dtype=np.int32), dst_pool=dst,
                             ckpt_every=every, ckpt_cu=ckpt_cu, ckpt_slots=ckpt_slots)
        assert err == 0
        q, k, v = np64(inp.q), np64(inp.k), np64(inp.v)
        g, b = np64(inp.g), np64(inp.beta)
        for sq in range(4):
            t0, t1 = int(cu[sq]), int(cu[sq + 1])
            for h in range(2):
                states, _ = brute_force_head(rule, init[sq, h], q[t0:t1, 0], k[t0:t1, 0], v[t0:t1, h],
                                             None if g is None else g[t0:t1, h], None if b is None else b[t0:t1, h])
                for j in range(n_ck[sq]):
                    close(S[ckpt_slots[ckpt_cu[sq] + j], h], states[(j + 1) * every - 1], 1e-9,
                          f"{rule} seq {sq} head {h} checkpoint {j}")
                close(S[sq, h], states[-1] if states else init[sq, h], 1e-9, f"{rule} final state")
    # one checkpoint too many for sequence 1 (7 tokens, every 4): reported, the rest still written
    bad_cu = ckpt_cu.copy()
    bad_cu[2:] += 1
    bad_slots = np.concatenate([ckpt_slots[:ckpt_cu[2]], [3], ckpt_slots[ckpt_cu[2]:]]).astype(np.int32)
    _, _, err = orc.scan("gated_delta", 1, cu, np64(inp.q), np64(inp.k), np64(inp.v), np64(inp.g), np64(inp.beta),
                         dst_pool=np.zeros_like(dst), ckpt_every=every, ckpt_cu=bad_cu, ckpt_slots=bad_slots)
    assert err == 4


def pin_kda_reductions(orc):
    """kda special cases: (1) every channel decaying by the same g is the gated_delta rule
    with that scalar gate, checked against the scalar transition products; (2) beta = 0
    leaves only the per-channel decay, S_T = Diag(prod_t alpha_t) S_0, and each output is
    the decayed initial state read by q_t."""
    inp = W.tiny("gated_delta", seed=19)
    gk = np.repeat(np64(inp.g)[:, :, None], 16, axis=2)  # [T, H, d_k], equal channels
    init = np.random.default_rng(8).standard_normal((2, 2, 16, 16)) * 0.5
    S_ref, o_ref = brute_force_all(inp, init)
    S, o, err = orc.scan("kda", 2, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k), np64(inp.v), gk,
                         np64(inp.beta), src_pool=init, read_slot=np.arange(2, dtype=np.int32))
    assert err == 0
    close(S, S_ref, 1e-9, "kda with equal channels = gated_delta (state)")
    close(o, o_ref, 1e-9, "kda with equal channels = gated_delta (output)")

    inp = W.scan_inputs(lengths=[37], n_qk_heads=1, n_v_heads=2, d_k=16, d_v=8, rule="kda",
                        state_dtype=torch.float32, io_dtype=torch.float32, seed=20, beta_mode="zero")
    init = np.random.default_rng(9).standard_normal((1, 2, 16, 8))
    S, o, err = run_scan_f64(orc, inp, init)
    assert err == 0
    a, q = np64(inp.g), np64(inp.q)
    decay = np.cumprod(a, axis=0)  # [T, H, d_k]: prod_{s<=t} alpha_s per channel
    for h in range(2):
        close(S[0, h], decay[-1, h][:, None] * init[0, h], 1e-12, "kda beta = 0 state")
        ref_o = np.einsum("ti,ij,ti->tj", decay[:, h], init[0, h], q[:, 0])
        close(o[:, h], ref_o, 1e-12, "kda beta = 0 outputs")


def pin_kda_wide_ranges_non_expansive(orc):
    """kda with alpha ~ U[-1, 1] per channel and beta ~ U[0, 2] ("Complex KDA" ranges),
    unit keys: the oracle follows the transition products, and because
    ||(I - beta k k^T) Diag(alpha)||_2 <= 1 the state norm obeys
    ||S_t||_F <= ||S_{t-1}||_F + beta ||v|| at every step."""
    inp = W.scan_inputs(lengths=[40], n_qk_heads=1, n_v_heads=2, d_k=16, d_v=16, rule="kda",
                        state_dtype=torch.float32, io_dtype=torch.float32, seed=21, g_mode="uniform_pm1",
                        beta_mode="uniform_0_2")
    init = np.random.default_rng(10).standard_normal((1, 2, 16, 16))
    S_ref, o_ref = brute_force_all(inp, init)
    S, o, err = run_scan_f64(orc, inp, init)
    assert err == 0
    close(S, S_ref, 1e-9, "kda wide-range state")
    close(o, o_ref, 1e-9, "kda wide-range output")
    pool = init.copy()
    q, k, v, g, b = np64(inp.q), np64(inp.k), np64(inp.v), np64(inp.g), np64(inp.beta)
    for t in range(40):
        prev = np.linalg.norm(pool.reshape(2, -1), axis=1)
        pool, _, _ = orc.step("kda", 1, pool, q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1], b[t:t + 1])
        now = np.linalg.norm(pool.reshape(2, -1), axis=1)
        assert np.all(now <= prev + b[t] * np.linalg.norm(v[t], axis=1) + 1e-12), t


def pin_query_groups(orc):
    """Query-group direction of the ONNX operator (each state head read by a group of query
    heads): 2 state heads, 6 query heads.  Each state head's states come from transition
    products of its own k, v; query head i reads the state of head i // 3 after the token.
    Checked for the scan and for sequential decode steps, for gated_delta and kda; with one
    query per state head it equals the default direction."""
    for rule in ("gated_delta", "kda"):
        inp = W.scan_inputs(lengths=[13, 6], n_qk_heads=2, n_v_heads=2, d_k=16, d_v=8, rule=rule,
                            state_dtype=torch.float32, io_dtype=torch.float32, seed=22, n_q_heads=6)
        init = np.random.default_rng(11).standard_normal((2, 2, 16, 8)) * 0.5
        q, k, v = np64(inp.q), np64(inp.k), np64(inp.v)
        g, b = np64(inp.g), np64(inp.beta)
        cu = inp.cu_seqlens.numpy()
        S, o, err = orc.scan_qgroups(rule, 6, cu, q, k, v, g, b, src_pool=init, read_slot=np.arange(2, dtype=np.int32))
        assert err == 0 and o.shape == (19, 6, 8)
        for sq in range(2):
            t0, t1 = int(cu[sq]), int(cu[sq + 1])
            for h in range(2):
                states, _ = brute_force_head(rule, init[sq, h], q[t0:t1, 0], k[t0:t1, h], v[t0:t1, h], g[t0:t1, h],
                                             b[t0:t1, h])
                close(S[sq, h], states[-1], 1e-9, f"{rule} query-group state")
                for i in range(3 * h, 3 * h + 3):
                    ref = np.stack([states[t].T.astype(np.float64) @ q[t0 + t, i] for t in range(t1 - t0)])
                    close(o[t0:t1, i], ref, 1e-9, f"{rule} query head {i}")
        # the same tokens as decode steps (sequence 1's 6 tokens)
        pool = init[1:2].copy()
        for t in range(int(cu[1]), int(cu[2])):
            pool, ot, err = orc.step_qgroups(rule, 6, pool, q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1], b[t:t + 1])
            assert err == 0
            close(ot[0], o[t], 1e-12, f"{rule} query-group step vs scan")
        close(pool[0], S[1], 1e-12, f"{rule} query-group step state")
    # one query per state head: identical to the default direction with H_qk = H_v
    inp = W.scan_inputs(lengths=[9], n_qk_heads=2, n_v_heads=2, d_k=16, d_v=16, rule="gated_delta",
                        state_dtype=torch.float32, io_dtype=torch.float32, seed=23)
    S1, o1, _ = run_scan_f64(orc, inp)
    S2, o2, _ = orc.scan_qgroups("gated_delta", 2, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k), np64(inp.v),
                                 np64(inp.g), np64(inp.beta))
    assert np.array_equal(S1, S2) and np.array_equal(o1, o2)


# ---------------------------------------------------------------------------------
# mixed INT8 / BF16 ("q8") state storage


def _q8_masks(H, dk, n_hp, seed):
    rng = np.random.default_rng(seed)
    masks = np.zeros((H, dk // 32), dtype=np.uint32)
    for h in range(H):
        for i in rng.choice(dk, n_hp, replace=False):
            masks[h, i // 32] |= np.uint32(1 << (i % 32))
    return masks


def _hp_rows(masks, h, dk):
    return [i for i in range(dk) if (int(masks[h, i // 32]) >> (i % 32)) & 1]


def pin_q8_page_figures(orc):
    """With 1/8 of the key channels in BF16, the q8 tile of a 128 x 128 head holds
    9.875 bits per value and saves 69.14 % of FP32 storage: the page's 9.9 bits and 69.1 %."""
    G = {}
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "page_sizes.txt")
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            k, v = line.split()[:2]
            G[k] = int(v)
    nbytes = orc.q8_tile_bytes(128, 128, 16)
    bits = 8.0 * nbytes / (128 * 128)
    assert round(bits * 10) == G["damp_bits_per_value_x10"], bits
    assert round((1 - bits / 32) * 1000) == G["damp_storage_reduction_pct_x10"], bits


def pin_q8_codec(orc):
    """The codec against its definition checked by properties: INT8 rows reproduce every
    value within half a group step (s / 2, s = group absmax / 127, plus the few FP32
    roundings of s and of the inverse scale: 1e-4 s), the group's largest
    magnitude lands on code +-127, all-zero groups decode to zero, values k * 2^e of a
    group whose absmax is 127 * 2^e come back exactly; BF16 rows equal torch's
    round-to-nearest-even conversion bit for bit."""
    rng = np.random.default_rng(12)
    H, dk, dv, n_hp = 3, 64, 64, 8
    masks = _q8_masks(H, dk, n_hp, 1)
    x = (rng.standard_normal((2, H, dk, dv)) * 10.0 ** rng.integers(-6, 6, (2, H, dk, 1))).astype(np.float32)
    x[0, 0, :, 32:] = 0.0                                                   # zero groups
    e = rng.integers(-10, 10, (2, H, dk, 2))
    x[1] = (rng.integers(-127, 128, (H, dk, dv)) * np.repeat(2.0 ** e[1], 32, axis=2)).astype(np.float32)
    x[1, :, :, 0] = 127 * 2.0 ** e[1][:, :, 0]                             # absmax 127 * 2^e per group
    x[1, :, :, 32] = -127 * 2.0 ** e[1][:, :, 1]
    b = orc.q8_encode(x, n_hp, masks)
    assert b.shape[2] == orc.q8_tile_bytes(dk, dv, n_hp)
    y = orc.q8_decode(b, dk, dv, n_hp, masks)
    for n in range(2):
        for h in range(H):
            hp = _hp_rows(masks, h, dk)
            assert len(hp) == n_hp
            ref = torch.tensor(x[n, h, hp]).to(torch.bfloat16).float().numpy()
            assert np.array_equal(y[n, h, hp].view(np.uint32), ref.view(np.uint32)), "bf16 rows"
            lo = [i for i in range(dk) if i not in hp]
            xg = x[n, h, lo].reshape(len(lo), dv // 32, 32).astype(np.float64)
            yg = y[n, h, lo].reshape(len(lo), dv // 32, 32).astype(np.float64)
            amax = np.abs(xg).max(axis=2, keepdims=True)
            step = amax / 127.0
            assert np.all(np.abs(yg - xg) <= step * (0.5 + 1e-4) + 1e-45), "int8 rows within s / 2"
            arg = np.abs(xg).argmax(axis=2)
            top = np.take_along_axis(yg, arg[..., None], axis=2)[..., 0]
            big = amax[..., 0] > 0
            assert np.allclose(np.abs(top[big]), amax[..., 0][big], rtol=1e-6), "absmax on code 127"
            assert np.all(yg[~big] == 0.0), "zero groups"
            if n == 1:
                assert np.array_equal(yg, xg), "exact dyadic groups"
    # codes and scales sit where the layout says: row r8, group g -> scale at n8 * dv + 4 (r8 * ng + g)
    n8, ng = dk - n_hp, dv // 32
    scales = b[1, 0, n8 * dv:n8 * dv + 4 * n8 * ng].view(np.float32).reshape(n8, ng)
    lo = [i for i in range(dk) if i not in _hp_rows(masks, 0, dk)]
    assert np.array_equal(scales, (2.0 ** e[1][0][lo]).astype(np.float32)), "scale layout"
    codes = b[1, 0, :n8 * dv].view(np.int8).reshape(n8, dv).astype(np.float64)
    assert np.array_equal(codes * np.repeat(scales, 32, axis=1), x[1, 0, lo]), "code layout"


def pin_q8_store_point(orc):
    """Decode step and scan with q8 destinations: every stored tile is the codec applied to
    the FP32-rounded state of the unquantised oracle, each head with its own mask."""
    H, dk, dv, n_hp = 2, 64, 64, 8
    masks = _q8_masks(H, dk, n_hp, 2)
    inp = W.step_inputs(B=3, n_qk_heads=1, n_v_heads=H, d_k=dk, d_v=dv, rule="gated_delta", slot_map="dense",
                        state_dtype=torch.float32, io_dtype=torch.float32, seed=24)
    args = (np64(inp.q), np64(inp.k), np64(inp.v), np64(inp.g), np64(inp.beta))
    ref, o_ref, _ = orc.step("gated_delta", 1, np64(inp.pool), *args, dst_dtype="f32")
    got, o, err = orc.step_q8("gated_delta", 1, np64(inp.pool), *args, masks=masks)
    assert err == 0 and np.array_equal(o, o_ref)
    want = orc.q8_decode(orc.q8_encode(ref.astype(np.float32), n_hp, masks), dk, dv, n_hp, masks)
    assert np.array_equal(got, want.astype(np.float64)), "step: q8 store"
    sc = W.scan_inputs(lengths=[11, 4], n_qk_heads=1, n_v_heads=H, d_k=dk, d_v=dv, rule="kda",
                       state_dtype=torch.float32, io_dtype=torch.float32, seed=25)
    cu = sc.cu_seqlens.numpy()
    args = (np64(sc.q), np64(sc.k), np64(sc.v), np64(sc.g), np64(sc.beta))
    ref, _, _ = orc.scan("kda", 1, cu, *args, dst_dtype="f32")
    got, _, err = orc.scan_q8("kda", 1, cu, *args, masks=masks)
    assert err == 0
    want = orc.q8_decode(orc.q8_encode(ref.astype(np.float32), n_hp, masks), dk, dv, n_hp, masks)
    assert np.array_equal(got, want.astype(np.float64)), "scan: q8 store"


# ---------------------------------------------------------------------------------
# short causal convolution ahead of the step


def _conv_operands(seed, H_qk=1, H=2, dk=16, dv=8, W=4, T=9):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((T, H_qk, dk)), rng.standard_normal((T, H_qk, dk)), rng.standard_normal((T, H, dv)),
            rng.standard_normal((H_qk, dk, W)), rng.standard_normal((H_qk, dk, W)), rng.standard_normal((H, dv, W)),
            rng.standard_normal((1, H, 2 * dk + dv, W - 1)))


def pin_conv_definition(orc):
    """Token by token, the convolution equals numpy's full convolution of each channel's
    input sequence (preceded by the W - 1 inputs of the initial history) with the reversed
    weights; SiLU is y * expit(y); the q/k normalisation gives unit vectors; the history
    after T tokens holds the last W - 1 inputs.  Two state heads over one q/k head both see
    that head's channels (each keeps its own copy)."""
    from scipy.special import expit
    for W in (2, 4):
        xq, xk, xv, wq, wk, wv, hist0 = _conv_operands(30 + W, W=W)
        T, dk, dv = xq.shape[0], xq.shape[2], xv.shape[2]
        for act, l2 in ((0, 0), (1, 0), (1, 1)):
            hist = hist0.copy()
            outs = []
            for t in range(T):
                q, k, v, hist = orc.conv(1, xq[t:t + 1], xk[t:t + 1], xv[t:t + 1], wq, wk, wv, hist, act=act,
                                         l2norm=l2)
                outs.append((q[0], k[0], v[0]))
            for h in range(2):
                for kind, xs, w, nch in (("q", xq[:, 0], wq[0], dk), ("k", xk[:, 0], wk[0], dk),
                                         ("v", xv[:, h], wv[h], dv)):
                    base = {"q": 0, "k": dk, "v": 2 * dk}[kind]
                    for c in range(nch):
                        seq = np.concatenate([hist0[0, h, base + c], xs[:, c]])
                        y = np.convolve(seq, w[c][::-1])[W - 1:W - 1 + T]
                        if act:
                            y = y * expit(y)
                        got = np.array([o[{"q": 0, "k": 1, "v": 2}[kind]][h, c] for o in outs])
                        if l2 and kind != "v":
                            ys = []
                            for t in range(T):
                                full = np.array([np.convolve(np.concatenate([hist0[0, h, base + cc], xs[:, cc]]),
                                                             w[cc][::-1])[W - 1 + t] for cc in range(nch)])
                                full = full * expit(full)
                                ys.append(full[c] / np.sqrt(np.sum(full ** 2) + 1e-6))
                            y = np.array(ys)
                        close(got, y, 1e-12, f"conv W={W} act={act} l2={l2} {kind}{c} head {h}")
                    last = np.concatenate([hist0[0, h, base:base + nch].T, xs.reshape(T, -1)[:, :nch]])[-(W - 1):].T
                    close(hist[0, h, base:base + nch], last, 0.0 + 1e-300, f"history {kind}")


def pin_conv_fused_step(orc):
    """The fused step equals the convolution followed by the recurrence: states and outputs
    against transition products of the post-convolution operands, and the histories go to
    the write slots."""
    xq, xk, xv, wq, wk, wv, hist = _conv_operands(40, T=3)
    rng = np.random.default_rng(41)
    B, H, dk, dv = 3, 2, 16, 8
    pool = rng.standard_normal((5, H, dk, dv)) * 0.3
    hists = rng.standard_normal((5, H, 2 * dk + dv, 3))
    g, beta = rng.uniform(0.2, 1.0, (B, H)), rng.uniform(0.0, 1.0, (B, H))
    rs, ws = np.array([4, 1, 2], np.int32), np.array([0, 1, 3], np.int32)
    new, hnew, o, err = orc.step_conv("gated_delta", 1, pool, xq, xk, xv, g, beta, 0.9, wq, wk, wv, hists, act=1,
                                      l2norm=1, read_slot=rs, write_slot=ws)
    assert err == 0
    q, k, v, hout = orc.conv(1, xq, xk, xv, wq, wk, wv, hists[rs], act=1, l2norm=1)
    for b in range(B):
        for h in range(H):
            states, outs = brute_force_head("gated_delta", pool[rs[b], h], q[b, h][None], k[b, h][None],
                                            v[b, h][None], g[b, h][None], beta[b, h][None], 0.9)
            close(new[ws[b], h], states[0], 1e-12, "fused step state")
            close(o[b, h], outs[0], 1e-12, "fused step output")
    close(hnew[ws], hout, 1e-300, "histories to the write slots")
    assert np.array_equal(hnew[4], hists[4]) and np.array_equal(new[4], pool[4]), "read-only slot untouched"


def pin_conv_scan(orc):
    """The scan with the convolution ahead equals one fused decode step per token with the
    history carried from step to step (sequences of unequal lengths, one empty, one shorter
    than the window), from read-slot histories; the final histories (the last W - 1
    inputs, the old history shifted in for short sequences) go to the write slots."""
    rng = np.random.default_rng(50)
    H, dk, dv, W = 2, 16, 8, 4
    lens = [5, 0, 2, 9]
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    xq, xk, xv = rng.standard_normal((T, 1, dk)), rng.standard_normal((T, 1, dk)), rng.standard_normal((T, H, dv))
    wq, wk, wv = rng.standard_normal((1, dk, W)), rng.standard_normal((1, dk, W)), rng.standard_normal((H, dv, W))
    g, beta = rng.uniform(0.3, 1.0, (T, H)), rng.uniform(0.0, 1.0, (T, H))
    pool = rng.standard_normal((6, H, dk, dv)) * 0.3
    hists = rng.standard_normal((6, H, 2 * dk + dv, W - 1))
    rs, ws = np.array([5, 2, 0, 3], np.int32), np.array([1, 4, 2, 0], np.int32)
    S, hnew, o, err = orc.scan_conv("gated_delta", 1, cu, xq, xk, xv, g, beta, 0.8, wq, wk, wv, act=1, l2norm=1,
                                    conv_src=hists, src_pool=pool, read_slot=rs, dst_pool=np.zeros((6, H, dk, dv)),
                                    conv_dst=np.zeros_like(hists), write_slot=ws)
    assert err == 0
    for s_ in range(4):
        st, hs = pool[rs[s_]][None].copy(), hists[rs[s_]][None].copy()
        for t in range(cu[s_], cu[s_ + 1]):
            st, hs2, ot, e = orc.step_conv("gated_delta", 1, st, xq[t:t + 1], xk[t:t + 1], xv[t:t + 1], g[t:t + 1],
                                           beta[t:t + 1], 0.8, wq, wk, wv, hs, act=1, l2norm=1)
            assert e == 0
            hs = hs2
            close(o[t], ot[0], 1e-12, f"seq {s_} token {t}")
        close(S[ws[s_]], st[0], 1e-12, f"seq {s_} final state")
        close(hnew[ws[s_]], hs[0], 1e-300, f"seq {s_} final history")


ALL_PINS = [pin_bf16_rounding, pin_brute_force_all_rules, pin_gqa_grouping, pin_exact_rational,
            pin_linear_closed_form, pin_gated_closed_form, pin_beta0_g1_identity, pin_delta_stores_value,
            pin_rearranged_readout, pin_scan_structure, pin_wide_ranges_non_expansive,
            pin_long_sequence_bounded, pin_storage_rounding_points, pin_slots, pin_pool_ops,
            pin_scan_checkpoints, pin_kda_reductions, pin_kda_wide_ranges_non_expansive, pin_query_groups,
            pin_q8_page_figures, pin_q8_codec, pin_q8_store_point, pin_conv_definition, pin_conv_fused_step,
            pin_conv_scan]
