"""Helpers of the GPU parity tests: run a workload through the C ABI (liblastate.so) and
through the CPU oracle on the same host-generated inputs, and compare."""
import numpy as np
import torch

import oracle
from gated_deltanet_recurrent_la_b200 import lastate as L

F32, BF16 = torch.float32, torch.bfloat16


def tolerances(state_dtype, io_dtype):
    """max|err| <= tol * max|ref|: 1e-4 for FP32 state (and FP32 io), 2e-2 where BF16
    storage or BF16 outputs are involved (the oracle rounds at the same points)."""
    st = 1e-4 if state_dtype == F32 else 2e-2
    o = 1e-4 if (state_dtype == F32 and io_dtype == F32) else 2e-2
    return st, o


def dname(dt):
    return {torch.float32: "f32", torch.bfloat16: "bf16", torch.float64: "f64"}[dt]


def assert_close(got, ref, tol, what):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    if ref.size == 0:
        return
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = float(np.max(np.abs(got - ref)))
    mx = float(np.max(np.abs(ref)))
    assert err <= tol * max(mx, 1e-30), f"{what}: max|err| {err:.3e} > {tol:g} * max|ref| {mx:.3e}"


def bf16_ulp_distance(got, ref):
    """Distance in BF16 units in the last place between two tensors of BF16-representable
    values (the oracle rounds to BF16 at the same points as the kernels): the bit patterns
    as sign-magnitude integers mapped onto one ordered integer line."""
    a = torch.as_tensor(np.asarray(got, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).int()
    b = torch.as_tensor(np.asarray(ref, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).int()
    oa = torch.where(a < 0, -(a & 0x7FFF), a)
    ob = torch.where(b < 0, -(b & 0x7FFF), b)
    return (oa - ob).abs()


def assert_bf16_ulps(got, ref, what, frac=0.999):
    """At least `frac` of the elements within one BF16 ulp of the oracle (the hard bound
    max|err| <= 2e-2 max|ref| is checked separately)."""
    d = bf16_ulp_distance(got, ref)
    within = float((d <= 1).double().mean()) if d.numel() else 1.0
    assert within >= frac, f"{what}: only {within:.5f} of the elements within 1 BF16 ulp (max {int(d.max())} ulp)"


def np64(t):
    return None if t is None else t.detach().cpu().double().numpy()


def dev(t):
    return None if t is None else t.cuda().contiguous()


def gpu_step(inp, *, pool_dev=None, read_slot=None, write_slot=None, guard=0):
    """One la_state_step on the device.  Returns (pool after, o, err word) on the host.
    `guard` > 0 surrounds o with sentinel elements and checks they survive."""
    pool_t = dev(inp.pool) if pool_dev is None else pool_dev
    pool = L.Pool(pool_t, inp.n_qk_heads)
    rs = dev(inp.read_slot if read_slot is None else read_slot)
    ws = dev(inp.write_slot if write_slot is None else write_slot)
    B = inp.q.shape[0]
    n = B * inp.n_v_heads * inp.d_v
    o_buf = torch.full((n + 2 * guard,), 7.0, dtype=inp.io_dtype, device="cuda")
    o = o_buf[guard:guard + n].view(B, inp.n_v_heads, inp.d_v)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = L.la_state_step(inp.rule, pool, rs, pool, ws, dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.g),
                         dev(inp.beta), inp.scale, o, err)
    L.check(st)
    torch.cuda.synchronize()
    if guard:
        assert torch.all(o_buf[:guard] == 7.0) and torch.all(o_buf[guard + n:] == 7.0), "o guard band overwritten"
    return pool_t.cpu(), o.cpu(), int(err.item())


def oracle_step(inp, pool_host=None, rows=None):
    """Oracle decode step on the requests `rows` (all by default), in dense mode on the
    gathered source tiles.  Returns (new states [len(rows), H, dk, dv], o, err)."""
    pool = inp.pool if pool_host is None else pool_host
    B = inp.q.shape[0]
    rows = np.arange(B) if rows is None else np.asarray(rows)
    rs = np.arange(B) if inp.read_slot is None else inp.read_slot.numpy()
    src = np64(pool[torch.as_tensor(rs[rows], dtype=torch.long)])
    sl = torch.as_tensor(rows, dtype=torch.long)
    new, o, err = oracle.step(inp.rule, inp.n_qk_heads, src, np64(inp.q[sl]), np64(inp.k[sl]), np64(inp.v[sl]),
                              np64(None if inp.g is None else inp.g[sl]), np64(None if inp.beta is None else inp.beta[sl]),
                              inp.scale, dst_dtype=dname(inp.state_dtype), io_dtype=dname(inp.io_dtype))
    return new, o, err


def check_step_against_oracle(inp, chunk=64, guard=16, ulps=False):
    """Full comparison of one decode step: every request's new state and output, plus
    bit-exact preservation of every slot that is not written.  ulps: BF16 states / outputs
    must also agree with the oracle to one BF16 ulp almost everywhere (the two round at the
    same points, so only values within an FP32 hair of a rounding tie may differ)."""
    before = inp.pool.clone()
    pool_after, o, err = gpu_step(inp, guard=guard)
    assert err == 0, f"device error bits {err}"
    B = inp.q.shape[0]
    ws = np.arange(B) if inp.write_slot is None else inp.write_slot.numpy()
    tol_s, tol_o = tolerances(inp.state_dtype, inp.io_dtype)
    for c0 in range(0, B, chunk):
        rows = np.arange(c0, min(B, c0 + chunk))
        new, o_ref, e = oracle_step(inp, before, rows)
        assert e == 0
        got_s = np64(pool_after[torch.as_tensor(ws[rows], dtype=torch.long)])
        got_o = np64(o[torch.as_tensor(rows, dtype=torch.long)])
        assert_close(got_s, new, tol_s, f"state rows {c0}..")
        assert_close(got_o, o_ref, tol_o, f"o rows {c0}..")
        if ulps and inp.state_dtype == BF16:
            assert_bf16_ulps(got_s, new, f"state rows {c0}..")
        if ulps and inp.io_dtype == BF16:
            assert_bf16_ulps(got_o, o_ref, f"o rows {c0}..")
    untouched = np.setdiff1d(np.arange(before.shape[0]), ws)
    ut = torch.as_tensor(untouched, dtype=torch.long)
    assert torch.equal(pool_after[ut].view(torch.int16) if before.dtype == BF16 else pool_after[ut].view(torch.int32),
                       before[ut].view(torch.int16) if before.dtype == BF16 else before[ut].view(torch.int32)), \
        "slots that are not written must stay bit-identical (checkpoints included)"
    return pool_after, o


def gpu_scan(inp, *, dst_dtype=None, seq_order=None, write_slot=None, n_dst=None, src_pool=None):
    n_seqs = inp.cu_seqlens.numel() - 1
    dst_dtype = inp.state_dtype if dst_dtype is None else dst_dtype
    dst_t = torch.full((n_dst or n_seqs, inp.n_v_heads, inp.d_k, inp.d_v), 3.0, dtype=dst_dtype, device="cuda")
    dst = L.Pool(dst_t, inp.n_qk_heads)
    src_t = dev(inp.pool if src_pool is None else src_pool)
    src = None if src_t is None else L.Pool(src_t, inp.n_qk_heads)
    T = inp.q.shape[0]
    o = torch.full((T, inp.n_v_heads, inp.d_v), 5.0, dtype=inp.io_dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = L.la_state_scan(inp.rule, src, dev(inp.read_slot), dst, dev(write_slot), dev(inp.cu_seqlens), dev(inp.q),
                         dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta), inp.scale, o, err,
                         seq_order=dev(seq_order))
    L.check(st)
    torch.cuda.synchronize()
    return dst_t.cpu(), o.cpu(), int(err.item())


def oracle_scan(inp, dst_dtype=None):
    dst_dtype = inp.state_dtype if dst_dtype is None else dst_dtype
    return oracle.scan(inp.rule, inp.n_qk_heads, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k), np64(inp.v),
                       np64(inp.g), np64(inp.beta), inp.scale, src_pool=np64(inp.pool),
                       read_slot=None if inp.read_slot is None else inp.read_slot.numpy(),
                       dst_dtype=dname(dst_dtype), io_dtype=dname(inp.io_dtype))


def gpu_step_qgroups(inp):
    """la_state_step_qgroups on the device (query-group direction)."""
    pool_t = dev(inp.pool)
    pool = L.Pool(pool_t, inp.n_qk_heads)
    B = inp.q.shape[0]
    o = torch.full((B, inp.n_q_heads, inp.d_v), 7.0, dtype=inp.io_dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = L.la_state_step_qgroups(inp.rule, pool, dev(inp.read_slot), pool, dev(inp.write_slot), dev(inp.q),
                                 dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta), inp.scale, o, err)
    L.check(st)
    torch.cuda.synchronize()
    return pool_t.cpu(), o.cpu(), int(err.item())


def oracle_step_qgroups(inp):
    """Oracle decode step in the query-group direction on the whole pool (slots as given)."""
    return oracle.step_qgroups(inp.rule, inp.n_q_heads, np64(inp.pool), np64(inp.q), np64(inp.k), np64(inp.v),
                               np64(inp.g), np64(inp.beta), inp.scale, dst_dtype=dname(inp.state_dtype),
                               io_dtype=dname(inp.io_dtype),
                               read_slot=None if inp.read_slot is None else inp.read_slot.numpy(),
                               write_slot=None if inp.write_slot is None else inp.write_slot.numpy())


def gpu_scan_qgroups(inp, dst_dtype=None):
    n_seqs = inp.cu_seqlens.numel() - 1
    dst_dtype = inp.state_dtype if dst_dtype is None else dst_dtype
    dst_t = torch.full((n_seqs, inp.n_v_heads, inp.d_k, inp.d_v), 3.0, dtype=dst_dtype, device="cuda")
    src_t = dev(inp.pool)
    src = None if src_t is None else L.Pool(src_t, inp.n_qk_heads)
    o = torch.full((inp.q.shape[0], inp.n_q_heads, inp.d_v), 5.0, dtype=inp.io_dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = L.la_state_scan_qgroups(inp.rule, src, dev(inp.read_slot), L.Pool(dst_t, inp.n_qk_heads), None,
                                 dev(inp.cu_seqlens), dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta),
                                 inp.scale, o, err)
    L.check(st)
    torch.cuda.synchronize()
    return dst_t.cpu(), o.cpu(), int(err.item())


def oracle_scan_qgroups(inp, dst_dtype=None):
    dst_dtype = inp.state_dtype if dst_dtype is None else dst_dtype
    return oracle.scan_qgroups(inp.rule, inp.n_q_heads, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k),
                               np64(inp.v), np64(inp.g), np64(inp.beta), inp.scale, src_pool=np64(inp.pool),
                               read_slot=None if inp.read_slot is None else inp.read_slot.numpy(),
                               dst_dtype=dname(dst_dtype), io_dtype=dname(inp.io_dtype))


def scan_unit_inputs(inp, picks):
    """The (sequence, head) units `picks` of a scan workload as one packed single-head input,
    each unit its own sequence (same tokens, gates and scale; zero initial state), so one
    oracle call recomputes them all."""
    cu = inp.cu_seqlens.numpy()
    ratio = inp.n_v_heads // inp.n_qk_heads
    parts = {"q": [], "k": [], "v": [], "g": [], "beta": []}
    lens = []
    for s, h in picks:
        t0, t1 = int(cu[s]), int(cu[s + 1])
        hq = h // ratio
        parts["q"].append(inp.q[t0:t1, hq:hq + 1])
        parts["k"].append(inp.k[t0:t1, hq:hq + 1])
        parts["v"].append(inp.v[t0:t1, h:h + 1])
        if inp.g is not None:
            parts["g"].append(inp.g[t0:t1, h:h + 1])
        if inp.beta is not None:
            parts["beta"].append(inp.beta[t0:t1, h:h + 1])
        lens.append(t1 - t0)
    cat = lambda xs: torch.cat(xs).contiguous() if xs else None  # noqa: E731
    cu_sub = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    from gated_deltanet_recurrent_la_b200 import workloads as W
    return W.Inputs("scan", inp.rule, 1, 1, inp.d_k, inp.d_v, inp.state_dtype, inp.io_dtype, cat(parts["q"]),
                    cat(parts["k"]), cat(parts["v"]), cat(parts["g"]), cat(parts["beta"]), inp.scale, None, None,
                    None, cu_sub)


def prefill_picks(inp, per_seq=2):
    """Every sequence on `per_seq` heads spread over the head range, and the longest sequence
    on every head."""
    cu = inp.cu_seqlens.numpy()
    n, H = len(cu) - 1, inp.n_v_heads
    picks = {(s, (s + i * H // per_seq) % H) for s in range(n) for i in range(per_seq)}
    longest = int(np.argmax(cu[1:] - cu[:-1]))
    picks |= {(longest, h) for h in range(H)}
    return sorted(picks)


def check_scan_units(inp, S, o, picks, tol_s, tol_o, batch=32, ref_fn=None):
    """Final states S [n_seqs, H, dk, dv] and outputs o [T, H, dv] of a scan against the
    oracle, unit by unit, the units recomputed `batch` at a time.  ref_fn(sub) -> (S_ref,
    o_ref) replaces the plain oracle scan (for example with the convolution ahead)."""
    cu = inp.cu_seqlens.numpy()
    for b0 in range(0, len(picks), batch):
        chunk = picks[b0:b0 + batch]
        sub = scan_unit_inputs(inp, chunk)
        if ref_fn is None:
            S_ref, o_ref, e = oracle_scan(sub)
            assert e == 0
        else:
            S_ref, o_ref = ref_fn(sub, chunk)
        ucu = sub.cu_seqlens.numpy()
        for i, (s, h) in enumerate(chunk):
            t0, t1 = int(cu[s]), int(cu[s + 1])
            assert_close(np64(S[s, h]), S_ref[i, 0], tol_s, f"seq {s} head {h} final state")
            assert_close(np64(o[t0:t1, h]), o_ref[int(ucu[i]):int(ucu[i + 1]), 0], tol_o, f"seq {s} head {h} outputs")
    assert torch.isfinite(o.float()).all() and torch.isfinite(S.float()).all()
