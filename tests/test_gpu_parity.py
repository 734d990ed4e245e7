"""GPU parity: the CUDA kernels, called through the C ABI, against the CPU oracle on the
same seeded inputs (element by element), at small sizes spanning several tiles with
ragged tails and at the full sizes of the named workloads.

Tolerances (max|err| <= tol * max|ref|, outputs and states checked separately): 1e-4
with FP32 state and io, 2e-2 where BF16 storage or BF16 io is involved; the oracle
rounds at the same points (state after each decode step, at the end of a scan; o to
the io type).  Slot operations and invariants are checked bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_recurrent_la_b200 import lastate as L
from gated_deltanet_recurrent_la_b200 import workloads as W
from gpu_helpers import (BF16, F32, assert_close, check_scan_units, check_step_against_oracle, dev, dname, gpu_scan,
                         gpu_scan_qgroups, gpu_step, gpu_step_qgroups, np64, oracle_scan, oracle_scan_qgroups,
                         oracle_step_qgroups, prefill_picks, tolerances)

pytestmark = pytest.mark.gpu

SHAPES = [(16, 16), (64, 64), (128, 64), (128, 128)]


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    L.lib()


# ---- the tiny workload: every rule, as 64 decode steps and as one scan ------------------

@pytest.mark.parametrize("rule", W.ALL_RULES)
def test_tiny_sequential_steps(rule):
    inp = W.tiny(rule)
    cu = inp.cu_seqlens.numpy()
    pool_t = torch.zeros(2, 2, 16, 16, dtype=F32, device="cuda")
    ref = np.zeros((2, 2, 16, 16))
    for t in range(64):
        rows = torch.as_tensor(cu[:-1] + t, dtype=torch.long)
        step_inp = W.Inputs("step", rule, 2, 2, 16, 16, F32, F32, inp.q[rows], inp.k[rows], inp.v[rows],
                            inp.g[rows], inp.beta[rows], 1.0, pool_t)
        after, o, err = gpu_step(step_inp, pool_dev=pool_t, guard=4)
        assert err == 0
        ref, o_ref, e = oracle.step(rule, 2, ref, np64(step_inp.q), np64(step_inp.k), np64(step_inp.v),
                                    np64(step_inp.g), np64(step_inp.beta), dst_dtype="f32", io_dtype="f32")
        assert e == 0
        assert_close(np64(after), ref, 1e-4, f"{rule} state after step {t}")
        assert_close(np64(o), o_ref, 1e-4, f"{rule} o at step {t}")


@pytest.mark.parametrize("rule", W.ALL_RULES)
def test_tiny_scan(rule):
    inp = W.tiny(rule)
    S, o, err = gpu_scan(inp)
    assert err == 0
    S_ref, o_ref, e = oracle_scan(inp)
    assert e == 0
    assert_close(np64(S), S_ref, 1e-4, f"{rule} final state")
    assert_close(np64(o), o_ref, 1e-4, f"{rule} outputs")


# ---- the full-size decode workloads ----------------------------------------------------

def test_decode64_full():
    check_step_against_oracle(W.decode64(), ulps=True)


def test_decode512_full_with_checkpoints():
    inp = W.decode512()
    rs, ws = inp.read_slot.numpy(), inp.write_slot.numpy()
    assert (rs != ws).sum() == 256 and len(set(ws)) == 512
    check_step_against_oracle(inp, ulps=True)  # also proves every checkpoint slot is bit-identical afterwards


def test_mamba2_full():
    check_step_against_oracle(W.mamba2(), ulps=True)


# ---- the full-size prefill workload ------------------------------------------------------

def test_prefill32_units():
    """The full prefill workload: every sequence on two heads and the longest on all 32
    against the oracle (94 (sequence, head) units)."""
    inp = W.prefill32()
    S, o, err = gpu_scan(inp)
    assert err == 0
    tol_s, tol_o = tolerances(inp.state_dtype, inp.io_dtype)
    check_scan_units(inp, S, o, prefill_picks(inp), tol_s, tol_o)


# ---- every rule x tile shape x dtype, small batches -----------------------------------------

@pytest.mark.parametrize("state", [F32, BF16], ids=["f32state", "bf16state"])
@pytest.mark.parametrize("io", [F32, BF16], ids=["f32io", "bf16io"])
@pytest.mark.parametrize("dk,dv", SHAPES, ids=[f"{a}x{b}" for a, b in SHAPES])
@pytest.mark.parametrize("rule", W.ALL_RULES)
def test_step_all_variants(rule, dk, dv, io, state):
    inp = W.step_inputs(B=5, n_qk_heads=2, n_v_heads=4, d_k=dk, d_v=dv, rule=rule, n_slots=11, state_dtype=state,
                        io_dtype=io, seed=dk + dv + len(rule), slot_map="perm", scale=0.9)
    check_step_against_oracle(inp)


@pytest.mark.parametrize("io", [F32, BF16], ids=["f32io", "bf16io"])
@pytest.mark.parametrize("dk,dv", SHAPES, ids=[f"{a}x{b}" for a, b in SHAPES])
@pytest.mark.parametrize("rule", W.ALL_RULES)
def test_scan_all_variants(rule, dk, dv, io):
    inp = W.scan_inputs(lengths=[3, 37, 0, 1, 16, 17], n_qk_heads=2, n_v_heads=4, d_k=dk, d_v=dv, rule=rule,
                        state_dtype=BF16, io_dtype=io, seed=7 + dk, init="slots", init_dtype=F32, scale=1.1)
    for dst in (F32, BF16):
        S, o, err = gpu_scan(inp, dst_dtype=dst)
        assert err == 0
        S_ref, o_ref, e = oracle_scan(inp, dst_dtype=dst)
        assert e == 0
        tol_s, tol_o = tolerances(dst, io)
        assert_close(np64(S), S_ref, tol_s, f"{rule} {dk}x{dv} final state ({dst})")
        assert_close(np64(o), o_ref, tol_o, f"{rule} {dk}x{dv} outputs")


def test_scan_ragged_multi_tile():
    inp = W.scan_inputs(lengths=[1, 17, 100, 0, 333, 64, 15, 2], n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128,
                        state_dtype=BF16, io_dtype=BF16, seed=21)
    S, o, err = gpu_scan(inp, dst_dtype=F32)
    assert err == 0
    S_ref, o_ref, _ = oracle_scan(inp, dst_dtype=F32)
    assert_close(np64(S), S_ref, 1e-4, "final FP32 state")
    assert_close(np64(o), o_ref, 2e-2, "BF16 outputs")


def test_scan_fp32_init_bf16_final():
    """The prefill layout with an FP32 initial state read from slots and a BF16 final state."""
    inp = W.scan_inputs(lengths=[1024, 1500, 1030], n_qk_heads=32, n_v_heads=32, d_k=128, d_v=128, seed=22,
                        init="slots", init_dtype=F32)
    S, o, err = gpu_scan(inp)
    assert err == 0
    S_ref, o_ref, _ = oracle_scan(inp)
    assert_close(np64(S), S_ref, 2e-2, "final BF16 state")
    assert_close(np64(o), o_ref, 2e-2, "outputs")


# ---- invariants and structure, bit for bit where the algebra is exact -----------------------

@pytest.mark.parametrize("state", [F32, BF16], ids=["f32", "bf16"])
@pytest.mark.parametrize("rule", ["delta", "gated_delta"])
def test_beta0_g1_leaves_state_bit_identical(rule, state):
    inp = W.step_inputs(B=6, n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128, rule=rule, n_slots=9, state_dtype=state,
                        io_dtype=BF16, g_mode="one", beta_mode="zero", slot_map="perm", seed=3)
    before = inp.pool.clone()
    after, _, err = gpu_step(inp)
    assert err == 0
    assert torch.equal(after.view(torch.int16 if state == BF16 else torch.int32),
                       before.view(torch.int16 if state == BF16 else torch.int32))
    S, _, err = gpu_scan(W.scan_inputs(lengths=[5, 9], n_qk_heads=1, n_v_heads=2, d_k=64, d_v=64, rule=rule,
                                       state_dtype=state, io_dtype=F32, g_mode="one", beta_mode="zero", init="slots",
                                       init_dtype=state, seed=4))
    assert err == 0


def test_delta_unit_key_stores_value():
    inp = W.step_inputs(B=8, n_qk_heads=4, n_v_heads=4, d_k=128, d_v=128, rule="delta", state_dtype=F32,
                        io_dtype=F32, beta_mode="one", slot_map="dense", seed=5, pool_std=1.0)
    inp.q = inp.k.clone()
    after, o, err = gpu_step(inp)
    assert err == 0
    k = np64(inp.k)
    k = k / np.linalg.norm(k, axis=-1, keepdims=True)
    stk = np.einsum("bhij,bhi->bhj", np64(after), k)
    assert_close(stk, np64(inp.v), 1e-5, "S^T k = v")
    assert_close(np64(o), np64(inp.v), 1e-5, "o = v for q = k")


def test_wide_gate_and_beta_ranges():
    """g in [-1, 1], beta in [0, 2] are not clamped (decode and scan)."""
    inp = W.step_inputs(B=7, n_qk_heads=1, n_v_heads=3, d_k=64, d_v=64, rule="gated_delta", n_slots=7,
                        state_dtype=F32, io_dtype=F32, g_mode="uniform_pm1", beta_mode="uniform_0_2", seed=8)
    check_step_against_oracle(inp)
    sc = W.scan_inputs(lengths=[40, 7], n_qk_heads=1, n_v_heads=3, d_k=64, d_v=64, state_dtype=F32, io_dtype=F32,
                       g_mode="uniform_pm1", beta_mode="uniform_0_2", seed=9, init="slots", init_dtype=F32)
    S, o, err = gpu_scan(sc)
    S_ref, o_ref, _ = oracle_scan(sc)
    assert err == 0
    assert_close(np64(S), S_ref, 1e-4, "wide-range scan state")
    assert_close(np64(o), o_ref, 1e-4, "wide-range scan outputs")


def test_gqa_heads_sharing_qk_agree_bitwise():
    inp = W.step_inputs(B=3, n_qk_heads=2, n_v_heads=8, d_k=128, d_v=128, slot_map="dense", seed=10)
    inp.v[:, 1] = inp.v[:, 0]
    inp.g[:, 1] = inp.g[:, 0]
    inp.beta[:, 1] = inp.beta[:, 0]
    inp.pool[:, 1] = inp.pool[:, 0]
    after, o, err = gpu_step(inp)
    assert err == 0
    assert torch.equal(after[:, 0], after[:, 1]) and torch.equal(o[:, 0], o[:, 1])
    assert not torch.equal(after[:, 4], after[:, 0])


def test_scan_equals_sequential_steps_fp32():
    inp = W.scan_inputs(lengths=[48, 48, 48], n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128, state_dtype=F32,
                        io_dtype=F32, seed=11)
    S_scan, o_scan, err = gpu_scan(inp)
    assert err == 0
    cu = inp.cu_seqlens.numpy()
    pool_t = torch.zeros(3, 4, 128, 128, dtype=F32, device="cuda")
    outs = torch.zeros_like(o_scan)
    for t in range(48):
        rows = torch.as_tensor(cu[:-1] + t, dtype=torch.long)
        si = W.Inputs("step", inp.rule, 2, 4, 128, 128, F32, F32, inp.q[rows], inp.k[rows], inp.v[rows],
                      inp.g[rows], inp.beta[rows], 1.0, pool_t)
        _, o, err = gpu_step(si, pool_dev=pool_t)
        assert err == 0
        outs[rows] = o
    assert_close(np64(pool_t.cpu()), np64(S_scan), 1e-4, "scan vs steps, state")
    assert_close(np64(outs), np64(o_scan), 1e-4, "scan vs steps, outputs")


def test_scan_seq_order_is_only_a_schedule():
    inp = W.scan_inputs(lengths=[30, 3, 0, 70, 12], n_qk_heads=2, n_v_heads=4, d_k=128, d_v=64, seed=12)
    S0, o0, e0 = gpu_scan(inp)
    S1, o1, e1 = gpu_scan(inp, seq_order=torch.tensor([3, 0, 4, 1, 2], dtype=torch.int32))
    assert e0 == e1 == 0
    assert torch.equal(S0, S1) and torch.equal(o0, o1)


def test_dense_past_present_equals_in_place():
    inp = W.step_inputs(B=4, n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128, slot_map="dense", seed=13)
    past = dev(inp.pool)
    present = torch.zeros_like(past)
    o = torch.empty(4, 4, 128, dtype=BF16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = L.la_state_step("gated_delta", L.Pool(past, 2), None, L.Pool(present, 2), None, dev(inp.q), dev(inp.k),
                         dev(inp.v), dev(inp.g), dev(inp.beta), 1.0, o, err)
    L.check(st)
    in_place, o2, _ = gpu_step(inp)
    torch.cuda.synchronize()
    assert torch.equal(past.cpu(), inp.pool), "past_state must not change"
    assert torch.equal(present.cpu(), in_place) and torch.equal(o.cpu(), o2)


def test_scan_write_slots_and_checkpoint_survives():
    inp = W.scan_inputs(lengths=[20, 5], n_qk_heads=1, n_v_heads=2, d_k=128, d_v=128, seed=14, init="slots",
                        init_dtype=BF16)
    ws = torch.tensor([3, 0], dtype=torch.int32)
    src = inp.pool.clone()  # slots 0, 1 hold the initial states (read_slot is a permutation of them)
    S, o, err = gpu_scan(inp, write_slot=ws, n_dst=4)
    assert err == 0
    S_ref, o_ref, _ = oracle_scan(inp)
    assert_close(np64(S[ws.long()]), S_ref, 2e-2, "final states at the write slots")
    assert torch.equal(S[1], torch.full_like(S[1], 3.0)) and torch.equal(S[2], torch.full_like(S[2], 3.0))
    assert torch.equal(inp.pool, src)


# ---- device-side error reporting (never a trap) -------------------------------------------

def test_step_bad_slots_are_skipped_and_reported():
    inp = W.step_inputs(B=6, n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128, n_slots=10, slot_map="perm", seed=15)
    good_ws = inp.write_slot.clone()
    inp.read_slot[1] = 10       # out of range
    inp.write_slot[4] = -1      # out of range
    before = inp.pool.clone()
    after, o, err = gpu_step(inp)
    assert err == (L.DEVERR_READ_SLOT | L.DEVERR_WRITE_SLOT)
    assert torch.all(o[1] == 7.0) and torch.all(o[4] == 7.0), "skipped requests leave o untouched"
    assert torch.equal(after[good_ws[1].long()], before[good_ws[1].long()])
    for b in (0, 2, 3, 5):
        sl = torch.tensor([b])
        one = W.Inputs("step", inp.rule, 2, 4, 128, 128, BF16, BF16, inp.q[sl], inp.k[sl], inp.v[sl], inp.g[sl],
                       inp.beta[sl], 1.0, before, inp.read_slot[sl], inp.write_slot[sl])
        new, o_ref, _ = oracle.step(one.rule, 2, np64(before[inp.read_slot[sl].long()]), np64(one.q), np64(one.k),
                                    np64(one.v), np64(one.g), np64(one.beta), dst_dtype="bf16", io_dtype="bf16")
        assert_close(np64(after[inp.write_slot[b].long()]), new[0], 2e-2, f"request {b}")
        assert_close(np64(o[b]), o_ref[0], 2e-2, f"request {b} o")


def test_scan_bad_cu_seqlens_and_order_reported():
    inp = W.scan_inputs(lengths=[4, 6], n_qk_heads=1, n_v_heads=2, d_k=64, d_v=64, seed=16)
    bad = inp.cu_seqlens.clone()
    bad[1] = 11  # beyond total_tokens
    inp2 = W.Inputs(**{**inp.__dict__, "cu_seqlens": bad})
    _, _, err = gpu_scan(inp2)
    assert err & L.DEVERR_CU_SEQLENS
    _, _, err = gpu_scan(inp, seq_order=torch.tensor([0, 5], dtype=torch.int32))
    assert err == L.DEVERR_CU_SEQLENS


def test_empty_calls_are_noops():
    pool_t = torch.zeros(2, 2, 64, 64, dtype=BF16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    e = torch.empty(0, 2, 64, dtype=BF16, device="cuda")
    st = L.la_state_step("gated_delta", L.Pool(pool_t, 1), None, L.Pool(pool_t, 1), None,
                         torch.empty(0, 1, 64, dtype=BF16, device="cuda"), torch.empty(0, 1, 64, dtype=BF16, device="cuda"),
                         e, torch.empty(0, 2, device="cuda"), torch.empty(0, 2, device="cuda"), 1.0, e, err)
    assert st == L.LA_OK
    st = L.la_state_scan("gated_delta", None, None, L.Pool(pool_t, 1), None, torch.zeros(1, dtype=torch.int32, device="cuda"),
                         torch.empty(0, 1, 64, dtype=BF16, device="cuda"), torch.empty(0, 1, 64, dtype=BF16, device="cuda"),
                         e, torch.empty(0, 2, device="cuda"), torch.empty(0, 2, device="cuda"), 1.0, e, err)
    assert st == L.LA_OK
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and not pool_t.any()


# ---- slot pool operations, bit for bit ---------------------------------------------------

@pytest.mark.parametrize("dtype", [F32, BF16], ids=["f32", "bf16"])
def test_pool_ops_bit_exact(dtype):
    g = torch.Generator().manual_seed(17)
    host = torch.randn(12, 4, 128, 64, generator=g).to(dtype)
    ints = torch.int16 if dtype == BF16 else torch.int32
    pool_t = host.cuda()
    pool = L.Pool(pool_t, 2)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    slots = torch.tensor([7, 2, 2, 11], dtype=torch.int32)
    dense = torch.empty(4, 4, 128, 64, dtype=dtype, device="cuda")
    L.check(L.la_state_pool_gather(pool, dev(slots), dense, err))
    ref, e = oracle.pool_gather(host.view(ints).numpy(), slots.numpy())
    assert e == 0 and np.array_equal(dense.cpu().view(ints).numpy(), ref)
    new = torch.randn(2, 4, 128, 64, generator=g).to(dtype)
    L.check(L.la_state_pool_scatter(pool, dev(torch.tensor([4, 9], dtype=torch.int32)), new.cuda(), err))
    L.check(L.la_state_pool_copy(pool, dev(torch.tensor([1, 3], dtype=torch.int32)),
                                 dev(torch.tensor([5, 0], dtype=torch.int32)), err))
    L.check(L.la_state_pool_zero(pool, dev(torch.tensor([6], dtype=torch.int32)), err))
    ref = host.view(ints).numpy().copy()
    assert oracle.pool_scatter(ref, np.array([4, 9], dtype=np.int32), new.view(ints).numpy()) == 0
    assert oracle.pool_copy(ref, np.array([1, 3], dtype=np.int32), np.array([5, 0], dtype=np.int32)) == 0
    assert oracle.pool_zero(ref, np.array([6], dtype=np.int32)) == 0
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(pool_t.cpu().view(ints).numpy(), ref)
    # out-of-range slots: skipped and reported
    L.check(L.la_state_pool_zero(pool, dev(torch.tensor([12], dtype=torch.int32)), err))
    L.check(L.la_state_pool_gather(pool, dev(torch.tensor([-3], dtype=torch.int32)), dense[:1], err))
    torch.cuda.synchronize()
    assert int(err.item()) == (L.DEVERR_READ_SLOT | L.DEVERR_WRITE_SLOT)
    assert np.array_equal(pool_t.cpu().view(ints).numpy(), ref)


def test_pool_checkpoint_roundtrip_full_size():
    """The decode64 pool: snapshot 64 live slots into checkpoint slots and back."""
    inp = W.decode64()
    pool_t = dev(inp.pool)
    pool = L.Pool(pool_t, 16)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    live = inp.write_slot
    others = torch.tensor([s for s in range(256) if s not in set(live.tolist())][:64], dtype=torch.int32)
    L.check(L.la_state_pool_copy(pool, dev(live), dev(others), err))
    torch.cuda.synchronize()
    after = pool_t.cpu()
    assert torch.equal(after[others.long()].view(torch.int16), inp.pool[live.long()].view(torch.int16))
    assert torch.equal(after[live.long()].view(torch.int16), inp.pool[live.long()].view(torch.int16))
    assert int(err.item()) == 0


# ---- scan with intermediate checkpoints ------------------------------------------------

def _ckpt_layout(lengths, every, extra_slot_base):
    n_ck = [l // every for l in lengths]
    cu = np.concatenate([[0], np.cumsum(n_ck)]).astype(np.int32)
    slots = (extra_slot_base + np.arange(cu[-1])).astype(np.int32)
    return cu, slots


def _gpu_scan_ckpt(inp, every, ckpt_cu, ckpt_slots, n_dst, dst_dtype, chunked=False):
    n_seqs = inp.cu_seqlens.numel() - 1
    dst_t = torch.full((n_dst, inp.n_v_heads, inp.d_k, inp.d_v), 3.0, dtype=dst_dtype, device="cuda")
    src = None if inp.pool is None else L.Pool(dev(inp.pool), inp.n_qk_heads)
    o = torch.full((inp.q.shape[0], inp.n_v_heads, inp.d_v), 5.0, dtype=inp.io_dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    fn = L.la_state_scan_chunked_checkpointed if chunked else L.la_state_scan_checkpointed
    st = fn(inp.rule, src, dev(inp.read_slot), L.Pool(dst_t, inp.n_qk_heads), None,
                                      dev(inp.cu_seqlens), dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.g),
                                      dev(inp.beta), inp.scale, o, every, dev(torch.as_tensor(ckpt_cu)),
                                      dev(torch.as_tensor(ckpt_slots)), err)
    L.check(st)
    torch.cuda.synchronize()
    assert n_seqs <= n_dst
    return dst_t.cpu(), o.cpu(), int(err.item())


@pytest.mark.parametrize("dst", [F32, BF16], ids=["f32", "bf16"])
@pytest.mark.parametrize("rule", W.ALL_RULES)
def test_scan_checkpoints(rule, dst):
    lengths, every = [37, 8, 0, 64, 5, 16], 8
    inp = W.scan_inputs(lengths=lengths, n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128, rule=rule, io_dtype=BF16,
                        seed=31, init="slots", init_dtype=F32)
    ckpt_cu, ckpt_slots = _ckpt_layout(lengths, every, len(lengths))
    n_dst = len(lengths) + int(ckpt_cu[-1])
    S, o, err = _gpu_scan_ckpt(inp, every, ckpt_cu, ckpt_slots, n_dst, dst)
    assert err == 0
    ref_pool = np.zeros((n_dst, 4, 128, 128))
    S_ref, o_ref, e = oracle.scan(rule, 2, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k), np64(inp.v),
                                  np64(inp.g), np64(inp.beta), inp.scale, src_pool=np64(inp.pool),
                                  read_slot=inp.read_slot.numpy(), dst_pool=ref_pool, dst_dtype=dname(dst),
                                  io_dtype="bf16", ckpt_every=every, ckpt_cu=ckpt_cu, ckpt_slots=ckpt_slots)
    assert e == 0
    tol_s, tol_o = tolerances(dst, BF16)
    assert_close(np64(S), S_ref, tol_s, f"{rule}: final states and checkpoints")
    assert_close(np64(o), o_ref, tol_o, f"{rule}: outputs (unchanged by checkpointing)")
    S_plain, o_plain, _ = gpu_scan(inp, dst_dtype=dst)
    assert torch.equal(o, o_plain), "checkpoints must not change the outputs"


def test_scan_checkpoint_errors_reported():
    lengths, every = [9, 4], 4
    inp = W.scan_inputs(lengths=lengths, n_qk_heads=1, n_v_heads=2, d_k=64, d_v=64, seed=32)
    cu = np.array([0, 3, 4], dtype=np.int32)            # sequence 0 fits only 2 checkpoints
    slots = np.array([2, 3, 4, 99], dtype=np.int32)      # slot 99 is outside the pool
    S, o, err = _gpu_scan_ckpt(inp, every, cu, slots, 5, BF16)
    assert err == (L.DEVERR_CU_SEQLENS | L.DEVERR_WRITE_SLOT)
    S_ref, _, _ = oracle.scan("gated_delta", 1, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k), np64(inp.v),
                              np64(inp.g), np64(inp.beta), dst_pool=np.zeros((5, 2, 64, 64)), dst_dtype="bf16",
                              io_dtype="bf16", ckpt_every=every, ckpt_cu=np.array([0, 2, 3], dtype=np.int32),
                              ckpt_slots=np.array([2, 3, 4], dtype=np.int32))
    assert_close(np64(S[:4]), S_ref[:4], 2e-2, "checkpoints that fit are written")


# ---- chunked tensor-core prefill (BF16 operands) -------------------------------------------
# Within a chunk the products take BF16 operands, so the chunked prefill agrees with the
# oracle to BF16 precision, not to the FP32 1e-4: over sequences of up to a few hundred
# tokens (every rule, gates and beta at the wide ranges too) its largest deviation stays
# under 1e-2 of the largest value, half the general BF16 bound of 2e-2, which the full-size
# prefill comparisons keep.
CHUNK_TOL = 1e-2

def _gpu_scan_chunked(inp, dst_dtype):
    n_seqs = inp.cu_seqlens.numel() - 1
    dst_t = torch.full((n_seqs, inp.n_v_heads, inp.d_k, inp.d_v), 3.0, dtype=dst_dtype, device="cuda")
    src = None if inp.pool is None else L.Pool(dev(inp.pool), inp.n_qk_heads)
    o = torch.full((inp.q.shape[0], inp.n_v_heads, inp.d_v), 5.0, dtype=inp.io_dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = L.la_state_scan_chunked(inp.rule, src, dev(inp.read_slot), L.Pool(dst_t, inp.n_qk_heads), None,
                                 dev(inp.cu_seqlens), dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta),
                                 inp.scale, o, err)
    L.check(st)
    torch.cuda.synchronize()
    return dst_t.cpu(), o.cpu(), int(err.item())


@pytest.mark.parametrize("dst", [F32, BF16], ids=["f32", "bf16"])
@pytest.mark.parametrize("rule", W.RULES)
def test_chunked_scan_vs_oracle(rule, dst):
    inp = W.scan_inputs(lengths=[100, 64, 1, 0, 200, 63, 129], n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128,
                        rule=rule, io_dtype=BF16, seed=41, init="slots", init_dtype=F32, scale=0.8)
    S, o, err = _gpu_scan_chunked(inp, dst)
    assert err == 0
    S_ref, o_ref, e = oracle_scan(inp, dst_dtype=dst)
    assert e == 0
    assert_close(np64(S), S_ref, CHUNK_TOL, f"{rule}: final states")
    assert_close(np64(o), o_ref, CHUNK_TOL, f"{rule}: outputs")


def test_chunked_scan_wide_gate_and_beta_ranges():
    inp = W.scan_inputs(lengths=[300, 70], n_qk_heads=1, n_v_heads=2, d_k=128, d_v=128, io_dtype=BF16, seed=42,
                        g_mode="uniform_pm1", beta_mode="uniform_0_2", init="slots", init_dtype=F32)
    S, o, err = _gpu_scan_chunked(inp, F32)
    S_ref, o_ref, _ = oracle_scan(inp, dst_dtype=F32)
    assert err == 0
    assert_close(np64(S), S_ref, CHUNK_TOL, "wide-range final states")
    assert_close(np64(o), o_ref, CHUNK_TOL, "wide-range outputs")


def _gpu_scan_chunked_ws(inp, dst_dtype):
    n_seqs = inp.cu_seqlens.numel() - 1
    dst_t = torch.full((n_seqs, inp.n_v_heads, inp.d_k, inp.d_v), 3.0, dtype=dst_dtype, device="cuda")
    src = None if inp.pool is None else L.Pool(dev(inp.pool), inp.n_qk_heads)
    o = torch.full((inp.q.shape[0], inp.n_v_heads, inp.d_v), 5.0, dtype=inp.io_dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    nbytes = max(16, L.la_scan_chunked_workspace_bytes_rule(inp.rule, inp.q.shape[0], n_seqs, inp.n_v_heads))
    ws = torch.full((nbytes,), 0xAB, dtype=torch.uint8, device="cuda")
    st = L.la_state_scan_chunked_ws(inp.rule, src, dev(inp.read_slot), L.Pool(dst_t, inp.n_qk_heads), None,
                                    dev(inp.cu_seqlens), dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.g),
                                    dev(inp.beta), inp.scale, o, ws, err)
    L.check(st)
    torch.cuda.synchronize()
    return dst_t.cpu(), o.cpu(), int(err.item())


@pytest.mark.parametrize("dst", [F32, BF16], ids=["f32", "bf16"])
@pytest.mark.parametrize("rule", W.RULES)
def test_chunked_two_launches_vs_oracle(rule, dst):
    """The two-launch form (intra-chunk inverses through the workspace, then for the delta
    rules the recurrence on tcgen05) against the oracle; the linear and gated rules take the
    fused kernel there, bit for bit.  The workspace size check is enforced for the delta
    rules."""
    inp = W.scan_inputs(lengths=[100, 64, 1, 0, 200, 63, 129], n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128,
                        rule=rule, io_dtype=BF16, seed=43, init="slots", init_dtype=F32, scale=0.8)
    S2, o2, e2 = _gpu_scan_chunked_ws(inp, dst)
    assert e2 == 0
    S_ref, o_ref, _ = oracle_scan(inp, dst_dtype=dst)
    assert_close(np64(S2), S_ref, CHUNK_TOL, f"{rule}: final states")
    assert_close(np64(o2), o_ref, CHUNK_TOL, f"{rule}: outputs")
    if rule in ("linear", "gated"):
        S1, o1, e1 = _gpu_scan_chunked(inp, dst)
        assert e1 == 0 and torch.equal(S1, S2) and torch.equal(o1, o2)
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    dst_t = torch.zeros(7, 4, 128, 128, dtype=F32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = L.la_state_scan_chunked_ws(rule, None, None, L.Pool(dst_t, 2), None, dev(inp.cu_seqlens), dev(inp.q),
                                    dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta), 1.0,
                                    torch.empty_like(dev(inp.v)), small, err)
    # the workspace exists for the delta rules' intra-chunk inverses; the other rules ignore it
    assert st == (L.LA_ERR_SHAPE if rule in ("delta", "gated_delta") else L.LA_OK)
    torch.cuda.synchronize()
    assert int(err.item()) == 0


@pytest.mark.parametrize("rule", ["delta", "gated_delta"])
def test_chunked_two_launches_special_ranges(rule):
    """Gates in [-1, 1] (negative products, ratios outside the factored range) and beta in
    [0, 2]; then beta = 0 with g = 1, which must leave the initial state as it is."""
    inp = W.scan_inputs(lengths=[300, 70, 5], n_qk_heads=1, n_v_heads=2, d_k=128, d_v=128, rule=rule,
                        io_dtype=BF16, seed=44, g_mode="uniform_pm1", beta_mode="uniform_0_2", init="slots",
                        init_dtype=F32)
    S, o, err = _gpu_scan_chunked_ws(inp, F32)
    S_ref, o_ref, _ = oracle_scan(inp, dst_dtype=F32)
    assert err == 0
    assert_close(np64(S), S_ref, CHUNK_TOL, f"{rule}: wide-range final states")
    assert_close(np64(o), o_ref, CHUNK_TOL, f"{rule}: wide-range outputs")
    inp = W.scan_inputs(lengths=[130, 64], n_qk_heads=1, n_v_heads=2, d_k=128, d_v=128, rule=rule,
                        io_dtype=BF16, seed=45, g_mode="one", beta_mode="zero", init="slots", init_dtype=F32)
    S, o, err = _gpu_scan_chunked_ws(inp, F32)
    assert err == 0
    S0 = inp.pool[inp.read_slot.long()].float()
    assert torch.equal(S, S0), "beta = 0, g = 1: the state passes through unchanged"
    S_ref, o_ref, _ = oracle_scan(inp, dst_dtype=F32)
    assert_close(np64(o), o_ref, CHUNK_TOL, f"{rule}: readout of the unchanged state")


@pytest.mark.parametrize("rule", ["delta", "gated_delta"])
def test_chunked_two_launches_all_sequences_empty(rule):
    """No tokens at all: every sequence stores its initial state (the tensor maps of the
    empty q / k / v are never used)."""
    inp = W.scan_inputs(lengths=[0, 0, 0], n_qk_heads=1, n_v_heads=2, d_k=128, d_v=128, rule=rule,
                        io_dtype=BF16, seed=46, init="slots", init_dtype=F32)
    S, o, err = _gpu_scan_chunked_ws(inp, F32)
    assert err == 0 and o.numel() == 0
    assert torch.equal(S, inp.pool[inp.read_slot.long()].float())


def test_chunked_two_launches_pool_slots_and_order():
    """Write slots into a larger pool (other slots untouched), a seq_order that reverses the
    sequences, BF16 final states: the pool semantics of the two-launch path."""
    inp = W.scan_inputs(lengths=[90, 200, 3, 64], n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128, io_dtype=BF16,
                        seed=47, init="slots", init_dtype=F32)
    n_seqs = 4
    dst_t = torch.full((9, 4, 128, 128), 3.0, dtype=BF16, device="cuda")
    write = torch.tensor([7, 2, 5, 0], dtype=torch.int32)
    o = torch.full((inp.q.shape[0], 4, 128), 5.0, dtype=BF16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(L.la_scan_chunked_workspace_bytes(inp.q.shape[0], n_seqs, 4), dtype=torch.uint8, device="cuda")
    st = L.la_state_scan_chunked_ws(inp.rule, L.Pool(dev(inp.pool), 2), dev(inp.read_slot), L.Pool(dst_t, 2),
                                    dev(write), dev(inp.cu_seqlens), dev(inp.q), dev(inp.k), dev(inp.v),
                                    dev(inp.g), dev(inp.beta), inp.scale, o, ws, err,
                                    seq_order=torch.tensor([3, 2, 1, 0], dtype=torch.int32, device="cuda"))
    L.check(st)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    S_ref, o_ref, _ = oracle_scan(inp, dst_dtype=BF16)
    got = dst_t.cpu()
    for s in range(n_seqs):
        assert_close(np64(got[int(write[s])]), S_ref[s], CHUNK_TOL, f"sequence {s} state in slot {int(write[s])}")
    untouched = [i for i in range(9) if i not in write.tolist()]
    assert torch.all(got[untouched] == 3.0)
    assert_close(np64(o.cpu()), o_ref, CHUNK_TOL, "outputs")


def test_chunked_two_launches_prefill32_units():
    """The full prefill workload through the two-launch path, as the benchmark runs it:
    every sequence on two heads and the longest on all 32 against the oracle."""
    inp = W.prefill32()
    S, o, err = _gpu_scan_chunked_ws(inp, BF16)
    assert err == 0
    check_scan_units(inp, S, o, prefill_picks(inp), 2e-2, 2e-2)


def test_chunked_prefill32_units():
    """The full prefill workload through the one-launch chunked prefill: every sequence on
    two heads and the longest on all 32 against the oracle."""
    inp = W.prefill32()
    S, o, err = _gpu_scan_chunked(inp, BF16)
    assert err == 0
    check_scan_units(inp, S, o, prefill_picks(inp), 2e-2, 2e-2)


@pytest.mark.parametrize("dst", [F32, BF16], ids=["f32", "bf16"])
@pytest.mark.parametrize("rule", W.RULES)
def test_chunked_checkpoints(rule, dst):
    """Prefix-cache checkpoints from the one-launch chunked prefill, every 128 tokens (chunk
    boundaries): every checkpoint and final state against the oracle's checkpointed scan at
    the BF16-operand tolerance; the outputs and final states are those of the plain chunked
    call, bit for bit (a checkpoint is a store of the state the recurrence already holds)."""
    lengths, every = [300, 64, 0, 129, 256, 5, 640], 128
    inp = W.scan_inputs(lengths=lengths, n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128, rule=rule, io_dtype=BF16,
                        seed=33, init="slots", init_dtype=F32, scale=0.8)
    ckpt_cu, ckpt_slots = _ckpt_layout(lengths, every, len(lengths))
    n_dst = len(lengths) + int(ckpt_cu[-1])
    S, o, err = _gpu_scan_ckpt(inp, every, ckpt_cu, ckpt_slots, n_dst, dst, chunked=True)
    assert err == 0
    S_ref, o_ref, e = oracle.scan(rule, 2, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k), np64(inp.v),
                                  np64(inp.g), np64(inp.beta), inp.scale, src_pool=np64(inp.pool),
                                  read_slot=inp.read_slot.numpy(), dst_pool=np.zeros((n_dst, 4, 128, 128)),
                                  dst_dtype=dname(dst), io_dtype="bf16", ckpt_every=every, ckpt_cu=ckpt_cu,
                                  ckpt_slots=ckpt_slots)
    assert e == 0
    assert_close(np64(S), S_ref, CHUNK_TOL, f"{rule}: final states and checkpoints")
    assert_close(np64(o), o_ref, CHUNK_TOL, f"{rule}: outputs")
    S1, o1, e1 = _gpu_scan_chunked(inp, dst)
    assert e1 == 0 and torch.equal(o, o1) and torch.equal(S[:len(lengths)], S1)


def test_chunked_checkpoints_supported_set_and_errors():
    """ckpt_every off the chunk grid is refused on the host; too many checkpoints for a
    sequence and a slot outside the pool are reported on the device, the others written."""
    lengths = [256, 130]
    inp = W.scan_inputs(lengths=lengths, n_qk_heads=1, n_v_heads=2, d_k=128, d_v=128, io_dtype=BF16, seed=34)
    with pytest.raises(L.LAError) as ei:
        _gpu_scan_ckpt(inp, 100, np.array([0, 2, 3], np.int32), np.array([2, 3, 4], np.int32), 5, BF16, chunked=True)
    assert ei.value.status == L.LA_ERR_UNSUPPORTED
    cu = np.array([0, 3, 4], dtype=np.int32)            # sequence 0 fits only 2 checkpoints of 128
    slots = np.array([2, 3, 4, 99], dtype=np.int32)      # slot 99 is outside the pool
    S, o, err = _gpu_scan_ckpt(inp, 128, cu, slots, 5, BF16, chunked=True)
    assert err == (L.DEVERR_CU_SEQLENS | L.DEVERR_WRITE_SLOT)
    S_ref, _, _ = oracle.scan("gated_delta", 1, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k), np64(inp.v),
                              np64(inp.g), np64(inp.beta), dst_pool=np.zeros((5, 2, 128, 128)), dst_dtype="bf16",
                              io_dtype="bf16", ckpt_every=128, ckpt_cu=np.array([0, 2, 3], dtype=np.int32),
                              ckpt_slots=np.array([2, 3, 4], dtype=np.int32))
    assert_close(np64(S[:4]), S_ref[:4], 2e-2, "checkpoints that fit are written")


# ---- channel-wise gate (kda): the full-size workloads, special cases, the supported set ----

def test_kda_decode64_full():
    check_step_against_oracle(W.kda_decode64())


def test_kda_prefill32_units():
    inp = W.kda_prefill32()
    S, o, err = gpu_scan(inp)
    assert err == 0
    tol_s, tol_o = tolerances(inp.state_dtype, inp.io_dtype)
    check_scan_units(inp, S, o, prefill_picks(inp), tol_s, tol_o)


def test_kda_wide_gate_and_beta_ranges():
    """alpha in [-1, 1] per channel and beta in [0, 2] are not clamped (decode and scan)."""
    inp = W.step_inputs(B=7, n_qk_heads=1, n_v_heads=3, d_k=128, d_v=64, rule="kda", n_slots=7, state_dtype=F32,
                        io_dtype=F32, g_mode="uniform_pm1", beta_mode="uniform_0_2", seed=51)
    check_step_against_oracle(inp)
    sc = W.scan_inputs(lengths=[60, 9], n_qk_heads=1, n_v_heads=3, d_k=64, d_v=64, rule="kda", state_dtype=F32,
                       io_dtype=F32, g_mode="uniform_pm1", beta_mode="uniform_0_2", seed=52, init="slots",
                       init_dtype=F32)
    S, o, err = gpu_scan(sc)
    S_ref, o_ref, _ = oracle_scan(sc)
    assert err == 0
    assert_close(np64(S), S_ref, 1e-4, "kda wide-range scan state")
    assert_close(np64(o), o_ref, 1e-4, "kda wide-range scan outputs")


def test_kda_equal_channels_matches_gated_delta():
    """Every channel decaying by the same g: the kda kernels (decode and scan) agree with the
    gated_delta kernels, a different code path, to FP32 precision."""
    sc = W.scan_inputs(lengths=[33, 70], n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128, rule="gated_delta",
                       state_dtype=F32, io_dtype=F32, seed=53, init="slots", init_dtype=F32)
    kda = W.Inputs(**{**sc.__dict__, "rule": "kda", "g": sc.g[:, :, None].expand(-1, -1, 128).contiguous()})
    S0, o0, e0 = gpu_scan(sc)
    S1, o1, e1 = gpu_scan(kda)
    assert e0 == e1 == 0
    assert_close(np64(S1), np64(S0), 1e-4, "scan state")
    assert_close(np64(o1), np64(o0), 1e-4, "scan outputs")
    st = W.step_inputs(B=6, n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128, rule="gated_delta", n_slots=9,
                       state_dtype=F32, io_dtype=F32, seed=54)
    st_kda = W.Inputs(**{**st.__dict__, "rule": "kda", "g": st.g[:, :, None].expand(-1, -1, 128).contiguous()})
    a0, p0, e0 = gpu_step(st)
    a1, p1, e1 = gpu_step(st_kda)
    assert e0 == e1 == 0
    assert_close(np64(a1), np64(a0), 1e-4, "step state")
    assert_close(np64(p1), np64(p0), 1e-4, "step outputs")


def test_kda_checkpointed_scan_and_chunked_refusal():
    lengths, every = [19, 40, 3], 8
    inp = W.scan_inputs(lengths=lengths, n_qk_heads=1, n_v_heads=2, d_k=128, d_v=128, rule="kda", io_dtype=BF16,
                        seed=55, init="slots", init_dtype=F32)
    ckpt_cu, ckpt_slots = _ckpt_layout(lengths, every, len(lengths))
    n_dst = len(lengths) + int(ckpt_cu[-1])
    S, o, err = _gpu_scan_ckpt(inp, every, ckpt_cu, ckpt_slots, n_dst, F32)
    assert err == 0
    S_ref, o_ref, e = oracle.scan("kda", 1, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k), np64(inp.v),
                                  np64(inp.g), np64(inp.beta), inp.scale, src_pool=np64(inp.pool),
                                  read_slot=inp.read_slot.numpy(), dst_pool=np.zeros((n_dst, 2, 128, 128)),
                                  dst_dtype="f32", io_dtype="bf16", ckpt_every=every, ckpt_cu=ckpt_cu,
                                  ckpt_slots=ckpt_slots)
    assert e == 0
    assert_close(np64(S), S_ref, 1e-4, "kda checkpoints and final states")
    assert_close(np64(o), o_ref, 2e-2, "kda outputs")
    with pytest.raises(L.LAError):
        _gpu_scan_chunked(inp, F32)


# ---- query-group direction (ONNX: query heads sharing a KV head and its state) ---------------

@pytest.mark.parametrize("group", [1, 2, 4, 8])
@pytest.mark.parametrize("state,io", [(F32, F32), (BF16, BF16), (BF16, F32)], ids=["f32", "bf16", "bf16state"])
@pytest.mark.parametrize("dk,dv", [(16, 16), (128, 64), (128, 128)], ids=["16x16", "128x64", "128x128"])
@pytest.mark.parametrize("rule", ["linear", "gated_delta", "kda"])
def test_qgroups_step(rule, dk, dv, state, io, group):
    inp = W.step_inputs(B=5, n_qk_heads=3, n_v_heads=3, d_k=dk, d_v=dv, rule=rule, n_slots=9, state_dtype=state,
                        io_dtype=io, seed=60 + group, slot_map="perm", scale=0.9, n_q_heads=3 * group)
    after, o, err = gpu_step_qgroups(inp)
    assert err == 0
    ref_pool, o_ref, e = oracle_step_qgroups(inp)
    assert e == 0
    tol_s, tol_o = tolerances(state, io)
    assert_close(np64(after), ref_pool, tol_s, f"{rule} group {group}: pool after the step")
    assert_close(np64(o), o_ref, tol_o, f"{rule} group {group}: outputs")


@pytest.mark.parametrize("group", [2, 8])
@pytest.mark.parametrize("io", [F32, BF16], ids=["f32io", "bf16io"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128)], ids=["64x64", "128x128"])
@pytest.mark.parametrize("rule", ["gated", "gated_delta", "kda"])
def test_qgroups_scan(rule, dk, dv, io, group):
    inp = W.scan_inputs(lengths=[3, 21, 0, 9], n_qk_heads=2, n_v_heads=2, d_k=dk, d_v=dv, rule=rule, state_dtype=BF16,
                        io_dtype=io, seed=70 + group, init="slots", init_dtype=F32, scale=1.1, n_q_heads=2 * group)
    for dst in (F32, BF16):
        S, o, err = gpu_scan_qgroups(inp, dst)
        assert err == 0
        S_ref, o_ref, e = oracle_scan_qgroups(inp, dst)
        assert e == 0
        tol_s, tol_o = tolerances(dst, io)
        assert_close(np64(S), S_ref, tol_s, f"{rule} group {group}: final states ({dst})")
        assert_close(np64(o), o_ref, tol_o, f"{rule} group {group}: outputs")


def test_qgroups_first_query_matches_default_direction_bitwise():
    """With one query per state head the query-group kernels give the default kernels' bits."""
    st = W.step_inputs(B=4, n_qk_heads=4, n_v_heads=4, d_k=128, d_v=128, seed=80, slot_map="perm", n_slots=6,
                       n_q_heads=4)
    a0, o0, e0 = gpu_step(st)
    a1, o1, e1 = gpu_step_qgroups(st)
    assert e0 == e1 == 0 and torch.equal(a0, a1) and torch.equal(o0, o1)
    sc = W.scan_inputs(lengths=[40, 17], n_qk_heads=2, n_v_heads=2, d_k=128, d_v=128, seed=81, n_q_heads=2)
    S0, o0, e0 = gpu_scan(sc)
    S1, o1, e1 = gpu_scan_qgroups(sc)
    assert e0 == e1 == 0 and torch.equal(S0, S1) and torch.equal(o0, o1)


def test_qgroups_decode_full():
    check = W.qgroup_decode256()
    after, o, err = gpu_step_qgroups(check)
    assert err == 0
    rows = torch.arange(0, 256, 37)  # sampled requests recomputed by the oracle (dense, gathered tiles)
    sub = W.Inputs(**{**check.__dict__, "q": check.q[rows], "k": check.k[rows], "v": check.v[rows],
                      "g": check.g[rows], "beta": check.beta[rows], "pool": check.pool[check.read_slot[rows].long()],
                      "read_slot": None, "write_slot": None})
    ref_states, o_ref, e = oracle_step_qgroups(sub)
    assert e == 0
    ws = check.write_slot[rows].long()
    assert_close(np64(after[ws]), ref_states, 2e-2, "sampled states")
    assert_close(np64(o[rows]), o_ref, 2e-2, "sampled outputs")
    untouched = np.setdiff1d(np.arange(check.pool.shape[0]), check.write_slot.numpy())
    assert torch.equal(after[untouched].view(torch.int16), check.pool[untouched].view(torch.int16))
