"""GPU parity of the mixed INT8 / BF16 (q8) state storage: the codec bit for bit against the
oracle's (codes decided in FP32 on both sides from the same FP32 values), and the decode
step and scans on q8 pools against the oracle at the BF16 tolerance (2e-2 * max|ref|; a
code may differ by one step, at most 1/127 of its group's largest magnitude, where the
two sides' FP32 states differ by rounding)."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_recurrent_la_b200 import lastate as L
from gated_deltanet_recurrent_la_b200 import workloads as W
from gpu_helpers import BF16, F32, assert_close, dev, dname, np64, tolerances

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    L.lib()


def masks_of(H, dk, n_hp, seed):
    return W.hp_masks(H, dk, n_hp, torch.Generator().manual_seed(seed))


def u32(mask):
    return mask.numpy().view(np.uint32)


def q8_pool(values, n_qk, n_hp, mask):
    """A q8 pool on the device holding `values` (float32 [n, H, dk, dv]) through the
    library's encoder; returns (pool, tensor)."""
    n, H, dk, dv = values.shape
    t = torch.zeros(n, H, L.q8_tile_bytes(dk, dv, n_hp), dtype=torch.uint8, device="cuda")
    pool = L.Pool.q8(t, n_qk, dk, dv, n_hp, mask.cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(L.la_state_pool_encode(pool, torch.arange(n, dtype=torch.int32, device="cuda"),
                                   values.float().cuda().contiguous(), err))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return pool, t


def test_codec_bit_exact():
    for (dk, dv, n_hp) in [(128, 128, 16), (128, 64, 0), (64, 64, 16), (128, 128, 32)]:
        g = torch.Generator().manual_seed(dk + dv + n_hp)
        H = 3
        x = torch.randn(5, H, dk, dv, generator=g) * 10.0 ** torch.randint(-5, 5, (5, H, dk, 1), generator=g)
        x[0, 0, :, :32] = 0.0
        x[1, 1, 3, 5] = 1e30
        mask = masks_of(H, dk, n_hp, dk + n_hp)
        pool, t = q8_pool(x, 1, n_hp, mask)
        ref = oracle.q8_encode(x.numpy(), n_hp, u32(mask))
        got = t.cpu().numpy()
        assert np.array_equal(got, ref), f"{dk}x{dv} n_hp {n_hp}: encoded bytes differ at {np.argwhere(got != ref)[:4]}"
        dense = torch.empty(5, H, dk, dv, dtype=torch.float32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        L.check(L.la_state_pool_decode(pool, torch.tensor([4, 0, 2, 1, 3], dtype=torch.int32, device="cuda"), dense,
                                       err))
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        back = oracle.q8_decode(ref, dk, dv, n_hp, u32(mask))[[4, 0, 2, 1, 3]]
        assert np.array_equal(dense.cpu().numpy().view(np.uint32), back.view(np.uint32)), "decoded values"


def test_codec_bad_slot_and_mask_reported():
    x = torch.randn(2, 2, 64, 64)
    mask = masks_of(2, 64, 8, 1)
    pool, t = q8_pool(x, 1, 8, mask)
    before = t.clone()
    bad = mask.clone()
    bad[1, 0] ^= 1  # head 1 now marks 7 or 9 rows
    badpool = L.Pool.q8(t, 1, 64, 64, 8, bad.cuda())
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(L.la_state_pool_encode(badpool, torch.tensor([0, 7], dtype=torch.int32, device="cuda"),
                                   torch.zeros(2, 2, 64, 64, device="cuda"), err))
    torch.cuda.synchronize()
    assert int(err.item()) == (L.DEVERR_Q8_MASK | L.DEVERR_WRITE_SLOT)
    # slot 0 head 0 was re-encoded (zeros); head 1 (bad mask) and slot 1 untouched
    assert torch.equal(t[1], before[1]) and torch.equal(t[0, 1], before[0, 1])
    assert int(t[0, 0].sum()) == 0


def _values_of(t, dk, dv, n_hp, mask):
    return oracle.q8_decode(t.cpu().numpy(), dk, dv, n_hp, u32(mask)).astype(np.float64)


@pytest.mark.parametrize("io", [F32, BF16], ids=["f32io", "bf16io"])
@pytest.mark.parametrize("dk,dv,n_hp", [(64, 64, 8), (64, 64, 6), (128, 64, 0), (128, 128, 16), (128, 128, 32),
                                        (128, 128, 2)],
                         ids=["64x64", "64x64hp6", "128x64", "128x128", "128x128hp32", "128x128hp2"])
@pytest.mark.parametrize("rule", ["gated", "gated_delta", "kda"])
def test_step_q8(rule, dk, dv, n_hp, io):
    inp = W.step_inputs(B=5, n_qk_heads=2, n_v_heads=4, d_k=dk, d_v=dv, rule=rule, n_slots=9, state_dtype=F32,
                        io_dtype=io, seed=90 + dk + n_hp, slot_map="perm", pool_std=0.3)
    mask = masks_of(4, dk, n_hp, 3)
    pool, t = q8_pool(inp.pool, 2, n_hp, mask)
    before = t.cpu()
    src_vals = _values_of(before, dk, dv, n_hp, mask)  # what the pool holds
    o = torch.empty(5, 4, dv, dtype=io, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(L.la_state_step(rule, pool, dev(inp.read_slot), pool, dev(inp.write_slot), dev(inp.q), dev(inp.k),
                            dev(inp.v), dev(inp.g), dev(inp.beta), inp.scale, o, err))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref, o_ref, e = oracle.step_q8(rule, 2, src_vals, np64(inp.q), np64(inp.k), np64(inp.v), np64(inp.g),
                                   np64(inp.beta), inp.scale, masks=u32(mask), io_dtype=dname(io),
                                   read_slot=inp.read_slot.numpy(), write_slot=inp.write_slot.numpy())
    assert e == 0
    after = t.cpu()
    ws = inp.write_slot.numpy()
    assert_close(_values_of(after, dk, dv, n_hp, mask)[ws], ref[ws], 2e-2, f"{rule}: q8 states")
    assert_close(np64(o.cpu()), o_ref, 1e-4 if io == F32 else 2e-2, f"{rule}: outputs")
    untouched = np.setdiff1d(np.arange(9), ws)
    assert torch.equal(after[untouched], before[untouched]), "slots not written keep their bytes"


@pytest.mark.parametrize("dst_mask_kind", ["copy", "other"])
@pytest.mark.parametrize("rule", ["gated_delta", "kda"])
def test_step_q8_separate_mask_arrays(rule, dst_mask_kind):
    """Source and destination with their own mask arrays (the kernel that locates rows
    through each mask): a copy of the source's mask on the same pool, or a second pool with
    another mask, against the oracle (source decoded through its mask, destination encoded
    through its own)."""
    dk, dv, n_hp, n_slots = 128, 128, 16, 9
    inp = W.step_inputs(B=5, n_qk_heads=2, n_v_heads=4, d_k=dk, d_v=dv, rule=rule, n_slots=n_slots,
                        state_dtype=F32, io_dtype=BF16, seed=131, slot_map="perm", pool_std=0.3)
    mask = masks_of(4, dk, n_hp, 11)
    pool, t = q8_pool(inp.pool, 2, n_hp, mask)
    src_vals = _values_of(t, dk, dv, n_hp, mask)
    if dst_mask_kind == "copy":
        dmask, dt = mask.clone(), t
        dst = L.Pool.q8(t, 2, dk, dv, n_hp, dmask.cuda())
    else:
        dmask = masks_of(4, dk, n_hp, 12)
        dt = torch.zeros_like(t)
        dst = L.Pool.q8(dt, 2, dk, dv, n_hp, dmask.cuda())
    assert dst.mask.data_ptr() != pool.mask.data_ptr()
    o = torch.empty(5, 4, dv, dtype=BF16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(L.la_state_step(rule, pool, dev(inp.read_slot), dst, dev(inp.write_slot), dev(inp.q), dev(inp.k),
                            dev(inp.v), dev(inp.g), dev(inp.beta), inp.scale, o, err))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref, o_ref, e = oracle.step_q8(rule, 2, src_vals, np64(inp.q), np64(inp.k), np64(inp.v), np64(inp.g),
                                   np64(inp.beta), inp.scale, masks=u32(dmask), io_dtype="bf16",
                                   read_slot=inp.read_slot.numpy(), write_slot=inp.write_slot.numpy())
    assert e == 0
    ws = inp.write_slot.numpy()
    assert_close(_values_of(dt, dk, dv, n_hp, dmask)[ws], ref[ws], 2e-2, f"{rule}: q8 states ({dst_mask_kind})")
    assert_close(np64(o.cpu()), o_ref, 2e-2, f"{rule}: outputs ({dst_mask_kind})")


def test_step_q8_nonfinite_group_takes_the_codec():
    """An infinite value input makes every row's group of that column infinite: the codec
    gives such a group the scale inf and all codes 0 (the infinite value's code is that of
    NaN), while the other groups of the same rows stay finite and match the oracle."""
    dk, dv, n_hp = 128, 128, 16
    inp = W.step_inputs(B=2, n_qk_heads=1, n_v_heads=1, d_k=dk, d_v=dv, rule="gated_delta", n_slots=2,
                        state_dtype=F32, io_dtype=F32, seed=132, slot_map="perm", pool_std=0.3)
    inp.v[0, 0, 37] = float("inf")       # column 37: group 1 of request 0
    mask = masks_of(1, dk, n_hp, 13)
    pool, t = q8_pool(inp.pool, 1, n_hp, mask)
    src_vals = _values_of(t, dk, dv, n_hp, mask)
    o = torch.empty(2, 1, dv, dtype=F32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(L.la_state_step("gated_delta", pool, dev(inp.read_slot), pool, dev(inp.write_slot), dev(inp.q),
                            dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta), 1.0, o, err))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    n8 = dk - n_hp
    tile = t.cpu()[int(inp.write_slot[0]), 0].numpy()
    codes = tile[:n8 * dv].view(np.int8).reshape(n8, dv)
    scales = tile[n8 * dv:n8 * dv + n8 * 4 * 4].view(np.float32).reshape(n8, 4)
    assert np.all(codes[:, 32:64] == 0) and np.all(np.isinf(scales[:, 1]))
    assert np.all(np.isfinite(scales[:, [0, 2, 3]]))
    ref, _, _ = oracle.step_q8("gated_delta", 1, src_vals, np64(inp.q), np64(inp.k), np64(inp.v), np64(inp.g),
                               np64(inp.beta), 1.0, masks=u32(mask), io_dtype="f32",
                               read_slot=inp.read_slot.numpy(), write_slot=inp.write_slot.numpy())
    got = _values_of(t, dk, dv, n_hp, mask)
    w0, w1 = int(inp.write_slot[0]), int(inp.write_slot[1])
    finite_cols = np.r_[0:32, 64:128]
    assert_close(got[w0][:, :, finite_cols], ref[w0][:, :, finite_cols], 2e-2, "finite groups of request 0")
    assert_close(got[w1], ref[w1], 2e-2, "request 1")


@pytest.mark.parametrize("src_kind,dst_kind", [("q8", "q8"), ("f32", "q8"), ("q8", "bf16")])
@pytest.mark.parametrize("rule", ["gated_delta", "kda"])
def test_scan_q8(rule, src_kind, dst_kind):
    dk, dv, n_hp = 128, 128, 16
    lengths = [37, 0, 5, 70]
    inp = W.scan_inputs(lengths=lengths, n_qk_heads=2, n_v_heads=2, d_k=dk, d_v=dv, rule=rule, state_dtype=BF16,
                        io_dtype=BF16, seed=95, init="slots", init_dtype=F32, pool_std=0.3)
    mask = masks_of(2, dk, n_hp, 4)
    if src_kind == "q8":
        src, st = q8_pool(inp.pool, 2, n_hp, mask)
        src_vals = _values_of(st, dk, dv, n_hp, mask)
    else:
        src = L.Pool(dev(inp.pool), 2)
        src_vals = np64(inp.pool)
    n = len(lengths)
    if dst_kind == "q8":
        dt = torch.zeros(n, 2, L.q8_tile_bytes(dk, dv, n_hp), dtype=torch.uint8, device="cuda")
        dst = L.Pool.q8(dt, 2, dk, dv, n_hp, mask.cuda())
    else:
        dt = torch.zeros(n, 2, dk, dv, dtype=BF16, device="cuda")
        dst = L.Pool(dt, 2)
    o = torch.empty(inp.q.shape[0], 2, dv, dtype=BF16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(L.la_state_scan(rule, src, dev(inp.read_slot), dst, None, dev(inp.cu_seqlens), dev(inp.q), dev(inp.k),
                            dev(inp.v), dev(inp.g), dev(inp.beta), inp.scale, o, err))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    args = (rule, 2, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k), np64(inp.v), np64(inp.g), np64(inp.beta),
            inp.scale)
    kw = dict(src_pool=src_vals, read_slot=inp.read_slot.numpy(), io_dtype="bf16")
    if dst_kind == "q8":
        ref, o_ref, e = oracle.scan_q8(*args, masks=u32(mask), **kw)
        got = _values_of(dt, dk, dv, n_hp, mask)
    else:
        ref, o_ref, e = oracle.scan(*args, dst_dtype="bf16", **kw)
        got = np64(dt.cpu())
    assert e == 0
    assert_close(got, ref, 2e-2, f"{rule} {src_kind}->{dst_kind}: final states")
    assert_close(np64(o.cpu()), o_ref, 2e-2, f"{rule} {src_kind}->{dst_kind}: outputs")


def test_step_q8_bad_mask_skips_and_reports():
    inp = W.step_inputs(B=3, n_qk_heads=1, n_v_heads=2, d_k=64, d_v=64, n_slots=4, state_dtype=F32, seed=97,
                        slot_map="perm")
    mask = masks_of(2, 64, 8, 5)
    pool, t = q8_pool(inp.pool, 1, 8, mask)
    before = t.clone()
    bad = mask.clone()
    bad[0, 1] = 0 if int(bad[0, 1]) != 0 else 1
    badpool = L.Pool.q8(t, 1, 64, 64, 8, bad.cuda())
    o = torch.full((3, 2, 64), 7.0, dtype=BF16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(L.la_state_step("gated_delta", badpool, dev(inp.read_slot), badpool, dev(inp.write_slot), dev(inp.q),
                            dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta), 1.0, o, err))
    torch.cuda.synchronize()
    assert int(err.item()) & L.DEVERR_Q8_MASK
    assert torch.equal(t[:, 0], before[:, 0]), "head 0 (bad mask) is skipped"
    assert torch.all(o[:, 0].float() == 7.0)
    assert not torch.equal(t[inp.write_slot.long(), 1], before[inp.write_slot.long(), 1]), "head 1 is updated"


def test_q8_decode64_full():
    inp = W.q8_decode64()
    n_hp, mask = inp.extra["n_hp"], inp.extra["hp_mask"]
    pool, t = q8_pool(inp.pool, 16, n_hp, mask)
    before = t.cpu()
    ref_bytes = oracle.q8_encode(inp.pool.numpy(), n_hp, u32(mask))
    assert np.array_equal(before.numpy(), ref_bytes), "full-size pool encodes bit for bit"
    o = torch.empty(64, 32, 128, dtype=BF16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(L.la_state_step("gated_delta", pool, dev(inp.read_slot), pool, dev(inp.write_slot), dev(inp.q),
                            dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta), 1.0, o, err))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rows = np.arange(0, 64, 9)
    rs, ws = inp.read_slot.numpy()[rows], inp.write_slot.numpy()[rows]
    src_vals = oracle.q8_decode(ref_bytes[rs], 128, 128, n_hp, u32(mask)).astype(np.float64)
    sl = torch.as_tensor(rows)
    ref, o_ref, e = oracle.step_q8("gated_delta", 16, src_vals, np64(inp.q[sl]), np64(inp.k[sl]), np64(inp.v[sl]),
                                   np64(inp.g[sl]), np64(inp.beta[sl]), 1.0, masks=u32(mask), io_dtype="bf16")
    assert e == 0
    after = t.cpu()
    assert_close(_values_of(after[torch.as_tensor(ws)], 128, 128, n_hp, mask), ref, 2e-2, "sampled q8 states")
    assert_close(np64(o.cpu()[sl]), o_ref, 2e-2, "sampled outputs")
    untouched = np.setdiff1d(np.arange(256), inp.write_slot.numpy())
    assert torch.equal(after[untouched], before[untouched])


# ---- q8 pools on the chunked prefill (one launch; BF16 operands inside the chunks, so the
#      states are compared at the chunked prefill's tolerance) ---------------------------

@pytest.mark.parametrize("src_kind,dst_kind", [("q8", "q8"), ("f32", "q8"), ("q8", "bf16"), ("q8", "f32")])
@pytest.mark.parametrize("rule", ["linear", "gated_delta"])
def test_chunked_scan_q8(rule, src_kind, dst_kind):
    dk, dv, n_hp = 128, 128, 16
    lengths = [37, 0, 130, 64]
    inp = W.scan_inputs(lengths=lengths, n_qk_heads=2, n_v_heads=2, d_k=dk, d_v=dv, rule=rule, state_dtype=BF16,
                        io_dtype=BF16, seed=96, init="slots", init_dtype=F32, pool_std=0.3)
    mask = masks_of(2, dk, n_hp, 6)
    if src_kind == "q8":
        src, st = q8_pool(inp.pool, 2, n_hp, mask)
        src_vals = _values_of(st, dk, dv, n_hp, mask)
    else:
        src = L.Pool(dev(inp.pool), 2)
        src_vals = np64(inp.pool)
    n = len(lengths)
    if dst_kind == "q8":
        dt = torch.zeros(n, 2, L.q8_tile_bytes(dk, dv, n_hp), dtype=torch.uint8, device="cuda")
        dst = L.Pool.q8(dt, 2, dk, dv, n_hp, mask.cuda())
    else:
        dt = torch.zeros(n, 2, dk, dv, dtype=BF16 if dst_kind == "bf16" else F32, device="cuda")
        dst = L.Pool(dt, 2)
    o = torch.empty(inp.q.shape[0], 2, dv, dtype=BF16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(L.la_state_scan_chunked(rule, src, dev(inp.read_slot), dst, None, dev(inp.cu_seqlens), dev(inp.q),
                                    dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta), inp.scale, o, err))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    args = (rule, 2, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k), np64(inp.v), np64(inp.g), np64(inp.beta),
            inp.scale)
    kw = dict(src_pool=src_vals, read_slot=inp.read_slot.numpy(), io_dtype="bf16")
    if dst_kind == "q8":
        ref, o_ref, e = oracle.scan_q8(*args, masks=u32(mask), **kw)
        got = _values_of(dt, dk, dv, n_hp, mask)
    else:
        ref, o_ref, e = oracle.scan(*args, dst_dtype=dst_kind, **kw)
        got = np64(dt.cpu())
    assert e == 0
    assert_close(got, ref, 1e-2, f"chunked {rule} {src_kind}->{dst_kind}: final states")
    assert_close(np64(o.cpu()), o_ref, 1e-2, f"chunked {rule} {src_kind}->{dst_kind}: outputs")
    # the empty sequence (index 1) stores its initial state through the destination's format
    assert_close(got[1], ref[1], 1e-5, f"chunked {rule} {src_kind}->{dst_kind}: empty sequence")


def test_chunked_scan_qgroups_q8():
    """The chunked prefill in the query-group direction from and to q8 pools: the state
    against the oracle's q8 scan, the outputs (taken before the state is encoded) against
    its query-group scan from the decoded initial states."""
    dk, dv, n_hp, H, group = 128, 128, 16, 2, 3
    lengths = [70, 0, 129]
    inp = W.scan_inputs(lengths=lengths, n_qk_heads=H, n_v_heads=H, d_k=dk, d_v=dv, rule="gated_delta",
                        state_dtype=BF16, io_dtype=BF16, seed=99, init="slots", init_dtype=F32, pool_std=0.3,
                        n_q_heads=H * group)
    mask = masks_of(H, dk, n_hp, 8)
    src, st = q8_pool(inp.pool, H, n_hp, mask)
    src_vals = _values_of(st, dk, dv, n_hp, mask)
    dt = torch.zeros(len(lengths), H, L.q8_tile_bytes(dk, dv, n_hp), dtype=torch.uint8, device="cuda")
    dst = L.Pool.q8(dt, H, dk, dv, n_hp, mask.cuda())
    o = torch.empty(inp.q.shape[0], H * group, dv, dtype=BF16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(L.la_state_scan_chunked_qgroups("gated_delta", src, dev(inp.read_slot), dst, None, dev(inp.cu_seqlens),
                                            dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta),
                                            inp.scale, o, err))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    cu = inp.cu_seqlens.numpy()
    q0 = np64(inp.q).reshape(-1, H, group, dk)[:, :, 0]
    ref, _, e = oracle.scan_q8("gated_delta", H, cu, q0, np64(inp.k), np64(inp.v), np64(inp.g), np64(inp.beta),
                               inp.scale, masks=u32(mask), src_pool=src_vals, read_slot=inp.read_slot.numpy(),
                               io_dtype="bf16")
    assert e == 0
    _, o_ref, e = oracle.scan_qgroups("gated_delta", H * group, cu, np64(inp.q), np64(inp.k), np64(inp.v),
                                      np64(inp.g), np64(inp.beta), inp.scale, src_pool=src_vals,
                                      read_slot=inp.read_slot.numpy(), dst_dtype="f32", io_dtype="bf16")
    assert e == 0
    assert_close(_values_of(dt, dk, dv, n_hp, mask), ref, 1e-2, "chunked query groups q8: final states")
    assert_close(np64(o.cpu()), o_ref, 1e-2, "chunked query groups q8: outputs")


def test_chunked_scan_q8_checkpoints_and_bad_mask():
    """Checkpoints every 64 tokens into a q8 pool (the chunked checkpointed entry point),
    against the oracle's checkpointed scan decoded through the same codec; then a mask with
    the wrong number of BF16 rows: that head is skipped and reported."""
    dk, dv, n_hp = 128, 128, 16
    lengths, every = [130, 64, 5], 64
    inp = W.scan_inputs(lengths=lengths, n_qk_heads=1, n_v_heads=2, d_k=dk, d_v=dv, rule="gated_delta",
                        state_dtype=BF16, io_dtype=BF16, seed=98, init="slots", init_dtype=F32, pool_std=0.3)
    mask = masks_of(2, dk, n_hp, 7)
    src, st = q8_pool(inp.pool, 1, n_hp, mask)
    src_vals = _values_of(st, dk, dv, n_hp, mask)
    n_ck = [l // every for l in lengths]
    ckpt_cu = np.concatenate([[0], np.cumsum(n_ck)]).astype(np.int32)
    n_dst = len(lengths) + int(ckpt_cu[-1])
    ckpt_slots = np.arange(len(lengths), n_dst, dtype=np.int32)
    dt = torch.zeros(n_dst, 2, L.q8_tile_bytes(dk, dv, n_hp), dtype=torch.uint8, device="cuda")
    dst = L.Pool.q8(dt, 1, dk, dv, n_hp, mask.cuda())
    o = torch.empty(inp.q.shape[0], 2, dv, dtype=BF16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(L.la_state_scan_chunked_checkpointed("gated_delta", src, dev(inp.read_slot), dst, None,
                                                 dev(inp.cu_seqlens), dev(inp.q), dev(inp.k), dev(inp.v),
                                                 dev(inp.g), dev(inp.beta), inp.scale, o, every,
                                                 dev(torch.from_numpy(ckpt_cu)), dev(torch.from_numpy(ckpt_slots)),
                                                 err))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref, o_ref, e = oracle.scan_q8("gated_delta", 1, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k), np64(inp.v),
                                   np64(inp.g), np64(inp.beta), inp.scale, masks=u32(mask), src_pool=src_vals,
                                   read_slot=inp.read_slot.numpy(), io_dtype="bf16",
                                   dst_pool=np.zeros((n_dst, 2, dk, dv)), ckpt_every=every,
                                   ckpt_cu=ckpt_cu, ckpt_slots=ckpt_slots)
    assert e == 0
    assert_close(_values_of(dt, dk, dv, n_hp, mask), ref, 1e-2, "q8 checkpoints and final states")
    bad = mask.clone()
    bad[1, 0] = 0 if int(bad[1, 0]) != 0 else 1
    dst_bad = L.Pool.q8(dt, 1, dk, dv, n_hp, bad.cuda())
    err.zero_()
    L.check(L.la_state_scan_chunked("gated_delta", src, dev(inp.read_slot), dst_bad, None, dev(inp.cu_seqlens),
                                    dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta), inp.scale, o, err))
    torch.cuda.synchronize()
    assert int(err.item()) & L.DEVERR_Q8_MASK
