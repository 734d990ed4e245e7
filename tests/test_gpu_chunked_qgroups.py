"""GPU parity of the chunked (WY/UT) prefill in the query-group direction of the ONNX
LinearAttention operator ("Seven Architectures ...", section "ONNX LinearAttention /
FlashInfer": a group of query heads reads each state head): the one-launch chunked pass
runs once per query of the group, and the state is written by the last of them.

Checked against the oracle's token-serial query-group scan at the chunked prefill's BF16
bound (1e-2 of the largest value, as for la_state_scan_chunked), and bit for bit against
la_state_scan_chunked given one query of the group at a time: the same kernel on the same
operands, so every output head and the states must agree exactly."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_recurrent_la_b200 import lastate as L
from gated_deltanet_recurrent_la_b200 import workloads as W
from gpu_helpers import BF16, F32, assert_close, dev, dname, np64, oracle_scan_qgroups

pytestmark = pytest.mark.gpu

CHUNK_TOL = 1e-2
SCALAR_RULES = ["linear", "gated", "delta", "gated_delta"]


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    L.lib()


def _run(inp, dst_t, src=None, read_slot=None, write_slot=None, seq_order=None):
    o = torch.full((inp.q.shape[0], inp.n_q_heads, inp.d_v), 5.0, dtype=BF16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(L.la_state_scan_chunked_qgroups(inp.rule, src, read_slot, L.Pool(dst_t, inp.n_qk_heads), write_slot,
                                            dev(inp.cu_seqlens), dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.g),
                                            dev(inp.beta), inp.scale, o, err, seq_order=seq_order))
    torch.cuda.synchronize()
    return o.cpu(), int(err.item())


@pytest.mark.parametrize("group", [2, 8])
@pytest.mark.parametrize("dst", [F32, BF16], ids=["f32", "bf16"])
@pytest.mark.parametrize("rule", SCALAR_RULES)
def test_chunked_qgroups_vs_oracle(rule, dst, group):
    H = 2
    inp = W.scan_inputs(lengths=[100, 1, 0, 200, 63, 129], n_qk_heads=H, n_v_heads=H, d_k=128, d_v=128, rule=rule,
                        io_dtype=BF16, seed=140 + group, init="slots", init_dtype=F32, scale=0.8,
                        n_q_heads=H * group)
    n = inp.cu_seqlens.numel() - 1
    dst_t = torch.full((n, H, 128, 128), 3.0, dtype=dst, device="cuda")
    o, err = _run(inp, dst_t, L.Pool(dev(inp.pool), H), dev(inp.read_slot))
    assert err == 0
    S_ref, o_ref, e = oracle_scan_qgroups(inp, dst)
    assert e == 0
    assert_close(np64(dst_t.cpu()), S_ref, CHUNK_TOL, f"{rule} group {group}: final states")
    assert_close(np64(o), o_ref, CHUNK_TOL, f"{rule} group {group}: outputs")


def test_chunked_qgroups_in_place_slots_and_order():
    """Each request reads and writes one slot of a shared pool (permuted), units dealt in a
    given order: every query pass reads the initial state, so the state is written only
    after the last of them."""
    H, group = 2, 4
    lengths = [70, 129, 5, 64]
    inp = W.scan_inputs(lengths=lengths, n_qk_heads=H, n_v_heads=H, d_k=128, d_v=128, rule="gated_delta",
                        io_dtype=BF16, seed=150, init="slots", init_dtype=F32, scale=0.9, n_q_heads=H * group)
    n_slots = inp.pool.shape[0]
    slots = torch.tensor([3, 0, 2, 1], dtype=torch.int32)
    assert int(slots.max()) < n_slots
    pool_t = dev(inp.pool).clone()
    order = torch.tensor([1, 0, 3, 2], dtype=torch.int32)
    o, err = _run(inp, pool_t, L.Pool(pool_t, H), dev(slots), dev(slots), dev(order))
    assert err == 0
    ref, o_ref, e = oracle.scan_qgroups("gated_delta", H * group, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k),
                                        np64(inp.v), np64(inp.g), np64(inp.beta), inp.scale, src_pool=np64(inp.pool),
                                        read_slot=slots.numpy(), dst_pool=np64(inp.pool).copy(), dst_dtype="f32",
                                        write_slot=slots.numpy(), io_dtype="bf16")
    assert e == 0
    assert_close(np64(pool_t.cpu()), ref, CHUNK_TOL, "pool after the in-place prefill")
    assert_close(np64(o), o_ref, CHUNK_TOL, "outputs")


@pytest.mark.parametrize("group", [1, 3, 8])
@pytest.mark.parametrize("rule", ["gated", "gated_delta"])
def test_chunked_qgroups_each_query_matches_chunked_scan_bitwise(rule, group):
    H = 2
    inp = W.scan_inputs(lengths=[64, 130, 17], n_qk_heads=H, n_v_heads=H, d_k=128, d_v=128, rule=rule,
                        io_dtype=BF16, seed=160 + group, init="slots", init_dtype=F32, n_q_heads=H * group)
    n = inp.cu_seqlens.numel() - 1
    dst_g = torch.zeros(n, H, 128, 128, dtype=F32, device="cuda")
    src = L.Pool(dev(inp.pool), H)
    o_g, err = _run(inp, dst_g, src, dev(inp.read_slot))
    assert err == 0
    T = inp.q.shape[0]
    q4 = inp.q.view(T, H, group, 128)
    for i in range(group):
        dst_1 = torch.zeros_like(dst_g)
        o_1 = torch.empty(T, H, 128, dtype=BF16, device="cuda")
        e1 = torch.zeros(1, dtype=torch.int32, device="cuda")
        L.check(L.la_state_scan_chunked(rule, src, dev(inp.read_slot), L.Pool(dst_1, H), None, dev(inp.cu_seqlens),
                                        dev(q4[:, :, i].contiguous()), dev(inp.k), dev(inp.v), dev(inp.g),
                                        dev(inp.beta), inp.scale, o_1, e1))
        torch.cuda.synchronize()
        assert int(e1.item()) == 0
        assert torch.equal(o_g.view(T, H, group, 128)[:, :, i], o_1.cpu()), f"query {i} of {group}"
        assert torch.equal(dst_g, dst_1)


def test_chunked_qgroups_full_prefill_sampled():
    """The query-group prefill at a serving size (8 state heads, 4 queries each, 16 ragged
    sequences up to 1000 tokens), with sampled (sequence, head) units recomputed by the
    oracle."""
    H, group = 8, 4
    g = torch.Generator().manual_seed(170)
    lengths = torch.randint(1, 1000, (16,), generator=g).tolist()
    inp = W.scan_inputs(lengths=lengths, n_qk_heads=H, n_v_heads=H, d_k=128, d_v=128, rule="gated_delta",
                        io_dtype=BF16, seed=171, n_q_heads=H * group)
    n = len(lengths)
    dst_t = torch.zeros(n, H, 128, 128, dtype=F32, device="cuda")
    o, err = _run(inp, dst_t)
    assert err == 0
    cu = inp.cu_seqlens.numpy()
    for s, h in [(0, 0), (5, 3), (11, 7), (15, 2)]:
        a, b = int(cu[s]), int(cu[s + 1])
        qs = np64(inp.q[a:b, h * group:(h + 1) * group])
        ks, vs = np64(inp.k[a:b, h:h + 1]), np64(inp.v[a:b, h:h + 1])
        S_ref, o_ref, e = oracle.scan_qgroups("gated_delta", group, np.array([0, b - a], dtype=np.int32), qs, ks, vs,
                                              np64(inp.g[a:b, h:h + 1]), np64(inp.beta[a:b, h:h + 1]), inp.scale,
                                              dst_dtype="f32", io_dtype="bf16")
        assert e == 0
        assert_close(np64(dst_t[s, h:h + 1].cpu())[None], S_ref, CHUNK_TOL, f"unit ({s}, {h}): state")
        assert_close(np64(o[a:b, h * group:(h + 1) * group]), o_ref, CHUNK_TOL, f"unit ({s}, {h}): outputs")
