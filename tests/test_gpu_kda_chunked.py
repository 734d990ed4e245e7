"""GPU parity of the chunked prefill for the channel-wise gate (rule kda, two launches:
the decay-scaled operands and intra-chunk products per (chunk, head), then the tcgen05
recurrence) against the oracle's token-serial kda scan.

Within a chunk the products take BF16 operands (the decays folded into them), so the
comparison is at the chunked prefill's BF16 tolerance: 1e-2 of the largest value on
sequences of up to a few hundred tokens, 2e-2 on the full prefill workload.  Decay
magnitudes below e^-8 act as e^-8 in the chunked form (zero included); the oracle takes
the decays as they are, and the difference stays far inside the tolerance."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_recurrent_la_b200 import lastate as L
from gated_deltanet_recurrent_la_b200 import workloads as W
from gpu_helpers import BF16, F32, assert_close, check_scan_units, dev, np64, oracle_scan, prefill_picks

pytestmark = pytest.mark.gpu

TOL = 1e-2


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    L.lib()


def gpu_kda_chunked(inp, dst_dtype, *, write_slot=None, n_dst=None, seq_order=None, ws_fill=0xAB):
    n_seqs = inp.cu_seqlens.numel() - 1
    n_dst = n_seqs if n_dst is None else n_dst
    dst_t = torch.full((n_dst, inp.n_v_heads, inp.d_k, inp.d_v), 3.0, dtype=dst_dtype, device="cuda")
    src = None if inp.pool is None else L.Pool(dev(inp.pool), inp.n_qk_heads)
    o = torch.full((inp.q.shape[0], inp.n_v_heads, inp.d_v), 5.0, dtype=inp.io_dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    nbytes = L.la_scan_chunked_workspace_bytes_rule("kda", inp.q.shape[0], n_seqs, inp.n_v_heads)
    ws = torch.full((nbytes,), ws_fill, dtype=torch.uint8, device="cuda")
    st = L.la_state_scan_chunked_ws("kda", src, dev(inp.read_slot), L.Pool(dst_t, inp.n_qk_heads),
                                    None if write_slot is None else dev(write_slot), dev(inp.cu_seqlens),
                                    dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta), inp.scale, o, ws,
                                    err, seq_order=None if seq_order is None else dev(seq_order))
    L.check(st)
    torch.cuda.synchronize()
    return dst_t.cpu(), o.cpu(), int(err.item())


@pytest.mark.parametrize("dst", [F32, BF16], ids=["f32", "bf16"])
def test_kda_chunked_vs_oracle(dst):
    """Ragged and empty sequences (1, 63, 64, 129, 200 tokens), two state heads per q/k
    head, an FP32 initial state read from slots, the workload's decay distribution."""
    inp = W.scan_inputs(lengths=[100, 64, 1, 0, 200, 63, 129], n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128,
                        rule="kda", io_dtype=BF16, seed=61, init="slots", init_dtype=F32, scale=0.8)
    S, o, err = gpu_kda_chunked(inp, dst)
    assert err == 0
    S_ref, o_ref, e = oracle_scan(inp, dst_dtype=dst)
    assert e == 0
    assert_close(np64(S), S_ref, TOL, "kda chunked: final states")
    assert_close(np64(o), o_ref, TOL, "kda chunked: outputs")


def test_kda_chunked_complex_kda_ranges():
    """Decays alpha in [-1, 1] per channel (signs of either kind, magnitudes down to zero) and
    beta in [0, 2], the "Complex KDA" ranges."""
    inp = W.scan_inputs(lengths=[300, 70, 5], n_qk_heads=1, n_v_heads=2, d_k=128, d_v=128, rule="kda",
                        io_dtype=BF16, seed=62, g_mode="uniform_pm1", beta_mode="uniform_0_2", init="slots",
                        init_dtype=F32)
    S, o, err = gpu_kda_chunked(inp, F32)
    assert err == 0
    S_ref, o_ref, _ = oracle_scan(inp, dst_dtype=F32)
    assert_close(np64(S), S_ref, TOL, "kda chunked, wide ranges: final states")
    assert_close(np64(o), o_ref, TOL, "kda chunked, wide ranges: outputs")


def test_kda_chunked_steep_and_vanishing_decays():
    """Channels decaying by up to e^-8 per token, and a tenth of the decays exactly zero or
    below e^-8 in magnitude (those act as e^-8): the factored ratios stay finite and the
    result stays within the tolerance of the oracle's exact decays."""
    inp = W.scan_inputs(lengths=[257, 64], n_qk_heads=1, n_v_heads=2, d_k=128, d_v=128, rule="kda",
                        io_dtype=BF16, seed=63, init="slots", init_dtype=F32)
    gen = torch.Generator().manual_seed(64)
    a = torch.exp(-8.0 * torch.rand(inp.g.shape, generator=gen))
    pick = torch.rand(inp.g.shape, generator=gen)
    a[pick < 0.05] = 0.0
    a[(pick >= 0.05) & (pick < 0.1)] *= 1e-6
    inp.g = a.float().contiguous()
    S, o, err = gpu_kda_chunked(inp, F32)
    assert err == 0
    assert torch.isfinite(S).all() and torch.isfinite(o.float()).all()
    S_ref, o_ref, _ = oracle_scan(inp, dst_dtype=F32)
    assert_close(np64(S), S_ref, TOL, "kda chunked, steep decays: final states")
    assert_close(np64(o), o_ref, TOL, "kda chunked, steep decays: outputs")


def test_kda_chunked_unit_decay_and_zero_beta_pass_the_state():
    """alpha = 1 and beta = 0 everywhere: every state passes through unchanged (up to its
    BF16 copy only feeding the readout) and the outputs are the readouts of S0."""
    inp = W.scan_inputs(lengths=[130, 64], n_qk_heads=1, n_v_heads=2, d_k=128, d_v=128, rule="kda",
                        io_dtype=BF16, seed=65, g_mode="one", beta_mode="zero", init="slots", init_dtype=F32)
    S, o, err = gpu_kda_chunked(inp, F32)
    assert err == 0
    assert torch.equal(S, inp.pool[inp.read_slot.long()].float())
    S_ref, o_ref, _ = oracle_scan(inp, dst_dtype=F32)
    assert_close(np64(o), o_ref, TOL, "kda chunked: readout of the unchanged state")


def test_kda_chunked_equals_gated_delta_for_equal_channels():
    """A decay equal on every channel is the scalar gate: kda then computes gated_delta, and
    both chunked paths agree with the oracle's gated_delta scan."""
    inp = W.scan_inputs(lengths=[150, 40], n_qk_heads=2, n_v_heads=2, d_k=128, d_v=128, rule="gated_delta",
                        io_dtype=BF16, seed=66, init="slots", init_dtype=F32)
    S_ref, o_ref, _ = oracle_scan(inp, dst_dtype=F32)
    kin = W.Inputs(**{**inp.__dict__, "rule": "kda",
                      "g": inp.g[:, :, None].expand(-1, -1, inp.d_k).contiguous()})
    S, o, err = gpu_kda_chunked(kin, F32)
    assert err == 0
    assert_close(np64(S), S_ref, TOL, "kda with equal channels = gated_delta: final states")
    assert_close(np64(o), o_ref, TOL, "kda with equal channels = gated_delta: outputs")


def test_kda_chunked_pool_slots_order_and_empty():
    """Write slots into a larger pool (other slots untouched), a reversed seq_order, BF16
    final states, an empty sequence storing its initial state; a workspace filled with NaN
    bytes (every tile the recurrence reads is written first)."""
    inp = W.scan_inputs(lengths=[90, 0, 200, 3, 64], n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128, rule="kda",
                        io_dtype=BF16, seed=67, init="slots", init_dtype=F32)
    write = torch.tensor([7, 2, 5, 0, 4], dtype=torch.int32)
    order = torch.tensor([4, 3, 2, 1, 0], dtype=torch.int32)
    S, o, err = gpu_kda_chunked(inp, BF16, write_slot=write, n_dst=9, seq_order=order, ws_fill=0xFF)
    assert err == 0
    S_ref, o_ref, _ = oracle_scan(inp, dst_dtype=BF16)
    for s in range(5):
        assert_close(np64(S[int(write[s])]), S_ref[s], TOL, f"sequence {s} state in slot {int(write[s])}")
    untouched = [i for i in range(9) if i not in write.tolist()]
    assert torch.all(S[untouched].float() == 3.0)
    assert_close(np64(o), o_ref, TOL, "outputs")


def test_kda_chunked_all_sequences_empty():
    inp = W.scan_inputs(lengths=[0, 0], n_qk_heads=1, n_v_heads=2, d_k=128, d_v=128, rule="kda", io_dtype=BF16,
                        seed=68, init="slots", init_dtype=F32)
    S, o, err = gpu_kda_chunked(inp, F32)
    assert err == 0 and o.numel() == 0
    assert torch.equal(S, inp.pool[inp.read_slot.long()].float())


def test_kda_chunked_workspace_checks():
    inp = W.scan_inputs(lengths=[70, 10], n_qk_heads=1, n_v_heads=2, d_k=128, d_v=128, rule="kda",
                        io_dtype=BF16, seed=69)
    dst_t = torch.zeros(2, 2, 128, 128, dtype=F32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    need = L.la_scan_chunked_workspace_bytes_rule("kda", 80, 2, 2)
    small = torch.zeros(need - 16, dtype=torch.uint8, device="cuda")
    st = L.la_state_scan_chunked_ws("kda", None, None, L.Pool(dst_t, 1), None, dev(inp.cu_seqlens), dev(inp.q),
                                    dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta), 1.0,
                                    torch.empty_like(dev(inp.v)), small, err)
    assert st == L.LA_ERR_SHAPE
    # the one-launch entry point has no kda form
    st = L.la_state_scan_chunked("kda", None, None, L.Pool(dst_t, 1), None, dev(inp.cu_seqlens), dev(inp.q),
                                 dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta), 1.0,
                                 torch.empty_like(dev(inp.v)), err)
    assert st == L.LA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert int(err.item()) == 0


def test_kda_prefill32_chunked_units():
    """The full kda prefill workload through the chunked path, as the benchmark runs it:
    every sequence on two heads and the longest on all 32 against the oracle."""
    inp = W.kda_prefill32()
    S, o, err = gpu_kda_chunked(inp, BF16)
    assert err == 0
    check_scan_units(inp, S, o, prefill_picks(inp), 2e-2, 2e-2)
