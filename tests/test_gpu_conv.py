"""GPU parity of the decode step with the short causal convolution fused ahead of it
(la_state_step_conv) against the oracle: states and outputs at the tolerances of
la_state_step (the convolution's outputs stay FP32 on both sides), the new histories bit
for bit (they are copies of inputs), slots that are not written untouched."""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_recurrent_la_b200 import lastate as L
from gated_deltanet_recurrent_la_b200 import workloads as W
from gpu_helpers import BF16, F32, assert_close, dev, dname, np64, prefill_picks, scan_unit_inputs, tolerances

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    L.lib()


def run_both(inp, width, act, l2, hist, n_hist_slots):
    H, dk, dv, B = inp.n_v_heads, inp.d_k, inp.d_v, inp.q.shape[0]
    g = torch.Generator().manual_seed(width * 10 + act * 2 + l2)
    wq = torch.randn(inp.n_qk_heads, dk, width, generator=g) / width ** 0.5
    wk = torch.randn(inp.n_qk_heads, dk, width, generator=g) / width ** 0.5
    wv = torch.randn(H, dv, width, generator=g) / width ** 0.5
    pool_t = dev(inp.pool)
    pool = L.Pool(pool_t, inp.n_qk_heads)
    hist_t = dev(hist)
    conv = L.Conv(dev(wq), dev(wk), dev(wv), hist_t, activation=act, qk_l2norm=l2)
    o = torch.full((B, H, dv), 7.0, dtype=inp.io_dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(L.la_state_step_conv(inp.rule, pool, dev(inp.read_slot), pool, dev(inp.write_slot), conv, dev(inp.q),
                                 dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta), inp.scale, o, err))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rs = None if inp.read_slot is None else inp.read_slot.numpy()
    ws = None if inp.write_slot is None else inp.write_slot.numpy()
    ref, href, o_ref, e = oracle.step_conv(inp.rule, inp.n_qk_heads, np64(inp.pool), np64(inp.q), np64(inp.k),
                                           np64(inp.v), np64(inp.g), np64(inp.beta), inp.scale, wq.double().numpy(),
                                           wk.double().numpy(), wv.double().numpy(), np64(hist), act=act, l2norm=l2,
                                           dst_dtype=dname(inp.state_dtype), io_dtype=dname(inp.io_dtype),
                                           read_slot=rs, write_slot=ws)
    assert e == 0
    return pool_t.cpu(), hist_t.cpu(), o.cpu(), ref, href, o_ref


@pytest.mark.parametrize("width", [2, 3, 4])
@pytest.mark.parametrize("act,l2", [(0, 0), (1, 1)], ids=["plain", "silu_norm"])
@pytest.mark.parametrize("state,io", [(F32, F32), (BF16, BF16)], ids=["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(16, 16), (64, 64), (128, 128)], ids=["16x16", "64x64", "128x128"])
@pytest.mark.parametrize("rule", ["gated_delta", "kda", "linear"])
def test_step_conv(rule, dk, dv, state, io, act, l2, width):
    inp = W.step_inputs(B=5, n_qk_heads=2, n_v_heads=4, d_k=dk, d_v=dv, rule=rule, n_slots=8, state_dtype=state,
                        io_dtype=io, seed=100 + width + dk, slot_map="perm", normalise_qk=False, pool_std=0.3)
    hist = torch.randn(8, 4, 2 * dk + dv, width - 1, generator=torch.Generator().manual_seed(7)).to(io)
    pool, hist_after, o, ref, href, o_ref = run_both(inp, width, act, l2, hist, 8)
    ws = inp.write_slot.numpy()
    tol_s, tol_o = tolerances(state, io)
    # without the normalisation keys are not unit vectors; compare relative to the largest value
    assert_close(np64(pool)[ws], ref[ws], tol_s, f"{rule} W={width}: states")
    assert_close(np64(o), o_ref, tol_o, f"{rule} W={width}: outputs")
    assert np.array_equal(np64(hist_after), href), "histories are exact copies of inputs"
    untouched = np.setdiff1d(np.arange(8), ws)
    assert torch.equal(pool[untouched], inp.pool[untouched])


def test_conv_decode64_full():
    inp = W.conv_decode64()
    x = inp.extra
    pool_t = dev(inp.pool)
    pool = L.Pool(pool_t, 16)
    hist_t = dev(x["hist"])
    conv = L.Conv(dev(x["w_q"]), dev(x["w_k"]), dev(x["w_v"]), hist_t, activation=1, qk_l2norm=1)
    o = torch.empty(64, 32, 128, dtype=BF16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(L.la_state_step_conv("gated_delta", pool, dev(inp.read_slot), pool, dev(inp.write_slot), conv,
                                 dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta), 1.0, o, err))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rows = torch.arange(0, 64, 7)
    rs, ws = inp.read_slot[rows].long(), inp.write_slot[rows].long()
    ref, href, o_ref, e = oracle.step_conv("gated_delta", 16, np64(inp.pool[rs]), np64(inp.q[rows]),
                                           np64(inp.k[rows]), np64(inp.v[rows]), np64(inp.g[rows]),
                                           np64(inp.beta[rows]), 1.0, np64(x["w_q"]), np64(x["w_k"]),
                                           np64(x["w_v"]), np64(x["hist"][rs]), act=1, l2norm=1, dst_dtype="bf16",
                                           io_dtype="bf16")
    assert e == 0
    after = pool_t.cpu()
    assert_close(np64(after[ws]), ref, 2e-2, "sampled states")
    assert_close(np64(o.cpu()[rows]), o_ref, 2e-2, "sampled outputs")
    assert np.array_equal(np64(hist_t.cpu()[ws]), href), "sampled histories"


def _conv_weights(nqk, H, dk, dv, width, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(nqk, dk, width, generator=g) / width ** 0.5,
            torch.randn(nqk, dk, width, generator=g) / width ** 0.5,
            torch.randn(H, dv, width, generator=g) / width ** 0.5)


def run_scan_conv(inp, wq, wk, wv, width, act, l2, hist_src, n_dst, dst_dtype, read_slot=None, write_slot=None):
    H, dk, dv = inp.n_v_heads, inp.d_k, inp.d_v
    dst_t = torch.full((n_dst, H, dk, dv), 3.0, dtype=dst_dtype, device="cuda")
    hist_dst = torch.full((n_dst, H, 2 * dk + dv, width - 1), 9.0, dtype=inp.io_dtype, device="cuda")
    src = None if inp.pool is None else L.Pool(dev(inp.pool), inp.n_qk_heads)
    hs = None if hist_src is None else dev(hist_src)
    conv = L.Conv(dev(wq), dev(wk), dev(wv), hs if hs is not None else hist_dst, hist_dst, activation=act,
                  qk_l2norm=l2)
    o = torch.full((inp.q.shape[0], H, dv), 5.0, dtype=inp.io_dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(L.la_state_scan_conv(inp.rule, src, dev(read_slot), L.Pool(dst_t, inp.n_qk_heads), dev(write_slot),
                                 dev(inp.cu_seqlens), conv, dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.g),
                                 dev(inp.beta), inp.scale, o, err))
    torch.cuda.synchronize()
    return dst_t.cpu(), hist_dst.cpu(), o.cpu(), int(err.item())


@pytest.mark.parametrize("width", [2, 4])
@pytest.mark.parametrize("act,l2", [(0, 0), (1, 1)], ids=["plain", "silu_norm"])
@pytest.mark.parametrize("io", [F32, BF16], ids=["f32io", "bf16io"])
@pytest.mark.parametrize("dk,dv", [(16, 16), (128, 64), (128, 128)], ids=["16x16", "128x64", "128x128"])
@pytest.mark.parametrize("rule", ["gated_delta", "kda", "gated"])
def test_scan_conv(rule, dk, dv, io, act, l2, width):
    lengths = [5, 0, 2, 37, 17]
    inp = W.scan_inputs(lengths=lengths, n_qk_heads=2, n_v_heads=4, d_k=dk, d_v=dv, rule=rule, state_dtype=F32,
                        io_dtype=io, seed=110 + width + dk, init="slots", init_dtype=F32, normalise_qk=False,
                        pool_std=0.3)
    wq, wk, wv = _conv_weights(2, 4, dk, dv, width, 3 + width)
    n = len(lengths)
    hist = torch.randn(n, 4, 2 * dk + dv, width - 1, generator=torch.Generator().manual_seed(8)).to(io)
    ws = torch.tensor([2, 0, 4, 1, 3], dtype=torch.int32)
    S, hnew, o, err = run_scan_conv(inp, wq, wk, wv, width, act, l2, hist, n, F32, read_slot=inp.read_slot,
                                    write_slot=ws)
    assert err == 0
    ref, href, o_ref, e = oracle.scan_conv(rule, 2, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k), np64(inp.v),
                                           np64(inp.g), np64(inp.beta), inp.scale, wq.double().numpy(),
                                           wk.double().numpy(), wv.double().numpy(), act=act, l2norm=l2,
                                           conv_src=np64(hist), src_pool=np64(inp.pool),
                                           read_slot=inp.read_slot.numpy(), dst_pool=np.zeros((n, 4, dk, dv)),
                                           conv_dst=np.zeros((n, 4, 2 * dk + dv, width - 1)), write_slot=ws.numpy(),
                                           dst_dtype="f32", io_dtype=dname(io))
    assert e == 0
    tol_s, tol_o = tolerances(F32, io)
    assert_close(np64(S), ref, tol_s, f"{rule} W={width}: final states")
    assert_close(np64(o), o_ref, tol_o, f"{rule} W={width}: outputs")
    assert np.array_equal(np64(hnew), href), "final histories are exact copies of inputs"


def test_scan_conv_then_step_conv_continues_the_sequence():
    """A fresh prefill through the convolution, then one fused decode step from its slot,
    equals the oracle scan over the whole sequence (state, last output, history)."""
    width = 4
    inp = W.scan_inputs(lengths=[30], n_qk_heads=1, n_v_heads=2, d_k=64, d_v=64, rule="gated_delta",
                        state_dtype=F32, io_dtype=F32, seed=120, normalise_qk=False)
    wq, wk, wv = _conv_weights(1, 2, 64, 64, width, 9)
    pre = W.Inputs(**{**inp.__dict__, "q": inp.q[:29], "k": inp.k[:29], "v": inp.v[:29], "g": inp.g[:29],
                      "beta": inp.beta[:29], "cu_seqlens": torch.tensor([0, 29], dtype=torch.int32)})
    S, hist, o_pre, err = run_scan_conv(pre, wq, wk, wv, width, 1, 1, None, 1, F32)
    assert err == 0
    pool_t, hist_t = dev(S), dev(hist)
    conv = L.Conv(dev(wq), dev(wk), dev(wv), hist_t, activation=1, qk_l2norm=1)
    o = torch.empty(1, 2, 64, dtype=F32, device="cuda")
    e = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(L.la_state_step_conv("gated_delta", L.Pool(pool_t, 1), None, L.Pool(pool_t, 1), None, conv,
                                 dev(inp.q[29:]), dev(inp.k[29:]), dev(inp.v[29:]), dev(inp.g[29:]),
                                 dev(inp.beta[29:]), 1.0, o, e))
    torch.cuda.synchronize()
    assert int(e.item()) == 0
    ref, href, o_ref, er = oracle.scan_conv("gated_delta", 1, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k),
                                            np64(inp.v), np64(inp.g), np64(inp.beta), 1.0, wq.double().numpy(),
                                            wk.double().numpy(), wv.double().numpy(), act=1, l2norm=1)
    assert er == 0
    assert_close(np64(pool_t.cpu()), ref, 1e-4, "state after prefill + one step")
    assert_close(np64(o.cpu())[0], o_ref[29], 1e-4, "the decode step's output")
    assert_close(np64(o_pre), o_ref[:29], 1e-4, "prefill outputs")
    assert np.array_equal(np64(hist_t.cpu()), href)


def test_conv_prefill32_units():
    """The full prefill workload with the convolution ahead of every token (fresh prefill):
    every sequence on two heads and the longest on all 32 against the oracle's convolved scan,
    including the final histories (exact copies of the last raw inputs)."""
    inp = W.conv_prefill32()
    x = inp.extra
    width, n = x["width"], inp.cu_seqlens.numel() - 1
    S, hnew, o, err = run_scan_conv(inp, x["w_q"], x["w_k"], x["w_v"], width, x["activation"], x["qk_l2norm"], None,
                                    n, inp.state_dtype)
    assert err == 0
    cu = inp.cu_seqlens.numpy()
    tol_s, tol_o = tolerances(inp.state_dtype, inp.io_dtype)
    by_head = {}
    for s_, h in prefill_picks(inp):
        by_head.setdefault(h, []).append(s_)
    for h, seqs in sorted(by_head.items()):
        sub = scan_unit_inputs(inp, [(s_, h) for s_ in seqs])
        ref, href, o_ref, e = oracle.scan_conv(
            inp.rule, 1, sub.cu_seqlens.numpy(), np64(sub.q), np64(sub.k), np64(sub.v), np64(sub.g), np64(sub.beta),
            inp.scale, x["w_q"][h:h + 1].double().numpy(), x["w_k"][h:h + 1].double().numpy(),
            x["w_v"][h:h + 1].double().numpy(), act=x["activation"], l2norm=x["qk_l2norm"],
            dst_dtype=dname(inp.state_dtype), io_dtype=dname(inp.io_dtype))
        assert e == 0
        ucu = sub.cu_seqlens.numpy()
        for i, s_ in enumerate(seqs):
            t0, t1 = int(cu[s_]), int(cu[s_ + 1])
            assert_close(np64(S[s_, h]), ref[i, 0], tol_s, f"seq {s_} head {h} final state")
            assert_close(np64(o[t0:t1, h]), o_ref[int(ucu[i]):int(ucu[i + 1]), 0], tol_o, f"seq {s_} head {h} outputs")
            assert np.array_equal(np64(hnew[s_, h]), href[i, 0]), f"seq {s_} head {h} final history"


# ---- the convolution inside the one-launch chunked prefill ------------------------------
# The chunked prefill rounds its operands to BF16 (the convolved q, k, v included), so its
# states and outputs are compared at the chunked tolerance (1e-2 of the largest value on
# these sizes); the histories are exact copies of raw inputs on both sides.
CHUNK_TOL = 1e-2


def run_chunked_conv(inp, wq, wk, wv, width, act, l2, hist_src, n_dst, dst_dtype, read_slot=None, write_slot=None,
                     seq_order=None, form="one"):
    """form "one": la_state_scan_chunked_conv (the convolution in the chunked kernel);
    "ws": la_state_scan_chunked_conv_ws (the convolution as its own launch, its output
    through a workspace filled with NaN bytes beforehand)."""
    H, dk, dv = inp.n_v_heads, inp.d_k, inp.d_v
    dst_t = torch.full((n_dst, H, dk, dv), 3.0, dtype=dst_dtype, device="cuda")
    hist_dst = torch.full((n_dst, H, 2 * dk + dv, width - 1), 9.0, dtype=inp.io_dtype, device="cuda")
    src = None if inp.pool is None else L.Pool(dev(inp.pool), inp.n_qk_heads)
    hs = None if hist_src is None else dev(hist_src)
    conv = L.Conv(dev(wq), dev(wk), dev(wv), hs if hs is not None else hist_dst, hist_dst, activation=act,
                  qk_l2norm=l2)
    o = torch.full((inp.q.shape[0], H, dv), 5.0, dtype=inp.io_dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    order = None if seq_order is None else dev(seq_order)
    if form == "ws":
        nbytes = L.la_scan_chunked_conv_workspace_bytes(inp.q.shape[0], H)
        ws = torch.full((nbytes,), 0xFF, dtype=torch.uint8, device="cuda")
        L.check(L.la_state_scan_chunked_conv_ws(inp.rule, src, dev(read_slot), L.Pool(dst_t, inp.n_qk_heads),
                                                dev(write_slot), dev(inp.cu_seqlens), conv, dev(inp.q), dev(inp.k),
                                                dev(inp.v), dev(inp.g), dev(inp.beta), inp.scale, o, ws, err,
                                                seq_order=order))
    else:
        L.check(L.la_state_scan_chunked_conv(inp.rule, src, dev(read_slot), L.Pool(dst_t, inp.n_qk_heads),
                                             dev(write_slot), dev(inp.cu_seqlens), conv, dev(inp.q), dev(inp.k),
                                             dev(inp.v), dev(inp.g), dev(inp.beta), inp.scale, o, err, seq_order=order))
    torch.cuda.synchronize()
    return dst_t.cpu(), hist_dst.cpu(), o.cpu(), int(err.item())


@pytest.mark.parametrize("form", ["one", "ws"])
@pytest.mark.parametrize("width", [2, 3, 4])
@pytest.mark.parametrize("rule,act,l2", [("linear", 0, 0), ("linear", 1, 1), ("gated", 0, 0), ("gated", 1, 1),
                                         ("delta", 0, 1), ("delta", 1, 1), ("gated_delta", 0, 1),
                                         ("gated_delta", 1, 1)])
def test_chunked_scan_conv(rule, act, l2, width, form):
    """Sequences shorter than the window, empty, across chunk boundaries (64, 65, 130
    tokens), two state heads per q/k head, histories read at permuted read slots and
    written at other write slots, against the oracle's convolved scan.  The delta rules
    take unit-length keys (their recurrence with raw convolution outputs, |k|^2 ~ d_k,
    diverges within a hundred tokens on both sides)."""
    lengths = [5, 0, 2, 130, 37, 64, 65]
    n = len(lengths)
    inp = W.scan_inputs(lengths=lengths, n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128, rule=rule, state_dtype=F32,
                        io_dtype=BF16, seed=130 + width + 3 * act, init="slots", init_dtype=F32, normalise_qk=False,
                        pool_std=0.3)
    wq, wk, wv = _conv_weights(2, 4, 128, 128, width, 13 + width)
    hist = torch.randn(n, 4, 384, width - 1, generator=torch.Generator().manual_seed(18)).to(BF16)
    ws = torch.tensor([2, 0, 4, 1, 3, 6, 5], dtype=torch.int32)
    S, hnew, o, err = run_chunked_conv(inp, wq, wk, wv, width, act, l2, hist, n, F32, read_slot=inp.read_slot,
                                       write_slot=ws, form=form)
    assert err == 0
    ref, href, o_ref, e = oracle.scan_conv(rule, 2, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k), np64(inp.v),
                                           np64(inp.g), np64(inp.beta), inp.scale, wq.double().numpy(),
                                           wk.double().numpy(), wv.double().numpy(), act=act, l2norm=l2,
                                           conv_src=np64(hist), src_pool=np64(inp.pool),
                                           read_slot=inp.read_slot.numpy(), dst_pool=np.zeros((n, 4, 128, 128)),
                                           conv_dst=np.zeros((n, 4, 384, width - 1)), write_slot=ws.numpy(),
                                           dst_dtype="f32", io_dtype="bf16")
    assert e == 0
    assert_close(np64(S), ref, CHUNK_TOL, f"{rule} W={width}: final states")
    assert_close(np64(o), o_ref, CHUNK_TOL, f"{rule} W={width}: outputs")
    assert np.array_equal(np64(hnew), href), "final histories are exact copies of inputs"


@pytest.mark.parametrize("form", ["one", "ws"])
def test_chunked_scan_conv_fresh_prefill_and_order(form):
    """No read slots (zero histories, zero initial states), the sequences dealt longest
    first, BF16 final states."""
    lengths = [300, 3, 64, 129]
    inp = W.scan_inputs(lengths=lengths, n_qk_heads=1, n_v_heads=2, d_k=128, d_v=128, rule="gated_delta",
                        io_dtype=BF16, seed=141, normalise_qk=False)
    wq, wk, wv = _conv_weights(1, 2, 128, 128, 4, 19)
    order = torch.tensor([0, 3, 2, 1], dtype=torch.int32)
    S, hnew, o, err = run_chunked_conv(inp, wq, wk, wv, 4, 1, 1, None, 4, BF16, seq_order=order, form=form)
    assert err == 0
    ref, href, o_ref, e = oracle.scan_conv("gated_delta", 1, inp.cu_seqlens.numpy(), np64(inp.q), np64(inp.k),
                                           np64(inp.v), np64(inp.g), np64(inp.beta), inp.scale, wq.double().numpy(),
                                           wk.double().numpy(), wv.double().numpy(), act=1, l2norm=1,
                                           dst_dtype="bf16", io_dtype="bf16")
    assert e == 0
    assert_close(np64(S), ref, CHUNK_TOL, "final states")
    assert_close(np64(o), o_ref, CHUNK_TOL, "outputs")
    assert np.array_equal(np64(hnew), href)


def test_chunked_scan_conv_unsupported():
    inp = W.scan_inputs(lengths=[10], n_qk_heads=1, n_v_heads=2, d_k=128, d_v=128, rule="kda", io_dtype=BF16,
                        seed=142, normalise_qk=False)
    wq, wk, wv = _conv_weights(1, 2, 128, 128, 4, 20)
    dst_t = torch.zeros(1, 2, 128, 128, dtype=F32, device="cuda")
    hist = torch.zeros(1, 2, 384, 3, dtype=BF16, device="cuda")
    conv = L.Conv(dev(wq), dev(wk), dev(wv), hist, hist, activation=1, qk_l2norm=1)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = torch.empty(10, 2, 128, dtype=BF16, device="cuda")
    st = L.la_state_scan_chunked_conv("kda", None, None, L.Pool(dst_t, 1), None, dev(inp.cu_seqlens), conv,
                                      dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta), 1.0, o, err)
    assert st == L.LA_ERR_UNSUPPORTED


@pytest.mark.parametrize("form", ["one", "ws"])
def test_conv_prefill32_chunked_units(form):
    """The full prefill workload with the convolution, through the chunked prefill with the
    convolution in the same launch: every sequence on two heads and the longest on all 32
    against the oracle's convolved scan, final histories exact."""
    inp = W.conv_prefill32()
    x = inp.extra
    width, n = x["width"], inp.cu_seqlens.numel() - 1
    S, hnew, o, err = run_chunked_conv(inp, x["w_q"], x["w_k"], x["w_v"], width, x["activation"], x["qk_l2norm"],
                                       None, n, inp.state_dtype, form=form)
    assert err == 0
    cu = inp.cu_seqlens.numpy()
    by_head = {}
    for s_, h in prefill_picks(inp):
        by_head.setdefault(h, []).append(s_)
    for h, seqs in sorted(by_head.items()):
        sub = scan_unit_inputs(inp, [(s_, h) for s_ in seqs])
        ref, href, o_ref, e = oracle.scan_conv(
            inp.rule, 1, sub.cu_seqlens.numpy(), np64(sub.q), np64(sub.k), np64(sub.v), np64(sub.g), np64(sub.beta),
            inp.scale, x["w_q"][h:h + 1].double().numpy(), x["w_k"][h:h + 1].double().numpy(),
            x["w_v"][h:h + 1].double().numpy(), act=x["activation"], l2norm=x["qk_l2norm"],
            dst_dtype=dname(inp.state_dtype), io_dtype=dname(inp.io_dtype))
        assert e == 0
        ucu = sub.cu_seqlens.numpy()
        for i, s_ in enumerate(seqs):
            t0, t1 = int(cu[s_]), int(cu[s_ + 1])
            assert_close(np64(S[s_, h]), ref[i, 0], 2e-2, f"seq {s_} head {h} final state")
            assert_close(np64(o[t0:t1, h]), o_ref[int(ucu[i]):int(ucu[i + 1]), 0], 2e-2, f"seq {s_} head {h} outputs")
            assert np.array_equal(np64(hnew[s_, h]), href[i, 0]), f"seq {s_} head {h} final history"
