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
from gpu_helpers import BF16, F32, assert_close, dev, dname, np64, tolerances

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
