"""GPU check of la_state_scan_chunked_noalloc, the two-launch chunked prefill on the
library's own fixed workspace: the same bits as the two-launch form on a caller's workspace,
parity with the oracle, and the size limit refused before any launch."""
import ctypes

import numpy as np
import pytest
import torch

from gated_deltanet_recurrent_la_b200 import lastate as L
from gated_deltanet_recurrent_la_b200 import workloads as W
from gpu_helpers import BF16, F32, assert_close, dev, np64, oracle_scan

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    L.lib()


def _run(fn, inp):
    n_seqs = inp.cu_seqlens.numel() - 1
    dst_t = torch.full((n_seqs, inp.n_v_heads, inp.d_k, inp.d_v), 3.0, dtype=F32, device="cuda")
    src = L.Pool(dev(inp.pool), inp.n_qk_heads)
    o = torch.full((inp.q.shape[0], inp.n_v_heads, inp.d_v), 5.0, dtype=BF16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.check(fn(inp.rule, src, dev(inp.read_slot), L.Pool(dst_t, inp.n_qk_heads), None, dev(inp.cu_seqlens),
               dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta), inp.scale, o, err))
    torch.cuda.synchronize()
    return dst_t.cpu(), o.cpu(), int(err.item())


def _chunked_ws(rule, src, read_slot, dst, write_slot, cu, q, k, v, g, beta, scale, o, err):
    nbytes = L.la_scan_chunked_workspace_bytes(q.shape[0], cu.numel() - 1, v.shape[1])
    ws = torch.empty((nbytes,), dtype=torch.uint8, device="cuda")
    return L.la_state_scan_chunked_ws(rule, src, read_slot, dst, write_slot, cu, q, k, v, g, beta, scale, o, ws, err)


@pytest.mark.parametrize("rule", ["delta", "gated_delta", "gated"])
def test_noalloc_matches_the_chunked_prefill(rule):
    inp = W.scan_inputs(lengths=[130, 0, 64, 7, 300], n_qk_heads=2, n_v_heads=4, d_k=128, d_v=128, rule=rule,
                        io_dtype=BF16, seed=61, init="slots", init_dtype=F32)
    S1, o1, e1 = _run(_chunked_ws, inp)
    S2, o2, e2 = _run(L.la_state_scan_chunked_noalloc, inp)
    S3, o3, e3 = _run(L.la_state_scan_chunked_noalloc, inp)  # the fixed workspace is reused
    assert e1 == e2 == e3 == 0
    assert torch.equal(S1, S2) and torch.equal(o1, o2) and torch.equal(S2, S3) and torch.equal(o2, o3)
    S_ref, o_ref, _ = oracle_scan(inp, dst_dtype=F32)
    assert_close(np64(S2), S_ref, 2e-2, f"{rule}: final states")
    assert_close(np64(o2), o_ref, 2e-2, f"{rule}: outputs")


def test_noalloc_refuses_work_beyond_its_workspace():
    # real buffers, but a token count whose workspace would pass 256 MiB: refused on the host
    inp = W.scan_inputs(lengths=[64], n_qk_heads=1, n_v_heads=32, d_k=128, d_v=128, io_dtype=BF16, seed=62)
    need = L.la_scan_chunked_workspace_bytes(1 << 20, 1, 32)
    assert need > (256 << 20)
    dst_t = torch.zeros(1, 32, 128, 128, dtype=F32, device="cuda")
    o = torch.zeros(64, 32, 128, dtype=BF16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, k, v, g, b, cu = dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.g), dev(inp.beta), dev(inp.cu_seqlens)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = L.lib().la_state_scan_chunked_noalloc(3, None, None, L.Pool(dst_t, 32).ref, None, 1, P(cu), 1 << 20, None,
                                               P(q), P(k), P(v), L.LA_BF16, P(g), P(b), 1.0, P(o), P(err),
                                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == L.LA_ERR_SHAPE
    torch.cuda.synchronize()
    assert int(err.item()) == 0
