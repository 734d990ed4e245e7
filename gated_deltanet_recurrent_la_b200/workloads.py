"""Seeded synthetic inputs for the recurrent-state step.

This module holds input generation only -- none of the method's arithmetic.  Tests,
the oracle side, the smoke check and the benchmark all draw their inputs from here,
on the host CPU with a seeded torch generator, so both sides see identical bytes.
BF16 values are rounded once here (torch's round-to-nearest-even conversion), before
either side sees them.

Distributions (the workloads the pages describe; no dataset is involved):
  q, k ~ N(0, 1), each head vector L2-normalised     (delta-rule keys are unit vectors)
  v    ~ N(0, 1)
  g    = exp(-softplus(N(0, 1)))                      gate in (0, 1); kda: one per key channel
  beta = sigmoid(N(0, 1))                             write strength in (0, 1)
  pool = N(0, 0.05) initial states (decode workloads)

Named workloads (sizes from the "SSM / linear-RNN decode" page, the ONNX section of
"Seven Architectures ...", and the serving scenario of the glossary pages):
  tiny        2 sequences x 64 tokens, 2 heads, d_k = d_v = 16, FP32, all four rules
  decode64    B=64 decode, 16 q/k heads : 32 state heads, 128 x 128, BF16 state, 256-slot pool
  decode512   B=512, same heads, 1024-slot pool, half the requests read a checkpoint slot
  prefill32   32 packed sequences, lengths U_int[1024, 8192], 32 heads, 128 x 128 scan
  mamba2      B=256 gated decode, 128 heads x 64, d_state 128 (Nemotron-H-8B layer sizes)
  kda_decode64, kda_prefill32   the same shapes with the channel-wise (kda) gate
  qgroup_decode256  B=256 decode, 16 state heads each read by 4 query heads (ONNX direction)
  q8_decode64 decode64 on the mixed INT8 / BF16 state storage (1/8 of the key channels BF16)
  conv_decode64  decode64 with the short causal convolution (width 4, SiLU, q/k norm) ahead
  conv_prefill32 prefill32 with the same convolution ahead of every token (fresh prefill)
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch

RULES = ("linear", "gated", "delta", "gated_delta")
# kda: the channel-wise gate of Kimi Delta Attention (g holds d_k decays per token and head)
ALL_RULES = RULES + ("kda",)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


@dataclass
class Inputs:
    """One call's worth of inputs (host tensors)."""
    kind: str                      # "step" or "scan"
    rule: str
    n_qk_heads: int
    n_v_heads: int
    d_k: int
    d_v: int
    state_dtype: torch.dtype       # dtype of the destination pool
    io_dtype: torch.dtype
    q: torch.Tensor                # [B|T, H_qk, d_k] io dtype
    k: torch.Tensor
    v: torch.Tensor                # [B|T, H_v, d_v] io dtype
    g: Optional[torch.Tensor]      # [B|T, H_v] float32 ([B|T, H_v, d_k] for kda)
    beta: Optional[torch.Tensor]
    scale: float = 1.0
    pool: Optional[torch.Tensor] = None        # source pool [n_slots, H_v, d_k, d_v]
    read_slot: Optional[torch.Tensor] = None   # int32
    write_slot: Optional[torch.Tensor] = None  # int32
    cu_seqlens: Optional[torch.Tensor] = None  # int32 [n_seqs + 1] (scan)
    extra: dict = field(default_factory=dict)
    # > 0: the query-group direction of the ONNX operator -- k has one head per state head
    # (n_qk_heads == n_v_heads), q and o have n_q_heads heads
    n_q_heads: int = 0

    @property
    def batch(self) -> int:
        return int(self.q.shape[0]) if self.kind == "step" else int(self.cu_seqlens.numel() - 1)


def token_operands(n_tok, n_qk_heads, n_v_heads, d_k, d_v, io_dtype, gen, *, normalise_qk=True,
                   g_mode="exp_neg_softplus", beta_mode="sigmoid", channel_gate=False):
    """q, k, v, g, beta for n_tok tokens (or requests), drawn in that order from gen.
    channel_gate: g has one decay per key channel, [n_tok, H_v, d_k] (kda)."""
    q = torch.randn(n_tok, n_qk_heads, d_k, generator=gen)
    k = torch.randn(n_tok, n_qk_heads, d_k, generator=gen)
    if normalise_qk:
        q, k = _unit(q), _unit(k)
    v = torch.randn(n_tok, n_v_heads, d_v, generator=gen)
    gshape = (n_tok, n_v_heads, d_k) if channel_gate else (n_tok, n_v_heads)
    zg = torch.randn(*gshape, generator=gen)
    zb = torch.randn(n_tok, n_v_heads, generator=gen)
    if g_mode == "exp_neg_softplus":
        g = torch.exp(-torch.nn.functional.softplus(zg))
    elif g_mode == "uniform_pm1":          # gate range [-1, 1] ("Complex KDA" section)
        g = torch.rand(*gshape, generator=gen) * 2 - 1
    elif g_mode == "one":
        g = torch.ones(*gshape)
    else:
        raise ValueError(g_mode)
    if beta_mode == "sigmoid":
        beta = torch.sigmoid(zb)
    elif beta_mode == "uniform_0_2":       # beta range [0, 2] ("Complex KDA" section)
        beta = torch.rand(n_tok, n_v_heads, generator=gen) * 2
    elif beta_mode == "zero":
        beta = torch.zeros(n_tok, n_v_heads)
    elif beta_mode == "one":
        beta = torch.ones(n_tok, n_v_heads)
    else:
        raise ValueError(beta_mode)
    return (q.to(io_dtype).contiguous(), k.to(io_dtype).contiguous(), v.to(io_dtype).contiguous(),
            g.float().contiguous(), beta.float().contiguous())


def random_pool(n_slots, n_v_heads, d_k, d_v, dtype, gen, std=0.05):
    """Initial states N(0, std^2), generated slot by slot to bound host memory."""
    out = torch.empty(n_slots, n_v_heads, d_k, d_v, dtype=dtype)
    for s in range(n_slots):
        out[s] = (torch.randn(n_v_heads, d_k, d_v, generator=gen) * std).to(dtype)
    return out


def _query_groups(inp: Inputs, n_q_heads: int, gen, normalise_qk: bool) -> Inputs:
    """Switch inputs to the query-group direction: n_q_heads queries per row, drawn after
    everything else (so the other operands are those of the default direction)."""
    if n_q_heads:
        assert inp.n_qk_heads == inp.n_v_heads and n_q_heads % inp.n_v_heads == 0
        q = torch.randn(inp.q.shape[0], n_q_heads, inp.d_k, generator=gen)
        inp.q = (_unit(q) if normalise_qk else q).to(inp.io_dtype).contiguous()
        inp.n_q_heads = n_q_heads
    return inp


def step_inputs(*, B, n_qk_heads, n_v_heads, d_k, d_v, rule="gated_delta", n_slots=None,
                state_dtype=torch.bfloat16, io_dtype=torch.bfloat16, seed=0, slot_map="perm",
                pool_std=0.05, g_mode="exp_neg_softplus", beta_mode="sigmoid", normalise_qk=True,
                scale=1.0, n_q_heads=0) -> Inputs:
    """A decode step.  slot_map: "perm" (read = write = randperm(n_slots)[:B]),
    "dense" (no slot arrays), or "checkpoint" (half of the requests read a checkpoint slot
    and write a distinct live slot, the rest update in place)."""
    gen = _gen(seed)
    n_slots = B if n_slots is None else n_slots
    pool = random_pool(n_slots, n_v_heads, d_k, d_v, state_dtype, gen, pool_std)
    read_slot = write_slot = None
    if slot_map == "perm":
        perm = torch.randperm(n_slots, generator=gen)[:B].to(torch.int32)
        read_slot, write_slot = perm.clone(), perm.clone()
    elif slot_map == "checkpoint":
        perm = torch.randperm(n_slots, generator=gen).to(torch.int32)
        live = perm[:B].clone()
        ckpt = perm[B:B + B // 2].clone()
        assert ckpt.numel() == B // 2, "checkpoint map needs n_slots >= 1.5 B"
        branch = torch.randperm(B, generator=gen)[:B // 2]
        read_slot = live.clone()
        read_slot[branch] = ckpt
        write_slot = live
    elif slot_map != "dense":
        raise ValueError(slot_map)
    q, k, v, g, beta = token_operands(B, n_qk_heads, n_v_heads, d_k, d_v, io_dtype, gen,
                                      normalise_qk=normalise_qk, g_mode=g_mode, beta_mode=beta_mode,
                                      channel_gate=rule == "kda")
    return _query_groups(Inputs("step", rule, n_qk_heads, n_v_heads, d_k, d_v, state_dtype, io_dtype, q, k, v, g,
                                beta, scale, pool, read_slot, write_slot), n_q_heads, gen, normalise_qk)


def scan_inputs(*, lengths, n_qk_heads, n_v_heads, d_k, d_v, rule="gated_delta",
                state_dtype=torch.bfloat16, io_dtype=torch.bfloat16, seed=0, init="zero",
                init_dtype=torch.float32, pool_std=0.05, g_mode="exp_neg_softplus",
                beta_mode="sigmoid", normalise_qk=True, scale=1.0, n_q_heads=0) -> Inputs:
    """Packed varlen prefill.  init: "zero" (no read slots) or "slots" (initial states
    read from a pool of init_dtype, read_slot = randperm)."""
    gen = _gen(seed)
    lengths = [int(x) for x in lengths]
    n_seqs = len(lengths)
    cu = torch.zeros(n_seqs + 1, dtype=torch.int32)
    if n_seqs:
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
    T = int(cu[-1])
    pool = read_slot = None
    if init == "slots":
        pool = random_pool(n_seqs, n_v_heads, d_k, d_v, init_dtype, gen, pool_std)
        read_slot = torch.randperm(n_seqs, generator=gen).to(torch.int32)
    elif init != "zero":
        raise ValueError(init)
    q, k, v, g, beta = token_operands(T, n_qk_heads, n_v_heads, d_k, d_v, io_dtype, gen,
                                      normalise_qk=normalise_qk, g_mode=g_mode, beta_mode=beta_mode,
                                      channel_gate=rule == "kda")
    return _query_groups(Inputs("scan", rule, n_qk_heads, n_v_heads, d_k, d_v, state_dtype, io_dtype, q, k, v, g,
                                beta, scale, pool, read_slot, None, cu), n_q_heads, gen, normalise_qk)


# ---- the named workloads ----------------------------------------------------------

def tiny(rule: str, seed: int = 0) -> Inputs:
    """2 sequences x 64 tokens, 2 heads, 16 x 16, FP32 state and io, zero initial state."""
    return scan_inputs(lengths=[64, 64], n_qk_heads=2, n_v_heads=2, d_k=16, d_v=16, rule=rule,
                       state_dtype=torch.float32, io_dtype=torch.float32, seed=seed)


def decode64(seed: int = 0) -> Inputs:
    """Batched decode: B=64, 16 q/k heads shared by 32 state heads, 128 x 128, BF16 state,
    256-slot pool, read = write = randperm(256)[:64]."""
    return step_inputs(B=64, n_qk_heads=16, n_v_heads=32, d_k=128, d_v=128, n_slots=256, seed=seed,
                       slot_map="perm")


def kda_decode64(seed: int = 0) -> Inputs:
    """decode64 with the channel-wise gate of Kimi Delta Attention (d_k decays per head)."""
    return step_inputs(B=64, n_qk_heads=16, n_v_heads=32, d_k=128, d_v=128, n_slots=256, seed=seed,
                       slot_map="perm", rule="kda")


def qgroup_decode256(seed: int = 0) -> Inputs:
    """Decode in the query-group direction of the ONNX operator: B=256, 16 KV (state) heads
    each read by 4 query heads (64 query heads), 128 x 128 BF16 state, 1024-slot pool,
    read = write = randperm(1024)[:256]."""
    return step_inputs(B=256, n_qk_heads=16, n_v_heads=16, d_k=128, d_v=128, n_slots=1024, seed=seed,
                       slot_map="perm", n_q_heads=64)


def hp_masks(n_v_heads: int, d_k: int, n_hp: int, gen: torch.Generator) -> torch.Tensor:
    """Channel masks of a q8 pool: for each head, n_hp key channels drawn at random (an
    offline calibration would choose them; none is done here).  int32 [H_v, d_k / 32]
    holding the uint32 mask words."""
    words = torch.zeros(n_v_heads, d_k // 32, dtype=torch.int64)
    for h in range(n_v_heads):
        for i in torch.randperm(d_k, generator=gen)[:n_hp].tolist():
            words[h, i // 32] |= 1 << (i % 32)
    return ((words + 2 ** 31) % 2 ** 32 - 2 ** 31).to(torch.int32)


def q8_decode64(seed: int = 0, n_hp: int = 16) -> Inputs:
    """decode64 on a q8 pool (INT8 state with 1/8 of the key channels in BF16, 9.875 bits
    per value): FP32 initial values N(0, 0.05) (encoded into the pool by the library),
    channel masks drawn at random, the masks and n_hp in `extra`."""
    inp = step_inputs(B=64, n_qk_heads=16, n_v_heads=32, d_k=128, d_v=128, n_slots=256, seed=seed,
                      slot_map="perm", state_dtype=torch.float32)
    inp.state_dtype = torch.uint8  # marks the q8 storage
    inp.extra = {"n_hp": n_hp, "hp_mask": hp_masks(32, 128, n_hp, _gen(seed + 7))}
    return inp


def conv_decode64(seed: int = 0, width: int = 4) -> Inputs:
    """decode64 with the short causal convolution ahead of the step: q, k, v are the
    convolution's inputs (N(0, 1), not normalised), weights N(0, 1 / W) per channel, the
    histories N(0, 1) in BF16 [256 slots, 32 heads, 2 * 128 + 128, W - 1]; SiLU and the q/k
    normalisation on (`extra`)."""
    inp = step_inputs(B=64, n_qk_heads=16, n_v_heads=32, d_k=128, d_v=128, n_slots=256, seed=seed,
                      slot_map="perm", normalise_qk=False)
    gen = _gen(seed + 11)
    W = width
    inp.extra = {
        "width": W, "activation": 1, "qk_l2norm": 1,
        "w_q": (torch.randn(16, 128, W, generator=gen) / W ** 0.5).contiguous(),
        "w_k": (torch.randn(16, 128, W, generator=gen) / W ** 0.5).contiguous(),
        "w_v": (torch.randn(32, 128, W, generator=gen) / W ** 0.5).contiguous(),
        "hist": torch.randn(256, 32, 3 * 128, W - 1, generator=gen).to(torch.bfloat16).contiguous(),
    }
    return inp


def decode512(seed: int = 0) -> Inputs:
    """Large decode: B=512, same heads, 1024-slot pool; half the requests read a
    checkpoint slot and write a distinct live slot, the rest update in place."""
    return step_inputs(B=512, n_qk_heads=16, n_v_heads=32, d_k=128, d_v=128, n_slots=1024, seed=seed,
                       slot_map="checkpoint")


def prefill32_lengths(seed: int = 0, n_seqs: int = 32, lo: int = 1024, hi: int = 8192):
    return [int(x) for x in torch.randint(lo, hi + 1, (n_seqs,), generator=_gen(seed))]


def prefill32(seed: int = 0, n_seqs: int = 32) -> Inputs:
    """Token-serial prefill: packed sequences with lengths U_int[1024, 8192], 32 heads,
    128 x 128, FP32 state on chip, zero initial state, BF16 final state and io."""
    return scan_inputs(lengths=prefill32_lengths(seed, n_seqs), n_qk_heads=32, n_v_heads=32, d_k=128,
                       d_v=128, seed=seed + 1)


def kda_prefill32(seed: int = 0, n_seqs: int = 32) -> Inputs:
    """prefill32 with the channel-wise gate of Kimi Delta Attention."""
    return scan_inputs(lengths=prefill32_lengths(seed, n_seqs), n_qk_heads=32, n_v_heads=32, d_k=128,
                       d_v=128, seed=seed + 1, rule="kda")


def conv_prefill32(seed: int = 0, n_seqs: int = 32, width: int = 4) -> Inputs:
    """prefill32 with the short causal convolution ahead of every token (fresh prefill:
    zero histories): q, k, v are the convolution's inputs (N(0, 1), not normalised),
    weights N(0, 1 / W), SiLU and the q/k normalisation on (`extra`)."""
    inp = scan_inputs(lengths=prefill32_lengths(seed, n_seqs), n_qk_heads=32, n_v_heads=32, d_k=128, d_v=128,
                      seed=seed + 1, normalise_qk=False)
    gen = _gen(seed + 13)
    inp.extra = {
        "width": width, "activation": 1, "qk_l2norm": 1,
        "w_q": (torch.randn(32, 128, width, generator=gen) / width ** 0.5).contiguous(),
        "w_k": (torch.randn(32, 128, width, generator=gen) / width ** 0.5).contiguous(),
        "w_v": (torch.randn(32, 128, width, generator=gen) / width ** 0.5).contiguous(),
    }
    return inp


def mamba2(seed: int = 0, B: int = 256) -> Inputs:
    """Mamba-2-style gated decode read as the gated rule: d_inner 8192 = 128 heads x 64
    (d_v), d_state N = 128 (d_k), one B/C group (H_qk = 1).  k := B_t, q := C_t (both
    N(0,1), not normalised), v := dt * x with x ~ N(0,1), g := exp(dt * A) with
    dt = softplus(N(0,1)) per (request, head) and A = -exp(U(0,2)) per head.  BF16 state,
    dense in-place pool of B slots."""
    gen = _gen(seed)
    H, N, P = 128, 128, 64
    pool = random_pool(B, H, N, P, torch.bfloat16, gen, 0.05)
    Bt = torch.randn(B, 1, N, generator=gen)
    Ct = torch.randn(B, 1, N, generator=gen)
    x = torch.randn(B, H, P, generator=gen)
    dt = torch.nn.functional.softplus(torch.randn(B, H, generator=gen))
    A = -torch.exp(torch.rand(H, generator=gen) * 2)
    g = torch.exp(dt * A[None, :]).float().contiguous()
    v = (dt[:, :, None] * x).to(torch.bfloat16).contiguous()
    return Inputs("step", "gated", 1, H, N, P, torch.bfloat16, torch.bfloat16,
                  Ct.to(torch.bfloat16).contiguous(), Bt.to(torch.bfloat16).contiguous(), v, g, None,
                  1.0, pool, None, None)


WORKLOADS = {
    "decode64": decode64,
    "decode512": decode512,
    "prefill32": prefill32,
    "mamba2": mamba2,
    "kda_decode64": kda_decode64,
    "kda_prefill32": kda_prefill32,
    "qgroup_decode256": qgroup_decode256,
    "q8_decode64": q8_decode64,
    "conv_decode64": conv_decode64,
    "conv_prefill32": conv_prefill32,
}
