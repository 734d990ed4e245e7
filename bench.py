"""Benchmark of the recurrent-state step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode512|decode64|mamba2|prefill32|...] [--rows all|none]

Prints ONE JSON line.  The headline workload is the largest single-GPU configuration of the
batched decode step the metric is quoted on (decode512: B=512 requests, 16 q/k heads shared
by 32 state heads, 128 x 128 BF16 state in a 1024-slot pool, half the requests reading a
prefix-cache checkpoint slot and writing a distinct live slot, gated_delta).  One step = one
call of la_state_step over the batch (slot gather, load, S^T k / S^T q reductions, delta
vector, update, readout, store: every row of the decode path).  `value` = algorithmic
state-update bytes of all ranks / device time of one step (max over ranks), in GB/s; `e2e`
is the same metric measured through the same C-ABI call with the step's inputs copied from
pinned host memory and its output copied back inside the timed region.

Timing: W untimed warm-up steps, then K steps back to back between CUDA events on the
launching stream, bracketed by a barrier and a device synchronize.  decode512 moves 1 GiB of
state per step through a 1 GiB pool (the 126 MB L2 holds an eighth of one step's traffic); a
second figure with an L2 flush (a 256 MiB write) before every step is reported beside it.
The other workloads (decode64, mamba2, the token-serial and chunked prefills, the kda /
query-group / q8 / convolution variants, the pool copy) are measured under `rows`, and a
compact summary of every row closes the line (`rows_summary`).

With --gpus N (launched by torchrun) every rank runs its own replica of the workload
on its own GPU: the step has no exchange between GPUs (every (request, head) tile is
independent), so there is no collective on the data path; ranks only meet at the
barriers and the final max-over-ranks of the elapsed time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "state-update HBM GB/s (% of B200 peak) and decode tokens/s per layer step"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_SM_MHZ = 1965.0
FALLBACK_BF16_TFLOPS = 1590.0
FP32_LANES_PER_SM = 128

# --------------------------------------------------------------------------------------
# byte / flop model (algorithmic: what the method must move, no re-reads)


def step_bytes_and_flops(*, B, n_qk_heads, n_v_heads, d_k, d_v, state_bytes, io_bytes, rule, state_only=False,
                         slot_arrays=0, n_q_heads=0):
    """Bytes and flops of one decode step over B requests.

    Bytes: the state is read and written once per (request, head) tile; q and k once
    per q/k head; v and o once per state head; g and beta (4 bytes) where the rule uses
    them (kda: d_k decays of 4 bytes); int32 slot ids.  Flops: 6 per state element
    (S^T k, S^T q and the update, 2 each), the count of the "SSM / linear-RNN decode"
    page.  Query-group direction (n_q_heads > 0): k per state head, n_q_heads query and
    output rows, 2 more flops per state element for each extra query of a group."""
    elems = B * n_v_heads * d_k * d_v
    state = 2 * elems * state_bytes
    group = n_q_heads // n_v_heads if n_q_heads else 1
    flops = (4 + 2 * group) * elems
    if state_only:
        return state, flops
    n_q = n_q_heads if n_q_heads else n_qk_heads
    n_o = n_q_heads if n_q_heads else n_v_heads
    qk = B * (n_q + n_qk_heads) * d_k * io_bytes
    vo = B * (n_v_heads + n_o) * d_v * io_bytes
    return state + qk + vo + B * gate_bytes_per_head(rule, d_k) * n_v_heads + 4 * B * slot_arrays, flops


def gate_bytes_per_head(rule, d_k):
    """FP32 gate and beta bytes of one token and state head."""
    g = {"gated": 4, "gated_delta": 4, "kda": 4 * d_k}.get(rule, 0)
    return g + (4 if rule in ("delta", "gated_delta", "kda") else 0)


def scan_bytes_and_flops(*, T, n_seqs, n_qk_heads, n_v_heads, d_k, d_v, io_bytes, rule, final_state_bytes,
                         init_state_bytes=0):
    """Bytes and flops of one scan: every token's q, k (per q/k head), v, o (per state
    head), gates; the final state stored once (and read once when initialised)."""
    per_tok = 2 * n_qk_heads * d_k * io_bytes + 2 * n_v_heads * d_v * io_bytes
    per_tok += n_v_heads * gate_bytes_per_head(rule, d_k)
    state = n_seqs * n_v_heads * d_k * d_v * (final_state_bytes + init_state_bytes)
    return T * per_tok + state + 4 * (n_seqs + 1), 6 * T * n_v_heads * d_k * d_v


# --------------------------------------------------------------------------------------
# peaks, clocks, traffic evidence


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return {"hbm_gbs": float(d["hbm_gbs"]), "sm_max_mhz": float(d.get("sm_max_mhz", FALLBACK_SM_MHZ)),
                "bf16_tflops": float(d.get("bf16_tflops", FALLBACK_BF16_TFLOPS)), "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "sm_max_mhz": FALLBACK_SM_MHZ, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "source": "fallback"}


def fp32_alu_peak_tflops(sm_count, mhz):
    """FP32 FMA roofline: SMs x 128 FP32 lanes x 2 flops x clock."""
    return sm_count * FP32_LANES_PER_SM * 2 * mhz * 1e6 / 1e12


def kernel_source_hash(files):
    """Hash of the kernel's source code with comments and blank lines dropped, so that a
    recorded capture stays attached to the code it measured and not to its comments."""
    import re
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "gated_deltanet_recurrent_la_b200", "csrc", f), "r", encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update("\n".join(l.rstrip() for l in text.splitlines() if l.strip()).encode())
    return h.hexdigest()[:16]


KERNEL_SOURCES = {
    "step": ["la_step.cuh", "la_device.cuh"],
    "step_q8": ["la_step_q8.cuh", "la_step.cuh", "la_device.cuh"],
    "scan": ["la_scan.cuh", "la_device.cuh"],
    "chunk": ["la_chunk.cuh", "la_device.cuh"],
    "chunk_tc": ["la_chunk.cuh", "la_chunk_tc.cuh", "la_umma.cuh", "la_device.cuh"],
    "chunk_fused": ["la_chunk.cuh", "la_chunk_fused.cuh", "la_chunk_tc.cuh", "la_umma.cuh", "la_device.cuh"],
    "chunk_kda": ["la_chunk.cuh", "la_chunk_kda.cuh", "la_chunk_fused.cuh", "la_chunk_tc.cuh", "la_umma.cuh",
                  "la_device.cuh"],
    "chunk_conv": ["la_chunk_conv.cuh", "la_chunk.cuh", "la_chunk_fused.cuh", "la_chunk_tc.cuh", "la_umma.cuh",
                   "la_device.cuh"],
    "pool": ["la_pool.cu"],
}


def step_kernel(workload):
    """(traffic key, kernel name) of a decode workload's kernel: q8 pools sharing one mask
    array run the storage-order q8 kernel, every other step the generic step kernel."""
    return ("step_q8", "la::step_q8s_kernel") if workload == "q8_decode64" else ("step", "la::step_kernel")


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary (profiles/traffic.json), or
    None when there is none or the kernel source changed since it was captured."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
            rec = json.load(fh).get(f"{kernel}/{workload}")
    except Exception:
        return None
    if not rec or rec.get("source_hash") != kernel_source_hash(KERNEL_SOURCES[kernel]):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML (read only) in a
    background thread; `window()` keeps the samples taken between mark_start/mark_end."""

    HW_BAD = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")

    def __init__(self, device_index, period_s=0.002):
        self.samples = []
        self.period = period_s
        self.ok = False
        self.t0 = self.t1 = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that, do not guess
            self.err = str(e)
        self._stop = threading.Event()
        self._th = threading.Thread(target=self._run, daemon=True)

    def _reasons(self, bits):
        nv = self.nv
        names = {"hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
                 "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
                 "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
                 "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
                 "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
                 "gpu_idle": getattr(nv, "nvmlClocksEventReasonGpuIdle", 0x1)}
        return [k for k, v in names.items() if bits & v]

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    bits = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, bits))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._th.start()

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def stop(self):
        if self.ok:
            self._stop.set()
            self._th.join(timeout=2)

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": "NVML unavailable"}
        win = [s for s in self.samples if self.t0 is not None and self.t0 <= s[0] <= (self.t1 or s[0])]
        if not win:  # region shorter than one poll: take the nearest samples
            win = sorted(self.samples, key=lambda s: abs(s[0] - (self.t0 or 0)))[:3]
        reasons = set()
        for _, _, bits in win:
            reasons.update(self._reasons(bits))
        return {"sm_mhz": statistics.median([m for _, m, _ in win]) if win else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(win)}


# --------------------------------------------------------------------------------------
# distributed plumbing (one process per GPU; replicas)


def dist_setup(n_gpus):
    """One process per GPU from torchrun's environment (RANK, LOCAL_RANK, WORLD_SIZE,
    MASTER_*).  NCCL when CUDA is present, gloo otherwise (the CPU tests of this logic).
    The process group only carries barriers and the max-over-ranks of the elapsed time."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(per_rank_units, max_ms, world):
    """Whole-job throughput: units processed by all ranks / the slowest rank's time."""
    return per_rank_units * world / (max_ms * 1e-3)


# --------------------------------------------------------------------------------------
# device workloads


def to_dev(t):
    return None if t is None else t.cuda().contiguous()


class DecodeRunner:
    """Holds one decode workload on the device and launches la_state_step on it, with
    `n_sets` disjoint slot sets rotated from step to step."""

    def __init__(self, inp, n_sets=1, seed=0):
        import torch
        from gated_deltanet_recurrent_la_b200 import lastate as L
        self.L = L
        self.torch = torch
        self.inp = inp
        if inp.state_dtype == torch.uint8:
            # q8 storage: the FP32 initial values are encoded into the pool by the library
            n_hp, mask = inp.extra["n_hp"], to_dev(inp.extra["hp_mask"])
            n, H, dk, dv = inp.pool.shape
            self.pool_t = torch.zeros(n, H, L.q8_tile_bytes(dk, dv, n_hp), dtype=torch.uint8, device="cuda")
            self.pool = L.Pool.q8(self.pool_t, inp.n_qk_heads, dk, dv, n_hp, mask)
            err = torch.zeros(1, dtype=torch.int32, device="cuda")
            L.check(L.la_state_pool_encode(self.pool, torch.arange(n, dtype=torch.int32, device="cuda"),
                                           to_dev(inp.pool.float()), err))
            torch.cuda.synchronize()
            if int(err.item()):
                raise RuntimeError(f"q8 encode reported {int(err.item())}")
        else:
            self.pool_t = to_dev(inp.pool)
            self.pool = L.Pool(self.pool_t, inp.n_qk_heads)
        self.conv = None
        if "width" in inp.extra:  # the short causal convolution ahead of the step
            x = inp.extra
            self.hist_t = to_dev(x["hist"])
            self.conv = L.Conv(to_dev(x["w_q"]), to_dev(x["w_k"]), to_dev(x["w_v"]), self.hist_t,
                               activation=x["activation"], qk_l2norm=x["qk_l2norm"])
        self.q, self.k, self.v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
        self.g, self.beta = to_dev(inp.g), to_dev(inp.beta)
        B = inp.q.shape[0]
        self.o = torch.empty(B, inp.n_q_heads or inp.n_v_heads, inp.d_v, dtype=inp.io_dtype, device="cuda")
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.sets = []
        if inp.read_slot is None:
            self.sets = [(None, None)]
        else:
            n_slots = inp.pool.shape[0]
            if n_sets > 1:
                assert n_sets * B <= n_slots
                rest = [s for s in range(n_slots) if s not in set(inp.write_slot.tolist()) | set(inp.read_slot.tolist())]
                g = torch.Generator().manual_seed(seed + 101)
                perm = torch.tensor(rest)[torch.randperm(len(rest), generator=g)]
                self.sets.append((inp.read_slot, inp.write_slot))
                for i in range(1, n_sets):
                    s = perm[(i - 1) * B:i * B].to(torch.int32)
                    self.sets.append((s, s))
            else:
                self.sets.append((inp.read_slot, inp.write_slot))
            self.sets = [(to_dev(r), to_dev(w)) for r, w in self.sets]
        self.B = B

    def call(self, r, w, q, k, v, g, beta, o, stream=None):
        """One decode step through the C ABI (the query-group entry point when the
        workload has query groups)."""
        if self.conv is not None:
            st = self.L.la_state_step_conv(self.inp.rule, self.pool, r, self.pool, w, self.conv, q, k, v, g, beta,
                                           self.inp.scale, o, self.err, stream=stream)
        else:
            fn = self.L.la_state_step_qgroups if self.inp.n_q_heads else self.L.la_state_step
            st = fn(self.inp.rule, self.pool, r, self.pool, w, q, k, v, g, beta, self.inp.scale, o, self.err,
                    stream=stream)
        if st != 0:
            raise self.L.LAError(st)

    def step(self, i=0, stream=None):
        r, w = self.sets[i % len(self.sets)]
        self.call(r, w, self.q, self.k, self.v, self.g, self.beta, self.o, stream)

    def bytes_flops(self):
        i = self.inp
        b, f = step_bytes_and_flops(B=self.B, n_qk_heads=i.n_qk_heads, n_v_heads=i.n_v_heads, d_k=i.d_k, d_v=i.d_v,
                                    state_bytes=state_bytes_per_value(i), io_bytes=i.q.element_size(), rule=i.rule,
                                    slot_arrays=0 if i.read_slot is None else 2, n_q_heads=i.n_q_heads)
        if self.conv is not None:
            # histories read and written per (request, head); the weights once
            x = i.extra
            b += 2 * self.B * i.n_v_heads * (2 * i.d_k + i.d_v) * (x["width"] - 1) * i.q.element_size()
            b += 4 * x["width"] * (2 * i.n_qk_heads * i.d_k + i.n_v_heads * i.d_v)
            f += 2 * self.B * i.n_v_heads * (2 * i.d_k + i.d_v) * x["width"]
        return b, f


CHUNK = 64  # tokens per chunk of the tensor-core prefill


def chunk_mma_flops(lengths, n_v_heads, d_k, d_v, rule):
    """Tensor-core flops the chunked prefill executes (whole chunks, the last one padded):
    per chunk and head Q K^T and (Q K^T . M) U (2 C^2 d_k and 2 C^2 d_v), Q S0 and the
    state update K^T U (2 C d_k d_v each); the delta rules add K K^T, W = T K, U~ = T V and
    W S0 (2 C^2 d_k, 2 C^2 d_k, 2 C^2 d_v, 2 C d_k d_v)."""
    C = CHUNK
    per = 2 * C * C * d_k + 2 * C * C * d_v + 4 * C * d_k * d_v
    if rule in ("delta", "gated_delta"):
        per += 4 * C * C * d_k + 2 * C * C * d_v + 2 * C * d_k * d_v
    elif rule == "kda":
        # [Q; K] against the decay-scaled keys by the ten 16 x 16 blocks on and below the
        # diagonal, in place of Q K^T; then W = Tw K+, U~ = Tw V and W S0
        per += 2 * (10 * 32 * 16) * d_k - 2 * C * C * d_k
        per += 2 * C * C * d_k + 2 * C * C * d_v + 2 * C * d_k * d_v
    chunks = sum((int(n) + C - 1) // C for n in lengths)
    return chunks * n_v_heads * per


def chunk_roofline(run, inp, ms, peaks):
    """Roofline object of the chunked prefill.  Its tensor-core work is a dense contraction
    that finishes below the HBM time, so the bound is HBM: the method's algorithmic bytes
    (q, k, v, o, gates of every token, the final state; no re-reads) over the device time,
    against the measured copy bandwidth.  The tensor rate is reported beside it twice: the
    method's own 6 flops per state element and token, and the chunked algorithm's MMA flops
    (which the measured dense BF16 GEMM peak bounds)."""
    lens = (inp.cu_seqlens[1:] - inp.cu_seqlens[:-1]).tolist()
    nbytes, flops = run.bytes_flops()
    gbs = nbytes / (ms * 1e-3) / 1e9
    mma_tf = chunk_mma_flops(lens, inp.n_v_heads, inp.d_k, inp.d_v, inp.rule) / (ms * 1e-3) / 1e12
    peak_tf = peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS)
    conv = run.conv is not None
    two = run.ws is not None and inp.rule in ("delta", "gated_delta") and not conv
    kda = inp.rule == "kda"
    kernel = "chunk_kda" if kda else "chunk_conv" if conv and run.ws is not None else ("chunk_tc" if two else "chunk_fused")
    out = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
           "traffic": recorded_traffic(kernel, ("kda_prefill32" if kda else "conv_prefill32" if conv else "prefill32") +
                                       (f"_ckpt{run.ckpt_every}" if run.ckpt_every else "")),
           "algorithmic_bytes_per_launch": nbytes,
           "method_tflops": flops / (ms * 1e-3) / 1e12,
           "mma_tflops": mma_tf, "mma_frac_of_bf16_peak": mma_tf / peak_tf,
           "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json hbm_gbs; bf16_tflops for mma_frac)"}
    out["kernel"] = ("la::chunk_kda_prep_kernel (mma.sync) + la::chunk_kda_kernel (tcgen05)" if kda else
                     "la::chunk_prep_kernel (mma.sync) + la::chunk_tc_kernel (tcgen05)" if two
                     else "la::chunk_conv_kernel + la::chunk_fused_kernel (tcgen05)" if conv and run.ws is not None
                     else "la::chunk_fused_kernel (tcgen05)" + (", the convolution in the same launch" if conv else ""))
    return out


class ScanRunner:
    """A prefill workload on the device.  ckpt_every > 0: la_state_scan_checkpointed with a
    checkpoint slot for every ckpt_every tokens of every sequence."""

    def __init__(self, inp, ckpt_every=0, chunked=False):
        import torch
        from gated_deltanet_recurrent_la_b200 import lastate as L
        self.L = L
        self.inp = inp
        n_seqs = inp.cu_seqlens.numel() - 1
        self.dst_t = torch.empty(n_seqs, inp.n_v_heads, inp.d_k, inp.d_v, dtype=inp.state_dtype, device="cuda")
        self.dst = L.Pool(self.dst_t, inp.n_qk_heads)
        self.src = None if inp.pool is None else L.Pool(to_dev(inp.pool), inp.n_qk_heads)
        self.read_slot = to_dev(inp.read_slot)
        self.cu = to_dev(inp.cu_seqlens)
        lens = (inp.cu_seqlens[1:] - inp.cu_seqlens[:-1]).tolist()
        order = sorted(range(n_seqs), key=lambda s: -lens[s])  # longest first
        self.order = torch.tensor(order, dtype=torch.int32, device="cuda")
        self.q, self.k, self.v = to_dev(inp.q), to_dev(inp.k), to_dev(inp.v)
        self.g, self.beta = to_dev(inp.g), to_dev(inp.beta)
        self.o = torch.empty(inp.q.shape[0], inp.n_v_heads, inp.d_v, dtype=inp.io_dtype, device="cuda")
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.T = int(inp.q.shape[0])
        self.n_seqs = n_seqs
        self.ckpt_every = ckpt_every
        self.chunked = chunked
        self.n_ckpt = 0
        if ckpt_every > 0:
            n_ck = [l // ckpt_every for l in lens]
            self.n_ckpt = sum(n_ck)
            cu = [0]
            for n in n_ck:
                cu.append(cu[-1] + n)
            self.ckpt_cu = torch.tensor(cu, dtype=torch.int32, device="cuda")
            self.ckpt_slots = torch.arange(n_seqs, n_seqs + self.n_ckpt, dtype=torch.int32, device="cuda")
            self.dst_t = torch.empty(n_seqs + self.n_ckpt, inp.n_v_heads, inp.d_k, inp.d_v, dtype=inp.state_dtype,
                                     device="cuda")
            self.dst = L.Pool(self.dst_t, inp.n_qk_heads)
        self.ws = None
        if chunked == "ws":  # the two-launch form: the caller-owned workspace of the intra-chunk part
            nb = (L.la_scan_chunked_conv_workspace_bytes(self.T, inp.n_v_heads) if "width" in inp.extra else
                  L.la_scan_chunked_workspace_bytes_rule(inp.rule, self.T, n_seqs, inp.n_v_heads))
            self.ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        self.conv = None
        if "width" in inp.extra:  # the short causal convolution ahead of every token (fresh prefill)
            x = inp.extra
            self.hist_t = torch.empty(n_seqs, inp.n_v_heads, 2 * inp.d_k + inp.d_v, x["width"] - 1,
                                      dtype=inp.io_dtype, device="cuda")
            self.conv = L.Conv(to_dev(x["w_q"]), to_dev(x["w_k"]), to_dev(x["w_v"]), self.hist_t, self.hist_t,
                               activation=x["activation"], qk_l2norm=x["qk_l2norm"])

    def step(self, i=0, stream=None):
        if self.conv is not None and self.ws is not None:
            st = self.L.la_state_scan_chunked_conv_ws(self.inp.rule, self.src, self.read_slot, self.dst, None, self.cu,
                                                      self.conv, self.q, self.k, self.v, self.g, self.beta,
                                                      self.inp.scale, self.o, self.ws, self.err, seq_order=self.order,
                                                      stream=stream)
        elif self.conv is not None and self.chunked:
            st = self.L.la_state_scan_chunked_conv(self.inp.rule, self.src, self.read_slot, self.dst, None, self.cu,
                                                   self.conv, self.q, self.k, self.v, self.g, self.beta,
                                                   self.inp.scale, self.o, self.err, seq_order=self.order,
                                                   stream=stream)
        elif self.conv is not None:
            st = self.L.la_state_scan_conv(self.inp.rule, self.src, self.read_slot, self.dst, None, self.cu,
                                           self.conv, self.q, self.k, self.v, self.g, self.beta, self.inp.scale,
                                           self.o, self.err, seq_order=self.order, stream=stream)
        elif self.ws is not None:
            st = self.L.la_state_scan_chunked_ws(self.inp.rule, self.src, self.read_slot, self.dst, None, self.cu,
                                                 self.q, self.k, self.v, self.g, self.beta, self.inp.scale, self.o,
                                                 self.ws, self.err, seq_order=self.order, stream=stream)
        elif self.chunked and self.ckpt_every > 0:
            st = self.L.la_state_scan_chunked_checkpointed(self.inp.rule, self.src, self.read_slot, self.dst, None,
                                                           self.cu, self.q, self.k, self.v, self.g, self.beta,
                                                           self.inp.scale, self.o, self.ckpt_every, self.ckpt_cu,
                                                           self.ckpt_slots, self.err, seq_order=self.order,
                                                           stream=stream)
        elif self.chunked:
            st = self.L.la_state_scan_chunked(self.inp.rule, self.src, self.read_slot, self.dst, None, self.cu, self.q,
                                              self.k, self.v, self.g, self.beta, self.inp.scale, self.o, self.err,
                                              seq_order=self.order, stream=stream)
        elif self.ckpt_every > 0:
            st = self.L.la_state_scan_checkpointed(self.inp.rule, self.src, self.read_slot, self.dst, None, self.cu,
                                                   self.q, self.k, self.v, self.g, self.beta, self.inp.scale, self.o,
                                                   self.ckpt_every, self.ckpt_cu, self.ckpt_slots, self.err,
                                                   seq_order=self.order, stream=stream)
        else:
            st = self.L.la_state_scan(self.inp.rule, self.src, self.read_slot, self.dst, None, self.cu, self.q,
                                      self.k, self.v, self.g, self.beta, self.inp.scale, self.o, self.err,
                                      seq_order=self.order, stream=stream)
        if st != 0:
            raise self.L.LAError(st)

    def bytes_flops(self):
        i = self.inp
        b, f = scan_bytes_and_flops(T=self.T, n_seqs=self.n_seqs, n_qk_heads=i.n_qk_heads, n_v_heads=i.n_v_heads,
                                    d_k=i.d_k, d_v=i.d_v, io_bytes=i.q.element_size(), rule=i.rule,
                                    final_state_bytes=self.dst_t.element_size(),
                                    init_state_bytes=0 if i.pool is None else i.pool.element_size())
        b += self.n_ckpt * i.n_v_heads * i.d_k * i.d_v * self.dst_t.element_size()
        if self.conv is not None:  # the final histories and the weights
            x = i.extra
            b += self.n_seqs * i.n_v_heads * (2 * i.d_k + i.d_v) * (x["width"] - 1) * i.q.element_size()
            b += 4 * x["width"] * (2 * i.n_qk_heads * i.d_k + i.n_v_heads * i.d_v)
            f += 2 * self.T * i.n_v_heads * (2 * i.d_k + i.d_v) * x["width"]
        return b, f


class PoolRunner:
    """Prefix-cache checkpoint copies of 64 slots of 1 MiB (the decode64 slot size) inside
    a 1024-slot pool (1 GiB, larger than L2): call i copies slot set 2i mod 16 onto set
    2i+1 mod 16 of 16 disjoint 64-slot sets, so no set is touched twice within 8 calls."""

    def __init__(self, n_sets=16, per_set=64, seed=0):
        import torch
        from gated_deltanet_recurrent_la_b200 import lastate as L
        self.L = L
        g = torch.Generator(device="cuda").manual_seed(seed)
        self.pool_t = torch.randint(-30000, 30000, (n_sets * per_set, 32, 128, 128), dtype=torch.int16,
                                    device="cuda", generator=g).view(torch.bfloat16)
        self.pool = L.Pool(self.pool_t, 16)
        perm = torch.randperm(n_sets * per_set, generator=torch.Generator().manual_seed(seed)).to(torch.int32)
        self.sets = [perm[i * per_set:(i + 1) * per_set].cuda() for i in range(n_sets)]
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step(self, i=0, stream=None):
        n = len(self.sets)
        st = self.L.la_state_pool_copy(self.pool, self.sets[(2 * i) % n], self.sets[(2 * i + 1) % n], self.err,
                                       stream=stream)
        if st != 0:
            raise self.L.LAError(st)

    def bytes_flops(self):
        return 2 * self.sets[0].numel() * self.pool_t[0].numel() * self.pool_t.element_size(), 0


# --------------------------------------------------------------------------------------
# timing


class L2Flush:
    def __init__(self):
        import torch
        props = torch.cuda.get_device_properties(torch.cuda.current_device())
        self.buf = torch.empty(max(2 * props.L2_cache_size, 64 << 20), dtype=torch.uint8, device="cuda")

    def __call__(self):
        self.buf.fill_(1)


def time_back_to_back(run, steps, warmup, world, sampler=None):
    """W warm-up steps, then K steps back to back between two CUDA events on the current
    stream; barrier + synchronize on both sides.  Returns ms per step (max over ranks)."""
    import torch
    for i in range(warmup):
        run.step(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.mark_start()
    e0.record(s)
    for i in range(steps):
        run.step(warmup + i)
    e1.record(s)
    torch.cuda.synchronize()
    if sampler:
        sampler.mark_end()
    barrier(world)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    return max_over_ranks(ms, world)


def time_flushed(run, steps, flush):
    """Each step timed alone between events after an L2 flush (flush outside the events)."""
    import torch
    s = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i, (a, b) in enumerate(evs):
        flush()
        a.record(s)
        run.step(i)
        b.record(s)
    torch.cuda.synchronize()
    return statistics.median([a.elapsed_time(b) for a, b in evs])


def time_e2e(run: DecodeRunner, steps, warmup, world):
    """The decode step through the same C-ABI call with every step's inputs (q, k, v, g,
    beta and the slot ids, one packed buffer) copied from pinned host memory and its
    output o copied back to pinned host memory, all inside the timed region.  The state
    stays resident in the device pool.  Steps are pipelined the way a serving loop would
    run them: device inputs and outputs are double buffered, the host-to-device copy of
    step i+1 and the device-to-host copy of step i-1 run on their own streams while step i
    computes, and chunks of steps are captured in a CUDA graph so that Python launch
    overhead does not bound the loop.  Returns (ms per step, H2D bytes, D2H bytes)."""
    import torch
    inp = run.inp
    L = run.L
    parts = [inp.q, inp.k, inp.v, inp.g, inp.beta]  # g / beta are None for rules that ignore them
    sizes = [0 if p is None else p.numel() * p.element_size() for p in parts] + [run.B * 4, run.B * 4]
    offs, total = [], 0
    for sz in sizes:
        offs.append(total)
        total += (sz + 255) // 256 * 256
    payload = sum(sizes[:5]) + (2 * run.B * 4 if inp.read_slot is not None else 0)
    hosts = []
    for r, w in run.sets:
        hb = torch.zeros(total, dtype=torch.uint8, pin_memory=True)
        for p, off in zip(parts, offs):
            if p is not None:
                hb[off:off + p.numel() * p.element_size()].copy_(p.contiguous().view(-1).view(torch.uint8))
        if r is not None:
            hb[offs[5]:offs[5] + run.B * 4].copy_(r.cpu().view(torch.uint8))
            hb[offs[6]:offs[6] + run.B * 4].copy_(w.cpu().view(torch.uint8))
        hosts.append(hb)
    devs = [torch.empty(total, dtype=torch.uint8, device="cuda") for _ in range(2)]
    outs = [torch.empty_like(run.o) for _ in range(2)]
    o_hosts = [torch.empty(run.o.shape, dtype=run.o.dtype, pin_memory=True) for _ in range(2)]
    o_bytes = o_hosts[0].numel() * o_hosts[0].element_size()

    def views(dev):
        def v(i, dtype, shape):
            n = 1
            for x in shape:
                n *= x
            return dev[offs[i]:offs[i] + n * torch.empty(0, dtype=dtype).element_size()].view(dtype).view(shape)
        return (v(0, inp.q.dtype, inp.q.shape), v(1, inp.k.dtype, inp.k.shape), v(2, inp.v.dtype, inp.v.shape),
                v(3, torch.float32, inp.g.shape) if inp.g is not None else None,
                v(4, torch.float32, inp.beta.shape) if inp.beta is not None else None,
                v(5, torch.int32, (run.B,)) if inp.read_slot is not None else None,
                v(6, torch.int32, (run.B,)) if inp.read_slot is not None else None)
    vs = [views(d) for d in devs]
    sh, sd = torch.cuda.Stream(), torch.cuda.Stream()

    def enqueue(n_steps, first):
        """n_steps pipelined steps on the current stream (+ the two copy streams)."""
        cs = torch.cuda.current_stream()
        fork = torch.cuda.Event()
        fork.record(cs)
        sh.wait_event(fork)
        sd.wait_event(fork)
        kev, dev_free = [None, None], [None, None]
        for j in range(n_steps):
            b = j % 2
            hev = torch.cuda.Event()
            with torch.cuda.stream(sh):
                if kev[b] is not None:
                    sh.wait_event(kev[b])          # step j-2 no longer reads devs[b]
                devs[b].copy_(hosts[(first + j) % len(hosts)], non_blocking=True)
                hev.record(sh)
            cs.wait_event(hev)
            if dev_free[b] is not None:
                cs.wait_event(dev_free[b])         # o of step j-2 has reached the host
            q, k, v, g, beta, rs, ws = vs[b]
            run.call(rs, ws, q, k, v, g, beta, outs[b])
            kev[b] = torch.cuda.Event()
            kev[b].record(cs)
            with torch.cuda.stream(sd):
                sd.wait_event(kev[b])
                o_hosts[b].copy_(outs[b], non_blocking=True)
                dev_free[b] = torch.cuda.Event()
                dev_free[b].record(sd)
        jh, jd = torch.cuda.Event(), torch.cuda.Event()
        jh.record(sh)
        jd.record(sd)
        cs.wait_event(jh)
        cs.wait_event(jd)

    chunk = next(c for c in (16, 8, 4, 2, 1) if steps % c == 0)
    graph = None
    try:
        enqueue(chunk, 0)  # warm-up outside capture
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            enqueue(chunk, 0)
        torch.cuda.synchronize()
    except Exception:
        graph = None  # capture not available: enqueue the same pipeline eagerly
        torch.cuda.synchronize()

    class R:
        @staticmethod
        def step(i):
            if i % chunk:
                return
            if graph is not None:
                graph.replay()
            else:
                enqueue(chunk, i)

    ms = time_back_to_back(R, steps, max(warmup, chunk), world)
    del graph
    return ms, payload, o_bytes


# --------------------------------------------------------------------------------------
# oracle on the host cores (baseline only)


def state_bytes_per_value(inp):
    """Stored bytes per state value of a workload (q8: the tile bytes over d_k x d_v)."""
    import torch
    if inp.state_dtype == torch.uint8:
        n_hp, dk, dv = inp.extra["n_hp"], inp.d_k, inp.d_v
        return ((dk - n_hp) * dv + (dk - n_hp) * (dv // 32) * 4 + n_hp * dv * 2) / (dk * dv)
    return inp.pool.element_size()


def cpu_baseline_decode(inp, budget_s=10.0):
    """The CPU oracle as it stands (fp64, OpenMP over tiles) on the decode workload: whole
    steps repeated until about budget_s of wall time.  Returns (ms per step, threads,
    sample description)."""
    import oracle
    import numpy as np
    pool = inp.pool.double().numpy()
    args = [inp.q.double().numpy(), inp.k.double().numpy(), inp.v.double().numpy(),
            None if inp.g is None else inp.g.double().numpy(), None if inp.beta is None else inp.beta.double().numpy()]
    rs = None if inp.read_slot is None else inp.read_slot.numpy().astype(np.int32)
    ws = None if inp.write_slot is None else inp.write_slot.numpy().astype(np.int32)
    st = "bf16" if inp.state_dtype.itemsize == 2 else "f32"
    io = "bf16" if inp.io_dtype.itemsize == 2 else "f32"
    dst = pool.copy()
    if "width" in inp.extra:
        hist = inp.extra["hist"].double().numpy()
        hist_out = hist.copy()
    times = []
    t_end = time.perf_counter() + budget_s
    while time.perf_counter() < t_end or not times:
        t0 = time.perf_counter()
        if "width" in inp.extra:
            x = inp.extra
            oracle.step_conv(inp.rule, inp.n_qk_heads, pool, *args, inp.scale, x["w_q"].double().numpy(),
                             x["w_k"].double().numpy(), x["w_v"].double().numpy(), hist, act=x["activation"],
                             l2norm=x["qk_l2norm"], dst_pool=dst, conv_dst=hist_out, dst_dtype=st, io_dtype=io,
                             read_slot=rs, write_slot=ws)
        elif inp.state_dtype.itemsize == 1:
            oracle.step_q8(inp.rule, inp.n_qk_heads, pool, *args, inp.scale, dst_pool=dst, io_dtype=io,
                           read_slot=rs, write_slot=ws, masks=inp.extra["hp_mask"].numpy().view(np.uint32))
        elif inp.n_q_heads:
            oracle.step_qgroups(inp.rule, inp.n_q_heads, pool, *args, inp.scale, dst_pool=dst, dst_dtype=st,
                                io_dtype=io, read_slot=rs, write_slot=ws)
        else:
            oracle.step(inp.rule, inp.n_qk_heads, pool, *args, inp.scale, dst_pool=dst, dst_dtype=st, io_dtype=io,
                        read_slot=rs, write_slot=ws)
        times.append(time.perf_counter() - t0)
    return 1e3 * statistics.median(times), oracle.num_threads(), f"{len(times)} whole decode steps of the workload"


def cpu_baseline_scan(inp, n_sub=4, budget_s=10.0, max_tokens=None):
    """The CPU oracle as it stands on a prefill workload, on a fixed subset: the first
    n_sub sequences (all heads; with max_tokens, only that many leading tokens of the first
    sequence), repeated until about budget_s; the rate is scaled to the whole workload by
    bytes and tokens (the oracle's cost is linear in tokens).  Returns (GB/s, tokens/s,
    threads, sample description) or None."""
    import oracle
    import numpy as np
    cu = inp.cu_seqlens.numpy()
    n = min(n_sub, len(cu) - 1)
    if max_tokens is not None:
        n = 1
        cu = np.array([0, min(int(cu[1]), int(max_tokens))], dtype=np.int64)
    t1 = int(cu[n])
    if t1 <= 0:
        return None
    sub = lambda t: None if t is None else t[:t1].double().numpy()  # noqa: E731
    st = "bf16" if inp.state_dtype.itemsize == 2 else "f32"
    io = "bf16" if inp.io_dtype.itemsize == 2 else "f32"
    times = []
    t_end = time.perf_counter() + budget_s
    while time.perf_counter() < t_end or not times:
        t0 = time.perf_counter()
        oracle.scan(inp.rule, inp.n_qk_heads, cu[:n + 1].astype(np.int32), sub(inp.q), sub(inp.k), sub(inp.v),
                    sub(inp.g), sub(inp.beta), inp.scale, dst_dtype=st, io_dtype=io)
        times.append(time.perf_counter() - t0)
    sec = statistics.median(times)
    b, _ = scan_bytes_and_flops(T=t1, n_seqs=n, n_qk_heads=inp.n_qk_heads, n_v_heads=inp.n_v_heads, d_k=inp.d_k,
                                d_v=inp.d_v, io_bytes=inp.q.element_size(), rule=inp.rule,
                                final_state_bytes=inp.state_dtype.itemsize)
    return (b / sec / 1e9, t1 / sec, oracle.num_threads(),
            (f"the first {t1} tokens of sequence 0" if max_tokens is not None else f"sequences 0..{n - 1}") +
            f" of the workload ({t1} tokens, all {inp.n_v_heads} heads), median of {len(times)} runs; rates "
            f"scaled to the whole workload by bytes and tokens")


def cpu_single_thread(fn, *args, **kw):
    """Runs a CPU baseline with the oracle held to one thread (restored afterwards)."""
    import oracle
    n = oracle.num_threads()
    oracle.set_threads(1)
    try:
        return fn(*args, **kw)
    finally:
        oracle.set_threads(n)


# --------------------------------------------------------------------------------------


def build_runner(name, seed=0, prefill_seqs=32, ckpt_every=0, chunked=False):
    from gated_deltanet_recurrent_la_b200 import workloads as W
    if name in ("prefill32", "kda_prefill32", "conv_prefill32"):
        inp = W.WORKLOADS[name](seed, prefill_seqs)
    else:
        inp = W.WORKLOADS[name](seed)
    if inp.kind == "scan":
        return ScanRunner(inp, ckpt_every, chunked), inp
    n_sets = 4 if name in ("decode64", "kda_decode64", "qgroup_decode256", "q8_decode64", "conv_decode64") else 1
    return DecodeRunner(inp, n_sets=n_sets, seed=seed), inp


def describe(name, inp):
    d = {"workload": name, "rule": inp.rule, "n_qk_heads": inp.n_qk_heads, "n_v_heads": inp.n_v_heads,
         "d_k": inp.d_k, "d_v": inp.d_v,
         "state": (f"q8 (INT8 codes, FP32 scale per 32 columns, {inp.extra['n_hp']} of {inp.d_k} key channels "
                   f"BF16)" if inp.state_dtype.itemsize == 1 else str(inp.state_dtype).replace("torch.", "")),
         "io": str(inp.io_dtype).replace("torch.", "")}
    if inp.n_q_heads:
        d["n_q_heads"] = inp.n_q_heads
    if inp.kind == "step":
        d.update(B=int(inp.q.shape[0]), pool_slots=int(inp.pool.shape[0]),
                 slot_map="dense" if inp.read_slot is None else
                 ("checkpoint" if not bool((inp.read_slot == inp.write_slot).all()) else "perm"))
    else:
        lens = (inp.cu_seqlens[1:] - inp.cu_seqlens[:-1])
        d.update(n_seqs=int(lens.numel()), total_tokens=int(inp.cu_seqlens[-1]), min_len=int(lens.min()),
                 max_len=int(lens.max()), init="slots" if inp.pool is not None else "zero",
                 final_state=str(inp.state_dtype).replace("torch.", ""))
    return d


def measure_row(name, steps, warmup, world, peaks, sm_count, flush=None, ckpt_every=0, chunked=False):
    run, inp = build_runner(name, ckpt_every=ckpt_every, chunked=chunked)
    ms = time_back_to_back(run, steps, warmup, world)
    nbytes, flops = run.bytes_flops()
    row = {"config": describe(name, inp), "ms_per_step": ms, "gb_s": nbytes / (ms * 1e-3) / 1e9}
    if inp.kind == "step":
        row["tokens_per_s"] = run.B / (ms * 1e-3)
        row["state_steps_per_s"] = run.B * inp.n_v_heads / (ms * 1e-3)
        row["roofline"] = {"bound": "hbm", "achieved": row["gb_s"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                           "frac": row["gb_s"] / peaks["hbm_gbs"], "traffic": recorded_traffic(step_kernel(name)[0], name),
                           "peak_source": peaks["source"]}
        row["pct_of_spec_8000"] = 100 * row["gb_s"] / SPEC_HBM_GBS
        if flush is not None:
            row["ms_per_step_l2_flushed"] = time_flushed(run, max(10, min(steps, 50)), flush)
    else:
        alu = fp32_alu_peak_tflops(sm_count, peaks["sm_max_mhz"])
        tf = flops / (ms * 1e-3) / 1e12
        row["tokens_per_s"] = run.T / (ms * 1e-3)
        if ckpt_every:
            row["config"]["ckpt_every"] = ckpt_every
            row["config"]["checkpoints"] = run.n_ckpt
        if chunked:
            row["config"]["algorithm"] = "chunked (64-token WY/UT form, BF16 tcgen05 products, FP32 state)" + \
                ("; the decay-scaled operands and intra-chunk products as a separate parallel launch through a "
                 "workspace, then the recurrence with the state in tensor memory" if chunked == "ws" and
                 inp.rule == "kda" else
                 "; intra-chunk inverses as a separate parallel launch through a workspace, then the recurrence "
                 "with the state in tensor memory" if chunked == "ws" else
                 "; one launch, the intra-chunk inverses computed on chip beside the recurrence") + \
                ("; the convolution as a launch of its own, its output through a workspace" if run.conv is not None
                 and chunked == "ws" else
                 "; the convolution of every staged chunk in the same launch" if run.conv is not None else "")
            row["roofline"] = chunk_roofline(run, inp, ms, peaks)
        else:
            row["roofline"] = {"bound": "alu", "achieved": tf, "peak": alu, "unit": "TFLOP/s", "frac": tf / alu,
                               "traffic": recorded_traffic("scan", name + (f"_ckpt{ckpt_every}" if ckpt_every else "")),
                               "hbm_gb_s": row["gb_s"],
                               "effective_state_gb_s": run.T * inp.n_v_heads * 2 * inp.d_k * inp.d_v * 4 /
                               (ms * 1e-3) / 1e9,
                               "peak_note": "SMs x 128 FP32 lanes x 2 x max SM clock"}
    del run
    return row


def build_runner_inputs(name, seed=0):
    """The host inputs of a workload (no device buffers)."""
    from gated_deltanet_recurrent_la_b200 import workloads as W
    return W.WORKLOADS[name](seed)


def rows_summary(rows):
    """One short entry per row (time, achieved rate, roofline fraction), so that every
    row's figures sit at the end of the printed line."""
    out = {}
    for name, r in rows.items():
        rf = r.get("roofline", {})
        e = {"ms": round(r.get("ms_per_step", r.get("ms_per_call", float("nan"))), 5)}
        if rf:
            e.update(bound=rf.get("bound"), achieved=round(rf.get("achieved", 0.0), 1), unit=rf.get("unit"),
                     frac=round(rf.get("frac", 0.0), 4))
        out[name] = e
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode512",
                    choices=["decode64", "decode512", "mamba2", "prefill32", "kda_decode64", "kda_prefill32",
                             "qgroup_decode256", "q8_decode64", "conv_decode64", "conv_prefill32"])
    ap.add_argument("--rows", default="all", choices=["all", "none"])
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--scan-algo", default="serial", choices=["serial", "chunked", "chunked_ws"],
                    help="prefill workload: token-serial scan, the chunked tensor-core form, or that form in "
                         "two launches through a workspace")
    ap.add_argument("--prefill-seqs", type=int, default=32,
                    help="sequences of the prefill workload (fewer only to profile a smaller case)")
    a = ap.parse_args()
    a.warmup = max(a.warmup, 3)

    rank, world, local = dist_setup(a.gpus)
    if a.impl == "reference":
        return reference_arm(a, rank, world)

    import torch
    from gated_deltanet_recurrent_la_b200 import lastate as L
    L.lib()  # fail loudly if the CUDA library is missing
    peaks = measured_peaks()
    sm_count = torch.cuda.get_device_properties(local).multi_processor_count
    sampler = ClockSampler(local)
    sampler.start()

    run, inp = build_runner(a.workload, prefill_seqs=a.prefill_seqs,
                            chunked={"serial": False, "chunked": True, "chunked_ws": "ws"}[a.scan_algo])
    nbytes, flops = run.bytes_flops()
    ms = time_back_to_back(run, a.steps, a.warmup, world, sampler)
    sampler.stop()
    flush = L2Flush()
    ms_flushed = time_flushed(run, min(a.steps, 50), flush) if inp.kind == "step" else None
    value = aggregate(nbytes, ms, world) / 1e9
    per_gpu = nbytes / (ms * 1e-3) / 1e9
    out = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
           "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
           "data": "synthetic (seeded host generator; no dataset)",
           "config": dict(describe(a.workload, inp), parallelism=f"replicas x{world}",
                          l2="inputs larger than L2: 4 disjoint 64-slot sets of the 256 MiB pool rotated step to step"
                          if a.workload == "decode64" else "inputs larger than L2 (1 GiB of state per step)"
                          if a.workload == "decode512" else "inputs larger than L2")}
    if inp.kind == "step":
        out["pct_of_peak"] = 100 * per_gpu / peaks["hbm_gbs"]
        out["pct_of_spec_8000"] = 100 * per_gpu / SPEC_HBM_GBS
        out["tokens_per_s"] = world * run.B / (ms * 1e-3)
        out["state_steps_per_s"] = world * run.B * inp.n_v_heads / (ms * 1e-3)
        out["ms_per_step_l2_flushed"] = ms_flushed
        out["roofline"] = {"bound": "hbm", "achieved": per_gpu, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                           "frac": per_gpu / peaks["hbm_gbs"],
                           "traffic": recorded_traffic(step_kernel(a.workload)[0], a.workload),
                           "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json hbm_gbs)" if peaks["source"] == "measured"
                           else "fallback 6650 GB/s", "algorithmic_bytes_per_launch": nbytes,
                           "kernel": step_kernel(a.workload)[1]}
    else:
        alu = fp32_alu_peak_tflops(sm_count, peaks["sm_max_mhz"])
        tf = flops / (ms * 1e-3) / 1e12
        out["tokens_per_s"] = world * run.T / (ms * 1e-3)
        if a.scan_algo != "serial":
            out["roofline"] = chunk_roofline(run, inp, ms, peaks)
        else:
            out["roofline"] = {"bound": "alu", "achieved": tf, "peak": alu, "unit": "TFLOP/s", "frac": tf / alu,
                               "traffic": recorded_traffic("scan", a.workload), "kernel": "la::scan_kernel"}
    out["gpu_launches"] = a.steps
    out["clocks"] = sampler.summary()

    if inp.kind == "step":
        e2e_ms, h2d, d2h = time_e2e(run, a.steps, a.warmup, world)
        out["e2e"] = {"value": aggregate(nbytes, e2e_ms, world) / 1e9, "unit": "GB/s", "ms_per_step": e2e_ms,
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                      "tokens_per_s": world * run.B / (e2e_ms * 1e-3),
                      "how": "pinned host buffers; H2D of step i+1 and D2H of step i-1 overlap step i; "
                             "chunks of 16 steps replayed as a CUDA graph"}
        out["gpu_launches"] += a.steps
    del run
    torch.cuda.empty_cache()

    if a.rows == "all":
        rows = {}
        for name in ("decode512", "decode64", "mamba2", "prefill32", "kda_decode64", "kda_prefill32",
                     "qgroup_decode256", "q8_decode64", "conv_decode64", "conv_prefill32"):
            if name == a.workload:
                continue
            k = a.steps if "prefill" not in name else max(3, min(a.steps, 20))
            rows[name] = measure_row(name, min(k, 500), a.warmup, world, peaks, sm_count, flush)
            torch.cuda.empty_cache()
        rows["prefill32_ckpt256"] = measure_row("prefill32", max(3, min(a.steps, 20)), a.warmup, world, peaks,
                                                sm_count, None, ckpt_every=256)
        torch.cuda.empty_cache()
        rows["prefill32_chunked"] = measure_row("prefill32", max(3, min(a.steps, 50)), a.warmup, world, peaks,
                                                sm_count, None, chunked=True)
        torch.cuda.empty_cache()
        rows["prefill32_chunked_two_launch"] = measure_row("prefill32", max(3, min(a.steps, 50)), a.warmup, world,
                                                           peaks, sm_count, None, chunked="ws")
        torch.cuda.empty_cache()
        rows["prefill32_chunked_ckpt256"] = measure_row("prefill32", max(3, min(a.steps, 50)), a.warmup, world,
                                                        peaks, sm_count, None, ckpt_every=256, chunked=True)
        torch.cuda.empty_cache()
        rows["kda_prefill32_chunked"] = measure_row("kda_prefill32", max(3, min(a.steps, 50)), a.warmup, world,
                                                    peaks, sm_count, None, chunked="ws")
        torch.cuda.empty_cache()
        rows["conv_prefill32_chunked"] = measure_row("conv_prefill32", max(3, min(a.steps, 50)), a.warmup, world,
                                                     peaks, sm_count, None, chunked=True)
        torch.cuda.empty_cache()
        rows["conv_prefill32_chunked_two_launch"] = measure_row("conv_prefill32", max(3, min(a.steps, 50)), a.warmup,
                                                                world, peaks, sm_count, None, chunked="ws")
        torch.cuda.empty_cache()
        pool_run = PoolRunner()
        pms = time_back_to_back(pool_run, min(a.steps, 500), a.warmup, world)
        pb, _ = pool_run.bytes_flops()
        rows["pool_copy64"] = {"ms_per_call": pms, "gb_s": pb / (pms * 1e-3) / 1e9,
                               "roofline": {"bound": "hbm", "achieved": pb / (pms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                                            "unit": "GB/s", "frac": pb / (pms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                            "traffic": recorded_traffic("pool", "copy64")},
                               "config": "64 slots x 1 MiB (32 heads x 128 x 128 BF16) copied to 64 others in a "
                                         "1024-slot pool; 16 disjoint slot sets rotated"}
        del pool_run
        out["rows"] = rows

    if rank == 0:
        if world == 1:
            if inp.kind == "step":
                cms, cores, sample = cpu_baseline_decode(inp, a.cpu_budget)
                out["cpu_baseline"] = {"value": nbytes / (cms * 1e-3) / 1e9, "unit": "GB/s", "cores": cores,
                                       "kind": "oracle", "sample": sample, "ms_per_step": cms}
                c1, _, s1 = cpu_single_thread(cpu_baseline_decode, inp, min(a.cpu_budget, 5.0))
                out["cpu_baseline"]["single_thread"] = {"value": nbytes / (c1 * 1e-3) / 1e9, "unit": "GB/s",
                                                        "cores": 1, "sample": s1, "ms_per_step": c1}
            else:
                cb = cpu_baseline_scan(inp, budget_s=a.cpu_budget)
                if cb is not None:
                    out["cpu_baseline"] = {"value": cb[0], "unit": "GB/s", "cores": cb[2], "kind": "oracle",
                                           "sample": cb[3], "tokens_per_s": cb[1], "scaled": True}
            if "rows" in out and "prefill32" in out["rows"]:
                # the prefill workload (all its forms share it): a fixed 4-sequence subset on all
                # host cores and a 1024-token prefix on one core, both scaled by tokens
                pin = build_runner_inputs("prefill32")
                cb = cpu_baseline_scan(pin, budget_s=a.cpu_budget)
                c1 = cpu_single_thread(cpu_baseline_scan, pin, budget_s=0.0, max_tokens=1024)
                if cb is not None and c1 is not None:
                    base = {"value": cb[0], "unit": "GB/s", "cores": cb[2], "kind": "oracle", "sample": cb[3],
                            "tokens_per_s": cb[1], "scaled": True,
                            "single_thread": {"value": c1[0], "unit": "GB/s", "cores": 1, "sample": c1[3],
                                              "tokens_per_s": c1[1], "scaled": True}}
                    for name in ("prefill32", "prefill32_chunked", "prefill32_chunked_two_launch"):
                        if name in out["rows"]:
                            out["rows"][name]["cpu_baseline"] = base
        if "rows" in out:
            out["rows_summary"] = rows_summary(out["rows"])
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def reference_arm(a, rank, world):
    """The oracle (CPU, fp64, OpenMP) timed on the host cores on the same workload, as the
    reference arm.  Under torchrun only rank 0 runs it; the other ranks exit."""
    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0
    from gated_deltanet_recurrent_la_b200 import workloads as W
    inp = W.WORKLOADS[a.workload](0)
    if inp.kind != "step":
        print(json.dumps({"impl": "reference", "unavailable": "the reference arm times decode workloads only"}))
        return 0
    nbytes, _ = step_bytes_and_flops(B=int(inp.q.shape[0]), n_qk_heads=inp.n_qk_heads, n_v_heads=inp.n_v_heads,
                                     d_k=inp.d_k, d_v=inp.d_v, state_bytes=state_bytes_per_value(inp),
                                     io_bytes=inp.q.element_size(), rule=inp.rule,
                                     slot_arrays=0 if inp.read_slot is None else 2, n_q_heads=inp.n_q_heads)
    budget = max(5.0, min(60.0, 0.5 * (a.steps + a.warmup)))
    cms, cores, sample = cpu_baseline_decode(inp, min(budget, a.cpu_budget * 3))
    value = nbytes / (cms * 1e-3) / 1e9
    out = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": a.steps,
           "warmup": a.warmup, "ms_per_step": cms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "f64", "data": "synthetic (seeded host generator; no dataset)",
           "config": describe(a.workload, inp),
           "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
