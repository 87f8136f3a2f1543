"""Benchmark of the CPR Gated DeltaNet path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

One step is one CPR forward (prefill / trainer forward: offsets, chunk
precompute, boundary chain, intra-chunk recurrence, output store) of the
prefill workload, B=4 sequences x T=4096 tokens, H=16 heads, d_k=d_v=128,
C=64, bf16 q/k/v, fp32 gates and state.  Inputs are synthetic, from the
device recipe of gated_deltanet_cpr_delta_b200.synth.  The line also
reports decode tokens/s for the decode workload (64 sequences x 32 heads,
prefilled to 2048 tokens, then 256 decode steps) and trainer fwd+bwd tokens/s
(B=2 x 8192 tokens, 32 heads, forward then gdn_cpr_backward) and varlen
tokens/s (32 packed sequences of 128..8192 tokens, 32 heads).

With N > 1 (torchrun, one rank per GPU) every rank runs its own sequences
(weak scaling, no data-path collective).  Timing is CUDA events on the
launching stream, the max over ranks: one event pair around each step of a
timed pass, then a second pass of the same steps with events inside the
calls for the per-kernel split (so the inner events do not inflate the
step).  L2 is flushed (a 256 MiB write) before every step.  Rank 0 prints
one JSON line.

Rank 0 checks the first forward against the oracle on two sampled (sequence,
head) pairs (the parity gate) before
it prints: if the gate fails, the line carries "value": null and the
process exits 1.  It also times the oracle on the host cores (cpu_baseline;
--no-cpu-baseline skips only that timing).

--impl reference times the CPU oracle (fp64 recurrence, OpenMP) on the host
cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
os.environ.setdefault("OMP_NUM_THREADS", str(os.cpu_count() or 1))

METRIC = "CPR GDN prefill & decode tokens/s on 1 B200; % of roofline; bitwise parity"
UNIT = "tokens/s"
WORKLOAD = dict(name="prefill B=4 H=16 T=4096 d_k=d_v=128 C=64 bf16", seed=1, B=4, H=16, T=4096, D=128, C=64)
DECODE = dict(name="decode 64 seqs H=32 d=128 C=64: prefill 2048, then 256 steps", seed=2, N=64, H=32, D=128,
              C=64, Lp=2048, steps=256)
TRAIN = dict(name="trainer fwd+bwd B=2 H=32 T=8192 d_k=d_v=128 C=64 bf16, dO ~ N(0,1) bf16", seed=4, B=2, H=32,
             T=8192, D=128, C=64)
VARLEN = dict(name="varlen 32 seqs L~U[128,8192] H=32 d_k=d_v=128 C=64 bf16", seed=3, N=32, H=32, D=128, C=64,
              lo=128, hi=8192)

# FP32 CUDA-core peak: 148 SMs x 128 FP32 lanes x 2 flop (fma) x 1.965 GHz (max SM clock)
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


# Algorithmic work of one forward, counted from the arithmetic schedule
# (fma = 2 flops).  Per (token, head): P_tok 7*dk*dv; chunk precompute
# (C-1)(2dk+dv) per token of a full chunk; boundary chain 4*dk*dv per token
# of a full chunk.
def forward_flops(tokens_heads: int, full_tokens_heads: int, dk: int, dv: int, C: int):
    return dict(tok=7 * dk * dv * tokens_heads,
                prep=(C - 1) * (2 * dk + dv) * full_tokens_heads,
                chain=4 * dk * dv * full_tokens_heads)


# Algorithmic bytes of one decode step's per-token kernel per (sequence, head):
# running state read + write (fp32), q, k, v read, o write, token appended to
# the buffer (k, v, alpha, beta), gates and position.
def decode_tok_bytes(dk: int, dv: int, esz: int, out_esz: int):
    return 8 * dk * dv + (2 * dk + dv) * esz + dv * out_esz + (dk + dv) * esz + 8 + 8 + 8


# Algorithmic work of the backward per (token, head), fma = 2 flops: the state
# recompute (u = S k, S <- alpha S + delta k^T: 3 dk*dv), G += dO q^T,
# ddelta = G k, <G, S_{t-1}>, dq = S_t^T dO, dk = G^T delta - ab S^T ddelta
# (2), G <- alpha G - ab ddelta k^T (2): 11 dk*dv fmas.
def backward_flops(tokens_heads: int, dk: int, dv: int):
    return 22 * dk * dv * tokens_heads


# Algorithmic work of k_bgrad per (chunk, head), the chunk form's dense
# products (fma = 2 flops, one product per pair of matrices, before the 3xTF32
# split): six d x d x C products (S0 w^T, S0 K^T, Y K^T, S0^T dO^T, S0^T Dd^T,
# Y^T Delta^T) = 12 C d^2, and the C x C x d products ([K; Q] K^T 4, U 2, Dd 4,
# [dO; Dd] Delta^T 4, dk 4, dq 2, and P_chunk part 1: Gram 1, u0 and w 2) =
# 23 C^2 d.
def bgrad_flops(chunks_heads: int, d: int, C: int):
    return (12 * C * d * d + 23 * C * C * d) * chunks_heads


# tf32 dense tensor-core peak from the measured (or fallback) bf16 peak and the
# nominal tf32 / bf16 ratio (1.1 / 2.25 PFLOP/s dense per GPU)
TF32_PER_BF16 = 1.1 / 2.25


# DRAM traffic per launch from ncu captures (dram__bytes_read.sum +
# dram__bytes_write.sum), keyed by kernel and by the sha256 of the sources that
# kernel is compiled from; a changed source drops the figure (reported null).
NCU_TRAFFIC = {
    ("k_chain_tok", "6ffe60d00cafadbf"): 787287552 + 328396544,
    ("k_dec_tok", "799efe9a357495b4"): 135929088 + 77861888,
    ("k_bgrad", "0a3b676036fe7e31"): 2770113280 + 2330992128,
}

KERNEL_SOURCES = {
    "k_tok": ("schedule.cuh", "k_ptok.cuh"),
    "k_chain_tok": ("schedule.cuh", "k_ptok.cuh", "k_tc.cuh", "k_pchunk.cuh"),
    "k_dec_tok": ("schedule.cuh", "k_ptok.cuh", "k_decode.cuh"),
    "k_bgrad": ("schedule.cuh", "k_ptok.cuh", "k_tc.cuh", "k_prep.cuh", "k_bgrad.cuh"),
}


def kernel_source_sha(kernel: str = "k_tok"):
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "gated_deltanet_cpr_delta_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measure_fp32_peak():
    """Sustained FP32 fma rate of this GPU (TFLOP/s), scalar and packed, from
    the probe kernels of libgdn_probe.so (run before the timed regions)."""
    import ctypes
    import torch
    path = os.path.join(ROOT, "gated_deltanet_cpr_delta_b200", "libgdn_probe.so")
    lib = ctypes.CDLL(path)
    lib.gdn_probe_fp32_tflops.restype = ctypes.c_int
    lib.gdn_probe_fp32_tflops.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                          ctypes.POINTER(ctypes.c_double), ctypes.c_void_p]
    sink = torch.zeros(148 * 64, dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    out = {}
    for name, packed in (("ffma", 0), ("ffma2", 1)):
        t = ctypes.c_double(0.0)
        if lib.gdn_probe_fp32_tflops(packed, 20, ctypes.c_void_p(sink.data_ptr()), ctypes.byref(t), stream) != 0:
            raise RuntimeError("FP32 peak probe failed")
        out[name] = t.value
    return out


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: str):
        self.dev = device_index
        self.proc = None
        self.path = os.path.join("/tmp", f"gdn_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.dev, f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) == 9 and p[1].replace(".", "").isdigit():
                    rows.append(p)
        if not rows:
            return None
        sm = sorted(float(r[1]) for r in rows)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows if r[3] != "[N/A]")}


def dist_setup(n_gpus: int):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return dist.get_rank(), world, local
    return 0, 1, 0


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Max of a per-rank timing over all ranks (the job's time is the slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_sequence_ids(rank: int, per_rank: int):
    """Weak scaling: rank r runs its own sequences r*per_rank .. (r+1)*per_rank-1
    of the seeded workload, so no rank repeats another's data and no data-path
    collective is needed."""
    return range(rank * per_rank, (rank + 1) * per_rank)


def job_throughput(tokens_per_rank: int, world: int, max_ms: float, steps: int) -> float:
    """Whole-job tokens/s: the tokens all ranks processed / the slowest rank's time."""
    return tokens_per_rank * world * steps / (max_ms / 1e3)


def barrier(world: int):
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(seed: int, B: int, H: int, D: int, C: int, T_s: int):
    """fp64 oracle on the first T_s tokens of every sequence and head of the
    prefill workload (host recipe inputs).  Returns (seconds, tokens)."""
    import numpy as np
    import oracle
    from gated_deltanet_cpr_delta_b200 import synth
    b = synth.make_batch(seed, [T_s] * B, H, D, D, "bf16")
    t0 = time.perf_counter()
    oracle.recurrent(b.q, b.k, b.v, b.alpha, b.beta, b.cu_seqlens, C)
    return time.perf_counter() - t0, B * T_s


def cpu_baseline(budget_s: float = 10.0):
    W = WORKLOAD
    T_s, secs, toks = 128, 0.0, 0
    while True:
        secs, toks = oracle_sample(W["seed"], W["B"], W["H"], W["D"], W["C"], T_s)
        if secs >= budget_s or T_s >= W["T"]:
            break
        T_s = min(W["T"], max(T_s * 2, int(T_s * budget_s / max(secs, 1e-3) * 1.1)))
    reps = 1
    if secs < budget_s:  # the whole workload is shorter than the budget: repeat it
        reps = max(1, int(budget_s / max(secs, 1e-3)))
        secs, toks = 0.0, 0
        for _ in range(reps):
            s_, t_ = oracle_sample(W["seed"], W["B"], W["H"], W["D"], W["C"], T_s)
            secs, toks = secs + s_, toks + t_
    return {"value": toks / secs, "unit": UNIT, "cores": int(os.environ["OMP_NUM_THREADS"]), "kind": "oracle",
            "sample": f"fp64 recurrence (oracle/recurrent_fp64.c, OpenMP over (sequence, head)) on the first "
                      f"{T_s} tokens of all {W['B']} sequences x {W['H']} heads of the prefill workload, "
                      f"{reps} run(s); {secs:.1f} s"}


def workload_config(world: int) -> dict:
    """The bench workload's config, shared by both arms of the benchmark."""
    W = WORKLOAD
    return {"workload": W["name"], "global_batch": W["B"] * world, "seq_len": W["T"], "heads": W["H"],
            "d_k": W["D"], "d_v": W["D"], "chunk": W["C"], "io_dtype": "bf16", "state_dtype": "f32",
            "parallelism": f"dp{world} (sequences sharded, no collective)",
            "l2": "flushed before every timed step (256 MiB write)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    import oracle
    oracle._load()
    W = WORKLOAD
    # size one step to ~5 s of oracle work
    T_s = 256
    secs, _ = oracle_sample(W["seed"], W["B"], W["H"], W["D"], W["C"], T_s)
    T_s = max(64, min(W["T"], int(T_s * 5.0 / max(secs, 1e-3))))
    for _ in range(args.warmup):
        oracle_sample(W["seed"], W["B"], W["H"], W["D"], W["C"], min(T_s, 64))
    tot_s, tot_tok = 0.0, 0
    for _ in range(args.steps):
        s, t = oracle_sample(W["seed"], W["B"], W["H"], W["D"], W["C"], T_s)
        tot_s += s
        tot_tok += t
    v = tot_tok / tot_s
    sample = (f"fp64 recurrence on the first {T_s} tokens of all {W['B']} sequences x {W['H']} heads "
              f"of the prefill workload per step")
    print(json.dumps({
        "metric": METRIC, "value": v, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(world),
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": int(os.environ["OMP_NUM_THREADS"]), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
    return 0


# ---------------------------------------------------------------- native
def parity_gate(d, snaps, C):
    """The first forward on sampled (sequence, head) pairs (snaps: (n, h, o
    rows, chunk-state rows) taken right after it): bitwise vs the fp32
    schedule model, and the max error vs the fp64 oracle.  Runs in the
    CPU-baseline leg (rank 0, one GPU), the one part of the native arm that
    runs the oracle."""
    import numpy as np
    import torch
    import oracle
    bits_all, rel_max, serr_max, err_max, names = True, 0.0, 0.0, 0.0, []
    for n, h, o_s, st_s in snaps:
        c0, c1 = d["cu_host"][n], d["cu_host"][n + 1]
        L = c1 - c0
        g = lambda t: t[c0:c1, h:h + 1].float().cpu().numpy()
        q, k, v, a, b = g(d["q"]), g(d["k"]), g(d["v"]), g(d["alpha"]), g(d["beta"])
        cu = np.array([0, L], np.int32)
        st_h = st_s.contiguous().cpu().numpy()
        mo, _, _ = oracle.schedule_tok_from_states(q, k, v, a, b, st_h, cu, C)
        r = oracle.recurrent(q, k, v, a, b, cu, C)
        got = o_s.contiguous().cpu()
        bits_all &= bool(np.array_equal(got.view(torch.int16).numpy().view(np.uint16), oracle.to_bf16_bits(mo)))
        err = float(np.max(np.abs(got.float().numpy().astype(np.float64) - r["o"])))
        err_max = max(err_max, err)
        rel_max = max(rel_max, err / float(np.max(np.abs(r["o"]))))
        serr_max = max(serr_max, float(np.max(np.abs(st_h.astype(np.float64) - r["states"]))) /
                       float(np.max(np.abs(r["states"]))))
        names.append(f"sequence {n}, head {h} ({L} tokens)")
    return {"p_tok_bitwise_vs_schedule_model": bits_all, "max_abs_err_vs_fp64": err_max,
            "max_err_rel_to_max_o": rel_max, "states_max_err_rel": serr_max, "tolerance_rel": 2e-2,
            "ok": bool(bits_all and rel_max <= 2e-2 and serr_max <= 2e-2), "sample": "; ".join(names)}


def bench_decode(rank: int, world: int, warmup: int):
    import torch
    from gated_deltanet_cpr_delta_b200 import gdn, synth
    Dc = DECODE
    N, H, D, C, Lp, S = Dc["N"], Dc["H"], Dc["D"], Dc["C"], Dc["Lp"], Dc["steps"]
    L = Lp + S
    d = synth.make_batch_device(Dc["seed"], [L] * N, H, D, D, "bf16", seq_ids=rank_sequence_ids(rank, N))
    idx = torch.cat([torch.arange(n * L, n * L + Lp) for n in range(N)]).cuda()
    cu_p = [n * Lp for n in range(N + 1)]
    cache = gdn.new_cache(N, H, D, D, C, torch.bfloat16)
    gdn.gdn_cpr_forward(d["q"][idx], d["k"][idx], d["v"][idx], d["alpha"][idx], d["beta"][idx],
                        torch.tensor(cu_p, dtype=torch.int32, device="cuda"), C, cu_seqlens_host=cu_p,
                        cache_out=cache)
    steps_in = []
    for s in range(S):
        t = torch.arange(N, device="cuda") * L + Lp + s
        steps_in.append([d[n][t].contiguous() for n in ("q", "k", "v", "alpha", "beta")])
    del d
    torch.cuda.empty_cache()   # only the cache and the step inputs stay on the device
    o = torch.empty(N, H, D, dtype=torch.bfloat16, device="cuda")
    # warm-up on a copy of the cache (the timed steps start at position Lp)
    wc = {k_: v_.clone() for k_, v_ in cache.items()}
    for s in range(max(warmup, 3)):
        gdn.gdn_decode_step(*steps_in[s], wc, C, o=o)
    del wc
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(S)]
    outer = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(S)]
    for e in ev:
        for x in e:
            x.record()
    c0 = {k_: v_.clone() for k_, v_ in cache.items()}  # the same start for the kernel-split pass
    # timed pass: one event pair around each step (L2 flushed before it), nothing inside the call
    barrier(world)
    for s in range(S):
        flush.zero_()
        outer[s][0].record()
        gdn.gdn_decode_step(*steps_in[s], cache, C, o=o)
        outer[s][1].record()
    barrier(world)
    step_ms = [a.elapsed_time(b) for a, b in outer]
    # second pass, from the same cache: events inside the call split each step into its kernels
    for s in range(S):
        flush.zero_()
        gdn.gdn_decode_step(*steps_in[s], c0, C, o=o, events=ev[s])
    torch.cuda.synchronize()
    tok_ms = [e[0].elapsed_time(e[1]) for e in ev]
    res_ms = [e[1].elapsed_time(e[2]) for e in ev]
    del c0
    total_ms = max_over_ranks(sum(step_ms), world)
    resync_steps = [s for s in range(S) if (Lp + s + 1) % C == 0]
    plain = [step_ms[s] for s in range(S) if s not in resync_steps]
    tb = decode_tok_bytes(D, D, 2, 2) * N * H
    mean_tok = sum(tok_ms) / S
    peaks, _ = load_peaks()
    return {"workload": Dc["name"], "value": N * world * S / (total_ms / 1e3), "unit": UNIT,
            "ms_per_step": total_ms / S, "plain_step_ms_mean": sum(plain) / len(plain),
            "resync_step_ms_mean": sum(step_ms[s] for s in resync_steps) / max(1, len(resync_steps)),
            "resync_kernel_ms_max": max(res_ms),
            "step_kernel_ms_mean": sum(tok_ms) / S,
            "resync_kernel_plain_ms_mean": sum(res_ms[s] for s in range(S) if s not in resync_steps) / len(plain),
            "roofline": {"kernel": "k_dec_tok", "bound": "hbm", "achieved": tb / (mean_tok / 1e3) / 1e9,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": tb / (mean_tok / 1e3) / 1e9 / peaks["hbm_gbs"],
                         "traffic": NCU_TRAFFIC.get(("k_dec_tok", kernel_source_sha("k_dec_tok"))),
                         "bytes_per_launch": tb}}


def bench_trainer(rank: int, world: int, warmup: int, steps: int, shape=None):
    """Trainer step: CPR forward + backward (gdn_cpr_backward) of the trainer
    workload on this rank's sequences; L2 flushed before every timed step.
    ``shape`` (B, H, T) replaces the workload's sizes (for profiling a smaller
    case of the same kernels)."""
    import torch
    from gated_deltanet_cpr_delta_b200 import gdn, synth
    Tr = dict(TRAIN)
    if shape is not None:
        Tr.update(B=shape[0], H=shape[1], T=shape[2],
                  name=f"trainer fwd+bwd B={shape[0]} H={shape[1]} T={shape[2]} d_k=d_v=128 C=64 bf16, "
                       f"dO ~ N(0,1) bf16")
    B, H, T, D, C = Tr["B"], Tr["H"], Tr["T"], Tr["D"], Tr["C"]
    d = synth.make_batch_device(Tr["seed"], [T] * B, H, D, D, "bf16", seq_ids=rank_sequence_ids(rank, B))
    g = torch.Generator(device="cuda")
    g.manual_seed(Tr["seed"] * 1_000_003 + 999 + rank)
    dO = torch.randn(B * T, H, D, device="cuda", generator=g).to(torch.bfloat16)
    o = torch.empty(B * T, H, D, dtype=torch.bfloat16, device="cuda")
    st = torch.empty(gdn.gdn_num_chunk_states(d["cu_host"], C), H, D, D, dtype=torch.float32, device="cuda")
    ws = torch.empty(gdn.gdn_cpr_workspace_size(B * T, B, H, D, D, C), dtype=torch.uint8, device="cuda")
    wsb = torch.empty(gdn.gdn_cpr_backward_workspace_size(B * T, B, H, D, D, C), dtype=torch.uint8, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    grads = (torch.empty(B * T, H, D, **f32), torch.empty(B * T, H, D, **f32), torch.empty(B * T, H, D, **f32),
             torch.empty(B * T, H, **f32), torch.empty(B * T, H, **f32), torch.empty(B, H, D, D, **f32))

    def step(fe=None, be=None):
        gdn.gdn_cpr_forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["cu_seqlens"], C,
                            cu_seqlens_host=d["cu_host"], o=o, chunk_states=st, workspace=ws, events=fe)
        gdn.gdn_cpr_backward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], dO, st, d["cu_seqlens"], C,
                             cu_seqlens_host=d["cu_host"], workspace=wsb, grads=grads, events=be)

    for _ in range(max(warmup, 3)):
        step()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    fev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    bev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for e in fev + bev:
        for x in e:
            x.record()
    outer = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    # timed pass: one event pair around each forward + backward, nothing inside the calls
    barrier(world)
    for s in range(steps):
        flush.zero_()
        outer[s][0].record()
        step()
        outer[s][1].record()
    barrier(world)
    tot = max_over_ranks(sum(a.elapsed_time(b) for a, b in outer), world)
    # second pass: events inside the calls split the step into forward, backward and kernels
    for s in range(steps):
        flush.zero_()
        step(fev[s], bev[s])
    torch.cuda.synchronize()
    fwd_ms = [e[0].elapsed_time(e[5]) for e in fev]
    bwd_ms = [e[0].elapsed_time(e[3]) for e in bev]
    kern = {n: sum(e[i].elapsed_time(e[i + 1]) for e in bev) / steps
            for i, n in enumerate(("k_tables + k_bwd_scan", "k_bprep", "k_bgrad"))}
    chunks = B * ((T + C - 1) // C) * H
    fl = bgrad_flops(chunks, D, C)
    tf = fl / (kern["k_bgrad"] / 1e3) / 1e12
    peaks, src = load_peaks()
    tpk = peaks["bf16_tflops"] * TF32_PER_BF16
    return {"workload": Tr["name"], "value": B * T * world / (tot / steps / 1e3), "unit": UNIT,
            "ms_per_step": tot / steps, "fwd_ms": sum(fwd_ms) / steps, "bwd_ms": sum(bwd_ms) / steps,
            "bwd_kernels_ms": kern,
            "roofline": {"kernel": "k_bgrad (per-chunk gradients on tcgen05, 3xTF32)", "bound": "tensor",
                         "achieved": tf, "peak": tpk, "unit": "TFLOP/s", "frac": tf / tpk,
                         "traffic": NCU_TRAFFIC.get(("k_bgrad", kernel_source_sha("k_bgrad"))),
                         "flops_per_launch": fl,
                         "peak_source": f"tf32 dense = bf16 dense ({src}) x 1.1/2.25 (nominal ratio)"}}


def bench_varlen(rank: int, world: int, warmup: int, steps: int):
    """Varlen workload: 32 packed sequences (lengths from the seeded draw in
    [128, 8192]), H=32; CPR forward tokens/s with L2 flushed before each step."""
    import torch
    from gated_deltanet_cpr_delta_b200 import gdn, synth
    V = VARLEN
    lens = synth.varlen_lengths(V["seed"], V["N"], V["lo"], V["hi"])
    H, D, C = V["H"], V["D"], V["C"]
    d = synth.make_batch_device(V["seed"], lens, H, D, D, "bf16", seq_ids=rank_sequence_ids(rank, V["N"]))
    T = sum(lens)
    o = torch.empty(T, H, D, dtype=torch.bfloat16, device="cuda")
    st = torch.empty(gdn.gdn_num_chunk_states(d["cu_host"], C), H, D, D, dtype=torch.float32, device="cuda")
    ws = torch.empty(gdn.gdn_cpr_workspace_size(T, len(lens), H, D, D, C), dtype=torch.uint8, device="cuda")
    fwd = lambda ev=None: gdn.gdn_cpr_forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["cu_seqlens"], C,
                                              cu_seqlens_host=d["cu_host"], o=o, chunk_states=st, workspace=ws,
                                              events=ev)
    for _ in range(max(warmup, 3)):
        fwd()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    outer = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(world)
    for s_ in range(steps):
        flush.zero_()
        outer[s_][0].record()
        fwd()
        outer[s_][1].record()
    barrier(world)
    total = max_over_ranks(sum(a.elapsed_time(b) for a, b in outer), world)
    full = sum((L // C) * C for L in lens)
    fl = forward_flops(T * H, full * H, D, D, C)
    return {"workload": V["name"], "tokens": T, "value": T * world * steps / (total / 1e3), "unit": UNIT,
            "ms_per_step": total / steps, "flops_per_step": sum(fl.values()),
            "frac_fp32_peak": sum(fl.values()) / (total / steps / 1e3) / 1e12 / FP32_PEAK_TFLOPS}


def run_native(args):
    import torch
    from gated_deltanet_cpr_delta_b200 import gdn, synth

    rank, world, local = dist_setup(args.gpus)
    gdn.load_library()
    fp32_meas = measure_fp32_peak()
    W = WORKLOAD
    B, H, T, D, C = W["B"], W["H"], W["T"], W["D"], W["C"]
    d = synth.make_batch_device(W["seed"], [T] * B, H, D, D, "bf16", seq_ids=rank_sequence_ids(rank, B))
    o = torch.empty(B * T, H, D, dtype=torch.bfloat16, device="cuda")
    st = torch.empty(gdn.gdn_num_chunk_states(d["cu_host"], C), H, D, D, dtype=torch.float32, device="cuda")
    ws = torch.empty(gdn.gdn_cpr_workspace_size(B * T, B, H, D, D, C), dtype=torch.uint8, device="cuda")
    fwd = lambda events=None: gdn.gdn_cpr_forward(d["q"], d["k"], d["v"], d["alpha"], d["beta"], d["cu_seqlens"],
                                                  C, cu_seqlens_host=d["cu_host"], o=o, chunk_states=st,
                                                  workspace=ws, events=events)
    fwd()
    torch.cuda.synchronize()
    # the first and the last (sequence, head) of this first forward; the CPU-baseline leg checks
    # them against the oracle
    snaps = []
    for n, h in sorted({(0, 0), (B - 1, H - 1)}):
        c0, c1 = d["cu_host"][n], d["cu_host"][n + 1]
        s0 = sum((d["cu_host"][m + 1] - d["cu_host"][m]) // C + 1 for m in range(n))
        snaps.append((n, h, o[c0:c1, h:h + 1].clone(), st[s0:s0 + (c1 - c0) // C + 1, h:h + 1].clone()))
    parity = None

    for _ in range(args.warmup):
        fwd()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    K = args.steps
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(K)]
    for e in kev:
        for x in e:
            x.record()
    outer = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    dev_index = os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local if world > 1 else 0]
    # timed pass: one event pair around each forward (L2 flushed before it), nothing inside the call
    with ClockSampler(dev_index) as clocks:
        barrier(world)
        for s in range(K):
            flush.zero_()
            outer[s][0].record()
            fwd()
            outer[s][1].record()
        barrier(world)
    step_ms = [a.elapsed_time(b) for a, b in outer]
    # second pass: events inside the call time each kernel on the launching stream
    for s in range(K):
        flush.zero_()
        fwd(kev[s])
    torch.cuda.synchronize()
    names = ["k_tables", "k_prep", "k_chain", "k_tok", "k_cache_fill"]
    kern_ms = {n: sum(e[i].elapsed_time(e[i + 1]) for e in kev) / K for i, n in enumerate(names)}
    total_ms = max_over_ranks(sum(step_ms), world)
    ms_step = total_ms / K
    tokens = B * T * world
    value = job_throughput(B * T, world, total_ms, K)

    # e2e: every step copies its inputs host (pinned) -> device, runs the
    # forward through the public API and copies o device -> host.  Steps are
    # pipelined the way a serving loop would run them: step i+1's inputs
    # upload on a copy stream while step i computes, and step i's o downloads
    # on a second copy stream (two device buffer sets alternate).
    hin = {n: d[n].cpu().pin_memory() for n in ("q", "k", "v", "alpha", "beta")}
    cu_pin = torch.tensor(d["cu_host"], dtype=torch.int32).pin_memory()
    dev_in = [{n: torch.empty_like(d[n]) for n in hin} for _ in range(2)]
    cu_dev = [torch.empty_like(d["cu_seqlens"]) for _ in range(2)]
    o_dev = [torch.empty_like(o) for _ in range(2)]
    o_host = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in hin.values()) + cu_pin.numel() * 4
    d2h = o.numel() * o.element_size()
    compute = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def upload(i):
        j = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(done[j])           # the forward two steps back is done with buffer set j
            for n in hin:
                dev_in[j][n].copy_(hin[n], non_blocking=True)
            cu_dev[j].copy_(cu_pin, non_blocking=True)
            in_ready[j].record(s_in)

    def run_steps(nsteps):
        for j in range(2):
            done[j].record(compute)
            out_done[j].record(compute)
        upload(0)
        for i in range(nsteps):
            j = i % 2
            if i + 1 < nsteps:
                upload(i + 1)
            compute.wait_event(in_ready[j])
            compute.wait_event(out_done[j])   # o buffer j has been downloaded
            gdn.gdn_cpr_forward(dev_in[j]["q"], dev_in[j]["k"], dev_in[j]["v"], dev_in[j]["alpha"],
                                dev_in[j]["beta"], cu_dev[j], C, cu_seqlens_host=d["cu_host"], o=o_dev[j],
                                chunk_states=st, workspace=ws)
            done[j].record(compute)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[j])
                o_host[j].copy_(o_dev[j], non_blocking=True)
                out_done[j].record(s_out)
        for j in range(2):
            compute.wait_event(out_done[j])
            compute.wait_event(in_ready[j])

    run_steps(2)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    run_steps(K)
    e1.record()
    barrier(world)
    assert torch.equal(o_dev[(K - 1) % 2].cpu(), o_host[(K - 1) % 2])
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / K

    dec = bench_decode(rank, world, args.warmup) if not args.no_decode else None
    tshape = tuple(int(x) for x in args.trainer_shape.split(",")) if args.trainer_shape else None
    trainer = bench_trainer(rank, world, args.warmup, min(K, 5), tshape) if not args.no_trainer else None
    varlen = bench_varlen(rank, world, args.warmup, min(K, 5)) if not args.no_varlen else None

    peaks, peak_src = load_peaks()
    flops = forward_flops(B * T * H, B * (T // C) * C * H, D, D, C)
    # with few (sequence, head) pairs the library runs the chain and P_tok as
    # one cooperative kernel; its events then give the chain no time of its own
    fused = kern_ms["k_chain"] < 0.01 and kern_ms["k_tok"] > 0
    if fused:
        kern_ms["k_chain_tok"] = kern_ms.pop("k_tok")
        kern_ms.pop("k_chain")
        flops["chain_tok"] = flops.pop("chain") + flops.pop("tok")
        names = ["k_tables", "k_prep", "k_chain_tok", "k_cache_fill"]
    main = "k_chain_tok" if fused else "k_tok"
    main_flops = flops["chain_tok" if fused else "tok"]
    tok_tf = main_flops / (kern_ms[main] / 1e3) / 1e12
    sha = kernel_source_sha(main)
    traffic = NCU_TRAFFIC.get((main, sha))
    kernels = {n: {"ms": kern_ms[n]} for n in names}
    for n in (("chain_tok", "prep") if fused else ("tok", "prep", "chain")):
        kernels["k_" + n]["tflops"] = flops[n] / (kern_ms["k_" + n] / 1e3) / 1e12 if kern_ms["k_" + n] > 0 else 0
        kernels["k_" + n]["frac_fp32_peak"] = kernels["k_" + n]["tflops"] / FP32_PEAK_TFLOPS
    total_flops = sum(flops.values())
    flops_tok_only = 7 * D * D * B * T * H
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": workload_config(world),
        "roofline": {"kernel": ("k_chain_tok (boundary chain on tcgen05 + intra-chunk P_tok, one cooperative "
                                "launch)") if fused else "k_tok (intra-chunk P_tok)",
                     "bound": "alu", "achieved": tok_tf,
                     "peak": FP32_PEAK_TFLOPS, "unit": "TFLOP/s", "frac": tok_tf / FP32_PEAK_TFLOPS,
                     "traffic": traffic, "flops_per_launch": main_flops,
                     "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 x 1.965 GHz",
                     "peak_measured": fp32_meas["ffma"], "frac_measured": tok_tf / fp32_meas["ffma"]},
        "forward_roofline": {"flops_per_step": total_flops,
                             "achieved_tflops": total_flops / (ms_step / 1e3) / 1e12 / world,
                             "frac": total_flops / (ms_step / 1e3) / 1e12 / world / FP32_PEAK_TFLOPS,
                             "frac_measured": total_flops / (ms_step / 1e3) / 1e12 / world / fp32_meas["ffma"],
                             "recurrence_only_flops": flops_tok_only,
                             "recurrence_only_frac": flops_tok_only / (ms_step / 1e3) / 1e12 / world /
                             FP32_PEAK_TFLOPS,
                             "peak": FP32_PEAK_TFLOPS, "peak_measured": fp32_meas["ffma"]},
        "kernels": kernels,
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "pipelining": "step i+1's upload and step i-1's download overlap step i's forward "
                              "(two device buffer sets, two copy streams)"},
        "gpu_launches": (3 if fused else 4) * K,
        "clocks": clocks.summary(),
        "parity": parity,
        "decode": dec,
        "trainer": trainer,
        "varlen": varlen,
        "peaks": {"hbm_gbs": peaks.get("hbm_gbs"), "source": peak_src,
                  "fp32_tflops_derived": FP32_PEAK_TFLOPS,
                  "fp32_tflops_measured": fp32_meas,
                  "fp32_measured_by": "libgdn_probe.so: 8 independent fma chains per thread, 8 CTAs x 256 "
                                      "threads per SM, 20 launches, timed in this run before the forward"},
        "kernel_source_sha": sha,
        "contract": {"id": gdn.gdn_contract_id(),
                     "numerical_policy": gdn.gdn_contract_identity(gdn.ID_NUMERICAL_POLICY, D, D, C, gdn.GDN_BF16,
                                                                   gdn.GDN_BF16),
                     "deployment": gdn.gdn_contract_identity(gdn.ID_DEPLOYMENT, D, D, C, gdn.GDN_BF16,
                                                             gdn.GDN_BF16)},
    }
    # The oracle leg, on rank 0 only: the parity gate on the first forward's
    # snapshot (always), and the oracle's own timing (one GPU, unless skipped).
    rc = 0
    if rank == 0:
        line["parity"] = parity_gate(d, snaps, C)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline()
        if not line["parity"]["ok"]:
            line["value"] = None  # no speed is reported for a result that failed its parity check
            line["parity_failed"] = True
            rc = 1
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))
    return rc


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-trainer", action="store_true")
    ap.add_argument("--no-varlen", action="store_true")
    ap.add_argument("--trainer-shape", default=None,
                    help="B,H,T of the trainer section (default: the trainer workload; for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    return run_reference(args) if args.impl == "reference" else run_native(args)


if __name__ == "__main__":
    sys.exit(main())
