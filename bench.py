"""Benchmark of the Lightning Attention hot path on B200.

One step = one la_prefill of the 32K-token workload shaped like the
MiniMax-01 attention layer: B=1, H=64, N=32768, d=128, bf16 q/k/v drawn
iid N(0,1)*128^-0.5, fp32 accumulation, bf16 output plus the final fp32
128x128 state of every head.  The step runs every prefill row of the hot path
(segment table + TMA staging + the four tcgen05 contractions + masking +
cross-SM segment hand-off + epilogue).  In the same run the fused batched
decode step is timed on its own workload (256 sequences x 64 heads, fp32
states initialised by a 4096-token prefill) and reported under "decode", and
the packed variable-length batch (8 sequences of 1024-65536 tokens, 64
heads) under "varlen", the 1M-token prefill (8 heads) under "long_context",
the local-prefix step of sequence parallelism (la_kv_aggregate) on the
prefill's k and v under "kv_aggregate", and the gradients of the prefill
(la_prefill_backward) under "backward".

  python bench.py [--gpus N] [--steps K] [--warmup W]      # CUDA path
  python bench.py --impl reference ...                     # fp64 CPU oracle arm

Under torchrun (N > 1) every rank runs its own independent batch (no
collective on the data path; weak scaling); timing is the max over ranks.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import la_inputs  # noqa: E402

METRIC = "lightning-attn prefill tok/s + TFLOP/s; decode tok/s; % of roofline"
B, N, H, D = 1, 32768, 64, 128
BLOCK = 128
E2E_CHUNK = 4096  # tokens per chunk of the host-memory pipeline timed as e2e
DEC_SEQS, DEC_PREFILL = 256, 4096
SEED = 20250101


# --------------------------------------------------------------------------- helpers
def prefill_bytes(tok_heads: int, heads: int, seqs: int) -> int:
    """Algorithmic HBM bytes of one prefill: read q, k, v (bf16), write out
    (bf16), write the final fp32 state of every (sequence, head)."""
    return tok_heads * D * 2 * 4 + seqs * heads * D * D * 4


LO_SPLIT_FROM = 32768  # segments ending past this token use S as bf16 hi + lo in Q S


def prefill_alg_flops(tok_heads: int, block: int) -> int:
    """Algorithmic FLOPs (2 per multiply-add) per the blocked definition:
    2*(Bk+1)*d per token-head for the causal triangle of its block including
    the diagonal, plus 4*d^2 for the inter-block term Q S and the update K^T V."""
    return tok_heads * (2 * (block + 1) * D + 4 * D * D)


def prefill_dense_flops(tok_heads: int, block: int) -> int:
    """The dense count 4*Bk*d + 4*d^2 per token-head (full score and P V tiles,
    one Q S and one K^T V), independent of how the kernel splits the work."""
    return tok_heads * (4 * block * D + 4 * D * D)


def prefill_mma_flops(lengths, heads: int, seg_len: int, want_state: bool = True, block: int = 128) -> int:
    """FLOPs the tensor pipe executes in la_prefill_kernel, counted MMA by MMA
    the way the kernel issues them (one unit = a 128 x 128 x 128 product,
    2 * 128^3 FLOPs), per segment of seg_len tokens of every sequence, over its
    128-row tiles:
      block 128: per tile Q K^T and P V (full tiles, masked or not), Q S (two
           units when the segment ends past LO_SPLIT_FROM tokens: S as bf16
           hi + lo), K^T V except for the segment's last tile (which gets it in
           the final segment when the state is wanted);
      block 64: per tile Q K^T, P V, Q S twice (once per 64-row block, each a
           full product writing half the rows; doubled again for hi + lo), K^T V
           of the first 64 rows always and of the last 64 rows as above;
      block 256: per pair of tiles Q K^T and P V three times (two diagonal
           tiles and the second tile against the first), Q S once per tile,
           K^T V for both tiles unless the pair is the segment's last (as above);
      and K^T V again in the segment-sum pass, one unit per tile of every
      segment that has a successor in its sequence."""
    unit = 2 * 128 ** 3
    units = 0.0
    for n in lengths:
        n = int(n)
        nseg = -(-n // seg_len) if n > 0 else 0
        for j in range(nseg):
            t0, t1 = j * seg_len, min(n, (j + 1) * seg_len)
            nblk = -(-(t1 - t0) // 128)
            last = j == nseg - 1
            qs = 2 if t1 > LO_SPLIT_FROM else 1          # Q S, bf16 S or hi + lo
            if block == 256:
                npair = (nblk + 1) // 2
                for m in range(npair):
                    ntp = 2 if 2 * m + 1 < nblk else 1
                    upd = m < npair - 1 or (last and want_state)
                    units += 2 * (ntp + (ntp == 2))         # Q K^T, P V (3 steps per full pair)
                    units += ntp * qs                       # Q S
                    units += ntp if upd else 0              # K^T V
            else:
                fin = 1 if (last and want_state) else 0
                units += 2 * nblk                           # Q K^T, P V
                if block == 64:
                    units += 2 * nblk * qs                  # Q S once per 64-row block
                    units += 0.5 * nblk + 0.5 * (nblk - 1 + fin)  # K^T V in two halves
                else:
                    units += nblk * qs
                    units += nblk - 1 + fin
            units += 0 if last else nblk                    # K^T V, segment sums
    return int(units * unit * heads)


def aggregate_bytes(tok_heads: int, pairs: int) -> int:
    """Read k and v (bf16), write one fp32 d x d sum per (sequence, head)."""
    return tok_heads * D * 2 * 2 + pairs * D * D * 4


def backward_bytes(tok_heads: int) -> int:
    """Read q, k, v and dout, write dq, dk and dv (all bf16)."""
    return tok_heads * D * 2 * 7


def decode_bytes(pairs: int) -> int:
    """Read + write the fp32 state, read q, k, v and write o (bf16)."""
    return pairs * (2 * D * D * 4 + 4 * D * 2)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), float(pk["bf16_tflops"]), float(pk.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


KERNEL_SOURCES = {
    "la_prefill_kernel": ("la_prefill.cuh", "la_ptx.cuh", "la_lib.cu"),
    "la_decode_kernel": ("la_decode.cuh", "la_lib.cu"),
    "la_kv_aggregate_kernel": ("la_aggregate.cuh", "la_prefill.cuh", "la_ptx.cuh", "la_lib.cu"),
}


def kernel_source_hash(kernel: str = "la_prefill_kernel") -> str:
    """Hash of the kernel's sources with // comments and blank lines removed, so
    that comment-only edits keep a recorded traffic figure valid."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "linear_attention_blocked_b200", "csrc", name), encoding="utf-8") as f:
            for line in f:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source; otherwise None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        e = rec[kernel][workload]
        if e.get("source_hash") == kernel_source_hash(kernel):
            return float(e["bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi samples (every 200 ms) tagged with host time."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.samples = []
        self.proc = None
        self.gpu = gpu_index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        rows = [s for (t, s) in self.samples if t0 <= t <= t1]
        if not rows:  # very short region: take the samples nearest to it
            rows = [s for (t, s) in self.samples if t0 - 0.5 <= t <= t1 + 0.5]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if len(r) > 6 + i and r[6 + i] == "Active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


class NvmlClockSampler:
    """SM clock and clock-event reasons read through NVML every `period`
    seconds from a background thread (a finer grid than nvidia-smi's 200 ms,
    so that a timed region of a few tens of milliseconds still gets samples).
    The GPU is found by its PCI bus id, so CUDA and NVML numbering may differ."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))
    # every other reason bit, reported so that a clock below the maximum is
    # never left unexplained by the record
    OTHER_REASONS = (("gpu_idle", "nvmlClocksEventReasonGpuIdle"),
                     ("applications_clocks_setting", "nvmlClocksEventReasonApplicationsClocksSetting"),
                     ("sync_boost", "nvmlClocksEventReasonSyncBoost"),
                     ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown"),
                     ("display_clock_setting", "nvmlClocksEventReasonDisplayClockSetting"))

    def __init__(self, dev: torch.device, period: float = 0.002):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml as nv
            self.nv = nv
            nv.nvmlInit()
            pr = torch.cuda.get_device_properties(dev)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            self.h = nv.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.masks = [(name, getattr(nv, attr)) for name, attr in self.REASONS]
            self.other_masks = [(name, getattr(nv, attr)) for name, attr in self.OTHER_REASONS if hasattr(nv, attr)]
            try:
                self.power_limit_w = nv.nvmlDeviceGetEnforcedPowerLimit(self.h) / 1000.0
            except Exception:
                self.power_limit_w = None
            self.period = period
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                try:
                    mw = nv.nvmlDeviceGetPowerUsage(self.h)
                except Exception:
                    mw = -1
                self.samples.append((time.time(), mhz, rs, mw))
            except Exception:
                pass
            time.sleep(self.period)

    def stop(self):
        self._stop.set()

    def summary(self, t0: float, t1: float):
        rows = [(m, r, w) for (t, m, r, w) in self.samples if t0 <= t <= t1]
        if not rows:
            return None
        reasons = sorted({name for (_, r, _) in rows for (name, mask) in self.masks if r & mask})
        other = sorted({name for (_, r, _) in rows for (name, mask) in self.other_masks if r & mask})
        watts = [w / 1000.0 for (_, _, w) in rows if w >= 0]
        out = {"sm_mhz": float(np.median([m for m, _, _ in rows])), "sm_max_mhz": float(self.max_mhz),
               "reasons": reasons, "other_reasons": other, "samples": len(rows), "source": "NVML, 2 ms period"}
        if watts:
            out["power_w_median"] = float(np.median(watts))
            out["power_w_max"] = float(np.max(watts))
            out["power_limit_w"] = self.power_limit_w
        return out


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    from linear_attention_blocked_b200.replicas import max_over_ranks as _max
    return _max(x)


# --------------------------------------------------------------------------- oracle arms
def oracle_sample_rate(budget_s: float, seed: int):
    """Time the fp64 oracle (recurrent form) on heads of the 32K workload until
    `budget_s` seconds of CPU work are spent.  Returns (tok/s scaled to all 64
    heads, threads used, description)."""
    import oracle
    oracle.build()
    q, k, v = la_inputs.qkv((N, H, D), seed)
    Q, K, V = la_inputs.bits(q), la_inputs.bits(k), la_inputs.bits(v)
    cu = np.array([0, N], np.int32)
    threads = oracle.max_threads()
    heads_done, elapsed = 0, 0.0
    step = max(1, min(H, threads))
    while heads_done < H and elapsed < budget_s:
        hs = list(range(heads_done, min(H, heads_done + step)))
        t = time.perf_counter()
        oracle.recurrent(Q, K, V, cu, heads=hs, threads=threads)
        elapsed += time.perf_counter() - t
        heads_done += len(hs)
    rate = N * heads_done / H / elapsed
    desc = (f"fp64 recurrent oracle, {heads_done} of {H} heads x {N} tokens in {elapsed:.1f} s on "
            f"{threads} OpenMP threads; tok/s scaled by {heads_done}/{H}")
    return rate, threads, desc


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    threads = oracle.max_threads()
    q, k, v = la_inputs.qkv((N, H, D), SEED)
    Q, K, V = la_inputs.bits(q), la_inputs.bits(k), la_inputs.bits(v)
    # each step: a bounded sample (tokens x heads) sized so the whole run takes ~--ref-seconds
    per_step_s = max(0.005, args.ref_seconds / max(1, args.steps + args.warmup))
    probe_tok = 1024
    t = time.perf_counter()
    oracle.recurrent(Q[:probe_tok], K[:probe_tok], V[:probe_tok], np.array([0, probe_tok], np.int32), heads=[0],
                     threads=1)
    per_tok = (time.perf_counter() - t) / probe_tok
    nh = max(1, min(H, threads))
    ntok = int(max(64, min(N, per_step_s / per_tok * 0.8)))
    cu = np.array([0, ntok], np.int32)
    hs = list(range(nh))
    # every call names its thread count: the 1-thread probe above must not
    # leave the oracle on one thread
    for _ in range(args.warmup):
        oracle.recurrent(Q[:ntok], K[:ntok], V[:ntok], cu, heads=hs, threads=threads)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle.recurrent(Q[:ntok], K[:ntok], V[:ntok], cu, heads=hs, threads=threads)
    dt = time.perf_counter() - t
    value = ntok * nh / H * args.steps / dt       # tok/s of the 64-head workload
    sample = (f"each step: fp64 recurrent oracle on the first {ntok} tokens of {nh} of {H} heads, "
              f"{threads} OpenMP threads (one (sequence, head) pair each); tok/s scaled by {nh}/{H}")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(args.gpus),
        "cpu_baseline": {"value": value, "unit": "tok/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(ngpu):
    return {"workload": "lightning-attn causal prefill B=1 H=64 N=32768 d=128 bf16 in/out + fp32 final state",
            "B": B, "N": N, "H": H, "d": D, "block": BLOCK, "global_batch": B * ngpu, "seq_len": N,
            "parallelism": f"replicas x{ngpu} (independent batches, no collective)",
            "l2": "inputs larger than L2 (1.61 GB of q/k/v read per step), no flush",
            "seed": SEED}


# --------------------------------------------------------------------------- CUDA arm
def run_cuda(args, world, rank, local):
    import linear_attention_blocked_b200 as la

    dev = torch.device("cuda", local if world > 1 else 0)
    stream = torch.cuda.current_stream(dev)
    hbm_peak, tc_peak, tc_sust, peak_src = load_peaks()

    q, k, v = la_inputs.qkv((B, N, H, D), SEED + rank, device=dev)
    out = torch.empty((B, N, H, D), dtype=torch.bfloat16, device=dev)
    st = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    ws = torch.empty(la.workspace_size(B, N, H, D, BLOCK), dtype=torch.uint8, device=dev)

    def step():
        la.prefill(q, k, v, block=BLOCK, out=out, state_out=st, workspace=ws)

    for _ in range(max(3, args.warmup)):
        step()
    if la.get_device_status() != la.LA_OK:
        raise RuntimeError("device status not OK after warm-up")

    sampler = ClockSampler(local if world > 1 else 0) if rank == 0 else None
    fast = NvmlClockSampler(dev) if rank == 0 else None
    time.sleep(0.3 if sampler else 0)
    launches0 = la.kernel_launches()
    barrier(world)
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_host0 = time.time()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    t_host1 = time.time()
    barrier(world)
    launches = la.kernel_launches() - launches0
    ms = ev0.elapsed_time(ev1) / args.steps
    ms_max = max_over_ranks(ms, world)
    status = la.get_device_status()
    clocks = None
    if fast is not None:
        clocks = fast.summary(t_host0, t_host1)
        fast.stop()
    if sampler:
        smi = sampler.summary(t_host0, t_host1)
        if clocks is None:
            clocks = smi
        else:
            clocks["nvidia_smi"] = smi
        sampler.stop()

    tok_heads = B * N * H
    tokens_all = B * N * world
    value = tokens_all / (ms_max * 1e-3)
    byts = prefill_bytes(tok_heads, H, B)
    L = la.last_segment_len()
    f_alg = prefill_alg_flops(tok_heads, BLOCK)
    f_mma = prefill_mma_flops([N] * B, H, L, want_state=True, block=BLOCK)
    f_dense = prefill_dense_flops(tok_heads, BLOCK)
    achieved_gbs = byts / (ms * 1e-3) / 1e9

    legs = set(args.legs.split(",")) if args.legs else None
    want = lambda name: legs is None or name in legs  # noqa: E731

    # ---------------- end to end through the public API with host buffers
    e2e_steps = max(3, min(args.steps, 20)) if want("e2e") else 0
    e2e_ms = None
    if e2e_steps:
        qh = q.cpu().pin_memory(); kh = k.cpu().pin_memory(); vh = v.cpu().pin_memory()
        oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        sh = torch.empty(st.shape, dtype=st.dtype).pin_memory()
        bufs = la.make_buffers(B, E2E_CHUNK, H, out.dtype, dev)

        def e2e_step():
            # the public host-memory entry point (la_prefill_from_host): chunks of
            # tokens copied in, scanned and copied out on three streams, the state
            # carried between chunks
            la.prefill_from_host(qh, kh, vh, chunk_tokens=E2E_CHUNK, out=oh, state_out=sh, buffers=bufs,
                                 device=dev)

        e2e_step()
        torch.cuda.synchronize(dev)
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
        del bufs, qh, kh, vh, oh, sh

    # ---------------- fused batched decode on its own workload
    dec = None
    if want("decode") and (rank == 0 or world > 1):
        dec = bench_decode(la, dev, stream, args, hbm_peak, world)

    # ---------------- the same workload at row blocks of 64 and 256
    by_block = {f"block{blk}": bench_prefill_block(la, dev, stream, q, k, v, blk, args, hbm_peak, tc_peak, world)
                for blk in (64, 256) if want(f"block{blk}")}
    # ---------------- the same workload with a per-head decay
    dec_pref = bench_prefill_decay(la, dev, stream, q, k, v, args, hbm_peak, world) if want("decay") else None

    # ---------------- the packed varlen batch and the 1M-token prefill
    varlen = bench_varlen(la, dev, stream, args, hbm_peak, tc_peak, world, rank) if want("varlen") else None
    longc = bench_long_context(la, dev, stream, args, hbm_peak, tc_peak, world, rank) if want("long") else None

    # ---------------- local prefix of sequence parallelism on the same k, v
    agg = bench_kv_aggregate(la, dev, stream, k, v, args, hbm_peak, world) if want("aggregate") else None
    # ---------------- gradients of the prefill on the same q, k, v
    bwd = bench_backward(la, dev, stream, q, k, v, args, hbm_peak, world) if want("backward") else None
    # ---------------- gradients of the packed varlen batch
    bwd_v = bench_backward_varlen(la, dev, stream, args, hbm_peak, world, rank) if want("backward_varlen") else None

    status2 = la.get_device_status()
    if rank != 0:
        return 0
    traffic = recorded_traffic("la_prefill_kernel", "prefill_B1_H64_N32768")
    cpu = None
    if world == 1 and args.cpu_seconds > 0:
        rate, cores, desc = oracle_sample_rate(args.cpu_seconds, SEED)
        cpu = {"value": rate, "unit": "tok/s", "cores": cores, "kind": "oracle", "sample": desc}
    line = {
        "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(world),
        "segment_len": L,
        "tflops_alg": f_alg / (ms * 1e-3) / 1e12,
        "tflops_mma": f_mma / (ms * 1e-3) / 1e12,
        "tensor_frac_mma": f_mma / (ms * 1e-3) / 1e12 / tc_peak,
        "tensor_frac_alg": f_alg / (ms * 1e-3) / 1e12 / tc_peak,
        "tensor_frac_dense_count": f_dense / (ms * 1e-3) / 1e12 / tc_peak,
        "tensor_note": ("tflops_mma counts every tcgen05 MMA the kernel issues (full 128-row tiles, Q S once "
                        "per block up to 32768 tokens into a sequence, twice beyond, K^T V in the scan and in the "
                        "segment-sum pass); "
                        "tflops_alg the blocked definition 2(Bk+1)d + 4d^2 per token-head; dense_count "
                        "4 Bk d + 4 d^2; fractions of the measured cuBLAS bf16 burst peak"),
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved_gbs / hbm_peak, "traffic": traffic,
                     "kernel": "la_prefill_kernel", "bytes_per_launch": byts,
                     "duration": "CUDA events around each la_prefill call (scheduler + prefill kernel)",
                     "peak_source": f"{peak_src} hbm_gbs"},
        "e2e": None if e2e_ms is None else {"value": tokens_all / (e2e_ms * 1e-3), "unit": "tok/s", "ms_per_step": e2e_ms,
                "steps": e2e_steps,
                "api": f"la_prefill_from_host (C ABI) through prefill_from_host, {E2E_CHUNK}-token chunks pipelined "
                       "over copy-in / compute / copy-out streams",
                "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
                "d2h_bytes_per_step": out.numel() * out.element_size() + st.numel() * st.element_size()},
        "gpu_launches": int(launches),
        "clocks": clocks,
        "prefill_by_block": by_block,
        "prefill_decay": dec_pref,
        "decode": dec,
        "varlen": varlen,
        "long_context": longc,
        "kv_aggregate": agg,
        "backward": bwd,
        "backward_varlen": bwd_v,
        "cpu_baseline": cpu,
        "device_status": [int(status), int(status2)],
    }
    print(json.dumps(line), flush=True)
    return 0


def bench_kv_aggregate(la, dev, stream, k, v, args, hbm_peak, world):
    """la_kv_aggregate (local prefix of sequence parallelism: sum of k_t^T v_t
    per head) over the prefill workload's k and v (1.07 GB, larger than L2)."""
    agg = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    ws = torch.empty(max(256, la.lib().la_kv_aggregate_workspace_size(B, N, H, D)), dtype=torch.uint8, device=dev)
    for _ in range(3):
        la.kv_aggregate(k, v, out=agg, workspace=ws)
    torch.cuda.synchronize(dev)
    barrier(world)
    steps = max(20, min(args.steps, 500))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        la.kv_aggregate(k, v, out=agg, workspace=ws)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    byts = aggregate_bytes(B * N * H, B * H)
    gbs = byts / (ms * 1e-3) / 1e9
    return {"workload": "kv_aggregate B=1 H=64 N=32768 d=128 (the prefill workload's k, v)",
            "ms_per_call": ms, "steps": steps,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": gbs / hbm_peak, "kernel": "la_kv_aggregate_kernel",
                         "traffic": recorded_traffic("la_kv_aggregate_kernel", "aggregate_B1_H64_N32768"),
                         "bytes_per_launch": byts,
                         "duration": "CUDA events around each la_kv_aggregate call (aggregate + reduce)"}}


def bench_backward_varlen(la, dev, stream, args, hbm_peak, world, rank):
    """la_prefill_backward_varlen on the packed varlen workload (8 sequences
    of lengths drawn in [1024, 65536], H=64; random dout), bf16 gradients."""
    lens = la_inputs.varlen_lengths(8, 1024, 65536, seed=3)
    cu = la_inputs.cu_seqlens_from_lengths(lens)
    T = int(cu[-1])
    q, k, v = la_inputs.qkv((T, H, D), seed=303 + rank, device=dev)
    g, _, _ = la_inputs.qkv((T, H, D), seed=313 + rank, device=dev)
    cu_d = torch.from_numpy(cu).to(dev)
    grads = [torch.empty_like(q) for _ in range(3)]
    ws = torch.empty(la.backward_varlen_workspace_size(len(lens), T, int(lens.max()), H, D), dtype=torch.uint8,
                     device=dev)

    def call():
        la.prefill_backward_varlen(q, k, v, g, cu_d, int(lens.max()), dq=grads[0], dk=grads[1], dv=grads[2],
                                   workspace=ws)

    for _ in range(3):
        call()
    torch.cuda.synchronize(dev)
    barrier(world)
    steps = max(5, min(args.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    byts = backward_bytes(T * H)
    gbs = byts / (ms * 1e-3) / 1e9
    del q, k, v, g, grads, ws
    return {"workload": f"packed varlen backward, 8 seqs U[1024, 65536] (seed 3), {T} tokens, H=64, d=128, "
                        "bf16 dq/dk/dv + fp32 dS_in",
            "tok_s": T / (ms * 1e-3), "ms_per_call": ms, "steps": steps,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                         "kernel": "la_prefill_kernel (dQ sweep + reversed paired dK/dV sweep)",
                         # DRAM bytes of both sweeps of one call
                         "traffic": recorded_traffic("la_prefill_kernel", "backward_varlen_S8_H64"),
                         "bytes_per_launch": byts,
                         "duration": "CUDA events around each la_prefill_backward_varlen call (two schedule kernels "
                                     "+ two sweeps)"}}


def bench_backward(la, dev, stream, q, k, v, args, hbm_peak, world):
    """la_prefill_backward (dq, dk, dv, dS_in for a random dout; no carried-in
    state or state gradient) on the prefill workload, bf16 gradients."""
    g, _, _ = la_inputs.qkv((B, N, H, D), SEED + 11, device=dev)
    grads = [torch.empty_like(q) for _ in range(3)]
    ws = torch.empty(la.backward_workspace_size(B, N, H, D), dtype=torch.uint8, device=dev)

    def call():
        la.prefill_backward(q, k, v, g, dq=grads[0], dk=grads[1], dv=grads[2], workspace=ws)

    for _ in range(3):
        call()
    torch.cuda.synchronize(dev)
    barrier(world)
    steps = max(5, min(args.steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    byts = backward_bytes(B * N * H)
    gbs = byts / (ms * 1e-3) / 1e9
    del g, grads, ws
    return {"workload": "prefill backward B=1 H=64 N=32768 d=128, bf16 dq/dk/dv + fp32 dS_in",
            "ms_per_call": ms, "steps": steps,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": gbs / hbm_peak, "kernel": "la_prefill_kernel (dQ sweep + reversed paired dK/dV sweep)",
                         # DRAM bytes of both sweeps of one call
                         "traffic": recorded_traffic("la_prefill_kernel", "backward_B1_H64_N32768"),
                         "bytes_per_launch": byts,
                         "duration": "CUDA events around each la_prefill_backward call (two schedule kernels + two sweeps)"}}


DATASHEET_HBM_GBS = 7700.0  # HGX B200 HBM3e datasheet figure (8000 on DGX), context only


def bench_decode(la, dev, stream, args, hbm_peak, world):
    """Decode workload: 256 sequences x 64 heads, states from a 4096-token
    prefill (run in chunks of sequences), then timed decode steps, each on its
    own freshly drawn q, k, v (one seeded set per step, generated before the
    timed region and read from HBM once)."""
    state = torch.empty((DEC_SEQS, H, D, D), dtype=torch.float32, device=dev)
    chunk = 16
    for s0 in range(0, DEC_SEQS, chunk):
        qp, kp, vp = la_inputs.qkv((chunk, DEC_PREFILL, H, D), SEED + 7 + s0, device=dev)
        la.prefill(qp, kp, vp, block=BLOCK, state_out=state[s0:s0 + chunk])
        del qp, kp, vp
    steps = max(16, min(args.steps, 1024))
    warm = 3
    qkv = torch.empty((warm + steps, 3, DEC_SEQS, H, D), dtype=torch.bfloat16, device=dev)
    for i in range(warm + steps):
        for j, t in enumerate(la_inputs.qkv((DEC_SEQS, H, D), la_inputs.decode_seed(SEED, i), device=dev)):
            qkv[i, j] = t
    o = torch.empty((DEC_SEQS, H, D), dtype=torch.bfloat16, device=dev)
    for i in range(warm):
        la.decode_step(qkv[i, 0], qkv[i, 1], qkv[i, 2], state, out=o)
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(warm, warm + steps):
        la.decode_step(qkv[i, 0], qkv[i, 1], qkv[i, 2], state, out=o)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    pairs = DEC_SEQS * H
    byts = decode_bytes(pairs)
    gbs = byts / (ms * 1e-3) / 1e9
    traffic = recorded_traffic("la_decode_kernel", "decode_S256_H64")
    del state, qkv
    roof = {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
            "frac": gbs / hbm_peak, "kernel": "la_decode_kernel", "traffic": traffic,
            "bytes_per_launch": byts,
            "datasheet_peak": DATASHEET_HBM_GBS, "frac_of_datasheet": gbs / DATASHEET_HBM_GBS}
    if traffic is not None:
        roof["achieved_dram"] = traffic / (ms * 1e-3) / 1e9
        roof["frac_dram"] = roof["achieved_dram"] / hbm_peak
    if roof["frac"] > 1.0:
        roof["frac_above_1"] = ("algorithmic bytes / time exceed the measured copy bandwidth: part of the "
                                "state is served from L2 between steps (ncu DRAM bytes below the "
                                "algorithmic bytes), so this is not a DRAM roofline fraction; frac_dram "
                                "and frac_of_datasheet bound it")
    return {"workload": "decode 256 seqs x H=64 x d=128, fp32 state (1 GiB) from a 4096-token prefill, "
                        "fresh q/k/v every step",
            "tok_s": DEC_SEQS * world / (ms * 1e-3), "ms_per_step": ms, "steps": steps, "roofline": roof}


def bench_prefill_block(la, dev, stream, q, k, v, block, args, hbm_peak, tc_peak, world):
    """The bench workload (B=1, H=64, N=32768, bf16 out + states) at another
    row-block length: 64 (two state snapshots per 128-row tile) or 256 (a
    snapshot per pair of tiles, plus the second tile's queries against the
    first tile's keys)."""
    out = torch.empty((B, N, H, D), dtype=torch.bfloat16, device=dev)
    st = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    ws = torch.empty(la.workspace_size(B, N, H, D, block), dtype=torch.uint8, device=dev)

    def call():
        la.prefill(q, k, v, block=block, out=out, state_out=st, workspace=ws)

    for _ in range(3):
        call()
    torch.cuda.synchronize(dev)
    barrier(world)
    steps = max(5, min(args.steps, 100))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    L = la.last_segment_len()
    byts = prefill_bytes(B * N * H, H, B)
    gbs = byts / (ms * 1e-3) / 1e9
    f_mma = prefill_mma_flops([N] * B, H, L, want_state=True, block=block)
    f_alg = prefill_alg_flops(B * N * H, block)
    f_dense = prefill_dense_flops(B * N * H, block)
    del out, st, ws
    return {"workload": f"causal prefill B=1 H=64 N=32768 d=128 at row blocks of {block}",
            "ms_per_call": ms, "steps": steps, "segment_len": L,
            "tflops_mma": f_mma / (ms * 1e-3) / 1e12, "tensor_frac_mma": f_mma / (ms * 1e-3) / 1e12 / tc_peak,
            "tflops_alg": f_alg / (ms * 1e-3) / 1e12, "tensor_frac_alg": f_alg / (ms * 1e-3) / 1e12 / tc_peak,
            "tensor_frac_dense_count": f_dense / (ms * 1e-3) / 1e12 / tc_peak,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                         "kernel": "la_prefill_kernel", "bytes_per_launch": byts,
                         "traffic": recorded_traffic("la_prefill_kernel", f"prefill_B1_H64_N32768_block{block}"),
                         "duration": "CUDA events around each la_prefill call (scheduler + prefill)"}}


def bench_prefill_decay(la, dev, stream, q, k, v, args, hbm_peak, world):
    """The bench workload with the per-head decay lambda_h = exp(-2^(-8 (h+1)/H))
    (la_prefill_decay: decay in the mask, the inter-block term and the state,
    the decayed keys of the state update as bf16 hi + lo)."""
    lam = torch.tensor(np.exp(-(2.0 ** (-8.0 * (np.arange(H) + 1) / H))), dtype=torch.float32, device=dev)
    out = torch.empty((B, N, H, D), dtype=torch.bfloat16, device=dev)
    st = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    ws = torch.empty(la.workspace_size(B, N, H, D, BLOCK), dtype=torch.uint8, device=dev)

    def call():
        la.prefill(q, k, v, block=BLOCK, out=out, state_out=st, workspace=ws, decay=lam)

    for _ in range(3):
        call()
    torch.cuda.synchronize(dev)
    barrier(world)
    steps = max(5, min(args.steps, 100))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    byts = prefill_bytes(B * N * H, H, B)
    gbs = byts / (ms * 1e-3) / 1e9
    del out, st, ws
    return {"workload": "causal prefill B=1 H=64 N=32768 d=128 with per-head decay exp(-2^(-8(h+1)/64))",
            "ms_per_call": ms, "steps": steps,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                         "kernel": "la_prefill_kernel (decay)", "bytes_per_launch": byts,
                         "traffic": recorded_traffic("la_prefill_kernel", "prefill_decay_B1_H64_N32768"),
                         "duration": "CUDA events around each la_prefill_decay call (scheduler + prefill)"}}


def bench_varlen(la, dev, stream, args, hbm_peak, tc_peak, world, rank):
    """Packed variable-length prefill: 8 sequences with lengths drawn uniform in
    [1024, 65536] from a seed, concatenated (cu_seqlens on the device), H=64,
    bf16 out + fp32 final states.  About 266K tokens, 17 GB of algorithmic
    traffic per call (inputs far larger than L2)."""
    lens = la_inputs.varlen_lengths(8, 1024, 65536, seed=3)
    cu = la_inputs.cu_seqlens_from_lengths(lens)
    T = int(cu[-1])
    q, k, v = la_inputs.qkv((T, H, D), seed=303 + rank, device=dev)
    cu_d = torch.from_numpy(cu).to(dev)
    out = torch.empty((T, H, D), dtype=torch.bfloat16, device=dev)
    st = torch.empty((len(lens), H, D, D), dtype=torch.float32, device=dev)
    ws = torch.empty(la.varlen_workspace_size(len(lens), T, int(lens.max()), H, D, BLOCK), dtype=torch.uint8,
                     device=dev)

    def call():
        la.prefill_varlen(q, k, v, cu_d, int(lens.max()), block=BLOCK, out=out, state_out=st, workspace=ws)

    for _ in range(3):
        call()
    torch.cuda.synchronize(dev)
    barrier(world)
    steps = max(5, min(args.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    L = la.last_segment_len()
    byts = prefill_bytes(T * H, H, len(lens))
    gbs = byts / (ms * 1e-3) / 1e9
    f_mma = prefill_mma_flops(lens, H, L, want_state=True)
    del q, k, v, out, st, ws
    return {"workload": f"packed varlen prefill, 8 seqs U[1024, 65536] (seed 3): lengths {lens.tolist()}, "
                        f"{T} tokens, H=64, d=128, bf16 in/out + fp32 final states",
            "tok_s": T * world / (ms * 1e-3), "ms_per_call": ms, "steps": steps, "segment_len": L,
            "tflops_alg": prefill_alg_flops(T * H, BLOCK) / (ms * 1e-3) / 1e12,
            "tflops_mma": f_mma / (ms * 1e-3) / 1e12, "tensor_frac_mma": f_mma / (ms * 1e-3) / 1e12 / tc_peak,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": gbs / hbm_peak, "kernel": "la_prefill_kernel", "bytes_per_launch": byts,
                         "traffic": recorded_traffic("la_prefill_kernel", "varlen_S8_H64"),
                         "duration": "CUDA events around each la_prefill_varlen call (scheduler + prefill)"}}


def bench_long_context(la, dev, stream, args, hbm_peak, tc_peak, world, rank):
    """Long-context prefill: B=1, H=8, N=1048576, bf16 out + fp32 final states
    (8.6 GB of algorithmic traffic per call).  Segments past 32768 tokens hand
    S to the inter-block product as bf16 hi + lo."""
    NL, HL = 1048576, 8
    q, k, v = la_inputs.qkv((1, NL, HL, D), seed=404 + rank, device=dev)
    out = torch.empty((1, NL, HL, D), dtype=torch.bfloat16, device=dev)
    st = torch.empty((1, HL, D, D), dtype=torch.float32, device=dev)
    ws = torch.empty(la.workspace_size(1, NL, HL, D, BLOCK), dtype=torch.uint8, device=dev)

    def call():
        la.prefill(q, k, v, block=BLOCK, out=out, state_out=st, workspace=ws)

    for _ in range(3):
        call()
    torch.cuda.synchronize(dev)
    barrier(world)
    steps = max(5, min(args.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    L = la.last_segment_len()
    byts = prefill_bytes(NL * HL, HL, 1)
    gbs = byts / (ms * 1e-3) / 1e9
    f_mma = prefill_mma_flops([NL], HL, L, want_state=True)
    del q, k, v, out, st, ws
    return {"workload": "long-context prefill B=1 H=8 N=1048576 d=128, bf16 in/out + fp32 final states",
            "tok_s": NL * world / (ms * 1e-3), "ms_per_call": ms, "steps": steps, "segment_len": L,
            "tflops_alg": prefill_alg_flops(NL * HL, BLOCK) / (ms * 1e-3) / 1e12,
            "tflops_mma": f_mma / (ms * 1e-3) / 1e12, "tensor_frac_mma": f_mma / (ms * 1e-3) / 1e12 / tc_peak,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": gbs / hbm_peak, "kernel": "la_prefill_kernel", "bytes_per_launch": byts,
                         "traffic": recorded_traffic("la_prefill_kernel", "prefill_B1_H8_N1048576"),
                         "duration": "CUDA events around each la_prefill call (scheduler + prefill)"}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="CPU time budget of the oracle baseline sample (rank 0, N=1)")
    ap.add_argument("--ref-seconds", type=float, default=60.0,
                    help="approximate total CPU time of the --impl reference run")
    ap.add_argument("--legs", default="",
                    help="comma-separated subset of the legs after the main prefill step to run (e2e, decode, "
                         "block64, block256, decay, varlen, long, aggregate, backward, backward_varlen); default all")
    args = ap.parse_args()
    if args.impl == "reference":
        # the oracle runs on the host cores of rank 0 only; no process group needed
        return run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
    world, rank, local = dist_setup()
    try:
        rc = run_cuda(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
