"""Benchmark of the ragged paged-KV attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fg|reference] [--config 2]

One step = one Dynamic SplitFuse forward pass of the attention path over the
Llama-2-7B-shape SplitFuse snapshot (32/32 heads, d=128, block 64, budget
2048 = 31 decodes + one 2017-token prompt chunk): batch put (metadata upload),
rotary + paged append, ragged attention (+ split-KV combine). Inputs are
resident in HBM when timing starts; L2 is flushed (256 MB written, then read
back) between steps, outside the timed events. Prints one JSON line (rank 0).

With N > 1 (torchrun) every rank runs its own replica of the step on its own
GPU (the path has no exchange step, so no collective is on the data path);
value = all ranks' tokens / the slowest rank's time.

--impl reference times the float64 oracle on the host cores instead, on a
bounded sample of the same workload per step (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ragged-attention tokens/s at Llama-2-7B shape; % of HBM/tensor roofline"
L2_FLUSH_BYTES = 256 << 20


# ---------------------------------------------------------------------------
# ranks
# ---------------------------------------------------------------------------
def world():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), \
        int(os.environ.get("LOCAL_RANK", 0))


def init_dist(backend: str):
    import datetime
    import torch.distributed as dist
    rank, ws, _ = world()
    if ws > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, rank=rank, world_size=ws,
                                timeout=datetime.timedelta(seconds=120))
    return rank, ws


def barrier():
    import torch.distributed as dist
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# roofline accounting (algorithmic bytes and flops of one pass)
# ---------------------------------------------------------------------------
def algorithmic_work(w):
    """Bytes each step must move at minimum and attention flops.

    attention bytes: every admitted cached K and V row read once per kv head
    (GQA sharing counted once), Q read and O written once;
    append bytes: new K, V read and written to the cache, Q read, Q_rot written.
    flops: 4 * d * Hq per admitted (query, key) pair (QK^T and PV)."""
    Hq, Hkv, d, W = w.n_q_heads, w.n_kv_heads, w.head_dim, w.sliding_window
    g = Hq // Hkv
    kv_rows = pairs = 0
    dec_rows = dec_tokens = 0      # one-token decodes: the decode kernels
    tc_pairs = tc_rows = 0         # everything else: the tensor-core kernel
    for q, c in zip(w.q_lens.tolist(), w.ctx_lens.tolist()):
        p = np.arange(c, c + q, dtype=np.int64)
        lo = np.maximum(0, p - W + 1) if W > 0 else np.zeros_like(p)
        rows = int(p[-1] + 1 - lo[0])
        prs = int((p - lo + 1).sum())
        kv_rows += rows
        pairs += prs
        if q == 1 and (g == 1 or (d == 128 and g <= 16)):   # the decode kernels
            dec_rows += rows
            dec_tokens += 1
        else:
            tc_rows += rows
            tc_pairs += prs
    T = w.n_tokens
    attn_bytes = kv_rows * Hkv * d * 2 * 2 + T * Hq * d * 2 * 2
    append_bytes = T * Hkv * d * 2 * 2 * 2 + T * Hq * d * 2 * 2
    return {"attn_bytes": attn_bytes, "append_bytes": append_bytes, "flops": 4 * d * Hq * pairs,
            "pairs": pairs, "kv_rows": kv_rows,
            "decode_bytes": dec_rows * Hkv * d * 2 * 2 + dec_tokens * Hq * d * 2 * 2,
            "decode_flops": 4 * d * Hq * (pairs - tc_pairs),
            "tc_flops": 4 * d * Hq * tc_pairs,
            "tc_bytes": tc_rows * Hkv * d * 2 * 2 + (T - dec_tokens) * Hq * d * 2 * 2}


# dram__bytes_read.sum + dram__bytes_write.sum per launch, from one ncu capture
# of the kernel on that config's batch with the block pool sized to what the
# batch uses (same kernel, same bytes); keyed by config, then kernel. Absent
# (null in the line) where no capture was taken or the kernel has changed
# since. Summaries with the commands are in profiles/.
NCU_TRAFFIC = {
    2: {"decode": 1263240448, "tc": 53038592},
    5: {"tc": 419401728},
}


def ncu_traffic(config, kernel):
    return NCU_TRAFFIC.get(config, {}).get(kernel)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return j["hbm_gbs"], j["bf16_tflops"], "measured"
    return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock and clock-event reasons during the timed region, read-only.

    Polls NVML every 0.5 ms (the timed region of a short run lasts only a few
    milliseconds; nvidia-smi could sample it once at best; the NVML calls go
    through ctypes, which lets the enqueuing thread run meanwhile), and falls
    back to nvidia-smi every 200 ms where NVML is unavailable."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.samples = []  # (sm_mhz, max_mhz, [reason names])
        self.source = None
        self._stop = threading.Event()
        self._t = threading.Thread(target=self._run, daemon=True)
        self._nvml = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            try:
                uuid = str(torch.cuda.get_device_properties(index).uuid)
                if not uuid.startswith("GPU-"):
                    uuid = "GPU-" + uuid
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self._nvml = (pynvml, h, pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.source = "nvml, 0.5 ms"
        except Exception:
            self._nvml = None

    def _run(self):
        if self._nvml is not None:
            nv, h, mx = self._nvml
            while not self._stop.is_set():
                try:
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((float(sm), float(mx), [n for n, m in self.REASONS if bits & m]))
                except Exception:
                    pass
                self._stop.wait(0.0005)
            return
        self.source = "nvidia-smi, 200 ms"
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                      "--format=csv,noheader,nounits"], capture_output=True,
                                     text=True, timeout=5).stdout.strip()
                if out:
                    f = [x.strip() for x in out.split(",")]
                    if f[0].replace(".", "").isdigit() and f[1].replace(".", "").isdigit():
                        self.samples.append((float(f[0]), float(f[1]),
                                             [n for i, (n, _) in enumerate(self.REASONS) if f[2 + i] == "Active"]))
            except Exception:
                pass
            self._stop.wait(0.2)

    def __enter__(self):
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._t.join(timeout=10)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock samples"]}
        sm = [x[0] for x in self.samples]
        reasons = sorted({r for x in self.samples for r in x[2]})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(x[1] for x in self.samples),
                "reasons": reasons, "samples": len(self.samples), "source": self.source}


# ---------------------------------------------------------------------------
# the oracle on the host cores (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------
def oracle_sample(w, max_chunk_rows=192):
    """A bounded slice of the workload for the float64 oracle: every decode
    sequence plus the first ``max_chunk_rows`` tokens of each prompt chunk
    (each such slice is itself a valid, shorter chunk at the same context)."""
    from ragged_paged_kv_b200 import workloads as W
    q = np.minimum(w.q_lens, max_chunk_rows)
    sub = W.Workload(name=w.name + "_sample", n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                     head_dim=w.head_dim, block_size=w.block_size, n_blocks=w.n_blocks,
                     rope_theta=w.rope_theta, sliding_window=w.sliding_window, seq_ids=w.seq_ids,
                     q_lens=q.astype(np.int32), ctx_lens=w.ctx_lens, block_tables=w.block_tables,
                     seed=w.seed, budget=int(q.sum()))
    return sub


def time_oracle(w, reps=1):
    """Seconds per oracle pass (rotary + append + attention) over workload w,
    with the prior context written into a fresh oracle cache first (untimed)."""
    from oracle import PagedCache
    from oracle.forward import splitfuse_pass
    q, k, v = w.qkv()
    times = []
    for _ in range(reps):
        pc = PagedCache(w.n_blocks, w.n_kv_heads, w.block_size, w.head_dim, fill=0)
        for s, kc, vc in w.contexts():
            pc.write_positions(w.block_tables[s], np.arange(kc.shape[0]), kc, vc)
        t0 = time.perf_counter()
        splitfuse_pass(pc, w.block_tables, w.q_lens, w.ctx_lens, q, k, v, w.rope_theta,
                       w.softmax_scale, w.sliding_window)
        times.append(time.perf_counter() - t0)
    return times


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return len(os.sched_getaffinity(0))


def cpu_baseline(w, max_chunk_rows=4096, reps=4):
    """The oracle over the measured batch (prompt chunks cut at max_chunk_rows
    tokens; the headline batch's 2017-token chunk is taken whole), `reps`
    passes (about 10 s of host work for the headline batch); the value is
    tokens over the mean pass time."""
    sub = oracle_sample(w, max_chunk_rows=max_chunk_rows)
    times = time_oracle(sub, reps=reps)
    t = sum(times) / len(times)
    whole = int(sub.n_tokens) == int(w.n_tokens)
    what = (f"the whole batch ({sub.n_tokens} tokens: {int((w.q_lens == 1).sum())} decodes + the prompt chunks)"
            if whole else
            f"{sub.n_tokens} tokens: all {int((w.q_lens == 1).sum())} decodes + first "
            f"{int(sub.q_lens.max())} tokens of each prompt chunk")
    return {"value": sub.n_tokens / t, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{what}, float64 numpy, {len(times)} passes of {t:.2f} s"}


def workload_config(w, ws):
    """The `config` object both arms print: the workload, by what it is."""
    return {"workload": f"{w.name} ({w.n_q_heads}/{w.n_kv_heads} heads, d={w.head_dim})",
            "tokens_per_gpu": w.n_tokens, "seqs": w.n_seqs, "q_heads": w.n_q_heads,
            "kv_heads": w.n_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size,
            "pool_blocks": w.n_blocks, "note": w.note, "parallelism": f"replicas x{ws}"}


def run_reference(args, w, rank, ws):
    if rank != 0:
        return 0
    sub = oracle_sample(w)
    for _ in range(args.warmup):
        time_oracle(sub)
    times = [time_oracle(sub)[0] for _ in range(args.steps)]
    ms = 1000 * sum(times) / len(times)
    value = sub.n_tokens / (ms / 1000)
    cores = blas_threads()
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": workload_config(w, ws),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{sub.n_tokens} tokens per step (all decodes + first "
                                       f"{int(sub.q_lens.max())} tokens of each chunk)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------
class FgPass:
    """Device state of one workload on one GPU: the cache with its prior
    context, a batch handle, q/k/v resident in HBM and the L2 flush buffer."""

    def __init__(self, w, dev, overlap=False):
        import torch
        from ragged_paged_kv_b200 import fg, fixtures
        self.w, self.dev = w, dev
        self.stream = torch.cuda.Stream(device=dev)
        self.cache = fg.KVCache(w.block_size, w.n_blocks, w.n_kv_heads, w.head_dim, device=dev)
        fixtures.fill(self.cache.tensor, 0)
        # prior context: seeded N(0,1) bf16 blocks (a pool of them, reused
        # across sequences: same sizes and distribution, fast for any pool)
        fixtures.write_context(w, self.cache.tensor, keep=(), others="pool")
        self.batch = fg.RaggedBatch(w.n_tokens, w.n_seqs, w.block_tables.shape[1])
        self.batch.set_overlap(overlap)
        self.q, self.k, self.v = fixtures.qkv_device(w, dev)
        self.q_rot, self.out = torch.empty_like(self.q), torch.empty_like(self.q)
        self.flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.host_parts = {"put": 0.0, "append": 0.0, "attention": 0.0}
        # fused: one fg_rotary_kv_attention call instead of the two calls
        self.fused = False
        torch.cuda.synchronize()

    def step(self, ev):
        from ragged_paged_kv_b200 import fg
        w, st = self.w, self.stream
        ev[0].record(st)
        t0 = time.perf_counter()
        self.batch.put(self.cache, w.seq_ids, w.q_lens, w.ctx_lens, w.block_tables, st)
        t1 = time.perf_counter()
        ev[3].record(st)
        if self.fused:
            t2 = time.perf_counter()
            ev[1].record(st)
            fg.rotary_kv_attention(self.cache, self.batch, self.q, self.k, self.v, self.q_rot, self.out,
                                   w.n_q_heads, w.rope_theta, w.softmax_scale, w.sliding_window, st)
            t3 = time.perf_counter()
            ev[2].record(st)
            self.host_parts["put"] += t1 - t0
            self.host_parts["attention"] += t3 - t2
            return
        fg.rotary_kv_append(self.cache, self.batch, self.q, self.k, self.v, self.q_rot, w.n_q_heads,
                            w.rope_theta, st)
        t2 = time.perf_counter()
        ev[1].record(st)
        fg.ragged_attention(self.cache, self.batch, self.q_rot, self.out, w.n_q_heads, w.softmax_scale,
                            w.sliding_window, st)
        t3 = time.perf_counter()
        ev[2].record(st)
        self.host_parts["put"] += t1 - t0
        self.host_parts["append"] += t2 - t1
        self.host_parts["attention"] += t3 - t2

    def flush_l2(self):
        # write a buffer larger than L2 (evicts every line of the step), then
        # read it back, so that the write-back of the dirty flush lines is
        # paid here and not by the first kernel of the next step
        import torch
        with torch.cuda.stream(self.stream):
            self.flush.zero_()
            self.flush.sum()

    def close(self):
        import torch
        torch.cuda.synchronize()
        self.cache.close()
        self.batch.close()
        del self.cache, self.batch, self.q, self.k, self.v, self.q_rot, self.out, self.flush
        torch.cuda.empty_cache()


def _events():
    import torch
    return [torch.cuda.Event(enable_timing=True) for _ in range(4)]


def device_timing(fp, steps, warmup, local_rank):
    """W untimed steps, then K timed steps (CUDA events on the launching
    stream, barrier + synchronize on both sides, L2 flushed before each step
    outside the events), with the clocks sampled during the timed region; then
    a second pass with the library's per-kernel events. Times are the max over
    ranks of each rank's mean."""
    import torch
    dev = fp.dev
    for _ in range(warmup):
        fp.step(_events())
        fp.flush_l2()
    torch.cuda.synchronize()
    fp.batch.device_status(fp.stream)
    evs = [_events() for _ in range(steps)]
    host_s = 0.0
    for k_ in fp.host_parts:
        fp.host_parts[k_] = 0.0
    fp.batch.host_profile_us(reset=True)
    # the sampler thread is started before the barrier, and every step
    # (the first included) is preceded by the L2 flush, so the device has
    # queued work while the host enqueues a step, as it does between steps;
    # a short interpreter switch interval lets the sampler thread run every
    # couple of milliseconds while the main thread enqueues
    switch = sys.getswitchinterval()
    sys.setswitchinterval(2e-4)
    with ClockSampler(local_rank) as clocks:
        barrier()
        torch.cuda.synchronize()
        for i in range(steps):
            # before the first step the flush is repeated (about 1.3 ms of
            # device work), so that the host has validated and enqueued the
            # first step before the device gets to it: batches of hundreds of
            # sequences take the host about 0.6 ms, and later steps find the
            # host ahead of the device, as in a serving loop
            for _ in range(16 if i == 0 else 1):
                fp.flush_l2()
            t0 = time.perf_counter()
            fp.step(evs[i])
            host_s += time.perf_counter() - t0
        torch.cuda.synchronize()
        barrier()
    sys.setswitchinterval(switch)
    lib_host = {k_: v_ / steps for k_, v_ in fp.batch.host_profile_us(reset=True).items()}
    step_ms = [e[0].elapsed_time(e[2]) for e in evs]
    put_ms = sum(e[0].elapsed_time(e[3]) for e in evs) / len(evs)
    append_ms = sum(e[3].elapsed_time(e[1]) for e in evs) / len(evs)
    attn_ms = [e[1].elapsed_time(e[2]) for e in evs]
    ms = max_over_ranks(sum(step_ms) / len(step_ms), dev)
    attn_ms_mean = max_over_ranks(sum(attn_ms) / len(attn_ms), dev)
    fp.batch.device_status(fp.stream)
    info = fp.batch.plan_info()
    host_parts = {k_: 1000 * v_ / steps for k_, v_ in fp.host_parts.items()}

    # per-kernel durations: the library's own CUDA events around each kernel,
    # on the stream it runs on (a separate pass, synchronised per step so
    # the events of every step can be read; the kernels run exactly as above)
    fp.batch.set_timing(True)
    kms = []
    for _ in range(steps):
        fp.step(_events())
        kms.append(fp.batch.kernel_ms())
        fp.flush_l2()
    fp.batch.set_timing(False)
    torch.cuda.synchronize()
    kernel_ms = {k: max_over_ranks(sum(d[k] for d in kms) / len(kms), dev) for k in kms[0]}
    return {"ms": ms, "attn_ms": attn_ms_mean, "put_ms": put_ms, "append_ms": append_ms,
            "kernel_ms": kernel_ms, "host_s": host_s, "host_parts": host_parts, "lib_host": lib_host,
            "info": info, "clocks": clocks.summary()}


def fused_timing(fp, steps, warmup, local_rank):
    """The same step through fg_rotary_kv_attention (one call: rotary +
    append + attention, the query tiles' Q rotated in the query-tile
    kernel's load): W untimed steps, then K timed steps, CUDA events on the
    launching stream around each step, L2 flushed before each step outside
    the events; the max over ranks of each rank's mean (ms)."""
    import torch
    fp.fused = True
    for _ in range(warmup):
        fp.step(_events())
        fp.flush_l2()
    torch.cuda.synchronize()
    evs = [_events() for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    for i in range(steps):
        for _ in range(16 if i == 0 else 1):
            fp.flush_l2()
        fp.step(evs[i])
    torch.cuda.synchronize()
    barrier()
    fp.fused = False
    fp.batch.device_status(fp.stream)
    return max_over_ranks(sum(e[0].elapsed_time(e[2]) for e in evs) / steps, fp.dev)


def roofline_of(w, config, m):
    """The `roofline` object for the dominant kernel of workload w (the one
    with the longest average launch), from the measurements `m`."""
    work = algorithmic_work(w)
    hbm, tf, src = load_peaks()
    kernel_ms = m["kernel_ms"]
    dom = max(("decode", "tc"), key=lambda k: kernel_ms[k])
    if dom == "decode":
        achieved = work["decode_bytes"] / (kernel_ms["decode"] / 1000) / 1e9
        roof = {"kernel": "decode (attn_decode_tc_kernel at d=128, attn_decode_kernel at d=64)", "bound": "hbm",
                "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": ncu_traffic(config, "decode"), "algorithmic_bytes": work["decode_bytes"]}
    elif work["tc_flops"] / (tf * 1e12) >= work["tc_bytes"] / (hbm * 1e9):
        achieved = work["tc_flops"] / (kernel_ms["tc"] / 1000) / 1e12
        roof = {"kernel": "attn_tc_kernel (tcgen05 tiles)", "bound": "tensor", "achieved": achieved,
                "peak": tf, "unit": "TFLOP/s", "frac": achieved / tf, "traffic": ncu_traffic(config, "tc"),
                "algorithmic_flops": work["tc_flops"]}
    else:  # its tiles are mostly grouped-query decodes: bound by the K/V bytes
        achieved = work["tc_bytes"] / (kernel_ms["tc"] / 1000) / 1e9
        roof = {"kernel": "attn_tc_kernel (tcgen05 tiles)", "bound": "hbm", "achieved": achieved,
                "peak": hbm, "unit": "GB/s", "frac": achieved / hbm, "traffic": ncu_traffic(config, "tc"),
                "algorithmic_bytes": work["tc_bytes"]}
    roof.update({"peak_source": f"{src} (MEASURED_PEAKS.json)" if src == "measured" else src,
                 "kernel_ms": kernel_ms,
                 "tc_TFLOPs": work["tc_flops"] / (kernel_ms["tc"] / 1000) / 1e12 if kernel_ms["tc"] else None,
                 "step_roofline_ms": 1000 * max((work["attn_bytes"] + work["append_bytes"]) / (hbm * 1e9),
                                                work["flops"] / (tf * 1e12))})
    roof["step_frac"] = roof["step_roofline_ms"] / m["ms"]
    return roof


def make_workload(config, compact_pool=False, local_rank=0, gpu=True):
    """Workload `config`; config 3's pool fills the GPU's free memory up to
    180 GB (less 8 GiB of headroom) when it runs on a GPU."""
    from ragged_paged_kv_b200 import workloads as W
    if config == 3 and gpu:
        import torch
        free, _ = torch.cuda.mem_get_info(local_rank)
        w = W.config3(n_blocks=int(min(180 * 10**9, free - 8 * 2**30) // (2 * 32 * 64 * 128 * 2)))
    else:
        w = W.CONFIGS[config]()
    if compact_pool:
        need = sum(w.blocks_used(s) for s in range(w.n_seqs))
        w = W._make(w.name, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block_size, w.seq_ids,
                    w.q_lens, w.ctx_lens, w.seed, w.budget, n_blocks=need + 16,
                    window=w.sliding_window, note=w.note + "; compact pool")
    return w


# the gates of the measured configurations: the dominant kernel's fraction of
# its roofline (HBM bandwidth for the decode-heavy batches, the bf16 tensor
# peak for the long-prompt batch)
GATES = {2: ("hbm", 0.70), 3: ("hbm", 0.70), 4: ("hbm", 0.70), 5: ("tensor", 0.50)}


def run_fg(args, w, rank, ws, local_rank):
    import torch
    from ragged_paged_kv_b200 import fg

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    fp = FgPass(w, dev, args.overlap)
    m = device_timing(fp, args.steps, args.warmup, local_rank)
    ms = m["ms"]
    fused_ms = fused_timing(fp, args.steps, args.warmup, local_rank)

    # end to end through the public API from pinned host buffers: each pass
    # uploads its q, k, v and downloads its output, pipelined across passes
    # (fg.HostPipeline: pass i + 1's upload and pass i - 1's download run
    # while pass i computes); the window runs from the first upload to the
    # last download, over K passes. The L2 flush still runs on the compute
    # stream after every pass.
    batch = fp.batch
    host_in = {n: t.cpu().pin_memory() for n, t in (("q", fp.q), ("k", fp.k), ("v", fp.v))}
    host_out = torch.empty(fp.out.shape, dtype=fp.out.dtype).pin_memory()
    pipe = fg.HostPipeline(fp.cache, w.n_tokens, w.n_q_heads, dev)

    def e2e_submit():
        pipe.submit(batch, w.seq_ids, w.q_lens, w.ctx_lens, w.block_tables, host_in["q"], host_in["k"],
                    host_in["v"], host_out, w.rope_theta, w.softmax_scale, w.sliding_window)
        with torch.cuda.stream(pipe.comp):
            fp.flush.zero_()
            fp.flush.sum()

    for _ in range(max(3, args.warmup)):
        e2e_submit()
    pipe.drain()
    torch.cuda.synchronize()
    barrier()
    # a continuous stream: warm-up passes are still in flight when the window
    # opens (at the end of the last warm-up upload), so the window holds the
    # K timed passes' uploads, computes and downloads in steady state, not
    # the pipeline's one-time fill and drain
    for _ in range(max(3, args.warmup)):
        e2e_submit()
    e2e_start, e2e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_start.record(pipe.up)
    for i in range(args.steps):
        e2e_submit()
    e2e_end.record(pipe.down)
    pipe.drain()
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e2e_start.elapsed_time(e2e_end) / args.steps, dev)
    batch.device_status(pipe.comp)
    # the link's own ceiling: the same q, k, v bytes as plain pinned
    # host-to-device copies, back to back (no compute, no download)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(pipe.up):
        c0.record(pipe.up)
        for _ in range(args.steps):
            for n in ("q", "k", "v"):
                pipe.bufs[0][n][:w.n_tokens].copy_(host_in[n], non_blocking=True)
        c1.record(pipe.up)
    c1.synchronize()
    h2d_only_ms = c0.elapsed_time(c1) / args.steps
    qkv_bytes = sum(t.numel() * 2 for t in host_in.values())
    # and both directions at once, as the pipeline runs them: the uploads on
    # one stream, the same number of output downloads on another
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(pipe.up)
    pipe.down.wait_event(d0)
    with torch.cuda.stream(pipe.up):
        for _ in range(args.steps):
            for n in ("q", "k", "v"):
                pipe.bufs[0][n][:w.n_tokens].copy_(host_in[n], non_blocking=True)
    with torch.cuda.stream(pipe.down):
        for _ in range(args.steps):
            host_out.copy_(pipe.bufs[1]["out"][:w.n_tokens], non_blocking=True)
    pipe.up.wait_stream(pipe.down)
    d1.record(pipe.up)
    d1.synchronize()
    both_ms = d0.elapsed_time(d1) / args.steps
    # the put's metadata upload: cu_q, ctx, bt_off, the per-row sequence,
    # position and block, and the compact block tables (int32)
    meta_bytes = 4 * (3 * w.n_seqs + 2 + 3 * w.n_tokens +
                      sum(w.blocks_used(s) for s in range(w.n_seqs)))
    h2d = sum(t.numel() * 2 for t in host_in.values()) + meta_bytes
    d2h = host_out.numel() * 2
    del host_in, host_out, pipe
    fp.close()

    # the other gated configurations, measured the same way in this run
    # (fewer steps), one object each under "per_config"
    per_config = {}
    launches = 2 * args.steps * (1 + m["info"]["launches"])
    if not args.no_per_config:
        for c in sorted(GATES):
            if c == args.config:
                continue
            wc = make_workload(c, args.compact_pool, local_rank)
            fpc = FgPass(wc, dev, args.overlap)
            mc = device_timing(fpc, args.per_config_steps, 3, local_rank)
            mc_fused = fused_timing(fpc, args.per_config_steps, 3, local_rank)
            fpc.close()
            rc = roofline_of(wc, c, mc)
            bound, gate = GATES[c]
            per_config[str(c)] = {
                "workload": f"{wc.name} ({wc.n_q_heads}/{wc.n_kv_heads} heads, d={wc.head_dim}, "
                            f"{wc.n_tokens} tokens, {wc.n_seqs} seqs, pool {wc.n_blocks} blocks)",
                "steps": args.per_config_steps, "warmup": 3, "ms_per_step": mc["ms"],
                "tokens_per_s": wc.n_tokens * ws / (mc["ms"] / 1000),
                "put_ms": mc["put_ms"], "append_ms": mc["append_ms"], "attention_call_ms": mc["attn_ms"],
                "dominant_kernel": rc["kernel"], "bound": rc["bound"], "achieved": rc["achieved"],
                "unit": rc["unit"], "peak": rc["peak"], "frac": rc["frac"], "traffic": rc["traffic"],
                "kernel_ms": rc["kernel_ms"], "tc_TFLOPs": rc["tc_TFLOPs"],
                "step_roofline_ms": rc["step_roofline_ms"], "step_frac": rc["step_frac"],
                "gate": {"bound": bound, "min_frac": gate, "met": rc["bound"] == bound and rc["frac"] >= gate},
                "clocks": mc["clocks"], "fused_q_rope_ms_per_step": mc_fused}
            launches += 2 * args.per_config_steps * (1 + mc["info"]["launches"])

    if rank != 0:
        return 0
    tokens = w.n_tokens * ws
    roof = roofline_of(w, args.config, m)
    work = algorithmic_work(w)
    roof.update({"attention_call_ms": m["attn_ms"],
                 "put_ms": m["put_ms"],
                 "append_ms": m["append_ms"],
                 "host_enqueue_ms_per_step": 1000 * m["host_s"] / args.steps,
                 "host_ms_per_call": m["host_parts"],
                 "library_host_us_per_step": m["lib_host"],
                 "attention_call_GBps": work["attn_bytes"] / (m["attn_ms"] / 1000) / 1e9})
    gb, gf = GATES.get(args.config, (None, None))
    if gb is not None:
        roof["gate"] = {"bound": gb, "min_frac": gf, "met": roof["bound"] == gb and roof["frac"] >= gf}
    line = {
        "metric": METRIC, "value": tokens / (ms / 1000), "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, ws),
        "l2": "flushed between steps (256 MB write, then the same 256 MB read back; outside the events)",
        "roofline": roof,
        "e2e": {"value": tokens / (e2e_ms / 1000), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "window": "K passes pipelined through fg.HostPipeline (upload of pass i+1 and download of pass "
                          "i-1 overlap pass i) in a continuous stream: from the end of the last warm-up upload "
                          "to the end of the K-th timed download, divided by K",
                "h2d_copy_only_ms_per_step": h2d_only_ms,
                "h2d_copy_only_GBps": qkv_bytes / (h2d_only_ms / 1000) / 1e9,
                "copies_both_directions_ms_per_step": both_ms},
        "fused_q_rope": {"ms_per_step": fused_ms, "value": tokens / (fused_ms / 1000), "unit": "tokens/s",
                         "entry": "fg_rotary_kv_attention",
                         "what": "the same pass in one call: the query-tile kernel reads its Q rows unrotated and "
                                 "rotates them in shared memory, the rotary kernel skips them; outputs and cache "
                                 "bit-identical to the two calls timed in value"},
        "gpu_launches": launches,
        "plan": dict(m["info"], overlap=args.overlap),
        "clocks": m["clocks"],
    }
    if per_config:
        line["per_config"] = per_config
    if ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)
    return 0


PHASES = {
    "softmax": ["wait_S", "load_S", "max", "rescale_O", "exp_and_store_P", "zero_V", "store_wait_and_arrive",
                "epilogue_wait", "epilogue_store", "unit_pop", None, "turn_wait"],
    "mma": ["unit_pop", "wait_K", "issue_S", "wait_V", "wait_P", "wait_O_free", "issue_PV"],
    "loader": ["unit_pop", "wait_Q_free", "wait_stage_free", "issue"],
}


def run_phase_trace(args, w):
    """Cycle accounting of the query-tile kernel's roles (the trace build,
    RAGGED_PAGED_KV_LIB=trace): the same steps as the bench, then one JSON
    line with, per role, the SM cycles spent in each phase summed over the
    CTAs and divided by the role's 64-key tiles, the mean kernel cycles per
    CTA, and per launch its event-timed duration beside the span from the
    first CTA's start to the last CTA's end (%globaltimer) and the spread of
    the CTA start times. Not a timing run: the marks themselves cost cycles,
    and the steps run without programmatic dependent launch (per-kernel
    events are on)."""
    import ctypes
    import torch
    from ragged_paged_kv_b200 import fg
    L = fg.lib()
    if not hasattr(L, "fg_phase_trace_read"):
        raise SystemExit("--phase-trace needs the trace build: python -m ragged_paged_kv_b200.build --trace "
                         "and RAGGED_PAGED_KV_LIB=trace")
    dev = torch.device("cuda", 0)
    fp = FgPass(w, dev)
    for _ in range(args.warmup):
        fp.step(_events())
        fp.flush_l2()
    buf = (ctypes.c_ulonglong * 64)()
    assert L.fg_phase_trace_read(buf, 64, 1) == 0
    # one launch per read: the table's timer slots then describe that launch;
    # the library's events give the same launch's duration on its stream
    fp.batch.set_timing(True)
    tot = [0] * 64
    spans = {"event_ms": [], "first_to_last_end_ms": [], "cta_start_skew_ms": []}
    for _ in range(args.steps):
        fp.step(_events())
        kms = fp.batch.kernel_ms()
        assert L.fg_phase_trace_read(buf, 64, 1) == 0
        tot = [a + b for a, b in zip(tot, list(buf))]
        spans["event_ms"].append(kms["tc"])
        spans["first_to_last_end_ms"].append((buf[60] - buf[58]) / 1e6)
        spans["cta_start_skew_ms"].append((buf[59] - buf[58]) / 1e6)
        fp.flush_l2()
    fp.batch.set_timing(False)
    v = tot
    out = {"kind": "phase_trace", "workload": w.name, "steps": args.steps,
           "ctas_per_launch": v[57] / args.steps, "cycles_per_cta": v[56] / max(1, v[57]),
           "launch_ms": {k: sum(x) / len(x) for k, x in spans.items()}}
    for t in range(2):
        base = 12 * t
        n = max(1, v[base + 10])
        out[f"softmax_tile{t}"] = {"tiles": v[base + 10],
                                   "cycles_per_tile": {k: v[base + i] / n for i, k in enumerate(PHASES["softmax"])
                                                       if k}}
        base = 24 + 8 * t
        n = max(1, v[base + 7])
        out[f"mma_tile{t}"] = {"tiles": v[base + 7],
                               "cycles_per_tile": {k: v[base + i] / n for i, k in enumerate(PHASES["mma"])}}
    for name, base in (("loader_K", 40), ("loader_V", 48)):
        n = max(1, v[base + 4])
        out[name] = {"tiles": v[base + 4],
                     "cycles_per_tile": {k: v[base + i] / n for i, k in enumerate(PHASES["loader"])}}
    print(json.dumps(out), flush=True)
    fp.close()
    return 0


def sweep_workload(n_tokens, n_decodes=32, seed=11):
    """Llama-2-7B-shape batch of n_tokens: n_decodes one-token decodes
    (contexts ~U[512, 4096]) plus one prompt chunk of the rest at context 1024."""
    from ragged_paged_kv_b200 import workloads as W
    rng = np.random.default_rng(seed)
    ctx = rng.integers(512, 4097, n_decodes).tolist()
    q = [1] * n_decodes
    if n_tokens > n_decodes:
        q.append(n_tokens - n_decodes)
        ctx.append(1024)
    return W._make(f"sweep_{n_tokens}", 32, 32, 128, 64, list(range(len(q))), q, ctx, seed=seed,
                   budget=int(sum(q)), note="token sweep")


def time_step(w, steps, warmup, dev):
    """Mean device time (ms) of put + rotary/append + attention over `steps`
    steps after `warmup`, L2 flushed (write + read of 256 MB) before each."""
    import torch
    from ragged_paged_kv_b200 import fg, fixtures
    stream = torch.cuda.Stream(device=dev)
    cache = fg.KVCache(w.block_size, w.n_blocks, w.n_kv_heads, w.head_dim, device=dev)
    fixtures.fill(cache.tensor, 0)
    fixtures.write_context(w, cache.tensor, keep=(), others="pool")
    batch = fg.RaggedBatch(w.n_tokens, w.n_seqs, w.block_tables.shape[1])
    q, k, v = fixtures.qkv_device(w, dev)
    q_rot, out = torch.empty_like(q), torch.empty_like(q)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    evs = []
    for i in range(warmup + steps):
        with torch.cuda.stream(stream):
            for _ in range(4 if i == warmup else 1):
                flush.zero_()
                flush.sum()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record(stream)
        batch.put(cache, w.seq_ids, w.q_lens, w.ctx_lens, w.block_tables, stream)
        fg.rotary_kv_append(cache, batch, q, k, v, q_rot, w.n_q_heads, w.rope_theta, stream)
        fg.ragged_attention(cache, batch, q_rot, out, w.n_q_heads, w.softmax_scale, w.sliding_window, stream)
        e[1].record(stream)
        if i >= warmup:
            evs.append(e)
    torch.cuda.synchronize()
    batch.device_status(stream)
    ms = sum(a.elapsed_time(b) for a, b in evs) / len(evs)
    cache.close()
    batch.close()
    return ms


def run_token_sweep(args):
    """Forward latency and throughput of the attention path against the
    tokens in a pass (the card's observation that latency follows the token
    count and throughput saturates, and its equal-split argument from the
    concavity of throughput): one JSON line per point, then the measured
    total time of splitting N tokens over two passes unevenly vs evenly."""
    import torch
    dev = torch.device("cuda", 0)
    pts = {}
    for n in (64, 128, 256, 512, 1024, 2048, 3072, 3584, 4096, 6144, 8192):
        ms = time_step(sweep_workload(n), args.steps, args.warmup, dev)
        pts[n] = ms
        print(json.dumps({"kind": "token_sweep", "tokens": n, "decodes": 32, "prefill_tokens": max(0, n - 32),
                          "ms_per_pass": ms, "tokens_per_s": n / ms * 1e3}), flush=True)
    for total, parts in ((4096, ((2048, 2048), (1024, 3072), (512, 3584))),
                         (8192, ((4096, 4096), (2048, 6144)))):
        for a, b in parts:
            print(json.dumps({"kind": "split_check", "total_tokens": total, "passes": [a, b],
                              "ms_total": pts[a] + pts[b]}), flush=True)
    return 0


def run_qkv_fused(args, w):
    """The Q/K/V projection fused with rotary + append, and the output
    projection, on the headline batch's tokens at Llama-2-7B width (hidden
    4096; 96 heads of 128 out, then 4096 -> 4096): one JSON line per GEMM with
    its device time, TFLOP/s and fraction of the measured bf16 peak (kinds
    "qkv_fused" and "out_proj", not the contract line)."""
    import torch
    from ragged_paged_kv_b200 import fg, fixtures
    dev = torch.device("cuda", 0)
    hidden = 4096
    stream = torch.cuda.Stream(device=dev)
    cache = fg.KVCache(w.block_size, w.n_blocks, w.n_kv_heads, w.head_dim, device=dev)
    fixtures.fill(cache.tensor, 0)
    fixtures.write_context(w, cache.tensor, keep=(), others="pool")
    batch = fg.RaggedBatch(w.n_tokens, w.n_seqs, w.block_tables.shape[1])
    g = torch.Generator(device=dev).manual_seed(7)
    x = torch.randn((w.n_tokens, hidden), generator=g, device=dev).to(torch.bfloat16)
    n_out = (w.n_q_heads + 2 * w.n_kv_heads) * w.head_dim
    wq = (torch.randn((n_out, hidden), generator=g, device=dev) / hidden ** 0.5).to(torch.bfloat16)
    q_rot = torch.empty((w.n_tokens, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    batch.put(cache, w.seq_ids, w.q_lens, w.ctx_lens, w.block_tables, stream)
    evs = []
    for i in range(args.warmup + args.steps):
        with torch.cuda.stream(stream):
            flush.zero_()
            flush.sum()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record(stream)
        fg.qkv_rotary_kv_append(cache, batch, x, wq, q_rot, w.n_q_heads, w.rope_theta, stream)
        e[1].record(stream)
        if i >= args.warmup:
            evs.append(e)
    torch.cuda.synchronize()
    batch.device_status(stream)
    ms = sum(a.elapsed_time(b) for a, b in evs) / len(evs)
    flops = 2.0 * w.n_tokens * hidden * n_out
    hbm, tf, src = load_peaks()
    print(json.dumps({"kind": "qkv_fused", "workload": f"{w.name}: T={w.n_tokens}, hidden={hidden}, out={n_out}",
                      "ms": ms, "tflops": flops / ms / 1e9, "peak_tflops": tf, "frac": flops / ms / 1e9 / tf,
                      "peak_source": src}), flush=True)

    # the output projection: the attention output [T, Hq d] times W_o^T
    k_in = w.n_q_heads * w.head_dim
    o = torch.randn((w.n_tokens, k_in), generator=g, device=dev).to(torch.bfloat16)
    wo = (torch.randn((hidden, k_in), generator=g, device=dev) / k_in ** 0.5).to(torch.bfloat16)
    y = torch.empty((w.n_tokens, hidden), dtype=torch.bfloat16, device=dev)
    evs = []
    for i in range(args.warmup + args.steps):
        with torch.cuda.stream(stream):
            flush.zero_()
            flush.sum()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record(stream)
        fg.output_projection(batch, o, wo, y, stream)
        e[1].record(stream)
        if i >= args.warmup:
            evs.append(e)
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in evs) / len(evs)
    flops = 2.0 * w.n_tokens * k_in * hidden
    print(json.dumps({"kind": "out_proj", "workload": f"{w.name}: T={w.n_tokens}, in={k_in}, out={hidden}",
                      "ms": ms, "tflops": flops / ms / 1e9, "peak_tflops": tf, "frac": flops / ms / 1e9 / tf,
                      "peak_source": src}), flush=True)
    return 0


class BlockAllocator:
    """Free list over the pool's block ids (host side of the paged cache):
    a sequence gets blocks as its context grows and returns them when it
    finishes."""

    def __init__(self, n_blocks, block_size, seed=0):
        ids = np.random.default_rng(seed).permutation(n_blocks)
        self.free = [int(b) for b in ids]
        self.B = block_size
        self.owned = {}

    def ensure(self, rid, length):
        have = self.owned.setdefault(rid, [])
        need = -(-length // self.B)
        while len(have) < need:
            if not self.free:
                raise RuntimeError("block pool exhausted")
            have.append(self.free.pop())
        return have

    def release(self, rid):
        self.free.extend(self.owned.pop(rid, []))


def run_serve_sim(args, policy="greedy"):
    """A timed Dynamic SplitFuse loop with attention only (no weights): the
    composer's closed loop of synthetic clients (32 active of 512 requests,
    prompt ~N(2600, 30 %), output ~N(60, 30 %), budget 2048: the card's
    workload, Key points) drives put + rotary/append + attention on one GPU
    at the Llama-2-7B attention shape, with blocks taken from a free list as
    contexts grow and returned when a request finishes; the cache is built
    through the API, chunk by chunk. Each iteration's device time (CUDA
    events) advances a clock; a request arrives when it becomes active, gets
    its first token at the end of the iteration that completes its prompt
    and one more at the end of every later iteration; a device spin queued
    ahead of each pass keeps a host pause out of its events. One JSON line (kind
    "serve_sim"): throughput, percentiles of time to first token and of the
    mean time per output token, and the requests per second that meet the
    latency targets (--sla-ttft-ms, --sla-tpot-ms). `policy` is the
    composer's chunking policy ("greedy": every pass filled while prompt
    tokens are pending; "equal_split": the pending prompt tokens spread evenly
    over the passes they need)."""
    import torch
    from ragged_paged_kv_b200 import fg, workloads as W
    dev = torch.device("cuda", 0)
    Hq = Hkv = 32
    d, B, budget = 128, 64, 2048
    n_blocks = 4096
    cache = fg.KVCache(B, n_blocks, Hkv, d, device=dev)
    alloc = BlockAllocator(n_blocks, B, seed=1)
    batch = fg.RaggedBatch(budget, 64, 128)
    g = torch.Generator(device=dev).manual_seed(3)
    q = torch.randn((budget, Hq, d), generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn((budget, Hkv, d), generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn((budget, Hkv, d), generator=g, device=dev).to(torch.bfloat16)
    q_rot, out = torch.empty_like(q), torch.empty_like(q)
    stream = torch.cuda.Stream(device=dev)
    scale = 1.0 / d ** 0.5
    # start-up work a server does once, outside the loop: the rotary table
    # for the longest context (prompts stay below 8192 tokens here), and one
    # untimed pass through the whole schedule, so that module loading, launch
    # set-up and the growth of the batch's staging and plan buffers to the
    # largest pass (a server sizes them once) are not counted
    cache.prepare_rotary(10000.0, 8191)

    def one_pass(bt, alloc_):
        rids = np.array([b[0] for b in bt], np.int32)
        ql = np.array([b[1] for b in bt], np.int32)
        cl = np.array([b[2] for b in bt], np.int32)
        tabs = [alloc_.ensure(int(r), int(c + n)) for r, n, c in zip(rids, ql, cl)]
        tab = np.full((len(bt), max(len(t) for t in tabs)), -1, np.int32)
        for i, t in enumerate(tabs):
            tab[i, :len(t)] = t
        T = int(ql.sum())
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        # about 1 ms of device spin ahead of the pass, so that the device is
        # still busy while the host validates and enqueues it: the events then
        # time the device's work, not a pause of the host (a garbage
        # collection, a page fault) between them
        with torch.cuda.stream(stream):
            torch.cuda._sleep(2_000_000)
        e0.record(stream)
        batch.put(cache, rids, ql, cl, tab, stream)
        fg.rotary_kv_append(cache, batch, q[:T], k[:T], v[:T], q_rot[:T], Hq, 10000.0, stream)
        fg.ragged_attention(cache, batch, q_rot[:T], out[:T], Hq, scale, 0, stream)
        e1.record(stream)
        e1.synchronize()
        return T, e0.elapsed_time(e1)

    warm_alloc = BlockAllocator(n_blocks, B, seed=1)
    warm_events = []
    warm_seen = 0
    for it, bt in W.splitfuse_schedule(seed=2, budget=budget, policy=policy, events=warm_events):
        for _, _, _, left in warm_events[warm_seen:]:
            for r in left:
                warm_alloc.release(r)
        warm_seen = len(warm_events)
        one_pass(bt, warm_alloc)
    torch.cuda.synchronize()

    events = []
    arrive = {rid: 0.0 for rid in range(32)}
    first, last, n_out = {}, {}, {}
    clock = 0.0
    iters = tokens = 0
    seen = 0
    pass_ms, pass_tokens = [], []

    def settle():
        # the composer reports an iteration's outcome when it is resumed for
        # the next one: tokens produced (at the clock's current value, the end
        # of that iteration), requests that left and those that joined
        nonlocal seen
        for _, produced, joined, left in events[seen:]:
            for r, is_first in produced:
                if is_first:
                    first[r] = clock
                last[r] = clock
                n_out[r] = n_out.get(r, 0) + 1
            for r in left:
                alloc.release(r)
            for r in joined:
                arrive[r] = clock
        seen = len(events)

    for it, bt in W.splitfuse_schedule(seed=2, budget=budget, events=events, policy=policy):
        settle()
        T, ms = one_pass(bt, alloc)
        pass_ms.append(ms)
        pass_tokens.append(T)
        clock += ms
        iters += 1
        tokens += T
    settle()
    batch.device_status(stream)
    done = sorted(first)
    ttft = np.array([first[r] - arrive[r] for r in done])
    tpot = np.array([(last[r] - first[r]) / (n_out[r] - 1) for r in done if n_out[r] > 1])
    meets = [r for r in done if first[r] - arrive[r] <= args.sla_ttft_ms and
             (n_out[r] <= 1 or (last[r] - first[r]) / (n_out[r] - 1) <= args.sla_tpot_ms)]
    pct = lambda a, p: float(np.percentile(a, p)) if len(a) else None
    print(json.dumps({
        "kind": "serve_sim", "policy": policy,
        "workload": "Llama-2-7B attention shape, 32 active of 512 requests, budget 2048",
        "iterations": iters, "tokens": tokens, "requests": len(done), "device_s": clock / 1e3,
        "tokens_per_s": tokens / clock * 1e3, "requests_per_s": len(done) / clock * 1e3,
        "ttft_ms": {"p50": pct(ttft, 50), "p95": pct(ttft, 95)},
        "tpot_ms": {"p50": pct(tpot, 50), "p95": pct(tpot, 95)},
        "pass_ms": {"p50": pct(pass_ms, 50), "p95": pct(pass_ms, 95), "max": max(pass_ms)},
        "pass_tokens": {"p50": pct(pass_tokens, 50), "min": min(pass_tokens), "max": max(pass_tokens)},
        "sla": {"ttft_ms": args.sla_ttft_ms, "tpot_ms": args.sla_tpot_ms,
                "effective_requests_per_s": len(meets) / clock * 1e3}}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["fg", "reference"], default="fg")
    ap.add_argument("--config", type=int, default=2, help="workload number (2 = the headline)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="measure only the chosen config (no per_config object for the other gated configs)")
    ap.add_argument("--per-config-steps", type=int, default=5)
    ap.add_argument("--overlap", action="store_true",
                    help="run the query-tile kernel beside the decode kernel on a second stream")
    ap.add_argument("--compact-pool", action="store_true",
                    help="size the block pool to what the batch uses (small ncu captures)")
    ap.add_argument("--qkv-fused", action="store_true",
                    help="time the fused Q/K/V projection + rotary + append and the output projection (one GPU; JSON lines, no contract line)")
    ap.add_argument("--phase-trace", action="store_true",
                    help="cycle accounting of the query-tile kernel's roles (trace build; JSON line, no contract line)")
    ap.add_argument("--serve-sim", action="store_true",
                    help="timed SplitFuse loop with closed-loop synthetic clients (one GPU; JSON line)")
    ap.add_argument("--policy", choices=["greedy", "equal_split", "both"], default="both",
                    help="--serve-sim: the composer's chunking policy (both: one line each)")
    ap.add_argument("--sla-ttft-ms", type=float, default=30.0)
    ap.add_argument("--sla-tpot-ms", type=float, default=1.0)
    ap.add_argument("--sweep-tokens", action="store_true",
                    help="latency/throughput against tokens per pass (one GPU; JSON lines, no contract line)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.sweep_tokens:
        return run_token_sweep(args)
    if args.serve_sim:
        from ragged_paged_kv_b200 import workloads as W
        for pol in (W.POLICIES if args.policy == "both" else (args.policy,)):
            rc = run_serve_sim(args, pol)
            if rc:
                return rc
        return 0
    w = make_workload(args.config, args.compact_pool, world()[2], gpu=args.impl == "fg")
    if args.qkv_fused:
        return run_qkv_fused(args, w)
    if args.phase_trace:
        return run_phase_trace(args, w)
    if args.impl == "reference":
        rank, ws = init_dist("gloo")
        rc = run_reference(args, w, rank, ws)
    else:
        import torch
        rank, ws = init_dist("nccl")
        rc = run_fg(args, w, rank, ws, world()[2])
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
