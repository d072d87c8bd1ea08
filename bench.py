"""Benchmark of the attention hot path on B200: one JSON line on rank 0.

A step is one pass of the hot path over one batch of synthetic inputs:
causal GQA prefill of the Llama-3-8B-shaped batch (B=4, Hq=32, Hkv=8,
N=4096, d=128) followed by one paged decode step of 64 sequences (context
uniform in [1024, 32768], Hq=32, Hkv=8, d=128, 16-token blocks). The headline
`value` is the prefill's TFLOP/s (causal FLOPs: only visible pairs count);
the decode's KV GB/s sits under "decode". Inputs are resident in HBM before
the timed region. Before every timed prefill L2 is flushed (a 256 MiB write).
An HBM-bound launch is flushed by a 256 MiB write followed by a 256 MiB read
of another buffer, which leaves L2 holding clean lines of neither the
workload nor the write (a write flush alone leaves dirty lines that would be
written back inside the timed region); a decode whose cache is more than twice
the L2 size is timed without a flush (its inputs are larger than L2: nothing it
reads can still be there).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

With N > 1 (launched by torch.distributed.run) every rank runs its own
independent batch (weak scaling, no collective on the data path); the time
is the max over ranks and `value` counts the work of all ranks.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_softmax_attention_causal_b200 import accounting, sharding, workloads  # noqa: E402

METRIC = "prefill causal-GQA TFLOP/s & paged-decode KV GB/s, % of B200 peak"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------------------
# environment
# ----------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return {"hbm_gbs": float(m["hbm_gbs"]), "bf16_tflops": float(m["bf16_tflops"]),
                "bf16_tflops_sustained": float(m.get("bf16_tflops_sustained", m["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, sampled while running.

    Reads NVML every 2 ms from a background thread (read-only queries; nothing
    about the GPU is changed), so even a timed region of a few tens of
    milliseconds gets many samples. Falls back to `nvidia-smi -lms 25` when
    NVML is unavailable.
    """

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, gpu_index: int, period_s: float = 0.002):
        self.gpu = gpu_index
        self.period = period_s
        self.proc = None
        self.lines = []
        self.samples = []  # (sm_mhz, max_mhz, reason bits)
        self.thread = None
        self.stop = threading.Event()
        self.source = None

    def _nvml_handle(self):
        import pynvml

        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _poll_nvml(self, nv, h):
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((float(sm), float(mx), int(bits)))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.thread = threading.Thread(target=self._poll_nvml, args=(nv, h), daemon=True)
            self.thread.start()
            self.source = "nvml, every 2 ms"
            return self
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "25"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            self.source = "nvidia-smi, every 25 ms"
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        self.stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        for s_mhz, m_mhz, bits in self.samples:
            sm.append(s_mhz)
            mx = m_mhz
            for name, bit in self.REASONS:
                if bits & bit:
                    reasons.add(name)
        names = [n for n, _ in self.REASONS]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0, "source": self.source}
        loaded = [s for s in sm if mx is None or s >= 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": self.source}


def kernel_source_hash(name: str) -> str:
    path = os.path.join(ROOT, "exact_softmax_attention_causal_b200", "csrc", name)
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel: str, source: str, kv_bytes: int | None = None):
    """DRAM bytes per launch from a committed ncu capture (profiles/traffic.json),
    or None once the kernel source has changed since the counters were taken.
    A capture of a smaller case is scaled to this launch by its KV bytes."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_sha256_16") != kernel_source_hash(source):
        return None
    if "bytes_per_launch" in rec:
        return rec["bytes_per_launch"]
    if "bytes_per_kv_byte" in rec and kv_bytes is not None:
        return int(rec["bytes_per_kv_byte"] * kv_bytes)
    return None


def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))

def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ----------------------------------------------------------------------------
# the fp64 CPU oracle, timed on the host cores (cpu_baseline and --impl reference)
# ----------------------------------------------------------------------------
def oracle_prefill_heads(x, cfg, heads, budget_s=None):
    """Run the oracle over whole (batch, head) slices of the prefill workload.

    Returns (flops, seconds, heads_done). Stops early once budget_s is spent
    (at least one head always runs).
    """
    import oracle  # the oracle is only ever loaded by the baseline legs

    B, Hq, N, d = cfg["B"], cfg["Hq"], cfg["N"], cfg["d"]
    kind = accounting.MASK_IDS[cfg["mask"]]
    per_head = 4 * d * accounting.visible_pairs(N, cfg["mask"], cfg["window"])
    scale = workloads.default_scale(d)
    rows = range(N)
    done = 0
    t0 = time.perf_counter()
    for i in range(heads):
        bh = (i * 37) % (B * Hq)  # spread the sample over batches and heads
        oracle.prefill_rows_ref(x.q, x.k, x.v, bh // Hq, bh % Hq, rows, kind, cfg["window"], scale)
        done += 1
        if budget_s is not None and time.perf_counter() - t0 >= budget_s:
            break
    return per_head * done, time.perf_counter() - t0, done


def oracle_config_rate(op, cfg, x, budget_s):
    """The oracle on a bounded sample of one workload: evenly spaced query rows
    of (batch, head) slices for a prefill (TFLOP/s over their visible pairs),
    whole sequences' heads for a decode (GB/s of the K/V they read)."""
    import oracle  # the oracle is only ever loaded by the baseline legs

    t0 = time.perf_counter()
    work, done = 0, []
    if op == "prefill":
        B, Hq, N, d = cfg["B"], cfg["Hq"], cfg["N"], cfg["d"]
        kind = accounting.MASK_IDS[cfg["mask"]]
        rows = list(range(0, N, max(1, N // 256)))
        for i in range(B * Hq):
            bh = (i * 37) % (B * Hq)
            oracle.prefill_rows_ref(x.q, x.k, x.v, bh // Hq, bh % Hq, rows, kind, cfg["window"],
                                    workloads.default_scale(d))
            work += 4 * d * sum(accounting.row_visible_keys(N, i, cfg["mask"], cfg["window"]) for i in rows)
            done.append(bh)
            if time.perf_counter() - t0 >= budget_s:
                break
        secs = time.perf_counter() - t0
        return {"value": work / secs / 1e12, "unit": "TFLOP/s",
                "sample": f"{len(rows)} evenly spaced rows of {len(done)} (batch, head) slices, {secs:.1f} s"}
    Hq, Hkv, d = cfg["Hq"], cfg["Hkv"], cfg["d"]
    for b in range(x.q.shape[0]):
        oracle.decode_rows_ref(x.q, x.k_cache, x.v_cache, x.block_table, x.seq_lens, b, range(Hq),
                               workloads.default_scale(d))
        work += int(x.seq_lens[b]) * Hkv * d * 4
        done.append(b)
        if time.perf_counter() - t0 >= budget_s:
            break
    secs = time.perf_counter() - t0
    return {"value": work / secs / 1e9, "unit": "GB/s",
            "sample": f"all {Hq} heads of {len(done)} sequence(s), {secs:.1f} s"}


def cpu_baseline(x, cfg, budget_s):
    flops, secs, done = oracle_prefill_heads(x, cfg, heads=cfg["B"] * cfg["Hq"], budget_s=budget_s)
    return {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
            "cpu_model": cpu_model(), "blas_threads": oracle_threads(),
            "sample": f"{done} of {cfg['B'] * cfg['Hq']} (batch, head) slices of the {cfg['name']} prefill, "
                      f"all {cfg['N']} rows each, fp64 NumPy (one process, BLAS-threaded matmuls), {secs:.1f} s"}


def run_reference(args, cfg):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0  # the oracle arm runs once, on rank 0
    x = workloads.prefill_inputs(cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["N"], cfg["d"], args.seed)
    heads_per_step = args.reference_heads
    for _ in range(args.warmup):
        oracle_prefill_heads(x, cfg, heads_per_step)
    flops = 0
    secs = 0.0
    for _ in range(args.steps):
        f, s, _ = oracle_prefill_heads(x, cfg, heads_per_step)
        flops += f
        secs += s
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(cfg, args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
                         "sample": f"{heads_per_step} (batch, head) slices of the {cfg['name']} prefill per step, "
                                   f"all {cfg['N']} rows each"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_block(cfg, n_gpus):
    return {"workload": cfg["name"], "B": cfg["B"], "Hq": cfg["Hq"], "Hkv": cfg["Hkv"], "N": cfg["N"],
            "d": cfg["d"], "mask": cfg["mask"], "window": cfg["window"], "global_batch": cfg["B"] * n_gpus,
            "seq_len": cfg["N"], "parallelism": f"independent batch per GPU x{n_gpus}",
            "l2": "prefill: flushed (256 MiB write) before every timed launch; decode: inputs larger than L2 "
                  "(a cache of more than twice the L2 size, timed without a flush)"}

# ----------------------------------------------------------------------------
# the CUDA path
# ----------------------------------------------------------------------------
def run_ours(args, pcfg, dcfg):
    import exact_softmax_attention_causal_b200 as attn

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)
    seed = sharding.rank_seed(args.seed, rank)  # every rank owns an independent batch

    B, Hq, Hkv, N, d = pcfg["B"], pcfg["Hq"], pcfg["Hkv"], pcfg["N"], pcfg["d"]
    xp = workloads.prefill_inputs(B, Hq, Hkv, N, d, seed)
    q, k, v = xp.q.to(dev), xp.k.to(dev), xp.v.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    p_flops = accounting.prefill_flops(B, Hq, N, d, pcfg["mask"], pcfg["window"])

    dB, dHq, dHkv, dd = dcfg["B"], dcfg["Hq"], dcfg["Hkv"], dcfg["d"]
    xd = workloads.paged_decode_inputs(dB, dHq, dHkv, dd, len_range=dcfg.get("len_range"),
                                       seq_lens=dcfg.get("seq_lens"), block_size=dcfg["block_size"], seed=seed)
    dq, kc, vc = xd.q.to(dev), xd.k_cache.to(dev), xd.v_cache.to(dev)
    bt, sl = xd.block_table.to(dev), xd.seq_lens.to(dev)
    sl_dev = sl
    xd_q_host, xd_bt_host, xd_sl_host = xd.q, xd.block_table, xd.seq_lens
    dout = torch.empty_like(dq)
    dlse = torch.empty((dB, dHq), dtype=torch.float32, device=dev)
    ws = torch.empty(attn.decode_workspace_bytes(dB, dHq, dHkv, dd, xd.max_seq_len, xd.block_size),
                     dtype=torch.uint8, device=dev)
    kv_bytes = accounting.decode_kv_bytes(xd.seq_lens.tolist(), dHkv, dd)
    del xd
    decode_flush = needs_flush(kv_bytes, dev)

    flush = L2Flush(dev)

    def step(ev=None):
        flush("write")
        if ev:
            ev[0].record()
        attn.prefill(q, k, v, mask=pcfg["mask"], window=pcfg["window"], out=o, lse=lse)
        if ev:
            ev[1].record()
        if decode_flush:
            flush("clean")
        if ev:
            ev[2].record()
        attn.decode_paged(dq, kc, vc, bt, sl, dcfg_max_len(dcfg), out=dout, lse=dlse, workspace=ws)
        if ev:
            ev[3].record()

    def barrier():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    region = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    with ClockSampler(local) as clk:
        for _ in range(args.warmup):
            step()
        barrier()
        region[0].record()
        for i in range(args.steps):
            step(events[i])
        region[1].record()
        barrier()
    p_ms = sum(e[0].elapsed_time(e[1]) for e in events)
    d_ms = sum(e[2].elapsed_time(e[3]) for e in events)
    region_ms = region[0].elapsed_time(region[1])

    # End to end through the public API: every step copies its Q, K, V in from
    # pinned host memory and its O and LSE back out. Steps are pipelined as a
    # server would run a stream of requests: step i's input copy (copy stream
    # in), step i - 1's prefill (compute stream) and step i - 2's result copy
    # (copy stream out) overlap, over two device buffer sets.
    hq, hk, hv = xp.q.pin_memory(), xp.k.pin_memory(), xp.v.pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    bufs = [(q, k, v, o, lse)] + [tuple(torch.empty_like(t) for t in (q, k, v, o, lse))]
    hout = [(torch.empty(o.shape, dtype=o.dtype, pin_memory=True),
             torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)) for _ in range(2)]
    d2h = sum(t.numel() * t.element_size() for t in hout[0])
    s_in, s_out, s_cmp = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    loaded = [torch.cuda.Event() for _ in range(2)]
    computed = [None, None]
    drained = [None, None]
    e2e_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    barrier()
    main = torch.cuda.current_stream(dev)
    e2e_ev[0].record(main)
    for st in (s_in, s_out, s_cmp):
        st.wait_event(e2e_ev[0])
    for i in range(args.steps):
        sl = i % 2
        bq, bk, bv, bo, bl = bufs[sl]
        with torch.cuda.stream(s_in):  # the previous prefill on this buffer set has read its inputs
            if computed[sl] is not None:
                s_in.wait_event(computed[sl])
            bq.copy_(hq, non_blocking=True)
            bk.copy_(hk, non_blocking=True)
            bv.copy_(hv, non_blocking=True)
            loaded[sl].record(s_in)
        with torch.cuda.stream(s_cmp):  # inputs landed; the previous result copy has read O and LSE
            s_cmp.wait_event(loaded[sl])
            if drained[sl] is not None:
                s_cmp.wait_event(drained[sl])
            attn.prefill(bq, bk, bv, mask=pcfg["mask"], window=pcfg["window"], out=bo, lse=bl, stream=s_cmp)
            computed[sl] = torch.cuda.Event()
            computed[sl].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[sl])
            hout[sl][0].copy_(bo, non_blocking=True)
            hout[sl][1].copy_(bl, non_blocking=True)
            drained[sl] = torch.cuda.Event()
            drained[sl].record(s_out)
    for ev in drained:
        if ev is not None:
            main.wait_event(ev)
    e2e_ev[1].record(main)
    barrier()
    e2e_ms = e2e_ev[0].elapsed_time(e2e_ev[1])

    # The decode half end to end: every step copies its new query tokens, block
    # table and context lengths in from pinned host memory, decodes against the
    # cache already resident in HBM, and copies O and LSE back out.
    hdq, hbt, hsl = (t.pin_memory() for t in (xd_q_host, xd_bt_host, xd_sl_host))
    dh2d = sum(t.numel() * t.element_size() for t in (hdq, hbt, hsl))
    hdo = torch.empty(dout.shape, dtype=dout.dtype, pin_memory=True)
    hdl = torch.empty(dlse.shape, dtype=dlse.dtype, pin_memory=True)
    dd2h = sum(t.numel() * t.element_size() for t in (hdo, hdl))
    dq2, bt2, sl2 = torch.empty_like(dq), torch.empty_like(bt), torch.empty_like(sl_dev)
    barrier()
    de2e_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    de2e_ev[0].record(main)
    for _ in range(args.steps):
        dq2.copy_(hdq, non_blocking=True)
        bt2.copy_(hbt, non_blocking=True)
        sl2.copy_(hsl, non_blocking=True)
        attn.decode_paged(dq2, kc, vc, bt2, sl2, dcfg_max_len(dcfg), out=dout, lse=dlse, workspace=ws)
        hdo.copy_(dout, non_blocking=True)
        hdl.copy_(dlse, non_blocking=True)
    de2e_ev[1].record(main)
    barrier()
    de2e_ms = de2e_ev[0].elapsed_time(de2e_ev[1])

    p_ms, d_ms, region_ms, e2e_ms, de2e_ms = sharding.max_over_ranks([p_ms, d_ms, region_ms, e2e_ms, de2e_ms],
                                                                      device=dev)

    # Every other configuration of the workload table, one entry point each,
    # timed the same way (CUDA events around each launch, L2 flushed before it,
    # max over ranks): the long-context causal and windowed prefills and the
    # GQA dial (MHA / GQA-8 / MQA) prefills and single-sequence decodes.
    del q, k, v, o, lse, dq, kc, vc, bt, dout, dlse, ws, bufs, dq2, bt2, sl2
    torch.cuda.empty_cache()
    peaks_all = measured_peaks()
    configs = []
    cfg_host = {}
    with ClockSampler(local) as clk_cfg:
        for op_name, wname in () if args.no_configs else CONFIG_SWEEP:
            op = setup_op(op_name, wname, dev, seed, peaks_all, keep_host=(rank == 0 and world == 1))
            ms = time_launches(op["launch"], args.config_steps, 3, flush, dist_on=world > 1, kind=op["flush"])
            (ms_max,) = sharding.max_over_ranks([ms], device=dev)
            per_launch_s = ms / args.config_steps / 1e3
            achieved = op["work"] / per_launch_s / op["scale_div"]
            configs.append({
                "workload": wname, "op": op_name, "unit": op["unit"],
                "value": sharding.job_throughput(op["work"], world, args.config_steps, ms_max) / op["scale_div"],
                "ms_per_launch": ms_max / args.config_steps, "work_per_launch": op["work"], "l2": op["l2"],
                "roofline": {"bound": op["bound"], "achieved": achieved, "peak": op["peak"], "unit": op["unit"],
                             "frac": achieved / op["peak"], "kernel": op["kernel"]},
            })
            if "host" in op["extra"]:
                cfg_host[wname] = (op_name, op["cfg"], op["extra"]["host"])
            del op
            torch.cuda.empty_cache()

    result = None
    if rank == 0:
        K = args.steps
        peaks = measured_peaks()
        tag = "of measured" if peaks["source"] == "measured" else "of fallback"
        p_avg_s = p_ms / K / 1e3
        d_avg_s = d_ms / K / 1e3
        p_tflops_launch = p_flops / p_avg_s / 1e12
        d_gbs_launch = kv_bytes / d_avg_s / 1e9
        result = {
            "metric": METRIC,
            "value": sharding.job_throughput(p_flops, world, K, p_ms) / 1e12,
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": (p_ms + d_ms) / K,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": config_block(pcfg, world),
            "roofline": {"bound": "tensor", "achieved": p_tflops_launch, "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": p_tflops_launch / peaks["bf16_tflops"],
                         "traffic": recorded_traffic("prefill_fwd_kernel", "prefill_sm100.cu"),
                         "peak_source": f"bf16_tflops (burst) {tag}",
                         "kernel": "prefill_fwd_kernel<128>", "flops_per_launch": p_flops},
            "e2e": {"value": sharding.job_throughput(p_flops, world, K, e2e_ms) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "schedule": "per step: Q, K, V in from pinned host memory, prefill, O and LSE out; "
                                "consecutive steps overlap on copy-in, compute and copy-out streams"},
            "gpu_launches": 2 * K,
            "gpu_launches_note": "timed step region: one prefill and one decode kernel per step; the end-to-end "
                                 "legs launch 2 * steps more and the configuration sweep config_steps per entry",
            "clocks": clk.summary(),
            "clocks_configs": clk_cfg.summary(),
            "decode": {
                "metric": "paged-decode KV GB/s", "value": sharding.job_throughput(kv_bytes, world, K, d_ms) / 1e9,
                "unit": "GB/s", "workload": dcfg["name"], "kv_bytes_per_step": kv_bytes, "ms_per_step": d_ms / K,
                "l2": (FLUSH_NOTE["clean"] if decode_flush else
                       f"inputs larger than L2 ({kv_bytes / 1e6:.0f} MB of K/V per launch): timed without a flush"),
                "roofline": {"bound": "hbm", "achieved": d_gbs_launch, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": d_gbs_launch / peaks["hbm_gbs"],
                             "traffic": recorded_traffic("decode_split_kernel", "decode_sm100.cu", kv_bytes),
                             "peak_source": f"hbm_gbs {tag}",
                             "kernel": "decode_split_kernel<128> (split-KV with the merge in the same launch)"},
                "e2e": {"value": sharding.job_throughput(kv_bytes, world, K, de2e_ms) / 1e9, "unit": "GB/s",
                        "h2d_bytes_per_step": dh2d, "d2h_bytes_per_step": dd2h,
                        "schedule": "per step: new query tokens, block table and context lengths in from pinned "
                                    "host memory, decode against the HBM-resident cache, O and LSE out"},
            },
            "region_ms": region_ms,
        }
        result["configs"] = configs
        if world == 1 and not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(xp, pcfg, args.cpu_seconds)
            # the oracle on a bounded sample of each configuration as well
            for c in configs:
                if c["workload"] in cfg_host:
                    op_name, cfg, host = cfg_host[c["workload"]]
                    c["cpu_baseline"] = dict(oracle_config_rate(op_name, cfg, host, args.cpu_seconds_per_config),
                                             kind="oracle", cores=oracle_threads())
                    c["gpu_over_cpu"] = c["value"] / c["cpu_baseline"]["value"]
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if result is not None:
        print(json.dumps(result), flush=True)
    return 0


# The configurations timed beside the headline step: long-context prefill
# (causal and sliding window, N = 32,768), the GQA dial of prefill (B = 2,
# N = 8,192) and of single-sequence decode (131,072 cached tokens).
CONFIG_SWEEP = (("prefill", "long_causal_n32768"), ("prefill", "long_window4096_n32768"),
                ("prefill", "gqa_dial_prefill_mha"), ("prefill", "gqa_dial_prefill_gqa8"),
                ("prefill", "gqa_dial_prefill_mqa"), ("decode", "gqa_dial_decode_mha"),
                ("decode", "gqa_dial_decode_gqa8"), ("decode", "gqa_dial_decode_mqa"))

LAUNCHES_PER_CALL = {"prefill": 1, "prefill_paged": 1, "prefill_backward": 3, "mla_decode": 2, "decode": 1,
                     "decode_window": 1}


def setup_op(op, name, dev, seed, peaks, keep_host=False):
    """Inputs on the device and a launch() closure for one entry point on one
    named workload, with its algorithmic work per launch and its roofline.

    prefill (TFLOP/s, tensor roofline), prefill_paged (TFLOP/s over the visible
    pairs of each chunk against its context), decode (KV GB/s, HBM roofline),
    decode_window (GB/s of the K/V bytes of the visible tokens only), mla_decode
    (GB/s of the latent cache, with its tensor-core rate reported beside it),
    prefill_backward (TFLOP/s counting 5 products per visible pair).
    """
    import exact_softmax_attention_causal_b200 as attn

    extra = {}
    if op == "prefill":
        cfg = workloads.PREFILL_WORKLOADS[name]
        x = workloads.prefill_inputs(cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["N"], cfg["d"], seed)
        q, k, v = x.q.to(dev), x.k.to(dev), x.v.to(dev)
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
        work = accounting.prefill_flops(cfg["B"], cfg["Hq"], cfg["N"], cfg["d"], cfg["mask"], cfg["window"])

        def launch():
            attn.prefill(q, k, v, mask=cfg["mask"], window=cfg["window"], out=o, lse=lse)
        unit, bound, peak, scale_div = "TFLOP/s", "tensor", peaks["bf16_tflops"], 1e12
        metric = "prefill TFLOP/s (visible pairs)"
        kernel = f"prefill_fwd_kernel<{cfg['d']}>"
    elif op == "prefill_paged":
        cfg = dict(workloads.PAGED_PREFILL_WORKLOADS[name])
        c = dict(cfg)
        mask, window = c.pop("mask"), c.pop("window")
        B, Hq, Hkv, Nq, d = (c.pop(kk) for kk in ("B", "Hq", "Hkv", "Nq", "d"))
        x = workloads.paged_prefill_inputs(B, Hq, Hkv, Nq, d, seed=seed, **c)
        q, kc, vc = x.q.to(dev), x.k_cache.to(dev), x.v_cache.to(dev)
        bt, sl = x.block_table.to(dev), x.seq_lens.to(dev)
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
        work = accounting.prefill_paged_flops(x.seq_lens.tolist(), Nq, Hq, d, mask, window)
        msl = x.max_seq_len

        def launch():
            attn.prefill_paged(q, kc, vc, bt, sl, msl, mask=mask, window=window, out=o, lse=lse)
        unit, bound, peak, scale_div = "TFLOP/s", "tensor", peaks["bf16_tflops"], 1e12
        metric = "chunked prefill TFLOP/s (visible pairs)"
        kernel = f"prefill_fwd_kernel<{d}, paged>"
    elif op == "decode_window":
        cfg = dict(workloads.WINDOW_DECODE_WORKLOADS[name])
        x = workloads.paged_decode_inputs(cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["d"], len_range=cfg.get("len_range"),
                                          seq_lens=cfg.get("seq_lens"), block_size=cfg["block_size"], seed=seed,
                                          learned_sinks=cfg["learned_sinks"])
        q, kc, vc = x.q.to(dev), x.k_cache.to(dev), x.v_cache.to(dev)
        bt, sl = x.block_table.to(dev), x.seq_lens.to(dev)
        sinks = None if x.sinks is None else x.sinks.to(dev)
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
        win, n_sink = cfg["window"], cfg["n_sink"]
        ws = torch.empty(attn.decode_window_workspace_bytes(cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["d"], x.max_seq_len,
                                                            x.block_size, win, n_sink), dtype=torch.uint8, device=dev)
        work = accounting.decode_window_kv_bytes(x.seq_lens.tolist(), cfg["Hkv"], cfg["d"], win, n_sink)
        msl = x.max_seq_len

        def launch():
            attn.decode_paged_window(q, kc, vc, bt, sl, msl, window=win, n_sink=n_sink, sinks=sinks, out=o, lse=lse,
                                     workspace=ws)
        unit, bound, peak, scale_div = "GB/s", "hbm", peaks["hbm_gbs"], 1e9
        metric = "windowed paged-decode KV GB/s (visible tokens)"
        kernel = f"decode_split_kernel<{cfg['d']}>"
    elif op == "prefill_backward":
        cfg = workloads.PREFILL_WORKLOADS[name]
        x = workloads.prefill_inputs(cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["N"], cfg["d"], seed)
        q, k, v = x.q.to(dev), x.k.to(dev), x.v.to(dev)
        gen = torch.Generator("cpu").manual_seed(10_000 + seed)
        d_o = torch.randn(q.shape, generator=gen, dtype=torch.float32).to(torch.bfloat16).to(dev)
        o, lse = attn.prefill(q, k, v, mask=cfg["mask"], window=cfg["window"])
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(attn.prefill_backward_workspace_bytes(cfg["B"], cfg["Hq"], cfg["N"]), dtype=torch.uint8,
                         device=dev)
        work = accounting.prefill_backward_flops(cfg["B"], cfg["Hq"], cfg["N"], cfg["d"], cfg["mask"], cfg["window"])

        def launch():
            attn.prefill_backward(q, k, v, o, lse, d_o, mask=cfg["mask"], window=cfg["window"], dq=dq, dk=dk, dv=dv,
                                  workspace=ws)
        unit, bound, peak, scale_div = "TFLOP/s", "tensor", peaks["bf16_tflops"], 1e12
        metric = "attention backward TFLOP/s (5 products per visible pair)"
        kernel = f"bwd_rowdot_kernel + bwd_dkdv_kernel<{cfg['d']}> + bwd_dq_kernel<{cfg['d']}>"
    elif op == "mla_decode":
        cfg = dict(workloads.MLA_DECODE_WORKLOADS[name])
        x = workloads.mla_decode_inputs(cfg["B"], cfg["H"], cfg["d_latent"], cfg["d_rope"], len_range=cfg["len_range"],
                                        block_size=cfg["block_size"], seed=seed)
        q, cache, bt, sl = x.q.to(dev), x.cache.to(dev), x.block_table.to(dev), x.seq_lens.to(dev)
        o = torch.empty((cfg["B"], cfg["H"], cfg["d_latent"]), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((cfg["B"], cfg["H"]), dtype=torch.float32, device=dev)
        ws = torch.empty(attn.mla_decode_workspace_bytes(cfg["B"], cfg["H"], x.max_seq_len), dtype=torch.uint8,
                         device=dev)
        work = accounting.mla_decode_bytes(x.seq_lens.tolist(), cfg["d_latent"], cfg["d_rope"])
        extra["mla_flops"] = accounting.mla_decode_flops(x.seq_lens.tolist(), cfg["H"], cfg["d_latent"],
                                                         cfg["d_rope"])
        msl = x.max_seq_len
        mla_scale = 1.0 / math.sqrt(cfg["d_head"] + cfg["d_rope"])

        def launch():
            attn.mla_decode_paged(q, cache, bt, sl, msl, mla_scale, out=o, lse=lse, workspace=ws)
        unit, bound, peak, scale_div = "GB/s", "hbm", peaks["hbm_gbs"], 1e9
        metric = "absorbed MLA decode latent-cache GB/s"
        kernel = "mla_split_kernel + decode_merge_kernel<512>"
    elif op == "decode":
        cfg = dict(workloads.DECODE_WORKLOADS[name])
        x = workloads.paged_decode_inputs(cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["d"], len_range=cfg.get("len_range"),
                                          seq_lens=cfg.get("seq_lens"), block_size=cfg["block_size"], seed=seed)
        q, kc, vc = x.q.to(dev), x.k_cache.to(dev), x.v_cache.to(dev)
        bt, sl = x.block_table.to(dev), x.seq_lens.to(dev)
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
        ws = torch.empty(attn.decode_workspace_bytes(cfg["B"], cfg["Hq"], cfg["Hkv"], cfg["d"], x.max_seq_len,
                                                     x.block_size), dtype=torch.uint8, device=dev)
        work = accounting.decode_kv_bytes(x.seq_lens.tolist(), cfg["Hkv"], cfg["d"])
        msl = x.max_seq_len

        def launch():
            attn.decode_paged(q, kc, vc, bt, sl, msl, out=o, lse=lse, workspace=ws)
        unit, bound, peak, scale_div = "GB/s", "hbm", peaks["hbm_gbs"], 1e9
        metric = "paged-decode KV GB/s"
        kernel = f"decode_split_kernel<{cfg['d']}>"
    else:
        raise ValueError(op)
    if keep_host:
        extra["host"] = x
    del x
    # HBM-bound entry points stream `work` bytes; prefill-type launches are always flushed
    kind = "write" if bound == "tensor" else ("clean" if needs_flush(work, dev) else None)
    l2 = (FLUSH_NOTE[kind] if kind else
          f"inputs larger than L2 ({work / 1e6:.0f} MB streamed per launch, more than twice the L2 size): "
          "timed without a flush")
    return dict(launch=launch, work=work, unit=unit, bound=bound, peak=peak, scale_div=scale_div, metric=metric,
                cfg=cfg, kernel=kernel, extra=extra, flush=kind, l2=l2)


def needs_flush(stream_bytes, dev):
    """An HBM-bound launch that streams more than twice the L2 capacity starts
    cold anyway (a streamed working set that large leaves nothing reusable in
    L2), so it is timed without a flush; anything smaller is flushed."""
    return stream_bytes < 2 * torch.cuda.get_device_properties(dev).L2_cache_size


FLUSH_NOTE = {
    "write": "flushed (256 MiB write) before every timed launch",
    "clean": "flushed (256 MiB write, then a 256 MiB read of another buffer: no dirty line left) before every "
             "timed launch",
}


class L2Flush:
    """Evicts the workload from L2 between timed launches. "write": fill a
    256 MiB buffer. "clean": the same write, then a read of another 256 MiB
    buffer, so that L2 ends up holding clean lines only and the timed kernel
    pays for no write-back of the flush's own lines."""

    def __init__(self, dev):
        self.wbuf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.rbuf = torch.ones(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
        self.acc = torch.empty((), dtype=torch.int64, device=dev)

    def __call__(self, kind):
        if kind is None:
            return
        self.wbuf.fill_(1)
        if kind == "clean":
            torch.sum(self.rbuf, dim=0, out=self.acc)


def time_launches(launch, steps, warmup, flush, dist_on=False, kind="write"):
    """CUDA-event time (ms, summed over `steps`) of launch(), each launch
    preceded by an L2 flush of the given kind (None: no flush) outside the
    events."""
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for _ in range(warmup):
        flush(kind)
        launch()
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    for e0, e1 in events:
        flush(kind)
        e0.record()
        launch()
        e1.record()
    torch.cuda.synchronize()
    return sum(e0.elapsed_time(e1) for e0, e1 in events)


def run_single_op(args):
    """Time one entry point on one named workload; one JSON line with its roofline.
    L2 is flushed before every timed launch; CUDA events on the launching stream.
    """
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    seed = sharding.rank_seed(args.seed, rank)
    peaks = measured_peaks()
    tag = "of measured" if peaks["source"] == "measured" else "of fallback"
    name = args.workload
    op = setup_op(args.op, name, dev, seed, peaks)
    flush = L2Flush(dev)
    with ClockSampler(local) as clk:
        ms = time_launches(op["launch"], args.steps, args.warmup, flush, dist_on=world > 1, kind=op["flush"])
    (ms_max,) = sharding.max_over_ranks([ms], device=dev)
    achieved = op["work"] / (ms / args.steps / 1e3) / op["scale_div"]
    if rank == 0:
        line = {
            "metric": op["metric"],
            "value": sharding.job_throughput(op["work"], world, args.steps, ms_max) / op["scale_div"],
            "unit": op["unit"], "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic", "op": args.op,
            "config": dict(workload=name, **{kk: vv for kk, vv in op["cfg"].items()},
                           l2=op["l2"]),
            "roofline": {"bound": op["bound"], "achieved": achieved, "peak": op["peak"], "unit": op["unit"],
                         "frac": achieved / op["peak"], "traffic": None, "peak_source": tag,
                         "kernel": op["kernel"]},
            "work_per_launch": op["work"],
            "gpu_launches": args.steps * LAUNCHES_PER_CALL[args.op],
            "clocks": clk.summary(),
        }
        if args.op == "mla_decode":  # the same launches against the tensor roofline, for context
            tf = op["extra"]["mla_flops"] / (ms / args.steps / 1e3) / 1e12
            line["tensor_context"] = {"achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                      "frac": tf / peaks["bf16_tflops"],
                                      "flops_per_launch": op["extra"]["mla_flops"]}
        print(json.dumps(line), flush=True)
    return 0


def dcfg_max_len(dcfg):
    if dcfg.get("len_range") is not None:
        return int(dcfg["len_range"][1])
    return int(max(dcfg["seq_lens"]))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--op", choices=["step", "prefill", "prefill_paged", "decode", "decode_window", "mla_decode",
                                     "prefill_backward"],
                    default="step",
                    help="step: the full hot-path step (default); otherwise time one entry point on --workload")
    ap.add_argument("--workload", default=None,
                    choices=sorted(list(workloads.PREFILL_WORKLOADS) + list(workloads.PAGED_PREFILL_WORKLOADS) +
                                   list(workloads.DECODE_WORKLOADS) + list(workloads.WINDOW_DECODE_WORKLOADS) +
                                   list(workloads.MLA_DECODE_WORKLOADS)))
    ap.add_argument("--decode-workload", default="paged_decode_b64", choices=sorted(workloads.DECODE_WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--reference-heads", type=int, default=2, help="oracle (batch, head) slices per step")
    ap.add_argument("--config-steps", type=int, default=20, help="timed launches per configuration of the sweep")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-configuration sweep")
    ap.add_argument("--cpu-seconds-per-config", type=float, default=3.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.op != "step":
        defaults = {"prefill": "llama3_8b_causal_gqa", "prefill_paged": "chunked_prefill_b4_q512",
                    "decode": "paged_decode_b64", "decode_window": "gptoss_window128_sinks_b64",
                    "mla_decode": "deepseek_v2_mla_b64", "prefill_backward": "llama3_8b_causal_gqa"}
        args.workload = args.workload or defaults[args.op]
        table = {"prefill": workloads.PREFILL_WORKLOADS, "prefill_paged": workloads.PAGED_PREFILL_WORKLOADS,
                 "decode": workloads.DECODE_WORKLOADS, "decode_window": workloads.WINDOW_DECODE_WORKLOADS,
                 "mla_decode": workloads.MLA_DECODE_WORKLOADS,
                 "prefill_backward": workloads.PREFILL_WORKLOADS}[args.op]
        if args.workload not in table:
            ap.error(f"--workload {args.workload} is not a {args.op} workload")
        if args.impl == "reference":
            ap.error("--op is only for the CUDA path")
        world, _, _ = dist_env()
        if world > 1:
            import torch.distributed as dist

            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                    device_id=torch.device("cuda", dist_env()[2]))
            try:
                return run_single_op(args)
            finally:
                dist.destroy_process_group()
        return run_single_op(args)
    args.workload = args.workload or "llama3_8b_causal_gqa"
    if args.workload not in workloads.PREFILL_WORKLOADS:
        ap.error("the full step takes a prefill workload")
    pcfg = dict(workloads.PREFILL_WORKLOADS[args.workload], name=args.workload)
    dcfg = dict(workloads.DECODE_WORKLOADS[args.decode_workload], name=args.decode_workload)
    world, _, _ = dist_env()
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.impl == "reference":
        return run_reference(args, pcfg)
    return run_ours(args, pcfg, dcfg)


if __name__ == "__main__":
    sys.exit(main())
