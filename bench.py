"""Throughput of the VideoMLA latent-KV attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 1]

One step = one chunk of an autoregressive rollout through the whole path, on one batch of
synthetic Wan2.1-1.3B-shaped input (the 6-frame window full, a 3-frame chunk of 4680 queries):
the down-projections of the chunk (query latent and chunk latents in one pass over x, whose
epilogue also writes the rotated positional keys of the ring and the chunk), attention over the
ring plus the chunk with the absorbed query heads (and their 3D-RoPE) formed inside the
attention kernel and the W_UV up-projection fused, and the ring append: three kernels.
(--unfused-query runs the query heads as their own GEMM and the key rotation as its own pass.)  Steps
advance the rollout (chunk 2, 3, 4, ... of a 6-frame window), so every step has the same work.

Timing: W untimed warm-up steps, then K steps between a barrier + device synchronisation on
both sides.  Each step's three kernels are captured beforehand as one CUDA graph per chunk
(rollout.ChunkGraph) and replayed, so the device runs them back to back.  L2 is flushed before
every step (a 256 MiB device memset, outside the per-step CUDA-event intervals).  Device time
per step = sum of per-step event intervals on the launch stream; the job time is the max over
ranks.  With N > 1 every rank runs its own independent
sample (weak scaling: no data-path collective exists on this path).

value      attention algorithmic TFLOP/s of the whole step: 2*(D + d_c) = 832 flop per
           (query row, attended key, head), divided by the whole-step device time
e2e        the same metric through the public API with host buffers: pinned host -> device copy
           of the step's tokens and device -> host copy of its output inside the timed interval,
           copies pipelined with the compute; independent rollouts served in turn, their rings
           together larger than L2 (each chunk's ring is cold without a flush in the interval;
           `flushed_value`: one rollout with the L2 flush inside the interval)
roofline   the attention call (the tensor-core kernel alone), timed with CUDA
           events recorded inside each step's graph around that call, against the measured
           bf16 peak
cpu_baseline  the float64 CPU oracle on a bounded sample of the same chunk (rank 0, N = 1)
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

METRIC = "MLA attention TFLOP/s & query tokens/s (Wan-1.3B shape), % of B200 BF16 peak"
REF_BUDGET_S = 90.0     # target wall time of a whole --impl reference run
CPU_BASELINE_S = 12.0   # CPU work of the cpu_baseline sample on the main line
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# --------------------------------------------------------------------------- clocks

REASON_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


class ClockSampler:
    """nvidia-smi sampled every 10 ms around the timed region.  The SM clock reported is the
    median over the samples stamped inside the timed region (begin() .. end(); by default the
    with-block), since the B200 lowers its clock under a sustained tensor load (power cap) and
    idle samples would hide that.  When no sample falls inside (a region shorter than the
    sampling interval), samples with GPU utilisation >= 50 % are used, then all samples.
    Two pollers run: one with nvidia-smi's timestamp field and one without it, so that a
    nvidia-smi that refuses the first query still leaves the unstamped samples."""

    FIELDS = "clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,utilization.gpu"

    def __init__(self, index: int):
        self.index = index
        self.procs = []
        self.lines = {"stamped": [], "plain": []}
        self.t_begin = None
        self.t_end = None

    def __enter__(self):
        for kind, query in (("stamped", "timestamp," + self.FIELDS), ("plain", self.FIELDS)):
            try:
                proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + query,
                     "--format=csv,noheader,nounits", "-lms", "10"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except (OSError, FileNotFoundError):
                continue
            thread = threading.Thread(target=self._read, args=(proc, self.lines[kind]),
                                      daemon=True)
            thread.start()
            self.procs.append((proc, thread))
        self.t_begin = time.time()
        return self

    def begin(self):
        self.t_begin = time.time()

    def end(self):
        self.t_end = time.time()

    @staticmethod
    def _read(proc, out):
        for line in proc.stdout:
            out.append(line.strip())

    def __exit__(self, *exc):
        if self.t_end is None:
            self.t_end = time.time()
        for proc, thread in self.procs:
            proc.terminate()
            try:
                proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                proc.kill()
            thread.join(timeout=2)

    @staticmethod
    def _stamp(text: str):
        """nvidia-smi's local-time stamp ("2026/12/02 17:05:01.123") as seconds since the epoch."""
        import datetime
        try:
            return datetime.datetime.strptime(text, "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    @staticmethod
    def _parse(lines, stamped: bool):
        rows = []
        for ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            ts = None
            if stamped:
                if len(parts) < 6:
                    continue
                ts = ClockSampler._stamp(parts[0])
                parts = parts[1:]
            if len(parts) < 5:
                continue
            try:
                s, m, pw = float(parts[0]), float(parts[1]), float(parts[2])
                bits = int(parts[3], 16) if parts[3].startswith("0x") else int(parts[3])
                util = float(parts[4])
            except ValueError:
                continue
            rows.append((ts, s, m, pw, bits, util))
        return rows

    def summary(self):
        rows = self._parse(self.lines["stamped"], True) or self._parse(self.lines["plain"], False)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        inside = []
        if self.t_begin is not None and self.t_end is not None:
            inside = [r for r in rows if r[0] is not None and self.t_begin <= r[0] <= self.t_end]
        loaded = [r for r in rows if r[5] >= 50.0]
        use = inside or loaded or rows
        reasons = set()
        for r in use:
            for bit, name in REASON_BITS.items():
                if r[4] & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[1] for r in use),
                "sm_max_mhz": max(r[2] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows), "samples_in_timed_region": len(inside),
                "samples_under_load": len(loaded),
                "from": "timed region" if inside else "utilisation >= 50 %" if loaded else "all samples",
                "power_w_max": max(r[3] for r in rows)}


# --------------------------------------------------------------------------- CPU oracle

class OracleSample:
    """The float64 oracle on sampled query rows of the measured chunk (window full).  Inputs and
    the window are prepared once; each call times one evaluation."""

    def __init__(self, cfg):
        import oracle
        from mla_latent_kv_attn_b200 import inputs
        self.cfg, self.oracle, self.inputs = cfg, oracle, inputs
        self.d = oracle.dims_from(cfg)
        self.lw = inputs.layer_weights(cfg)
        self.win = oracle.SlidingWindow(self.d)
        for ch in range(cfg.measured_chunk):
            x = inputs.chunk_x(cfg, ch)[0]
            c, k = oracle.down_project(x, self.lw.w_dkv, self.lw.w_kr)
            self.win.append_chunk(cfg.first_frame(ch), c, k)
        self.x = inputs.chunk_x(cfg, cfg.measured_chunk)[0]

    def __call__(self, rows: int, seed_tag: int = 7):
        cfg = self.cfg
        sel = self.inputs.sample_rows(cfg.n_q, rows, tag=seed_tag)
        t0 = time.perf_counter()
        self.oracle.chunk_step(self.d, self.lw, self.x, self.win,
                               cfg.first_frame(cfg.measured_chunk), rows=sel, append=False)
        dt = time.perf_counter() - t0
        flops = 2.0 * (cfg.d_latent + cfg.d_c) * len(sel) * \
            cfg.keys_per_query(cfg.measured_chunk) * cfg.n_heads
        return flops, dt, len(sel)


class OracleRows:
    """The oracle's work per sampled query row of the measured chunk, with the chunk's keys built
    once: the steps of oracle.chunk_step, in its order, split in two.  The setup (the chunk's
    down-projection, the window's and chunk's per-head keys and values, the rotated positional
    keys) is timed once (`setup_s`); each call times the rows' query latent, query heads, their
    rotation and the attention over all keys.  Setup plus the calls is what one chunk_step call
    over all those rows costs."""

    def __init__(self, sample: OracleSample):
        o, cfg, lw = sample.oracle, sample.cfg, sample.lw
        self.sample, self.o, self.cfg, self.lw, self.d = sample, o, cfg, lw, sample.d
        first = cfg.first_frame(cfg.measured_chunk)
        t0 = time.perf_counter()
        c_kv, k_r = o.down_project(sample.x, lw.w_dkv, lw.w_kr)
        self.pos_chunk = o.token_positions(range(first, first + cfg.chunk_frames), self.d)
        c_win, k_win, pos_win = sample.win.keys()
        self.c_all = np.concatenate([c_win, c_kv])
        k_r_all = np.concatenate([k_win, k_r])
        pos_all = np.concatenate([pos_win, self.pos_chunk])
        self.k_nope, self.v = o.key_value_heads(self.c_all, lw.w_uk, lw.w_uv)
        self.k_rope = o.rope3d(k_r_all, pos_all, self.d)
        self.setup_s = time.perf_counter() - t0

    def evaluate(self, sel):
        """The rows' part of chunk_step for the query rows `sel`: their attention results."""
        o, lw, d = self.o, self.lw, self.d
        c_q = o.query_latent(self.sample.x[sel], lw.w_dq)
        q_nope, q_r = o.query_heads(c_q, lw.w_uq, lw.w_qr)
        q_rope = o.rope3d(q_r, self.pos_chunk[sel], d)
        return o.attend(q_nope, q_rope, self.k_nope, self.k_rope, self.v, d.softmax_scale,
                        c_keys=self.c_all)

    def __call__(self, rows: int, seed_tag: int = 7):
        cfg = self.cfg
        sel = self.sample.inputs.sample_rows(cfg.n_q, rows, tag=seed_tag)
        t0 = time.perf_counter()
        self.evaluate(sel)
        dt = time.perf_counter() - t0
        flops = 2.0 * (cfg.d_latent + cfg.d_c) * len(sel) * \
            cfg.keys_per_query(cfg.measured_chunk) * cfg.n_heads
        return flops, dt, len(sel)


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


def run_reference(args, cfg):
    """--impl reference: the CPU oracle as it stands, each step a bounded row sample of the
    measured chunk.  The chunk's keys are built once (OracleRows: the setup that a chunk_step
    call over all the steps' rows would do once), and its time counts in full in the total; each
    step then evaluates its rows.  The rows per step are sized from a calibration sample so that
    the whole --warmup + --steps run takes about REF_BUDGET_S seconds (at most --ref-rows rows,
    at least 1)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    sample = OracleSample(cfg)
    prep = OracleRows(sample)
    f, dt, n = prep(16, seed_tag=99)                 # calibration (not counted)
    per_row = dt / max(n, 1)
    rows = int(max(REF_BUDGET_S - prep.setup_s, 1.0) / max(args.warmup + args.steps, 1) /
               max(per_row, 1e-6))
    rows = max(1, min(args.ref_rows, rows))
    times, flops = [], 0.0
    for i in range(args.warmup + args.steps):
        f, dt, n = prep(rows, seed_tag=100 + i)
        if i >= args.warmup:
            times.append(dt)
            flops += f
    total = prep.setup_s + sum(times)
    value = flops / total / 1e12
    tok = rows * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "batch": cfg.batch, "n_q": cfg.n_q,
                   "keys_per_query": cfg.keys_per_query(cfg.measured_chunk),
                   "sample": f"{rows} query rows x all heads per step; the chunk's keys "
                             f"built once ({prep.setup_s:.1f} s, counted in the total)"},
        "query_tokens_per_s": tok,
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(),
                         "kind": "oracle",
                         "sample": f"{rows} sampled query rows of one chunk per step, the "
                                   f"chunk's keys built once"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- ranks

def rank_samples(rank: int, batch: int) -> range:
    """Sample indices a rank draws: every rank runs its own, disjoint samples."""
    return range(rank * batch, (rank + 1) * batch)


def max_over_ranks(value: float, device=None) -> float:
    """The largest value over all ranks (the local value without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------- GPU path

def probe_sm_clock(stream, spin_us: int = 200):
    """Launches the library's clock probe (one warp per SM reads the SM cycle counter against
    the global timer while spinning spin_us) on `stream`; returns a function that, after the
    stream has run it, gives the median SM clock in MHz over the SMs."""
    import torch
    from mla_latent_kv_attn_b200 import _lib
    n = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    out = torch.zeros((n, 4), dtype=torch.int64, device="cuda")
    st = _lib.lib().mla_probe_sm_clock(out.data_ptr(), n, spin_us, stream.cuda_stream)
    if st != 0:
        raise RuntimeError("mla_probe_sm_clock: " + _lib.last_error())

    def result():
        v = out.cpu().numpy().astype(np.float64)
        mhz = 1000.0 * v[:, 1] / np.maximum(v[:, 2], 1.0)
        return float(np.median(mhz))
    return result


def time_calls(fn, flush, stream, reps: int):
    """Mean device time (ms) of fn() over reps launches, each after an L2 flush that lies
    outside its CUDA-event interval."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    for _ in range(3):
        flush.zero_()
        fn()
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in ev)


def bandwidth_entry(nbytes: float, ms: float, hbm_gbs: float, workload: str, **extra):
    gbs = nbytes / (ms * 1e-3) / 1e9
    d = {"bytes": int(nbytes), "us": 1e3 * ms, "gbs": gbs, "frac": gbs / hbm_gbs,
         "workload": workload}
    d.update(extra)
    return d


def measure_bandwidth(cfg, flush, stream, hbm_gbs: float, reps: int = 20):
    """The memory-bound calls of the path, each timed alone with CUDA events (L2 flushed before
    every launch), at the benchmark workload and at a batch whose arrays exceed the 126 MB L2:
    achieved GB/s = the call's algorithmic bytes / its time, against the measured HBM copy
    bandwidth.  Algorithmic bytes: ring append 2 * D * sizeof(T) per chunk token (read the chunk
    latent, write the ring row); ring-key rotation 2 * d_rope * sizeof(T) per ring key (read k_R,
    write the rotated key); query RoPE 2 * d_rope * sizeof(T) per (token, head); KV
    down-projection x + [W_down^KV; W_R^K] read, [c_KV || k_R] written once; the step's
    x-projection x + w_x read, [c_Q || c_KV || k_R] written once, and with the rotated keys also
    k_R of every ring key read and the rotated key of every ring and chunk key written."""
    import torch
    from mla_latent_kv_attn_b200 import api, rollout
    res = {}
    for tag, batch in (("bench", cfg.batch), ("large", 32)):
        c = api.make_config(cfg, batch=batch)
        dt = api.torch_dtype(c)
        es = 2 if dt == torch.bfloat16 else 4
        tpf, n_q, D = cfg.tokens_per_frame, cfg.n_q, cfg.d_latent
        W = cfg.window_frames
        ring = rollout.Ring(c)
        lat = torch.randn((batch, n_q, D), device="cuda").to(dt)
        first = W * 4            # a chunk whose frames wrap into a full ring
        for ch in range(W // cfg.chunk_frames):
            api.mla_cache_append(c, None, None, lat, ring.cache, ring.slot_frame,
                                 ch * cfg.chunk_frames, api.MLA_APPEND)
        wl = f"{cfg.name}, batch {batch}"
        ms = time_calls(lambda: api.mla_cache_append(c, None, None, lat, ring.cache,
                                                     ring.slot_frame, first, api.MLA_APPEND),
                        flush, stream, reps)
        res[f"ring_append_{tag}"] = bandwidth_entry(2.0 * batch * n_q * D * es, ms, hbm_gbs, wl,
                                                    kernel="ring_append_kernel")
        ws = torch.empty(api.mla_attention_workspace_bytes(c, W), device="cuda", dtype=torch.uint8)
        ms = time_calls(lambda: api.mla_rotate_ring_keys(c, ring.cache, ring.slot_frame, W, ws),
                        flush, stream, reps)
        res[f"rope_ring_keys_{tag}"] = bandwidth_entry(2.0 * batch * W * tpf * cfg.d_rope * es, ms,
                                                       hbm_gbs, wl, kernel="rope_keys_vec_kernel")
        q = torch.randn((batch, n_q, cfg.n_heads, D), device="cuda").to(dt)
        q3 = q.view(batch, n_q, cfg.n_heads * D)
        ms = time_calls(lambda: api.mla_rope3d(c, q3, n_vec=cfg.n_heads, col_offset=cfg.d_c,
                                               vec_stride=D, first_frame=first),
                        flush, stream, reps)
        res[f"rope_query_{tag}"] = bandwidth_entry(2.0 * batch * n_q * cfg.n_heads * cfg.d_rope * es,
                                                   ms, hbm_gbs, wl, kernel="rope3d_kernel")
        if tag == "bench" or batch * n_q * cfg.d_model * es <= 2 ** 30:
            x = torch.randn((batch, n_q, cfg.d_model), device="cuda").to(dt)
            wkv = torch.randn((D, cfg.d_model), device="cuda").to(dt)
            ms = time_calls(lambda: api.mla_cache_append(c, x, wkv, lat, None, None, first,
                                                         api.MLA_PROJECT),
                            flush, stream, reps)
            nbytes = (batch * n_q * cfg.d_model + D * cfg.d_model + batch * n_q * D) * es
            flops = 2.0 * batch * n_q * cfg.d_model * D
            res[f"kv_down_projection_{tag}"] = bandwidth_entry(
                nbytes, ms, hbm_gbs, wl, kernel="gemm_tc_kernel", tflops=flops / (ms * 1e-3) / 1e12)
            # the step's x-projection (c_Q || chunk latents in one pass over x), without and with
            # the rotated keys of the ring and the chunk written from its epilogue
            wx = torch.randn((cfg.d_cq + D, cfg.d_model), device="cuda").to(dt)
            cq = torch.empty((batch, n_q, cfg.d_cq), device="cuda", dtype=dt)
            n_x = cfg.d_cq + D
            nbytes = (batch * n_q * cfg.d_model + n_x * cfg.d_model + batch * n_q * n_x) * es
            flops = 2.0 * batch * n_q * cfg.d_model * n_x
            ms = time_calls(lambda: api.mla_project_latents(c, x, wx, cq, lat), flush, stream, reps)
            res[f"x_projection_{tag}"] = bandwidth_entry(
                nbytes, ms, hbm_gbs, wl, kernel="gemm_tc_kernel", tflops=flops / (ms * 1e-3) / 1e12)
            ms = time_calls(lambda: api.mla_project_latents_rotated(
                c, x, wx, cq, lat, ring.cache, ring.slot_frame, W, first, ws), flush, stream, reps)
            nbytes += batch * (W * tpf * 2 + n_q) * cfg.d_rope * es
            res[f"x_projection_rotated_keys_{tag}"] = bandwidth_entry(
                nbytes, ms, hbm_gbs, wl, kernel="gemm_tc_kernel", tflops=flops / (ms * 1e-3) / 1e12)
            del x, wkv, wx, cq
        del ring, lat, ws, q, q3
        torch.cuda.empty_cache()
    return res



def run_ours(args, cfg):
    import torch
    import torch.distributed as dist
    from mla_latent_kv_attn_b200 import api, inputs, rollout

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    c = api.make_config(cfg, kernel_path=kernel_path(args))
    lw = inputs.layer_weights(cfg)
    w = rollout.upload_weights(c, lw, device=dev)
    ring = rollout.Ring(c, device=dev)
    buf = rollout.ChunkBuffers(c, device=dev)
    # independent sample per rank: inputs drawn with the rank as the sample index
    n_pool = 4
    samples = rank_samples(rank, cfg.batch)
    pool = [torch.from_numpy(inputs.chunk_x(cfg, cfg.measured_chunk + i, samples=samples))
            .to(device=dev, dtype=torch.bfloat16) for i in range(n_pool)]
    for ch in range(cfg.measured_chunk):
        buf.x.copy_(torch.from_numpy(inputs.chunk_x(cfg, ch, samples=samples)).to(torch.bfloat16))
        rollout.prefill_chunk(c, w, ring, buf, ch)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    # the query heads formed inside the attention kernel where the shape allows
    fused_q = rollout.fused_query_supported(c) and not args.unfused_query
    # fused: x GEMM (c_Q || chunk latents || rotated keys), attention (+W_UV), ring append;
    # otherwise x GEMM, Q' GEMM + RoPE, rotated-key pass, attention (+W_UV), ring append
    launches_per_step = 3 if fused_q else 5

    first_chunk = cfg.measured_chunk
    flops_step = cfg.attention_flops(first_chunk)   # same for every later chunk (window full)

    def step(i, ev=None, x=None):
        ch = first_chunk + i
        x = pool[i % n_pool] if x is None else x
        first, n_valid = rollout.chunk_schedule(cfg.chunk_frames, cfg.window_frames, ch)
        if fused_q:
            api.mla_project_latents_rotated(c, x, w.w_x, buf.c_q, buf.chunk_lat, ring.cache,
                                            ring.slot_frame, n_valid, first, buf.workspace,
                                            dev_status=buf.dev_status)
        else:
            api.mla_project_chunk(c, x, w.w_x, w.w_qcat, buf.c_q, buf.q, buf.chunk_lat, first)
        if ev is not None:
            ev[0].record(stream)
        if fused_q:
            api.mla_attention_fwd_from_cq(c, buf.c_q, w.w_qcat, buf.chunk_lat, ring.cache,
                                          ring.slot_frame, n_valid, first, w.w_uv, buf.o, buf.lse,
                                          buf.workspace, buf.dev_status, prerotated=True)
        else:
            api.mla_attention_fwd(c, buf.q, buf.chunk_lat, ring.cache, ring.slot_frame, n_valid,
                                  first, w.w_uv, buf.o, buf.lse, buf.workspace, buf.dev_status)
        if ev is not None:
            ev[1].record(stream)
        api.mla_cache_append(c, None, None, buf.chunk_lat, ring.cache, ring.slot_frame, first,
                             api.MLA_APPEND)

    # Each step is one CUDA graph (rollout.ChunkGraph): the chunk's kernels replay back to back
    # without per-launch host overhead, each kernel's set-up overlapping the previous kernel's
    # tail (programmatic launches).  Graphs are captured before the timed region (host set-up,
    # like encoding a plan); capturing launches nothing.  The per-call breakdown is measured
    # afterwards on graphs of further chunks with timing events between the calls (an event
    # between two kernels keeps the second from starting early, so the timed steps have none).
    graphs = [rollout.ChunkGraph(c, w, ring, buf, first_chunk + i, x=pool[i % n_pool],
                                 fused_q=fused_q)
              for i in range(args.warmup + args.steps)]
    # warm-up
    for i in range(args.warmup):
        flush.zero_()
        graphs[i].replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    # ---- device-timed region
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        time.sleep(0.25)
        clk.begin()
        for i in range(args.steps):
            flush.zero_()
            ev_s[i].record(stream)
            graphs[args.warmup + i].replay()
            ev_e[i].record(stream)
        # the SM clock read on the device right after the last timed step (nvidia-smi's samples
        # are 10 ms apart, longer than a short timed region)
        clock_after = probe_sm_clock(stream)
        torch.cuda.synchronize()
        clk.end()
        time.sleep(0.25)
    if world > 1:
        dist.barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(ev_s, ev_e)]
    sm_mhz_device = clock_after()
    total_ms = max_over_ranks(sum(step_ms), device=dev)
    status = int(buf.dev_status.item())
    if status != 0:
        raise RuntimeError(f"a kernel reported status {status}")
    base = args.warmup + args.steps

    # ---- the step's calls, timed by events recorded inside the step graphs (further chunks of
    # the same rollout, same work per chunk)
    bd_graphs = [rollout.ChunkGraph(c, w, ring, buf, first_chunk + base + i, x=pool[i % n_pool],
                                    events=True, fused_q=fused_q) for i in range(args.steps)]
    for g in bd_graphs:
        flush.zero_()
        g.replay()
    torch.cuda.synchronize()
    attn_ms = [g.attention_ms() for g in bd_graphs]
    proj_ms = [g.projection_ms() for g in bd_graphs]
    app_ms = [g.append_ms() for g in bd_graphs]
    base += args.steps
    del bd_graphs

    # ---- end to end through the public API with host buffers
    # Pinned host tokens in, pinned host output back, every copy inside the timed interval.
    # Pipelined (rollout.HostStreamer): chunk n's copy-in overlaps chunk n-1's compute and its
    # copy-out overlaps chunk n+1's compute; one interval from before the first copy-in to after
    # the last copy-out.  Two forms: (1) one rollout with the L2 flush before every chunk inside
    # the interval (`flushed_value`); (2) the headline: R independent rollouts served in turn,
    # their rings together larger than L2 (so each chunk finds its ring cold, with no flush
    # in the interval).  The serial variant (copy-in, compute, copy-out one after the other on
    # one stream; flushes outside its per-step intervals) is reported beside them.
    x_host = [p.cpu().pin_memory() for p in pool]
    o_host = [torch.empty(buf.o.shape, dtype=buf.o.dtype).pin_memory() for _ in range(2)]
    h2d = x_host[0].numel() * x_host[0].element_size()
    d2h = o_host[0].numel() * o_host[0].element_size()
    streamer = rollout.HostStreamer(c, w, ring, device=dev, compute_stream=stream)
    for i in range(args.warmup):          # warm the streamer's own buffers and streams
        flush.zero_()
        streamer.submit(first_chunk + base + i, x_host[i % n_pool], o_host[i % 2], fused_q=fused_q)
    streamer.finish()
    torch.cuda.synchronize()
    base += args.warmup
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e2e_a, e2e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_a.record(stream)
    streamer.begin(e2e_a)
    for i in range(args.steps):
        flush.zero_()
        streamer.submit(first_chunk + base + i, x_host[(base + i) % n_pool], o_host[i % 2],
                        fused_q=fused_q)
    streamer.finish()
    e2e_b.record(stream)
    torch.cuda.synchronize()
    streamer.check_device_status()
    e2e_flushed_ms = max_over_ranks(e2e_a.elapsed_time(e2e_b), device=dev)
    base += args.steps
    # R independent rollouts, each prefilled to the measured chunk's state (from the device input
    # pool: the values do not matter for timing), served in turn
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    ring_bytes = ring.cache.numel() * ring.cache.element_size()
    n_rings = max(2, -(-int(1.25 * l2_bytes) // ring_bytes))
    rings = [rollout.Ring(c, device=dev) for _ in range(n_rings)]
    pbuf = rollout.ChunkBuffers(c, device=dev)
    for r in rings:
        for ch in range(first_chunk):
            pbuf.x.copy_(pool[ch % n_pool])
            rollout.prefill_chunk(c, w, r, pbuf, ch)
    del pbuf
    next_chunk = [first_chunk] * n_rings
    def submit_rotating(i):
        r = i % n_rings
        streamer.submit(next_chunk[r], x_host[i % n_pool], o_host[i % 2], fused_q=fused_q,
                        ring=rings[r])
        next_chunk[r] += 1
    for i in range(args.warmup):
        submit_rotating(i)
    streamer.finish()
    flush.zero_()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e2e_a, e2e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_a.record(stream)
    streamer.begin(e2e_a)
    for i in range(args.steps):
        submit_rotating(args.warmup + i)
    streamer.finish()
    e2e_b.record(stream)
    torch.cuda.synchronize()
    streamer.check_device_status()
    e2e_ms = max_over_ranks(e2e_a.elapsed_time(e2e_b), device=dev)
    rings_mb = n_rings * ring_bytes / 1e6
    del rings
    # serial variant
    ser_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ser_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        ser_s[i].record(stream)
        buf.x.copy_(x_host[(base + i) % n_pool], non_blocking=True)
        step(base + i, x=buf.x)
        o_host[0].copy_(buf.o, non_blocking=True)
        ser_e[i].record(stream)
    torch.cuda.synchronize()
    ser_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(ser_s, ser_e)), device=dev)
    if world > 1:
        dist.barrier()

    peaks, peak_kind = load_peaks()
    bandwidth = measure_bandwidth(cfg, flush, stream, peaks["hbm_gbs"]) if not args.no_bandwidth \
        else None
    # the step's three calls, timed by events inside the step graphs (means over the timed steps)
    n_x = cfg.d_cq + cfg.d_latent
    # with the query heads formed inside the attention kernel the projection call is the
    # x-projection alone; otherwise it also runs the Q' GEMM
    proj_flops = 2.0 * cfg.batch * cfg.n_q * (
        cfg.d_model * n_x + (0 if fused_q else cfg.d_cq * cfg.n_heads * cfg.d_latent))
    app_bytes = 2.0 * cfg.batch * cfg.n_q * cfg.d_latent * 2
    step_breakdown = {
        "projections_us": 1e3 * statistics.mean(proj_ms),
        "projections_tflops": proj_flops / (statistics.mean(proj_ms) * 1e-3) / 1e12,
        "attention_call_us": 1e3 * statistics.mean(attn_ms),
        "append_us": 1e3 * statistics.mean(app_ms),
        "append_gbs": app_bytes / (statistics.mean(app_ms) * 1e-3) / 1e9,
        "step_us": 1e3 * statistics.mean(step_ms),
        "calls": ("mla_project_latents_rotated (x-projection GEMM, rotated keys from its "
                  "epilogue) | mla_attention_fwd_from_cq_prerotated (attention with the query "
                  "heads formed inside it) | mla_cache_append(MLA_APPEND)") if fused_q else
                 ("mla_project_chunk (x-projection GEMM, Q' GEMM + RoPE) | mla_attention_fwd "
                  "(rotated-key pre-pass + attention) | mla_cache_append(MLA_APPEND)")}
    n_units_all = world * cfg.batch
    ms_per_step = total_ms / args.steps
    value = world * flops_step * args.steps / (total_ms * 1e-3) / 1e12
    tok_s = world * cfg.batch * cfg.n_q * args.steps / (total_ms * 1e-3)
    attn_avg_ms = statistics.mean(attn_ms)
    achieved = flops_step / (attn_avg_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    traffic = None
    tr_path = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tr_path):
        tr = json.load(open(tr_path))
        # counters taken on this workload, from the kernel source as it is now
        if tr.get("kernel_sha") == kernel_sha() and tr.get("workload") == cfg.name:
            traffic = tr.get("bytes_per_launch")
    result = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": cfg.name, "batch": cfg.batch, "n_q": cfg.n_q,
                   "window_frames": cfg.window_frames, "chunk_frames": cfg.chunk_frames,
                   "keys_per_query": cfg.keys_per_query(first_chunk), "heads": cfg.n_heads,
                   "d_c": cfg.d_c, "d_rope": cfg.d_rope,
                   "parallelism": f"replicas x{world} (independent samples)",
                   "l2": "flushed before every step (256 MiB memset outside the event intervals)"},
        "query_tokens_per_s": tok_s,
        "pct_of_bf16_peak": 100.0 * value / peak,
        "attention_call_ms": attn_avg_ms,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": ("mla_attention_fwd_from_cq_prerotated (attention_tc_kernel)"
                                if fused_q else "mla_attention_fwd (rotated-key pre-pass + " +
                                ("attention_pair_kernel" if args.kernel_path == "pair"
                                 and cfg.n_heads % 2 == 0 and cfg.d_c in (128, 192)
                                 else "attention_tc_kernel") + ")"),
                     "peak_kind": f"{peak_kind} burst bf16",
                     "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"]},
        "e2e": {"value": world * flops_step * args.steps / (e2e_ms * 1e-3) / 1e12,
                "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms / args.steps,
                "mode": f"pipelined: copy-in of chunk n+1 and copy-out of chunk n-1 overlap "
                        f"chunk n (rollout.HostStreamer); one interval; {n_rings} independent "
                        f"rollouts served in turn, rings {rings_mb:.0f} MB in all (> L2), so "
                        f"each chunk's ring is cold; no flush inside the interval",
                "flushed_value": world * flops_step * args.steps / (e2e_flushed_ms * 1e-3) / 1e12,
                "flushed_mode": "one rollout, the 256 MiB L2 flush before every chunk inside the "
                                "interval",
                "serial_value": world * flops_step * args.steps / (ser_ms * 1e-3) / 1e12,
                "serial_ms_per_step": ser_ms / args.steps},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": dict(clk.summary(), sm_mhz_device=sm_mhz_device,
                       sm_mhz_device_method="mla_probe_sm_clock right after the last timed step: "
                                            "median over SMs of cycles / global-timer ns"),
        "step_breakdown": step_breakdown,
        "bandwidth": bandwidth,
    }
    result["roofline"]["sm_mhz"] = sm_mhz_device
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle on the same chunk: its keys built once (time counted), then batches of
        # --cpu-rows sampled rows until about CPU_BASELINE_S seconds of CPU work in all
        prep = OracleRows(OracleSample(cfg))
        flops, spent, rows, k = 0.0, prep.setup_s, 0, 0
        while spent < CPU_BASELINE_S or k == 0:
            f, dt, n = prep(args.cpu_rows, seed_tag=200 + k)
            flops, spent, rows, k = flops + f, spent + dt, rows + n, k + 1
        result["cpu_baseline"] = {"value": flops / spent / 1e12, "unit": "TFLOP/s",
                                  "cores": blas_threads(), "kind": "oracle",
                                  "sample": f"{rows} sampled query rows x {cfg.n_heads} heads of "
                                            f"one chunk in {k} batches, the chunk's keys built "
                                            f"once ({prep.setup_s:.1f} s); {spent:.1f} s in all"}
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_stack(args, cfg):
    """Workloads with a stack of layers and several denoising steps per chunk (the 30-layer
    preset): one step = one whole rollout (every chunk, step and layer), each chunk replayed as
    one CUDA graph (rollout.LayerStack.capture_chunk: ring keys rotated once per chunk and layer,
    cached-ring attention, appends after the last step).  value = algorithmic attention flops of
    the rollout / its device time.  Inputs: a pool of 8 seeded chunk inputs on the device,
    cycled over (step, layer); the stack's rings and weights (over 700 MB) exceed L2, which is
    also flushed before every rollout."""
    import torch
    import torch.distributed as dist
    from mla_latent_kv_attn_b200 import api, inputs, rollout

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    steps = args.steps if args.steps_given else 3
    c = api.make_config(cfg)
    stack = rollout.LayerStack(c, [rollout.upload_weights(c, inputs.layer_weights(cfg, l), device=dev)
                                   for l in range(cfg.n_layers)], device=dev)
    samples = rank_samples(rank, cfg.batch)
    pool = [torch.from_numpy(inputs.chunk_x(cfg, k, samples=samples)).to(device=dev,
                                                                          dtype=torch.bfloat16)
            for k in range(8)]
    x_of = lambda s, l: pool[(s * cfg.n_layers + l) % len(pool)]
    graphs = [stack.capture_chunk(ch, cfg.n_steps, x_of) for ch in range(cfg.n_chunks)]
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    flops = sum(cfg.attention_flops(ch) for ch in range(cfg.n_chunks)) * cfg.n_steps * cfg.n_layers
    calls = cfg.n_chunks * cfg.n_steps * cfg.n_layers
    for _ in range(args.warmup):
        flush.zero_()
        for g in graphs:
            g.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    with ClockSampler(local) as clk:
        for i in range(steps):
            flush.zero_()
            ev[i][0].record(stream)
            for g in graphs:
                g.replay()
            ev[i][1].record(stream)
        clock_after = probe_sm_clock(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), device=dev)
    rollout.check_device_status(stack.buf)
    peaks, peak_kind = load_peaks()
    value = world * flops * steps / (total_ms * 1e-3) / 1e12
    result = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": total_ms / steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": cfg.name, "batch": cfg.batch, "n_q": cfg.n_q, "layers": cfg.n_layers,
                   "denoising_steps": cfg.n_steps, "chunks": cfg.n_chunks,
                   "window_frames": cfg.window_frames, "chunk_frames": cfg.chunk_frames,
                   "attention_calls_per_step": calls,
                   "parallelism": f"replicas x{world} (independent samples)",
                   "l2": "inputs larger than L2 (30 layers' rings and weights), and flushed before "
                         "every rollout"},
        "query_tokens_per_s": world * cfg.batch * cfg.n_q * cfg.n_chunks * cfg.n_steps *
                              cfg.n_layers * steps / (total_ms * 1e-3),
        "pct_of_bf16_peak": 100.0 * value / peaks["bf16_tflops"],
        # a rollout is seconds of back-to-back tensor work under the 1 kW cap: the sustained
        # figure is its peak (the burst one is reported beside it)
        "roofline": {"bound": "tensor", "achieved": value,
                     "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                     "frac": value / peaks["bf16_tflops_sustained"], "traffic": None,
                     "kernel": "whole rollout (attention flops / all kernels' time)",
                     "peak_kind": f"{peak_kind} sustained bf16",
                     "frac_of_burst": value / peaks["bf16_tflops"]},
        "e2e": None,
        # per call: x-projection GEMM (with the chunk-key rotation in its epilogue) and attention
        # with the query heads formed inside it where supported, else x-projection, Q' GEMM,
        # chunk-key rotation and attention; per chunk and layer: the ring-key rotation (chunks
        # with a non-empty window) and the append
        "gpu_launches": steps * (calls * (2 if stack.fused_q else 4) + cfg.n_layers * (
            cfg.n_chunks + sum(1 for ch in range(cfg.n_chunks) if cfg.valid_frames(ch) > 0))),
        "clocks": dict(clk.summary(), sm_mhz_device=clock_after()),
    }
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_backward(args, cfg):
    """--backward: the gradient call mla_attention_bwd on the preset's measured chunk (window
    full), inputs drawn directly (seeded queries, chunk and ring latents, upstream gradient) and
    the forward's o_lat / lse computed first.  Algorithmic work per (query row, key, head):
    recomputed scores 2D, dP 2d_c, dq 2D, key gradient 2D, value gradient 2d_c."""
    import torch
    from mla_latent_kv_attn_b200 import api, inputs, rollout

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    c = api.make_config(cfg)
    dt = api.torch_dtype(c)
    ring = rollout.Ring(c, device=dev)
    lat = torch.empty((cfg.batch, cfg.n_q, cfg.d_latent), device=dev, dtype=dt)
    chunk = cfg.measured_chunk
    for ch in range(chunk):
        lat.copy_(torch.from_numpy(inputs.direct_latents(cfg, ch)).to(dt))
        api.mla_cache_append(c, None, None, lat, ring.cache, ring.slot_frame, cfg.first_frame(ch),
                             api.MLA_APPEND)
    first, n_valid = rollout.chunk_schedule(cfg.chunk_frames, cfg.window_frames, chunk)
    q = torch.from_numpy(inputs.direct_queries(cfg, chunk)).to(device=dev, dtype=dt)
    lat.copy_(torch.from_numpy(inputs.direct_latents(cfg, chunk)).to(dt))
    g = torch.from_numpy(inputs.upstream_gradient(cfg, chunk, cfg.d_c)).to(device=dev, dtype=dt)
    o_lat = torch.empty((cfg.batch, cfg.n_q, cfg.n_heads, cfg.d_c), device=dev, dtype=dt)
    lse = torch.empty((cfg.batch, cfg.n_heads, cfg.n_q), device=dev, dtype=torch.float32)
    ws = torch.empty(api.mla_attention_workspace_bytes(c, n_valid), device=dev, dtype=torch.uint8)
    api.mla_attention_fwd(c, q, lat, ring.cache, ring.slot_frame, n_valid, first, None, o_lat, lse, ws)
    d_q, d_lat, d_cache = torch.empty_like(q), torch.empty_like(lat), torch.empty_like(ring.cache)
    bws = torch.empty(api.mla_attention_bwd_workspace_bytes(c, n_valid), device=dev,
                      dtype=torch.uint8)
    call = lambda: api.mla_attention_bwd(c, q, lat, ring.cache, ring.slot_frame, n_valid, first,
                                         o_lat, lse, g, d_q, d_lat, d_cache, bws)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    steps = args.steps if args.steps_given else 5
    for _ in range(args.warmup):
        flush.zero_()
        call()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    with ClockSampler(local) as clk:
        for i in range(steps):
            flush.zero_()
            ev[i][0].record()
            call()
            ev[i][1].record()
        clock_after = probe_sm_clock(torch.cuda.current_stream())
        torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    per = 2.0 * (3 * cfg.d_latent + 2 * cfg.d_c)
    flops = per * cfg.n_q * cfg.keys_per_query(chunk) * cfg.n_heads * cfg.batch
    peaks, peak_kind = load_peaks()
    value = flops / (ms * 1e-3) / 1e12
    print(json.dumps({
        "metric": "MLA attention backward TFLOP/s (Wan-1.3B shape)", "value": value,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
        "data": "synthetic",
        "config": {"workload": cfg.name, "call": "mla_attention_bwd", "batch": cfg.batch,
                   "n_q": cfg.n_q, "keys_per_query": cfg.keys_per_query(chunk),
                   "flop_per_row_key_head": per,
                   "l2": "flushed before every call (256 MiB memset outside the event intervals)"},
        "roofline": {"bound": "tensor", "achieved": value, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": value / peaks["bf16_tflops"], "traffic": None,
                     "kernel": "mla_attention_bwd (" + ("tensor-core" if api.mla_attention_uses_tensor_cores(c, False) and cfg.d_c == 192 and cfg.d_rope == 32 and cfg.n_q % 4 == 0 else "CUDA-core") + " kernels)",
                     "peak_kind": f"{peak_kind} burst bf16"},
        "e2e": None, "gpu_launches": 5 * steps,
        "clocks": dict(clk.summary(), sm_mhz_device=clock_after())}), flush=True)
    return 0


def kernel_path(args) -> int:
    from mla_latent_kv_attn_b200 import api
    return {"auto": api.MLA_PATH_AUTO, "pair": api.MLA_PATH_TC_PAIR}[args.kernel_path]


def run_bandwidth_only(args, cfg):
    """--bandwidth-only: the stand-alone timing of the memory-bound calls (measure_bandwidth) and
    nothing else, one JSON object; used to profile those kernels on their own."""
    import torch
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    peaks, _ = load_peaks()
    reps = args.steps if args.steps_given else 20
    bw = measure_bandwidth(cfg, flush, torch.cuda.current_stream(), peaks["hbm_gbs"], reps=reps)
    print(json.dumps({"bandwidth": bw, "hbm_gbs": peaks["hbm_gbs"], "reps": reps}), flush=True)
    return 0


def kernel_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ("attention_sm100.cu", "attention_pair_sm100.cu", "sm100.cuh", "common.cuh",
              "kernels.h", "exp2.cuh"):
        h.update(open(os.path.join(ROOT, "mla_latent_kv_attn_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--cpu-rows", type=int, default=64)
    ap.add_argument("--ref-rows", type=int, default=64)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-bandwidth", action="store_true",
                    help="skip the stand-alone timing of the memory-bound calls")
    ap.add_argument("--kernel-path", choices=("auto", "pair"), default="auto",
                    help="attention kernel: auto (one CTA per head and query tile) or pair (the "
                         "CTA-pair kernel, for comparison)")
    ap.add_argument("--unfused-query", action="store_true",
                    help="project Q' with its own GEMM (mla_project_chunk + mla_attention_fwd) "
                         "instead of forming it inside the attention kernel")
    ap.add_argument("--bandwidth-only", action="store_true",
                    help="only time the memory-bound calls (append, RoPE, KV down-projection)")
    ap.add_argument("--backward", action="store_true",
                    help="time the attention backward call instead of the forward step")
    ap.add_argument("--d-c", type=int, default=None,
                    help="content-latent width (latent-size ablation shapes; default: the preset's)")
    ap.add_argument("--d-rope", type=int, default=None,
                    help="positional-key width (16, 32 or 64; default: the preset's)")
    args = ap.parse_args(argv)
    args.steps_given = args.steps is not None
    if args.steps is None:
        args.steps = 200
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from mla_latent_kv_attn_b200 import inputs
    cfg = inputs.CONFIGS[args.config]
    if args.d_c is not None or args.d_rope is not None:
        cfg = inputs.with_latent_shape(cfg, args.d_c or cfg.d_c, args.d_rope or cfg.d_rope)
    if args.impl == "reference":
        return run_reference(args, cfg)
    if args.bandwidth_only:
        return run_bandwidth_only(args, cfg)
    if args.backward:
        return run_backward(args, cfg)
    if cfg.n_layers > 1:
        return run_stack(args, cfg)
    return run_ours(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
