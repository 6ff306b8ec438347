"""Benchmark of the context-extended attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole hot path over one batch of synthetic input
(K rotation, tensor-core attention with the Q rotation fused in its tile load,
and for ring workloads the ring schedule, whose LSE merges run in the epilogue
of each later block's attention), through the C ABI.  The default workload is the 1M-token ring configuration (64 Q / 8 KV
heads, d 128, NTK s = 128, 16 ring blocks of 65,536 keys); the 128K sliding-
window configuration is timed in the same run and reported under "secondary".

Multi-GPU: the path has no data-path exchange on one GPU; N ranks run N
independent replicas of the workload (weak scaling), timed on the device, the
max over ranks.

--impl reference times the float64 CPU oracle on a bounded sample of the same
workload (rank 0 only) and prints the same metric.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "causal attention fwd TFLOP/s and % of B200 BF16 tensor peak at 128K and 1M"
# DRAM bytes (read + write) per attention launch of the named workload from
# ncu captures of the attention kernel as currently built, reported as
# roofline.traffic (remove an entry when the kernel changes).  32K: one launch
# captured.  1M: not captured at full size; the four launch forms of its ring
# were captured on the three-block 192K ring (same heads, block size and
# schedule) and weighted by their counts in the 1M step (1 direct, 15 first,
# 105 middle, 15 last).
ATTN_TRAFFIC_PER_LAUNCH = {"llama3_70b_32k_yarn": 1.193e9, "llama3_70b_1m_ring": 5.676e9}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def useful_flops(w):
    """4 * d * Hq * visible pairs per batch element (QK^T and PV, visible pairs only)."""
    from rope_context_extension_scaled_b200.configs import WORKLOADS  # noqa: F401
    return 4.0 * w.d * w.Hq * w.B * visible_pairs(w.N, w.window, w.n_sink)


def visible_pairs(N, window, n_sink):
    if window <= 0 or window >= N:
        return N * (N + 1) // 2
    # rows i < window see i + 1 keys; later rows see window keys plus min(n_sink, i - window + 1) sinks
    full = window * (window + 1) // 2 + (N - window) * window
    extra = 0
    if n_sink > 0:
        t = N - window                      # rows i >= window, with i - window + 1 = 1 .. t
        k = min(n_sink, t)
        extra = k * (k + 1) // 2 + max(0, t - k) * n_sink
    return full + extra


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        except Exception:
            pass
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- CPU oracle

def oracle_sample(w, get_q, get_kv, n_rows, seed=1):
    """Run the float64 oracle on n_rows seeded rows of batch 0: query heads of
    KV group 0 (every group costs the same), tokens uniform over the sequence.

    get_q(h, toks) -> [len(toks), 1, d] array; get_kv(g, last) -> k, v [last, 1, d].
    Returns (useful FLOPs of those rows, seconds, description)."""
    from oracle import rcx_oracle as orc
    rng = np.random.default_rng(seed)
    G = w.Hq // w.Hkv
    heads = rng.integers(0, G, size=n_rows)
    toks = rng.integers(0, w.N, size=n_rows)
    rows = {}
    for h, t in zip(heads, toks):
        rows.setdefault(int(h), set()).add(int(t))
    rows = {h: np.array(sorted(t)) for h, t in rows.items()}
    flops = sum(4.0 * w.d * visible_pairs_row(int(t), w.window, w.n_sink) for ts in rows.values() for t in ts)
    last = int(toks.max()) + 1
    k, v = get_kv(0, last)
    qs = {h: get_q(h, ts) for h, ts in rows.items()}
    t0 = time.perf_counter()
    inv, temp = orc.rope_freqs(w.scheme, w.base, w.d, w.L_train, w.L_target, w.alpha, w.beta)
    kk = orc.rope_rotate(k, np.arange(last), inv)
    for h, ts in rows.items():
        qq = orc.rope_rotate(qs[h], ts, inv)
        orc.attention(qq, kk, v, 1.0 / (math.sqrt(w.d) * temp), window=w.window, n_sink=w.n_sink,
                      q_index=ts, k_index=np.arange(last))
    dt = time.perf_counter() - t0
    return flops, dt, (f"{n_rows} seeded (head, token) rows of {w.name} (heads of KV group 0, tokens uniform), "
                       f"float64 numpy oracle incl. the K rotation")


def visible_pairs_row(i, window, n_sink):
    if window <= 0 or window > i:
        return i + 1
    return window + min(n_sink, i - window + 1)


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [x.get("num_threads", 0) for x in threadpool_info() if x.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


# ---------------------------------------------------------------- arms

def run_reference(args, w):
    """The oracle, as it stands, on a bounded sample per step (host cores)."""
    import torch
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    # Seeded N(0,1) inputs rounded to the storage dtype, drawn for the slices
    # the sampled rows read (one KV group; the sampled query rows).
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    g = torch.Generator().manual_seed(0)
    kf = torch.randn(w.N, 1, w.d, generator=g).to(dt).float().numpy()
    vf = torch.randn(w.N, 1, w.d, generator=g).to(dt).float().numpy()

    def get_q(h, toks):
        gq = torch.Generator().manual_seed(1000 + h)
        full = torch.randn(len(toks), 1, w.d, generator=gq).to(dt).float().numpy()
        return full

    def get_kv(grp, last):
        return kf[:last], vf[:last]

    rows = args.ref_rows
    for i in range(args.warmup):
        oracle_sample(w, get_q, get_kv, rows, seed=100 + i)
    fl, secs = 0.0, 0.0
    desc = ""
    for i in range(args.steps):
        f, s_, desc = oracle_sample(w, get_q, get_kv, rows, seed=1 + i)
        fl += f
        secs += s_
    val = fl / secs / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic N(0,1) rounded to bf16, seed 0",
            "config": config_dict(w),
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": desc + f"; per step, {args.steps} steps"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_dict(w):
    from rope_context_extension_scaled_b200.configs import PI, NTK, DYN_NTK, NTK_PARTS, YARN
    names = {0: "plain", PI: "pi", NTK: "ntk", DYN_NTK: "dyn_ntk", NTK_PARTS: "ntk_parts", YARN: "yarn"}
    d = {"workload": w.name, "batch": w.B, "seq_len": w.N, "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.d,
         "rope": f"{names[w.scheme]} base {w.base:g} L_train {w.L_train} L_target {w.L_target}",
         "window": w.window, "n_sink": w.n_sink, "causal": True,
         "ring_blocks": (w.N + w.kv_block - 1) // w.kv_block if (w.ring and w.kv_block) else 1,
         "l2": "inputs larger than L2 (126 MB)", "parallelism": "replicas"}
    return d


def max_over_ranks(x, dist, device="cuda"):
    """Max of a per-rank float over all ranks (identity without a process group)."""
    if dist is None or dist.get_world_size() == 1:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(world, flops_per_rank_step, ms_per_step):
    """Whole-job throughput: every rank's useful FLOPs over the slowest rank's time."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


def time_steps(run, steps, warmup, stream, dist, world):
    import torch
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        run()
    e1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), dist)
    return ms / steps


def run_ours(args, w):
    import torch
    from rope_context_extension_scaled_b200 import _lib
    from rope_context_extension_scaled_b200.configs import WORKLOADS
    from rope_context_extension_scaled_b200.inputs import make_qkv
    from rope_context_extension_scaled_b200.runner import run_workload

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist_mod
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                    device_id=torch.device("cuda", local))
        dist = dist_mod
    _lib.load()
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream()
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16

    # ---------------- secondary: the 128K sliding-window workload (short)
    secondary = None
    if args.secondary and w.name != "llama3_8b_128k_window":
        w2 = WORKLOADS["llama3_8b_128k_window"]
        q2, k2, v2 = make_qkv(w2.B, w2.N, w2.Hq, w2.Hkv, w2.d, torch.bfloat16, seed=0, device="cuda")
        run2 = run_workload(w2, q2, k2, v2)
        ms2 = time_steps(run2, max(args.steps, 10), max(args.warmup, 3), stream, dist, world)
        _lib.stats_reset()
        _lib.stats_enable_timing(True)
        for _ in range(5):
            run2()
        st2 = _lib.stats_read()
        _lib.stats_enable_timing(False)
        _lib.stats_reset()
        f2 = useful_flops(w2)
        attn_ms2 = st2["attn_tc"][1] / 5
        secondary = {"workload": w2.name, "value": aggregate_tflops(world, f2, ms2), "unit": "TFLOP/s",
                     "ms_per_step": ms2, "attn_kernel_tflops": f2 / (attn_ms2 * 1e-3) / 1e12,
                     "pct_of_peak": 100.0 * f2 / (ms2 * 1e-3) / 1e12 / peaks["bf16_tflops"],
                     "peak": f"bf16_tflops {peaks['bf16_tflops']} ({peak_src}, burst)",
                     "tokens_per_s": world * w2.B * w2.N / (ms2 * 1e-3)}
        del q2, k2, v2, run2
        torch.cuda.empty_cache()

    # ---------------- main workload
    q, k, v = make_qkv(w.B, w.N, w.Hq, w.Hkv, w.d, dt, seed=0, device="cuda")
    run = run_workload(w, q, k, v)
    with ClockSampler(local) as clk:
        ms = time_steps(run, args.steps, args.warmup, stream, dist, world)
    clocks = clk.summary()
    flops = useful_flops(w)
    value = aggregate_tflops(world, flops, ms)

    # per-kernel time over one more timed pass (CUDA events on the launching stream)
    _lib.stats_reset()
    _lib.stats_enable_timing(True)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    reps = max(1, min(args.steps, 2))
    for _ in range(reps):
        run()
    e1.record(stream)
    torch.cuda.synchronize()
    st = _lib.stats_read()
    _lib.stats_enable_timing(False)
    launches = sum(n for n, _ in st.values()) // reps
    kern = {}
    attn_key = "attn_tc" if w.dtype == "bf16" else "attn_simt"
    attn_n, attn_ms = st[attn_key][0] / reps, st[attn_key][1] / reps
    kern[attn_key] = {"launches_per_step": attn_n, "ms_per_step": attn_ms,
                      "tflops": flops / (attn_ms * 1e-3) / 1e12 if attn_ms else None}
    rope_bytes = 2.0 * w.B * w.N * w.Hkv * w.d * (2 if w.dtype == "bf16" else 4) + 8.0 * w.N * 0
    if st["rope_apply"][0]:
        r_ms = st["rope_apply"][1] / reps
        kern["rope_apply"] = {"launches_per_step": st["rope_apply"][0] / reps, "ms_per_step": r_ms,
                              "gbs": rope_bytes / (r_ms * 1e-3) / 1e9 if r_ms else None,
                              "pct_hbm": 100 * rope_bytes / (r_ms * 1e-3) / 1e9 / peaks["hbm_gbs"] if r_ms else None}
    if st["merge"][0]:
        m_ms = st["merge"][1] / reps
        P = (w.N + w.kv_block - 1) // w.kv_block
        # causal ring: shard r merges r partials; each merge reads two fp32 rows
        # and LSEs and writes one (the last merge of a shard writes bf16 O)
        rows_per_merge = w.B * w.Hq * w.kv_block
        n_merge = P * (P - 1) // 2
        m_bytes = rows_per_merge * (n_merge * (12 * w.d + 12) - (P - 1) * 2 * w.d)
        kern["merge"] = {"launches_per_step": st["merge"][0] / reps, "ms_per_step": m_ms,
                         "gbs": m_bytes / (m_ms * 1e-3) / 1e9 if m_ms else None,
                         "pct_hbm": 100 * m_bytes / (m_ms * 1e-3) / 1e9 / peaks["hbm_gbs"] if m_ms else None}
    # ---------------- decode: one new query token per head against the same KV cache
    decode = None
    if args.decode and w.dtype == "bf16":
        qd = q[:, -1:].contiguous()
        od = torch.empty_like(qd)
        ld = torch.empty(w.B, w.Hq, 1, dtype=torch.float32, device="cuda")
        inv_d, t_d = _lib.rope_freqs(w.scheme, w.base, w.d, w.L_train, w.L_target, w.alpha, w.beta)
        wsd = torch.empty(max(_lib.load().rcx_attn_decode_workspace_size(_lib.view(qd), _lib.view(k)), 256),
                          dtype=torch.uint8, device="cuda")

        def dstep():
            _lib.attn_decode_fwd(qd, k, v, od, ld, window=w.window, n_sink=w.n_sink, temperature=t_d,
                                 q_index=w.N - 1, inv_freq=inv_d, rope_flags=_lib.ROTATE_Q, workspace=wsd)
        d_ms = time_steps(dstep, 20, 5, stream, dist, world)
        kv_bytes = 2.0 * k.numel() * k.element_size()
        decode = {"workload": f"decode: 1 query token per head, {w.N}-token KV cache, {w.Hq}/{w.Hkv} heads",
                  "ms": d_ms, "gbs": kv_bytes / (d_ms * 1e-3) / 1e9,
                  "pct_hbm": 100.0 * kv_bytes / (d_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                  "tokens_per_s": world * w.B / (d_ms * 1e-3)}
        # the same decode over the int8 copy of the cache (codes made outside the timed region)
        kc, ks = _lib.kv_quantize_int8(k)
        vc, vs = _lib.kv_quantize_int8(v)
        ws8 = torch.empty(max(_lib.load().rcx_attn_decode_int8_workspace_size(_lib.view(qd), _lib.view(kc)), 256),
                          dtype=torch.uint8, device="cuda")

        def dstep8():
            _lib.attn_decode_int8_fwd(qd, kc, ks, vc, vs, od, ld, window=w.window, n_sink=w.n_sink,
                                      temperature=t_d, q_index=w.N - 1, inv_freq=inv_d, rope_flags=_lib.ROTATE_Q,
                                      workspace=ws8)
        d8_ms = time_steps(dstep8, 20, 5, stream, dist, world)
        kv8_bytes = 2.0 * (kc.numel() + 4 * ks.numel())
        decode["int8_cache"] = {"ms": d8_ms, "gbs": kv8_bytes / (d8_ms * 1e-3) / 1e9,
                                "pct_hbm": 100.0 * kv8_bytes / (d8_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                "tokens_per_s": world * w.B / (d8_ms * 1e-3),
                                "bytes_per_step": kv8_bytes}
        # the append path: quantising the bf16 K cache (read bf16, write codes and scales)
        kq_out = torch.empty_like(kc)
        ksc_out = torch.empty_like(ks)
        q_ms = time_steps(lambda: _lib.kv_quantize_int8(k, codes=kq_out, scale=ksc_out), 10, 3, stream, dist, world)
        q_bytes = k.numel() * k.element_size() + kq_out.numel() + 4 * ksc_out.numel()
        decode["int8_quantize"] = {"workload": f"quantise the {w.N}-token K cache ({w.Hkv} heads)", "ms": q_ms,
                                   "gbs": q_bytes / (q_ms * 1e-3) / 1e9,
                                   "pct_hbm": 100.0 * q_bytes / (q_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
        del kq_out, ksc_out
        del qd, od, ld, wsd, kc, ks, vc, vs, ws8
    peak_key = "bf16_tflops_sustained" if ms > 1000 else "bf16_tflops"
    peak = peaks.get(peak_key, FALLBACK_PEAKS[peak_key])
    achieved = flops / (attn_ms * 1e-3) / 1e12
    traffic = args.traffic if args.traffic is not None else ATTN_TRAFFIC_PER_LAUNCH.get(w.name)
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": traffic, "kernel": attn_key,
                "peak_source": f"{peak_key} ({peak_src})"}
    del run
    torch.cuda.empty_cache()

    # ---------------- e2e: host buffers through the C ABI (H2D and D2H inside the timed region)
    qh = q.cpu()
    kh = k.cpu()
    vh = v.cpu()
    del q, k, v
    torch.cuda.empty_cache()
    e2e = None
    need_host = 2.2 * (qh.numel() * qh.element_size() + 2 * kh.numel() * kh.element_size())
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = float("inf")
    if args.e2e and need_host * world < avail:
        qp, kp, vp = qh.pin_memory(), kh.pin_memory(), vh.pin_memory()
        op = torch.empty_like(qp).pin_memory()
        lp = torch.empty(w.B, w.Hq, w.N, dtype=torch.float32).pin_memory()
        inv, temp = _lib.rope_freqs(w.scheme, w.base, w.d, w.L_train, w.L_target, w.alpha, w.beta)

        def host_step():
            _lib.ring_attn_fwd_host(qp, kp, vp, op, lp, kv_block=w.kv_block if w.ring else 0, window=w.window,
                                    n_sink=w.n_sink, temperature=temp, inv_freq=inv,
                                    rope_flags=_lib.ROTATE_Q | _lib.ROTATE_K)
        host_step()
        if dist is not None:
            dist.barrier()
        t0 = time.perf_counter()
        for _ in range(args.e2e_steps):
            host_step()
        e_ms = max_over_ranks((time.perf_counter() - t0) * 1e3 / args.e2e_steps, dist)
        h2d = sum(x.numel() * x.element_size() for x in (qp, kp, vp))
        d2h = op.numel() * op.element_size() + lp.numel() * 4
        e2e = {"value": aggregate_tflops(world, flops, e_ms), "unit": "TFLOP/s", "ms_per_step": e_ms,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "api": "rcx_ring_attn_fwd_host (pinned host buffers; copies, device staging and compute)"}
        del qp, kp, vp, op, lp
    elif args.e2e:
        e2e = {"value": None, "unit": "TFLOP/s", "skipped": "not enough host memory for pinned copies"}

    # ---------------- CPU baseline: the oracle on a bounded sample (rank 0, N = 1)
    cpu = None
    if rank == 0 and world == 1 and args.cpu_rows > 0:
        G = w.Hq // w.Hkv

        def get_q(h, toks):
            return qh[0, torch.as_tensor(toks), h:h + 1].float().numpy()

        def get_kv(grp, last):
            return kh[0, :last, grp:grp + 1].float().numpy(), vh[0, :last, grp:grp + 1].float().numpy()
        f, s_, desc = oracle_sample(w, get_q, get_kv, args.cpu_rows)
        cpu = {"value": f / s_ / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": desc + f"; {s_:.1f} s"}

    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic N(0,1) rounded to bf16, seed 0",
            "config": config_dict(w),
            "pct_of_peak": 100.0 * value / world / peak, "peak": f"{peak_key} {peak} ({peak_src})",
            "tokens_per_s": world * w.B * w.N / (ms * 1e-3),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(launches * args.steps),
            "kernels": kern, "clocks": clocks, "secondary": secondary, "decode": decode}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama3_70b_1m_ring")
    ap.add_argument("--cpu-rows", type=int, default=24, help="oracle rows for cpu_baseline (0 = skip)")
    ap.add_argument("--ref-rows", type=int, default=12, help="oracle rows per reference-arm step")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--e2e-steps", type=int, default=1)
    ap.add_argument("--no-secondary", dest="secondary", action="store_false")
    ap.add_argument("--no-decode", dest="decode", action="store_false")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per attention launch from an ncu capture (reported as roofline.traffic)")
    args = ap.parse_args()
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    from rope_context_extension_scaled_b200.configs import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
