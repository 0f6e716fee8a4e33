"""Benchmark of one hot-path step: corrected attention of the current chunk over the packed
INT2 cache plus the unquantised chunk, then quantise-append of the finished chunk.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints ONE JSON line (rank 0). The default workload is the chunked-prefill shape (B4, 32 query /
8 KV heads, d128, 512-query chunk over a 131072-token INT2 cache), the largest of the five.
`value` is attention TFLOP/s of the whole job (algorithmic 4*d FLOPs per (query, visible key)
pair) over the device-timed steps, max over ranks. Inputs are resident in HBM; L2 is flushed (a
256 MiB write) between timed steps, outside the timed events. The `configs` block gives the same
figures for the other workloads (attention and whole-cache quantise-append of each), `decode` the
few-query-rows regime, `fidelity` the attention-fidelity diagnostics with and without the
correction at INT2 and INT4. `--impl reference` times the CPU oracle instead (bounded samples of
the same workload).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_kv_cache_19_b200 import api, shard  # noqa: E402
from quantized_kv_cache_19_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "corrected INT2-KV attention TFLOP/s & packed-cache GB/s, % of B200 roofline"
DEFAULT_WORKLOAD = "prefill_gqa"
# the other workloads of the bench's `configs` block (tiny_f32 is a correctness-only case)
CONFIG_WORKLOADS = ("bf16_int4", "bf16_int2", "video_dit", "long_video")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------------------------ ncu traffic
# DRAM bytes per launch come from one ncu capture per kernel and workload, stored with a hash of
# the kernel's sources; a stored figure is reported only while the sources still hash the same.
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
CSRC = os.path.join(ROOT, "quantized_kv_cache_19_b200", "csrc")
KERNEL_SOURCES = {
    "corrected_attention_kernel": ["attention.cu", "qkv_common.cuh", "qkv_jensen.cuh", "qkv_internal.h", "tile_ops.cuh"],
    "quantize_append_kernel": ["quant_append.cu", "qkv_common.cuh", "qkv_internal.h"],
    "attention_fidelity_kernel": ["fidelity.cu", "fidelity.h", "qkv_common.cuh", "qkv_jensen.cuh"],
}


def source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()


def ncu_traffic(kernel: str, workload: str):
    """DRAM read+write bytes per launch from the stored capture, or None if absent or stale."""
    try:
        with open(TRAFFIC_FILE) as f:
            entry = json.load(f).get(kernel, {}).get(workload)
    except (OSError, ValueError):
        return None
    if not entry or entry.get("source_sha256") != source_hash(kernel):
        return None
    return entry["dram_bytes_per_launch"]


def record_traffic(report: str, workload: str, command: str) -> None:
    """Reads dram__bytes_{read,write}.sum of every kernel in an ncu report and stores them."""
    import csv
    import io
    import subprocess
    out = subprocess.run(["ncu", "-i", report, "--page", "raw", "--csv"], check=True,
                         capture_output=True, text=True).stdout
    rows = list(csv.reader(io.StringIO(out)))
    hdr = rows[0]
    col = {name: hdr.index(name) for name in ("Kernel Name", "dram__bytes_read.sum", "dram__bytes_write.sum")}
    units = rows[1]
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    try:
        with open(TRAFFIC_FILE) as f:
            data = json.load(f)
    except (OSError, ValueError):
        data = {}
    for r in rows[2:]:
        name = r[col["Kernel Name"]].split("(")[0].split("<")[0].strip()
        kernel = next((k for k in KERNEL_SOURCES if k in name), None)
        if kernel is None:
            continue
        total = sum(float(r[col[m]].replace(",", "")) * scale[units[col[m]]]
                    for m in ("dram__bytes_read.sum", "dram__bytes_write.sum"))
        data.setdefault(kernel, {})[workload] = {
            "dram_bytes_per_launch": int(round(total)), "source_sha256": source_hash(kernel),
            "command": command}
    with open(TRAFFIC_FILE, "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
        f.write("\n")


def describe(w) -> str:
    return (f"{w.name}: B{w.B} Hq{w.Hq} Hkv{w.Hkv} d{w.d} Lq{w.Lq} Lcur{w.Lcur} Lc{w.Lc} "
            f"INT{w.bits} G{w.group} meta {w.meta} {w.dtype}{' causal' if w.causal else ''}")


# ------------------------------------------------------------------------------------ ranks
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def reduce_max(x: float, world: int, device) -> float:
    """Max of a float over ranks (the slowest rank's time decides a multi-GPU number)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                self.reasons |= int(self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._nv is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples),
                "reasons": [n for bit, n in self.REASONS.items() if self.reasons & bit]}


# ------------------------------------------------------------------------------------ CPU oracle
class OracleSample:
    """The oracle on a bounded sample of one step: the quantise-append of the whole current chunk,
    then corrected attention of sampled query rows of sampled (batch, KV head) pairs over their full
    cache. The sampled heads' caches are built once, outside the timing (they are the state the
    step starts from); the time of the whole step is extrapolated linearly in (query row, KV head)
    pairs."""

    def __init__(self, w, x_cpu, n_heads: int = 2):
        import oracle
        self.oracle, self.w = oracle, w
        K = {k: v.float().numpy() for k, v in x_cpu.items()}
        pairs = [(0, 0), (w.B - 1, w.Hkv - 1)]
        pairs = list(dict.fromkeys(pairs))[:n_heads]
        r = w.Hq // w.Hkv
        self.heads = []
        for b, h in pairs:
            sub = {"Q": K["Q"][b:b + 1, h * r:(h + 1) * r], "K_cur": K["K_cur"][b:b + 1, h:h + 1],
                   "V_cur": K["V_cur"][b:b + 1, h:h + 1]}
            cache = oracle.build_cache(K["K_src"][b:b + 1, h:h + 1], K["V_src"][b:b + 1, h:h + 1],
                                       w.bits, w.group, w.meta) if w.Lc else None
            self.heads.append((sub, cache))
        self.K_cur, self.V_cur = K["K_cur"], K["V_cur"]

    def time(self, budget_s: float, seed: int = 0):
        """Returns (seconds extrapolated to the whole step, flops of the step, sample text, cores)."""
        from threadpoolctl import threadpool_info
        w, oracle = self.w, self.oracle
        scale = 1.0 / math.sqrt(w.d)
        t0 = time.perf_counter()
        oracle.build_cache(self.K_cur, self.V_cur, w.bits, w.group, w.meta)      # the step's append
        t_quant = time.perf_counter() - t0
        rng = np.random.default_rng(seed)
        total_rows = (w.Hq // w.Hkv) * w.Lq
        spent, pairs_done = 0.0, 0
        for sub, cache in self.heads:
            order = rng.permutation(total_rows)        # rows drawn without replacement, in batches
            n, start, head_spent = 8, 0, 0.0
            while start < total_rows and head_spent < budget_s / len(self.heads):
                rows = np.sort(order[start:start + n])
                t0 = time.perf_counter()
                oracle.corrected_attention(sub["Q"], cache, sub["K_cur"], sub["V_cur"], correct=1,
                                           causal=w.causal, scale=scale, rows=rows)
                head_spent += time.perf_counter() - t0
                pairs_done += len(rows)
                start += len(rows)
                n *= 2
            spent += head_spent
        blas = sum(i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas")
        cores = blas or os.cpu_count()
        all_pairs = total_rows * w.B * w.Hkv
        est_s = t_quant + spent * all_pairs / pairs_done           # linear in (query row, KV head) pairs
        full_flops = api.attention_flops(w.B, w.Hq, w.Lq, w.Lc, w.Lcur, w.d, w.causal)
        text = (f"oracle (numpy fp64 attention, fp32 quantiser): quantise-append of the whole {w.Lcur}-token "
                f"chunk ({t_quant:.2f} s) + corrected attention of {pairs_done} of {all_pairs} (query row, "
                f"KV head) pairs, rows drawn at random in {len(self.heads)} KV head(s) ({spent:.2f} s); "
                f"full step extrapolated linearly in those pairs to {est_s:.1f} s")
        return est_s, full_flops, text, cores


# ------------------------------------------------------------------------------------ GPU arm
def timed_ms(fn, stream, flush, steps: int, warmup: int = 3) -> float:
    """Mean CUDA-event time (ms) of fn() on `stream` over `steps` launches after `warmup`, with L2
    flushed (a 256 MiB write) before every launch, outside the events."""
    ts = []
    for i in range(steps + warmup):
        flush.fill_(i & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        if i >= warmup:
            ts.append(a.elapsed_time(b))
    return statistics.mean(ts)


def qa_row_bytes(w) -> int:
    """Algorithmic HBM bytes of quantise-append per (token, KV head): read K and V, write both rows
    of codes and both rows of (step, zero-point)."""
    esz = 4 if w.dtype == "f32" else 2
    return 2 * w.d * esz + 2 * (w.d * w.bits // 8) + 2 * w.n_groups * 2 * (2 if w.meta == "f16" else 4)


def workload_figures(w, dev, peaks, flush, steps: int = 10):
    """One workload's attention (correct=1) and quantise-append, each timed alone: attention TFLOP/s
    against the measured bf16 peak and its packed-cache GB/s; the whole-cache quantise-append (every
    previous chunk in one call) and the append of one chunk against measured HBM."""
    x = make_inputs(w, device=dev)
    cache = api.KVCache(w.B, w.Hkv, w.d, w.bits, w.group, api.round_capacity(w.Lc + w.Lcur), w.meta,
                        device=dev)
    stream = torch.cuda.current_stream(dev)
    hbm, peak_t = float(peaks["hbm_gbs"]), float(peaks["bf16_tflops"])

    def build():
        cache.length = 0
        api.kv_quantize_append(cache, x["K_src"], x["V_src"])

    def chunk():
        cache.length = w.Lc
        api.kv_quantize_append(cache, x["K_cur"], x["V_cur"])

    full_ms = timed_ms(build, stream, flush, steps)
    chunk_ms = timed_ms(chunk, stream, flush, steps)
    cache.length = w.Lc
    O = torch.empty_like(x["Q"])
    LSE = torch.empty(w.B, w.Hq, w.Lq, dtype=torch.float32, device=dev)
    attn_ms = timed_ms(lambda: api.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=1,
                                                       causal=w.causal, out=O, lse=LSE), stream, flush, steps)
    if api.device_status() != 0:
        raise RuntimeError(f"device status after the {w.name} figures")
    flops = api.attention_flops(w.B, w.Hq, w.Lq, w.Lc, w.Lcur, w.d, w.causal)
    tf = flops / (attn_ms * 1e-3) / 1e12
    full_bytes = w.B * w.Hkv * w.Lc * qa_row_bytes(w)
    chunk_bytes = w.B * w.Hkv * w.Lcur * qa_row_bytes(w)
    out = {"workload": describe(w),
           "attention": {"kernel": "corrected_attention_kernel", "bound": "tensor",
                         "ms_per_launch": round(attn_ms, 5), "flops_per_launch": flops,
                         "achieved_tflops": round(tf, 2), "peak_tflops": peak_t, "frac": round(tf / peak_t, 4),
                         "packed_cache_gbs": round(cache.packed_bytes(w.Lc) / (attn_ms * 1e-3) / 1e9, 1)},
           "quant_append_full_cache": {"kernel": "quantize_append_kernel", "bound": "hbm", "tokens": w.Lc,
                                       "ms_per_launch": round(full_ms, 5), "bytes_per_launch": full_bytes,
                                       "achieved_gbs": round(full_bytes / (full_ms * 1e-3) / 1e9, 1),
                                       "peak_gbs": hbm, "frac": round(full_bytes / (full_ms * 1e-3) / 1e9 / hbm, 4)},
           "quant_append_chunk": {"tokens": w.Lcur, "ms_per_launch": round(chunk_ms, 5),
                                  "bytes_per_launch": chunk_bytes,
                                  "achieved_gbs": round(chunk_bytes / (chunk_ms * 1e-3) / 1e9, 1)}}
    del x, cache, O, LSE
    torch.cuda.empty_cache()
    return out


def decode_sweep(dev, peaks, flush, steps: int = 20):
    """Few query rows per KV head over the chunked-prefill workload's 131072-token INT2 cache
    (B4, 32 query / 8 KV heads): the regime where attention reads the packed cache once and the
    cached keys are split over CTAs. Packed-cache GB/s against the measured HBM peak."""
    base = WORKLOADS["prefill_gqa"]
    x = make_inputs(base.with_(Lq=16, Lcur=16), device=dev)
    cache = api.KVCache(base.B, base.Hkv, base.d, base.bits, base.group, api.round_capacity(base.Lc),
                        base.meta, device=dev)
    api.kv_quantize_append(cache, x["K_src"], x["V_src"])
    stream = torch.cuda.current_stream(dev)
    out = {"workload": "prefill_gqa cache (B4 Hq32 Hkv8 d128 Lc131072 INT2 G64 f32 meta), Lcur = Lq, causal",
           "bound": "hbm", "peak_gbs": float(peaks["hbm_gbs"]), "points": []}
    for Lq in (1, 4, 16):
        Q = x["Q"][:, :, :Lq].contiguous()
        Kc = x["K_cur"][:, :, :Lq].contiguous()
        Vc = x["V_cur"][:, :, :Lq].contiguous()
        O = torch.empty_like(Q)
        L = torch.empty(base.B, base.Hq, Lq, dtype=torch.float32, device=dev)
        nws = api.attention_workspace_bytes(cache, base.Hq, Lq, Lq)
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
        ms = timed_ms(lambda: api.corrected_attention(Q, cache, Kc, Vc, correct=1, causal=True, out=O, lse=L,
                                                      workspace=ws), stream, flush, steps)
        gbs = cache.packed_bytes(base.Lc) / (ms * 1e-3) / 1e9
        out["points"].append({"Lq": Lq, "rows_per_kv_head": 4 * Lq, "ms": round(ms, 4),
                              "workspace_bytes": nws, "packed_cache_gbs": round(gbs, 1),
                              "frac": round(gbs / float(peaks["hbm_gbs"]), 4)})
    if api.device_status() != 0:
        raise RuntimeError("device status after the decode sweep")
    del x, cache
    torch.cuda.empty_cache()
    return out


def fidelity_means(st) -> dict:
    return {"mass_ref": round(st[..., 2].mean().item(), 5), "mass_q": round(st[..., 3].mean().item(), 5),
            "kl": round(st[..., 4].mean().item(), 5), "token_drift": round(1.0 - st[..., 5].mean().item(), 5),
            "top5_recall": round(st[..., 6].mean().item(), 5)}


def fidelity_leg(dev, flush, steps: int = 10):
    """Attention-fidelity diagnostics (cached mass under the reference and the quantised softmax,
    KL(P_ref || P_q), token drift, top-5 recall), row means, without (correct=0) and with (correct=1)
    the correction, at INT2 and INT4, on the bf16 workload and on the video-DiT workload. The kernel
    (fp32 CUDA cores) is timed on bf16_int2 with correct=1 and top lists written: 4d FLOP per (query
    row, cached key) pair (two dot products) and 2d per visible current key, against the fp32 FMA
    peak 148 SMs x 128 lanes x 2 FLOP x the maximum SM clock."""
    props = torch.cuda.get_device_properties(dev)
    sm_mhz = float(load_peaks()[0].get("sm_max_mhz", 1965.0))
    peak = props.multi_processor_count * 128 * 2 * sm_mhz * 1e6 / 1e12
    stream = torch.cuda.current_stream(dev)
    out = {"kernel": "attention_fidelity_kernel", "compared": []}
    cases = [("bf16_int2", WORKLOADS["bf16_int2"]), ("bf16_int4", WORKLOADS["bf16_int4"]),
             ("video_dit", WORKLOADS["video_dit"]), ("video_dit at INT4", WORKLOADS["video_dit"].with_(bits=4))]
    for label, w in cases:
        x = make_inputs(w, device=dev)
        cache = api.KVCache(w.B, w.Hkv, w.d, w.bits, w.group, api.round_capacity(w.Lc), w.meta, device=dev)
        api.kv_quantize_append(cache, x["K_src"], x["V_src"])
        rec = {"workload": label, "bits": w.bits, "group": w.group}
        for correct in (0, 1):
            st, _ = api.attention_fidelity(x["Q"], cache, x["K_src"], x["K_cur"], correct=correct, causal=w.causal)
            rec[f"correct{correct}"] = fidelity_means(st)
        out["compared"].append(rec)
        if label == "bf16_int2":
            rows = w.B * w.Hq * w.Lq
            vis_cur = rows * w.Lcur
            flops = 4 * w.d * rows * w.Lc + 2 * w.d * vis_cur
            ms = timed_ms(lambda: api.attention_fidelity(x["Q"], cache, x["K_src"], x["K_cur"], correct=1,
                                                         causal=w.causal), stream, flush, steps)
            tf = flops / (ms * 1e-3) / 1e12
            out.update({"timed_on": "bf16_int2, correct=1, top lists written", "bound": "alu",
                        "ms_per_launch": round(ms, 4), "flops_per_launch": flops, "achieved": round(tf, 2),
                        "peak": round(peak, 1), "unit": "TFLOP/s",
                        "peak_kind": "fp32 FMA: SMs x 128 lanes x 2 x max SM clock", "frac": round(tf / peak, 4),
                        "traffic": ncu_traffic("attention_fidelity_kernel", w.name)})
        del x, cache
        torch.cuda.empty_cache()
    if api.device_status() != 0:
        raise RuntimeError("device status after the fidelity diagnostics")
    return out


def key_channel_leg(dev, flush, T: int = 32, steps: int = 10):
    """Per-channel keys along tokens (blocks of T positions, KIVI's group size of 32) on the bf16
    INT2 workload: the whole-cache quantise-append (keys per channel, values per token; HBM-bound),
    corrected attention with correct=1 on the tensor-core kernel for this layout (against the bf16
    peak), and with correct=2 on the fp32 CUDA-core kernel that serves the fourth-order term
    (against the fp32 FMA peak)."""
    w = WORKLOADS["bf16_int2"]
    x = make_inputs(w, device=dev)
    props = torch.cuda.get_device_properties(dev)
    peaks = load_peaks()[0]
    sm_mhz = float(peaks.get("sm_max_mhz", 1965.0))
    fp32_peak = props.multi_processor_count * 128 * 2 * sm_mhz * 1e6 / 1e12
    hbm = float(peaks["hbm_gbs"])
    bf16_peak = float(peaks["bf16_tflops"])
    cache = api.KVCache(w.B, w.Hkv, w.d, w.bits, w.group, api.round_capacity(w.Lc), w.meta, device=dev,
                        key_block=T)
    stream = torch.cuda.current_stream(dev)

    def quant():
        cache.length = 0
        api.kv_quantize_append(cache, x["K_src"], x["V_src"])

    q_ms = timed_ms(quant, stream, flush, steps)
    in_bytes = x["K_src"].element_size()
    q_bytes = 2 * w.B * w.Hkv * w.Lc * w.d * in_bytes + cache.packed_bytes(w.Lc)
    O = torch.empty_like(x["Q"])
    LSE = torch.empty(w.B, w.Hq, w.Lq, dtype=torch.float32, device=dev)
    flops = api.attention_flops(w.B, w.Hq, w.Lq, w.Lc, w.Lcur, w.d, w.causal)
    out = {"workload": describe(w), "key_block": T,
           "quantize_append_full_cache": {"bound": "hbm", "ms": round(q_ms, 4), "bytes": q_bytes,
                                          "achieved_gbs": round(q_bytes / (q_ms * 1e-3) / 1e9, 1),
                                          "peak_gbs": hbm,
                                          "frac": round(q_bytes / (q_ms * 1e-3) / 1e9 / hbm, 4)}}
    for correct, key, kernel, bound, peak, kind in (
            (1, "attention", "chan_attention_kernel (tensor cores)", "tensor", bf16_peak,
             "bf16 dense, of measured"),
            (2, "attention_correct2", "attention_f32_kernel (per-channel keys, CUDA cores)", "alu",
             fp32_peak, "fp32 FMA: SMs x 128 lanes x 2 x max SM clock")):
        a_ms = timed_ms(lambda: api.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=correct,
                                                        causal=w.causal, out=O, lse=LSE), stream, flush, steps)
        if api.device_status() != 0:
            raise RuntimeError("device status after the per-channel key leg")
        tf = flops / (a_ms * 1e-3) / 1e12
        out[key] = {"kernel": kernel, "correct": correct, "bound": bound, "ms_per_launch": round(a_ms, 4),
                    "flops_per_launch": flops, "achieved": round(tf, 2), "peak": round(peak, 1),
                    "unit": "TFLOP/s", "peak_kind": kind, "frac": round(tf / peak, 4)}
    del cache, x
    torch.cuda.empty_cache()
    return out


def e2e_leg(w, x, cache, dev, flush, n_steps: int):
    """The step through the public API with host buffers: every step uploads its Q, K_cur and V_cur
    from pinned host memory and reads O and LSE back into pinned host memory. Uploads and read-backs
    run on two copy streams with two sets of device buffers, so that step i+1's upload and step
    i-1's read-back overlap step i's kernels, as a serving loop would run it. Returns (ms per step,
    H2D bytes per step, D2H bytes per step); the time runs from the first upload to the last
    read-back, on the device."""
    comp = torch.cuda.current_stream(dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    names = ("Q", "K_cur", "V_cur")
    pin = [{k: x[k].cpu().pin_memory() for k in names} for _ in range(2)]
    d_in = [{k: torch.empty_like(x[k]) for k in names} for _ in range(2)]
    d_o = [torch.empty_like(x["Q"]) for _ in range(2)]
    d_l = [torch.empty(w.B, w.Hq, w.Lq, dtype=torch.float32, device=dev) for _ in range(2)]
    h_o = [torch.empty(d_o[0].shape, dtype=d_o[0].dtype).pin_memory() for _ in range(2)]
    h_l = [torch.empty(d_l[0].shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    uploaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    read = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def upload(i):
        s = i % 2
        with torch.cuda.stream(up):
            if used[s]:
                up.wait_event(computed[s])         # step i-2 has finished reading these inputs
            for k in names:
                d_in[s][k].copy_(pin[s][k], non_blocking=True)
            uploaded[s].record(up)

    def run(n, timed):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if timed:
            start.record(up)
        upload(0)
        for i in range(n):
            s = i % 2
            if i + 1 < n:
                upload(i + 1)
            comp.wait_event(uploaded[s])
            if used[s]:
                comp.wait_event(read[s])             # step i-2's outputs have been read back
            cache.length = w.Lc
            api.corrected_attention(d_in[s]["Q"], cache, d_in[s]["K_cur"], d_in[s]["V_cur"], correct=1,
                                    causal=w.causal, out=d_o[s], lse=d_l[s])
            api.kv_quantize_append(cache, d_in[s]["K_cur"], d_in[s]["V_cur"])
            computed[s].record(comp)
            used[s] = True
            with torch.cuda.stream(down):
                down.wait_event(computed[s])
                h_o[s].copy_(d_o[s], non_blocking=True)
                h_l[s].copy_(d_l[s], non_blocking=True)
                read[s].record(down)
        if timed:
            end.record(down)
        torch.cuda.synchronize()
        return start.elapsed_time(end) / n if timed else 0.0

    flush.fill_(0)
    run(3, False)
    torch.cuda.synchronize()
    ms = run(n_steps, True)
    h2d = sum(t.numel() * t.element_size() for t in pin[0].values())
    d2h = d_o[0].numel() * d_o[0].element_size() + d_l[0].numel() * 4
    return ms, h2d, d2h


def run_ours(args, world, rank, local):
    w_full = w = WORKLOADS[args.workload]
    if args.cache_tokens is not None:
        # the same shape with a shorter cache: small enough for a profiler capture of one launch
        w_full = w = w.with_(Lc=args.cache_tokens)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks, peak_kind = load_peaks()
    api.load_library()

    split = args.split_heads and world > 1
    if split:
        # one problem, its (batch, KV head) pairs split over the ranks with no exchange (strong scaling)
        if w.B * w.Hkv < world:
            raise SystemExit(f"--split-heads: {w.B * w.Hkv} (batch, KV head) pairs for {world} ranks")
        start, stop = shard.pair_ranges(w.B * w.Hkv, world)[rank]
        x_full = make_inputs(w, device="cuda")
        x = {k: v.contiguous() for k, v in shard.shard_inputs(x_full, w.B, w.Hq, w.Hkv, start, stop).items()}
        del x_full
        w = w.with_(B=stop - start, Hq=w.Hq // w.Hkv, Hkv=1)
    else:
        x = make_inputs(w, device="cuda", seed=w.seed + rank)  # each rank: its own problem (weak scaling)
    cap = api.round_capacity(w.Lc + w.Lcur)
    cache = api.KVCache(w.B, w.Hkv, w.d, w.bits, w.group, cap, w.meta, device=dev)
    for t0 in range(0, w.Lc, max(w.Lcur, 1)):                   # previous chunks, appended one by one
        t1 = min(w.Lc, t0 + max(w.Lcur, 1))
        api.kv_quantize_append(cache, x["K_src"][:, :, t0:t1].contiguous(), x["V_src"][:, :, t0:t1].contiguous())
    O = torch.empty_like(x["Q"])
    LSE = torch.empty(w.B, w.Hq, w.Lq, dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    ws_bytes = api.attention_workspace_bytes(cache, w.Hq, w.Lq, w.Lcur)
    launches_per_step = 2 + (1 if ws_bytes else 0)            # attention (+ merge of a key split) + append

    def step():
        cache.length = w.Lc
        api.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=1, causal=w.causal, out=O, lse=LSE)
        api.kv_quantize_append(cache, x["K_cur"], x["V_cur"])

    for _ in range(args.warmup):
        step()
        flush.fill_(1)
    torch.cuda.synchronize()
    assert api.device_status() == 0

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for i in range(K):
            cache.length = w.Lc
            ev[i][0].record(stream)
            api.corrected_attention(x["Q"], cache, x["K_cur"], x["V_cur"], correct=1, causal=w.causal,
                                    out=O, lse=LSE)
            ev[i][1].record(stream)
            api.kv_quantize_append(cache, x["K_cur"], x["V_cur"])
            ev[i][2].record(stream)
            flush.fill_(i & 0xFF)
        torch.cuda.synchronize()
    barrier(world)
    attn_ms = [e[0].elapsed_time(e[1]) for e in ev]
    qa_ms = [e[1].elapsed_time(e[2]) for e in ev]
    step_ms = [a + q for a, q in zip(attn_ms, qa_ms)]
    status = api.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed steps")

    # end to end through the public API with host buffers (pipelined uploads and read-backs)
    e2e_ms, h2d_bytes, d2h_bytes = e2e_leg(w, x, cache, dev, flush, min(K, 50))

    # whole-cache build: every previous chunk quantised in one call (the HBM-bound figure of the
    # quantiser; a single chunk is too small to leave launch latency behind)
    def build():
        cache.length = 0
        api.kv_quantize_append(cache, x["K_src"], x["V_src"])
    full_ms = timed_ms(build, stream, flush, 20)
    cache.length = w.Lc

    flops = api.attention_flops(w.B, w.Hq, w.Lq, w.Lc, w.Lcur, w.d, w.causal)
    # work of the whole job: every rank's own problem (replicas), or the one problem split over them
    job_flops = (api.attention_flops(w_full.B, w_full.Hq, w_full.Lq, w_full.Lc, w_full.Lcur, w_full.d, w_full.causal)
                 if split else world * flops)
    mean_step = statistics.mean(step_ms)
    mean_attn = statistics.mean(attn_ms)
    mean_qa = statistics.mean(qa_ms)
    ms_step = reduce_max(mean_step, world, dev)
    ms_attn = reduce_max(mean_attn, world, dev)
    ms_e2e = reduce_max(e2e_ms, world, dev)
    packed = cache.packed_bytes(w.Lc)
    qa_bytes = w.B * w.Hkv * w.Lcur * qa_row_bytes(w)
    full_bytes = w.B * w.Hkv * w.Lc * qa_row_bytes(w)
    peak_t = float(peaks["bf16_tflops"])
    achieved = flops / (ms_attn * 1e-3) / 1e12
    clk = clocks.summary()
    if clk.get("sm_mhz") and clk.get("sm_max_mhz"):
        # the attention time the kernel would take at the maximum SM clock, if it scaled with it
        clk["attention_ms_at_max_clock"] = round(ms_attn * clk["sm_mhz"] / clk["sm_max_mhz"], 5)
    result = {
        "metric": METRIC,
        "value": round(job_flops / (ms_step * 1e-3) / 1e12, 3),
        "unit": "TFLOP/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "strong" if split else "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": describe(w_full), "step": "corrected attention (correct=1) + quantise-append of the chunk",
                   "l2": "flushed between timed steps (256 MiB write, outside the timed events)",
                   "parallelism": (f"(batch, KV head) pairs split over {world} ranks, no exchange" if split
                                   else f"replicas x{world} (independent problems per GPU)")},
        "packed_cache_gbs": round(packed / (ms_attn * 1e-3) / 1e9, 1),
        "roofline": {"bound": "tensor", "kernel": "corrected_attention_kernel",
                     "achieved": round(achieved, 2), "peak": peak_t, "unit": "TFLOP/s",
                     "frac": round(achieved / peak_t, 4), "peak_kind": f"{peak_kind} bf16 dense (burst)",
                     "traffic": ncu_traffic("corrected_attention_kernel", w.name),
                     "ms_per_launch": round(ms_attn, 5),
                     "flops_per_launch": flops},
        "quant_append": {"bound": "hbm", "ms_per_launch": round(mean_qa, 5),
                         "bytes_per_launch": qa_bytes,
                         "traffic": ncu_traffic("quantize_append_kernel", w.name),
                         "achieved_gbs": round(qa_bytes / (mean_qa * 1e-3) / 1e9, 1),
                         "peak_gbs": float(peaks["hbm_gbs"]),
                         "frac": round(qa_bytes / (mean_qa * 1e-3) / 1e9 / float(peaks["hbm_gbs"]), 4),
                         "full_cache": {"tokens": w.Lc, "ms_per_launch": round(full_ms, 5),
                                        "bytes_per_launch": full_bytes,
                                        "traffic": ncu_traffic("quantize_append_kernel", w.name + "/full_cache"),
                                        "achieved_gbs": round(full_bytes / (full_ms * 1e-3) / 1e9, 1),
                                        "frac": round(full_bytes / (full_ms * 1e-3) / 1e9 /
                                                      float(peaks["hbm_gbs"]), 4)}},
        "e2e": {"value": round(job_flops / (ms_e2e * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(ms_e2e, 5), "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
                "how": "pinned host buffers; uploads and read-backs on two copy streams, double-buffered"},
        "gpu_launches": launches_per_step * K,
        "clocks": clk,
    }
    del x, cache, O, LSE
    torch.cuda.empty_cache()
    if not args.no_configs:
        result["configs"] = [workload_figures(WORKLOADS[n], dev, peaks, flush) for n in CONFIG_WORKLOADS
                             if n != w.name]
    if not args.no_fidelity:
        result["fidelity"] = fidelity_leg(dev, flush)
    if not args.no_key_channel:
        result["key_per_channel"] = key_channel_leg(dev, flush)
    if not args.no_decode:
        result["decode"] = decode_sweep(dev, peaks, flush)
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        x_cpu = make_inputs(w, device="cpu")
        est_s, full_flops, text, cores = OracleSample(w, x_cpu).time(args.cpu_budget)
        result["cpu_baseline"] = {"value": round(full_flops / est_s / 1e12, 6), "unit": "TFLOP/s",
                                  "cores": cores, "kind": "oracle", "sample": text}
    return result


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle, as it stands, on bounded samples of the same workload."""
    if rank != 0:
        return None
    w = WORKLOADS[args.workload]
    x_cpu = make_inputs(w, device="cpu")
    sample = OracleSample(w, x_cpu)
    per_step = max(0.5, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    times, text, cores = [], "", os.cpu_count()
    for i in range(args.warmup + args.steps):
        est_s, full_flops, text, cores = sample.time(per_step, seed=i)
        if i >= args.warmup:
            times.append(est_s)
    mean_s = statistics.mean(times)
    value = full_flops / mean_s / 1e12
    return {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "impl": "reference",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(mean_s * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": describe(w), "step": "corrected attention (correct=1) + quantise-append of the chunk"},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"each step: {text}"},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip the few-query-rows (decode) sweep")
    ap.add_argument("--no-fidelity", action="store_true", help="skip the attention-fidelity diagnostics")
    ap.add_argument("--no-key-channel", action="store_true", help="skip the per-channel key layout leg")
    ap.add_argument("--no-configs", action="store_true", help="skip the other workloads' figures")
    ap.add_argument("--cache-tokens", type=int, default=None,
                    help="override the workload's cache length (for profiler captures of a smaller case)")
    ap.add_argument("--split-heads", action="store_true",
                    help="with several ranks: split one problem by (batch, KV head) instead of replicas")
    ap.add_argument("--record-traffic", metavar="NCU_REP", default=None,
                    help="store the DRAM bytes per launch of an ncu report (taken on --workload) and exit")
    ap.add_argument("--record-command", default="", help="the command line that made the report")
    ap.add_argument("--record-key", default=None, help="key to store the figures under (default: --workload)")
    args = ap.parse_args(argv)
    if args.record_traffic:
        record_traffic(args.record_traffic, args.record_key or args.workload, args.record_command)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            res = run_reference(args, world, rank)
        else:
            res = run_ours(args, world, rank, local)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
