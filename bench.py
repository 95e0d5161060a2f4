#!/usr/bin/env python
"""Decode-step benchmark of the compressed KV-cache path.

One step = one decode token through every layer of the Llama-3.1-8B-shaped
workload (32 layers, batch 8, 32 q / 8 kv heads, head_dim 128, 512 hot fp16
tokens + 32256 compressed cold tokens, b_r = b_theta = 3, m = 128): per
layer tq_evict_window (the new token enters the hot ring, the oldest hot
token is compressed into the cold store) then tq_decode_attention (q-prep,
hot + cold attention, combine).  Inputs are seeded synthetic tensors with
the workload's value recipe, generated on the device; the 32 layers' caches
(8.4 GB) are far larger than L2, and every layer has its own buffers.

Prints ONE JSON line (rank 0).  ``--impl reference`` times the fp64 CPU
oracle on the same metric instead (a bounded sample per step).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "cold-KV decode attention keys/s and achieved HBM GB/s (% of B200 peak)"
UNIT = "keys/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--workload", default="llama8b")
    ap.add_argument("--layers", type=int, default=0, help="0: the workload's layer count")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--gate-quantile", type=float, default=None,
                    help="decode with the threshold-gated cold tier; each layer's threshold is this "
                         "quantile of its heads' hot-window maxima q.k at the start")
    ap.add_argument("--tensor-cache", action="store_true",
                    help="decode with the Tensor Cache tier: evicted tokens go to an outer-product "
                         "memory instead of the compressed cold store")
    ap.add_argument("--promotion", action="store_true",
                    help="decode with attention-weighted promotion (threshold 0.15, sticky 3)")
    ap.add_argument("--encode", action="store_true",
                    help="time the prefill encode (tq_encode_append of 4096-token chunks) instead")
    return ap.parse_args()


# DRAM bytes (read + write) of one attention launch on the default workload,
# from an ncu capture, keyed by the SHA-1 of the kernel source it was taken
# on; any other source reports null (the counters no longer describe it).
# DRAM bytes (read + write) of one attention launch on the llama8b workload,
# from an ncu capture of such a launch, keyed by the
# SHA-1 of the kernel's source; a changed kernel reports null until captured
# again.
ATTEND_TRAFFIC = {
    "d16f271aa746a9be5796851f85296458defa66c1": 261319680 + 3596544,
}


def attend_traffic(same_workload: bool):
    import hashlib
    src = os.path.join(ROOT, "compressed_decode_attention_encode_b200", "csrc", "tq_attend.cuh")
    h = hashlib.sha1(open(src, "rb").read()).hexdigest()
    return ATTEND_TRAFFIC.get(h) if same_workload else None


# --------------------------------------------------------------------------
# ranks: one process per GPU (torchrun); every rank runs the full per-GPU
# workload (weak scaling, no data-path collective)
# --------------------------------------------------------------------------
def rank_env():
    """(world size, rank, local rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, device) -> float:
    """The largest per-rank value over the process group (x with one rank):
    a job's time is its slowest rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, units_per_rank: float, ms_max: float) -> float:
    """Whole-job rate of a weak-scaling run: every rank processes
    `units_per_rank` in the slowest rank's `ms_max` milliseconds."""
    return world * units_per_rank / (ms_max / 1e3)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# --------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"tq_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), smax=float(f[2]), hw=f[5], hwt=f[6], swt=f[7],
                                 pcap=f[8]))
            except ValueError:
                continue
        if not rows:
            return None
        reasons = set()
        for r in rows:
            if r["hw"] == "Active": reasons.add("hw_slowdown")
            if r["hwt"] == "Active": reasons.add("hw_thermal_slowdown")
            if r["swt"] == "Active": reasons.add("sw_thermal_slowdown")
            if r["pcap"] == "Active": reasons.add("sw_power_cap")
        return {"sm_mhz": statistics.median(r["sm"] for r in rows),
                "sm_max_mhz": max(r["smax"] for r in rows), "samples": len(rows),
                "reasons": sorted(reasons)}


# --------------------------------------------------------------------------
# oracle timing (cpu_baseline and the reference arm)
# --------------------------------------------------------------------------
def oracle_sample(wl, seed: int, kv_heads: int):
    """One batch row, `kv_heads` kv heads of layer 0: oracle-encoded records
    (built once, untimed) and the query."""
    import numpy as np
    from compressed_decode_attention_encode_b200.inputs import kv_stream, queries
    from oracle import tq_oracle as O
    d = wl.head_dim
    signs = O.rotation_signs(seed, d)
    S = O.qjl_matrix(seed, wl.qjl_bits, d)
    ck, cv, hk, hv = [], [], [], []
    for h in range(kv_heads):
        k = kv_stream(wl, 0, seed, 0, 0, h, 0, wl.cold + wl.hot).astype(np.float64)
        v = kv_stream(wl, 0, seed, 1, 0, h, 0, wl.cold + wl.hot).astype(np.float64)
        ck.append(O.encode(k[: wl.cold], signs, S, wl.b_r, wl.b_theta))
        cv.append(O.encode(v[: wl.cold], signs, None, wl.b_r, wl.b_theta))
        hk.append(k[wl.cold:])
        hv.append(v[wl.cold:])
    q = queries(wl, 0, seed)[0, : kv_heads * wl.group].astype(np.float64)
    return dict(q=q, hk=np.stack(hk), hv=np.stack(hv), ck=ck, cv=cv, signs=signs, S=S,
                kv_heads=kv_heads)


def time_oracle(sample):
    """Seconds and keys of one oracle decode over the sample."""
    from oracle import tq_oracle as O
    t0 = time.perf_counter()
    O.decode_attention(sample["q"], sample["hk"], sample["hv"], sample["ck"], sample["cv"],
                       sample["signs"], sample["S"], sample["kv_heads"])
    dt = time.perf_counter() - t0
    keys = sample["kv_heads"] * (sample["hk"].shape[1] + sample["ck"][0].s16.shape[0])
    return dt, keys


def oracle_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 1) for i in info), default=1)
        return int(n)
    except Exception:
        return 1


def run_reference(args, wl):
    _, rank, _ = rank_env()
    if rank != 0:              # the reference arm runs on rank 0 only
        return
    sample = oracle_sample(wl, args.seed, kv_heads=2)
    for _ in range(args.warmup):
        time_oracle(sample)
    tot_t, tot_k = 0.0, 0
    for _ in range(args.steps):
        dt, k = time_oracle(sample)
        tot_t += dt
        tot_k += k
    v = tot_k / tot_t
    desc = (f"per step: oracle decode attention of 1 batch row x 2 kv heads (8 q heads) of "
            f"layer 0, {wl.cold} cold + {wl.hot} hot tokens")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.name, "layers": wl.layers, "batch": wl.batch,
                   "num_q_heads": wl.num_q_heads, "num_kv_heads": wl.num_kv_heads,
                   "head_dim": wl.head_dim, "hot": wl.hot, "cold": wl.cold,
                   "b_r": wl.b_r, "b_theta": wl.b_theta, "qjl_bits": wl.qjl_bits},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# --------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------
def gen_kv(wl, layer, seed, which, b_rows, start, count, device, gen):
    """fp16 [B, Hkv, count, d] with the workload's channel scales (device RNG)."""
    import torch
    from compressed_decode_attention_encode_b200.inputs import channel_scales
    sc = torch.from_numpy(channel_scales(wl, layer, seed, which)).to(device=device, dtype=torch.float32)
    z = torch.randn((b_rows, wl.num_kv_heads, count, wl.head_dim), generator=gen, device=device,
                    dtype=torch.float32)
    return (z * sc[None, :, None, :]).to(torch.float16)


def run_gpu(args, wl):
    import numpy as np
    import torch
    import torch.distributed as dist

    from compressed_decode_attention_encode_b200 import build as B
    from compressed_decode_attention_encode_b200 import tq

    world, rank, local = rank_env()
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        B.build()
    if world > 1:
        dist.barrier()
    tq.lib()

    L = args.layers or wl.layers
    total_steps = args.warmup + 3 * args.steps + 2
    cap = wl.cold + total_steps + 64
    cfg = tq.make_config(wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.hot, cap,
                         wl.b_r, wl.b_theta, wl.qjl_bits, seed=args.seed)
    stream = torch.cuda.current_stream()
    gen = torch.Generator(device=dev)
    caches = []
    chunk = 4096
    for layer in range(L):
        gen.manual_seed(1_000_003 * (args.seed + 1) + 7919 * layer + rank)
        c = tq.TQCache(cfg, device=dev)
        if args.tensor_cache:      # fixed synthetic decay, write rate and gate
            c.enable_tensor_cache([0.995] * wl.num_kv_heads, [0.05] * wl.num_kv_heads,
                                  [0.0] * wl.num_q_heads)
        pos = 0
        while pos < wl.cold:
            n = min(chunk, wl.cold - pos)
            k = gen_kv(wl, layer, args.seed, 0, wl.batch, pos, n, dev, gen)
            v = gen_kv(wl, layer, args.seed, 1, wl.batch, pos, n, dev, gen)
            if args.tensor_cache:  # the whole context streams through the ring into A
                c.evict_window(k, v)
            else:
                c.encode_append(k, v)
            pos += n
        k = gen_kv(wl, layer, args.seed, 0, wl.batch, 0, wl.hot, dev, gen)
        v = gen_kv(wl, layer, args.seed, 1, wl.batch, 0, wl.hot, dev, gen)
        c.evict_window(k, v)
        if args.promotion:         # the page's benchmark setting
            c.enable_promotion(0.15, 3)
        if c.get_status() != 0:
            raise RuntimeError("device status after prefill")
        caches.append(c)
    # per-step inputs (new token K/V per layer, queries per layer)
    knew = [gen_kv(wl, l, args.seed, 0, wl.batch, 0, total_steps, dev, gen) for l in range(L)]
    vnew = [gen_kv(wl, l, args.seed, 1, wl.batch, 0, total_steps, dev, gen) for l in range(L)]
    knew = [[x[:, :, s:s + 1].contiguous() for s in range(total_steps)] for x in knew]
    vnew = [[x[:, :, s:s + 1].contiguous() for s in range(total_steps)] for x in vnew]
    qs = [torch.randn((wl.batch, wl.num_q_heads, wl.head_dim), generator=gen, device=dev).half()
          for _ in range(L)]
    outs = [torch.empty((wl.batch, wl.num_q_heads, wl.head_dim), dtype=torch.float32, device=dev)
            for _ in range(L)]
    torch.cuda.synchronize()

    units = wl.batch * wl.num_kv_heads
    kc = wl.head_dim // 2 * (wl.b_r + wl.b_theta) // 8
    cold_tok_bytes = 2 * kc + wl.qjl_bits // 8 + 6     # K and V record bytes
    hot_tok_bytes = 4 * wl.head_dim                     # K and V fp16

    gate_tau = None
    skip_bufs = None
    if args.gate_quantile is not None:
        # per-layer thresholds: a quantile of max_t q.k over each head's hot
        # window (a configuration choice made once, outside the timed path)
        G = wl.num_q_heads // wl.num_kv_heads
        gate_tau = []
        for l in range(L):
            hk, _ = caches[l].hot_ring()
            qf = qs[l].float().view(wl.batch, wl.num_kv_heads, G, wl.head_dim)
            sc = torch.einsum("bhgd,bhtd->bhgt", qf, hk.float())
            gate_tau.append(float(torch.quantile(sc.amax(dim=-1).flatten(), args.gate_quantile)))
        skip_bufs = [torch.zeros((wl.batch, wl.num_q_heads), dtype=torch.int32, device=dev)
                     for _ in range(L)]

    def attend(l, q, out):
        if gate_tau is None:
            caches[l].decode_attention(q, out=out)
        else:
            caches[l].decode_attention_gated(q, gate_tau[l], out=out, head_skip=skip_bufs[l])

    step_idx = [0]
    seen = [wl.cold + wl.hot] * L        # tokens inserted per (row, kv head), per layer
    tc_bytes = 12 * wl.head_dim * wl.head_dim   # A read + written (update), read (decode), float32

    def one_step(ev_pairs=None):
        s = step_idx[0]
        step_idx[0] += 1
        keys = 0
        abytes = 0
        for l in range(L):
            caches[l].evict_window(knew[l][s], vnew[l][s])
            nc, nh, _ = caches[l].counts()
            seen[l] += 1
            if args.tensor_cache:
                keys += units * seen[l]
                abytes += units * (nh * hot_tok_bytes + tc_bytes)
            else:
                keys += units * (nc + nh)
                abytes += units * (nc * cold_tok_bytes + nh * hot_tok_bytes)
                if args.promotion:      # the attention kernel also writes every cold logit
                    abytes += units * nc * wl.group * 4
            if ev_pairs is not None:
                caches[l].set_attend_events(*ev_pairs[l])
            attend(l, qs[l], outs[l])
            if ev_pairs is not None:
                caches[l].set_attend_events(None, None)
        return keys, abytes

    for _ in range(args.warmup):
        one_step()
    for c in caches:
        if c.get_status() != 0:
            raise RuntimeError("device status after warm-up")

    # ---- timed region: device-resident inputs --------------------------
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(L)] for _ in range(args.steps)]
    for row in ev:                       # torch creates CUDA events lazily
        for a_, b_ in row:
            a_.record(stream)
            b_.record(stream)
    clock = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clock.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    # pass 1: the steps alone (no event between the kernels of a step, so
    # the programmatic launches overlap as they do in use)
    t0.record(stream)
    keys_total = 0
    for s in range(args.steps):
        k_, _ = one_step()
        keys_total += k_
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    # pass 2: the same number of steps with CUDA events around every
    # attention launch, for the kernel's own duration
    bytes_total = 0
    for s in range(args.steps):
        _, b_ = one_step(ev[s])
        bytes_total += b_
    torch.cuda.synchronize()
    clocks = clock.stop()
    attend_ms = sum(a.elapsed_time(b) for row in ev for (a, b) in row)
    for c in caches:
        if c.get_status() != 0:
            raise RuntimeError("device status in timed region")
    ms = max_over_ranks(ms, dev)
    # evict: per-token encode (ring write fused); decode: qprep, [gate,] attend, combine
    launches_per_step = L * (1 + 3 + (gate_tau is not None))
    if args.promotion:   # evict: dequant, encode, ring positions; decode: + the mass kernel
        launches_per_step = L * (3 + 4)

    # ---- e2e: host buffers through the public API ------------------------
    # Each step's inputs (every layer's new K, V token and queries) travel in
    # one host->device copy from pinned memory, and the step's outputs come
    # back in one device->host copy.
    kn, vn, qn = knew[0][0].numel(), vnew[0][0].numel(), qs[0].numel()
    per_layer = kn + vn + qn
    nsteps_in = len(knew[0])
    hin = torch.empty((nsteps_in, L * per_layer), dtype=torch.float16).pin_memory()
    for st_i in range(nsteps_in):
        for l in range(L):
            o = l * per_layer
            hin[st_i, o:o + kn] = knew[l][st_i].reshape(-1).cpu()
            hin[st_i, o + kn:o + kn + vn] = vnew[l][st_i].reshape(-1).cpu()
            hin[st_i, o + kn + vn:o + per_layer] = qs[l].reshape(-1).cpu()
    din = torch.empty((L * per_layer,), dtype=torch.float16, device=dev)
    on = outs[0].numel()
    dout = torch.empty((L, on), dtype=torch.float32, device=dev)
    hout = torch.empty((L, on), dtype=torch.float32).pin_memory()
    views = []
    for l in range(L):
        o = l * per_layer
        views.append((din[o:o + kn].view(knew[0][0].shape), din[o + kn:o + kn + vn].view(vnew[0][0].shape),
                      din[o + kn + vn:o + per_layer].view(qs[0].shape), dout[l].view(outs[0].shape)))
    e2e_steps = args.steps
    h2d = d2h = 0
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_keys = 0
    for _ in range(e2e_steps):
        s = step_idx[0] % nsteps_in
        step_idx[0] += 1
        din.copy_(hin[s], non_blocking=True)
        h2d = din.numel() * 2
        for l in range(L):
            dk, dv, dq, do = views[l]
            caches[l].evict_window(dk, dv)
            nc, nh, _ = caches[l].counts()
            seen[l] += 1
            e2e_keys += units * (seen[l] if args.tensor_cache else nc + nh)
            attend(l, dq, do)
        hout.copy_(dout, non_blocking=True)
        d2h = dout.numel() * 4
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, dev)

    value = job_rate(world, keys_total, ms)
    e2e_value = job_rate(world, e2e_keys, e2e_ms)
    hbm_peak, peak_kind = peaks()
    attend_launches = L * args.steps
    achieved = bytes_total / (attend_ms / 1e3) / 1e9
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16-in/f32-acc", "data": "synthetic",
        "config": {"workload": wl.name, "layers": L, "batch": wl.batch,
                   "num_q_heads": wl.num_q_heads, "num_kv_heads": wl.num_kv_heads,
                   "head_dim": wl.head_dim, "hot": wl.hot, "cold": wl.cold,
                   "b_r": wl.b_r, "b_theta": wl.b_theta, "qjl_bits": wl.qjl_bits,
                   "l2": "inputs larger than L2 (each of the layers has its own "
                         f"{caches[0].bytes['cold'] / 1e6:.0f} MB cold store)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "hbm": {"step_gbs": bytes_total / (ms / 1e3) / 1e9, "attend_gbs": achieved,
                "frac_of_measured": achieved / hbm_peak, "frac_of_8tbs_spec": achieved / 8000.0},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": attend_traffic(wl.name == "llama8b"),
                     "kernel": "attend_kernel",
                     "peak_kind": peak_kind,
                     "avg_launch_us": 1e3 * attend_ms / attend_launches,
                     "bytes_per_launch": bytes_total / attend_launches,
                     "timing": "ms_per_step from a timed pass with no per-kernel events; the "
                               "attention kernel's duration from a second pass of as many steps "
                               "with CUDA events around each launch"},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / e2e_steps},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if gate_tau is not None:
        # what the gate skipped (last step's decisions) and what it changed:
        # the gated output against the ungated one on the same cache state
        G = wl.num_q_heads // wl.num_kv_heads
        sk = torch.stack(skip_bufs).bool()                       # [L, B, Hq]
        whole = sk.view(L, wl.batch, wl.num_kv_heads, G).all(dim=-1)
        errs = []
        for l in range(L):
            a_ = caches[l].decode_attention(qs[l])
            b_ = caches[l].decode_attention_gated(qs[l], gate_tau[l])
            errs.append(((b_ - a_).norm(dim=-1) / a_.norm(dim=-1).clamp_min(1e-30)).flatten())
        errs = torch.cat(errs)
        nc, nh, _ = caches[0].counts()
        read = (~whole).sum().item() * nc * cold_tok_bytes + L * units * nh * hot_tok_bytes
        achieved_g = read / L / (attend_ms / attend_launches / 1e3) / 1e9
        result["metric"] = "gated decode: context keys/s (cold tier read only below the hot-max threshold)"
        result["config"]["gate_quantile"] = args.gate_quantile
        result["gate"] = {
            "thresholds_first_layers": gate_tau[:4],
            "heads_skipped_frac": sk.float().mean().item(),
            "units_skipped_frac": whole.float().mean().item(),
            "out_rel_l2_vs_ungated": {"max": errs.max().item(), "mean": errs.mean().item(),
                                      "heads_over_2e-3": int((errs > 2e-3).sum().item())},
        }
        result["roofline"].update({"achieved": achieved_g, "frac": achieved_g / hbm_peak,
                                   "traffic": None,
                                   "bytes_per_launch": read / L,
                                   "bytes_note": "cold bytes of the units the last step read"})
        result["hbm"] = None
    if args.promotion:
        st = [caches[l].promotion_state() for l in range(L)]
        result["metric"] = ("decode with attention-weighted promotion: context keys/s "
                            "(threshold 0.15, sticky count 3)")
        result["config"]["promotion"] = {"threshold": 0.15, "sticky": 3}
        result["promotion"] = {
            "counted_tokens_last_step": sum(len(u["counts"]) for x in st for u in x),
            "pending_promotions_last_step": sum(len(u["pending"]) for x in st for u in x),
        }
        result["roofline"]["traffic"] = None
        result["roofline"]["bytes_note"] = ("cold and hot bytes plus the cold tokens' logits "
                                            "the attention kernel writes (4 B per token and head)")
    if args.tensor_cache:
        step_gbs = bytes_total / (ms / 1e3) / 1e9
        result["metric"] = ("Tensor Cache decode: context tokens/s (softmax over the ring + "
                            "outer-product memory of the evicted tokens)")
        result["config"]["tensor_cache"] = {"lambda": 0.995, "eta": 0.05, "gate": 0.0,
                                            "memory_per_unit_bytes": 4 * wl.head_dim ** 2}
        result["roofline"] = {"bound": "hbm", "achieved": step_gbs, "peak": hbm_peak, "unit": "GB/s",
                              "frac": step_gbs / hbm_peak, "traffic": None,
                              "kernel": "whole decode step (ring attention, A update, A read)",
                              "peak_kind": peak_kind,
                              "bytes_note": "512 B per ring token + 12 d^2 B of A per unit and layer"}
        result["hbm"] = None
        result["gpu_launches"] = L * (2 + 2 + 1) * args.steps   # no q-prep without cold tokens
    if rank == 0 and world == 1 and not args.no_cpu_baseline and gate_tau is None and \
            not args.tensor_cache and not args.promotion:
        sample = oracle_sample(wl, args.seed, kv_heads=1)
        time_oracle(sample)

        def rate(seconds):
            tt, kk = 0.0, 0
            while tt < seconds:
                dt, k_ = time_oracle(sample)
                tt += dt
                kk += k_
            return kk / tt
        v_all = rate(10.0)
        v_one = None
        try:
            import threadpoolctl
            with threadpoolctl.threadpool_limits(limits=1):
                v_one = rate(5.0)
        except Exception:
            pass
        result["cpu_baseline"] = {
            "value": v_all, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
            "value_1_thread": v_one, "cores_1_thread": 1,
            "sample": f"fp64 oracle decode attention, 1 batch row x 1 kv head (4 q heads) of "
                      f"layer 0 ({wl.cold} cold + {wl.hot} hot tokens), repeated for ~10 s on "
                      f"all threads, then ~5 s with the thread pools limited to one thread"}
    for c in caches:
        c.close()
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# --------------------------------------------------------------------------
# prefill encode: tq_encode_append of 4096-token chunks into one layer handle
# --------------------------------------------------------------------------
ENCODE_METRIC = "prefill encode token-heads/s (K and V of one token of one kv head)"
FP64_PEAK_TFLOPS = 148 * 64 * 2 * 1965e6 / 1e12   # SMs x FP64 FMA/clk x 2 x max SM clock


def run_encode(args, wl):
    import torch

    from compressed_decode_attention_encode_b200 import build as B
    from compressed_decode_attention_encode_b200 import tq
    from compressed_decode_attention_encode_b200.inputs import WORKLOADS  # noqa: F401

    world, rank, local = rank_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        B.build()
    tq.lib()
    chunk = 4096
    nsteps = args.warmup + 2 * args.steps
    cfg = tq.make_config(wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.hot,
                         nsteps * chunk, wl.b_r, wl.b_theta, wl.qjl_bits, seed=args.seed)
    cache = tq.TQCache(cfg, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000 + rank)
    k = gen_kv(wl, 0, args.seed, 0, wl.batch, 0, chunk, dev, gen)
    v = gen_kv(wl, 0, args.seed, 1, wl.batch, 0, chunk, dev, gen)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        cache.encode_append(k, v)
    torch.cuda.synchronize()
    if cache.get_status() != 0:
        raise RuntimeError("device status after warm-up")
    clock = ClockSampler(local)
    clock.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        cache.encode_append(k, v)
    t1.record(stream)
    torch.cuda.synchronize()
    clocks = clock.stop()
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, dev)
    units = wl.batch * wl.num_kv_heads
    per_step = units * chunk                        # token-heads (K and V) per append
    value = job_rate(world, per_step, ms)
    # e2e: the chunk from pinned host memory, then the device status back
    hk = k.cpu().pin_memory()
    hv = v.cpu().pin_memory()
    dk, dv = torch.empty_like(k), torch.empty_like(v)
    hstat = torch.empty(1, dtype=torch.int32).pin_memory()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        cache.encode_append(dk, dv)
        hstat.copy_(cache.ws[:4].view(torch.int32), non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)
    if cache.get_status() != 0:
        raise RuntimeError("device status after timing")
    kc = wl.head_dim // 2 * (wl.b_r + wl.b_theta) // 8
    rec_bytes = 2 * kc + wl.qjl_bits // 8 + 6            # K and V records per token-head
    flops = 2.0 * wl.qjl_bits * wl.head_dim * per_step   # S r in float64, one per key
    achieved = flops / (ms / 1e3) / 1e12
    result = {
        "metric": ENCODE_METRIC, "value": value, "unit": "token-heads/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 decisions, fp16 in", "data": "synthetic",
        "config": {"workload": wl.name + "-prefill-encode", "batch": wl.batch,
                   "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim, "chunk": chunk,
                   "b_r": wl.b_r, "b_theta": wl.b_theta, "qjl_bits": wl.qjl_bits,
                   "l2": "inputs 134 MB per chunk (> L2)"},
        "records_gbs": value * rec_bytes / 1e9,
        "roofline": {"bound": "alu", "achieved": achieved, "peak": FP64_PEAK_TFLOPS,
                     "unit": "TFLOP/s (fp64)", "frac": achieved / FP64_PEAK_TFLOPS, "traffic": None,
                     "kernel": "encode_kernel", "peak_kind": "derived: 148 SMs x 64 FP64 FMA/clk x 1965 MHz",
                     "flop_per_step": flops},
        "e2e": {"value": job_rate(world, per_step, e2e_ms), "unit": "token-heads/s",
                "h2d_bytes_per_step": 2 * k.numel() * 2, "d2h_bytes_per_step": 4,
                "ms_per_step": e2e_ms},
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    cache.close()
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


# --------------------------------------------------------------------------
# vector-search workload (1M x 200 database, 1024 queries, top-10)
# --------------------------------------------------------------------------
SEARCH_METRIC = "estimated inner products/s (vector search, top-10)"


def _search_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return float(json.load(open(p))["bf16_tflops"]), "measured (bf16 cuBLAS burst; fp16 runs at the same rate)"
    return 1590.0, "fallback"


def run_search(args, sw):
    import numpy as np
    import torch
    from compressed_decode_attention_encode_b200 import build as B
    from compressed_decode_attention_encode_b200 import tq
    from compressed_decode_attention_encode_b200.inputs import mixture_centres

    world, rank, local = rank_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        B.build()
    tq.lib()
    gen = torch.Generator(device=dev)
    gen.manual_seed(12345 + rank)
    centres = torch.from_numpy(mixture_centres(sw, args.seed)).to(dev, torch.float32)

    def mixture(count):
        comp = torch.randint(0, sw.components, (count,), generator=gen, device=dev)
        x = centres[comp] + torch.randn((count, sw.dim), generator=gen, device=dev)
        return (x / x.norm(dim=1, keepdim=True)).contiguous()

    index = tq.TQVecIndex(sw.dim, sw.n, sw.b_r, sw.b_theta, sw.qjl_bits, seed=args.seed,
                          max_queries=sw.n_queries, device=dev)
    for s in range(0, sw.n, 200_000):
        index.encode(mixture(min(200_000, sw.n - s)), start=s)
    q = mixture(sw.n_queries)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        index.search(q, k=sw.k)
    torch.cuda.synchronize()
    clock = ClockSampler(local)
    clock.start()
    time.sleep(0.3)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        index.search(q, k=sw.k)
    t1.record(stream)
    torch.cuda.synchronize()
    clocks = clock.stop()
    ms = t0.elapsed_time(t1) / args.steps
    ms = max_over_ranks(ms, dev)
    ips = sw.n_queries * sw.n
    value = job_rate(world, ips, ms)
    # e2e: queries from pinned host memory, results back to the host
    hq = q.cpu().pin_memory()
    hs = torch.empty((sw.n_queries, sw.k), dtype=torch.float32).pin_memory()
    hi = torch.empty((sw.n_queries, sw.k), dtype=torch.int32).pin_memory()
    dq = torch.empty_like(q)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        dq.copy_(hq, non_blocking=True)
        sc, ix = index.search(dq, k=sw.k)
        hs.copy_(sc, non_blocking=True)
        hi.copy_(ix, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)
    flops = 2.0 * ips * (256 + sw.qjl_bits)        # algorithmic: polar d=256 + m sign terms
    peak, peak_kind = _search_peak()
    achieved = flops / (ms / 1e3) / 1e12
    result = {
        "metric": SEARCH_METRIC, "value": value, "unit": "inner products/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16-in/f32-acc", "data": "synthetic",
        "config": {"workload": sw.name, "n": sw.n, "dim": sw.dim, "queries": sw.n_queries,
                   "k": sw.k, "b_r": sw.b_r, "b_theta": sw.b_theta, "qjl_bits": sw.qjl_bits,
                   "l2": "database codes 164 MB (> L2) read once per search"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None, "kernel": "tq_ip_search (q-prep, search, merge)",
                     "peak_kind": peak_kind, "flop_per_step": flops},
        "e2e": {"value": job_rate(world, ips, e2e_ms), "unit": "inner products/s",
                "h2d_bytes_per_step": q.numel() * 4, "d2h_bytes_per_step": sw.n_queries * sw.k * 8,
                "ms_per_step": e2e_ms},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import tq_oracle as O
        from compressed_decode_attention_encode_b200.inputs import mixture_queries, mixture_vectors
        nb, nqs = 50_000, 16
        x = mixture_vectors(sw, args.seed, 0, nb).astype(np.float64)
        d = 256
        signs, S = O.rotation_signs(args.seed, d), O.qjl_matrix(args.seed, sw.qjl_bits, d)
        codes = O.encode(x, signs, S, sw.b_r, sw.b_theta)
        qs = mixture_queries(sw, args.seed, nqs).astype(np.float64)
        def rate(seconds):
            tt, reps = 0.0, 0
            while tt < seconds:
                t_ = time.perf_counter()
                sc = O.ip_scores(qs, signs, S, codes)
                O.top_k(sc, sw.k)
                tt += time.perf_counter() - t_
                reps += 1
            return reps * nb * nqs / tt
        v_all = rate(10.0)
        v_one = None
        try:
            import threadpoolctl
            with threadpoolctl.threadpool_limits(limits=1):
                v_one = rate(5.0)
        except Exception:
            pass
        result["cpu_baseline"] = {
            "value": v_all, "unit": "inner products/s", "cores": oracle_threads(), "kind": "oracle",
            "value_1_thread": v_one, "cores_1_thread": 1,
            "sample": f"fp64 oracle scores + top-10 of {nqs} queries over {nb} encoded vectors, repeated "
                      f"~10 s on all threads, then ~5 s with the thread pools limited to one thread"}
    index.close()
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    from compressed_decode_attention_encode_b200.inputs import SEARCH_WORKLOADS, WORKLOADS
    if args.workload in SEARCH_WORKLOADS:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the vector-search reference arm "
                              "is not timed; run the default workload"}))
            return
        run_search(args, SEARCH_WORKLOADS[args.workload])
        return
    wl = WORKLOADS[args.workload]
    if args.encode:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the encode reference arm is not "
                              "timed; run the default workload"}))
            return
        run_encode(args, wl)
        return
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_gpu(args, wl)


if __name__ == "__main__":
    main()
