#!/usr/bin/env python
"""Benchmark of one MLA decode step on B200 through libmla's C ABI.

A step is the whole hot path over one batch: append the new tokens' latent
rows (mla_append_latent), absorb the query (mla_absorb_q), split-KV
attention over the latent cache (mla_decode_attention) and the combine +
W_UV up-projection (mla_decode_combine).  The default workload is the
V3-shaped batch-64 x 4096 decode (128 heads, d_c 512, d_R 64, paged cache of
64-token blocks with a permuted block table).

Prints one JSON line on rank 0.  Under torchrun each rank runs the same
workload on its own GPU (independent batches, no data-path collective);
timings are the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mla|reference] [--config NAME]
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode TFLOP/s & latent-KV GB/s vs B200 roofline (bf16, V3 shapes)"
UNIT = "TFLOP/s"


def _args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="mla", choices=["mla", "reference"])
    p.add_argument("--config", default="v3_bf16")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-prefill", action="store_true", help="skip the prefill measurement (single-GPU runs only)")
    p.add_argument("--no-configs", action="store_true",
                   help="skip the other decode workloads (V2-Lite, V3 ragged, V3 long; single-GPU runs only)")
    p.add_argument("--repeats", type=int, default=10,
                   help="extra blocks of --steps steps timed after the headline block, for the spread")
    p.add_argument("--only", default="all", choices=["all", "decode", "prefill", "configs"],
                   help="run one part alone (for profiler captures of a single kernel family)")
    p.add_argument("--prefill-seqlens", default=None,
                   help="comma-separated prefill sequence lengths instead of the workload's 8192,8192 (profiling)")
    return p.parse_args()


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        j = json.load(open(path))
        return dict(hbm_gbs=j["hbm_gbs"], bf16_tflops=j["bf16_tflops"],
                    bf16_tflops_sustained=j.get("bf16_tflops_sustained"), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def _config_json(case, n_gpus):
    d = case.dims
    sl = case.seqlens
    return {"workload": f"{case.name}: MLA decode step (append + absorb + split-KV attention + combine/W_UV)",
            "batch_per_gpu": case.batch, "global_batch": case.batch * n_gpus, "n_q": case.n_q,
            "seqlens": list(sl), "heads": d.n_heads, "d_c": d.d_c, "d_rope": d.d_rope, "d_nope": d.d_nope,
            "d_v": d.d_v, "d_model": d.d_model, "block_size": case.block_size,
            "block_table": "seeded random permutation" if case.paged else "contiguous",
            "parallelism": f"replicas x{n_gpus} (independent batches per GPU)",
            "l2": "inputs larger than L2: the latent cache streamed each step exceeds the 126 MB L2"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.p:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()

    def summary(self):
        self.f.flush()
        rows = []
        try:
            for line in open(self.f.name):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        finally:
            os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# Sources an attention kernel's DRAM traffic depends on; a recorded figure holds only while they are unchanged.
_TRAFFIC_SOURCES = {"decode_tc.cu": ("decode_tc.cu", "decode_tc.cuh", "sm100.cuh", "common.cuh", "kernels.cuh"),
                    "attn_simt.cu": ("attn_simt.cu", "common.cuh", "kernels.cuh")}


def traffic_source_hash(kernel_file):
    """Hash of the kernel's sources with // comments and blank lines removed (comment edits keep the figure)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in _TRAFFIC_SOURCES[kernel_file]:
        text = open(os.path.join(ROOT, "mla_latent_kv_40_b200", "csrc", f), encoding="utf-8").read()
        code = [re.sub(r"\s*//.*$", "", ln).rstrip() for ln in text.splitlines()]
        h.update("\n".join(ln for ln in code if ln).encode())
    return h.hexdigest()[:16]


def _traffic_for(kernel_file):
    """dram bytes per launch from the committed ncu summary, if the kernel's sources are unchanged since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    ent = json.load(open(path)).get(kernel_file)
    if not ent or ent.get("source_sha256_16") != traffic_source_hash(kernel_file):
        return None
    return ent.get("dram_bytes_per_launch")


def cpu_baseline(case, target_s=12.0, inp=None):
    """The fp64 oracle, as it stands, on a bounded sample of the same workload."""
    import oracle
    from workloads import make_decode_inputs
    try:
        from threadpoolctl import threadpool_info
        cores = max([t.get("num_threads", 1) for t in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    if inp is None:
        inp = make_decode_inputs(case)
    d = case.dims
    H = d.n_heads
    S0 = int(inp["seqlens"][0])
    heads, t0, done = [], time.time(), 0
    flops = 0
    while time.time() - t0 < target_s and done < H:
        picks = [(0, j, done) for j in range(case.n_q)]
        oracle.decode(d, inp["q_nope"], inp["q_pe"], inp["pool"], inp["block_table"], inp["block_size"],
                      inp["seqlens"], inp["w_uk"], inp["w_uv"], picks=picks)
        for j in range(case.n_q):
            vis = S0 - case.n_q + j + 1
            flops += vis * (2 * (d.d_c + d.d_rope) + 2 * d.d_c) + 2 * d.d_nope * d.d_c + 2 * d.d_c * d.d_v
        done += 1
    el = time.time() - t0
    return {"value": flops / el / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"sequence 0 (S={S0}), {done} of {H} heads, all {case.n_q} query tokens; fp64 unabsorbed "
                      f"form, FLOPs counted as absorbed-form work; {el:.1f} s"}


def rank_info():
    """(rank, world size, local rank) of this process, as torchrun sets them (1 process by default)."""
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks_of(x, world, device):
    """The largest x over all ranks (one all-reduce); x itself on a single process."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(step_flops_per_rank, world, ms_max):
    """Whole-job TFLOP/s: every rank does one step of the same work; the slowest rank sets the time."""
    return step_flops_per_rank * world / (ms_max * 1e-3) / 1e12


def run_reference(args):
    rank, _, _ = rank_info()
    if rank != 0:
        return
    from workloads import DECODE_CASES, make_decode_inputs
    case = DECODE_CASES[args.config]
    inp = make_decode_inputs(case)
    vals, last = [], None
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(case, target_s=2.0, inp=inp)
        if i >= args.warmup:
            vals.append(r["value"])
            last = r
    v = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1) cache rows and queries)",
            "config": _config_json(case, 1),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": last["cores"], "kind": "oracle",
                             "sample": "each step: " + last["sample"]},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def measure_prefill(mla, torch, peaks, seqlens=None, calls=10):
    """The causal prefill (the secondary path row) on its workload: V3 shapes, 2 sequences x 8192 tokens,
    128 heads, 64-token pages.  Device-side seeded inputs; 2 warm-up calls, then `calls` timed calls of
    mla_prefill, each bracketed by CUDA events (median and spread reported)."""
    import dataclasses
    from workloads import PREFILL_CASES, prefill_flops
    case = PREFILL_CASES["v3_prefill_bf16"]
    if seqlens:
        case = dataclasses.replace(case, seqlens=tuple(seqlens))
    d = case.dims
    B, T = len(case.seqlens), sum(case.seqlens)
    g = torch.Generator(device="cuda").manual_seed(case.seed)
    dims = mla.make_dims(d.n_heads, d.d_c, d.d_rope, d.d_nope, d.d_v, d.d_model, case.block_size, d.dtype)
    cu = torch.zeros(B + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(case.seqlens, dtype=torch.int32), 0)
    mbps = max((s_ + case.block_size - 1) // case.block_size for s_ in case.seqlens)
    num_blocks = B * mbps
    bt = torch.randperm(num_blocks, generator=torch.Generator().manual_seed(case.seed)).to(torch.int32).view(B, mbps)
    pool = torch.randn(num_blocks * case.block_size, d.d_c + d.d_rope, generator=g, device="cuda").to(torch.bfloat16)
    q_nope = torch.randn(T, d.n_heads, d.d_nope, generator=g, device="cuda").to(torch.bfloat16)
    q_pe = torch.randn(T, d.n_heads, d.d_rope, generator=g, device="cuda").to(torch.bfloat16)
    w_uk = (torch.randn(d.n_heads, d.d_c, d.d_nope, generator=g, device="cuda") / d.d_c ** 0.5).to(torch.bfloat16)
    w_uv = (torch.randn(d.n_heads, d.d_c, d.d_v, generator=g, device="cuda") / d.d_c ** 0.5).to(torch.bfloat16)
    out = torch.empty(T, d.n_heads, d.d_v, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(T, d.n_heads, dtype=torch.float32, device="cuda")
    ms_ = max(case.seqlens)
    ws = mla.alloc_workspace(mla.mla_prefill_workspace_size(dims, B, T, ms_))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    cu_d, bt_d = cu.cuda(), bt.cuda()

    def run():
        mla.mla_prefill(dims, cu_d, ms_, q_nope, q_pe, pool, pool[:, d.d_c:], bt_d, mbps, num_blocks, w_uk, w_uv,
                        out, lse, ws, st)

    for _ in range(2):
        run()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(calls)]
    for a, b in evs:
        a.record()
        run()
        b.record()
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} in the prefill")
    times = sorted(a.elapsed_time(b) for a, b in evs)
    ms = statistics.median(times)
    fl = prefill_flops(d, list(case.seqlens))
    t_roof = fl["total"] / (peaks["bf16_tflops"] * 1e12)
    del q_nope, q_pe, ws, out
    torch.cuda.empty_cache()
    return {"workload": f"v3_prefill_bf16: causal prefill, {B} x {max(case.seqlens)} tokens, 128 heads, keys 192, "
                        "values 128",
            "ms": ms, "ms_min": times[0], "ms_max": times[-1], "calls": calls,
            "tflops": fl["total"] / (ms * 1e-3) / 1e12, "flops": fl["total"],
            "roofline": {"bound": "tensor", "t_us": t_roof * 1e6, "frac": t_roof / (ms * 1e-3),
                         "peak_tflops": peaks["bf16_tflops"], "peak_source": peaks["source"]}}


def measure_decode_configs(mla, torch, peaks, steps, names=("v2lite_bf16", "v3_ragged_bf16", "v3_long_bf16")):
    """The other decode workloads at full size, each timed through one public call per step
    (mla_decode: absorb + split-KV attention + combine/W_UV), inputs resident on the device.
    Reported per workload: TFLOP/s, latent-KV GB/s, decode tokens/s and the fraction of the roofline
    max(latent bytes / HBM peak, decode FLOPs / bf16 peak)."""
    from workloads import DECODE_CASES, decode_flops, latent_bytes, make_decode_inputs_device
    res = {}
    for name in names:
        case = DECODE_CASES[name]
        d = case.dims
        inp = make_decode_inputs_device(case)
        tiled = d.dtype == "bf16" and case.block_size % 64 == 0 and (d.d_c + d.d_rope) % 64 == 0
        dims = mla.make_dims(d.n_heads, d.d_c, d.d_rope, d.d_nope, d.d_v, d.d_model, case.block_size, d.dtype,
                             rope_base=d.rope_base, rms_eps=d.rms_eps, cache_layout=1 if tiled else 0)
        pool = inp["pool"]
        if tiled:
            packed = torch.empty_like(pool)
            mla.mla_cache_pack(dims, pool, packed)
            torch.cuda.synchronize()
            del pool
            inp["pool"] = pool = packed
        c_kv, k_pe = (pool, pool) if tiled else (pool, pool[:, d.d_c:])
        B, n_q, H = case.batch, case.n_q, d.n_heads
        sl = inp["seqlens"]
        max_seqlen = int(sl.max())
        bt = inp["block_table"].cuda() if case.paged else None
        sl_d = sl.cuda()
        ws = mla.alloc_workspace(mla.mla_decode_workspace_size(dims, B, n_q, max_seqlen))
        out = torch.empty((B, n_q, H, d.d_v), dtype=d.torch_dtype, device="cuda")
        lse = torch.empty((B, n_q, H), dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")

        def run():
            mla.mla_decode(dims, inp["q_nope"], inp["q_pe"], c_kv, k_pe, bt, inp["max_blocks_per_seq"],
                           inp["num_blocks"], sl_d, max_seqlen, inp["w_uk"], inp["w_uv"], out, lse, ws, st)

        for _ in range(3):
            run()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            run()
        e1.record()
        torch.cuda.synchronize()
        if int(st.item()) != 0:
            raise RuntimeError(f"device status {int(st.item())} in {name}")
        ms = e0.elapsed_time(e1) / steps
        fl = decode_flops(d, sl.tolist(), n_q)["total"]
        lb = latent_bytes(d, sl.tolist())
        t_roof = max(lb / (peaks["hbm_gbs"] * 1e9), fl / (peaks["bf16_tflops"] * 1e12))
        res[name] = {"ms": ms, "tflops": fl / (ms * 1e-3) / 1e12, "latent_kv_gbs": lb / (ms * 1e-3) / 1e9,
                     "decode_tokens_per_s": B * n_q / (ms * 1e-3), "roofline_us": t_roof * 1e6,
                     "roofline_frac": t_roof / (ms * 1e-3), "batch": B, "n_q": n_q,
                     "seqlens": list(case.seqlens), "latent_bytes": lb, "flops": fl, "call": "mla_decode"}
        del inp, pool, c_kv, k_pe, ws, out
        torch.cuda.empty_cache()
    return res


def measure_absorbed(mla, torch, peaks, steps, d_cq=1536):
    """Decode from hidden states with folded weights (mla_decode_absorbed) on the V3 batch-64 x 4096
    workload, d_cq = 1536: c_Q = h W_DQ, latent and RoPE queries through W_UQK and W_QR, attention, the
    merge, and the output through W_UVO, per call (the weight folds run once, untimed).  Roofline: the
    four weights and the latent cache read once against HBM, or the products' FLOPs against bf16."""
    from workloads import DECODE_CASES, make_decode_inputs_device, make_query_path_inputs, latent_bytes, decode_flops
    case = DECODE_CASES["v3_bf16"]
    d = case.dims
    inp = make_decode_inputs_device(case)
    qp = {k: v.cuda() for k, v in make_query_path_inputs(case, d_cq, seed=case.seed + 1).items()}
    dims = mla.make_dims(d.n_heads, d.d_c, d.d_rope, d.d_nope, d.d_v, d.d_model, case.block_size, d.dtype,
                         rope_base=d.rope_base, rms_eps=d.rms_eps, cache_layout=1)
    packed = torch.empty_like(inp["pool"])
    mla.mla_cache_pack(dims, inp["pool"], packed)
    torch.cuda.synchronize()
    inp["pool"] = packed
    B, n_q, H, D = case.batch, case.n_q, d.n_heads, d.d_model
    w_uqk = torch.empty(H, d_cq, d.d_c, dtype=d.torch_dtype, device="cuda")
    w_uvo = torch.empty(H, d.d_c, D, dtype=d.torch_dtype, device="cuda")
    mla.mla_fold_query_weights(dims, qp["w_uq"], inp["w_uk"], w_uqk)
    mla.mla_fold_output_weights(dims, inp["w_uv"], qp["w_o"], w_uvo)
    w_qr = qp["w_qr"].reshape(d_cq, H * d.d_rope).contiguous()
    sl = inp["seqlens"]
    ws = mla.alloc_workspace(mla.mla_decode_absorbed_workspace_size(dims, d_cq, B, n_q, int(sl.max())))
    out = torch.empty((B, n_q, D), dtype=d.torch_dtype, device="cuda")
    lse = torch.empty((B, n_q, H), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    bt, sl_d = inp["block_table"].cuda(), sl.cuda()

    def run():
        mla.mla_decode_absorbed(dims, qp["h"], qp["w_dq"], w_uqk, w_qr, packed, packed, bt, inp["max_blocks_per_seq"],
                                inp["num_blocks"], sl_d, int(sl.max()), w_uvo, out, lse, ws, st)

    for _ in range(3):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        run()
    e1.record()
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} in the absorbed decode")
    ms = e0.elapsed_time(e1) / steps
    T = B * n_q
    w_bytes = 2 * (D * d_cq + H * d_cq * d.d_c + d_cq * H * d.d_rope + H * d.d_c * D)
    seqlens = [int(x) for x in sl]
    bytes_ = w_bytes + latent_bytes(d, seqlens)
    flops = 2 * T * (D * d_cq + H * d_cq * d.d_c + d_cq * H * d.d_rope + H * d.d_c * D) + decode_flops(d, seqlens, n_q)["attention"]
    t_roof = max(bytes_ / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12))
    res = {"workload": f"v3_bf16 from hidden states, d_cq {d_cq}, folded W_UQK and W_UVO", "ms": ms,
           "tflops": flops / (ms * 1e-3) / 1e12, "gbs": bytes_ / (ms * 1e-3) / 1e9, "bytes": bytes_,
           "decode_tokens_per_s": T / (ms * 1e-3), "roofline_us": t_roof * 1e6, "roofline_frac": t_roof / (ms * 1e-3),
           "call": "mla_decode_absorbed (c_Q, queries, attention, merge, output through W_UVO)"}
    del inp, packed, ws, w_uqk, w_uvo, qp
    torch.cuda.empty_cache()
    return res


def measure_sparse(mla, torch, peaks, steps, topk=2048):
    """Sparse decode (mla_decode_sparse) on the V3 batch-64 x 4096 workload with `topk` tokens selected
    per query token (seeded random distinct positions): the gather of the selected rows, absorption,
    attention over them and the combine, per call.  Roofline: the selected rows read once
    (gathered, then streamed) against HBM, or the attention FLOPs over the selected keys."""
    import numpy as np
    from workloads import DECODE_CASES, make_decode_inputs_device
    case = DECODE_CASES["v3_bf16"]
    d = case.dims
    inp = make_decode_inputs_device(case)
    dims = mla.make_dims(d.n_heads, d.d_c, d.d_rope, d.d_nope, d.d_v, d.d_model, case.block_size, d.dtype,
                         rope_base=d.rope_base, rms_eps=d.rms_eps, cache_layout=1)
    packed = torch.empty_like(inp["pool"])
    mla.mla_cache_pack(dims, inp["pool"], packed)
    torch.cuda.synchronize()
    inp["pool"] = packed
    B, n_q, H = case.batch, case.n_q, d.n_heads
    sl = inp["seqlens"]
    g = np.random.default_rng(case.seed)
    sel = np.stack([np.stack([g.permutation(int(sl[b]) - n_q + j + 1)[:topk] for j in range(n_q)]) for b in range(B)])
    sel_d = torch.from_numpy(sel.astype(np.int32)).cuda()
    ws = mla.alloc_workspace(mla.mla_decode_sparse_workspace_size(dims, B, n_q, topk))
    out = torch.empty((B, n_q, H, d.d_v), dtype=d.torch_dtype, device="cuda")
    lse = torch.empty((B, n_q, H), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    bt, sl_d = inp["block_table"].cuda(), sl.cuda()

    def run():
        mla.mla_decode_sparse(dims, inp["q_nope"], inp["q_pe"], packed, packed, bt, inp["max_blocks_per_seq"],
                              inp["num_blocks"], sl_d, int(sl.max()), sel_d, inp["w_uk"], inp["w_uv"], out, lse, ws, st)

    for _ in range(3):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        run()
    e1.record()
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} in the sparse decode")
    ms = e0.elapsed_time(e1) / steps
    keys = B * n_q * topk
    W = d.d_c + d.d_rope
    att_flops = keys * H * (2 * W + 2 * d.d_c)
    flops = att_flops + B * n_q * H * 2 * d.d_c * (d.d_nope + d.d_v)
    sel_bytes = keys * W * 2
    t_roof = max(sel_bytes / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12))
    res = {"workload": f"v3_bf16 with {topk} selected tokens per query", "ms": ms,
           "tflops": flops / (ms * 1e-3) / 1e12, "selected_kv_gbs": sel_bytes / (ms * 1e-3) / 1e9,
           "decode_tokens_per_s": B * n_q / (ms * 1e-3), "roofline_us": t_roof * 1e6,
           "roofline_frac": t_roof / (ms * 1e-3), "call": "mla_decode_sparse (gather + absorb + attention + combine)"}
    del inp, packed, ws
    torch.cuda.empty_cache()
    return res


def measure_split_kv(mla, torch, peaks, steps, world=4):
    """The V3 long workload (4 x 131072 keys, 2 query tokens) split into `world` key ranges, each
    range's partial (mla_decode_partial) timed alone on this GPU, as one of `world` devices would
    run it, and the merge of the `world` partials (mla_merge_partials).  The all-gather between
    devices (world x 1 MB here) is not part of it: every run here has one GPU."""
    import importlib
    sharded = importlib.import_module("mla_latent_kv_40_b200.sharded")
    from workloads import DECODE_CASES, decode_flops, latent_bytes, make_decode_inputs_device
    case = DECODE_CASES["v3_long_bf16"]
    d = case.dims
    inp = make_decode_inputs_device(case)
    dims = mla.make_dims(d.n_heads, d.d_c, d.d_rope, d.d_nope, d.d_v, d.d_model, case.block_size, d.dtype,
                         rope_base=d.rope_base, rms_eps=d.rms_eps, cache_layout=1)
    packed = torch.empty_like(inp["pool"])
    mla.mla_cache_pack(dims, inp["pool"], packed)
    torch.cuda.synchronize()
    inp["pool"] = packed
    B, n_q, H = case.batch, case.n_q, d.n_heads
    sl = inp["seqlens"]
    max_seqlen = int(sl.max())
    bt, sl_d = inp["block_table"].cuda(), sl.cuda()
    ws = mla.alloc_workspace(mla.mla_decode_workspace_size(dims, B, n_q, max_seqlen))
    o_parts = torch.empty((world, B, n_q, H, d.d_c), dtype=d.torch_dtype, device="cuda")
    l_parts = torch.empty((world, B, n_q, H), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ranges = sharded.kv_shard_ranges(max_seqlen, world)
    part_ms = []
    for r, (k0, k1) in enumerate(ranges):
        def run():
            mla.mla_decode_partial(dims, inp["q_nope"], inp["q_pe"], packed, packed, bt, inp["max_blocks_per_seq"],
                                   inp["num_blocks"], sl_d, max_seqlen, k0, k1, inp["w_uk"], o_parts[r], l_parts[r],
                                   ws, st)
        for _ in range(3):
            run()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            run()
        e1.record()
        torch.cuda.synchronize()
        part_ms.append(e0.elapsed_time(e1) / steps)
    out = torch.empty((B, n_q, H, d.d_v), dtype=d.torch_dtype, device="cuda")
    lse = torch.empty((B, n_q, H), dtype=torch.float32, device="cuda")
    mws = mla.alloc_workspace(mla.mla_merge_workspace_size(dims, B, n_q, world))
    for _ in range(3):
        mla.mla_merge_partials(dims, o_parts, l_parts, inp["w_uv"], out, lse, mws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        mla.mla_merge_partials(dims, o_parts, l_parts, inp["w_uv"], out, lse, mws)
    e1.record()
    torch.cuda.synchronize()
    merge_ms = e0.elapsed_time(e1) / steps
    if int(st.item()) != 0:
        raise RuntimeError(f"device status {int(st.item())} in the split decode")
    fl = decode_flops(d, sl.tolist(), n_q)["total"]
    lb = latent_bytes(d, sl.tolist())
    per_dev = max(part_ms) + merge_ms
    t_roof = max(lb / world / (peaks["hbm_gbs"] * 1e9), fl / world / (peaks["bf16_tflops"] * 1e12))
    res = {"workload": f"v3_long_bf16 split over {world} key ranges", "ranges": ranges, "partial_ms": part_ms,
           "merge_ms": merge_ms, "ms_per_device": per_dev, "tflops_per_device": fl / world / (per_dev * 1e-3) / 1e12,
           "roofline_us_per_device": t_roof * 1e6, "roofline_frac": t_roof / (per_dev * 1e-3),
           "note": "per device: its own range's partial plus the merge; the all-gather is not included"}
    del inp, packed, ws
    torch.cuda.empty_cache()
    return res


def run_mla(args):
    import torch
    import torch.distributed as dist
    rank, world, local = rank_info()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    import mla_latent_kv_40_b200 as mla
    from workloads import DECODE_CASES, append_flops, decode_flops, latent_bytes, make_decode_step_inputs

    if args.only in ("prefill", "configs"):   # profiling helpers: one kernel family alone, no JSON contract
        peaks = _peaks()
        if args.only == "prefill":
            sl = [int(x) for x in args.prefill_seqlens.split(",")] if args.prefill_seqlens else None
            print(json.dumps({"prefill": measure_prefill(mla, torch, peaks, sl, calls=max(args.steps, 1))}), flush=True)
        else:
            print(json.dumps({"configs": measure_decode_configs(mla, torch, peaks, max(args.steps, 1))}), flush=True)
        return

    case = DECODE_CASES[args.config]
    d = case.dims
    inp = make_decode_step_inputs(case)
    # bf16 pools with 64-token pages use the tiled page layout (pages move by contiguous bulk copies);
    # the seeded row pool is packed into it once, before anything is timed.
    tiled = d.dtype == "bf16" and case.block_size % 64 == 0 and (d.d_c + d.d_rope) % 64 == 0
    dims = mla.make_dims(d.n_heads, d.d_c, d.d_rope, d.d_nope, d.d_v, d.d_model, case.block_size, d.dtype,
                         rope_base=d.rope_base, rms_eps=d.rms_eps, cache_layout=1 if tiled else 0)
    dev = {k: inp[k].cuda() for k in ("pool", "block_table", "seqlens", "q_nope", "q_pe", "w_uk", "w_uv", "h_new",
                                      "w_dkv", "w_kr", "gamma", "seq_idx", "pos")}
    if tiled:
        packed = torch.empty_like(dev["pool"])
        mla.mla_cache_pack(dims, dev["pool"], packed)
        torch.cuda.synchronize()
        dev["pool"] = packed
    B, n_q, H = case.batch, case.n_q, d.n_heads
    max_seqlen = int(inp["seqlens"].max())
    T = B * n_q
    pool = dev["pool"]
    c_kv, k_pe = (pool, pool) if tiled else (pool, pool[:, d.d_c:])
    bt = dev["block_table"] if case.paged else None
    ws = mla.alloc_workspace(mla.mla_decode_workspace_size(dims, B, n_q, max_seqlen))
    q_abs = torch.empty((B, n_q, H, d.d_c + d.d_rope), dtype=d.torch_dtype, device="cuda")
    out = torch.empty((B, n_q, H, d.d_v), dtype=d.torch_dtype, device="cuda")
    lse = torch.empty((B, n_q, H), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    app_ws_bytes = mla.mla_append_workspace_size(dims, T)
    app_ws = mla.alloc_workspace(app_ws_bytes) if app_ws_bytes else None

    # The append (cache write of the new tokens) and the query absorption are independent: the
    # append runs on a side stream, and the attention, which reads the new tokens, waits for it.
    side = torch.cuda.Stream()
    appended = torch.cuda.Event()

    def append():
        side.wait_stream(stream)   # after everything already queued (the previous step's readers)
        mla.mla_append_latent(dims, dev["h_new"], dev["w_dkv"], dev["w_kr"], dev["gamma"], dev["seq_idx"],
                              dev["pos"], c_kv, k_pe, bt, B, inp["max_blocks_per_seq"], inp["num_blocks"], status,
                              workspace=app_ws, stream=side)
        appended.record(side)

    def step(ev=None):
        append()
        mla.mla_absorb_q(dims, dev["q_nope"], dev["q_pe"], dev["w_uk"], dev["seqlens"], q_abs)
        stream.wait_event(appended)
        if ev is not None:
            ev[0].record(stream)
        mla.mla_decode_attention(dims, q_abs, c_kv, k_pe, bt, inp["max_blocks_per_seq"], inp["num_blocks"],
                                 dev["seqlens"], max_seqlen, ws, status)
        if ev is not None:
            ev[1].record(stream)
        mla.mla_decode_combine(dims, B, n_q, dev["seqlens"], max_seqlen, dev["w_uv"], out, lse, ws)


    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return max_over_ranks_of(x, world, "cuda")

    def timed_block(instrumented):
        """Exactly --steps steps between a barrier + synchronize on each side: (ms per step, attention ms
        per launch or None), each the max over ranks.  An instrumented block records events around every
        attention launch; those events cut the programmatic overlap of the attention kernel with its
        neighbours (~4 us a step), so the headline block runs without them."""
        att_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)] if instrumented else [None] * args.steps
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(args.steps):
            step(att_ev[i])
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        att = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in att_ev)) if instrumented else None
        return max_over_ranks(e0.elapsed_time(e1) / args.steps), att

    # The headline block (plain steps), then --repeats (at least one) blocks of the same steps with the
    # attention launches bracketed by events, for the attention kernel's duration and the spread; the
    # clocks are sampled across all of them.
    # The W warm-up steps run inside the sampler's context, right before the timed blocks (the sampler
    # start leaves the GPU idle for a moment).
    with ClockSampler(local) as clk:
        for _ in range(max(args.warmup, 3)):
            step()
        torch.cuda.synchronize()
        if int(status.item()) != 0:
            raise RuntimeError(f"device status {int(status.item())} during warm-up")
        ms, _ = timed_block(False)
        reps = [timed_block(True) for _ in range(max(args.repeats, 1))]
    clocks = clk.summary()
    all_ms = sorted([ms] + [r[0] for r in reps])
    all_att = sorted(r[1] for r in reps)
    att_ms = statistics.median(all_att)

    # The same step through the single public decode call: append, then mla_decode (absorb + attention +
    # combine/W_UV in one call) on one stream.
    dec_ws = mla.alloc_workspace(mla.mla_decode_workspace_size(dims, B, n_q, max_seqlen))

    def api_step():
        mla.mla_append_latent(dims, dev["h_new"], dev["w_dkv"], dev["w_kr"], dev["gamma"], dev["seq_idx"],
                              dev["pos"], c_kv, k_pe, bt, B, inp["max_blocks_per_seq"], inp["num_blocks"], status,
                              workspace=app_ws)
        mla.mla_decode(dims, dev["q_nope"], dev["q_pe"], c_kv, k_pe, bt, inp["max_blocks_per_seq"], inp["num_blocks"],
                       dev["seqlens"], max_seqlen, dev["w_uk"], dev["w_uv"], out, lse, dec_ws, status)

    for _ in range(3):
        api_step()
    torch.cuda.synchronize()
    barrier()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(args.steps):
        api_step()
    a1.record(stream)
    torch.cuda.synchronize()
    barrier()
    api_ms = max_over_ranks(a0.elapsed_time(a1) / args.steps)

    # The whole step as one call: mla_decode_step (append of the new tokens and the query absorption
    # in one launch on these shapes, then attention and combine).
    step_ws = mla.alloc_workspace(mla.mla_decode_step_workspace_size(dims, B, n_q, max_seqlen))
    h_step = dev["h_new"].view(B, n_q, -1)

    def fused_step():
        mla.mla_decode_step(dims, h_step, dev["w_dkv"], dev["w_kr"], dev["gamma"], dev["q_nope"], dev["q_pe"], c_kv,
                            k_pe, bt, inp["max_blocks_per_seq"], inp["num_blocks"], dev["seqlens"], max_seqlen,
                            dev["w_uk"], dev["w_uv"], out, lse, step_ws, status)

    for _ in range(3):
        fused_step()
    torch.cuda.synchronize()
    barrier()
    a0.record(stream)
    for _ in range(args.steps):
        fused_step()
    a1.record(stream)
    torch.cuda.synchronize()
    barrier()
    fused_ms = max_over_ranks(a0.elapsed_time(a1) / args.steps)

    # End to end through the public calls a user makes for a step (mla_append_latent, then mla_decode):
    # pinned host inputs in, result out, every step's copies inside the timed region.  The inputs of step i+1 are copied (copy stream) while step i computes, into the other of
    # two device buffer sets, and step i's result goes back (a second copy stream) while step i+1 computes.
    e2e = None
    if not args.no_e2e:
        # The step's inputs sit in ONE pinned host buffer (each at a 256-byte aligned offset) and move
        # with one copy per step into one of two device buffers, whose views are the call arguments.
        in_keys = ("h_new", "q_nope", "q_pe", "seqlens", "seq_idx", "pos")
        offs, nbytes = {}, 0
        for k in in_keys:
            offs[k] = nbytes
            nbytes += (inp[k].numel() * inp[k].element_size() + 255) // 256 * 256
        host_blob = torch.empty(nbytes, dtype=torch.uint8).pin_memory()

        def views(blob):
            return {k: blob[offs[k]:offs[k] + inp[k].numel() * inp[k].element_size()].view(inp[k].dtype)
                    .view(inp[k].shape) for k in in_keys}

        for k, v in views(host_blob).items():
            v.copy_(inp[k])
        host_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
        h2d = nbytes   # the bytes of the one copy (inputs plus alignment padding)
        d2h = host_out[0].numel() * host_out[0].element_size()
        dev_blobs = [torch.empty(nbytes, dtype=torch.uint8, device="cuda") for _ in range(2)]
        e2e_ws = mla.alloc_workspace(mla.mla_decode_workspace_size(dims, B, n_q, max_seqlen))
        bufs = [views(b) for b in dev_blobs]
        outs = [torch.empty_like(out) for _ in range(2)]
        h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
        in_ready = [torch.cuda.Event() for _ in range(2)]
        in_free = [torch.cuda.Event() for _ in range(2)]
        out_ready = [torch.cuda.Event() for _ in range(2)]
        out_read = [torch.cuda.Event() for _ in range(2)]
        for e in in_free + out_read:
            e.record(stream)

        def h2d_copy(i):
            j = i % 2
            h2d_s.wait_event(in_free[j])              # step i-2 no longer reads buffer set j
            with torch.cuda.stream(h2d_s):
                dev_blobs[j].copy_(host_blob, non_blocking=True)
            in_ready[j].record(h2d_s)

        def e2e_step(i, last):
            j = i % 2
            if not last:
                h2d_copy(i + 1)
            x = bufs[j]
            stream.wait_event(in_ready[j])
            stream.wait_event(out_read[j])            # step i-2's result has left outs[j]
            # The calls a user makes for a step: append the new tokens, then one mla_decode.
            mla.mla_append_latent(dims, x["h_new"], dev["w_dkv"], dev["w_kr"], dev["gamma"], x["seq_idx"], x["pos"],
                                  c_kv, k_pe, bt, B, inp["max_blocks_per_seq"], inp["num_blocks"], status,
                                  workspace=app_ws)
            mla.mla_decode(dims, x["q_nope"], x["q_pe"], c_kv, k_pe, bt, inp["max_blocks_per_seq"], inp["num_blocks"],
                           x["seqlens"], max_seqlen, dev["w_uk"], dev["w_uv"], outs[j], lse, e2e_ws, status)
            in_free[j].record(stream)
            out_ready[j].record(stream)
            d2h_s.wait_event(out_ready[j])
            with torch.cuda.stream(d2h_s):
                host_out[j].copy_(outs[j], non_blocking=True)
            out_read[j].record(d2h_s)

        def e2e_run(n):
            f0 = torch.cuda.Event(enable_timing=True)
            f1 = torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            h2d_s.wait_event(f0)
            h2d_copy(0)
            for i in range(n):
                e2e_step(i, i == n - 1)
            stream.wait_stream(d2h_s)                  # the last result is back on the host
            f1.record(stream)
            return f0, f1

        e2e_run(3)
        torch.cuda.synchronize()
        barrier()
        f0, f1 = e2e_run(args.steps)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(f0.elapsed_time(f1) / args.steps)
        e2e = {"h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} in the timed region")

    fl = decode_flops(d, inp["seqlens"].tolist(), n_q)
    step_flops = fl["total"] + append_flops(d, T)
    lat_bytes = latent_bytes(d, inp["seqlens"].tolist())
    peaks = _peaks()
    value = weak_scaling_value(step_flops, world, ms)
    att_gbs = lat_bytes / (att_ms * 1e-3) / 1e9
    # append (projection + finish with a workspace, one fused kernel without), then absorb + attention + combine
    launches_per_step = (2 if app_ws is not None else 1) + mla.mla_decode_launches(dims, n_q)
    t_hbm = lat_bytes / (peaks["hbm_gbs"] * 1e9)
    t_flop = fl["total"] / (peaks["bf16_tflops"] * 1e12)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if d.dtype == "bf16" else "f32",
        "data": "synthetic (seeded N(0,1) latent cache rows and queries, N(0,1)/sqrt(fan_in) weights)",
        "config": _config_json(case, world),
        "latent_kv_gbs": lat_bytes * world / (ms * 1e-3) / 1e9,
        "decode_tokens_per_s": T * world / (ms * 1e-3),
        "step_roofline": {"t_hbm_us": t_hbm * 1e6, "t_tensor_us": t_flop * 1e6,
                          "frac": max(t_hbm, t_flop) / (ms * 1e-3),
                          "note": "roofline time = max(latent bytes / HBM, decode FLOPs / bf16 peak) of measured "
                                  "peaks, over the whole step time"},
        "roofline": {"kernel": "split-KV attention (mla_decode_attention)", "bound": "hbm",
                     "achieved": att_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": att_gbs / peaks["hbm_gbs"],
                     "traffic": _traffic_for("decode_tc.cu" if mla.mla_decode_path(dims, n_q) == mla.PATH_TCGEN05
                                             else "attn_simt.cu"),
                     "peak_source": peaks["source"], "kernel_ms": att_ms,
                     "algorithmic_bytes_per_launch": lat_bytes},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "spread": {"blocks": len(all_ms), "steps_per_block": args.steps,
                   "note": "the first block runs plain steps (the headline); the others bracket every attention "
                           "launch with events (the attention figures), which costs the step ~4 us of overlap",
                   "ms_per_step_median": statistics.median(all_ms), "ms_per_step_min": all_ms[0],
                   "ms_per_step_max": all_ms[-1], "attention_ms_median": statistics.median(all_att),
                   "attention_ms_min": all_att[0], "attention_ms_max": all_att[-1],
                   "attention_frac_median": lat_bytes / (statistics.median(all_att) * 1e-3) / 1e9 / peaks["hbm_gbs"]},
        "api_step": {"calls": "mla_append_latent + mla_decode, one stream", "ms_per_step": api_ms,
                     "tflops": step_flops * world / (api_ms * 1e-3) / 1e12,
                     "roofline_frac": max(t_hbm, t_flop) / (api_ms * 1e-3)},
        "fused_step": {"calls": "mla_decode_step (append + absorption in one launch, attention, combine)",
                       "ms_per_step": fused_ms, "tflops": step_flops * world / (fused_ms * 1e-3) / 1e12,
                       "roofline_frac": max(t_hbm, t_flop) / (fused_ms * 1e-3)},
    }
    if e2e:
        line["e2e"] = {"value": step_flops * world / (e2e["ms_per_step"] * 1e-3) / 1e12, "unit": UNIT,
                       "h2d_bytes_per_step": e2e["h2d_bytes_per_step"], "d2h_bytes_per_step": e2e["d2h_bytes_per_step"],
                       "ms_per_step": e2e["ms_per_step"]}
    del dec_ws, step_ws
    if world == 1 and rank == 0 and not args.no_prefill and args.only == "all":
        line["prefill"] = measure_prefill(mla, torch, peaks)
    if world == 1 and rank == 0 and not args.no_configs and args.only == "all":
        del dev, pool, c_kv, k_pe, ws
        torch.cuda.empty_cache()
        line["configs"] = measure_decode_configs(mla, torch, peaks, max(args.steps, 5))
        line["sparse"] = measure_sparse(mla, torch, peaks, max(args.steps, 5))
        line["absorbed"] = measure_absorbed(mla, torch, peaks, max(args.steps, 5))
        line["split_kv"] = measure_split_kv(mla, torch, peaks, max(args.steps, 5))
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(case)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    args = _args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_mla(args)


if __name__ == "__main__":
    main()
