#!/usr/bin/env python
"""Benchmark of the elastic-depth forward pass of the Dory-shape looped nGPT.

Workload (one B200 per rank): Dory1.0-4B shapes (d 2560, 16/4 heads of 160,
blocks 8/20/8, SwiGLU 10240, vocab 131072), seeded random-init BF16 weights,
batch 1, a 2048-token uniform-random prompt, then greedy decode, last_loop KV
cache, at k = 1, 2 and 4 loops.  A step is one decode step: one token through
embedding, 16 + 20k blocks and the LM head.  The headline value is decode
tokens/s at k = 2 (the recommended default loop count); decode and prefill
tokens/s at every k and their roofline fractions are in "breakdown".

More than one GPU: independent replicas (one per rank, no collective on the
data path); the value is the sum of tokens over ranks / the slowest rank's
time.  `--impl reference` times the CPU oracle on a bounded sample instead.
"""
import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("decode tok/s & prefill tok/s at k=1/2/4 (1 B200); "
          "% of HBM / TC roofline")
PROMPT = 2048
HEADLINE_K = 2


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=4)
    ap.add_argument("--impl", default="dory", choices=["dory", "reference"])
    ap.add_argument("--loops", default="1,2,3,4")
    ap.add_argument("--kv-mode", default="last_loop")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prompt", type=int, default=PROMPT)
    ap.add_argument("--no-long", action="store_true",
                    help="skip the long-context batched-decode workloads")
    ap.add_argument("--long-steps", type=int, default=8)
    ap.add_argument("--no-quant", action="store_true",
                    help="skip the MXFP8 / NVFP4 weight-only models (B=1 at "
                         "2048 context and B=4 at 131072 context, k=2)")
    ap.add_argument("--no-spec", action="store_true",
                    help="skip self-speculative decoding (k=1 draft, k=4 "
                         "verify, 4 drafts per step)")
    ap.add_argument("--no-per-loop", action="store_true",
                    help="skip the per_loop rows of the 2048-token workload")
    ap.add_argument("--profile-decode", type=int, default=0, metavar="K",
                    help="only: prefill, warm up, then one decode step at "
                         "k=K inside the NVTX range 'decode_step' (for ncu)")
    ap.add_argument("--profile-blocks", default="",
                    help="profile runs only: input,recurrent,output block "
                         "counts of a reduced-depth Dory-width model")
    ap.add_argument("--profile-quant", default="", choices=["", "mxfp8", "nvfp4"],
                    help="profile decode runs only: weight format of the "
                         "block projections (context from the synthetic "
                         "cache fill)")
    ap.add_argument("--profile-prefill", type=int, default=0, metavar="K",
                    help="only: one prefill at k=K inside the NVTX range "
                         "'prefill' (for ncu)")
    return ap.parse_args()


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# one ncu capture of the named kernel (profiles/gemv_gateup_dory_full.md),
# valid only for the source it was taken on (sha256 prefix of the file).
NCU_TRAFFIC = {
    "gemv_gateup": ("looped_ngpt_b200/csrc/k_gemv.cu", "12dc52a58b07d94a",
                    (104.955392 + 2.960640) * 1e6),
}


def dram_traffic(kernel):
    import hashlib
    entry = NCU_TRAFFIC.get(kernel)
    if not entry:
        return None
    path, sha, nbytes = entry
    try:
        with open(os.path.join(ROOT, path), "rb") as f:
            cur = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    return nbytes if cur == sha else None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,"
         "clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return
        # the sampler takes a moment to start: let it run before the timed
        # region so that its 50 ms samples fall inside it
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        self.proc.wait()
        self.f.flush()
        rows = []
        with open(self.f.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == 8:
                    rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if r[4 + i].lower().startswith("active")})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(
                    ".", "").isdigit() else None,
                "samples": len(rows), "reasons": reasons}


# ------------------------------------------------------------------ ranks --
def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device(f"cuda:{local}"))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    """The largest of the ranks' values (every rank gets it): the timed
    region of a replica run is as long as its slowest rank."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info()
             if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


# --------------------------------------------------------------- oracle arm --
def arm_config(prompt, world, kv_mode):
    """The workload both arms name in their JSON line."""
    return {"workload": (f"Dory-shape BF16 looped nGPT decode, batch 1 per GPU "
                         f"at a {prompt}-token context, k={HEADLINE_K}, "
                         f"{kv_mode}"),
            "global_batch": world, "seq_len": prompt,
            "parallelism": f"replicas x{world}",
            "l2": "no flush: 12 GB of weights streamed per token > L2"}


def oracle_at_context(w, n_ctx, kv_mode="last_loop", n_loops=HEADLINE_K,
                      extra=64):
    """The oracle holding n_ctx tokens of seeded synthetic context (the same
    counter generator the library's cache fill uses), every slot sized for
    `extra` more tokens."""
    from oracle.model import Model
    from synthetic import DORY
    from synthetic.kvgen import kv_rows
    m = Model(DORY, w, batch=1, kv_mode=kv_mode)
    _, grec, _ = DORY.block_groups()
    pos = np.arange(n_ctx)
    for i in range(DORY.n_blocks):
        per_loop = i in grec and kv_mode == "per_loop"
        for slot in (range(1, n_loops + 1) if per_loop else [0]):
            K = np.zeros((1, DORY.n_kv_heads, n_ctx + extra, DORY.head_dim))
            V = np.zeros_like(K)
            for h in range(DORY.n_kv_heads):
                K[0, h, :n_ctx], V[0, h, :n_ctx] = kv_rows(DORY, 2, i, slot, 0,
                                                          h, pos)
            m.cache[(i, slot)] = (K, V)
    m.n_ctx = n_ctx
    if kv_mode == "per_loop":
        m.n_loops_fixed = n_loops
    return m


def oracle_decode_sample(w, n_loops, n_ctx, tokens=1):
    """Time the oracle on a bounded sample of the decode workload: `tokens`
    greedy decode steps at a context of n_ctx cached tokens."""
    m = oracle_at_context(w, n_ctx, n_loops=n_loops, extra=tokens + 1)
    t0 = time.perf_counter()
    tok = 7
    for _ in range(tokens):
        z = m.decode_step([tok], n_loops)
        tok = int(np.argmax(z[0]))
    dt = time.perf_counter() - t0
    return tokens / dt, dt


# ------------------------------------------------------------------ GPU arm --
# ------------------------------------------------------------------ GPU arm --
def decode_prefill_at(gm, prompt, k, kv_mode, ws, K, W, world, max_ctx,
                      tc_peak, hbm_peak, clocks=None):
    """The 2048-token workload at k loops in one KV mode: the prompt's
    prefill (one warm-up call, one timed, one profiled for FLOPs), then W + K
    greedy decode steps (CUDA-graph replays; the argmax of each step is
    written straight into the token buffer the next step reads), then P
    profiled eager steps (CUDA events around every kernel)."""
    import torch
    ev = lambda: torch.cuda.Event(enable_timing=True)
    cache = gm.new_cache(1, max_ctx, prompt.shape[1], kv_mode=kv_mode,
                         max_loops=k)
    t_pre = None
    for rep in range(3):
        cache.reset()
        if rep == 2:
            gm.profile(True)
        torch.cuda.synchronize()
        e0, e1 = ev(), ev()
        e0.record()
        _, am = gm.prefill(cache, prompt, k, ws)
        e1.record()
        torch.cuda.synchronize()
        if rep == 1:
            t_pre = e0.elapsed_time(e1) / 1e3
    pst = gm.profile_read()
    gm.profile(False)
    pflops = sum(v["flops"] for v in pst.values())
    gm.decode_step(cache, am, k, ws, want_logits=False)
    tok = cache._dec_bufs[0]
    for _ in range(W):
        gm.decode_step(cache, tok, k, ws, argmax=tok, want_logits=False)
    torch.cuda.synchronize()
    barrier(world)
    if clocks:
        clocks.start()
    e0, e1 = ev(), ev()
    e0.record()
    for _ in range(K):
        gm.decode_step(cache, tok, k, ws, argmax=tok, want_logits=False)
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    dt = e0.elapsed_time(e1) / 1e3
    ck = clocks.stop() if clocks else None
    gm.profile(True)
    P = 4
    for _ in range(P):
        gm.decode_step(cache, tok, k, ws, argmax=tok, want_logits=False)
    st = gm.profile_read()
    gm.profile(False)
    assert gm.sync_status() == 0, "device-side check failed"
    bytes_tok = sum(v["bytes"] for v in st.values()) / P
    return dict(
        prefill_tok_s=prompt.shape[1] / t_pre, prefill_flops=pflops,
        prefill_tc_frac=pflops / t_pre / (tc_peak * 1e12),
        decode_tok_s=K / dt, decode_bytes_per_token=bytes_tok,
        decode_hbm_frac=bytes_tok * K / dt / (hbm_peak * 1e9),
        kv_cache_gb=cache.nbytes / 1e9,
        dt=dt, clocks=ck, stats=st, P=P, cache=cache,
        launches=sum(v["launches"] for v in st.values()) / P)


def run_gpu(args, rank, world, local):
    import torch
    import looped_ngpt_b200 as lb
    from synthetic import DORY, make_weights, make_prompt

    hbm_peak, tc_peak, peak_kind = peaks()
    w = make_weights(DORY, seed=0)
    dev = torch.device(f"cuda:{local}")
    gm = lb.DoryModel(DORY, w, device=dev)
    prompt = torch.from_numpy(make_prompt(DORY, 1, args.prompt)).to(dev)
    ks = [int(k) for k in args.loops.split(",")]
    if HEADLINE_K not in ks:
        ks.append(HEADLINE_K)
    K, W = args.steps, args.warmup
    max_ctx = args.prompt + 2 * (W + K) + 16
    ws = gm.workspace(1, args.prompt)
    modes = [args.kv_mode]
    if not args.no_per_loop:
        modes += [m for m in ("last_loop", "per_loop") if m != args.kv_mode]
    out = {}
    headline = None
    for mode in modes:
        rows = {"decode_tok_s": {}, "prefill_tok_s": {}, "decode_hbm_frac": {},
                "prefill_tc_frac": {}, "decode_bytes_per_token": {},
                "prefill_flops": {}, "kv_cache_gb": {}}
        for k in ks:
            head = mode == args.kv_mode and k == HEADLINE_K
            r = decode_prefill_at(gm, prompt, k, mode, ws, K, W, world, max_ctx,
                                  tc_peak, hbm_peak,
                                  Clocks(local) if head else None)
            for key in rows:
                rows[key][f"k{k}"] = r[key]
            if head:
                headline = r
            else:
                del r["cache"]
        out[mode] = rows
    # end-to-end through host buffers at the headline k
    k = HEADLINE_K
    cache = headline["cache"]
    cache.reset()
    _, am = gm.prefill(cache, prompt, k, ws)
    host_tok = torch.empty(1, dtype=torch.int32, pin_memory=True)
    host_out = torch.empty(1, dtype=torch.int32, pin_memory=True)
    host_tok.copy_(am.cpu())
    tok = cache._dec_bufs[0]
    for _ in range(W):
        tok.copy_(host_tok, non_blocking=True)
        gm.decode_step(cache, tok, k, ws, argmax=tok, want_logits=False)
        host_out.copy_(tok, non_blocking=True)
        torch.cuda.synchronize()
        host_tok.copy_(host_out)
    torch.cuda.synchronize()
    barrier(world)
    t0 = time.perf_counter()
    for _ in range(K):
        tok.copy_(host_tok, non_blocking=True)
        gm.decode_step(cache, tok, k, ws, argmax=tok, want_logits=False)
        host_out.copy_(tok, non_blocking=True)
        torch.cuda.synchronize()
        host_tok.copy_(host_out)
    e2e_dt = time.perf_counter() - t0
    barrier(world)
    del cache, headline["cache"]
    torch.cuda.empty_cache()
    if not args.no_spec:
        sp = run_spec(gm, prompt)
        ar = out.get("per_loop", {}).get("decode_tok_s", {}).get("k4")
        if ar:
            sp["autoregressive_k4_per_loop_tok_s"] = ar
            sp["speedup_vs_autoregressive"] = sp["tok_s"] / ar
            sp["break_even_tokens_per_step"] = sp["ms_per_step"] / 1e3 * ar
        out["self_speculative_b1_k1_draft_k4_verify"] = sp
    if not args.no_long:
        out["long_context"] = run_long(gm, args, hbm_peak, dev)
        out["prefill_t8192_k4_per_loop"] = run_prefill_long(gm, tc_peak, dev)
    if not args.no_quant:
        del gm
        torch.cuda.empty_cache()
        out["quantized"] = run_quant(w, args, hbm_peak, dev)
    return dict(out=out, headline=headline, e2e_dt=e2e_dt, w=w,
                hbm_peak=hbm_peak, tc_peak=tc_peak, peak_kind=peak_kind)


def run_spec(gm, prompt, steps=64, gamma=4, k_draft=1, k_verify=4):
    """Self-speculative greedy decoding after the prompt (per_loop cache):
    gamma drafts at k_draft loops, one verify pass at k_verify.  Every step
    synchronises once (the emitted count); wall-clock timing."""
    import torch
    T = prompt.shape[1]
    cache = gm.new_cache(1, T + (steps + 4) * (gamma + 1) + 16, T,
                         kv_mode="per_loop", max_loops=k_verify)
    ws = gm.workspace(1, T)
    sws = gm.spec_workspace(1, gamma)
    _, a = gm.prefill(cache, prompt, k_verify, ws)
    last = a.clone()
    for _ in range(3):
        out, n = gm.spec_decode_step(cache, last, gamma, k_draft, k_verify, sws)
        last = out[:, n - 1].contiguous()
    torch.cuda.synchronize()
    emitted = []
    t0 = time.perf_counter()
    for _ in range(steps):
        out, n = gm.spec_decode_step(cache, last, gamma, k_draft, k_verify, sws)
        last = out[:, n - 1].contiguous()
        emitted.append(n)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert gm.sync_status() == 0, "device-side check failed"
    # cost of one step when no draft is kept, and the break-even count
    res = {"tok_s": sum(emitted) / dt, "ms_per_step": dt / steps * 1e3,
           "tokens_per_step": sum(emitted) / steps, "gamma": gamma,
           "k_draft": k_draft, "k_verify": k_verify, "emitted": emitted}
    del cache, ws, sws
    torch.cuda.empty_cache()
    return res


def timed_decode(gm, B, ctx, k, mode, steps, hbm_peak, dev, prompt=None):
    """Decode `steps` tokens (CUDA-graph replays) after `ctx` tokens of
    context (prefill of `prompt`, else seeded synthetic cache)."""
    import torch
    cache = gm.new_cache(B, ctx + steps + 16, 1 if prompt is None else ctx,
                         kv_mode=mode, max_loops=k)
    ws = gm.workspace(B, 1 if prompt is None else ctx)
    if prompt is None:
        cache.fill_synthetic(ctx, seed=2)
    else:
        for t in range(prompt.shape[1]):      # quantised models: T = 1 calls
            gm.decode_step(cache, prompt[:, t].contiguous(), k, ws,
                           want_logits=False)
    tok = torch.zeros(B, dtype=torch.int32, device=dev)
    gm.decode_step(cache, tok, k, ws, want_logits=False)
    tb = cache._dec_bufs[0]
    for _ in range(2):
        gm.decode_step(cache, tb, k, ws, argmax=tb, want_logits=False)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        gm.decode_step(cache, tb, k, ws, argmax=tb, want_logits=False)
    e1.record()
    torch.cuda.synchronize()
    dt = e0.elapsed_time(e1) / 1e3
    gm.profile(True)
    gm.decode_step(cache, tb, k, ws, argmax=tb, want_logits=False)
    st = gm.profile_read()
    gm.profile(False)
    assert gm.sync_status() == 0, "device-side check failed"
    step_bytes = sum(v["bytes"] for v in st.values())
    res = {"tok_s": B * steps / dt, "ms_per_step": dt / steps * 1e3,
           "kv_cache_gb": cache.nbytes / 1e9, "bytes_per_step_gb": step_bytes / 1e9,
           "hbm_frac": step_bytes * steps / dt / (hbm_peak * 1e9),
           "kernels_us": {n: round(v["ms"] * 1e3, 1)
                          for n, v in sorted(st.items(), key=lambda kv: -kv[1]["ms"])}}
    del cache, ws
    torch.cuda.empty_cache()
    return res


def run_quant(w, args, hbm_peak, dev):
    """MXFP8 / NVFP4 weight-only models (embedding and head BF16)."""
    import torch
    import looped_ngpt_b200 as lb
    from synthetic import DORY, make_prompt
    from synthetic.quantize import quantize_weights
    res = {}
    for fmt in ("mxfp8", "nvfp4"):
        t0 = time.time()
        qw = quantize_weights(w, fmt)
        gm = lb.DoryModel(DORY, qw, device=dev)
        del qw
        r = {"encode_s": time.time() - t0}
        r["b1_ctx2k_k2_last_loop"] = timed_decode(gm, 1, 2048, 2, "last_loop",
                                                  32, hbm_peak, dev)
        r["b4_ctx131k_k2_last_loop"] = timed_decode(gm, 4, 131072, 2,
                                                    "last_loop", 8, hbm_peak, dev)
        res[fmt] = r
        del gm
        torch.cuda.empty_cache()
    return res


def run_long(gm, args, hbm_peak, dev):
    """Decode over seeded synthetic cached context: B=64 x 32768 tokens at
    k=2 in both KV modes, and B=4 x 131072 tokens at k=2, last_loop."""
    import torch
    res = {}
    K, W = args.long_steps, 2
    for name, B, ctx, k, mode in (("b64_ctx32k_k2_per_loop", 64, 32768, 2, "per_loop"),
                                   ("b64_ctx32k_k2_last_loop", 64, 32768, 2, "last_loop"),
                                   ("b4_ctx131k_k2_last_loop", 4, 131072, 2, "last_loop")):
        cache = gm.new_cache(B, ctx + K + W + 8, 1, kv_mode=mode, max_loops=k)
        cache.fill_synthetic(ctx, seed=2)
        ws = gm.workspace(B, 1)
        tok = torch.zeros(B, dtype=torch.int32, device=dev)
        gm.decode_step(cache, tok, k, ws, want_logits=False)
        tb = cache._dec_bufs[0]
        for _ in range(W):
            gm.decode_step(cache, tb, k, ws, argmax=tb, want_logits=False)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(K):
            gm.decode_step(cache, tb, k, ws, argmax=tb, want_logits=False)
        e1.record()
        torch.cuda.synchronize()
        dt = e0.elapsed_time(e1) / 1e3
        gm.profile(True)
        gm.decode_step(cache, tb, k, ws, argmax=tb, want_logits=False)
        st = gm.profile_read()
        gm.profile(False)
        assert gm.sync_status() == 0, "device-side check failed"
        step_bytes = sum(v["bytes"] for v in st.values())
        res[name] = {"tok_s": B * K / dt, "ms_per_step": dt / K * 1e3,
                     "kv_cache_gb": cache.nbytes / 1e9,
                     "bytes_per_step_gb": step_bytes / 1e9,
                     "hbm_frac": step_bytes * K / dt / (hbm_peak * 1e9),
                     "kernels_us": {n: round(v["ms"] * 1e3, 1)
                                    for n, v in sorted(st.items(),
                                                       key=lambda kv: -kv[1]["ms"])}}
        del cache, ws
        torch.cuda.empty_cache()
    return res


def run_prefill_long(gm, tc_peak, dev, T=8192, k=4, mode="per_loop"):
    """Prefill of one T-token prompt (seeded uniform tokens) at k loops: one
    warm-up call, one timed call, one profiled call (FLOPs per kernel)."""
    import torch
    from synthetic import DORY, make_prompt
    prompt = torch.from_numpy(make_prompt(DORY, 1, T)).to(dev)
    cache = gm.new_cache(1, T + 16, T, kv_mode=mode, max_loops=k)
    ws = gm.workspace(1, T)
    t = None
    for rep in range(3):
        cache.reset()
        if rep == 2:
            gm.profile(True)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        gm.prefill(cache, prompt, k, ws)
        e1.record()
        torch.cuda.synchronize()
        if rep == 1:
            t = e0.elapsed_time(e1) / 1e3
    st = gm.profile_read()
    gm.profile(False)
    assert gm.sync_status() == 0, "device-side check failed"
    flops = sum(v["flops"] for v in st.values())
    res = {"tok_s": T / t, "ms": t * 1e3, "flops": flops,
           "tc_frac": flops / t / (tc_peak * 1e12),
           "kernels_ms": {n: round(v["ms"], 2)
                          for n, v in sorted(st.items(), key=lambda kv: -kv[1]["ms"])}}
    del cache, ws
    torch.cuda.empty_cache()
    return res


def profile_run(args):
    """A minimal run for profilers: one NVTX-marked decode step or prefill."""
    import torch
    import looped_ngpt_b200 as lb
    from synthetic import DORY, make_weights, make_prompt, dory_with_blocks
    shape = DORY
    if args.profile_blocks:
        shape = dory_with_blocks(*[int(x) for x in args.profile_blocks.split(",")])
    w = make_weights(shape, seed=0)
    if args.profile_quant:
        from synthetic.quantize import quantize_weights
        w = quantize_weights(w, args.profile_quant)
    gm = lb.DoryModel(shape, w, device="cuda:0")
    prompt = torch.from_numpy(make_prompt(shape, 1, args.prompt)).to("cuda:0")
    k = args.profile_decode or args.profile_prefill
    cache = gm.new_cache(1, args.prompt + 64, 1 if args.profile_quant else args.prompt,
                         kv_mode=args.kv_mode, max_loops=k)
    ws = gm.workspace(1, args.prompt)
    if args.profile_quant:
        # block projections are quantised: T = 1 calls only, so the context
        # comes from the seeded cache fill
        cache.fill_synthetic(args.prompt, seed=3)
        tok = torch.zeros(1, dtype=torch.int32, device="cuda:0")
        for _ in range(4):
            gm.decode_step(cache, tok, k, ws, argmax=tok, want_logits=False)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_push("decode_step")
        gm.decode_step(cache, tok, k, ws, argmax=tok, want_logits=False)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
        assert gm.sync_status() == 0
        return 0
    if args.profile_prefill:
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_push("prefill")
        gm.prefill(cache, prompt, k, ws)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
        return 0
    _, am = gm.prefill(cache, prompt, k, ws)
    gm.decode_step(cache, am, k, ws, want_logits=False)
    tok = cache._dec_bufs[0]
    for _ in range(3):
        gm.decode_step(cache, tok, k, ws, argmax=tok, want_logits=False)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("decode_step")
    gm.decode_step(cache, tok, k, ws, argmax=tok, want_logits=False)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    assert gm.sync_status() == 0
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return main_reference(args)
    if args.profile_decode or args.profile_prefill:
        return profile_run(args)
    rank, world, local = dist_setup()
    r = run_gpu(args, rank, world, local)
    h = r["headline"]
    dt = max_over_ranks(h["dt"], world)
    K, W = args.steps, args.warmup
    value = world * K / dt
    e2e_dt = max_over_ranks(r["e2e_dt"], world)
    st = h["stats"]
    # dominant kernel: largest share of the profiled (eager) step
    dom = max(st, key=lambda n: st[n]["ms"])
    d = st[dom]
    bound = "hbm" if d["flops"] / max(d["bytes"], 1) < 100 else "tensor"
    if bound == "hbm":
        achieved = d["bytes"] / d["launches"] / (d["ms"] / d["launches"] / 1e3) / 1e9
        peak, unit = r["hbm_peak"], "GB/s"
    else:
        achieved = d["flops"] / d["launches"] / (d["ms"] / d["launches"] / 1e3) / 1e12
        peak, unit = r["tc_peak"], "TFLOP/s"
    eager_ms = sum(v["ms"] for v in st.values())
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, secs = oracle_decode_sample(r["w"], HEADLINE_K, args.prompt)
        cpu = {"value": tps, "unit": "tok/s", "cores": blas_threads(),
               "kind": "oracle",
               "sample": (f"1 greedy decode step at k={HEADLINE_K}, "
                          f"{args.kv_mode}, at a {args.prompt}-token context "
                          f"(seeded synthetic cached entries from the "
                          f"generator the library's cache fill uses), "
                          f"Dory-shape weights, fp64 NumPy ({secs:.1f} s)")}
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": dt / K * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": arm_config(args.prompt, world, args.kv_mode),
        "roofline": {"bound": bound, "kernel": dom, "achieved": achieved,
                     "peak": peak, "unit": unit, "frac": achieved / peak,
                     "peak_source": r["peak_kind"], "traffic": dram_traffic(dom),
                     "share_of_eager_pass": d["ms"] / eager_ms},
        "cpu_baseline": cpu,
        "e2e": {"value": world * K / e2e_dt, "unit": "tok/s",
                "h2d_bytes_per_step": 4, "d2h_bytes_per_step": 4},
        "gpu_launches": int(round(h["launches"] * K)),
        "clocks": h["clocks"],
        "breakdown": r["out"],
        # per-kernel figures of P extra steps launched eagerly with CUDA
        # events around every kernel (no graph, no overlap between
        # kernels): their sum exceeds the graph-replayed step time, so they
        # rank kernels and give each one's own rate, not shares of the
        # timed step (the ncu launch list under profiles/ gives those)
        "kernels_eager": {
            "eager_pass_ms": eager_ms / h["P"],
            "timed_step_ms": dt / K * 1e3,
            "per_kernel": {n: {"launches_per_step": v["launches"] / h["P"],
                               "us_per_step": v["ms"] / h["P"] * 1e3,
                               "GBps": v["bytes"] / (v["ms"] / 1e3) / 1e9
                               if v["ms"] > 0 else None}
                           for n, v in sorted(st.items(),
                                              key=lambda kv: -kv[1]["ms"])}},
    }
    print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main_reference(args):
    """The oracle on the host cores, on the GPU arm's workload (Dory shapes,
    batch 1, k=2, decode at the prompt-length context) and metric.  One
    oracle decode token takes about 20 s, so a step is a bounded sample: 1/C
    of a token, C the smallest divisor of --steps that keeps the timed run
    at 3 tokens or fewer; the K steps run as K / C whole tokens, timed
    together."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from synthetic import DORY, make_weights
    K, W = max(1, args.steps), max(0, args.warmup)
    C = next(c for c in range(1, K + 1) if K % c == 0 and K // c <= 3)
    n_tok, n_warm = K // C, -(-W // C)
    w = make_weights(DORY, seed=0)
    m = oracle_at_context(w, args.prompt, args.kv_mode, HEADLINE_K,
                          extra=n_tok + n_warm + 1)
    tok = 7
    for _ in range(n_warm):
        tok = int(np.argmax(m.decode_step([tok], HEADLINE_K)[0]))
    t0 = time.perf_counter()
    for _ in range(n_tok):
        tok = int(np.argmax(m.decode_step([tok], HEADLINE_K)[0]))
    secs = time.perf_counter() - t0
    tps = n_tok / secs
    sample = (f"{K} steps of 1/{C} decode token each, run as {n_tok} whole "
              f"greedy decode tokens at k={HEADLINE_K}, {args.kv_mode}, "
              f"after a {args.prompt}-token seeded synthetic cached context "
              f"({n_warm} warm-up tokens), Dory-shape weights, fp64 NumPy "
              f"({secs:.1f} s timed)")
    line = {"metric": METRIC, "value": tps, "unit": "tok/s", "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": secs / K * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": arm_config(args.prompt, world, args.kv_mode),
            "cpu_baseline": {"value": tps, "unit": "tok/s",
                             "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": tps, "unit": "tok/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
