#!/usr/bin/env python
"""LFM3-1.7B decode / prefill throughput on B200 through liblfm3.so (one JSON line on rank 0).

Headline (value): greedy decode tok/s of the bf16 24-layer model, batch 1, at a 2048-token
context (the prompt is prefilled by the library first); one step = embed -> 24 layers -> tied
head -> argmax for one token, with the next token fed back on the device. Inputs are synthetic
(seeded random-init weights, uniform token ids); every step streams the 3.46 GB of weights, far
more than the 126 MB L2, so no explicit L2 flush is needed between steps.

Also reported under "extra": prefill tok/s of an 8192-token prompt in 2048-token chunks over
shuffled 64-token pages (bf16), and NVFP4-FFN decode tok/s at 1 / 8 streams (2048 context) and
64 streams (contexts uniform in [256, 8192] on drawn state).

--impl reference times the CPU oracle (float64 NumPy) on the same metric.
Multi-GPU (torchrun, --gpus N): independent replicas, no collective on the data path; value is
the sum over ranks (N x steps / max-over-ranks time).
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tok/s @1/8/64 streams; prefill tok/s @8k; % of HBM/TC roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------------------------------- clocks
class Clocks:
    """nvidia-smi sampled every 100 ms while the GPU phases run."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--id={index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                       "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.count(",") >= 8]
        os.unlink(self.f.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
                pw = float(r[3])
            except ValueError:
                continue
            if pw < 200:  # idle samples (between phases) do not describe the load
                continue
            for i, nm in enumerate(names):
                if r[5 + i].strip().lower() in ("active", "1"):
                    reasons.add(nm)
        loaded = [float(r[1]) for r in rows if len(r) > 3 and _f(r[3]) >= 200]
        return {"sm_mhz": statistics.median(loaded) if loaded else (statistics.median(sm) if sm else None),
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons), "samples": len(loaded)}


def _f(x):
    try:
        return float(x)
    except ValueError:
        return 0.0


# ---------------------------------------------------------------------------------------- oracle baseline
def oracle_decode_rate(max_steps=3, prompt=64, warm=1):
    """The CPU oracle (float64 NumPy, all host cores) on a bounded sample of the decode workload:
    the bf16 24-layer model, a `prompt`-token prompt, then timed greedy decode steps."""
    from lfm3_inputs import lfm3_1p7b, make_weights, make_tokens
    from oracle import Lfm3Oracle
    g = lfm3_1p7b()
    o = Lfm3Oracle(make_weights(g, 0))
    st = o.new_state()
    out = o.forward_chunk(st, tokens=make_tokens(1, "prompt", prompt, g.vocab))
    tok = int(np.argmax(out["logits"]))
    for _ in range(warm):
        tok = int(np.argmax(o.forward_chunk(st, tokens=np.array([tok]))["logits"]))
    t0 = time.perf_counter()
    for _ in range(max_steps):
        tok = int(np.argmax(o.forward_chunk(st, tokens=np.array([tok]))["logits"]))
    dt = time.perf_counter() - t0
    threads = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            threads = max(i.get("num_threads", 0) for i in info)
    except Exception:
        pass
    return max_steps / dt, threads, dt


# ---------------------------------------------------------------------------------------- GPU arm
def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world, cuda=True):
    """All ranks meet; then (on a GPU) the device is drained."""
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if cuda:
        torch.cuda.synchronize()


def max_over_ranks(world, x, device="cuda"):
    """The largest of the ranks' values (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def timed(world, fn, steps, stream):
    """Device time of `steps` calls of fn(), CUDA events on the launching stream, max over ranks."""
    import torch
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(world, e0.elapsed_time(e1))


def traffic_record(key):
    """The committed ncu traffic record `key` (profiles/traffic.json), or None once any kernel
    source it was measured on has changed."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)[key]
        for src, sha in rec["sources"].items():
            if hashlib.sha256(open(os.path.join(ROOT, src), "rb").read()).hexdigest() != sha:
                return None
        return rec
    except Exception:
        return None


def decode_step_bytes(g, positions, nvfp4=False, logits=True):
    """Algorithmic HBM bytes of one decode step: every weight once (bf16, or NVFP4 codes + E4M3
    scales for the FFN), the cached keys and values each stream's new row attends to (all earlier
    positions on full layers, the last 256 on sliding ones) plus the new row written, the conv
    columns read and written, and the fp32 logits written. Activations between kernels (a few KB
    per layer) are left out."""
    from lfm3_inputs.gen import CONV, FULL
    d, f, hd, kv = g.d_model, g.d_ffn, g.head_dim, g.n_kv
    w = 0
    for t in g.layer_types:
        w += 2 * 4 * d
        if t == CONV:
            w += 2 * (3 * d * d + d * g.conv_taps + d * d)
        else:
            w += 2 * (g.qkvg_rows * d + 2 * hd + d * g.n_q * hd)
        w += 3 * (f * d // 2 + f * d // 16) if nvfp4 else 2 * 3 * f * d
    if g.has_head:
        w += 2 * (g.vocab * d + d)
    state = 0
    row = 2 * 2 * kv * hd  # K and V of one position, bf16
    for p in positions:
        for t in g.layer_types:
            if t == CONV:
                state += 2 * 2 * (g.conv_taps - 1) * d
            else:
                seen = p + 1 if t == FULL else min(p + 1, g.window)
                state += row * seen + row
        if g.has_head and logits:
            state += 4 * g.vocab
    return w + state


def run_ours(args):
    import torch
    from attention_decoder_b200.model import Lfm3Model
    from lfm3_inputs import lfm3_1p7b, make_weights, make_tokens, page_permutation, context_lengths

    world, rank, local = dist_setup(args)
    pk, pk_kind = peaks()
    hbm = float(pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    stream = torch.cuda.current_stream()
    K, Wm = args.steps, args.warmup
    clocks = Clocks(local)
    g = lfm3_1p7b()
    if args.small:
        # profiling case: 4 layers (conv, sliding, full, conv) + the tied head, 256-token context
        g = lfm3_1p7b(layer_types=(0, 2, 1, 0))
        args.no_extra = True
    res = {}

    # ---------------- bf16 model: decode at batch 1 (headline) and prefill 8k
    W = make_weights(g, 0)
    ctx0 = 256 if args.small else 2048
    need = ctx0 + Wm + K + 8
    mpp = max(128, (need + 63) // 64 + 1)
    m = Lfm3Model(W, max_streams=1, max_pages_per_stream=mpp, max_batch=1)
    del W
    prompt = torch.from_numpy(make_tokens(1, "prompt", 2048, g.vocab)[:ctx0]).cuda()

    def fresh_state(model, page_table=None):
        st = model.new_state(page_table=page_table)
        o = model.prefill(st, 0, tokens=prompt)
        return st, o

    if args.only == "prefill":
        return run_prefill_only(args, world, m, g, stream, clocks, Wm)
    if args.only == "nvfp4":
        del m
        torch.cuda.empty_cache()
        r = nvfp4_leg(world, g, stream, prompt, K, Wm, hbm, hi=2048 if args.small else 8192)
        if rank == 0:
            print(json.dumps({"profiling_case": "NVFP4 decode at 1/4/8/64 streams", **r, "clocks": clocks.stop()}),
                  flush=True)
        return
    st, o = fresh_state(m)
    bufs = {"argmax": o["argmax"].clone(), "logits": torch.empty(1, g.vocab, device="cuda")}
    slots_d = torch.zeros(1, dtype=torch.int32, device="cuda")

    def step():
        m.decode(st, [0], tokens=bufs["argmax"], d_slots=slots_d, out=bufs)

    for _ in range(Wm):
        step()
    ms = timed(world, step, K, stream)
    launches_per_step = m.last_launch_count()
    res["decode_b1"] = {"ms_per_step": ms / K, "tok_s": K / (ms / 1e3)}

    # the projections' own rate, event-bracketed: this pass runs the step launch by launch (no
    # graph, an event pair around each projection), so it is reported beside the roofline only
    st, o = fresh_state(m)
    bufs["argmax"].copy_(o["argmax"])
    m.profile(True, capacity=200 * (K + 1))
    for _ in range(K):
        step()
    prof = m.profile_read()
    m.profile(False)
    gemv_gbs = prof["bytes"] / (prof["ms"] / 1e3) / 1e9
    # the timed steps ran at positions ctx0 + Wm .. ctx0 + Wm + K - 1
    step_bytes = sum(decode_step_bytes(g, [p]) for p in range(ctx0 + Wm, ctx0 + Wm + K)) / K

    # end to end through the public API with host buffers: pinned token in, greedy id out, each step
    st, o = fresh_state(m)
    h_tok = torch.empty(1, dtype=torch.int32).pin_memory()
    h_out = torch.empty(1, dtype=torch.int32).pin_memory()
    h_tok.copy_(o["argmax"].cpu())
    d_tok = torch.empty(1, dtype=torch.int32, device="cuda")

    def e2e_step():
        d_tok.copy_(h_tok, non_blocking=True)
        m.decode(st, [0], tokens=d_tok, d_slots=slots_d, out=bufs)
        h_out.copy_(bufs["argmax"], non_blocking=True)
        stream.synchronize()
        h_tok.copy_(h_out)

    for _ in range(min(Wm, 3)):
        e2e_step()
    barrier(world)
    t0 = time.perf_counter()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(world, e0.elapsed_time(e1))

    # prefill 8k (chunks of 2048) over shuffled pages
    if not args.no_extra and args.only is None:
        n8 = 8192
        mp = Lfm3Model(make_weights(g, 0), max_streams=1, max_pages_per_stream=n8 // 64, max_batch=1)
        pt = page_permutation(1, "pages8k", n8 // 64).reshape(1, -1)
        tok8 = torch.from_numpy(make_tokens(1, "prompt8k", n8, g.vocab)).cuda()
        sts = [mp.new_state(page_table=pt) for _ in range(2)]
        it = [0]

        def pstep():
            s = sts[it[0] % 2]
            it[0] += 1
            s.h_seq_len[:] = 0
            s.seq_len.zero_()
            mp.prefill(s, 0, tokens=tok8)

        for _ in range(2):
            pstep()
        pk_steps = max(2, min(K, 8))
        pms = timed(world, pstep, pk_steps, stream)
        mp.profile(True, capacity=400)
        pstep()
        pprof = mp.profile_read()
        mp.profile(False)
        pf = prefill_flops(g, n8)
        p_tf = pf / (pms / pk_steps / 1e3) / 1e12
        res["prefill_8k"] = {"tok_s": n8 * pk_steps / (pms / 1e3), "ms": pms / pk_steps,
                             "flops": pf, "tflops": p_tf,
                             "tc_frac": p_tf / float(pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])),
                             "tc_frac_sustained": p_tf / float(pk.get("bf16_tflops_sustained",
                                                                      pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))),
                             "gemm_tflops": pprof["flops"] / (pprof["ms"] / 1e3) / 1e12,
                             "gemm_share": pprof["ms"] / (pms / pk_steps)}
        del mp, sts
    # prefill 32k (chunks of 2048) over shuffled pages: opt-in (--long)
    if args.long and args.only is None:
        n32 = 32768
        mp = Lfm3Model(make_weights(g, 0), max_streams=1, max_pages_per_stream=n32 // 64, max_batch=1)
        s32 = mp.new_state(page_table=page_permutation(1, "pages32k", n32 // 64).reshape(1, -1))
        tok32 = torch.from_numpy(make_tokens(1, "prompt32k", n32, g.vocab)).cuda()

        def lstep():
            s32.h_seq_len[:] = 0
            s32.seq_len.zero_()
            mp.prefill(s32, 0, tokens=tok32)

        lstep()
        lms = timed(world, lstep, 2, stream)
        lf = prefill_flops(g, n32)
        l_tf = lf / (lms / 2 / 1e3) / 1e12
        res["prefill_32k"] = {"tok_s": n32 * 2 / (lms / 1e3), "ms": lms / 2, "flops": lf, "tflops": l_tf,
                              "tc_frac": l_tf / float(pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))}
        del mp, s32
    del m, st
    torch.cuda.empty_cache()

    # ---------------- NVFP4 FFN model: decode at 1 / 4 / 8 streams (2048 ctx) and 64 streams
    if not args.no_extra and args.only is None:
        res.update(nvfp4_leg(world, g, stream, prompt, K, Wm, hbm))
    clk = clocks.stop()

    tok_s_rank = res["decode_b1"]["tok_s"]
    step_s = res["decode_b1"]["ms_per_step"] / 1e3
    achieved = step_bytes / step_s / 1e9
    trec = traffic_record("decode_step_b1")
    value = world * tok_s_rank
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "tok/s", "n_gpus": world, "steps": K, "warmup": Wm,
        "ms_per_step": round(res["decode_b1"]["ms_per_step"], 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded random-init weights, uniform token ids)",
        "config": {"workload": ("LFM3-1.7B bf16 24-layer decode, 1 stream per GPU, greedy, 2048-token context "
                                "(prefilled), tied 128000 head") if not args.small else
                               "profiling case: 4-layer LFM3 slice + head, bf16 decode, 256-token context",
                   "streams_per_gpu": 1, "context": ctx0,
                   "l2": "no flush: each step streams %.2f GB of weights and K/V, > 126 MB L2" % (step_bytes / 1e9),
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm",
                     "kernel": ("the decode step as timed: one CUDA-graph replay of %d kernels (k_wstream "
                                "projections, k_attn_decode_fused, bookkeeping)" % launches_per_step),
                     "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s", "frac": round(achieved / hbm, 4),
                     "peak_kind": pk_kind,
                     "traffic": None if trec is None else round(trec["dram_per_algorithmic"] * step_bytes),
                     "traffic_note": None if trec is None else trec["note"],
                     "bytes_per_step": round(step_bytes),
                     "projections_graph_off": {"gbs": round(gemv_gbs, 1), "frac": round(gemv_gbs / hbm, 4),
                                               "launches": prof["launches"],
                                               "note": "k_wstream only, event pair around each launch, no graph"}},
        "e2e": {"value": round(world * K / (e2e_ms / 1e3), 2), "unit": "tok/s", "h2d_bytes_per_step": 4,
                "d2h_bytes_per_step": 4},
        "gpu_launches": launches_per_step * K,
        "clocks": clk,
        "extra": res,
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        rate, threads, dt = oracle_decode_rate()
        line["cpu_baseline"] = {"value": round(rate, 4), "unit": "tok/s", "cores": threads, "kind": "oracle",
                                "sample": f"float64 NumPy oracle, bf16 24-layer model, 64-token prompt then 3 timed "
                                          f"greedy decode steps ({dt:.1f} s)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def prefill_flops(g, n):
    """Algorithmic FLOPs of one n-token prompt pass: every projection GEMM (2 M N K), causal
    attention (Q K^T and P V over the keys each query sees: all earlier positions on full layers,
    at most the window on sliding ones) and the head on the last row. The 7-tap convolution and the
    norms are left out (under 0.01 %)."""
    from lfm3_inputs.gen import CONV, FULL
    d, f, hd = g.d_model, g.d_ffn, g.head_dim
    per_tok = 0
    for t in g.layer_types:
        per_tok += 2 * d * f * 3
        per_tok += 2 * d * 3 * d + 2 * d * d if t == CONV else 2 * d * g.qkvg_rows + 2 * g.n_q * hd * d
    keys_full = n * (n + 1) // 2
    keys_win = sum(min(p + 1, g.window) for p in range(n))
    attn = 0
    for t in g.layer_types:
        if t != CONV:
            attn += 4 * hd * g.n_q * (keys_full if t == FULL else keys_win)
    return n * per_tok + attn + 2 * d * g.vocab


def nvfp4_leg(world, g, stream, prompt, K, Wm, hbm, hi=8192):
    """The NVFP4-FFN model: decode tok/s and HBM fraction at 1 / 4 / 8 streams (the prompt's
    context, prefilled) and at 64 streams on drawn state (contexts uniform in [256, hi])."""
    import torch
    import numpy as np
    from attention_decoder_b200.model import Lfm3Model
    from lfm3_inputs import make_weights, make_tokens, page_permutation, context_lengths
    res = {}
    Wq = make_weights(g, 0, ffn="nvfp4")
    S = 64
    ctx64 = context_lengths(1, "ctx64", S, 256, hi)
    steps_q = max(4, min(K, 32))
    mpp_q = (hi + Wm + steps_q + 16) // 64 + 2
    mq = Lfm3Model(Wq, max_streams=S, max_pages_per_stream=mpp_q, max_batch=S)
    del Wq
    stq = mq.new_state(page_table=page_permutation(1, "pages64", S * mpp_q).reshape(S, mpp_q))
    for s in range(8):
        mq.prefill(stq, s, tokens=prompt)
    qb, qfrac = {}, {}
    for B in (1, 4, 8):
        sl = torch.arange(B, dtype=torch.int32, device="cuda")
        ob = {"argmax": torch.zeros(B, dtype=torch.int32, device="cuda"),
              "logits": torch.empty(B, g.vocab, device="cuda")}

        def qstep():
            mq.decode(stq, list(range(B)), tokens=ob["argmax"], d_slots=sl, out=ob)

        for _ in range(Wm):
            qstep()
        p0 = int(stq.h_seq_len[0])
        qms = timed(world, qstep, steps_q, stream)
        qb[B] = B * steps_q / (qms / 1e3)
        qbytes = decode_step_bytes(g, [p0 + steps_q // 2] * B, nvfp4=True)
        qfrac[B] = qbytes * (steps_q / (qms / 1e3)) / 1e9 / hbm
    # 64 streams on drawn state: K/V, rings and conv columns N(0,1) drawn on the device
    gen = torch.Generator(device="cuda").manual_seed(1)
    for t in (stq.kv_k, stq.kv_v, stq.ring_k, stq.ring_v, stq.conv):
        t.normal_(generator=gen)
    stq.h_seq_len[:] = ctx64
    stq.seq_len.copy_(torch.from_numpy(stq.h_seq_len))
    sl = torch.arange(S, dtype=torch.int32, device="cuda")
    ob = {"argmax": torch.from_numpy(make_tokens(1, "tok64", S, g.vocab)).cuda(),
          "logits": torch.empty(S, g.vocab, device="cuda")}

    def q64():
        mq.decode(stq, list(range(S)), tokens=ob["argmax"], d_slots=sl, out=ob)

    for _ in range(Wm):
        q64()
    qms = timed(world, q64, steps_q, stream)
    qb[64] = S * steps_q / (qms / 1e3)
    qbytes = decode_step_bytes(g, [int(c) + Wm + steps_q // 2 for c in ctx64], nvfp4=True)
    qfrac[64] = qbytes * (steps_q / (qms / 1e3)) / 1e9 / hbm
    res["decode_nvfp4"] = {f"b{b}_tok_s": v for b, v in qb.items()}
    res["decode_nvfp4"].update({f"b{b}_hbm_frac": round(v, 4) for b, v in qfrac.items()})
    res["decode_nvfp4"]["b64_contexts"] = "uniform [256, %d], mean %.0f" % (hi, float(np.mean(ctx64)))
    del mq, stq
    torch.cuda.empty_cache()
    return res


def run_prefill_only(args, world, m, g, stream, clocks, Wm):
    """Profiling leg: the 8192-token prompt pass (chunks of 2048, shuffled pages), timed."""
    import torch
    from lfm3_inputs import make_tokens, page_permutation
    del m
    torch.cuda.empty_cache()
    from attention_decoder_b200.model import Lfm3Model
    from lfm3_inputs import make_weights
    n8 = 8192
    mp = Lfm3Model(make_weights(g, 0), max_streams=1, max_pages_per_stream=n8 // 64, max_batch=1)
    pt = page_permutation(1, "pages8k", n8 // 64).reshape(1, -1)
    tok8 = torch.from_numpy(make_tokens(1, "prompt8k", n8, g.vocab)).cuda()
    st = mp.new_state(page_table=pt)

    def pstep():
        st.h_seq_len[:] = 0
        st.seq_len.zero_()
        mp.prefill(st, 0, tokens=tok8)

    for _ in range(Wm):
        pstep()
    K = max(1, args.steps)
    ms = timed(world, pstep, K, stream)
    clk = clocks.stop()
    if int(os.environ.get("RANK", "0")) == 0:
        print(json.dumps({"profiling_case": "prefill 8k", "ms": ms / K, "tok_s": n8 * K / (ms / 1e3),
                          "launches_per_prefill": mp.last_launch_count(), "clocks": clk}), flush=True)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    K = min(args.steps, 30)
    rate, threads, dt = oracle_decode_rate(max_steps=K, prompt=64, warm=min(args.warmup, 1))
    line = {
        "impl": "reference", "metric": METRIC, "value": round(rate, 4), "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 / rate, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded random-init weights)",
        "config": {"workload": "LFM3-1.7B bf16 24-layer decode, 1 stream, greedy (CPU oracle)"},
        "cpu_baseline": {"value": round(rate, 4), "unit": "tok/s", "cores": threads, "kind": "oracle",
                         "sample": f"float64 NumPy oracle: 64-token prompt, then {K} timed greedy decode steps "
                                   f"({dt:.1f} s; at most 30 steps are timed)"},
        "e2e": {"value": round(rate, 4), "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true", help="headline decode only")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--small", action="store_true", help="4-layer profiling case (not a bench line)")
    ap.add_argument("--long", action="store_true", help="also time the 32768-token prefill")
    ap.add_argument("--only", choices=["decode", "prefill", "nvfp4"], default=None,
                    help="profiling: run only the bf16 decode, the 8k prefill or the NVFP4 decode leg")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
