#!/usr/bin/env python
"""Benchmark of the fine-grained-scaled FP8 GEMM  D = C + A @ B^T  on B200.

One step = one pass over the dense NT FP8 sweep of DeepSeek-V3 projection
shapes: M in {64, 128, 4096} x (N, K) in {(2112,7168), (24576,1536),
(32768,512), (7168,16384), (4096,7168), (7168,2048)}, A/B ~ N(0,1) quantised
with 1x128 / 128x128 UE8M0 scales, C ~ N(0,1) bf16 (synthetic, seeded).
Each GEMM call is timed with CUDA events on its stream after an L2 flush (a
256 MB write followed by a 256 MB read, so L2 holds clean unrelated lines),
so no call reads its inputs from a warm L2; each step is
enqueued behind a short device-side sleep so that no timed call waits for the
host to launch it.

  value   = total FLOPs of the sweep (all ranks) / device time (max over ranks)
  e2e     = the same sweep through the C ABI from pinned HOST buffers, the
            host->device copies of A, SFA, B, SFB, C and the device->host copy
            of D inside the timed region
  roofline: the dominant kernel (largest share of step time) against the
            measured peak (MEASURED_PEAKS.json), FP8 peak = measured bf16 x 2;
            beside it frac_vs_probe (the library's own block-scaled FP8
            tcgen05 loop, measured in the same run: tensor_peak_probe) and
            frac_vs_spec (nominal dense FP8, 4.5 PFLOP/s)
  per_config: the other configurations timed the same way after the sweep:
            the small dense case, MoE prefill (contiguous), MoE decode
            (masked) and FP8 x FP4 (dense and contiguous)
  cpu_baseline: the CPU oracle on a bounded sample of the same sweep

Multi-GPU: the sweep does not shard (replicas only); with --gpus N each rank
runs the full sweep on its own GPU and value aggregates all ranks ("weak").

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                  [--shape M,N,K] [--no-e2e] [--no-cpu]
                  [--no-configs]
                  [--workload dense | contiguous | nn_contiguous | kgrouped_tn | masked
                              | fp4 | moe_decode_fp4 | bf16 | promotion] [--graph]

The default workload (dense) is the headline line.  The others time each case
alone after an L2 flush and report per-case TFLOPS and roofline fractions:
MoE prefill (contiguous, NT and NN), the MoE weight gradient (K-grouped TN),
decode (masked, plain or as a CUDA graph with --graph), FP8 x FP4, the FP8 x
FP4 decode step with SwiGLU, BF16 against cuBLAS, and the two ways of
applying the scales (block-scaled MMA vs per-K-block promotion).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FP8 TFLOPS per shape & % of B200 dense FP8 peak (GB/s vs HBM for decode)"
UNIT = "TFLOPS"
DENSE_NK = [(2112, 7168), (24576, 1536), (32768, 512), (7168, 16384), (4096, 7168), (7168, 2048)]
DENSE_M = [64, 128, 4096]
FLUSH_BYTES = 256 << 20
HOLD_CYCLES = 6_000_000  # ~3 ms at 2 GHz: longer than the host needs to enqueue one step
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_PER_BF16 = 2.0  # nominal dense FP8 : BF16 tensor throughput (4.5 : 2.25 PFLOP/s)
FP8_SPEC_TFLOPS = 4500.0  # nominal dense FP8 peak of one B200


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--shape", default=None, help="run one M,N,K shape instead of the sweep")
    ap.add_argument("--workload", default="dense",
                    choices=["dense", "contiguous", "masked", "fp4", "moe_decode_fp4", "bf16", "nn_contiguous",
                             "kgrouped_tn", "promotion"],
                    help="dense: the DeepSeek-V3 dense sweep (default); contiguous / masked / fp4: the "
                         "M-grouped prefill, masked decode and FP8 x FP4 cases, one JSON line each")
    ap.add_argument("--graph", action="store_true",
                    help="grouped workloads: capture each case's call in a CUDA graph and time its replay")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="time the dense sweep only (skip the grouped, decode and FP8 x FP4 cases)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    return ap.parse_args()


def shapes_from(args):
    if args.shape:
        m, n, k = (int(v) for v in args.shape.split(","))
        return [(m, n, k)]
    return [(m, n, k) for (n, k) in DENSE_NK for m in DENSE_M]


# ---------------------------------------------------------------- ranks

def max_over_ranks(x: float, use_dist: bool, device) -> float:
    """The largest of x over all ranks (the slowest rank sets the job's time);
    x itself when the run is not distributed.  Every rank calls it at the same
    point, in the same order."""
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if use_dist:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_rank: float, ms_max: float) -> float:
    """Whole-job throughput: every rank does flops_per_rank in a step whose
    time is the maximum over ranks ("weak" scaling: work per GPU fixed)."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


def flops(m, n, k):
    return 2.0 * m * n * k


def alg_bytes(m, n, k, with_c=True):
    """A + SFA + B + SFB (128x128 block codes) + D (+ C), in bytes."""
    sfa = m * (k // 128)
    sfb = ((n + 127) // 128) * (k // 128)
    return m * k + sfa + n * k + sfb + 2 * m * n + (2 * m * n if with_c else 0)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash():
    h = hashlib.sha1()
    for name in ("dg_gemm.cuh", "dg_ptx.cuh", "dg_lib.cu"):
        with open(os.path.join(ROOT, "moe_grouped_gemm_06_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def recorded_traffic(workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    src = kernel_source_hash()
    for line in open(path):
        parts = line.split()
        if len(parts) >= 3 and not line.startswith("#") and parts[0] == src and parts[1] == workload:
            return float(parts[2])
    return None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        rows = []
        with open(self.file.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.file.name)
        if not rows:
            return None

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None

        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        power = [num(r[3]) for r in rows if num(r[3]) is not None]
        pmax = max(power) if power else 0.0
        loaded = [num(r[1]) for r in rows if num(r[3]) is not None and num(r[3]) >= 0.5 * pmax]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(loaded or sm) if sm else None,
                "sm_max_mhz": num(rows[0][2]), "power_w_max": pmax, "samples": len(rows),
                "reasons": reasons}


# ---------------------------------------------------------------- inputs

def make_inputs(dg, torch, m, n, k, gen):
    """Device-resident inputs, quantised and packed by the library's own kernels."""
    dev = "cuda"
    xa = torch.randn((m, k), generator=gen, device=dev, dtype=torch.float32)
    xb = torch.randn((n, k), generator=gen, device=dev, dtype=torch.float32)
    a = torch.empty((m, k), dtype=torch.uint8, device=dev)
    b = torch.empty((n, k), dtype=torch.uint8, device=dev)
    ea = torch.empty((m, k // 128), dtype=torch.uint8, device=dev)
    eb = torch.empty(((n + 127) // 128, k // 128), dtype=torch.uint8, device=dev)
    dg.dg_quantize_fp8(xa, a, ea, 1)
    dg.dg_quantize_fp8(xb, b, eb, 128)
    sfa = torch.empty(dg.dg_packed_sf_words(m, k // 128), dtype=torch.int32, device=dev)
    sfb = torch.empty(dg.dg_packed_sf_words(n, k // 128), dtype=torch.int32, device=dev)
    dg.dg_pack_sf(ea, m, sfa, row_div=1)
    dg.dg_pack_sf(eb, n, sfb, row_div=128)
    c = torch.randn((m, n), generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
    d = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
    del xa, xb, ea, eb
    return {"a": a, "sfa": sfa, "b": b, "sfb": sfb, "c": c, "d": d}


# ---------------------------------------------------------------- grouped / FP4 cases

GROUPED_NK = [(4096, 7168), (7168, 2048)]
CONTIG_GROUPS, CONTIG_ROWS = 8, (6000, 10000)
MASKED_GROUPS, MASKED_MAX_M, MASKED_EXPECTED = 32, 256, (16, 64, 128)


def quant_a_dev(dg, torch, rows, k, gen, groups=1):
    """e4m3 A [groups*rows, k] with 1x128 scales, packed per group."""
    x = torch.randn((groups * rows, k), generator=gen, device="cuda", dtype=torch.float32)
    a = torch.empty((groups * rows, k), dtype=torch.uint8, device="cuda")
    ea = torch.empty((groups * rows, k // 128), dtype=torch.uint8, device="cuda")
    dg.dg_quantize_fp8(x, a, ea, 1)
    del x
    words = dg.dg_packed_sf_words(rows, k // 128)
    sfa = torch.empty(groups * words, dtype=torch.int32, device="cuda")
    for g in range(groups):
        dg.dg_pack_sf(ea[g * rows:(g + 1) * rows], rows, sfa[g * words:(g + 1) * words], row_div=1)
    return a, sfa


def quant_b_dev(dg, torch, groups, n, k, gen, fp4=False):
    """B [groups, n, k] e4m3 with 128x128 scales, or e2m1 [groups, n, k/2]
    with 1x32 scales; scale words packed per group."""
    b = torch.empty((groups, n, k // 2 if fp4 else k), dtype=torch.uint8, device="cuda")
    cols = k // 32 if fp4 else k // 128
    words = dg.dg_packed_sf_words(n, cols)
    sfb = torch.empty(groups * words, dtype=torch.int32, device="cuda")
    for g in range(groups):
        x = torch.randn((n, k), generator=gen, device="cuda", dtype=torch.float32)
        if fp4:
            e = torch.empty((n, cols), dtype=torch.uint8, device="cuda")
            dg.dg_quantize_fp4(x, b[g], e)
            dg.dg_pack_sf(e, n, sfb[g * words:(g + 1) * words], row_div=1)
        else:
            e = torch.empty(((n + 127) // 128, cols), dtype=torch.uint8, device="cuda")
            dg.dg_quantize_fp8(x, b[g], e, 128)
            dg.dg_pack_sf(e, n, sfb[g * words:(g + 1) * words], row_div=128)
        del x, e
    return b, sfb


def grouped_cases(dg, torch, workload, gen, seed):
    """[(name, call, flops, algorithmic bytes)] for the grouped / FP4 configs:
    contiguous (MoE prefill, 8 groups of U[6000,10000] rows padded to 128),
    masked (MoE decode, 32 groups, max_m 256, masked_m ~ U[0, 2 expected_m]),
    fp4 (dense M=4096 and contiguous with e2m1 weights)."""
    import numpy as np
    rng = np.random.default_rng(seed)
    cases = []

    def contiguous(n, k, fp4, nn=False):
        rows = rng.integers(CONTIG_ROWS[0], CONTIG_ROWS[1] + 1, CONTIG_GROUPS)
        mi = np.concatenate([np.concatenate([np.full(r, g, np.int32), np.full(-r % 128, -1, np.int32)])
                             for g, r in enumerate(rows)])
        m_total, valid = mi.size, int(rows.sum())
        a, sfa = quant_a_dev(dg, torch, m_total, k, gen)
        b, sfb = quant_b_dev(dg, torch, CONTIG_GROUPS, n, k, gen, fp4)
        d = torch.empty((m_total, n), dtype=torch.bfloat16, device="cuda")
        t_mi = torch.from_numpy(mi).cuda()
        fn = dg.dg_m_grouped_fp8_fp4_gemm_nt_contiguous if fp4 else dg.dg_m_grouped_fp8_gemm_nt_contiguous
        if nn:
            # the same weights stored [G][K][N] (not transposed)
            b = b.transpose(1, 2).contiguous()
            fn = dg.dg_m_grouped_fp8_gemm_nn_contiguous
        bb = CONTIG_GROUPS * n * k // (2 if fp4 else 1)
        by = valid * k + bb + 2 * valid * n + (sfa.numel() + sfb.numel()) * 4 + 4 * m_total
        kind = "nn-contiguous" if nn else "contiguous"
        name = f"{kind}{'-fp4' if fp4 else ''} G={CONTIG_GROUPS} M={m_total} ({valid} valid) N={n} K={k}"
        cases.append((name, lambda: fn(a, sfa, b, sfb, None, d, t_mi), 2.0 * valid * n * k, by))

    if workload == "contiguous":
        for (n, k) in GROUPED_NK:
            contiguous(n, k, False)
    elif workload == "nn_contiguous":
        for (n, k) in GROUPED_NK:
            contiguous(n, k, False, nn=True)
    elif workload == "kgrouped_tn":
        # weight gradient of the contiguous configuration's projections:
        # forward D[tokens, n] = X[tokens, k] W[n, k]^T per expert, so
        # dW[g] [n, k] = dY_g^T X_g, K-grouped over the 8 experts' tokens
        # (U[6000, 10000] per expert, padded to 128); dY and X quantised 1x128
        # along the token axis (one scale per column and 128 tokens)
        for (n, k) in GROUPED_NK:
            toks = rng.integers(CONTIG_ROWS[0], CONTIG_ROWS[1] + 1, CONTIG_GROUPS)
            ks = ((toks + 127) // 128 * 128).astype(np.int32)
            kt = int(ks.sum())

            def col_quant(cols):
                x = torch.randn((cols, kt), generator=gen, device="cuda", dtype=torch.float32)
                q = torch.empty((cols, kt), dtype=torch.uint8, device="cuda")
                e = torch.empty((cols, kt // 128), dtype=torch.uint8, device="cuda")
                dg.dg_quantize_fp8(x, q, e, 1)
                del x
                sf = torch.empty(dg.dg_packed_sf_words(cols, kt // 128), dtype=torch.int32, device="cuda")
                dg.dg_pack_sf(e, cols, sf, row_div=1)
                return q.t().contiguous(), sf

            a, sfa = col_quant(n)
            b, sfb = col_quant(k)
            d = torch.empty((CONTIG_GROUPS, n, k), dtype=torch.bfloat16, device="cuda")
            t_ks = torch.from_numpy(ks).cuda()
            by = kt * n + kt * k + 2 * CONTIG_GROUPS * n * k + (sfa.numel() + sfb.numel()) * 4
            name = f"k-grouped-tn G={CONTIG_GROUPS} K={kt} M={n} N={k}"
            cases.append((name, (lambda a=a, sfa=sfa, b=b, sfb=sfb, d=d, t_ks=t_ks:
                                 dg.dg_k_grouped_fp8_gemm_tn_contiguous(a, sfa, b, sfb, None, d, t_ks)),
                          2.0 * kt * n * k, by))
    elif workload == "masked":
        G, max_m = MASKED_GROUPS, MASKED_MAX_M
        for (n, k) in GROUPED_NK:
            b, sfb = quant_b_dev(dg, torch, G, n, k, gen)
            for em in MASKED_EXPECTED:
                mm = np.minimum(rng.integers(0, 2 * em + 1, G), max_m).astype(np.int32)
                a, sfa = quant_a_dev(dg, torch, max_m, k, gen, groups=G)
                a = a.view(G, max_m, k)
                d = torch.empty((G, max_m, n), dtype=torch.bfloat16, device="cuda")
                t_mm = torch.from_numpy(mm).cuda()
                valid = int(mm.sum())
                by = valid * k + G * n * k + 2 * valid * n + (valid * (k // 128)) + sfb.numel() * 4
                name = f"masked G={G} max_m={max_m} expected_m={em} ({valid} valid rows) N={n} K={k}"
                cases.append((name, (lambda a=a, sfa=sfa, b=b, sfb=sfb, d=d, t_mm=t_mm, em=em:
                                     dg.dg_m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, d, t_mm, expected_m=em)),
                              2.0 * valid * n * k, by))
    elif workload == "moe_decode_fp4":
        # one MoE decode step per expected_m with FP4 expert weights:
        # linear1 (N = 2 x 2048 gate/up rows interleaved by 64, K = 7168) with
        # SwiGLU fused, then linear2 (N = 7168, K = 2048)
        G, max_m = MASKED_GROUPS, MASKED_MAX_M
        b1, sfb1 = quant_b_dev(dg, torch, G, 4096, 7168, gen, fp4=True)
        b2, sfb2 = quant_b_dev(dg, torch, G, 7168, 2048, gen, fp4=True)
        for em in MASKED_EXPECTED:
            mm = np.minimum(rng.integers(0, 2 * em + 1, G), max_m).astype(np.int32)
            t_mm = torch.from_numpy(mm).cuda()
            valid = int(mm.sum())
            a1, sfa1 = quant_a_dev(dg, torch, max_m, 7168, gen, groups=G)
            a1 = a1.view(G, max_m, 7168)
            act = torch.empty((G, max_m, 2048), dtype=torch.bfloat16, device="cuda")
            a2, sfa2 = quant_a_dev(dg, torch, max_m, 2048, gen, groups=G)
            a2 = a2.view(G, max_m, 2048)
            out = torch.empty((G, max_m, 7168), dtype=torch.bfloat16, device="cuda")
            by1 = valid * 7168 + G * 4096 * 7168 // 2 + 2 * valid * 2048 + sfb1.numel() * 4
            by2 = valid * 2048 + G * 7168 * 2048 // 2 + 2 * valid * 7168 + sfb2.numel() * 4
            cases.append((f"linear1+SwiGLU fp4 G={G} expected_m={em} ({valid} valid rows) N=4096 K=7168",
                          (lambda a=a1, sfa=sfa1, d=act, t=t_mm, em=em:
                           dg.dg_m_grouped_fp8_fp4_gemm_nt_masked_swiglu(a, sfa, b1, sfb1, d, t, expected_m=em)),
                          2.0 * valid * 4096 * 7168, by1))
            cases.append((f"linear2 fp4 G={G} expected_m={em} ({valid} valid rows) N=7168 K=2048",
                          (lambda a=a2, sfa=sfa2, d=out, t=t_mm, em=em:
                           dg.dg_m_grouped_fp8_fp4_gemm_nt_masked(a, sfa, b2, sfb2, d, t, expected_m=em)),
                          2.0 * valid * 7168 * 2048, by2))
    elif workload == "bf16":
        # dense bf16 at the M = 4096 sweep shapes, with cuBLAS (torch.matmul)
        # on the same operands as a library reference
        for (n, k) in DENSE_NK:
            m = 4096
            a = torch.randn((m, k), generator=gen, device="cuda", dtype=torch.float32).to(torch.bfloat16)
            b = torch.randn((n, k), generator=gen, device="cuda", dtype=torch.float32).to(torch.bfloat16)
            d = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
            d_ref = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
            cases.append((f"bf16 M={m} N={n} K={k}", (lambda a=a, b=b, d=d: dg.dg_bf16_gemm_nt(a, b, None, d)),
                          2.0 * m * n * k, 2 * (m * k + n * k + m * n),
                          (lambda a=a, b=b, d_ref=d_ref: torch.matmul(a, b.t(), out=d_ref))))
    elif workload == "promotion":
        # the two ways of applying the scales on the same operands: inside the
        # block-scaled MMA (the library's plan, and forced to 128-wide tiles
        # like the promotion kernel), and per-K-block promotion
        for (m, n, k) in [(4096, 7168, 16384), (64, 7168, 16384), (4096, 4096, 7168), (4096, 7168, 2048)]:
            x = make_inputs(dg, torch, m, n, k, gen)
            f, by = flops(m, n, k), alg_bytes(m, n, k)

            def scaled(x=x, bn=0):
                if bn:
                    dg.dg_set_tile_config(bn, 0)
                try:
                    dg.dg_fp8_gemm_nt(x["a"], x["sfa"], x["b"], x["sfb"], x["c"], x["d"])
                finally:
                    if bn:
                        dg.dg_set_tile_config(0, 0)
            cases.append((f"block-scaled MMA M={m} N={n} K={k}", scaled, f, by))
            cases.append((f"block-scaled MMA, 128-wide tiles M={m} N={n} K={k}",
                          (lambda x=x: scaled(x, 128)), f, by))
            cases.append((f"per-K-block promotion M={m} N={n} K={k}",
                          (lambda x=x: dg.dg_fp8_gemm_nt_promoted(x["a"], x["sfa"], x["b"], x["sfb"], x["c"], x["d"])),
                          f, by))
    elif workload == "fp4":
        for (n, k) in GROUPED_NK:
            m = 4096
            a, sfa = quant_a_dev(dg, torch, m, k, gen)
            b, sfb = quant_b_dev(dg, torch, 1, n, k, gen, fp4=True)
            b = b[0]
            d = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
            by = m * k + n * k // 2 + 2 * m * n + (sfa.numel() + sfb.numel()) * 4
            cases.append((f"dense-fp4 M={m} N={n} K={k}",
                          (lambda a=a, sfa=sfa, b=b, sfb=sfb, d=d: dg.dg_fp8_fp4_gemm_nt(a, sfa, b, sfb, None, d)),
                          2.0 * m * n * k, by))
        for (n, k) in GROUPED_NK:
            contiguous(n, k, True)
    return cases


def make_flush(torch):
    """L2 flush between timed calls: write 256 MB (> 126 MB L2), then read
    another 256 MB so that L2 ends up holding clean lines of unrelated data:
    no input of the timed call is cached and no dirty line of the flush is
    written back inside it."""
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    flush_rd = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device="cuda")

    def flush_l2():
        flush.zero_()
        flush_rd.max()
    return flush_l2


def time_calls(torch, calls, steps, warmup, flush_l2):
    """Mean CUDA-event time (ms) of each call over `steps` steps, each call
    alone after an L2 flush; every step is enqueued behind a short device
    sleep so no timed call waits for the host.  Returns (ms list, launches of
    this library inside the timed steps)."""
    import moe_grouped_gemm_06_b200 as dg
    stream = torch.cuda.current_stream()

    def step(events):
        torch.cuda._sleep(HOLD_CYCLES)
        for i, call in enumerate(calls):
            flush_l2()
            if events is not None:
                events[i][0].record(stream)
            call()
            if events is not None:
                events[i][1].record(stream)

    for _ in range(warmup):
        step(None)
    torch.cuda.synchronize()
    if steps <= 0:
        return [], 0
    events = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in calls]
              for _ in range(steps)]
    launches0 = dg.dg_launch_count()
    for s_ in range(steps):
        step(events[s_])
    torch.cuda.synchronize()
    launches = dg.dg_launch_count() - launches0
    ms = [sum(events[s_][i][0].elapsed_time(events[s_][i][1]) for s_ in range(steps)) / steps
          for i in range(len(calls))]
    return ms, launches


def case_entries(cases, ms, tensor_peak, hbm, ref_ms=None):
    """Per-case TFLOP/s, GB/s, the binding roofline and the fraction of it."""
    ridge = tensor_peak * 1e12 / (hbm * 1e9)
    out = []
    for i, ((name, _, f, by), m_) in enumerate(zip(cases, ms)):
        tf, gbs = f / (m_ * 1e-3) / 1e12, by / (m_ * 1e-3) / 1e9
        bound = "tensor" if f / by >= ridge else "hbm"
        entry = {"case": name, "us": round(m_ * 1e3, 2), "tflops": round(tf, 1), "gbs": round(gbs, 1),
                 "bound": bound, "frac": round(tf / tensor_peak if bound == "tensor" else gbs / hbm, 4)}
        if ref_ms is not None and ref_ms[i] is not None:
            entry["cublas_us"] = round(ref_ms[i] * 1e3, 2)
            entry["cublas_tflops"] = round(f / (ref_ms[i] * 1e-3) / 1e12, 1)
        out.append(entry)
    return out


def run_grouped(args, dg, torch, rank, world, use_dist, local_rank):
    """--workload contiguous | masked | fp4 | ...: each case timed alone (L2
    flushed before every call), one JSON line with per-case TFLOPS, GB/s
    and roofline fraction."""
    gen = torch.Generator(device="cuda")
    gen.manual_seed(4321 + rank)
    cases = grouped_cases(dg, torch, args.workload, gen, 99 + rank)
    graphs = []
    if args.graph:
        # one CUDA graph per case (the calls read their group metadata on the
        # device, so a captured launch is replayable); first call eager
        cap = torch.cuda.Stream()
        for i, case in enumerate(cases):
            name, call = case[0], case[1]
            with torch.cuda.stream(cap):
                call()
            cap.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                call()
            # the graph holds raw pointers into the case's tensors: keep the
            # original call (whose closure owns them) alive with the graph
            graphs.append((g, call))
            cases[i] = (name, g.replay) + tuple(case[2:])
    flush_l2 = make_flush(torch)

    refs = [c[4] if len(c) > 4 else None for c in cases]
    cases = [c[:4] for c in cases]
    time_calls(torch, [c[1] for c in cases], 0, max(args.warmup, 1), flush_l2)   # warm-up only
    err = dg.dg_get_last_error()
    assert err == 0, f"device error during warm-up: {dg.status_string(err)} ({err})"
    sampler = ClockSampler(local_rank)
    if use_dist:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    ms, launches = time_calls(torch, [c[1] for c in cases], args.steps, 0, flush_l2)
    clocks = sampler.stop()
    err = dg.dg_get_last_error()
    assert err == 0, f"device error during timing: {dg.status_string(err)} ({err})"
    # library references (cuBLAS for bf16), timed the same way, after ours
    ref_ms = [None] * len(cases)
    if any(r is not None for r in refs):
        idx = [i for i, r in enumerate(refs) if r is not None]
        rms, _ = time_calls(torch, [refs[i] for i in idx], args.steps, args.warmup, flush_l2)
        for i, v in zip(idx, rms):
            ref_ms[i] = v
    step_ms_max = max_over_ranks(sum(ms), use_dist, "cuda")
    peaks, peak_kind = load_peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_PER_BF16
    hbm = peaks["hbm_gbs"]
    tensor_peak = peaks["bf16_tflops"] if args.workload == "bf16" else fp8_peak
    per_case = case_entries(cases, ms, tensor_peak, hbm, ref_ms)
    dom = max(range(len(cases)), key=lambda i: ms[i])
    pc = per_case[dom]
    roofline = {"bound": pc["bound"], "achieved": pc["tflops"] if pc["bound"] == "tensor" else pc["gbs"],
                "peak": round(tensor_peak, 1) if pc["bound"] == "tensor" else hbm,
                "unit": "TFLOP/s" if pc["bound"] == "tensor" else "GB/s", "frac": pc["frac"], "traffic": None,
                "kernel": f"gemm_kernel on {pc['case']}",
                "peak_source": f"{peak_kind}: FP8 = bf16 burst {peaks['bf16_tflops']} x {FP8_PER_BF16}; HBM {hbm} GB/s"}
    if rank == 0:
        value = whole_job_tflops(world, sum(c[2] for c in cases), step_ms_max)
        line = {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": round(step_ms_max, 4), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
                "config": {"workload": args.workload, "cases": len(cases), "cuda_graph": bool(args.graph),
                           "l2": "flushed before every timed call: 256 MB write then 256 MB read, not timed",
                           "parallelism": f"replicas x{world}"},
                "roofline": roofline, "cpu_baseline": None, "e2e": None, "gpu_launches": int(launches),
                "clocks": clocks, "per_case": per_case}
        print(json.dumps(line), flush=True)


def measure_configs(dg, torch, rank, steps, warmup, flush_l2, fp8_peak, hbm):
    """The other configurations, each case timed alone after an L2 flush
    like the sweep: the small dense case (128 x 512 x 1024, C = 0), the MoE
    prefill (contiguous, 2 cases), the MoE decode (masked, 6 cases) and
    FP8 x FP4 (dense and contiguous, 4 cases).  Returns {name: [per-case]}
    and the library launches inside their timed steps."""
    gen = torch.Generator(device="cuda")
    gen.manual_seed(4321 + rank)
    out, launches = {}, 0
    small = make_inputs(dg, torch, 128, 512, 1024, gen)
    small_case = [("dense M=128 N=512 K=1024 C=0",
                   lambda x=small: dg.dg_fp8_gemm_nt(x["a"], x["sfa"], x["b"], x["sfb"], None, x["d"]),
                   flops(128, 512, 1024), alg_bytes(128, 512, 1024, with_c=False))]
    groups = [("dense_small", small_case)]
    for key, wl in (("contiguous_prefill", "contiguous"), ("masked_decode", "masked"), ("fp8xfp4", "fp4")):
        groups.append((key, [c[:4] for c in grouped_cases(dg, torch, wl, gen, 99 + rank)]))
    for key, cases in groups:
        ms, n = time_calls(torch, [c[1] for c in cases], steps, warmup, flush_l2)
        launches += n
        out[key] = case_entries(cases, ms, fp8_peak, hbm)
    del groups, small
    torch.cuda.empty_cache()
    return out, launches


def probe_tensor_peaks(dg, torch, kblocks=4096, reps=3):
    """TFLOP/s of the tensor pipe alone: the library's own tcgen05 loop (one
    CTA per SM, operands resident in shared memory, no global traffic), best
    of `reps` launches timed with CUDA events, for the block-scaled FP8 MMA
    the GEMMs issue (also at N = 32, 64 and 192: the cost of other widths), the
    plain FP8 MMA and bf16, at N = 128 and 256."""
    stream = torch.cuda.current_stream()
    out = {}
    for kind in ("fp8_block_scaled", "fp8_plain", "bf16"):
        for bn in ((32, 64, 128, 192, 256) if kind == "fp8_block_scaled" else (128, 256)):
            dg.dg_probe_mma_peak(kind, bn, 256)
            best = None
            for _ in range(reps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                f = dg.dg_probe_mma_peak(kind, bn, kblocks)
                e1.record(stream)
                torch.cuda.synchronize()
                t = f / (e0.elapsed_time(e1) * 1e-3) / 1e12
                best = t if best is None else max(best, t)
            out[f"{kind}_n{bn}"] = round(best, 1)
    err = dg.dg_get_last_error()
    assert err == 0, f"device error in the tensor probe: {dg.status_string(err)} ({err})"
    return out


# ---------------------------------------------------------------- CPU oracle

def oracle_prepare(shapes, seed=0):
    """Host inputs for the CPU oracle: for each shape, R = min(threads, M)
    rows of A (so every OpenMP thread of the oracle's row loop has a row)
    and the whole B, quantised by the oracle; B is shared per (N, K)."""
    import oracle
    import synth
    oracle.build()
    threads = oracle.num_threads()
    bcache, prepared = {}, []
    for (m, n, k) in shapes:
        if (n, k) not in bcache:
            bcache[(n, k)] = oracle.quantize_fp8(synth.normal_f32(seed + n + k, (n, k)), 128)
        qb, eb = bcache[(n, k)]
        r = min(threads, m)
        qa, ea = oracle.quantize_fp8(synth.normal_f32(seed + m + n + k, (r, k)), 1)
        c = synth.normal_bf16_bits(seed + 7 + m, (r, n))
        prepared.append((r, n, k, qa, ea, qb, eb, c))
    return prepared, threads


def oracle_step(prepared):
    """One pass of the CPU oracle over the sample; returns its FLOPs."""
    import oracle
    f = 0.0
    for (r, n, k, qa, ea, qb, eb, c) in prepared:
        oracle.gemm(qa, ea, qb, eb, c=c)
        f += 2.0 * r * n * k
    return f


def oracle_sample_text(prepared, threads, passes):
    rows = sorted({p[0] for p in prepared})
    return (f"{passes} pass(es) over the {len(prepared)} sweep shapes; per shape R = min(threads, M) "
            f"= {rows} full output rows (all N columns, full K); CPU FP64 oracle, {threads} OpenMP threads")


def oracle_sample_tflops(shapes, seconds):
    """The CPU oracle, as it stands, on a bounded sample of the sweep (about
    `seconds` of wall time).  Returns (TFLOPS, threads, description)."""
    prepared, threads = oracle_prepare(shapes)
    total, passes = 0.0, 0
    t0 = time.perf_counter()
    while True:
        total += oracle_step(prepared)
        passes += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return total / dt / 1e12, threads, oracle_sample_text(prepared, threads, passes)


def reference_arm(args, rank):
    """--impl reference: the CPU oracle timed per step on a bounded sample of
    the same sweep (rank 0 only; other ranks exit without work)."""
    if rank != 0:
        return
    shapes = shapes_from(args)
    prepared, threads = oracle_prepare(shapes)
    for _ in range(args.warmup):
        oracle_step(prepared)
    t0 = time.perf_counter()
    total = 0.0
    for _ in range(args.steps):
        total += oracle_step(prepared)
    dt = time.perf_counter() - t0
    value = total / dt / 1e12
    sample = "per step: " + oracle_sample_text(prepared, threads, 1)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": "dense NT FP8 sweep (sampled rows), DeepSeek-V3 shapes", "shapes": len(shapes)},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- main

def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, rank)
        return

    import torch
    import torch.distributed as dist
    import moe_grouped_gemm_06_b200 as dg

    torch.cuda.set_device(local_rank)
    use_dist = world > 1
    if use_dist:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local_rank))

    if args.workload != "dense":
        run_grouped(args, dg, torch, rank, world, use_dist, local_rank)
        if use_dist:
            dist.barrier()
            dist.destroy_process_group()
        return

    shapes = shapes_from(args)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(1234 + rank)
    inputs = [make_inputs(dg, torch, m, n, k, gen) for (m, n, k) in shapes]
    flush_l2 = make_flush(torch)
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()

    def call(x):
        dg.dg_fp8_gemm_nt(x["a"], x["sfa"], x["b"], x["sfb"], x["c"], x["d"], stream=stream)

    def sweep(events):
        # Hold the stream in a short device-side sleep while the host enqueues
        # the whole step, so no timed call waits for the host to launch it.
        torch.cuda._sleep(HOLD_CYCLES)
        for i, x in enumerate(inputs):
            flush_l2()
            if events is not None:
                events[i][0].record(stream)
            call(x)
            if events is not None:
                events[i][1].record(stream)

    for _ in range(max(args.warmup, 1)):
        sweep(None)
    err = dg.dg_get_last_error()
    assert err == 0, f"device error during warm-up: {dg.status_string(err)} ({err})"
    probe = probe_tensor_peaks(dg, torch)

    events = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in shapes] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank)
    if use_dist:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    launches0 = dg.dg_launch_count()
    wall0 = time.perf_counter()
    for s in range(args.steps):
        sweep(events[s])
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    launches = dg.dg_launch_count() - launches0
    peaks, peak_kind = load_peaks()
    fp8_peak = peaks["bf16_tflops"] * FP8_PER_BF16
    hbm = peaks["hbm_gbs"]
    per_config, config_launches = None, 0
    if not args.shape and not args.no_configs:
        per_config, config_launches = measure_configs(dg, torch, rank, args.steps, args.warmup, flush_l2,
                                                      fp8_peak, hbm)
    if use_dist:
        dist.barrier()
    clocks = sampler.stop()
    err = dg.dg_get_last_error()
    assert err == 0, f"device error during timing: {dg.status_string(err)} ({err})"

    per_shape_ms = [sum(events[s][i][0].elapsed_time(events[s][i][1]) for s in range(args.steps)) / args.steps
                    for i in range(len(shapes))]
    step_ms = sum(per_shape_ms)
    step_ms_max = max_over_ranks(step_ms, use_dist, "cuda")

    sweep_flops = sum(flops(*s) for s in shapes)
    value = whole_job_tflops(world, sweep_flops, step_ms_max)

    ridge = fp8_peak * 1e12 / (hbm * 1e9)
    per_shape = []
    for (m, n, k), ms in zip(shapes, per_shape_ms):
        f, by = flops(m, n, k), alg_bytes(m, n, k)
        tf = f / (ms * 1e-3) / 1e12
        gbs = by / (ms * 1e-3) / 1e9
        bound = "tensor" if f / by >= ridge else "hbm"
        frac = tf / fp8_peak if bound == "tensor" else gbs / hbm
        per_shape.append({"m": m, "n": n, "k": k, "us": round(ms * 1e3, 2), "tflops": round(tf, 1),
                          "gbs": round(gbs, 1), "bound": bound, "frac": round(frac, 4)})

    dom = max(range(len(shapes)), key=lambda i: per_shape_ms[i])
    (dm, dn, dk) = shapes[dom]
    dom_bound = per_shape[dom]["bound"]
    dom_workload = f"dense_{dm}x{dn}x{dk}"
    if dom_bound == "tensor":
        achieved = flops(dm, dn, dk) / (per_shape_ms[dom] * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(fp8_peak, 1),
                    "unit": "TFLOP/s", "frac": round(achieved / fp8_peak, 4)}
    else:
        achieved = alg_bytes(dm, dn, dk) / (per_shape_ms[dom] * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                    "frac": round(achieved / hbm, 4)}
    fp8_probe = max(probe["fp8_block_scaled_n128"], probe["fp8_block_scaled_n256"])
    if dom_bound == "tensor":
        roofline["frac_vs_probe"] = round(achieved / fp8_probe, 4)
        roofline["frac_vs_spec"] = round(achieved / FP8_SPEC_TFLOPS, 4)
    roofline["traffic"] = recorded_traffic(dom_workload)
    roofline["kernel"] = f"gemm_kernel on {dom_workload} ({per_shape_ms[dom] / step_ms * 100:.0f}% of step time)"
    roofline["peak_source"] = (f"{peak_kind}: FP8 = bf16 burst {peaks['bf16_tflops']} x {FP8_PER_BF16} "
                               f"(nominal FP8:BF16 ratio); HBM {hbm} GB/s; beside it the block-scaled FP8 "
                               f"tcgen05 loop measured in this run, {fp8_probe} TFLOP/s (frac_vs_probe), and the "
                               f"nominal dense FP8 peak {FP8_SPEC_TFLOPS} TFLOP/s (frac_vs_spec)")

    # ---- end to end through the C ABI from pinned host buffers
    e2e = None
    if not args.no_e2e:
        host = []
        h2d = d2h = 0
        for x in inputs:
            hx = {key: x[key].cpu().pin_memory() for key in ("a", "sfa", "b", "sfb", "c")}
            hx["d"] = torch.empty(x["d"].shape, dtype=x["d"].dtype).pin_memory()
            host.append(hx)
            h2d += sum(hx[key].numel() * hx[key].element_size() for key in ("a", "sfa", "b", "sfb", "c"))
            d2h += hx["d"].numel() * hx["d"].element_size()

        # Copies in, GEMM and copy out of each shape on three streams, ordered
        # by events: the inputs of shape i+1 travel to the device while shape
        # i computes and its D travels back (host-to-device and device-to-host
        # copies use separate copy engines), as a client pipelining its calls
        # would; a step's inputs are not overwritten before the previous
        # step's GEMM of that shape has read them, nor its D before it is out.
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        done_prev = [None] * len(inputs)   # GEMM of shape i finished (last step)
        out_prev = [None] * len(inputs)    # D of shape i copied out (last step)

        def e2e_step():
            for i, (x, hx) in enumerate(zip(inputs, host)):
                if done_prev[i] is not None:
                    s_in.wait_event(done_prev[i])
                with torch.cuda.stream(s_in):
                    for key in ("a", "sfa", "b", "sfb", "c"):
                        x[key].copy_(hx[key], non_blocking=True)
                    arrived = ev()
                    arrived.record(s_in)
                stream.wait_event(arrived)
                if out_prev[i] is not None:
                    stream.wait_event(out_prev[i])
                call(x)
                done = ev()
                done.record(stream)
                s_out.wait_event(done)
                with torch.cuda.stream(s_out):
                    hx["d"].copy_(x["d"], non_blocking=True)
                    out = ev()
                    out.record(s_out)
                done_prev[i], out_prev[i] = done, out

        e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_steps = max(1, min(args.steps, 5))
        if use_dist:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(s_in)
        for _ in range(e2e_steps):
            e2e_step()
        s_in.wait_stream(s_out)
        e1.record(s_in)
        torch.cuda.synchronize()
        ems = e0.elapsed_time(e1) / e2e_steps
        ems_max = max_over_ranks(ems, use_dist, "cuda")
        e2e = {"value": round(whole_job_tflops(world, sweep_flops, ems_max), 2), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(ems_max, 3),
               "pipeline": "per shape: H2D of the inputs, GEMM, D2H of D on three streams ordered by events"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        v, cores, sample = oracle_sample_tflops(shapes, args.cpu_seconds)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(step_ms_max, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
            "config": {"workload": ("dense NT FP8 sweep, DeepSeek-V3 shapes M in {64,128,4096} x (N,K) in "
                                    "{(2112,7168),(24576,1536),(32768,512),(7168,16384),(4096,7168),(7168,2048)}"
                                    if not args.shape else f"dense NT FP8 {args.shape}"),
                       "shapes": len(shapes), "accumulate": "f32 (TMEM)", "out": "bf16", "c": "N(0,1) bf16",
                       "scales": "UE8M0 1x128 (A), 128x128 (B)",
                       "l2": "flushed before every timed GEMM call: 256 MB write then 256 MB read, not timed",
                       "parallelism": f"replicas x{world}", "wall_s_timed_region": round(wall, 3)},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(launches),
            "clocks": clocks, "per_shape": per_shape,
            "per_config": per_config, "per_config_launches": int(config_launches),
            "tensor_peak_probe": probe,
        }
        print(json.dumps(line), flush=True)
    if use_dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
