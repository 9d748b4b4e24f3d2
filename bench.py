"""Benchmark of the optimizer-step hot path on synthetic layer sets.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl mine|reference]

One "step" applies the whole hot path to one full synthetic layer set resident
in HBM: a Muon step, a SOAP step (eigenbasis refresh every step) and a FOAM step
(adaptive refresh check every 10 steps), all on the same weights and gradients
(per rank: N ranks each own one layer set, no collective on the data path =
weak scaling).  Rank 0 prints one JSON line.

Timing: W untimed warm-up steps; K timed steps between a barrier and
cudaDeviceSynchronize on both sides, CUDA events on the launching stream, max
over ranks.  Inputs exceed the 126 MB L2 many times over.  Every library launch
inside the timed region is bracketed by events (mao_profile_start), which gives
each kernel's live duration for the roofline entry and the launch count.
"""

from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

WORKLOADS = {
    # name: (description, optimizers run per step, default gradient dtype bf16?)
    "dense8b_moe": ("8B-dense block (7 matrices) + 256-expert MoE bank (768 matrices), bf16 G ~ N(0,0.01^2)*s_e",
                    True),
    "dense8b_block": ("8B-dense block alone (7 matrices), bf16 G ~ N(0,0.01^2)", True),
    "moe_bank": ("256-expert MoE bank alone (768 matrices), bf16 G ~ N(0,0.01^2)*s_e", True),
    "gpt2_124m": ("GPT-2-124M-shaped set, 48 matrices, bf16 G ~ N(0,0.02^2), Muon+ Col-Row", True),
    "gpt2_760m": ("GPT-2-760M-shaped set, 96 matrices, fp32 G ~ N(0,0.01^2)", False),
    "muon_single": ("one 256x512 fp32 weight", False),
}
MUON_NORM = {"gpt2_124m": "col_row"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["mine", "reference"], default="mine")
    ap.add_argument("--mode", choices=["sets", "layerwise"], default="sets",
                    help="sets: every rank steps its own layer set (weak scaling, no collective); layerwise: one "
                         "layer set split over the ranks by owner, updated weights exchanged by all-gather-V "
                         "(strong scaling)")
    ap.add_argument("--workload", default="dense8b_moe", choices=sorted(WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--experts", type=int, default=256,
                    help="experts of the MoE bank (moe_bank, dense8b_moe); fewer make a small case of the same "
                         "shapes for profiling")
    ap.add_argument("--optimizers", default="muon,soap,foam", help="comma list of muon, soap, foam")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--soap-k", type=int, default=1, help="SOAP refreshes its bases every k steps")
    ap.add_argument("--foam-kinds", type=int, default=0,
                    help="instead of the bench line: FOAM alone for steps t = 1..N, each timed on its own, "
                         "and the median ms of plain, check-only and check+refresh steps")
    ap.add_argument("--cpu-budget-s", type=float, default=20.0)
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other configurations' timings (Muon+ on the GPT-2-124M set, FOAM step kinds on "
                         "the GPT-2-760M set) added to the bench line")
    ap.add_argument("--cpu-baseline-full", action="store_true",
                    help="instead of the bench line: time the float64 oracle once on every distinct shape of the "
                         "workload for each optimizer (minutes) and print the table as JSON")
    ap.add_argument("--launch-log", default=None,
                    help="after the measurement, run one more step and write its launch list (kernel, work) here")
    ap.add_argument("--traffic-csv", default=None,
                    help="offline: ncu CSV (dram__bytes_read/write.sum, gpu__time_duration.sum) of a run made with "
                         "--launch-log; folds the last step's launches into --traffic-out (no GPU needed)")
    ap.add_argument("--traffic-out", default=os.path.join(ROOT, "profiles", "ncu_traffic.json"))
    return ap.parse_args()


EXPERTS = [256]  # experts of the MoE bank (set from --experts)


def specs_for(workload, seed):
    from matrix_aware_optimizers_02_b200 import synth
    if workload == "dense8b_moe":
        return synth.specs_dense8b_moe(EXPERTS[0], seed)
    if workload == "moe_bank":
        return synth.specs_moe_bank(EXPERTS[0], seed)
    return synth.WORKLOADS[workload]()


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- peaks / traffic
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    cs = os.path.join(ROOT, "matrix_aware_optimizers_02_b200", "csrc")
    for fn in sorted(os.listdir(cs)):
        if fn.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(cs, fn), "rb") as f:
                h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_name, flops_per_launch, bytes_per_launch):
    """DRAM bytes per launch of a kernel from the committed ncu traffic summary, if the kernel
    sources still match it.  The summary is measured on a workload small enough for ncu; its
    DRAM bytes per algorithmic FLOP (or byte) scale to this launch's work."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("source_hash") != kernel_source_hash():
        return None
    e = d.get("kernels", {}).get(kernel_name)
    if e is None:
        return None
    if flops_per_launch > 0 and e.get("dram_bytes_per_flop") is not None:
        return {"bytes": round(e["dram_bytes_per_flop"] * flops_per_launch),
                "scaled_from": d.get("measured_on"), "by": "algorithmic flops"}
    if bytes_per_launch > 0 and e.get("dram_bytes_per_alg_byte") is not None:
        return {"bytes": round(e["dram_bytes_per_alg_byte"] * bytes_per_launch),
                "scaled_from": d.get("measured_on"), "by": "algorithmic bytes"}
    return None


def roofline_of(name, e, peaks, peak_src, traffic):
    """The roofline object of the bench line for one profiler id: `e` sums its launches
    (n, ms, flops = executed useful FLOP, tc = tensor-core operations issued, planned =
    the host's count of the ungated problems, bytes = algorithmic bytes); `traffic` is
    ncu_traffic()'s scaled DRAM bytes per launch, or None."""
    avg_ms = e["ms"] / e["n"]
    if e["flops"] > 0:
        # tensor-pipe work: the bf16 products issued (six per fp32-faithful multiply-add of
        # three-plane operands), against the bf16 peak
        achieved = (e["tc"] / e["n"]) / (avg_ms * 1e-3) / 1e12
        useful = (e["flops"] / e["n"]) / (avg_ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops_sustained"]
        roof = {"bound": "tensor", "kernel": name, "achieved": round(achieved, 1),
                "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "useful_tflops": round(useful, 1),
                "peak_source": f"{peak_src} bf16 sustained (kernel timed inside a long step); achieved counts "
                               "the bf16 tensor-core products the kernel issued (6 per fp32-faithful "
                               "multiply-add), over the tiles it computed (device counters: the passes "
                               "decided on the device included)"}
        if e["planned"] < e["flops"]:
            roof["useful_tflops_host_counted"] = round((e["planned"] / e["n"]) / (avg_ms * 1e-3) / 1e12, 1)
    else:
        achieved = (e["bytes"] / e["n"]) / (avg_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "kernel": name, "achieved": round(achieved, 1),
                "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                "peak_source": f"{peak_src} HBM copy"}
    roof["traffic"] = traffic["bytes"] if traffic else None
    if traffic:
        roof["traffic_source"] = f"ncu DRAM bytes per {traffic['by']} on {traffic['scaled_from']}, scaled to this launch"
    roof["launches"] = e["n"]
    roof["avg_launch_ms"] = round(avg_ms, 4)
    return roof


def write_launch_log(args, lib, L, LS, t, stream):
    """One more step with the launch profiler recording kernel ids and work only."""
    import torch
    torch.cuda.synchronize()
    lib.mao_profile_start(None, None, 0)
    LS.step(t, stream)
    n = lib.mao_profile_stop()
    torch.cuda.synchronize()
    info = (L.LaunchInfo * max(n, 1))()
    L.check(lib.mao_profile_start(None, info, n))
    # the range lets a profiler capture this step alone (ncu --nvtx --nvtx-include)
    with torch.cuda.nvtx.range("mao.bench.logged_step"):
        LS.step(t, stream)  # the same t: the same launch plan
    m = lib.mao_profile_stop()
    torch.cuda.synchronize()
    # executed work (device counters for the table-mode products), and the host's count
    rows = [{"kernel": L.KERNEL_NAMES.get(info[i].kernel, str(info[i].kernel)), "flops": info[i].exec_flops,
             "bytes": info[i].bytes, "tc_flops": info[i].exec_tc_flops, "planned_flops": info[i].flops}
            for i in range(min(n, m))]
    with open(args.launch_log, "w") as f:
        json.dump({"workload": args.workload, "optimizers": args.optimizers, "source_hash": kernel_source_hash(),
                   "launches": rows}, f)


def fold_traffic(args):
    """Per kernel id: launches, ncu time and share, DRAM bytes per launch / per algorithmic
    FLOP / per algorithmic byte, and the time-weighted tensor-pipe and DRAM utilisation,
    from the ncu CSV of a --launch-log run (its last len(launches) library launches are the
    logged step).  Metrics absent from the CSV are left out.  Writes --traffic-out (JSON)
    and prints a markdown table."""
    import csv
    with open(args.launch_log) as f:
        log = json.load(f)
    rows = list(csv.reader(open(args.traffic_csv)))
    head = None
    per = {}
    names = {}
    for r in rows:
        if "Kernel Name" in r:
            head = r
            continue
        if head is None or len(r) != len(head):
            continue
        d = dict(zip(head, r))
        try:
            i = int(d["ID"])
        except ValueError:
            continue
        e = per.setdefault(i, {})
        try:
            e[d["Metric Name"]] = float(d["Metric Value"].replace(",", ""))
        except ValueError:
            pass
        names[i] = d["Kernel Name"].split("(")[0].split("<")[0].split()[-1].split("::")[-1]
    ids = sorted(i for i in per if names.get(i, "").startswith(("gemm_tc", "muon_", "pc_", "soap_", "foam_", "qr_",
                                                                   "mop_")))
    launches = log["launches"]
    tail = ids[-len(launches):]
    if len(tail) != len(launches):
        raise SystemExit("fewer ncu launches than logged launches")
    # each profiler id is launched by these kernels (first word of ncu's kernel name)
    fam = {"muon_prep": ["muon_prep_kernel"], "muon_scale": ["muon_scale_kernel"], "muon_stats": ["muon_stats_kernel"],
           "muon_update": ["muon_update_kernel"], "muon_colsq": ["muon_norm_tile_kernel"],
           "muon_colscale": ["muon_norm_final_kernel"], "muon_rowscale": ["muon_norm_tile_kernel",
                                                                          "muon_norm_final_kernel"],
           "mop_init": ["mop_init_kernel"],
           "pc_elementwise": ["pc_momentum_kernel", "pc_split_kernel", "soap_adam_kernel", "foam_rc_partial_kernel",
                              "foam_tau_kernel", "foam_n_kernel"],
           "pc_sort": ["pc_keys_kernel", "pc_argsort_kernel", "pc_gather_cols_kernel", "soap_vperm_kernel"],
           "pc_check": ["pc_check_kernel"], "pc_chol": ["qr_chol_kernel"], "pc_qr_reduce": ["pc_coef_reduce_kernel"],
           "pc_stats": ["pc_stats_kernel"],
           "pc_panel": ["gemm_tc_table_kernel", "gemm_tc_pair_kernel", "qr_gram_reduce_kernel"]}
    for rec, i in zip(launches, tail):
        ok = fam.get(rec["kernel"], ["gemm_tc_table_kernel", "gemm_tc_pair_kernel", "gemm_tc_kernel",
                                     "gemm_tc_pair_class_kernel"])
        if names[i] not in ok:
            raise SystemExit(f"launch {i}: ncu saw {names[i]}, the log says {rec['kernel']}: not aligned")
    agg = {}
    for rec, i in zip(launches, tail):
        m = per[i]
        a = agg.setdefault(rec["kernel"], {"launches": 0, "dram": 0.0, "flops": 0.0, "bytes": 0.0, "ns": 0.0,
                                           "tc_ns": 0.0, "dt_ns": 0.0, "has_dram": False, "has_tc": False})
        ns = m.get("gpu__time_duration.sum", 0.0)
        a["launches"] += 1
        if "dram__bytes_read.sum" in m or "dram__bytes_write.sum" in m:
            a["has_dram"] = True
            a["dram"] += m.get("dram__bytes_read.sum", 0.0) + m.get("dram__bytes_write.sum", 0.0)
        if "sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_elapsed" in m:
            a["has_tc"] = True
            a["tc_ns"] += ns * m["sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_elapsed"]
        if "dram__throughput.avg.pct_of_peak_sustained_elapsed" in m:
            a["dt_ns"] += ns * m["dram__throughput.avg.pct_of_peak_sustained_elapsed"]
        a["flops"] += rec["flops"]
        a["bytes"] += rec["bytes"]
        a["ns"] += ns
    total_ns = sum(a["ns"] for a in agg.values()) or 1.0
    out = {"source_hash": log["source_hash"], "measured_on": log["workload"], "kernels": {}}
    for k, a in sorted(agg.items()):
        rec = {"launches": a["launches"], "ncu_ms": a["ns"] / 1e6, "share": a["ns"] / total_ns}
        if a["has_dram"]:
            rec["dram_bytes_per_launch"] = a["dram"] / a["launches"]
            rec["dram_bytes_per_flop"] = (a["dram"] / a["flops"]) if a["flops"] > 0 else None
            rec["dram_bytes_per_alg_byte"] = (a["dram"] / a["bytes"]) if a["bytes"] > 0 else None
        if a["has_tc"] and a["ns"] > 0:
            rec["tensor_pipe_pct"] = a["tc_ns"] / a["ns"]
        if a["dt_ns"] > 0 and a["ns"] > 0:
            rec["dram_pct"] = a["dt_ns"] / a["ns"]
        out["kernels"][k] = rec
    with open(args.traffic_out, "w") as f:
        json.dump(out, f, indent=1)
    print(f"| kernel id | launches | ncu ms | share | tensor pipe % | DRAM % | DRAM B / alg B | DRAM B / FLOP |")
    print("|---|---|---|---|---|---|---|---|")
    for k, r in sorted(out["kernels"].items(), key=lambda kv: -kv[1]["share"]):
        def f(x, fmt):
            return fmt.format(x) if x is not None else ""
        print(f"| {k} | {r['launches']} | {r['ncu_ms']:.3f} | {r['share']:.3f} | {f(r.get('tensor_pipe_pct'), '{:.1f}')} | "
              f"{f(r.get('dram_pct'), '{:.1f}')} | {f(r.get('dram_bytes_per_alg_byte'), '{:.2f}')} | "
              f"{f(r.get('dram_bytes_per_flop'), '{:.4f}')} |")


# ----------------------------------------------------------------------------- CPU (oracle) leg
def _ns_flops(m, n):
    a, b = min(m, n), max(m, n)
    return 5 * (4 * a * a * b + 2 * a ** 3)


def _soap_flops(m, n):
    # factors, power step, QR (Householder with explicit Q), two rotations in, one back
    return 2 * m * m * n + 2 * m * n * n + 2 * (m ** 3 + n ** 3) + 8 / 3 * (m ** 3 + n ** 3) + 6 * (m * m * n + m * n * n)


def _foam_flops(m, n, check):
    f = 8 * m * n * n
    if check:
        f += 4 * n ** 3 + 2 * n ** 3 + 8 / 3 * n ** 3
    return f


def cpu_oracle_sample(workload, budget_s, seed, optimizers, t_foam=1):
    """Time the float64 oracle on a bounded sample of the workload's matrices and
    scale to one full layer set.  Returns (ms per layer set, cores, sample text)."""
    from oracle import mao_oracle as O
    specs = specs_for(workload, seed)
    norm = {"col_row": O.NORM_COL_ROW}.get(MUON_NORM.get(workload, "none"), O.NORM_NONE)
    shapes = {}
    for s in specs:
        shapes[(s.m, s.n)] = shapes.get((s.m, s.n), 0) + 1
    models = {"muon": _ns_flops, "soap": _soap_flops, "foam": lambda m, n: _foam_flops(m, n, True)}
    rng = np.random.default_rng(seed)
    total_ms = 0.0
    parts = []
    per_opt_budget = budget_s / max(len(optimizers), 1)
    for opt in optimizers:
        flops = models[opt]
        order = sorted(shapes, key=lambda k: flops(*k))
        timed, spent = {}, 0.0
        for (m, n) in order:
            if spent > per_opt_budget * 0.5 and timed:
                break
            if timed and flops(m, n) / max(flops(*k) / v for k, v in timed.items()) > per_opt_budget:
                break  # one more shape would blow the budget: extrapolate instead
            W = rng.standard_normal((m, n)) * 0.02
            G = rng.standard_normal((m, n)) * 0.01
            t0 = time.perf_counter()
            if opt == "muon":
                O.muon_step(W, G, np.zeros((m, n)), mu=0.95, lr=0.02, norm=norm)
            elif opt == "soap":
                O.soap_step(W, G, O.SoapState.init(m, n), t=1, beta1=0.95, beta2=0.95, eps=1e-8, lr=3e-3)
            else:
                O.foam_step(W, G, O.FoamState.init(m, n), t=1, beta1=0.95, beta2=0.95, eps=1e-8, lr=3e-3)
            dt = time.perf_counter() - t0
            timed[(m, n)] = dt
            spent += dt
        rate = max(flops(*k) / v for k, v in timed.items())
        opt_s = sum(cnt * (timed[k] if k in timed else flops(*k) / rate) for k, cnt in shapes.items())
        total_ms += opt_s * 1e3
        parts.append(f"{opt}: timed {', '.join(f'{m}x{n}' for (m, n) in timed)} ({spent:.1f} s)" +
                     ("" if len(timed) == len(shapes) else ", other shapes scaled by the step's FLOP model"))
    cores = len(os.sched_getaffinity(0))
    sample = ("float64 NumPy oracle, each distinct shape's step time x its multiplicity (SOAP and FOAM steps "
              "with a basis refresh); " + "; ".join(parts))
    return total_ms, cores, sample, blas_threads()


def blas_threads():
    """Threads of the BLAS library NumPy calls (threadpoolctl), or None."""
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads") for d in threadpool_info() if d.get("user_api") == "blas"]
        return max(n) if n else None
    except Exception:
        return None


def cpu_full_table(workload, seed, optimizers):
    """The float64 oracle timed once on every distinct shape of the workload, per optimizer
    (SOAP and FOAM with a basis refresh), and the layer-set total = sum of time x count."""
    from oracle import mao_oracle as O
    specs = specs_for(workload, seed)
    norm = {"col_row": O.NORM_COL_ROW}.get(MUON_NORM.get(workload, "none"), O.NORM_NONE)
    shapes = {}
    for sp in specs:
        shapes[(sp.m, sp.n)] = shapes.get((sp.m, sp.n), 0) + 1
    rng = np.random.default_rng(seed)
    rows, total = [], 0.0
    for opt in optimizers:
        for (m, n), cnt in sorted(shapes.items()):
            W = rng.standard_normal((m, n)) * 0.02
            G = rng.standard_normal((m, n)) * 0.01
            t0 = time.perf_counter()
            if opt == "muon":
                O.muon_step(W, G, np.zeros((m, n)), mu=0.95, lr=0.02, norm=norm)
            elif opt == "soap":
                O.soap_step(W, G, O.SoapState.init(m, n), t=1, beta1=0.95, beta2=0.95, eps=1e-8, lr=3e-3)
            else:
                O.foam_step(W, G, O.FoamState.init(m, n), t=1, beta1=0.95, beta2=0.95, eps=1e-8, lr=3e-3)
            dt = time.perf_counter() - t0
            rows.append({"optimizer": opt, "m": m, "n": n, "count": cnt, "s": round(dt, 3)})
            total += dt * cnt
            print(json.dumps(rows[-1]), file=sys.stderr, flush=True)
    return {"workload": workload, "unit": "ms", "value": round(total * 1e3, 1), "cores": len(os.sched_getaffinity(0)),
            "blas_threads": blas_threads(), "rows": rows}


def committed_cpu_table(workload):
    """The every-shape oracle timing committed under profiles/ for this workload (measured on
    a GPU machine's host by --cpu-baseline-full), or None."""
    p = os.path.join(ROOT, "profiles", f"cpu_oracle_{workload}.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    return {"value": d["value"], "unit": d["unit"], "cores": d["cores"], "blas_threads": d.get("blas_threads"),
            "source": f"profiles/cpu_oracle_{workload}.json (bench.py --cpu-baseline-full, every distinct shape "
                      "timed once, times its count)"}


# ----------------------------------------------------------------------------- ranks
def rank_seed(seed, rank):
    """Each rank owns its own synthetic layer set (weak scaling, no data-path collective)."""
    return seed + 7919 * rank


def reduce_times(values, dist, device):
    """Max over ranks of each per-rank duration: the slowest rank bounds the job."""
    import torch
    tt = torch.tensor(list(values), device=device, dtype=torch.float64)
    if dist is not None:
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return tt.tolist()


def per_layer_set(ms_max, world):
    """ms per layer set for the whole job: `world` layer sets processed in ms_max."""
    return ms_max / world


# ----------------------------------------------------------------------------- the layer set on the GPU
class LayerSet:
    """W, the optimizer states and `n_grad` gradient sets of one synthetic layer set,
    plus, per optimizer, one batch object per gradient set (all sharing W, the states
    and one workspace).  Step k uses gradient set k mod n_grad, so consecutive steps
    see different gradients without any copy between them."""

    def __init__(self, specs, seed, dev, g_bf16, optimizers, norm, soap_k=1, n_grad=3):
        import torch

        from matrix_aware_optimizers_02_b200 import api, synth
        self.torch = torch
        base = synth.torch_muon_inputs(specs, seed, dev, g_bf16=g_bf16)
        self.W = [w for (w, _, _) in base]
        self.G_sets = [[g for (_, g, _) in base]]
        del base
        gen = torch.Generator(device=dev)
        for k in range(1, n_grad):
            gen.manual_seed(seed * 1000003 + k)
            self.G_sets.append([synth.torch_gaussian((sp.m, sp.n), sp.g_std * sp.g_scale, gen, dev,
                                                     torch.bfloat16 if g_bf16 else torch.float32) for sp in specs])
        self.G = self.G_sets[0]
        self.n_grad = n_grad
        self.batches = {}
        z = torch.zeros
        if "muon" in optimizers:
            M = [z(w.shape, device=dev) for w in self.W]
            self.batches["muon"] = [api.MuonBatch(list(zip(self.W, Gs, M)), mu=0.95, lr=0.02, norm=norm,
                                                  with_stats=True, allocate=False) for Gs in self.G_sets]
        if "soap" in optimizers:
            st = []
            for w in self.W:
                m, n = w.shape
                st.append({"M": z((m, n), device=dev), "V": z((m, n), device=dev),
                           "L": torch.eye(m, device=dev) * 1e-6, "R": torch.eye(n, device=dev) * 1e-6,
                           "QL": torch.eye(m, device=dev), "QR": torch.eye(n, device=dev)})
            self.batches["soap"] = [api.SoapBatch([dict(d, W=w, G=g) for d, w, g in zip(st, self.W, Gs)], beta1=0.95,
                                                  beta2=0.95, eps=1e-8, lr=3e-3, refresh="every_k", k=soap_k,
                                                  with_stats=True, allocate=False) for Gs in self.G_sets]
        if "foam" in optimizers:
            st = []
            for w in self.W:
                m, n = w.shape
                st.append({"M": z((m, n), device=dev), "r": z(m, device=dev), "c": z(n, device=dev),
                           "R": torch.eye(n, device=dev) * 1e-6, "QR": torch.eye(n, device=dev)})
            self.batches["foam"] = [api.FoamBatch([dict(d, W=w, G=g) for d, w, g in zip(st, self.W, Gs)], beta1=0.95,
                                                  beta2=0.95, eps=1e-8, lr=3e-3, refresh="adaptive", pf=10, tol=0.1,
                                                  with_stats=True, allocate=False) for Gs in self.G_sets]
        self.order = [o for o in ("muon", "soap", "foam") if o in self.batches]
        # the steps run in order on one stream, so one workspace serves all of them
        ws_bytes = max(b.ws_bytes for bs in self.batches.values() for b in bs)
        self.workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        for bs in self.batches.values():
            for b in bs:
                b.attach_workspace(self.workspace)

    def step(self, t, stream, events=None):
        """Step t (1-based) of every optimizer, on gradient set (t - 1) mod n_grad."""
        gi = (t - 1) % self.n_grad
        for name in self.order:
            b = self.batches[name][gi]
            if events is not None:
                events[name][0].record(stream)
            if name == "muon":
                b()
            else:
                b(t)
            if events is not None:
                events[name][1].record(stream)

    def stats_tensor(self, t):
        """The stats array the first optimizer's step t writes."""
        return self.batches[self.order[0]][(t - 1) % self.n_grad].stats

    def status(self):
        for name, bs in self.batches.items():
            st = bs[0].device_status()
            if st != 0:
                return name, st
        return None


class LayerwiseSet:
    """One layer set split over the ranks by the layer-wise optimizer (whole matrices
    owned by ranks, balanced by the cost model; the updated weights exchanged by the
    all-gather-V).  Every rank holds W and the gradient sets in full (identical on all
    ranks, as after a data-parallel gradient all-reduce) and optimizer state only for
    the matrices it owns.  Same interface as LayerSet."""

    def __init__(self, specs, seed, dev, g_bf16, optimizers, norm, dist, soap_k=1, n_grad=3):
        import torch

        from matrix_aware_optimizers_02_b200 import api, synth
        from matrix_aware_optimizers_02_b200 import layerwise as LW
        self.torch = torch
        base = synth.torch_muon_inputs(specs, seed, dev, g_bf16=g_bf16)
        self.W = [w for (w, _, _) in base]
        self.G_sets = [[g for (_, g, _) in base]]
        del base
        gen = torch.Generator(device=dev)
        for k in range(1, n_grad):
            gen.manual_seed(seed * 1000003 + k)
            self.G_sets.append([synth.torch_gaussian((sp.m, sp.n), sp.g_std * sp.g_scale, gen, dev,
                                                     torch.bfloat16 if g_bf16 else torch.float32) for sp in specs])
        self.G = self.G_sets[0]
        self.n_grad = n_grad
        world, rank = dist.get_world_size(), dist.get_rank()
        kws = {"muon": dict(mu=0.95, lr=0.02, norm=norm),
               "soap": dict(beta1=0.95, beta2=0.95, eps=1e-8, lr=3e-3, refresh="every_k", k=soap_k),
               "foam": dict(beta1=0.95, beta2=0.95, eps=1e-8, lr=3e-3, refresh="adaptive", pf=10, tol=0.1)}
        shapes = [(sp.m, sp.n) for sp in specs]
        z = torch.zeros
        self.order = [o for o in ("muon", "soap", "foam") if o in optimizers]
        self.steps, self.owners, self.owned_count = {}, {}, {}
        batches = []
        for o in self.order:
            owners = LW.assign_owners(shapes, world, o, LW.cost_for(o, kws[o]))
            self.owners[o] = owners
            mine = [i for i, r in enumerate(owners) if r == rank]
            self.owned_count[o] = len(mine)
            state = {}
            for i in mine:
                m, n = shapes[i]
                if o == "muon":
                    state[i] = {"M": z((m, n), device=dev)}
                elif o == "soap":
                    state[i] = {"M": z((m, n), device=dev), "V": z((m, n), device=dev),
                                "L": torch.eye(m, device=dev) * 1e-6, "R": torch.eye(n, device=dev) * 1e-6,
                                "QL": torch.eye(m, device=dev), "QR": torch.eye(n, device=dev)}
                else:
                    state[i] = {"M": z((m, n), device=dev), "r": z(m, device=dev), "c": z(n, device=dev),
                                "R": torch.eye(n, device=dev) * 1e-6, "QR": torch.eye(n, device=dev)}
            exchange = LW.AllGatherV(self.W, owners, dist)
            per_set = []
            for Gs in self.G_sets:
                if o == "muon":
                    mats = [(self.W[i], Gs[i], state[i]["M"] if i in state else None) for i in range(len(specs))]
                else:
                    mats = [dict(state.get(i, {}), W=self.W[i], G=Gs[i]) for i in range(len(specs))]

                def make_batch(owned, o=o):
                    b = {"muon": api.MuonBatch, "soap": api.SoapBatch, "foam": api.FoamBatch}[o](
                        owned, with_stats=True, allocate=False, **kws[o])
                    batches.append(b)
                    return b
                per_set.append(LW.LayerwiseStep(mats, o, dist, make_batch=make_batch, grads_reduced=True,
                                                exchange=exchange, **kws[o]))
            self.steps[o] = per_set
        ws_bytes = max([b.ws_bytes for b in batches] + [256])
        self.workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        for b in batches:
            b.attach_workspace(self.workspace)
        self._dummy_stats = torch.zeros((1, 4), dtype=torch.float32, device=dev)

    def step(self, t, stream, events=None):
        gi = (t - 1) % self.n_grad
        for name in self.order:
            lw = self.steps[name][gi]
            if events is not None:
                events[name][0].record(stream)
            if name == "muon":
                lw()
            else:
                lw(t)
            if events is not None:
                events[name][1].record(stream)

    def stats_tensor(self, t):
        b = self.steps[self.order[0]][(t - 1) % self.n_grad].batch
        return b.stats if b is not None else self._dummy_stats

    def status(self):
        for name in self.order:
            b = self.steps[name][0].batch
            if b is not None and b.device_status() != 0:
                return name, b.device_status()
        return None


# ----------------------------------------------------------------------------- main (mine)
def run_mine(args, rank, world, dist):
    import torch

    from matrix_aware_optimizers_02_b200 import _lib as L

    lib = L.load()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    desc, g_bf16 = WORKLOADS[args.workload]
    specs = specs_for(args.workload, args.seed)
    optimizers = [o.strip() for o in args.optimizers.split(",") if o.strip()]
    norm = MUON_NORM.get(args.workload, "none")
    layerwise = args.mode == "layerwise"
    if layerwise:
        if dist is None:
            raise SystemExit("--mode layerwise needs a process group (run under torchrun)")
        LS = LayerwiseSet(specs, args.seed, dev, g_bf16, optimizers, norm, dist, soap_k=args.soap_k)
    else:
        LS = LayerSet(specs, rank_seed(args.seed, rank), dev, g_bf16, optimizers, norm, soap_k=args.soap_k)
    stream = torch.cuda.current_stream()

    def barrier():
        if dist is not None:
            dist.barrier()

    t = 0
    for _ in range(args.warmup):
        t += 1
        LS.step(t, stream)
    torch.cuda.synchronize()
    bad = LS.status()
    if bad:
        raise RuntimeError(f"device status {bad} after warm-up")

    # launch profiler: one probe step counts the launches, then events for the timed steps
    lib.mao_profile_start(None, None, 0)
    t += 1
    LS.step(t, stream)
    per_step_launches = lib.mao_profile_stop()
    torch.cuda.synchronize()
    # check and refresh steps launch more than the probe step: leave room for them
    cap = min(int(per_step_launches * args.steps * 1.6) + 1024, 150000)
    Ev = ctypes.c_void_p * (2 * cap)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * cap)]
    for e in evs:  # torch creates the CUDA event object on its first record
        e.record(stream)
    opt_ev = {o: [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps)] for o in LS.order}
    torch.cuda.synchronize()
    ev_arr = Ev(*[ctypes.c_void_p(e.cuda_event) for e in evs])
    info = (L.LaunchInfo * cap)()

    clocks = ClockSampler(dev.index) if rank == 0 else None
    barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
        time.sleep(0.3)
    # the timed region: K steps as a caller runs them (the library only counts its launches)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    lib.mao_profile_start(None, None, 0)
    t_start.record(stream)
    for k in range(args.steps):
        t += 1
        LS.step(t, stream, {o: (opt_ev[o][2 * k], opt_ev[o][2 * k + 1]) for o in LS.order})
    t_end.record(stream)
    n_launch = lib.mao_profile_stop()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop() if clocks else None
    ms = t_start.elapsed_time(t_end) / args.steps
    opt_ms = {o: round(sum(opt_ev[o][2 * k].elapsed_time(opt_ev[o][2 * k + 1]) for k in range(args.steps))
                       / args.steps, 3) for o in LS.order}
    bad = LS.status()
    if bad:
        raise RuntimeError(f"device status {bad} after timed steps")

    # the kernel table and the roofline: K more steps with every library launch bracketed
    # by events on its stream (the events themselves cost time, so this region is not the
    # step time above)
    barrier()
    torch.cuda.synchronize()
    k_start = torch.cuda.Event(enable_timing=True)
    k_end = torch.cuda.Event(enable_timing=True)
    L.check(lib.mao_profile_start(ev_arr, info, cap))
    k_start.record(stream)
    for k in range(args.steps):
        t += 1
        LS.step(t, stream)
    k_end.record(stream)
    n_prof = lib.mao_profile_stop()
    torch.cuda.synchronize()
    barrier()
    ms_instrumented = k_start.elapsed_time(k_end) / args.steps
    bad = LS.status()
    if bad:
        raise RuntimeError(f"device status {bad} after the instrumented steps")

    # per-kernel live durations
    per = {}
    for i in range(min(n_prof, cap)):
        kk = info[i].kernel
        d = evs[2 * i].elapsed_time(evs[2 * i + 1])
        e = per.setdefault(kk, {"ms": 0.0, "n": 0, "flops": 0.0, "bytes": 0.0, "tc": 0.0, "planned": 0.0})
        e["ms"] += d
        e["n"] += 1
        # the work the device executed (table-mode products count their computed tiles on
        # the device, so the passes it decides to run are included)
        e["flops"] += info[i].exec_flops
        e["bytes"] += info[i].bytes
        e["tc"] += info[i].exec_tc_flops
        e["planned"] += info[i].flops

    # end-to-end: this step's gradient set from pinned host memory, the step, stats back to host
    host_sets = [[g.cpu().pin_memory() for g in Gs] for Gs in LS.G_sets]
    h2d = sum(g.numel() * g.element_size() for g in host_sets[0])
    stats_host = torch.empty_like(LS.stats_tensor(1), device="cpu").pin_memory()
    d2h = stats_host.numel() * stats_host.element_size()
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        t += 1
        gi = (t - 1) % LS.n_grad
        for g, hg in zip(LS.G_sets[gi], host_sets[gi]):
            g.copy_(hg, non_blocking=True)
        LS.step(t, stream)
        stats_host.copy_(LS.stats_tensor(t), non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    del host_sets
    e2e_ms = e0.elapsed_time(e1) / args.steps

    if args.launch_log and rank == 0:
        write_launch_log(args, lib, L, LS, t + 1, stream)
    order = list(LS.order)
    del LS
    torch.cuda.empty_cache()

    ms_max, e2e_max = reduce_times([ms, e2e_ms], dist, dev)
    if rank != 0:
        return None

    peaks, peak_src = measured_peaks()
    names = L.KERNEL_NAMES
    dom = max(per, key=lambda k: per[k]["ms"]) if per else None
    roof = None
    if dom is not None:
        e = per[dom]
        name = names.get(dom, str(dom))
        tr = ncu_traffic(name, e["flops"] / e["n"], e["bytes"] / e["n"])
        roof = roofline_of(name, e, peaks, peak_src, tr)
    tot = max(sum(x["ms"] for x in per.values()), 1e-9)
    kernels = {}
    for k, v in sorted(per.items()):
        rec = {"launches": v["n"], "ms_total": round(v["ms"], 3), "share": round(v["ms"] / tot, 4)}
        if v["flops"] > 0:
            rec["tflops"] = round(v["flops"] / (v["ms"] * 1e-3) / 1e12, 1)
            rec["tc_tflops"] = round(v["tc"] / (v["ms"] * 1e-3) / 1e12, 1)
        elif v["bytes"] > 0:
            rec["gbs"] = round(v["bytes"] / (v["ms"] * 1e-3) / 1e9, 1)
        kernels[names.get(k, str(k))] = rec

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu_ms, cores, sample, blas = cpu_oracle_sample(args.workload, args.cpu_budget_s, args.seed, order)
        cpu = {"value": round(cpu_ms, 1), "unit": "ms", "cores": cores, "blas_threads": blas, "kind": "oracle",
               "sample": sample}
        full = committed_cpu_table(args.workload)
        if full is not None:
            cpu["every_shape_timed"] = full

    n_elems = sum(s.m * s.n for s in specs)
    line = {
        "metric": "Muon/SOAP/FOAM step ms per layer set; % of tensor-core peak and HBM GB/s",
        "value": round(per_layer_set(ms_max, 1 if layerwise else world), 4),
        "unit": "ms",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max, 4),
        "higher_is_better": False,
        "scaling": "strong" if layerwise else "weak",
        "vs_baseline": None,
        "dtype": "bf16/fp32",
        "data": "synthetic (seeded Gaussian gradients, random weights)",
        "config": {"workload": args.workload, "description": desc, "experts": args.experts, "optimizers": order,
                   "arithmetic": ("bf16 tensor-core operands with fp32 accumulation (Newton-Schulz); "
                                  "fp32-faithful three-plane bf16 products and fp32 states and passes (SOAP, FOAM)"),
                   "optimizer_ms": opt_ms,
                   "muon": {"mu": 0.95, "lr": 0.02, "ns_steps": 5, "norm": norm},
                   "soap": {"beta1": 0.95, "beta2": 0.95, "eps": 1e-8,
                            "refresh": "every step, sorted" if args.soap_k == 1 else
                            f"every {args.soap_k} steps, sorted"},
                   "foam": {"beta1": 0.95, "beta2": 0.95, "eps": 1e-8, "refresh": "adaptive pf=10 tol=0.1"},
                   "timed_steps_t": [args.warmup + 2, args.warmup + 1 + args.steps],
                   "kernel_table": (f"per-launch CUDA events over {args.steps} further steps (t = "
                                    f"{args.warmup + 2 + args.steps}..{args.warmup + 1 + 2 * args.steps}); "
                                    f"{round(ms_instrumented, 1)} ms per step with the events"),
                   "matrices_per_rank": len(specs), "elements_per_rank": n_elems,
                   "gradient_sets": 3,
                   "inputs": "three device-resident seeded gradient sets, step t uses set (t - 1) mod 3",
                   "l2_policy": "inputs larger than L2 (no flush)",
                   "parallelism": (f"layer-wise: one layer set, matrices owned by {world} ranks, all-gather-V of the "
                                   "updated weights" if layerwise else f"independent layer sets x{world}")},
        "roofline": roof,
        "kernels": kernels,
        "cpu_baseline": cpu,
        "e2e": {"value": round(per_layer_set(e2e_max, 1 if layerwise else world), 4), "unit": "ms",
                "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": int(n_launch),
        "clocks": clk,
    }
    if world == 1 and not args.no_extra:
        # the other configurations, timed on this GPU after the layer set above was freed
        c4 = foam_kinds("gpt2_760m", 21, args.seed)
        line["other_configs"] = {
            "gpt2_124m_muon_plus_col_row": muon_set_ms("gpt2_124m", 20, 3, args.seed),
            "gpt2_760m_foam_step_kinds": {"median_ms": c4["median_ms"], "steps": c4["steps"],
                                          "note": "fresh fp32 gradient each step; medians over t >= 2"},
        }
    return line


def foam_kinds(workload, steps, seed):
    """FOAM alone on the workload for t = 1..steps (adaptive, pf = 10, tol = 0.1, a fresh
    gradient each step, drawn outside the timed region), each step bracketed by its own
    events and followed by a read of the per-matrix refresh flags.  A step is plain
    ((t - 1) mod pf != 0), check-only (a check step where no matrix refreshed) or
    check+refresh.  Returns the median ms of each kind over t >= 2 (t = 1 also builds
    the step's launch plan on the host while the GPU waits) and the per-step record."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device())
    desc, g_bf16 = WORKLOADS[workload]
    specs = specs_for(workload, seed)
    LS = LayerSet(specs, seed, dev, g_bf16, ["foam"], "none", n_grad=1)
    b = LS.batches["foam"][0]
    stream = torch.cuda.current_stream()
    kinds = {"plain": [], "check": [], "check+refresh": []}
    per_t = []
    gen = torch.Generator(device=dev).manual_seed(seed + 1)
    for t in range(1, steps + 1):
        for g, sp in zip(LS.G, specs):  # a fresh gradient each step, outside the timed region
            g.normal_(0.0, sp.g_std * sp.g_scale, generator=gen)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        b(t)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        nref = sum(1 for r in b.stats_dict()["refreshed"] if r & 1)
        kind = "plain" if (t - 1) % 10 else ("check+refresh" if nref else "check")
        if t > 1:
            kinds[kind].append(ms)
        per_t.append({"t": t, "kind": kind, "ms": round(ms, 3), "refreshed": nref})
    if LS.status():
        raise RuntimeError(f"device status {LS.status()}")
    del LS, b
    torch.cuda.empty_cache()
    return {"workload": workload, "description": desc, "steps": steps,
            "median_ms": {k: (round(statistics.median(v), 3) if v else None) for k, v in kinds.items()},
            "per_step": per_t}


def muon_set_ms(workload, steps, warmup, seed):
    """Muon (+ the workload's Muon+ norm) alone on the workload: ms per step over `steps`
    timed steps after `warmup`, three gradient sets in rotation."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device())
    _, g_bf16 = WORKLOADS[workload]
    specs = specs_for(workload, seed)
    norm = MUON_NORM.get(workload, "none")
    LS = LayerSet(specs, seed, dev, g_bf16, ["muon"], norm)
    stream = torch.cuda.current_stream()
    t = 0
    for _ in range(warmup):
        t += 1
        LS.step(t, stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        t += 1
        LS.step(t, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    if LS.status():
        raise RuntimeError(f"device status {LS.status()}")
    ms = e0.elapsed_time(e1) / steps
    del LS
    torch.cuda.empty_cache()
    return {"workload": workload, "norm": norm, "matrices": len(specs), "ms_per_step": round(ms, 4),
            "steps": steps, "warmup": warmup}


def run_foam_kinds(args):
    import torch
    torch.cuda.set_device(0)
    out = foam_kinds(args.workload, args.foam_kinds, args.seed)
    out.update({"metric": "FOAM step ms by step kind", "unit": "ms"})
    return out


def run_reference(args, rank, world):
    """The oracle as the reference arm, on the host cores, rank 0 only."""
    if rank != 0:
        return None
    optimizers = [o.strip() for o in args.optimizers.split(",") if o.strip()]
    per_step = []
    info = None
    for i in range(args.warmup + args.steps):
        ms, cores, sample, _ = cpu_oracle_sample(args.workload, args.cpu_budget_s / max(args.steps, 1),
                                                 args.seed + i, optimizers)
        if i >= args.warmup:
            per_step.append(ms)
            info = (cores, sample)
    v = statistics.median(per_step)
    desc, _ = WORKLOADS[args.workload]
    return {
        "impl": "reference",
        "metric": "Muon/SOAP/FOAM step ms per layer set; % of tensor-core peak and HBM GB/s",
        "value": round(v, 1), "unit": "ms", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(v, 1), "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded Gaussian)",
        "config": {"workload": args.workload, "description": desc, "optimizers": optimizers},
        "cpu_baseline": {"value": round(v, 1), "unit": "ms", "cores": info[0], "kind": "oracle", "sample": info[1]},
        "e2e": {"value": round(v, 1), "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    EXPERTS[0] = args.experts
    if args.traffic_csv:
        fold_traffic(args)
        return 0
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.foam_kinds > 0:
        print(json.dumps(run_foam_kinds(args)), flush=True)
        return 0
    if args.cpu_baseline_full:
        opts = [o.strip() for o in args.optimizers.split(",") if o.strip()]
        print(json.dumps(cpu_full_table(args.workload, args.seed, opts)), flush=True)
        return 0
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    dist = None
    if world > 1 or args.mode == "layerwise":
        import datetime

        import torch
        import torch.distributed as D
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        if "MASTER_ADDR" in os.environ:
            D.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        else:  # one process without torchrun: a one-rank group
            import socket
            with socket.socket() as sk:
                sk.bind(("127.0.0.1", 0))
                port = sk.getsockname()[1]
            D.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                 timeout=datetime.timedelta(seconds=120))
        dist = D
    try:
        line = run_mine(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
