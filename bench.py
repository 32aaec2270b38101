#!/usr/bin/env python
"""Benchmark of the SparsePR sparse attention call on B200.

    python bench.py [--gpus N --steps K --warmup W] [--workload mid|hunyuan|wan|sweep|tiny]
                    [--impl ours|reference]

One step = one whole SparsePR call (partition, route, routed attention with
exact probe rows, probe-fitted reconstruction and un-permute) over a batch of
seeded synthetic Voronoi-center video tokens.  The default workload is the
HunyuanVideo-13B-shaped attention call: 24 heads x 118,800 tokens (33x45x80
latent grid), d = 128, bf16, 256 K/V and 256 query groups, budget routing at
rho_exec = 25% including probes, M = 1024 probes, r = 32.

Metric: dense-equivalent TFLOP/s = 4 d N^2 (heads) / call time (higher is
better); the JSON line also carries ms per call, executed-pair TFLOP/s, the
stage breakdown, the attention kernel's roofline fraction, an end-to-end figure
through host buffers, and the fp64 CPU oracle timed on this host as a baseline.

Multi-GPU (torchrun): every rank runs its own heads (weak scaling); there is
no collective on the data path, only a barrier and a max-reduction of the
timings.  --impl reference times the CPU oracle (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from synthetic import voronoi_qkv, workload  # noqa: E402

METRIC = "SparsePR ms/call & dense-equiv TFLOP/s at ρ_exec≈25%; rel-L2 vs dense"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def profiled_traffic(workload_name: str, heads: int):
    """DRAM bytes per attention launch from the committed ncu summary, or None.

    The summary states the DRAM bytes of one launch over `heads_captured`
    heads of the workload (a capture of every head of the long workloads
    would break the capture-size rule); heads are independent units of equal
    size, so the figure scales by heads / heads_captured.  It holds only for
    the kernel source it was captured from: a changed source (its hash no
    longer matches) or another workload gives None.
    """
    import hashlib
    prof = os.path.join(ROOT, "profiles", f"k_attend_tc_{workload_name}.md")
    src = os.path.join(ROOT, "free_block_sparse_means_b200", "csrc", "k_attend_tc.cu")
    if not (os.path.exists(prof) and os.path.exists(src)):
        return None
    fields = {}
    with open(prof) as f:
        for line in f:
            k, sep, v = line.strip().partition(":")
            if sep and k in ("kernel_source_sha256_16", "workload", "traffic_bytes_per_launch",
                             "heads_captured"):
                fields[k] = v.strip()
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    if fields.get("kernel_source_sha256_16") != sha or fields.get("workload") != workload_name:
        return None
    captured = int(fields.get("heads_captured", heads))
    return int(round(int(fields["traffic_bytes_per_launch"]) * heads / captured))


def dist_info():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def shard_heads(BH: int, rank: int, world: int):
    """Flat head indices of one rank under weak scaling (each rank its own BH heads)."""
    return list(range(rank * BH, (rank + 1) * BH))


def reduce_max(values, world, device):
    """Element-wise max over ranks of a list of floats (timing only)."""
    if world == 1:
        return list(values)
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.dev)], stdout=open(self.path, "w"),
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        pw = [num(r[3]) for r in rows if num(r[3]) is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(pw) if pw else None}


def blas_cores():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        return os.cpu_count() or 1


ORACLE_WHOLE_HEAD_MAX_N = 16384  # longer heads: attention on sampled query groups, scaled


class OracleHead:
    """The fp64 oracle on one head of a workload, as it stands.

    Up to ORACLE_WHOLE_HEAD_MAX_N tokens a head runs whole.  Longer heads
    run their partition, route, probes (exact dense rows) and fit once
    (t_fixed); the hard-drop attention, which the oracle evaluates query group
    by query group (one gather of the routed keys per group), is timed on
    every row of a sample of whole query groups and scaled by routed pairs
    (all groups / the sampled ones) to the whole head."""

    def __init__(self, wl, bh):
        import numpy as np
        from oracle import Params, sparsepr_head
        self.wl = wl
        self.prm = Params(Ms=wl.Ms, p=wl.p, Gk=wl.Gk, Gq=wl.Gq, iters=wl.iters,
                          route_mode=wl.route_mode, tau=wl.tau, rho_target=wl.rho_target,
                          M=wl.M, r=wl.r, lam=wl.lam, seed=wl.index, partition=wl.partition,
                          weights=wl.weights, probe_select=wl.probes)
        Q, K, V = voronoi_qkv(wl, heads=[bh])
        self.q, self.k, self.v = (t[0, 0].double().numpy() for t in (Q, K, V))
        self.whole = wl.N <= ORACLE_WHOLE_HEAD_MAX_N
        t0 = time.perf_counter()
        self.out = sparsepr_head(self.q, self.k, self.v, self.prm, bh=bh,
                                 rows=None if self.whole else np.arange(min(16, wl.N)))
        self.t_fixed = time.perf_counter() - t0
        if not self.whole:
            o = self.out
            cq, ck, rp, ci = o["counts_q"], o["counts_k"], o["row_ptr"], o["col_idx"]
            self.pairs = np.array([cq[i] * ck[ci[rp[i]:rp[i + 1]]].sum() for i in range(len(cq))],
                                  np.float64)
            self.live = np.nonzero(self.pairs > 0)[0]
            self.rng = np.random.default_rng(bh)
            t, p = self._time(self.live[:1])
            self.per_pair = max(t / max(p, 1.0), 1e-15)

    def _time(self, groups):
        import numpy as np
        from oracle import hard_drop_attention
        o = self.out
        rows = np.nonzero(np.isin(o["lab_q"], groups))[0]
        t0 = time.perf_counter()
        hard_drop_attention(self.q, self.k, self.v, o["lab_q"], o["lab_k"], o["row_ptr"],
                            o["col_idx"], o["scale"], rows=rows)
        return time.perf_counter() - t0, float(self.pairs[groups].sum())

    def groups_for(self, seconds):
        """Query groups whose attention takes about `seconds`."""
        g = seconds / (self.per_pair * float(self.pairs[self.live].mean()))
        return int(min(len(self.live), max(1, g)))

    def head_seconds(self, groups=None):
        """One estimate of the whole head's time (a fresh group sample)."""
        if self.whole:
            return self.t_fixed
        gs = self.rng.choice(self.live, groups, replace=False)
        t, p = self._time(gs)
        return self.t_fixed + t * float(self.pairs.sum()) / p

    def describe(self, groups=None):
        if self.whole:
            return "whole head"
        return (f"partition, route, probes and fit of the head; hard-drop attention of every "
                f"row of {groups} random query groups, scaled by routed pairs")


def oracle_baseline(wl, budget_s=10.0):
    """The oracle as it stands on heads of the workload, ~budget_s of CPU work
    beyond one head's fixed part (at least one head), scaled to all heads."""
    heads, t_tot, how = 0, 0.0, ""
    while heads < wl.BH and (heads == 0 or t_tot < budget_s):
        h = OracleHead(wl, heads)
        g = None if h.whole else h.groups_for(budget_s / 2)
        t_tot += h.head_seconds(g)
        how = h.describe(g)
        heads += 1
    flops = 4.0 * wl.d * wl.N * wl.N * heads
    return {"value": flops / t_tot / 1e12, "unit": "TFLOP/s (dense-equivalent)",
            "cores": blas_cores(), "kind": "oracle",
            "sample": f"{heads} of {wl.BH} heads of {wl.name} ({how}), fp64 numpy, "
                      f"{t_tot:.1f} s estimated"}


def partition_bytes(wl):
    """Algorithmic HBM bytes of the partition stage per call: every pass reads
    its input once and writes its output once.  Per head, with row bytes
    qb = kb = 2d (bf16) and zb = 128 (32 fp32 key coordinates):
      query RMS pass and T query assignments: (T + 1) qb N;
      key projection: kb N read + zb N written; T key assignments: T zb N;
      group-major copies of Q, K and V: 3 (read + write) 2d N;
      group means of the permuted keys and queries: 2 qb N."""
    qb, zb, T, N = 2.0 * wl.d, 128.0, wl.iters, wl.N
    per_head = ((T + 1) * qb + qb + zb + T * zb + 3 * 2 * qb + 2 * qb) * N
    return per_head * wl.BH


def config_of(wl, world):
    return {"workload": f"{wl.name}: B={wl.B} H={wl.H} N={wl.N} ({'x'.join(map(str, wl.grid))}) "
                        f"d={wl.d}", "heads_per_gpu": wl.BH, "tokens": wl.N, "head_dim": wl.d,
            "Ms": wl.Ms, "p": wl.p, "Gk": wl.Gk, "Gq": wl.Gq, "iters": wl.iters,
            "routing": (f"budget rho_target={wl.rho_target}" if wl.route_mode == "budget"
                        else f"tau={wl.tau}"),
            "M": wl.M, "r": wl.r, "lambda": wl.lam, "partition": wl.partition,
            "probe_weights": wl.weights,
            "probes": wl.probes,
            "parallelism": f"heads x{world} (weak)",
            "l2": "flushed (256 MiB write) before every timed call"}


REF_BUDGET_S = 120.0  # wall-clock target of a whole reference-arm run (steps + warm-up)


def run_reference(args, wl):
    """The oracle as the reference arm, on a bounded sample of the workload
    (OracleHead): head 0 is set up once; every step is a fresh estimate of its
    time (whole head, or a fresh sample of whole query groups sized so that
    the warm-up and the steps take about REF_BUDGET_S)."""
    world, rank, _ = dist_info()
    if rank != 0:
        return 0
    nsteps = args.warmup + args.steps
    h = OracleHead(wl, 0)
    g = None if h.whole else h.groups_for(max(REF_BUDGET_S - h.t_fixed, 10.0) / nsteps)
    times = []
    for s in range(nsteps):
        t = h.head_seconds(g) if not h.whole else OracleHead(wl, s % wl.BH).t_fixed
        if s >= args.warmup:
            times.append(t)
    sample = f"head 0 of {wl.name}: {h.describe(g)} (fp64 numpy)"
    t = statistics.mean(times)
    val = 4.0 * wl.d * wl.N * wl.N / t / 1e12
    unit = "TFLOP/s (dense-equivalent)"
    line = {"metric": METRIC, "value": val, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": dict(config_of(wl, 1), kmeans_start="seeded"),
            "cpu_baseline": {"value": val, "unit": unit, "cores": blas_cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def quality_vs_dense(spr, prm, ws, Q, K, V, O, wl, rows_per_head=1024, seed=0):
    """Attention-reconstruction error against dense attention on sampled rows
    (the same rows in every head), as measurement only (dense rows in fp32,
    the fit below in fp64, both with torch outside the timed region):
      - relative L2 over the sample of the hard-drop output (routed cells
        only) and of the SparsePR output;
      - the O3 split of the hard-drop residual R = dense - hard drop: its
        least-squares affine fit on [hard-drop output, 1] per head and the
        remainder; reported as the affine-explainable fraction sum ||P||^2 /
        sum ||R||^2 and the orthogonal energy sum ||R - P||^2 relative to the
        dense output's energy (estimated on the sampled rows)."""
    BH, N, d = wl.BH, wl.N, wl.d
    dev = Q.device
    g = torch.Generator().manual_seed(seed)
    rows = torch.randperm(N, generator=g)[: min(rows_per_head, N)].to(dev)
    perm_q = spr.workspace_tensor(prm, ws, "perm_q", torch.int32, (BH, N)).long()
    inv = torch.empty_like(perm_q)
    inv.scatter_(1, perm_q, torch.arange(N, device=dev).expand(BH, N).contiguous())
    osp = spr.workspace_tensor(prm, ws, "o_sparse", torch.float32, (BH, N, d))
    q, k, v, o = (t.reshape(BH, N, d) for t in (Q, K, V, O))
    scale = 1.0 / d ** 0.5
    num_hd = num_sp = den = e_res = e_aff = e_orth = 0.0
    row_hd, row_sp = [], []
    for bh in range(BH):
        s = (q[bh, rows].float() @ k[bh].float().T) * scale
        dense = torch.softmax(s, dim=-1) @ v[bh].float()
        hd = osp[bh, inv[bh, rows]]
        sp = o[bh, rows].float()
        num_hd += float(((hd - dense) ** 2).sum())
        num_sp += float(((sp - dense) ** 2).sum())
        dn = dense.norm(dim=1).clamp_min(1e-30)
        row_hd.append(((hd - dense).norm(dim=1) / dn).double().cpu())
        row_sp.append(((sp - dense).norm(dim=1) / dn).double().cpu())
        den += float((dense ** 2).sum())
        R = (dense - hd).double()
        F = torch.cat([hd.double(), torch.ones(hd.shape[0], 1, dtype=torch.float64, device=dev)], 1)
        P = F @ torch.linalg.lstsq(F.cpu(), R.cpu()).solution.to(dev)
        e_res += float((R * R).sum())
        e_aff += float((P * P).sum())
        e_orth += float(((R - P) ** 2).sum())
    row_hd, row_sp = torch.cat(row_hd), torch.cat(row_sp)
    return {"rows_sampled_per_head": int(rows.numel()), "dense": 0.0,
            "hard_drop": (num_hd / den) ** 0.5, "sparsepr": (num_sp / den) ** 0.5,
            "row_error_hard_drop": {"mean": float(row_hd.mean()),
                                    "p99": float(torch.quantile(row_hd, 0.99))},
            "row_error_sparsepr": {"mean": float(row_sp.mean()),
                                   "p99": float(torch.quantile(row_sp, 0.99))},
            "o3_affine_fraction": e_aff / e_res if e_res > 0 else 0.0,
            "o3_orthogonal_energy_rel": e_orth / den}


def dense_sdpa_context(Q, K, V, wl, ms_per_call, flush, stream, reps=3):
    """Context only, outside the timed region: dense attention on the same
    inputs with torch's scaled_dot_product_attention (a library kernel), the
    time a call without any sparsity would take on this GPU."""
    import torch.nn.functional as F
    F.scaled_dot_product_attention(Q, K, V)  # warm-up (backend selection)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        F.scaled_dot_product_attention(Q, K, V)
        b.record(stream)
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in ev)
    flop = 4.0 * wl.d * wl.N * wl.N * wl.BH
    return {"kernel": "torch scaled_dot_product_attention (dense, bf16)", "ms": ms,
            "tflops": flop / (ms * 1e-3) / 1e12, "sparsepr_speedup": ms / ms_per_call}


def support_and_mass(P, keep, alpha=0.9, pool=8):
    """O1 / O2 on sampled query rows (measurement only, torch).

    P: [n, N] attention probabilities of n sampled queries, consecutive blocks
    of `pool` rows from the same query group; keep: [n, N] bool, the keys each
    query's route keeps.  Returns (per-query minimal-support fractions at mass
    alpha, the pooled support fraction of each block, retained masses).  A
    query's support: keys by decreasing probability (ties to the lower index)
    until the running mass reaches alpha.
    """
    n, N = P.shape
    ps, order = torch.sort(P, dim=1, descending=True, stable=True)
    cs = torch.cumsum(ps, dim=1)
    k = ((cs < alpha * P.sum(1, keepdim=True)).sum(1) + 1).clamp(max=N)
    per = k.double() / N
    in_sorted = torch.arange(N, device=P.device)[None, :] < k[:, None]
    member = torch.zeros_like(in_sorted).scatter_(1, order, in_sorted)
    pooled = member.view(n // pool, pool, N).any(1).sum(1).double() / N
    mass = (P * keep).sum(1).double()
    return per, pooled, mass


def diagnostics(spr, prm, ws, Q, K, V, wl, alpha=0.9, pool=8, groups_per_head=16, seed=0):
    """O1 pooled support and O2 retained mass vs error [paperlayer §3.1] on
    query groups sampled from every head (pool members each), measurement
    only: dense probabilities in fp32 here, the hard-drop rows from the
    workspace."""
    BH, N, d = wl.BH, wl.N, wl.d
    dev = Q.device
    g = torch.Generator().manual_seed(seed)
    q_off = spr.workspace_tensor(prm, ws, "q_off", torch.int32, (BH, wl.Gq + 1)).long().cpu()
    perm_q = spr.workspace_tensor(prm, ws, "perm_q", torch.int32, (BH, N)).long()
    lab_k = spr.workspace_tensor(prm, ws, "lab_k", torch.int32, (BH, N)).long()
    row_ptr = spr.workspace_tensor(prm, ws, "row_ptr", torch.int32, (BH, wl.Gq + 1)).long().cpu()
    col_idx = spr.workspace_tensor(prm, ws, "col_idx", torch.int32, (BH, wl.Gq * wl.Gk)).long()
    osp = spr.workspace_tensor(prm, ws, "o_sparse", torch.float32, (BH, N, d))
    q, k, v = (t.reshape(BH, N, d) for t in (Q, K, V))
    scale = 1.0 / d ** 0.5
    pers, pooleds, masses, errs = [], [], [], []
    for bh in range(BH):
        sizes = q_off[bh, 1:] - q_off[bh, :-1]
        big = torch.nonzero(sizes >= pool).flatten()
        if len(big) == 0:
            continue
        groups = big[torch.randperm(len(big), generator=g)[:groups_per_head]]
        pos, keep_groups = [], []
        for gi in groups.tolist():
            o0, cnt = int(q_off[bh, gi]), int(sizes[gi])
            pos.append(o0 + torch.randperm(cnt, generator=g)[:pool])
            routed = col_idx[bh, int(row_ptr[bh, gi]):int(row_ptr[bh, gi + 1])]
            keep_groups.append(torch.isin(lab_k[bh], routed))
        pos = torch.cat(pos).to(dev)
        rows = perm_q[bh, pos]
        keep = torch.stack(keep_groups).repeat_interleave(pool, dim=0)
        P = torch.softmax((q[bh, rows].float() @ k[bh].float().T) * scale, dim=-1)
        per, pooled, mass = support_and_mass(P, keep, alpha, pool)
        dense = P @ v[bh].float()
        err = (osp[bh, pos] - dense).norm(dim=1) / dense.norm(dim=1)
        pers.append(per)
        pooleds.append(pooled)
        masses.append(mass)
        errs.append(err.double())
    if not pers:
        return {"alpha": alpha, "queries": 0, "pool": pool}
    per, pooled, mass, err = (torch.cat(x).cpu() for x in (pers, pooleds, masses, errs))
    # O2: how far retained mass ranks the errors (Spearman), and the spread of
    # the error among the fifth of the queries closest to the median mass
    rank = lambda x: torch.argsort(torch.argsort(x)).double()
    rm, re = rank(mass), rank(err)
    rm, re = rm - rm.mean(), re - re.mean()
    spearman = float((rm * re).sum() / (rm.norm() * re.norm()))
    near = torch.argsort((mass - mass.median()).abs())[: max(2, len(mass) // 5)]
    e_near = err[near]
    return {"alpha": alpha, "queries": int(len(per)), "pool": pool,
            "o1_support_median": float(per.median()), "o1_pooled_median": float(pooled.median()),
            "o2_mass_median": float(mass.median()), "o2_spearman_mass_error": spearman,
            "o2_error_p90_over_p10_at_median_mass":
                float(torch.quantile(e_near, 0.9) / torch.quantile(e_near, 0.1))}


def run_ours(args, wl):
    import free_block_sparse_means_b200 as spr
    world, rank, local = dist_info()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    spr.load_library()
    heads = shard_heads(wl.BH, rank, world)
    Qc, Kc, Vc = voronoi_qkv(wl, heads=heads)
    shape = (wl.B, wl.H, wl.N, wl.d)
    Qc, Kc, Vc = (t.reshape(shape).contiguous() for t in (Qc, Kc, Vc))
    Q, K, V = (t.to(dev) for t in (Qc, Kc, Vc))
    O = torch.empty_like(Q)
    prm = spr.make_params(Q, K, V, O, Ms=wl.Ms, p=wl.p, Gk=wl.Gk, Gq=wl.Gq, iters=wl.iters,
                          seed=wl.index, route_mode=wl.route_mode, tau=wl.tau,
                          rho_target=wl.rho_target, M=wl.M, r=wl.r, lam=wl.lam,
                          partition=wl.partition, weights=wl.weights, probes=wl.probes)
    ws = spr.alloc_workspace(prm, device=dev)
    prm_seeded = prm
    if args.warm_iters > 0:  # every call after the first starts from the previous centroids
        prm = spr.make_params(Q, K, V, O, Ms=wl.Ms, p=wl.p, Gk=wl.Gk, Gq=wl.Gq,
                              iters=args.warm_iters, seed=wl.index, route_mode=wl.route_mode,
                              tau=wl.tau, rho_target=wl.rho_target, M=wl.M, r=wl.r, lam=wl.lam,
                              partition=wl.partition, weights=wl.weights, probes=wl.probes,
                              init="warm")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def call_staged(ev=None, prm=prm):
        if ev is not None:
            ev[0].record(stream)
        spr.sparsepr_partition(prm, Q, K, V, ws, stream)
        if ev is not None:
            ev[1].record(stream)
        spr.sparsepr_route(prm, ws, stream)
        if ev is not None:
            ev[2].record(stream)
        spr.sparsepr_attend(prm, ws, stream)
        if ev is not None:
            ev[3].record(stream)
        spr.sparsepr_reconstruct(prm, ws, O, stream)
        if ev is not None:
            ev[4].record(stream)

    for w in range(args.warmup):
        flush.zero_()
        call_staged(prm=prm_seeded if w == 0 else prm)
    torch.cuda.synchronize(dev)
    stats, err = spr.sparsepr_get_stats(prm, ws, stream)
    if err:
        raise SystemExit(f"device error word {err}")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    n0 = spr.sparsepr_launch_count()
    with ClockSampler(local) as clk:
        for s in range(args.steps):
            flush.zero_()
            call_staged(evs[s])
        torch.cuda.synchronize(dev)
    n1 = spr.sparsepr_launch_count()
    if world > 1:
        torch.distributed.barrier()
    stage = [[evs[s][i].elapsed_time(evs[s][i + 1]) for i in range(4)] for s in range(args.steps)]
    per_call = [sum(x) for x in stage]
    total_ms = sum(per_call)
    stage_mean = [statistics.mean(x[i] for x in stage) for i in range(4)]
    srt = sorted(per_call)
    med = statistics.median(srt)
    p90 = srt[min(len(srt) - 1, int(0.9 * (len(srt) - 1) + 0.5))]
    mx = reduce_max([total_ms] + stage_mean + [med, p90], world, dev)
    total_ms_max, stage_max, med_max, p90_max = mx[0], mx[1:5], mx[5], mx[6]
    ms_per_call = total_ms_max / args.steps
    dense_flop = 4.0 * wl.d * wl.N * wl.N * wl.BH  # per rank
    value = dense_flop * world / (ms_per_call * 1e-3) / 1e12
    pairs = sum(h["routed_pairs"] + h["probe_pairs"] for h in stats)
    tile_pairs = sum(h["tile_pairs"] for h in stats)
    rho = pairs / (wl.N * wl.N * wl.BH)
    exec_tflops = 4.0 * wl.d * pairs / (ms_per_call * 1e-3) / 1e12
    peaks, peak_kind = load_peaks()
    attend_ms = stage_max[2]
    att_achieved = 4.0 * wl.d * pairs / (attend_ms * 1e-3) / 1e12
    roof = {"bound": "tensor", "kernel": "k_attend (routed cells + probe rows)",
            "achieved": att_achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": att_achieved / peaks["bf16_tflops"], "peak_source": f"{peak_kind} bf16 burst",
            "traffic": profiled_traffic(wl.name, wl.BH),
            "algorithmic_flop_per_launch": 4.0 * wl.d * pairs,
            "executed_tile_pairs": tile_pairs, "true_pairs": pairs,
            # the same kernel against the sustained (power-capped) bf16 peak, and
            # on executed tile pairs (padding included) against the burst peak
            "frac_sustained": att_achieved / peaks.get("bf16_tflops_sustained",
                                                       FALLBACK_PEAKS["bf16_tflops_sustained"]),
            "frac_executed_pairs": (att_achieved * tile_pairs / pairs / peaks["bf16_tflops"]
                                    if pairs > 0 else 0.0)}
    part_bytes = partition_bytes(wl)
    part_gbs = part_bytes / (stage_max[0] * 1e-3) / 1e9
    # end to end through the public API with host buffers (pinned): the
    # host-buffer call pipelined over chunks of heads (copies of one chunk
    # overlap the computation of the next); every byte of the inputs and of
    # the output crosses PCIe inside the timed region
    Qh, Kh, Vh = (t.pin_memory() for t in (Qc, Kc, Vc))
    Oh = torch.empty(shape, dtype=torch.bfloat16).pin_memory()
    e2e_chunk = max(1, -(-wl.BH // args.e2e_chunks))
    pipe = spr.HostPipeline(shape, e2e_chunk, device=dev, Ms=wl.Ms, p=wl.p, Gk=wl.Gk,
                            Gq=wl.Gq, iters=wl.iters, seed=wl.index, route_mode=wl.route_mode,
                            tau=wl.tau, rho_target=wl.rho_target, M=wl.M, r=wl.r, lam=wl.lam,
                            partition=wl.partition, weights=wl.weights, probes=wl.probes)
    e2e_steps = max(3, min(args.steps, 10))
    ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(e2e_steps)]
    flush.zero_()
    pipe(Qh, Kh, Vh, Oh, stream)  # warm-up of the pipeline's own buffers
    for s in range(e2e_steps):
        flush.zero_()
        ee[s][0].record(stream)
        pipe(Qh, Kh, Vh, Oh, stream)
        ee[s][1].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = reduce_max([statistics.mean(a.elapsed_time(b) for a, b in ee)], world, dev)[0]
    h2d = 3 * Q.numel() * 2
    d2h = O.numel() * 2
    clocks = clk.summary()
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s (dense-equivalent)",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_call, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 (fp32 accumulate)", "data": "synthetic",
            "config": dict(config_of(wl, world), **(
                {"iters": args.warm_iters,
                 "kmeans_start": "warm (previous call's centroids; first warm-up call seeded)"}
                if args.warm_iters > 0 else {"kmeans_start": "seeded"})),
            "ms_per_call": ms_per_call, "ms_per_call_median": med_max, "ms_per_call_p90": p90_max,
            "exec_pair_tflops": exec_tflops * world, "rho_exec": rho,
            "stage_ms": {"partition": stage_max[0], "route": stage_max[1], "attend": stage_max[2],
                         "reconstruct": stage_max[3]},
            "roofline": roof,
            "partition_hbm": {"achieved_gbs": part_gbs, "peak_gbs": peaks["hbm_gbs"],
                              "frac": part_gbs / peaks["hbm_gbs"], "algorithmic_bytes": part_bytes},
            "e2e": {"value": dense_flop * world / (e2e_ms * 1e-3) / 1e12,
                    "unit": "TFLOP/s (dense-equivalent)", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "api": f"HostPipeline: pinned host Q, K, V in and O out, "
                           f"{len(pipe.chunks())} chunks of {e2e_chunk} heads, the copies "
                           f"of one chunk overlapping the computation of the next"},
            "gpu_launches": int(n1 - n0), "clocks": clocks, "device_error": err}
    line["rel_l2_vs_dense"] = quality_vs_dense(spr, prm, ws, Q, K, V, O, wl)
    line["dense_context"] = dense_sdpa_context(Q, K, V, wl, ms_per_call, flush, stream)
    if args.diagnostics:
        line["diagnostics"] = diagnostics(spr, prm, ws, Q, K, V, wl)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_baseline(wl, budget_s=args.cpu_budget)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


E2E_CHUNKS = 4  # head chunks of the pipelined host-buffer call
SWEEP_RHO = (0.10, 0.20, 0.25, 0.35, 0.50)
SWEEP_M = (64, 256, 1024)
SWEEP_R = (8, 32)
SWEEP_LAMBDA = (1e-2, 1e-1, 1.0)  # ridge strengths beside the workload's, at rho 0.25, r 8


def run_sweep(args, wl):
    """Density / probe-budget / rank sweep on one GPU (the sweep workload by
    default): every executed-pair density in SWEEP_RHO with the method's
    response-coupled partition for every probe budget M x rank r, and with
    the semantic comparator at the workload's M and r; then, at rho 0.25 and
    r 8, every M with the ridge strengths of SWEEP_LAMBDA.  One JSON line per
    point: ms per call (median of the timed calls, L2 flushed before each),
    dense-equivalent and executed-pair TFLOP/s, realised rho_exec and the
    errors against dense attention on sampled rows (quality_vs_dense)."""
    import free_block_sparse_means_b200 as spr
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    dev = torch.device("cuda", 0)
    spr.load_library()
    Qc, Kc, Vc = voronoi_qkv(wl)
    shape = (wl.B, wl.H, wl.N, wl.d)
    Q, K, V = (t.reshape(shape).contiguous().to(dev) for t in (Qc, Kc, Vc))
    O = torch.empty_like(Q)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    points = [("response", rho, M, r, wl.lam) for rho in SWEEP_RHO for M in SWEEP_M
              for r in SWEEP_R]
    points += [("semantic", rho, wl.M, wl.r, wl.lam) for rho in SWEEP_RHO]
    points += [("response", 0.25, M, 8, lam) for M in SWEEP_M for lam in SWEEP_LAMBDA]
    ws = None
    for part, rho, M, r, lam in points:
        pw = wl.replace(partition=part, route_mode="budget", rho_target=rho, M=M, r=r, lam=lam)
        prm = spr.make_params(Q, K, V, O, Ms=pw.Ms, p=pw.p, Gk=pw.Gk, Gq=pw.Gq, iters=pw.iters,
                              seed=pw.index, route_mode="budget", rho_target=rho, M=M, r=r,
                              lam=lam, partition=part, weights=pw.weights, probes=pw.probes)
        need = spr.sparsepr_workspace_size(prm)
        if ws is None or ws.numel() < need:
            ws = spr.alloc_workspace(prm, device=dev)
        for _ in range(args.warmup):
            flush.zero_()
            spr.sparsepr_call(prm, Q, K, V, O, ws, stream)
        times = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            spr.sparsepr_call(prm, Q, K, V, O, ws, stream)
            b.record(stream)
            times.append((a, b))
        torch.cuda.synchronize(dev)
        ms = statistics.median(x.elapsed_time(y) for x, y in times)
        stats, err = spr.sparsepr_get_stats(prm, ws, stream)
        if err:
            raise SystemExit(f"device error word {err} at {part} rho={rho} M={M} r={r} "
                             f"lambda={lam}")
        pairs = sum(h["routed_pairs"] + h["probe_pairs"] for h in stats)
        q = quality_vs_dense(spr, prm, ws, Q, K, V, O, pw, rows_per_head=512)
        print(json.dumps({
            "sweep": pw.name, "partition": part, "rho_target": rho, "M": M, "r": r,
            "lambda": lam,
            "rho_exec": pairs / (wl.N * wl.N * wl.BH), "ms_per_call_median": ms,
            "dense_equiv_tflops": 4.0 * wl.d * wl.N * wl.N * wl.BH / (ms * 1e-3) / 1e12,
            "exec_pair_tflops": 4.0 * wl.d * pairs / (ms * 1e-3) / 1e12,
            "rel_l2_hard_drop": q["hard_drop"], "rel_l2_sparsepr": q["sparsepr"],
            "row_error_hard_drop": q["row_error_hard_drop"],
            "row_error_sparsepr": q["row_error_sparsepr"],
            "o3_affine_fraction": q["o3_affine_fraction"]}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[1])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="hunyuan")
    ap.add_argument("--heads", type=int, default=0,
                    help="H > 0: that many heads of the workload (a smaller case of the same "
                         "kernels, for profiler captures)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--warm-iters", type=int, default=0,
                    help="T > 0: the first warm-up call is seeded, every later call starts its "
                         "k-means from the previous call's centroids and runs T iterations")
    ap.add_argument("--weights", default="coverage", choices=["coverage", "uniform"],
                    help="uniform: the unweighted estimator of the ablation")
    ap.add_argument("--probes", default="stratified", choices=["stratified", "ranked"],
                    help="ranked: each group's probes are its rows nearest the centroid")
    ap.add_argument("--rank", type=int, default=0,
                    help="r of the residual fit (0: the workload's; d: no subspace restriction)")
    ap.add_argument("--diagnostics", action="store_true",
                    help="add the O1 pooled-support and O2 retained-mass diagnostics")
    ap.add_argument("--rho", type=float, default=0.0,
                    help="executed-pair density target (0: the workload's), for density sweeps")
    ap.add_argument("--e2e-chunks", type=int, default=E2E_CHUNKS,
                    help="head chunks of the pipelined host-buffer call timed as e2e")
    ap.add_argument("--sweep", action="store_true",
                    help="density x probe budget x rank sweep (one JSON line per point; "
                         "default workload: sweep)")
    ap.add_argument("--partition", default="response", choices=["response", "semantic"],
                    help="semantic: the raw-row k-means comparator instead of the method's "
                         "response-coupled partition")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = workload(args.workload, partition=args.partition, weights=args.weights,
                  probes=args.probes)
    if args.heads > 0:
        wl = wl.replace(H=args.heads)
    if args.rank > 0:
        wl = wl.replace(r=args.rank)
    if args.rho > 0:
        wl = wl.replace(route_mode="budget", rho_target=args.rho)
    if args.sweep:
        if args.workload == "hunyuan":
            wl = workload("sweep", weights=args.weights, probes=args.probes)
        return run_sweep(args, wl)
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
