#!/usr/bin/env python
"""Benchmark of the chunk-adaptive mixed-bitwidth KV-cache path on B200.

One step = one pass of the whole path over one batch:
  route (router scores, argmax, vote, freezing)  ->  layout (regroup by
  precision)  ->  pack every layer  ->  one decode step per layer,
all through the C ABI of libmqkv, on synthetic inputs already resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the CPU oracle, timed as a baseline

Default workload: llama2_13b_128k (Llama-2-13B shape, 40 layers sharing one
routing map, 1 x 131072 tokens, chunk 256, INT2-heavy map; every layer's K/V
is drawn and packed in turn, so only the packed cache of the 40 layers stays
resident).  Multi-GPU (torchrun): every rank runs its own batch (seeded by
rank), no data-path collective; the timed region is bracketed by barriers
and the max over ranks is reported.

Printed: one JSON line on rank 0.  value = decode tokens per second of the
whole step (sequences x decode steps / step time, summed over ranks).
"""
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

METRIC = "decode attn tokens/s & packed-KV HBM GB/s (% of B200 peak); pack GB/s"
DEFAULT_WORKLOAD = "llama2_13b_128k"
L2_BYTES = 126 * 2 ** 20


def l2_evict(buf):
    """Reads a buffer of twice the L2 size (written once, at setup): every
    line the L2 held is evicted (dirty ones written back now) and what stays
    is clean, so the next timed kernel reads its input from HBM and pays for
    no other data's write-backs."""
    import torch
    return buf.view(-1).view(torch.int64).max()
SPEC_HBM_GBS = 8000.0   # B200 HBM3e data-sheet bandwidth (context beside the measured peak)


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--router", default="moqae", choices=["moqae", "similarity"],
                   help="chunk map from MoQAE's router or from Cocktail's chunk-query similarity")
    p.add_argument("--layers", type=int, default=0,
                   help="override the workload's layer count (small profiling cases)")
    p.add_argument("--seqs", type=int, default=0,
                   help="override the workload's sequence count (small profiling cases)")
    p.add_argument("--lam", type=float, default=0.0,
                   help="memory-pressure knob for the router map: subtracts lam * bits/16 from "
                        "each expert's bias (more INT2 as lam grows, more FP16 below 0)")
    p.add_argument("--context-split", action="store_true",
                   help="every rank holds a contiguous range of chunks of the same batch; "
                        "per-rank partial records are all-gathered and merged (strong scaling)")
    p.add_argument("--grow", action="store_true",
                   help="decode-time cache growth: every decode step appends one token per "
                        "sequence; full tails are routed and sealed into their segments")
    p.add_argument("--no-rs", action="store_true",
                   help="routing sharing off: one router, map and layout per layer")
    return p.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# DRAM bytes (read + write) of one full-size pack launch of the default
# workload, from an ncu capture (the command and counters are recorded under
# profiles/), valid only for the pack kernel source (pack.cu) with this
# SHA-256.
# DRAM bytes (read + write) of one full-size pack launch per workload, from
# the ncu captures summarised in profiles/pack_kernel_*_traffic.md, with the
# SHA-256 of the pack.cu they ran
PACK_TRAFFIC = {
    "llama2_7b_32l": {"sha256": "8a9960beeb72542fc97eda5327348a6f19cbddb77bc9d45c775727e1d8600141",
                      "bytes_per_launch": 2148355840 + 843005952},
    "llama2_13b_128k": {"sha256": "8a9960beeb72542fc97eda5327348a6f19cbddb77bc9d45c775727e1d8600141",
                        "bytes_per_launch": 2685038080 + 757476608},
}


def pack_sources_sha256():
    import hashlib
    h = hashlib.sha256()
    for f in ("pack.cu",):
        with open(os.path.join(ROOT, "chunk_adaptive_mixed_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def pack_traffic(w, S, seed):
    """Measured DRAM bytes per pack launch, or None when the capture does not
    describe this kernel and workload."""
    from chunk_adaptive_mixed_b200 import workloads as W
    cap = PACK_TRAFFIC.get(w.name)
    if (cap is None or seed != 0 or w.num_seqs != W.get(w.name).num_seqs or S.router != "moqae"
            or S.lam or not S.rs):
        return None
    return cap["bytes_per_launch"] if pack_sources_sha256() == cap["sha256"] else None


def peaks_all():
    """{hbm GB/s, bf16 TFLOP/s burst and sustained}: the measured copy
    bandwidth and the measured bf16 GEMM rates (the router's MMAs are bf16).
    The router runs inside a seconds-long step under the power cap, so its
    fraction is taken against the sustained rate; the burst one is kept beside
    it."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        burst = float(d["bf16_tflops"])
        return {"hbm": float(d["hbm_gbs"]), "bf16": burst,
                "bf16_sustained": float(d.get("bf16_tflops_sustained", burst)), "source": "measured"}
    return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def route_summary(S, route_ms, peaks):
    """Rate of the chunk-map step (all maps of one step) against its roofline."""
    amount, unit, bound = S.route_work()
    maps = len(S.routers)
    rate = amount * maps / (route_ms / 1e3) / (1e9 if unit == "GB/s" else 1e12)
    peak = peaks["hbm"] if bound == "hbm" else peaks["bf16_sustained"]
    out = {"router": S.router, "maps_per_step": maps, "avg_ms_per_step": route_ms,
           "achieved": rate, "unit": unit, "bound": bound, "peak": peak, "frac": rate / peak,
           "peak_source": peaks["source"] + (" (sustained bf16 GEMM)" if bound == "tensor" else ""),
           "algorithmic_per_map": amount, "includes": "map kernels only (layout excluded)"}
    if bound == "tensor":
        # bf16 hi*hi + hi*lo + lo*hi: the tensor cores do 3x the algorithmic work
        out["tensor_passes"] = 3
        out["tensor_frac"] = 3 * rate / peak
        out["tensor_frac_of_burst"] = 3 * rate / peaks["bf16"]
    return out


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi during a region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ ranks

def workload(args):
    """The named workload, with the layer / sequence overrides applied."""
    from chunk_adaptive_mixed_b200 import workloads as W
    w = W.get(args.workload)
    ch = {}
    if args.layers:
        ch["layers"] = args.layers
    if args.seqs:
        ch["num_seqs"] = args.seqs
    return W.scaled(w, **ch) if ch else w


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own batch: independent problems, no exchange."""
    return seed + 1009 * rank


def reduce_timing(ms_local: float, device=None) -> float:
    """Max over ranks of the locally measured time (the job ends when the
    slowest rank ends).  A single process returns its own time."""
    import torch
    import torch.distributed as tdist
    if not (tdist.is_available() and tdist.is_initialized()) or tdist.get_world_size() == 1:
        return ms_local
    t = torch.tensor([ms_local], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time."""
    return units_per_rank * world / (ms_max / 1e3)


def reduce_sum(x_local: float, device=None) -> float:
    """Sum over ranks (bytes every rank moved).  A single process returns its
    own value."""
    import torch
    import torch.distributed as tdist
    if not (tdist.is_available() and tdist.is_initialized()) or tdist.get_world_size() == 1:
        return x_local
    t = torch.tensor([x_local], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.SUM)
    return float(t.item())


def e2e_result(units_per_rank: float, world: int, ms_max: float, h2d_all: float, d2h_all: float,
               steps: int, shared_batch: bool) -> dict:
    """The end-to-end entry: whole-job tokens/s over the slowest rank's time
    (every rank decodes the same sequences when the context is split), and the
    bytes all ranks copied per step."""
    value = (units_per_rank / (ms_max / 1e3) if shared_batch
             else job_throughput(units_per_rank, world, ms_max))
    return {"value": value, "unit": "tokens/s", "ms_per_step": ms_max, "steps": steps,
            "h2d_bytes_per_step": int(h2d_all), "d2h_bytes_per_step": int(d2h_all)}


# ------------------------------------------------------------------ our path

class Setup:
    """Device-resident inputs and outputs of one batch of the workload."""

    def __init__(self, w, seed, device, routing_sharing=True, router="moqae", lam=0.0,
                 grow=False, shard=None):
        import torch
        from chunk_adaptive_mixed_b200 import context_split as CS
        from chunk_adaptive_mixed_b200 import mqkv as M
        from chunk_adaptive_mixed_b200 import workloads as W
        self.w = w
        # shard = (rank, world): this rank holds a contiguous range of whole
        # chunks of every sequence of one shared batch (context split)
        self.shard = shard
        self.full_lens = W.seq_lens(w, seed)
        if shard is not None:
            rank, world = shard
            self.lo, self.hi = CS.shard_ranges(self.full_lens, w.chunk_len, rank, world)
            self.lens = CS.shard_lengths(self.full_lens, w.chunk_len, rank, world)
            self.freeze = CS.routing_freeze(rank)
        else:
            self.lens = self.full_lens
            self.freeze = True
        self.B = len(self.lens)
        self.T = int(self.lens.sum())
        self.N = int(W.num_chunks(self.lens, w.chunk_len).sum())
        self.shape = M.shape(self.B, w.num_q_heads, w.num_kv_heads, w.head_dim, w.chunk_len)
        self.cu = torch.as_tensor(W.cu_seqlens(self.lens), device=device)
        self.rs = routing_sharing
        # with routing sharing one router serves every layer; without it each
        # layer has its own router (weights drawn from seed + layer) over the
        # same router input, so each layer gets its own map and layout
        nr = 1 if routing_sharing else w.layers
        self.routers = [W.router_weights(w, seed + (l if not routing_sharing else 0), device)
                        for l in range(nr)]
        self.lam = lam
        if lam:
            # MoQAE trades accuracy for memory with a weight lambda on the
            # memory term; at inference the same pressure is a bias against
            # the wider experts
            pen = torch.tensor([16.0, 4.0, 2.0], device=device) / 16.0 * lam
            self.routers = [(W1, W2, W3, b3 - pen) for W1, W2, W3, b3 in self.routers]
        self.W1, self.W2, self.W3, self.b3 = self.routers[0]
        self.router = router
        if router == "similarity":
            # one query vector per sequence (per layer and sequence without
            # routing sharing); thresholds at the workload's target mix
            self.u = [W.similarity_query(w, seed + (l if not routing_sharing else 0), device)
                      for l in range(nr)]
            self.tau = W.similarity_thresholds(w)
        take = (lambda x: CS.shard_rows(x, self.full_lens, self.lo, self.hi)) if shard else \
            (lambda x: x)
        self.C = take(W.router_input(w, self.full_lens, seed, device))
        # every layer's K/V resident, or (streamed workloads) one layer's at a
        # time, drawn just before that layer's pack
        self.streamed = w.kv_streamed
        self.seed, self.device, self.take = seed, device, take
        self.K, self.V, self.q = [], [], []
        for layer in range(w.layers):
            if not self.streamed:
                K, V = W.kv_layer(w, self.full_lens, layer, seed, device)
                self.K.append(take(K))
                self.V.append(take(V))
                del K, V
            self.q.append([W.query(w, layer, s, seed, device) for s in range(w.decode_steps)])
        if self.streamed:
            self.K_cur, self.V_cur = self.draw_kv(0)
            self.flush_buf = torch.ones(2 * L2_BYTES, dtype=torch.uint8, device=device)
        u8 = torch.uint8
        self.route_ws = torch.empty(M.mq_route_workspace_bytes(self.shape, self.lens, w.router_dim,
                                                                w.router_hidden),
                                    dtype=u8, device=device)
        self.token_expert = torch.empty(self.T, dtype=u8, device=device)
        self.chunk_experts = [torch.empty(max(self.N, 16), dtype=u8, device=device)
                              for _ in range(nr)]
        self.layouts = [torch.empty(M.mq_layout_bytes(self.shape, self.lens), dtype=u8,
                                    device=device) for _ in range(nr)]
        self.chunk_expert = self.chunk_experts[0]
        self.layout = self.layouts[0]
        # packed buffers: the inputs are the same every step, so the map is
        # too; route once here and size every buffer at the packed bytes of
        # its layout (no host round trip separates routing from packing in
        # the timed steps; a larger map would be caught by the pack kernel's
        # capacity check)
        self._route_maps()
        self._build_layouts()
        need = max(M.mq_packed_bytes(lay) for lay in self.layouts)
        self.packed = [torch.empty(max(need, 16), dtype=u8, device=device)
                       for _ in range(w.layers)]
        self.out = [torch.empty(self.B, w.num_q_heads, w.head_dim, dtype=torch.float32,
                                device=device) for _ in range(w.layers)]
        self.ws = torch.empty(M.mq_decode_workspace_bytes(self.shape, self.lens), dtype=u8,
                              device=device)
        self.grow = grow
        if grow:
            if shard is not None:
                raise SystemExit("--grow and --context-split are separate variants")
            self._setup_grow(seed, device)
        if shard is not None:
            # this rank's records, all ranks' records, the merged output
            d4 = M.partial_floats(w.head_dim)
            self.rec = torch.empty(self.B, w.num_q_heads, d4, dtype=torch.float32, device=device)
        if self.streamed:
            self.kv_bytes = self.K_cur.numel() * self.K_cur.element_size() * 2
        else:
            self.kv_bytes = sum(K.numel() * K.element_size() * 2 for K in self.K) // w.layers
        torch.cuda.synchronize()

    def draw_kv(self, layer):
        """K, V of one layer (streamed workloads): the workload's draw for
        that layer, on the device."""
        from chunk_adaptive_mixed_b200 import workloads as W
        K, V = W.kv_layer(self.w, self.full_lens, layer, self.seed, self.device)
        return self.take(K), self.take(V)

    def kv_of(self, layer, loader=None):
        """K, V that the pack of `layer` reads.  Streamed workloads first
        draw them (or copy them in with `loader`) and then read a 2 x L2
        buffer (l2_evict), so that the pack reads its input from HBM like the
        resident workloads do; both happen outside the timed spans."""
        if not self.streamed:
            return self.K[layer], self.V[layer]
        if loader is not None:
            loader(layer, self.K_cur, self.V_cur)
        else:
            self.K_cur, self.V_cur = None, None
            self.K_cur, self.V_cur = self.draw_kv(layer)
        l2_evict(self.flush_buf)
        return self.K_cur, self.V_cur

    def _setup_grow(self, seed, device):
        """Growable layout sized for decode_steps more tokens, the appended
        tokens' K/V and router-input rows, and which sequences fill a chunk at
        which step (lengths are known on the host)."""
        import torch
        from chunk_adaptive_mixed_b200 import mqkv as M
        from chunk_adaptive_mixed_b200 import workloads as W
        w, u8 = self.w, torch.uint8
        if self.router != "moqae" or not self.rs:
            raise SystemExit("--grow runs with the MoQAE router and routing sharing")
        n = w.decode_steps
        lay_b, pk_b, ws_b = M.mq_grow_sizes(self.shape, self.lens, n)
        self.cap_lens = self.lens + n
        self.layouts = [torch.empty(lay_b, dtype=u8, device=device)]
        self.layout = self.layouts[0]
        self.packed = [torch.empty(pk_b, dtype=u8, device=device) for _ in range(w.layers)]
        self.ws = torch.empty(ws_b, dtype=u8, device=device)
        self.kv_new = [[W.new_token_kv(w, l, s, seed, device) for s in range(n)]
                       for l in range(w.layers)]
        self.c_new = [W.new_token_router_input(w, s, seed, device) for s in range(n)]
        L, B = w.chunk_len, self.B
        # router input of every sequence's open tail, [B * L, D]: the prefill's
        # partial chunk, then one row per appended token
        self.tail_c0 = torch.zeros(B * L, w.router_dim, dtype=torch.float32, device=device)
        cu = W.cu_seqlens(self.lens)
        for b in range(B):
            t = int(self.lens[b]) % L
            if t:
                self.tail_c0[b * L:b * L + t] = self.C[int(cu[b + 1]) - t:int(cu[b + 1])]
        self.tail_c = self.tail_c0.clone()
        self.tail_lens = np.full(B, L, np.int32)
        self.tail_cu = torch.as_tensor(W.cu_seqlens(self.tail_lens), device=device)
        self.tail_te = torch.empty(B * L, dtype=u8, device=device)
        self.tail_ce = torch.empty(max(B, 16), dtype=u8, device=device)
        self.tail_ws = torch.empty(M.mq_route_workspace_bytes(self.shape, self.tail_lens,
                                                              w.router_dim, w.router_hidden),
                                   dtype=u8, device=device)
        self.sealed = torch.full((max(B, 16),), 255, dtype=u8, device=device)
        self.no_seal = torch.full((max(B, 16),), 255, dtype=u8, device=device)
        self.tail_row, self.fill_mask, self.fills = [], [], []
        lens = self.lens.astype(np.int64).copy()
        for s in range(n):
            pos = lens % L                          # row of the new token in its tail
            self.tail_row.append(torch.as_tensor(np.arange(B) * L + pos, device=device))
            lens += 1
            full = lens % L == 0
            mask = np.zeros(max(B, 16), bool)
            mask[:B] = full
            self.fill_mask.append(torch.as_tensor(mask, device=device))
            self.fills.append(int(full.sum()))

    def step_grow(self, timers=None):
        """Prefill (route, growable layout, pack) then decode_steps decode
        steps that each append one token per sequence before attending."""
        import torch
        from chunk_adaptive_mixed_b200 import mqkv as M
        w, n = self.w, self.w.decode_steps
        if timers:
            timers["route"][0].record()
        M.mq_route_chunks(self.shape, self.lens, self.cu, self.C, self.W1, self.W2, self.W3,
                          self.b3, self.token_expert, self.chunk_expert, self.route_ws)
        if timers:
            timers["route"][1].record()
        M.mq_grow_build_layout(self.shape, self.lens, n, self.cu, self.chunk_expert, self.layout)
        for layer in range(w.layers):
            if timers:
                timers["pack"][layer][0].record()
            M.mq_grow_pack_kv(self.shape, self.lens, n, self.layout, self.K[layer], self.V[layer],
                              self.packed[layer])
            if timers:
                timers["pack"][layer][1].record()
        self.tail_c.copy_(self.tail_c0)
        pending = False
        for s in range(n):
            M.mq_grow_commit(self.shape, self.layout, self.sealed if pending else None, True)
            self.tail_c.index_copy_(0, self.tail_row[s], self.c_new[s])
            for layer in range(w.layers):
                Kn, Vn = self.kv_new[layer][s]
                M.mq_grow_append_kv(self.shape, self.layout, Kn, Vn, self.packed[layer])
                if timers:
                    timers["decode"][s * w.layers + layer][0].record()
                M.mq_decode_attn(self.shape, self.cap_lens, self.layout, self.packed[layer],
                                 self.q[layer][s], self.out[layer], self.ws)
                if timers:
                    timers["decode"][s * w.layers + layer][1].record()
            pending = self.fills[s] > 0
            if pending:
                # route the full tails (all B tails are scored; only the full
                # ones are sealed)
                M.mq_route_chunks(self.shape, self.tail_lens, self.tail_cu, self.tail_c, self.W1,
                                  self.W2, self.W3, self.b3, self.tail_te, self.tail_ce,
                                  self.tail_ws, routing_freeze=False)
                torch.where(self.fill_mask[s], self.tail_ce, self.no_seal, out=self.sealed)
                for layer in range(w.layers):
                    M.mq_grow_seal(self.shape, self.layout, self.sealed, self.packed[layer])

    def step(self, timers=None, loader=None):
        """One pass of the whole path (launches only; asynchronous).  With a
        streamed workload, each layer's K/V are drawn (or copied in by
        `loader`) between the timed spans."""
        from chunk_adaptive_mixed_b200 import mqkv as M
        w = self.w
        if self.grow:
            return self.step_grow(timers)
        if timers:
            timers["route"][0].record()
        self._route_maps()
        if timers:
            timers["route"][1].record()
            timers["layout"][0].record()
        self._build_layouts()
        if timers:
            timers["layout"][1].record()
        for layer in range(w.layers):
            K, V = self.kv_of(layer, loader)
            if timers:
                timers["pack"][layer][0].record()
            M.mq_pack_kv(self.shape, self.lens, self.layout_of(layer), K, V, self.packed[layer])
            if timers:
                timers["pack"][layer][1].record()
        for s in range(w.decode_steps):
            for layer in range(w.layers):
                if timers:
                    timers["decode"][s * w.layers + layer][0].record()
                if self.shard is None:
                    M.mq_decode_attn(self.shape, self.lens, self.layout_of(layer),
                                     self.packed[layer], self.q[layer][s], self.out[layer],
                                     self.ws)
                else:
                    self.decode_split(layer, s)
                if timers:
                    timers["decode"][s * w.layers + layer][1].record()

    def _route_maps(self):
        from chunk_adaptive_mixed_b200 import mqkv as M
        for r, (W1, W2, W3, b3) in enumerate(self.routers):
            if self.router == "similarity":
                M.mq_similarity_route(self.shape, self.lens, self.cu, self.C, self.u[r],
                                      self.tau[0], self.tau[1], self.chunk_experts[r])
            else:
                M.mq_route_chunks(self.shape, self.lens, self.cu, self.C, W1, W2, W3, b3,
                                  self.token_expert, self.chunk_experts[r], self.route_ws,
                                  routing_freeze=self.freeze)

    def _build_layouts(self):
        from chunk_adaptive_mixed_b200 import mqkv as M
        for r in range(len(self.routers)):
            M.mq_build_layout(self.shape, self.lens, self.cu, self.chunk_experts[r],
                              self.layouts[r])

    def decode_split(self, layer, s):
        """This rank's records, the all-gather over every rank, the merge."""
        from chunk_adaptive_mixed_b200 import context_split as CS
        from chunk_adaptive_mixed_b200 import mqkv as M
        M.mq_decode_attn_partial(self.shape, self.lens, self.layout_of(layer), self.packed[layer],
                                 self.q[layer][s], self.rec, self.ws)
        M.mq_combine_partials(CS.gather_records(self.rec), self.out[layer])

    def layout_of(self, layer):
        return self.layouts[0 if self.rs else layer]

    def launches_per_step(self):
        return launches_per_step(self.w, len(self.routers), self.router,
                                 sum(1 for f in self.fills if f) if self.grow else None,
                                 self.shard is not None)

    def route_work(self):
        """Algorithmic work of one map: (amount, unit, bound).  The router is
        two D x H projections per token (the small W3 product aside); the
        similarity search reads C and u once and writes one byte per chunk."""
        w = self.w
        if self.router == "similarity":
            return (self.T * w.router_dim * 4 + self.B * w.router_dim * 4 + self.N, "GB/s", "hbm")
        return (4.0 * self.T * w.router_dim * w.router_hidden, "TFLOP/s", "tensor")


def decode_kernels_per_call(w) -> int:
    """The library's kernels in one decode call: with fp16 queries, d = 128 and
    one or four query heads per kv-head the tensor-core decode comes with its
    prep kernel (work-order table, counters) and the merge; the other decode
    kernels with the merge only (a memset clears their counter)."""
    tc = w.kv_dtype == "f16" and w.head_dim == 128 and w.num_q_heads // w.num_kv_heads in (1, 4)
    return 3 if tc else 2


def launches_per_step(w, n_maps: int, router: str, fill_steps=None, split: bool = False) -> int:
    """The library's kernel launches in one step.  Per map: weight split +
    router + vote (or one similarity kernel) and 2 layout kernels; one pack per
    layer; one decode call per layer and decode step.  Growth (fill_steps =
    decode steps that seal full tails): per decode step a commit (2 kernels)
    and per layer an append before the decode call; per sealing step the
    tails' routing (3) and one seal per layer.  A split context: a partial
    decode call and a combine per layer and decode step."""
    dk = decode_kernels_per_call(w)
    if split:
        return 5 * n_maps + w.layers + (dk + 1) * w.layers * w.decode_steps
    if fill_steps is not None:
        n = w.decode_steps
        return 5 + w.layers + n * (2 + (1 + dk) * w.layers) + fill_steps * (3 + w.layers)
    per_map = 3 if router == "similarity" else 5
    return per_map * n_maps + w.layers + dk * w.layers * w.decode_steps


DTYPE_DETAIL = ("router: fp32 operands, each product formed from bf16 parts (hi*hi + hi*lo + "
                "lo*hi, about 2^-16 relative per product) with fp32 accumulation on the tensor "
                "cores; pack: IEEE fp32; decode: codes and fp16 queries (or fp32 queries on the "
                "CUDA cores) as exact products, fp32 accumulation and softmax")


def line_config(w, full_lens, rs, router, lam, grow, context_split, world):
    """The workload description both arms print (identical for the same
    arguments)."""
    flush = kv_fits_l2(w, full_lens)
    return {"workload": w.name, "layers": w.layers, "num_seqs": len(full_lens),
            "seq_len": int(full_lens.max()), "total_tokens": int(full_lens.sum()),
            "q_heads": w.num_q_heads, "kv_heads": w.num_kv_heads,
            "head_dim": w.head_dim, "chunk_len": w.chunk_len,
            "router_D": w.router_dim, "router_H": w.router_hidden,
            "kv_dtype": w.kv_dtype, "decode_steps": w.decode_steps,
            "routing_sharing": rs, "router": router, "lam": lam, "grow": bool(grow),
            "kv": ("each layer's K/V drawn, then packed, in turn: only the packed cache "
                   "stays resident") if w.kv_streamed else "every layer's K/V resident",
            "step_time": ("sum of the library spans (route, layout, each pack, each decode); "
                          "the K/V draws and L2 flushes between them excluded")
            if w.kv_streamed and not grow and not context_split
            else "whole step on the device (CUDA events)",
            "parallelism": (f"cp{world} (context split, records all-gathered)"
                            if context_split else f"dp{world} (independent batches)"),
            "l2": ("2 x L2 buffer read before every step (outside its events; L2 left "
                   "clean); unflushed time in no_flush") if flush
            else ("inputs larger than 2 x L2; each layer's pack input follows a 2 x L2 read "
                  "(L2 left clean)" if w.kv_streamed else "inputs larger than 2 x L2 (no flush needed)")}


def kv_fits_l2(w, full_lens):
    """Whether one layer's K/V fit twice in L2 (then a flush precedes every step)."""
    elem = 4 if w.kv_dtype == "f32" else 2
    return int(full_lens.sum()) * w.num_kv_heads * w.head_dim * elem * 2 < 2 * L2_BYTES


def run_ours(args, rank, world, local_rank):
    import torch
    from chunk_adaptive_mixed_b200 import build as Bld
    from chunk_adaptive_mixed_b200 import mqkv as M
    from chunk_adaptive_mixed_b200 import workloads as W
    Bld.build()
    M.lib()
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    w = workload(args)
    # independent batches per rank (weak scaling), or one shared batch split
    # by context (strong scaling)
    seed = args.seed if args.context_split else rank_seed(args.seed, rank)
    if args.lam and args.router != "moqae":
        raise SystemExit("--lam applies to the MoQAE router only")
    S = Setup(w, seed, device, routing_sharing=not args.no_rs, router=args.router, lam=args.lam,
              grow=args.grow, shard=(rank, world) if args.context_split else None)
    dist = world > 1
    if dist:
        import torch.distributed as tdist

    def barrier():
        if dist:
            tdist.barrier()

    for _ in range(args.warmup):
        S.step()
    torch.cuda.synchronize()
    assert M.mq_device_status() == 0, "device-side check failed during warm-up"
    if S.grow:
        # bytes the prefill map occupies (a growable layout's header counts
        # its reservations too): a fixed layout of the same map
        fixed = torch.empty(M.mq_layout_bytes(S.shape, S.lens), dtype=torch.uint8, device=device)
        M.mq_build_layout(S.shape, S.lens, S.cu, S.chunk_expert, fixed)
        pb = M.mq_packed_bytes(fixed)
        del fixed
    else:
        pb = int(np.mean([M.mq_packed_bytes(S.layout_of(l)) for l in range(w.layers)]))
    mix = np.bincount(S.chunk_expert[:S.N].cpu().numpy(), minlength=3) / max(S.N, 1)

    # per-kernel events for every pack launch and every decode call.
    # Workloads whose K/V fit twice in L2 would leave the next step's inputs
    # cached: those read a 2 x L2 buffer before every step (l2_evict),
    # outside the step's events, and report the unflushed time beside it.
    E = torch.cuda.Event
    flush = S.kv_bytes < 2 * L2_BYTES
    flush_buf = torch.ones(2 * L2_BYTES, dtype=torch.uint8, device=device) if flush else None
    if S.streamed and w.decode_steps != 1:
        raise SystemExit("streamed K/V workloads time one decode step per layer")

    def timed_steps(with_flush):
        timers, spans = [], []
        for _ in range(args.steps):
            if with_flush:
                l2_evict(flush_buf)
            tm = {"route": (E(enable_timing=True), E(enable_timing=True)),
                  "layout": (E(enable_timing=True), E(enable_timing=True)),
                  "pack": [(E(enable_timing=True), E(enable_timing=True)) for _ in range(w.layers)],
                  # every decode call of the step (layers x decode steps)
                  "decode": [(E(enable_timing=True), E(enable_timing=True))
                             for _ in range(w.layers * w.decode_steps)]}
            if with_flush or not spans:
                spans.append((E(enable_timing=True), E(enable_timing=True)))
                spans[-1][0].record()
            S.step(tm)
            if with_flush:
                spans[-1][1].record()
            timers.append(tm)
        if not with_flush:
            spans[-1][1].record()
        return timers, spans

    no_flush = None
    if flush:
        barrier()
        torch.cuda.synchronize()
        _, spans_nf = timed_steps(False)
        torch.cuda.synchronize()
        ms_nf = reduce_timing(sum(a.elapsed_time(b) for a, b in spans_nf), device)
        no_flush = {"ms_per_step": ms_nf / args.steps,
                    "value": job_throughput(S.B * w.decode_steps, world, ms_nf / args.steps)
                    if not args.context_split else S.B * w.decode_steps / (ms_nf / args.steps / 1e3)}
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()
    timers_all, spans = timed_steps(flush)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    assert M.mq_device_status() == 0, "device-side check failed in the timed region"
    if S.streamed:
        # the step is the sum of its library spans (route, layout, every pack
        # and decode); the draws of each layer's K/V and the L2 flush after
        # them lie between the spans and are not the method's work
        def step_spans(tm):
            pairs = [tm["route"], tm["layout"]] + list(tm["pack"]) + list(tm["decode"])
            return sum(a.elapsed_time(b) for a, b in pairs)
        ms = reduce_timing(sum(step_spans(tm) for tm in timers_all), device)
    else:
        ms = reduce_timing(sum(a.elapsed_time(b) for a, b in spans), device)
    ms_step = ms / args.steps
    pack_ms = [a.elapsed_time(b) for tm in timers_all for a, b in tm["pack"]]
    dec_ms = [a.elapsed_time(b) for tm in timers_all for a, b in tm["decode"]]
    route_ms = float(np.mean([tm["route"][0].elapsed_time(tm["route"][1]) for tm in timers_all]))
    pack_avg = float(np.mean(pack_ms))
    dec_avg = float(np.mean(dec_ms))

    def spread(xs):
        """Median, 10th and 90th percentile of per-launch times (ms)."""
        return {"median_ms": float(np.median(xs)), "p10_ms": float(np.percentile(xs, 10)),
                "p90_ms": float(np.percentile(xs, 90)), "launches": len(xs)}

    tokens_per_step = S.B * w.decode_steps
    if args.context_split:
        value = tokens_per_step / (ms_step / 1e3)    # every rank works on the same sequences
    else:
        value = job_throughput(tokens_per_step, world, ms_step)
    peak, peak_kind = measured_peaks()
    pack_bytes = S.kv_bytes + pb                                   # read K/V, write packed
    dec_bytes = pb + sum(x.numel() * x.element_size() for x in (S.q[0][0], S.out[0]))
    pack_gbs = pack_bytes / (pack_avg / 1e3) / 1e9
    dec_gbs = dec_bytes / (dec_avg / 1e3) / 1e9

    # end to end through the same calls, inputs in pinned host memory
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(S, args, device)
    cpu = routing = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gpu_maps = None
        if S.router == "moqae" and S.rs and not S.grow and not S.lam:
            gpu_maps = (S.token_expert[:S.T].cpu().numpy(), S.chunk_expert[:S.N].cpu().numpy())
        cpu, routing = cpu_baseline(w, S.lens, seed, tokens_per_step, S.router, len(S.routers),
                                    one_core=flush, gpu_maps=gpu_maps, draw_device=device)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "strong" if args.context_split else "weak",
            "vs_baseline": None, "dtype": "f32", "dtype_detail": DTYPE_DETAIL,
            "data": "synthetic (seeded; random tensors of the model's shape, no checkpoint)",
            "config": line_config(w, S.full_lens, S.rs, S.router, S.lam, S.grow,
                                  args.context_split, world),
            "roofline": {"bound": "hbm", "kernel": "pack_kernel",
                         "achieved": pack_gbs, "peak": peak, "unit": "GB/s",
                         "frac": pack_gbs / peak, "traffic": pack_traffic(w, S, seed),
                         "peak_source": peak_kind,
                         "algorithmic_bytes_per_launch": pack_bytes,
                         "avg_launch_ms": pack_avg},
            "decode_attn": {"GB/s": dec_gbs, "frac": dec_gbs / peak, "avg_ms_per_layer": dec_avg,
                            "timed": "every decode call of every timed step (layers x decode steps)",
                            "frac_of_spec": dec_gbs / SPEC_HBM_GBS,
                            "tokens_per_s_attention_only": S.B / (dec_avg * w.layers / 1e3),
                            "algorithmic_bytes_per_layer": dec_bytes, **spread(dec_ms)},
            "route": route_summary(S, route_ms, peaks_all()),
            "pack": {"GB/s": pack_gbs, "frac": pack_gbs / peak, "avg_ms_per_layer": pack_avg,
                     "frac_of_spec": pack_gbs / SPEC_HBM_GBS, **spread(pack_ms)},
            "no_flush": no_flush,
            "packed_bytes_per_layer": pb,
            "chunk_mix": [round(float(x), 4) for x in mix],
            "avg_bits": float(np.dot(mix, [16, 4, 2])),
            "routing": routing,
            "clocks": clocks,
            "gpu_launches": S.launches_per_step() * args.steps,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def run_e2e(S, args, device):
    """Same step through the same ABI calls, with every step's inputs copied
    from pinned host memory inside the timed region and each layer's output
    read back."""
    import torch
    w = S.w
    def pinned_copy(t):
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        return h

    host = {}
    host["C"] = pinned_copy(S.C)
    if S.streamed:
        # a pool of two layers' K/V in pinned host memory (layer l copies
        # pool entry l % 2 in before its pack): every layer's bytes cross the
        # host link, with host memory bounded; the packed contents then
        # follow the pool, not the layer's own draw
        pool = [S.draw_kv(l) for l in range(min(2, w.layers))]
        host["K"] = [pinned_copy(K) for K, _ in pool]
        host["V"] = [pinned_copy(V) for _, V in pool]
        del pool
    else:
        host["K"] = [pinned_copy(K) for K in S.K]
        host["V"] = [pinned_copy(V) for V in S.V]
    host["q"] = [[pinned_copy(q) for q in qs] for qs in S.q]
    host["u"] = [pinned_copy(u) for u in S.u] if S.router == "similarity" else []
    # decode-time growth: every appended token's K/V and router-input row
    host["kv_new"] = ([[(pinned_copy(k), pinned_copy(v)) for k, v in per] for per in S.kv_new]
                      if S.grow else [])
    host["c_new"] = [pinned_copy(c) for c in S.c_new] if S.grow else []
    out_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in S.out]
    h2d = (host["C"].numel() * 4 + sum(u.numel() * 4 for u in host["u"])
           + sum(k.numel() * k.element_size() * 2 for per in host["kv_new"] for k, _ in per)
           + sum(c.numel() * 4 for c in host["c_new"])
           + (S.kv_bytes * w.layers if S.streamed
              else sum(x.numel() * x.element_size() for x in host["K"] + host["V"]))
           + sum(q.numel() * q.element_size() for qs in host["q"] for q in qs))

    def load_layer(layer, K, V):
        K.copy_(host["K"][layer % len(host["K"])], non_blocking=True)
        V.copy_(host["V"][layer % len(host["V"])], non_blocking=True)
    # each layer's output after the step's last decode step
    d2h = sum(o.numel() * o.element_size() for o in out_host)

    def e2e_step():
        S.C.copy_(host["C"], non_blocking=True)
        for r, u in enumerate(host["u"]):
            S.u[r].copy_(u, non_blocking=True)
        for layer, per in enumerate(host["kv_new"]):
            for s_, (k, v) in enumerate(per):
                S.kv_new[layer][s_][0].copy_(k, non_blocking=True)
                S.kv_new[layer][s_][1].copy_(v, non_blocking=True)
        for s_, c in enumerate(host["c_new"]):
            S.c_new[s_].copy_(c, non_blocking=True)
        for layer in range(w.layers):
            if not S.streamed:
                S.K[layer].copy_(host["K"][layer], non_blocking=True)
                S.V[layer].copy_(host["V"][layer], non_blocking=True)
            for s in range(w.decode_steps):
                S.q[layer][s].copy_(host["q"][layer][s], non_blocking=True)
        S.step(loader=load_layer if S.streamed else None)
        for layer in range(w.layers):
            out_host[layer].copy_(S.out[layer], non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    world = 1
    import torch.distributed as tdist
    if tdist.is_available() and tdist.is_initialized():
        world = tdist.get_world_size()
        tdist.barrier()
    E = torch.cuda.Event
    a, b = E(enable_timing=True), E(enable_timing=True)
    a.record()
    for _ in range(args.e2e_steps):
        e2e_step()
    b.record()
    torch.cuda.synchronize()
    ms = reduce_timing(a.elapsed_time(b) / args.e2e_steps, device)
    del host
    res = e2e_result(S.B * w.decode_steps, world, ms, reduce_sum(h2d, device),
                     reduce_sum(d2h, device), args.e2e_steps, bool(args.context_split))
    res["timed"] = ("whole step including every host-to-device and device-to-host copy"
                    + ("; K/V from a two-layer pinned pool" if S.streamed else ""))
    return res


# ------------------------------------------------------------------ CPU oracle

def route_sample_chunks(N, count, group=4):
    """Chunk indices of the routing sample: `count` chunks in groups of
    `group` consecutive chunks spread evenly over the batch (first and last
    chunk included)."""
    count = min(count, N)
    ng = max(1, count // group)
    starts = np.unique(np.linspace(0, max(N - group, 0), ng).round().astype(np.int64))
    out = sorted({int(c) for s0 in starts for c in range(s0, min(s0 + group, N))} | {N - 1})
    return out[:max(count, 1)] if len(out) > count else out


def oracle_step_estimate(w, lens, seed, route_chunks=32, pack_tokens=32768, router="moqae",
                         maps=1, gpu_maps=None, draw_device="cpu"):
    """Times the CPU oracle on a bounded sample of one step: the map of
    `route_chunks` chunks spread over the batch, and pack + decode of the
    first `pack_tokens` tokens of one layer of the first sequence.  Each
    phase's time is scaled by its share of the full step.

    gpu_maps = (token_expert, chunk_expert) of the GPU (numpy, whole batch):
    the sampled chunks' choices are then compared with the oracle's, near
    ties counted (MoQAE router, fp64 top-2 gap below 1e-3).  The router
    weights and the sampled router-input rows are then drawn on draw_device
    (the GPU run's device: torch's CPU and CUDA generators give different
    streams) and copied to the host.

    Returns a dict: projected (s per full step), measured (s of the sample),
    sample (text), cores, routing (the comparison, or None)."""
    from chunk_adaptive_mixed_b200 import workloads as W
    from oracle import oracle as O
    L = w.chunk_len
    W1, W2, W3, b3 = (x.cpu().numpy() for x in W.router_weights(w, seed, draw_device))
    T = int(lens.sum())
    counts_all = W.chunk_token_counts(lens, L).astype(np.int64)
    row0 = np.concatenate([[0], np.cumsum(counts_all)])
    N = len(counts_all)
    chunks = route_sample_chunks(N, route_chunks)
    # contiguous runs of sampled chunks: one router-input draw each
    runs, r = [], [chunks[0], chunks[0] + 1]
    for c in chunks[1:]:
        if c == r[1]:
            r[1] += 1
        else:
            runs.append(tuple(r))
            r = [c, c + 1]
    runs.append(tuple(r))
    Cs = [W.router_input(w, lens, seed, draw_device, chunk_range=rr).cpu().numpy()
          for rr in runs]
    counts = counts_all[chunks].astype(np.int32)
    t_route = 0.0
    routing = None
    if router == "similarity":
        u = W.similarity_query(w, seed, "cpu").numpy()[:1]
        tau_hi, tau_lo = W.similarity_thresholds(w)
        for C in Cs:
            t0 = time.perf_counter()
            O.similarity_route(np.array([C.shape[0]], np.int32), L, C, u, tau_hi, tau_lo)
            t_route += time.perf_counter() - t0
    else:
        z32s, z64s = [], []
        for C in Cs:
            t0 = time.perf_counter()
            z32, z64 = O.router_logits(C, W1, W2, W3, b3)
            t_route += time.perf_counter() - t0
            z32s.append(z32)
            z64s.append(z64)
        z32, z64 = np.concatenate(z32s), np.concatenate(z64s)
        te_o = O.token_argmax(z32)
        t0 = time.perf_counter()
        ce_o = O.vote(counts, L, te_o, False)
        t_route += time.perf_counter() - t0
        if gpu_maps is not None:
            te_g, ce_g = gpu_maps
            rows = np.concatenate([np.arange(row0[c], row0[c + 1]) for c in chunks])
            near = O.top2_gap(z64) < 1e-3
            te_s = te_g[rows]
            mism = int(((te_s != te_o) & ~near).sum())
            first = set((np.concatenate([[0], np.cumsum((lens + L - 1) // L)])[:-1])[lens > 0]
                        .tolist())
            exempt = chunk_mism = 0
            off = 0
            for i, c in enumerate(chunks):
                n = int(counts[i])
                want = 0 if c in first else int(ce_o[i])   # routing freezing
                if int(ce_g[c]) != want:
                    cnt = np.sort(np.bincount(te_o[off:off + n], minlength=3))
                    if cnt[-1] - cnt[-2] <= int(near[off:off + n].sum()) and c not in first:
                        exempt += 1
                    else:
                        chunk_mism += 1
                off += n
            routing = {"sampled_chunks": len(chunks), "sampled_tokens": int(counts.sum()),
                       "near_tie_tokens": int(near.sum()), "exempt_chunks": exempt,
                       "token_mismatches_outside_band": mism,
                       "chunk_mismatches_outside_band": chunk_mism}
    t_route_full = t_route * T / max(int(counts.sum()), 1) * maps
    # packing and decode: 1 layer of the first sequence, capped at pack_tokens
    Tp = int(min(lens[0], pack_tokens))
    lens1 = np.array([Tp], np.int32)
    K, V = W.kv_layer(w, lens1, 0, seed, "cpu")
    cmap = W.synthetic_chunk_map(lens1, L, mix=w.target_mix, seed=1)
    Kn, Vn = K.numpy(), V.numpy()
    t0 = time.perf_counter()
    packed = O.pack(w.num_kv_heads, w.head_dim, L, lens1, cmap, Kn, Vn)
    t_pack = time.perf_counter() - t0
    # decode: 1 layer of the same sample
    q = W.query(w, 0, 0, seed, "cpu").numpy()[:1]
    t0 = time.perf_counter()
    O.decode(w.num_q_heads, w.num_kv_heads, w.head_dim, L, lens1, cmap, packed, q)
    t_dec = time.perf_counter() - t0
    full = (t_route_full + t_pack * (T / Tp) * w.layers
            + t_dec * (T / Tp) * w.layers * w.decode_steps)
    sample = (f"{router} map of {int(counts.sum())} tokens ({len(chunks)} chunks spread over "
              f"the batch, x {maps} maps), pack + decode of {Tp} tokens of 1 layer; each "
              f"phase scaled to {T} tokens x {w.layers} layers x {w.decode_steps} decode "
              f"step(s)")
    return {"projected": full, "measured": t_route + t_pack + t_dec, "sample": sample,
            "cores": O.num_threads(), "routing": routing}


def cpu_baseline(w, lens, seed, tokens_per_step, router="moqae", maps=1, one_core=False,
                 gpu_maps=None, draw_device="cpu"):
    """The oracle on all host cores; with one_core (the small workloads) also
    on a single core.  The value is a projection: the sample's measured time
    of each phase scaled to the full step."""
    est = oracle_step_estimate(w, lens, seed, route_chunks=128, router=router, maps=maps,
                               gpu_maps=gpu_maps, draw_device=draw_device)
    out = {"value": tokens_per_step / est["projected"], "unit": "tokens/s", "cores": est["cores"],
           "kind": "oracle", "sample": est["sample"], "projected_s_per_step": est["projected"],
           "measured_sample_s": est["measured"], "value_is": "projection from the sample"}
    if one_core:
        from oracle import oracle as O
        prev = O.num_threads()
        O.set_num_threads(1)
        try:
            e1 = oracle_step_estimate(w, lens, seed, route_chunks=128, router=router, maps=maps)
        finally:
            O.set_num_threads(prev)
        out["one_core"] = {"value": tokens_per_step / e1["projected"],
                           "projected_s_per_step": e1["projected"]}
    return out, est["routing"]


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands, on bounded samples.
    Each timed step runs one sample (the map of a few chunks spread over the
    batch, pack + decode of a slice of one layer); ms_per_step is that
    sample's measured time and value the step's tokens over the sample's
    time scaled, phase by phase, to the full step."""
    if rank != 0:
        return
    from chunk_adaptive_mixed_b200 import workloads as W
    w = workload(args)
    lens = W.seq_lens(w, args.seed)
    tokens_per_step = len(lens) * w.decode_steps
    # a smaller sample per step than the cpu_baseline leg, so that K + W
    # steps stay within a few minutes
    kw = dict(route_chunks=8, pack_tokens=8192, router=args.router,
              maps=w.layers if args.no_rs else 1)
    for _ in range(args.warmup):
        oracle_step_estimate(w, lens, args.seed, **kw)
    proj, meas = [], []
    t_start = time.perf_counter()
    for _ in range(args.steps):
        est = oracle_step_estimate(w, lens, args.seed, **kw)
        proj.append(est["projected"])
        meas.append(est["measured"])
    wall = time.perf_counter() - t_start
    t_full = float(np.mean(proj))
    value = tokens_per_step / t_full
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": float(np.mean(meas)) * 1e3, "higher_is_better": True,
            "scaling": "strong" if args.context_split else "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": line_config(w, lens, not args.no_rs, args.router, args.lam, args.grow,
                                  args.context_split, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": est["cores"],
                             "kind": "oracle", "sample": est["sample"],
                             "value_is": "projection: each phase's sample time scaled to the "
                                         "full step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "ms_per_step_is": "measured time of one step's bounded sample",
            "projected_ms_per_full_step": t_full * 1e3,
            "sample_wall_s": wall}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus > 1 and world == 1:
        raise SystemExit("--gpus > 1 needs torchrun (one process per GPU)")
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                 device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as tdist
            tdist.destroy_process_group()


if __name__ == "__main__":
    main()
