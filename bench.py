#!/usr/bin/env python
"""Benchmark of the equivariant message-passing convolution on B200.

One step = one pass of the whole hot path over one batch of synthetic input
already resident in HBM: receiver-sorted CSR indexing of the edge list
(e3conv_build_csr) followed by the fused forward (e3conv_forward: gather,
channelwise CG product, scalar mix, segmented sum, 1/N scale, store).

Default workload: the large mixed-precision graph (100,000 nodes, ~4.0M
edges, 128x(0e+1o+2e+3o) float16 node features, Y for l <= 3, float16 edge
scalars, float32 accumulation and output, outputs l <= 3).  Its inputs
(~37 GB) are larger than L2, so no flush is needed between steps.

Prints one JSON line (rank 0).  `--impl reference` times the float64 CPU
oracle on a bounded sample of the same workload instead.
Multi-GPU (torchrun): one graph, its receiver rows partitioned into contiguous
CSR row ranges (one per rank, balanced on edges + rows); each step every rank
builds its rows' CSR, receives the node features its senders need from the
other ranks (NCCL all-gather, or a halo all-to-all with --exchange halo) and
runs e3conv_forward_rows on its rows (strong scaling: the total work is fixed).
Times are the max over ranks; edges/s counts every rank's edges.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "edges/sec and achieved fraction of roofline (HBM GB/s or FP32 FMA) at 1 B200"
UNIT = "edges/s"
SMS = 148
FP32_LANES_PER_SM = 128
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="large_f16")
    ap.add_argument("--nodes", type=int, default=None,
                    help="override the node count at the same density (profiling cases)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--channels-per-lane", type=int, default=0)
    ap.add_argument("--block-threads", type=int, default=0)
    ap.add_argument("--stages", type=int, default=-1)
    ap.add_argument("--contract-first", type=int, default=-1)
    ap.add_argument("--path-split", type=int, default=-1,
                    help="warps that split a receiver row's paths (E3CONV_OPT_PATH_SPLIT)")
    ap.add_argument("--edge-vectors", type=int, default=0,
                    help="1: edge vectors as input, harmonics evaluated in the kernel")
    ap.add_argument("--tensor-cores", type=int, default=0,
                    help="1: the tensor-core forward variant (float16 inputs, 128 channels)")
    ap.add_argument("--exchange", choices=["allgather", "halo"], default="allgather",
                    help="multi-GPU: how a rank receives its senders' node features")
    ap.add_argument("--direct-pipeline", type=int, default=-1,
                    help="small channel counts: 1 loads the next edge during this edge's products")
    ap.add_argument("--copy-group", type=int, default=-1,
                    help="edges per ring group of the staged variant (1..4)")
    ap.add_argument("--a-layout", type=int, default=-1,
                    help="shared-memory layout of the contract-first A entries (0, 1, 2)")
    ap.add_argument("--radial", action="store_true",
                    help="edge scalars from the radial MLP on the tensor cores every step "
                         "(workloads with MLP scalars)")
    ap.add_argument("--next-rows", dest="next_rows", action="store_true", default=True,
                    help="after the timed region, time the backward and the irreps linear layer "
                         "on the same workload (supplementary entries with their rooflines; on "
                         "by default)")
    ap.add_argument("--no-next-rows", dest="next_rows", action="store_false",
                    help="skip the supplementary next-row timings")
    ap.add_argument("--backward-parts", type=int, default=-1,
                    help="launches of each backward kernel in the next-row timing (-1 automatic)")
    ap.add_argument("--no-graphs", action="store_true",
                    help="launch the step's kernels one by one instead of replaying CUDA graphs "
                         "of the CSR build and of the forward")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the supplementary timing of the tensor-core variant")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# accounting

def peaks():
    hbm, sm_max, src = FALLBACK_HBM_GBS, 1965.0, "fallback"
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        hbm = float(d.get("hbm_gbs", hbm))
        sm_max = float(d.get("sm_max_mhz", sm_max))
        src = "measured"
    fp32_tflops = SMS * FP32_LANES_PER_SM * 2 * sm_max * 1e6 / 1e12
    f16 = 1590.0
    if src == "measured":
        f16 = float(json.load(open(p)).get("bf16_tflops", f16))
    return {"hbm_gbs": hbm, "fp32_tflops": fp32_tflops, "f16_tflops": f16, "sm_max_mhz": sm_max,
            "source": src}


def algorithmic(conv, N, E, in_bytes):
    """Algorithmic bytes and FLOPs of one forward.

    bytes = E (ny b + P C b) + 4E (senders) + N (nx C b + 4 nout C + 4 (row_ptr)):
            every edge's Y and s once, every node's features once, every output once
            (with edge vectors as input, 16 bytes per edge replace the ny b of Y).
    flops = 2 E C (sum of CG nonzeros over paths + sum over paths of (2 l3 + 1)).
    """
    import numpy as np
    nnz = sum(int((np.abs(conv.cg(p)) > 1e-12).sum()) for p in range(conv.num_paths))
    mix = sum(2 * q.l3 + 1 for q in conv.paths)
    y_bytes = 16 if conv.edge_vectors else conv.ny * in_bytes   # vectors: float32 [E][4]
    nbytes = E * (y_bytes + conv.num_paths * conv.C * in_bytes) + 4 * E + \
        N * (conv.nx * conv.C * in_bytes + 4 * conv.nout * conv.C + 4)
    flops = 2 * E * conv.C * (nnz + mix)
    return nbytes, flops, nnz, mix


class Clocks:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""
    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.ident = str(device_index)

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.ident, "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == len(self.FIELDS):
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        power = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(power) if power else None}


def kernel_hash(conv) -> str:
    return hashlib.sha1(conv.kernel_source().encode()).hexdigest()[:16]


def traffic_for(workload, conv, N, E, edge_vectors=False):
    """DRAM bytes of one forward launch from a committed ncu capture of this same
    configuration (workload, node count, unchanged kernel source), else None.  A capture of a
    smaller graph is not scaled: the node table's L2 residency changes with the size."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if workload is None or edge_vectors or not os.path.exists(p):
        return None, None
    d = json.load(open(p)).get(f"{workload}@{N}")
    if not d or d.get("kernel_sha1") != kernel_hash(conv) or d.get("edges") != E:
        return None, None
    return float(d["dram_read_bytes"] + d["dram_write_bytes"]), d.get("source")


# ---------------------------------------------------------------------------
# oracle sample (CPU baseline and reference arm)

def prepare_sample(graph, rows, x_rows_fn, Y_fn, s_fn):
    """The oracle's float64 inputs for the receivers `rows` and all their edges (generated once)."""
    import numpy as np
    rp = np.zeros(graph.num_nodes + 1, np.int64)
    np.cumsum(np.bincount(graph.receivers, minlength=graph.num_nodes), out=rp[1:])
    edges = np.concatenate([np.arange(rp[b], rp[b + 1]) for b in rows])
    senders = graph.senders[edges]
    uniq, inv = np.unique(senders, return_inverse=True)
    x = x_rows_fn(uniq).astype(np.float64)
    n = max(len(rows), len(uniq))
    xr = np.zeros((n,) + x.shape[1:])
    xr[:len(uniq)] = x
    return {"x": xr, "Y": Y_fn(edges).astype(np.float64), "s": s_fn(edges).astype(np.float64),
            "senders": inv, "receivers": np.repeat(np.arange(len(rows)), np.diff(rp)[rows]),
            "n": n, "edges": len(edges)}


def run_oracle(spec, graph, prep, threads=0):
    """Times one oracle forward on a prepared sample; returns (edges/s, edges, secs)."""
    import oracle
    t0 = time.perf_counter()
    oracle.forward(spec.irreps_node, spec.irreps_sh, spec.irreps_out, prep["x"], prep["Y"],
                   prep["s"], prep["senders"], prep["receivers"], prep["n"],
                   graph.avg_num_neighbors, threads=threads)
    dt = time.perf_counter() - t0
    return prep["edges"] / dt, prep["edges"], dt


def oracle_sample_rate(spec, graph, rows, x_rows_fn, Y_fn, s_fn, threads=0):
    """Times the oracle on the receivers `rows` (all their edges); returns (edges/s, edges, secs)."""
    return run_oracle(spec, graph, prepare_sample(graph, rows, x_rows_fn, Y_fn, s_fn), threads)


def calibrated_rows(spec, graph, x_rows_fn, Y_fn, s_fn, target_s, seed=2024):
    """Seeded receivers whose oracle run takes about target_s seconds.  The oracle's rate
    grows with the sample (fixed per-call cost, OpenMP balance over few receivers), so the
    probe grows geometrically until one run takes at least a quarter of the target, and the
    sample is scaled from that last probe."""
    import numpy as np
    order = np.random.default_rng(seed).permutation(graph.num_nodes)
    n = min(16, graph.num_nodes)
    while True:
        rate, ne, dt = oracle_sample_rate(spec, graph, order[:n], x_rows_fn, Y_fn, s_fn)
        if n >= graph.num_nodes:
            return np.sort(order[:n])
        if dt >= 0.25 * target_s:
            want = int(min(graph.num_nodes, n * target_s / max(dt, 1e-9)))
            return np.sort(order[:max(want, n)])
        n = int(min(graph.num_nodes, n * min(8.0, max(2.0, 0.3 * target_s / max(dt, 1e-9)))))


def oracle_input_fns(spec, graph, x_dev=None, s_dev=None):
    """Host inputs of an oracle sample, as functions of the rows / edges it takes: x and
    drawn s from the seeded generator (read back from its device form when given: the
    numpy form draws ~6M values/s), Y and radial s from the oracle's own harmonics and
    radial MLP of the edge vectors, rounded to the workload dtype as the GPU's inputs are."""
    import numpy as np
    import torch

    import oracle
    from workloads import configs
    dt = configs.np_dtype(spec)

    def xf(rows):
        if x_dev is None:
            return configs.node_features_np(spec, graph.num_nodes, rows)
        return x_dev[torch.from_numpy(rows).to(x_dev.device)].cpu().numpy()

    def yf(edges):
        v = graph.vec[edges]
        return oracle.sh(spec.lmax, v / np.linalg.norm(v, axis=1, keepdims=True)).astype(dt)

    if spec.scalars == "normal":
        def sf(edges):
            if s_dev is None:
                return configs.scalars_np(spec, graph, edges)
            return s_dev[torch.from_numpy(edges).to(s_dev.device)].cpu().numpy()
    else:
        ws = configs.radial_weights(spec)

        def sf(edges):
            d = np.linalg.norm(graph.vec[edges], axis=1)
            s = oracle.radial_mlp(d, spec.graph["r"], ws)
            return s.reshape(len(edges), spec.num_paths, spec.C).astype(dt)
    return xf, yf, sf


# ---------------------------------------------------------------------------

def reduce_over_ranks(times_ms, edges, world, device=None):
    """Max of each time and sum of edges over the ranks (identity for one rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(times_ms), dtype=torch.float64, device=device)
    e = torch.tensor([float(edges)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(e, op=dist.ReduceOp.SUM)
    return t.tolist(), e.item()


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np

    import oracle
    from workloads import configs
    spec = configs.SPECS[args.workload]
    g = configs.make_graph(spec, args.nodes)
    try:
        import torch
        on_gpu = torch.cuda.is_available()
    except ImportError:
        on_gpu = False
    if on_gpu:
        # the drawn inputs come from the counter generator's device form (faster than the
        # numpy form); the harmonics and radial scalars from the oracle; it runs on the host
        dev = torch.device("cuda", 0)
        xf, yf, sf = oracle_input_fns(
            spec, g, configs.node_features_torch(spec, g.num_nodes, dev),
            configs.scalars_torch(spec, g, dev) if spec.scalars == "normal" else None)
    else:
        xf, yf, sf = oracle_input_fns(spec, g)
    per_step = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    rows = calibrated_rows(spec, g, xf, yf, sf, per_step)
    prep = prepare_sample(g, rows, xf, yf, sf)    # inputs generated once; steps time the oracle
    for _ in range(args.warmup):
        run_oracle(spec, g, prep)
    tot_e, tot_t = 0, 0.0
    for _ in range(args.steps):
        _, ne, dt = run_oracle(spec, g, prep)
        tot_e += ne
        tot_t += dt
    value = tot_e / tot_t
    cores = oracle.max_threads()
    sample = (f"{len(rows)} seeded receivers of {g.num_nodes} with all their "
              f"{tot_e // max(1, args.steps)} edges per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": spec.name, "description": spec.description, "nodes": g.num_nodes,
                   "edges": g.num_edges},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def edge_inputs(conv, configs, spec, g, e0, e1, vectors, dev):
    """The forward's per-edge operands for edges e0..e1-1 on the device: the harmonics
    [E][ny] in the workload dtype (e3conv_edge_harmonics of the edge vectors), or the edge
    vectors float32 [E][4] themselves; and the edge scalars, drawn, or the radial MLP of
    the edge vectors (e3conv_radial_scalars with the workload's seeded weights)."""
    import torch
    v4 = torch.from_numpy(configs.edge_vectors_np(g, e0, e1)).to(dev)
    Y = v4 if vectors else conv.edge_harmonics(v4)
    if spec.scalars == "normal":
        s = configs.scalars_torch(spec, g, dev, edges=(e0, e1))
    else:
        s = conv.radial_scalars(v4)
    torch.cuda.synchronize()
    return v4, Y, s


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import equivariant_graph_message_b200 as e3
    from workloads import configs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    spec = configs.SPECS[args.workload]
    g = configs.make_graph(spec, args.nodes)     # every rank: the same graph
    N, E = g.num_nodes, g.num_edges
    conv = e3.Conv(spec.irreps_node, spec.irreps_sh, spec.irreps_out, g.avg_num_neighbors,
                   dtype=spec.dtype)
    if args.channels_per_lane or args.block_threads or args.stages != -1:
        conv.set_launch_config(args.channels_per_lane, args.block_threads, args.stages)
    if args.contract_first != -1:
        conv.set_contract_first(args.contract_first)
    if args.tensor_cores:
        conv.set_tensor_cores(1)
    if args.path_split != -1:
        conv.set_path_split(args.path_split)
    if args.a_layout != -1:
        conv.set_a_layout(args.a_layout)
    if args.copy_group != -1:
        conv.set_copy_group(args.copy_group)
    if args.direct_pipeline != -1:
        conv.set_direct_pipeline(args.direct_pipeline)
    if spec.scalars == "radial":
        conv.set_radial_mlp(spec.graph["r"], [w.astype(np.float32)
                                               for w in configs.radial_weights(spec)])
    if args.radial:
        # the edge scalars come from the radial MLP on the tensor cores every step
        if spec.scalars != "radial":
            raise SystemExit("--radial needs a workload whose scalars are the radial MLP (mace)")
        args.edge_vectors = 1
    if args.edge_vectors:
        conv.set_edge_vectors(1)
    stream = torch.cuda.current_stream()
    sh = e3._stream_handle(stream)
    shard = None
    if world == 1:
        rows, E_loc = N, E
        x = configs.node_features_torch(spec, N, dev)
        _, Y, s = edge_inputs(conv, configs, spec, g, 0, E, args.edge_vectors, dev)
        senders = torch.from_numpy(g.senders.astype(np.int32)).to(dev)
        receivers = torch.from_numpy(g.receivers.astype(np.int32)).to(dev)
        table = x
    else:
        # receiver sharding: this rank's CSR row range, its edges, its own node rows; the
        # sender table is filled by the exchange step every forward
        from equivariant_graph_message_b200 import sharding
        rp_host = np.zeros(N + 1, np.int64)
        np.cumsum(np.bincount(g.receivers, minlength=N), out=rp_host[1:])
        shard = sharding.shard_graph(rp_host, g.senders, rank, world, args.exchange,
                                     requests=sharding.torch_requests(device=dev))
        b0, e0, e1 = shard.row_begin, shard.edge_begin, shard.edge_end
        rows, E_loc = shard.rows, e1 - e0
        own = configs.node_features_torch(spec, shard.own_rows, dev, first=b0)
        if args.exchange == "allgather":
            x = torch.zeros((shard.block_rows, conv.nx, conv.C), dtype=own.dtype, device=dev)
            x[:shard.own_rows] = own
        else:
            x = own
            send_idx = torch.from_numpy(shard.send_idx).to(dev)
            send_buf = torch.empty((len(shard.send_idx), conv.nx, conv.C), dtype=own.dtype,
                                   device=dev)
        del own
        table = torch.empty((shard.table_rows, conv.nx, conv.C), dtype=x.dtype, device=dev)
        _, Y, s = edge_inputs(conv, configs, spec, g, e0, e1, args.edge_vectors, dev)
        senders = torch.from_numpy(shard.senders).to(dev)
        receivers = torch.from_numpy((g.receivers[e0:e1] - b0).astype(np.int32)).to(dev)
    row_ptr = torch.empty(rows + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(max(E_loc, 1), dtype=torch.int32, device=dev)
    ws = torch.empty(e3.csr_workspace_size(E_loc, rows), dtype=torch.uint8, device=dev)
    out = torch.empty((rows, conv.nout, conv.C), dtype=torch.float32, device=dev)
    pY, ps, psend, prp, pout = (e3._ptr(t) for t in (Y, s, senders, row_ptr, out))
    ptab = e3._ptr(table)
    precv, pperm, pws = e3._ptr(receivers), e3._ptr(perm), e3._ptr(ws)
    ws_bytes = ws.numel()

    def exchange():
        if args.exchange == "halo":
            sharding.pack_halo(x, send_idx, out=send_buf)
            sharding.exchange_rows(shard, send_buf, table)
        else:
            sharding.exchange_rows(shard, x, table)

    def csr_part(h):
        e3._ok(e3._build_csr(precv, E_loc, rows, prp, pperm, pws, ws_bytes, h), "e3conv_build_csr")

    def radial_part(h):
        e3._ok(e3._radial_scalars(conv._h, pY, E_loc, ps, h), "e3conv_radial_scalars")

    def forward_part(h):
        if shard is None:
            conv.forward_raw(ptab, pY, ps, psend, prp, N, pout, h)
        else:
            conv.forward_rows_raw(ptab, shard.table_rows, pY, ps, psend, prp, 0, rows, pout, h)

    graphs = None

    def step(fwd_events=None, radial_events=None):
        if graphs:
            graphs["csr"].replay()
        else:
            csr_part(sh)
        if shard is not None:
            exchange()
        if args.radial:
            if radial_events:
                radial_events[0].record(stream)
            if graphs:
                graphs["radial"].replay()
            else:
                radial_part(sh)
            if radial_events:
                radial_events[1].record(stream)
        if fwd_events:
            fwd_events[0].record(stream)
        if graphs:
            graphs["forward"].replay()
        else:
            forward_part(sh)
        if fwd_events:
            fwd_events[1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert e3.csr_check(ws) and conv.check(), "bad index met during warm-up"
    if not args.no_graphs and world == 1:
        # one CUDA graph per part of the step (the library's calls launch on the capture
        # stream and neither allocate nor synchronise): a replay per part and step
        graphs = {}
        parts = [("csr", csr_part), ("forward", forward_part)]
        if args.radial:
            parts.insert(1, ("radial", radial_part))
        for name, fn in parts:
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                fn(e3._stream_handle(torch.cuda.current_stream()))
            graphs[name] = gr
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        assert e3.csr_check(ws) and conv.check(), "bad index met during the graph warm-up"
    info = conv.kernel_info()

    # inputs that fit in L2 would be read from it by the next step: then L2 is flushed before
    # every step, outside the step's own events, and the steps' event times are summed
    global _flush
    in_bytes = 2 if spec.dtype == "f16" else 4
    step_bytes = algorithmic(conv, N, E, in_bytes)[0] / world
    _flush = L2Flush(stream) if needs_l2_flush(step_bytes) else None
    clocks = Clocks(local)
    clocks.start()
    steps_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)]
    fwd = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    rad = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)] if args.radial else [None] * args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for k in range(args.steps):
        if _flush is not None:
            _flush()
            steps_ev[k][0].record(stream)
        step(fwd[k], rad[k])
        if _flush is not None:
            steps_ev[k][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = t0.elapsed_time(t1) if _flush is None else sum(a.elapsed_time(b) for a, b in steps_ev)
    fwd_ms = statistics.mean(a.elapsed_time(b) for a, b in fwd)
    rad_ms = statistics.mean(a.elapsed_time(b) for a, b in rad) if args.radial else 0.0
    (ms, fwd_ms, rad_ms), total_edges = reduce_over_ranks([ms, fwd_ms, rad_ms], E_loc, world, dev)
    ms_per_step = ms / args.steps
    value = total_edges / (ms_per_step / 1000.0)

    pk = peaks()
    in_bytes = 2 if spec.dtype == "f16" else 4
    # per GPU: the whole graph's algorithmic bytes and FLOPs over the ranks (the partition
    # balances edges + rows), against the slowest rank's forward time
    nbytes, flops, nnz, mix = algorithmic(conv, N, E, in_bytes)
    nbytes, flops = nbytes / world, flops / world
    traffic, traffic_src = traffic_for(spec.name if world == 1 else None, conv, N, E,
                                       bool(args.edge_vectors))
    sec = fwd_ms / 1000.0
    t_hbm = nbytes / (pk["hbm_gbs"] * 1e9)
    if info.get("tensor_cores"):
        # tensor-core variant: the CG x Y contraction runs as two tcgen05 MMAs per edge
        # (M = C, N = path outputs padded to 16, K = 16); only the s-scaling stays on FP32.
        ncols = -(-mix // 16) * 16
        tc_flops = 2 * 2 * E * conv.C * ncols * 16 / world
        fp32_flops = 2 * E * conv.C * mix / world
        times = {"hbm": t_hbm, "tensor": tc_flops / (pk["f16_tflops"] * 1e12),
                 "alu": fp32_flops / (pk["fp32_tflops"] * 1e12)}
    else:
        tc_flops, fp32_flops = 0, flops
        times = {"hbm": t_hbm, "alu": flops / (pk["fp32_tflops"] * 1e12)}
    bound = max(times, key=times.get)
    if bound == "hbm":
        achieved = nbytes / sec / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "traffic": traffic,
                "peak_source": f"hbm_gbs ({pk['source']})"}
    elif bound == "tensor":
        achieved = tc_flops / sec / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk["f16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / pk["f16_tflops"], "traffic": traffic,
                "peak_source": f"bf16_tflops ({pk['source']}); f16 dense = bf16 dense"}
    else:
        achieved = fp32_flops / sec / 1e12
        roof = {"bound": "alu", "achieved": achieved, "peak": pk["fp32_tflops"],
                "unit": "TFLOP/s", "frac": achieved / pk["fp32_tflops"], "traffic": traffic,
                "peak_source": f"derived: {SMS} SMs x {FP32_LANES_PER_SM} FP32 lanes x 2 x "
                               f"{pk['sm_max_mhz']:.0f} MHz (sm_max_mhz, {pk['source']})"}
    roof.update({"kernel": "e3conv_fwd", "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
                 "fp32_flops": fp32_flops, "tensor_flops": tc_flops, "forward_ms": fwd_ms,
                 "hbm_frac": nbytes / sec / 1e9 / pk["hbm_gbs"],
                 "fp32_equivalent_tflops": flops / sec / 1e12,
                 "roofline_times_ms": {k: 1000 * v for k, v in times.items()},
                 "traffic_source": traffic_src})

    radial = None
    if args.radial:
        # the radial kernel: tensor FLOPs of the hidden and output layers (3 MMAs per product
        # for the hi/lo splits) and the scalars it writes
        H = 64
        tflop = 3 * 2 * E * H * (H + conv.num_paths * conv.C) / world
        s_bytes = E * conv.num_paths * conv.C * in_bytes / world
        radial = {"kernel": "k_radial", "radial_ms": rad_ms,
                  "tensor_flops": tflop, "achieved_tflops": tflop / (rad_ms / 1000) / 1e12,
                  "tensor_peak_tflops": pk["f16_tflops"],
                  "tensor_frac": tflop / (rad_ms / 1000) / 1e12 / pk["f16_tflops"],
                  "scalars_bytes_written": s_bytes,
                  "write_gbs": s_bytes / (rad_ms / 1000) / 1e9,
                  "note": "edge scalars s = MLP(bessel x cutoff of |r|) computed every step; "
                          "the forward reads them back (value counts radial + forward)"}

    variants = None
    if world == 1 and not info.get("tensor_cores") and not args.no_variants and not args.radial:
        variants = {"tensor_cores": time_tensor_core_variant(args, spec, g, conv, x, Y, s, senders,
                                                            row_ptr, out, stream)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        xf, yf, sf = oracle_input_fns(spec, g, x, s if spec.scalars == "normal" else None)
        sample_rows = calibrated_rows(spec, g, xf, yf, sf, args.cpu_seconds)
        rate, ne, dt = oracle_sample_rate(spec, g, sample_rows, xf, yf, sf)
        cpu = {"value": rate, "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
               "sample": f"{len(sample_rows)} seeded receivers of {N} with all their {ne} edges "
                         f"({dt:.1f} s, float64 loops, OpenMP over receivers)"}

    e2e = None
    if not args.no_e2e:
        def device_step():
            # the public calls a user makes: CSR build, (exchange,) forward
            e3.build_csr(receivers, rows, row_ptr=row_ptr, perm=perm[:E_loc], workspace=ws)
            if args.radial:
                conv.radial_scalars(Y, out=s)
            if shard is None:
                conv.forward(table, Y, s, senders, row_ptr, out=out)
            else:
                exchange()
                conv.forward_rows(table, Y, s, senders, row_ptr, 0, rows, out=out)
        inputs = [x, Y, senders, receivers] if args.radial else [x, Y, s, senders, receivers]
        e2e = run_e2e(args, inputs, out, device_step, E_loc, world, dev)

    per_step = e3.csr_kernel_count(E_loc, rows) + 1 + (1 if args.exchange == "halo" and
                                                       world > 1 else 0) + (1 if args.radial else 0)
    launches = args.steps * per_step
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None,
        "dtype": "f16 inputs, f32 accumulation" if spec.dtype == "f16" else "f32",
        "data": "synthetic",
        "config": {"workload": spec.name, "description": spec.description, "nodes": N,
                   "edges": E, "edges_total": int(total_edges), "channels": conv.C,
                   "irreps_node": spec.irreps_node, "irreps_sh": spec.irreps_sh,
                   "irreps_out": spec.irreps_out, "input_dtype": spec.dtype,
                   "step": ("e3conv_build_csr + e3conv_forward" if world == 1 else
                            f"e3conv_build_csr (own rows) + node-feature {args.exchange} (NCCL) "
                            "+ e3conv_forward_rows"),
                   "parallelism": ("one GPU" if world == 1 else
                                   f"receiver rows sharded over {world} ranks "
                                   f"(e3conv_partition_rows), {args.exchange} exchange"),
                   "l2": (f"inputs larger than L2 ({nbytes / 1e9:.1f} GB read per forward per GPU)"
                          if _flush is None else
                          f"L2 flushed before every step ({nbytes / 1e6:.0f} MB read per forward "
                          "per GPU fits in L2; 256 MiB written outside the step's events, "
                          "steps timed one by one and summed)"),
                   "launch": ("CUDA graph replays (one graph per part of the step)" if graphs
                              else "eager launches"),
                   "forward_edges_per_s": total_edges / (fwd_ms / 1000.0),
                   "kernel": info},
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk,
    }
    if variants is not None:
        line["variants"] = variants
    if args.next_rows and world == 1:
        line["next_rows"] = time_next_rows(args, spec, g, conv, x, Y, s, senders, receivers,
                                           row_ptr, out, stream, pk)
    if radial is not None:
        line["radial"] = radial
        line["config"]["step"] = ("e3conv_build_csr + e3conv_radial_scalars + e3conv_forward "
                                  "(edge vectors)")
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


L2_BYTES = 126e6   # B200 L2


class L2Flush:
    """Evicts L2 between timed launches of a workload whose inputs would otherwise stay in it
    (outside the launch's own events): a 256 MiB device buffer is overwritten, then another
    one is read, so that the written lines are also written back before the launch and the
    launch meets a clean L2 that holds none of its inputs."""

    def __init__(self, stream):
        import torch
        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        self.clean = torch.ones(64 << 20, dtype=torch.float32, device="cuda")
        self.sink = torch.empty((), dtype=torch.float32, device="cuda")
        self.stream = stream

    def __call__(self):
        import torch
        with torch.cuda.stream(self.stream):
            self.buf.fill_(1)
            torch.sum(self.clean, dim=0, out=self.sink)


_flush = None   # set for workloads whose inputs fit in L2


def needs_l2_flush(step_bytes: float) -> bool:
    """Inputs smaller than twice the L2 would be partly read from it by the next step."""
    return step_bytes < 2 * L2_BYTES


def _event_ms(fn, reps, stream):
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    for a, b in ev:
        if _flush is not None:
            _flush()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in ev)


def time_next_rows(args, spec, g, conv, x, Y, s, senders, receivers, row_ptr, out, stream, pk):
    """Supplementary, after the timed region, on the same resident inputs: the backward
    (gradients of x, Y and s for a seeded upstream gradient) and the irreps linear layer on
    the forward's output (the output irreps mixed C -> C); CUDA events, inputs larger than L2."""
    import numpy as np
    import torch

    import equivariant_graph_message_b200 as e3
    N, E = g.num_nodes, g.num_edges
    res = {}
    reps = max(3, min(args.steps, 10))
    if args.backward_parts != -1:
        conv.set_backward_parts(args.backward_parts)
    if not conv.edge_vectors and conv.C <= (256 if spec.dtype == "f16" else 128):
        gout = torch.randn(out.shape, generator=torch.Generator(device=out.device).manual_seed(7),
                           device=out.device)
        srp, sperm, _ = e3.build_csr(senders, N)
        conv.backward(x, Y, s, senders, row_ptr, gout, receivers=receivers,
                      sender_row_ptr=srp, sender_perm=sperm)      # compile and warm up
        torch.cuda.synchronize()
        ms = _event_ms(lambda: conv.backward(x, Y, s, senders, row_ptr, gout, receivers=receivers,
                                             sender_row_ptr=srp, sender_perm=sperm), reps, stream)
        assert conv.check(), "backward reported a bad index"
        # each kernel alone: grad_Y and grad_s (receiver order), grad_x (sender order)
        ms_edges = _event_ms(lambda: conv.backward(x, Y, s, senders, row_ptr, gout, need_x=False),
                             reps, stream)
        ms_nodes = _event_ms(lambda: conv.backward(x, Y, s, senders, row_ptr, gout, receivers=receivers,
                                                   sender_row_ptr=srp, sender_perm=sperm,
                                                   need_edges=False), reps, stream)
        b = 2 if spec.dtype == "f16" else 4
        nnz = sum(int((np.abs(conv.cg(p)) > 1e-12).sum()) for p in range(conv.num_paths))
        mix = sum(2 * q.l3 + 1 for q in conv.paths)
        # edges kernel reads Y, s, senders, x rows, grad_out rows; writes grad_Y and grad_s (f32);
        # nodes kernel reads Y, s, receivers, perm, grad_out rows; writes grad_x
        nbytes = (2 * E * (conv.ny + conv.num_paths * conv.C) * b + 12 * E
                  + E * (conv.ny + conv.num_paths * conv.C) * 4
                  + N * (conv.nx * conv.C * b + 2 * 4 * conv.nout * conv.C + 4 * conv.nx * conv.C))
        flops = 2 * E * conv.C * (4 * nnz + mix)
        res["backward"] = {
            "kernels": "e3conv_bwd_edges + e3conv_bwd_nodes", "ms": ms, "edges_ms": ms_edges,
            "nodes_ms": ms_nodes, "edges_per_s": E / (ms / 1e3),
            "algorithmic_bytes": nbytes, "hbm_gbs": nbytes / (ms / 1e3) / 1e9,
            "hbm_frac": nbytes / (ms / 1e3) / 1e9 / pk["hbm_gbs"],
            "fp32_flops": flops, "fp32_tflops": flops / (ms / 1e3) / 1e12,
            "fp32_frac": flops / (ms / 1e3) / 1e12 / pk["fp32_tflops"],
            "note": "definition FLOPs: grad_s and grad_Y (3 per CG nonzero and channel), grad_x (1), "
                    "the s-scaling (one per output component); float32 accumulation"}
        del gout, srp, sperm
    irreps = "+".join(f"{conv.C}x{l}{'e' if p > 0 else 'o'}" for l, p, _ in conv.outputs)
    if conv.C in (32, 64, 128):
        lin = e3.IrrepsLinear(irreps, irreps, 1.0)
        rng = np.random.default_rng(3)
        lin.set_weights([rng.normal(size=(conv.C, conv.C)).astype(np.float32)
                         for _ in range(lin.num_weight_blocks)])
        yl = torch.empty_like(out)
        flat = out.view(N, -1)
        lin(flat, out=yl.view(N, -1))
        torch.cuda.synchronize()
        ms = _event_ms(lambda: lin(flat, out=yl.view(N, -1)), reps, stream)
        kernel = "k_linear_tma" if lin.uses_tma else "k_linear"
        lin.set_tma(False)                 # the row-per-thread kernel, for comparison
        ms_rows = _event_ms(lambda: lin(flat, out=yl.view(N, -1)), reps, stream)
        assert lin.check()
        nbytes = 2 * out.numel() * 4
        flops = 3 * 2 * N * conv.nout * conv.C * conv.C
        res["irreps_linear"] = {
            "kernel": kernel, "irreps": irreps, "ms": ms, "row_per_thread_kernel_ms": ms_rows,
            "algorithmic_bytes": nbytes,
            "hbm_gbs": nbytes / (ms / 1e3) / 1e9, "hbm_frac": nbytes / (ms / 1e3) / 1e9 / pk["hbm_gbs"],
            "tensor_flops": flops, "tensor_tflops": flops / (ms / 1e3) / 1e12,
            "note": "x read and y written once (HBM bound); tensor FLOPs count the three "
                    "float16 hi/lo MMAs per product"}
        del lin, yl
    if not args.radial and g.vec is not None and conv.C >= 32:
        # the radial MLP at this workload's size and dtype: seeded weights (8 bases, 64 x 2
        # hidden, P*C outputs), the scalars written over this workload's s (last use of it)
        rng = np.random.default_rng(11)
        sizes = [8, 64, 64, conv.num_paths * conv.C]
        ws = [(rng.normal(size=(a_, b_)) / np.sqrt(a_)).astype(np.float32)
              for a_, b_ in zip(sizes[:-1], sizes[1:])]
        v = np.zeros((E, 4), np.float32)
        v[:, :3] = g.vec
        r_max = float(np.linalg.norm(g.vec, axis=1).max()) * 1.01
        conv.set_radial_mlp(r_max, ws)
        v4 = torch.from_numpy(v).to(out.device)
        conv.radial_scalars(v4, out=s)
        torch.cuda.synchronize()
        ms = _event_ms(lambda: conv.radial_scalars(v4, out=s), reps, stream)
        assert conv.check()
        nbytes = s.numel() * s.element_size()
        flops = 3 * 2 * E * 64 * (64 + conv.num_paths * conv.C)
        res["radial_mlp"] = {
            "kernel": "k_radial", "outputs": conv.num_paths * conv.C, "dtype": spec.dtype, "ms": ms,
            "scalars_bytes_written": nbytes, "write_gbs": nbytes / (ms / 1e3) / 1e9,
            "hbm_frac": nbytes / (ms / 1e3) / 1e9 / pk["hbm_gbs"],
            "tensor_flops": flops, "tensor_tflops": flops / (ms / 1e3) / 1e12,
            "note": "edge scalars from the edge vectors (bessel x cutoff, SiLU MLP) at this "
                    "workload's size, seeded weights; supplementary"}
        del v4
    return res


def time_tensor_core_variant(args, spec, g, conv, x, Y, s, senders, row_ptr, out, stream):
    """Supplementary: the opt-in tensor-core forward on the same resident inputs, after the
    timed region (CUDA events, inputs larger than L2); None where the variant does not apply."""
    import torch

    import equivariant_graph_message_b200 as e3
    tc = e3.Conv(spec.irreps_node, spec.irreps_sh, spec.irreps_out, g.avg_num_neighbors,
                 dtype=spec.dtype)
    tc.set_tensor_cores(1)
    if not tc.kernel_info()["tensor_cores"]:
        return None
    N, E = g.num_nodes, g.num_edges
    out_tc = torch.empty_like(out)
    sh = e3._stream_handle(stream)
    ptrs = [e3._ptr(t) for t in (x, Y, s, senders, row_ptr)]
    for _ in range(max(3, args.warmup)):
        tc.forward_raw(*ptrs, N, e3._ptr(out_tc), sh)
    reps = max(5, min(args.steps, 20))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in ev:
        a.record(stream)
        tc.forward_raw(*ptrs, N, e3._ptr(out_tc), sh)
        b.record(stream)
    torch.cuda.synchronize()
    assert tc.check(), "tensor-core variant reported a bad index or a wait timeout"
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    diff = ((out_tc - out).abs().max() / out.abs().max().clamp_min(1e-30)).item()
    return {"forward_ms": ms, "edges_per_s": E / (ms / 1000.0), "launches": reps,
            "max_abs_diff_vs_default_over_max_abs": diff, "kernel": tc.kernel_info(),
            "note": "opt-in tcgen05/TMA/tensor-memory forward; not the headline (see roofline)"}


def run_e2e(args, tensors, out, device_step, edges, world, dev):
    """The same step through the public API, with this step's inputs copied from pinned host
    memory and its result copied back, every step, inside the timed region."""
    import torch
    import torch.distributed as dist
    h2d = sum(t.numel() * t.element_size() for t in tensors)
    d2h = out.numel() * out.element_size()
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = 0
    ok = torch.tensor([1 if avail > 1.3 * (h2d + d2h) + (8 << 30) else 0], device=dev)
    if world > 1:
        dist.all_reduce(ok, op=dist.ReduceOp.MIN)
    if not ok.item():
        return {"value": None, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "skipped": f"host memory available {avail / 2**30:.0f} GiB < needed pinned "
                           f"{(h2d + d2h) / 2**30:.0f} GiB"}
    host = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in tensors]
    for h, t in zip(host, tensors):
        h.copy_(t)
    out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    steps = max(1, min(args.steps, 5))

    def step():
        for h, t in zip(host, tensors):
            t.copy_(h, non_blocking=True)
        device_step()
        out_h.copy_(out, non_blocking=True)

    step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    a.record()
    for _ in range(steps):
        step()
    b.record()
    torch.cuda.synchronize()
    (ms,), total = reduce_over_ranks([a.elapsed_time(b) / steps], edges, world, dev)
    del host, out_h
    return {"value": total / (ms / 1000.0), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": ms}


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
