"""Benchmark of the deformable sampling core on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-rows] [--no-cpu]

One step = one dcn_core_forward over one batch of the DCNv4 YOLO-P4 workload
(B=8 per GPU, 40x40, G=16 x C=32, 3x3, fp16 storage, fp32 accumulation, raw
modulation).  Inputs rotate over enough resident copies to exceed 4x the L2
size, so every step reads HBM.  The K timed steps are replayed from CUDA
graphs and bracketed by a barrier and synchronisations; the time is the max
over ranks of CUDA-event time on the launching stream.  Rank 0 prints one
JSON line.  Under torchrun each rank runs its own batch (weak scaling, no
collective on the data path; the only collectives are the barrier and the
max-over-ranks of the time).

--impl reference times the fp64 CPU oracle (the reference this build is
checked against) on the host cores, on rank 0, on a bounded sample of the
same workload; other ranks exit without work.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic_inputs as si  # noqa: E402

METRIC = "deform-sample fwd Gsamples/s & achieved HBM GB/s (% of peak), DCNv4 P4 shape"
WORKLOAD = ("DCNv4 core forward, YOLO-P4 shape: B=8 per GPU, H=W=40, 512 ch as G=16 x C=32, 3x3, "
            "stride 1, pad 1, dil 1, raw modulation, fp16 storage / fp32 accumulate; x~N(0,1), "
            "offsets~N(0,3), mask~N(0,1)")
FALLBACK_HBM_GBS = 6650.0
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
# Sources of the timed forward kernel: the recorded DRAM traffic is used only
# while these are unchanged.
KERNEL_SOURCES = [os.path.join(ROOT, "deformable_convolution_sampling_dcn_b200", "csrc", f)
                  for f in ("dcn_forward_plane.cu", "dcn_forward_staged.cuh", "dcn_forward_staged_f16.cu",
                            "dcn_tma.cuh", "dcn_common.cuh", "dcn_device.h")]


def kernel_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """Polls SM clock and throttle reasons through NVML while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clocks_setting": 0x100,
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML unavailable: report no clocks
            self.ok = False
        self._period = period_s
        self._t = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": len(self.samples)}
        names = [n for n, bit in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------- our arm
def build_sets(shape, seed, dev, l2_bytes):
    inp = si.core_inputs(shape, seed, offset_std=3.0)
    x, off, m = (inp[k].to(dev) for k in ("x", "offset", "mask"))
    out_shape = (shape.B, shape.Ho, shape.Wo, shape.G * shape.C)
    footprint = shape.compulsory_bytes()
    R = max(2, math.ceil(4 * l2_bytes / footprint))
    sets = []
    for _ in range(R):
        sets.append((x.clone(), off.clone(), m.clone(), torch.empty(out_shape, dtype=x.dtype, device=dev)))
    return inp, sets, R, footprint


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest `value` over all ranks (the job is as slow as its slowest
    rank); identity on one process."""
    if world <= 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def capture(fn_list, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for fn in fn_list:
            fn()
    return g


def time_steps(make_call, sets, K, W, stream, barrier, world):
    """Replay K calls (rotating over `sets`) from CUDA graphs; returns ms (max over ranks)."""
    R = len(sets)
    calls = [make_call(s) for s in sets]
    for c in calls:  # eager warm-up of each set (also validates the launch)
        c()
    torch.cuda.synchronize()
    g_full = capture(calls, stream)
    rem = K % R
    g_rem = capture(calls[:rem], stream) if rem else None
    full = K // R
    wfull = max(1, math.ceil(W / R))
    for _ in range(wfull):
        g_full.replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(full):
            g_full.replay()
        if g_rem is not None:
            g_rem.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), world, "cuda")
    del g_full, g_rem
    return ms


def run_ours(args, world, rank, local):
    import deformable_convolution_sampling_dcn_b200 as dcn

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)

        def barrier():
            torch.distributed.barrier()
    else:
        def barrier():
            pass

    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))
    shape = si.DCNV4_P4
    inp, sets, R, footprint = build_sets(shape, si.SEEDS["dcnv4_p4"] + 1000 * rank, dev, l2)
    stream = torch.cuda.Stream(dev)

    def make_call(s):
        x, off, m, out = s
        return lambda: dcn.dcn_core_forward(x, off, m, group=shape.G, out=out)

    K, W = args.steps, args.warmup
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    with sampler:
        ms = time_steps(make_call, sets, K, W, stream, barrier, world)
    clocks = sampler.summary()
    step_s = ms / 1e3 / K
    samples_all = shape.samples * world
    value = samples_all / step_s / 1e9  # Gsamples/s, whole job
    bytes_per_launch = shape.compulsory_bytes()
    achieved = bytes_per_launch / step_s / 1e9
    peak, peak_kind = peaks()
    traffic = None
    issue = None
    if os.path.exists(TRAFFIC_FILE):
        with open(TRAFFIC_FILE) as f:
            tr = json.load(f)
        ent = tr.get("dcnv4_p4_forward")
        if ent and ent.get("kernel_hash") == kernel_hash():
            traffic = ent["bytes_per_launch"]  # DRAM reads + the launch's L2 writes (its output)
            insts = ent.get("warp_instructions_per_launch")
            if insts and clocks.get("sm_mhz"):
                # the ceiling that binds this gather: one warp instruction per
                # scheduler per clock (148 SMs x 4 schedulers at the sampled clock)
                ceil_t = torch.cuda.get_device_properties(dev).multi_processor_count * 4 * clocks["sm_mhz"] * 1e6
                ach_t = insts / step_s
                issue = {"warp_instructions_per_launch": insts, "achieved": round(ach_t / 1e12, 4),
                         "ceiling": round(ceil_t / 1e12, 4), "unit": "T warp-instructions/s",
                         "frac": round(ach_t / ceil_t, 4)}

    # end to end through the public API with host buffers (pinned), copies timed
    e2e = measure_e2e(dcn, shape, inp, dev, stream, min(K, args.e2e_steps), barrier, world)

    rows = measure_rows(dcn, dev, stream, l2, barrier, world) if (args.rows and world == 1) else None

    cpu = None
    if rank == 0 and world == 1 and args.cpu:
        cpu = cpu_baseline(args.cpu_seconds)

    if world > 1:
        torch.distributed.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "Gsamples/s", "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": round(ms / K, 6), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B_per_gpu": shape.B, "global_batch": shape.B * world,
                       "H": shape.H, "W": shape.W, "G": shape.G, "C": shape.C, "kernel": [3, 3],
                       "storage": "f16", "accumulate": "f32",
                       "samples_per_step_per_gpu": shape.samples,
                       "l2": f"{R} rotating resident input sets ({R * footprint / 1e6:.0f} MB) > 4x L2 "
                             f"({l2 / 1e6:.0f} MB); no flush",
                       "timing": "CUDA graphs of the rotating launches, CUDA events on the launching stream",
                       "parallelism": f"batch shard x{world}, no data-path collective" if world > 1 else "1 GPU"},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic,
                         "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                         else "fallback 6.65 TB/s",
                         "algorithmic_bytes_per_launch": bytes_per_launch,
                         "kernel": "dcn_core_forward (one launch per step)", "issue": issue},
            "clocks": clocks,
            "e2e": e2e,
            "gpu_launches": K,
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        if rows is not None:
            line["rows"] = rows
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def measure_e2e(dcn, shape, inp, dev, stream, E, barrier, world):
    """Same metric through dcn_core_forward with host buffers: every step copies
    its inputs from pinned host memory, calls the forward and copies the
    output back to pinned host memory, all inside the timed region.  Steps are
    pipelined over two buffer slots and three streams (host-to-device copies,
    compute, device-to-host copies), so one step's copies overlap the
    neighbouring steps' work; events order every reuse of a slot."""
    # x, offset and mask live back to back in one pinned host buffer (256-byte
    # aligned views), so each step uploads them with one copy
    srcs = [inp[k] for k in ("x", "offset", "mask")]
    offs, total = [], 0
    for t in srcs:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    hbuf = torch.empty(total, dtype=torch.uint8).pin_memory()

    def views(buf):
        return [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for o, t in zip(offs, srcs)]

    hx, hoff, hm = views(hbuf)
    for h, t in zip((hx, hoff, hm), srcs):
        h.copy_(t)
    out_shape = (shape.B, shape.Ho, shape.Wo, shape.G * shape.C)
    slots = 2
    hout = [torch.empty(out_shape, dtype=hx.dtype).pin_memory() for _ in range(slots)]
    dbufs = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(slots)]
    dins = [views(b) for b in dbufs]
    douts = [torch.empty(out_shape, dtype=hx.dtype, device=dev) for _ in range(slots)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    copied = [ev() for _ in range(slots)]     # inputs of the slot are on the device
    computed = [ev() for _ in range(slots)]   # the slot's forward is done (inputs free, output ready)
    returned = [ev() for _ in range(slots)]   # the slot's output is back on the host (output free)
    used = [False] * slots
    E = max(1, E)

    def step(i):
        k = i % slots
        dx, doff, dm = dins[k]
        with torch.cuda.stream(s_in):
            if used[k]:
                s_in.wait_event(computed[k])
            dbufs[k].copy_(hbuf, non_blocking=True)  # x, offset and mask in one upload
            copied[k].record(s_in)
        with torch.cuda.stream(stream):
            stream.wait_event(copied[k])
            if used[k]:
                stream.wait_event(returned[k])
            dcn.dcn_core_forward(dx, doff, dm, group=shape.G, out=douts[k])
            computed[k].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[k])
            hout[k].copy_(douts[k], non_blocking=True)
            returned[k].record(s_out)
        used[k] = True

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(E):
        step(3 + i)
    # the timed region ends when the last output is on the host and every stream is idle
    for st_ in (s_in, stream):
        s_out.wait_stream(st_)
    e1.record(s_out)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), world, "cuda")
    h2d = total  # the one upload per step (x, offset, mask and at most 3 x 255 bytes of alignment)
    d2h = hout[0].numel() * hout[0].element_size()
    return {"value": round(shape.samples * world / (ms / 1e3 / E) / 1e9, 3), "unit": "Gsamples/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": E,
            "ms_per_step": round(ms / E, 4),
            "pipeline": "2 buffer slots; one H2D copy of x+offset+mask, compute and D2H on three streams"}


def measure_rows(dcn, dev, stream, l2, barrier, world, steps=280):
    """Per-workload device times of every hot-path row (context for the headline)."""
    out = {}

    def core_fwd(name):
        shape, inp = si.workload_core(name)
        x, off, m = (inp[k].to(dev) for k in ("x", "offset", "mask"))
        R = min(64, max(2, math.ceil(4 * l2 / shape.compulsory_bytes())))
        sets = [(x.clone(), off.clone(), m.clone(),
                 torch.empty((shape.B, shape.Ho, shape.Wo, shape.G * shape.C), dtype=x.dtype, device=dev))
                for _ in range(R)]
        cfg = dict(group=shape.G, kernel=(shape.kh, shape.kw), stride=(shape.stride_h, shape.stride_w),
                   pad=(shape.pad_h, shape.pad_w), dil=(shape.dil_h, shape.dil_w), softmax=shape.softmax)

        def mk(s):
            return lambda: dcn.dcn_core_forward(s[0], s[1], s[2], out=s[3], **cfg)

        ms = time_steps(mk, sets, steps, 3 * R, stream, barrier, world) / steps
        out[name] = {"us": round(ms * 1e3, 2), "Gsamples_s": round(shape.samples / ms / 1e6, 2),
                     "GB_s": round(shape.compulsory_bytes() / ms / 1e6, 1), "R": R}
        del sets

    for n in ("dcnv3_tiny", "dcnv3_p3", "dcnv3_p3_dil2"):
        core_fwd(n)

    # DCNv3 softmax-mode backward, bf16, at the P3 shape
    shape, inp = si.workload_core("dcnv3_p3_bwd")
    t = [inp[k].to(dev) for k in ("x", "offset", "mask", "grad_out")]
    R = max(2, math.ceil(4 * l2 / shape.compulsory_bytes(backward=True)))
    sets = [[u.clone() for u in t] + [torch.empty_like(t[0]), torch.empty_like(t[1]), torch.empty_like(t[2])]
            for _ in range(R)]

    def mkb3(s):
        return lambda: dcn.dcn_core_backward(s[0], s[1], s[2], s[3], group=shape.G, softmax=True, grad_x=s[4],
                                             grad_offset=s[5], grad_mask=s[6])

    ms = time_steps(mkb3, sets, steps, 3 * R, stream, barrier, world) / steps
    out["dcnv3_p3_bwd_softmax_bf16"] = {"us": round(ms * 1e3, 2), "Gsamples_s": round(shape.samples / ms / 1e6, 2),
                                        "R": R}
    del sets

    # DCNv4 backward at the P4 shape, fp32
    shape, inp = si.workload_core("dcnv4_p4_bwd")
    t = [inp[k].to(dev) for k in ("x", "offset", "mask", "grad_out")]
    R = max(2, math.ceil(4 * l2 / shape.compulsory_bytes(backward=True)))
    sets = [[u.clone() for u in t] + [torch.empty_like(t[0]), torch.empty_like(t[1]), torch.empty_like(t[2])]
            for _ in range(R)]

    def mkb(s):
        return lambda: dcn.dcn_core_backward(s[0], s[1], s[2], s[3], group=shape.G, grad_x=s[4],
                                             grad_offset=s[5], grad_mask=s[6])

    ms = time_steps(mkb, sets, steps, 3 * R, stream, barrier, world) / steps
    out["dcnv4_p4_bwd"] = {"us": round(ms * 1e3, 2), "Gsamples_s": round(shape.samples / ms / 1e6, 2),
                           "GB_s": round(shape.compulsory_bytes(backward=True) / ms / 1e6, 1), "R": R}
    del sets

    # Sparse4D aggregation forward
    a = si.SPARSE4D
    inp = si.agg_inputs(a, si.SEEDS["sparse4d"])
    keys = ("feat", "spatial_shape", "scale_start_index", "sampling_location", "weights")
    t = [inp[k].to(dev) for k in keys]
    R = max(2, math.ceil(4 * l2 / a.compulsory_bytes()))
    sets = [[u.clone() for u in t] + [torch.empty((a.B, a.num_anchors, a.G * a.C), device=dev)] for _ in range(R)]

    def mka(s):
        return lambda: dcn.deform_agg_forward(*s[:5], out=s[5])

    ms = time_steps(mka, sets, steps, 3 * R, stream, barrier, world) / steps
    out["sparse4d"] = {"us": round(ms * 1e3, 2), "Gsamples_s": round(a.samples / ms / 1e6, 2),
                       "GB_s": round(a.compulsory_bytes() / ms / 1e6, 1), "R": R}
    del sets

    # Sparse4D aggregation backward
    inp = si.agg_inputs(a, si.SEEDS["sparse4d"], with_grad_out=True)
    t = [inp[k].to(dev) for k in keys + ("grad_out",)]
    R = max(2, math.ceil(4 * l2 / (2 * a.compulsory_bytes())))
    sets = [[u.clone() for u in t] + [torch.empty_like(t[0]), torch.empty_like(t[3]), torch.empty_like(t[4])]
            for _ in range(R)]

    def mkab(s):
        return lambda: dcn.deform_agg_backward(*s[:6], grad_feat=s[6], grad_loc=s[7], grad_weights=s[8])

    ms = time_steps(mkab, sets, steps, 3 * R, stream, barrier, world) / steps
    out["sparse4d_bwd"] = {"us": round(ms * 1e3, 2), "Gsamples_s": round(a.samples / ms / 1e6, 2), "R": R}
    del sets

    # deformable RoI pooling
    rs = si.ROI_POOL
    inp = si.roi_inputs(rs, si.SEEDS["roi_pool"])
    t = [inp[k].to(dev) for k in ("x", "rois", "offset")]
    R = max(2, math.ceil(4 * l2 / rs.compulsory_bytes()))
    sets = [[u.clone() for u in t] + [torch.empty((rs.N, rs.PH, rs.PW, rs.C), device=dev)] for _ in range(R)]

    def mkr(s):
        return lambda: dcn.deform_roi_pool_forward(s[0], s[1], s[2], pooled=(rs.PH, rs.PW), sampling=rs.S,
                                                   spatial_scale=rs.spatial_scale, gamma=rs.gamma, out=s[3])

    ms = time_steps(mkr, sets, steps, 3 * R, stream, barrier, world) / steps
    out["roi_pool"] = {"us": round(ms * 1e3, 2), "Gsamples_s": round(rs.samples / ms / 1e6, 2),
                       "GB_s": round(rs.compulsory_bytes() / ms / 1e6, 1), "R": R}
    del sets

    # DCNv4 P4 core followed by its 512 -> 512 projection (tensor cores): the
    # workspace route (core kernel into a workspace, then the library's GEMM),
    # the one fused kernel, and for context the core kernel followed by a
    # cuBLAS GEMM through torch on the stored core output.
    shape, inp = si.workload_proj()
    t = [inp[k].to(dev) for k in ("x", "offset", "mask", "weight", "bias")]
    cout = t[3].shape[0]
    pbytes = shape.compulsory_bytes() + (t[3].numel() + t[4].numel()) * 2 + \
        shape.B * shape.Ho * shape.Wo * (cout - shape.G * shape.C) * 2
    R = max(2, math.ceil(4 * l2 / pbytes))
    sets = [[u.clone() for u in t] + [torch.empty((shape.B, shape.Ho, shape.Wo, cout), dtype=t[0].dtype, device=dev),
                                      torch.empty((shape.B, shape.Ho, shape.Wo, shape.G * shape.C),
                                                  dtype=t[0].dtype, device=dev)] for _ in range(R)]

    def mkp(s):  # workspace route; the core-output buffer is its workspace
        return lambda: dcn.dcn_core_forward_proj(s[0], s[1], s[2], s[3], s[4], group=shape.G, out=s[5],
                                                 workspace=s[6])

    ms = time_steps(mkp, sets, steps, 3 * R, stream, barrier, world) / steps

    def mkf(s):
        return lambda: dcn.dcn_core_forward_proj(s[0], s[1], s[2], s[3], s[4], group=shape.G, out=s[5], fused=True)

    ms_f = time_steps(mkf, sets, steps, 3 * R, stream, barrier, world) / steps

    def mku(s):
        def call():
            dcn.dcn_core_forward(s[0], s[1], s[2], group=shape.G, out=s[6])
            torch.addmm(s[4], s[6].view(-1, shape.G * shape.C), s[3].t(), out=s[5].view(-1, cout))
        return call

    ms_u = time_steps(mku, sets, steps, 3 * R, stream, barrier, world) / steps
    flops = 2.0 * shape.B * shape.Ho * shape.Wo * cout * shape.G * shape.C
    out["dcnv4_p4_proj"] = {"us": round(ms * 1e3, 2), "Gsamples_s": round(shape.samples / ms / 1e6, 2),
                            "GB_s": round(pbytes / ms / 1e6, 1), "gemm_TFLOP_s": round(flops / ms / 1e9, 1),
                            "route": "workspace (core kernel + tcgen05 GEMM)", "fused_one_kernel_us":
                            round(ms_f * 1e3, 2), "unfused_core_then_cublas_us": round(ms_u * 1e3, 2),
                            "Cout": cout, "R": R}
    del sets

    # modulated deformable convolution (a dense weight per kernel point) at the
    # P4 shape, 512 -> 512, fp16
    shape, inp = workload_deform_conv()
    t = [inp[k].to(dev) for k in ("x", "offset", "mask", "weight", "bias")]
    cout = t[3].shape[0]
    R = max(2, math.ceil(4 * l2 / pbytes))
    sets = [[u.clone() for u in t] + [torch.empty((shape.B, shape.Ho, shape.Wo, cout), dtype=t[0].dtype, device=dev)]
            for _ in range(R)]

    def mkd(s):
        return lambda: dcn.dcn_deform_conv_forward(s[0], s[1], s[2], s[3], s[4], group=shape.G, out=s[5])

    ms = time_steps(mkd, sets, steps, 3 * R, stream, barrier, world) / steps
    flops = 2.0 * shape.B * shape.Ho * shape.Wo * cout * shape.K * shape.G * shape.C
    out["dcnv2_p4_deform_conv"] = {"us": round(ms * 1e3, 2), "Gsamples_s": round(shape.samples / ms / 1e6, 2),
                                   "gemm_TFLOP_s": round(flops / ms / 1e9, 1), "Cout": cout, "R": R}
    return out


def workload_deform_conv():
    """DCNv4-P4 inputs with a 512 -> 512 dense weight per kernel point."""
    shape, inp = si.workload_core("dcnv4_p4")
    inp.update(si.deform_conv_weights(shape.K, shape.G * shape.C, 512, shape.dtype, 9))
    return shape, inp


# ----------------------------------------------------------------------------- CPU oracle
def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(seconds: float):
    """The fp64 oracle as it stands on all host cores: whole DCNv4-P4 batches,
    repeated until `seconds` of wall time have passed (at least once)."""
    import oracle

    n = oracle.set_threads(cpu_threads())
    shape, inp = si.workload_core("dcnv4_p4")
    x, off, m = (inp[k].double().numpy() for k in ("x", "offset", "mask"))
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.dcn_forward(x, off, m, G=shape.G)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    # the same oracle on one core, for a shorter while
    oracle.set_threads(1)
    reps1, t1 = 0, time.perf_counter()
    while True:
        oracle.dcn_forward(x, off, m, G=shape.G)
        reps1 += 1
        el1 = time.perf_counter() - t1
        if el1 >= seconds / 5:
            break
    oracle.set_threads(n)
    return {"value": round(shape.samples * reps / el / 1e9, 5), "unit": "Gsamples/s", "cores": n,
            "kind": "oracle",
            "sample": f"{reps} whole DCNv4-P4 batches (B=8, {shape.samples} samples each) in {el:.1f} s, "
                      f"fp64 C loops, OpenMP over (b, output row)",
            "single_core": {"value": round(shape.samples * reps1 / el1 / 1e9, 5), "unit": "Gsamples/s",
                            "sample": f"{reps1} whole batches in {el1:.1f} s on 1 thread"}}


def run_reference(args, world, rank):
    """The oracle as it stands, on the host cores, one bounded sample per step.

    Groups are independent, so a step runs the oracle on `ng` whole groups of
    one image (every output pixel and tap of those groups), sized so that the
    W + K steps take about a minute."""
    if rank != 0:
        return
    import numpy as np

    import oracle

    n = oracle.set_threads(cpu_threads())
    shape, inp = si.workload_core("dcnv4_p4")
    x, off, m = (inp[k].double().numpy() for k in ("x", "offset", "mask"))
    C, G = shape.C, shape.G

    def group_slice(b, g0, ng):
        return (np.ascontiguousarray(x[b:b + 1, :, :, g0 * C:(g0 + ng) * C]),
                np.ascontiguousarray(off[b:b + 1, :, :, g0:g0 + ng]),
                np.ascontiguousarray(m[b:b + 1, :, :, g0:g0 + ng]))

    t0 = time.perf_counter()
    xs, os_, ms_ = group_slice(0, 0, 1)
    for _ in range(3):
        oracle.dcn_forward(xs, os_, ms_, G=1)
    per_group = (time.perf_counter() - t0) / 3
    budget = 60.0 / max(1, args.steps + args.warmup)
    ng = int(max(1, min(G, budget / max(per_group, 1e-9))))
    slices = [group_slice(b, g0, ng) for b in range(shape.B) for g0 in range(0, G - ng + 1, ng)]

    def step(i):
        xs, os_, ms_ = slices[i % len(slices)]
        oracle.dcn_forward(xs, os_, ms_, G=ng)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    el = time.perf_counter() - t0
    per_step_samples = shape.Ho * shape.Wo * ng * shape.K
    v = per_step_samples * args.steps / el / 1e9
    sample = (f"each step: {ng} of {G} groups of one DCNv4-P4 image, all {shape.Ho}x{shape.Wo} pixels and "
              f"{shape.K} taps ({per_step_samples} samples); fp64 C oracle, OpenMP")
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": "Gsamples/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B_per_gpu": shape.B, "global_batch": shape.B,
                       "parallelism": "host cores"},
            "cpu_baseline": {"value": round(v, 6), "unit": "Gsamples/s", "cores": n, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(v, 6), "unit": "Gsamples/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


CASES = ("dcnv4_p4", "dcnv3_p3", "dcnv3_p3_dil2", "dcnv4_p4_bwd", "sparse4d", "sparse4d_bwd", "roi_pool",
         "dcnv4_p4_proj", "dcnv2_p4_deform_conv")


def run_case(name: str, calls: int) -> None:
    """Call one workload's entry point `calls` times on cuda:0, untimed (for
    profilers: `ncu ... python bench.py --case NAME --steps 2`)."""
    import deformable_convolution_sampling_dcn_b200 as dcn

    dev = torch.device("cuda:0")
    if name in ("dcnv4_p4", "dcnv3_p3", "dcnv3_p3_dil2"):
        shape, inp = si.workload_core(name)
        t = [inp[k].to(dev) for k in ("x", "offset", "mask")]
        cfg = dict(group=shape.G, kernel=(shape.kh, shape.kw), stride=(shape.stride_h, shape.stride_w),
                   pad=(shape.pad_h, shape.pad_w), dil=(shape.dil_h, shape.dil_w), softmax=shape.softmax)
        call = lambda: dcn.dcn_core_forward(*t, **cfg)
    elif name == "dcnv4_p4_bwd":
        shape, inp = si.workload_core(name)
        t = [inp[k].to(dev) for k in ("x", "offset", "mask", "grad_out")]
        call = lambda: dcn.dcn_core_backward(*t, group=shape.G)
    elif name in ("sparse4d", "sparse4d_bwd"):
        bwd = name == "sparse4d_bwd"
        inp = si.agg_inputs(si.SPARSE4D, si.SEEDS["sparse4d"], with_grad_out=bwd)
        keys = ("feat", "spatial_shape", "scale_start_index", "sampling_location", "weights")
        t = [inp[k].to(dev) for k in keys + (("grad_out",) if bwd else ())]
        call = (lambda: dcn.deform_agg_backward(*t)) if bwd else (lambda: dcn.deform_agg_forward(*t))
    elif name == "roi_pool":
        rs = si.ROI_POOL
        inp = si.roi_inputs(rs, si.SEEDS["roi_pool"])
        t = [inp[k].to(dev) for k in ("x", "rois", "offset")]
        call = lambda: dcn.deform_roi_pool_forward(*t, pooled=(rs.PH, rs.PW), sampling=rs.S,
                                                   spatial_scale=rs.spatial_scale, gamma=rs.gamma)
    elif name == "dcnv4_p4_proj":
        shape, inp = si.workload_proj()
        t = [inp[k].to(dev) for k in ("x", "offset", "mask", "weight", "bias")]
        call = lambda: dcn.dcn_core_forward_proj(*t, group=shape.G)
    else:
        shape, inp = workload_deform_conv()
        t = [inp[k].to(dev) for k in ("x", "offset", "mask", "weight", "bias")]
        call = lambda: dcn.dcn_deform_conv_forward(*t, group=shape.G)
    for _ in range(calls):
        call()
    torch.cuda.synchronize()
    err = dcn._binding.take_device_error()
    if err:
        raise SystemExit(f"device error word {err}")
    print(f"ok {name} x{calls}")


def run_ceilings(reps_scale: float) -> None:
    """Measure the on-chip rates that bound the sampling kernels (dcn_probe_rate:
    one CTA per SM, SM-clock cycles) and print them, per SM per clock, with the
    lower bound each implies for the DCNv4 P4 forward (1,843,200 samples on all
    SMs at the maximum SM clock).  One JSON line at the end."""
    import deformable_convolution_sampling_dcn_b200 as dcn

    dev = torch.device("cuda:0")
    props = torch.cuda.get_device_properties(dev)
    sms = props.multi_processor_count
    clk_mhz = float(_nvml_max_sm_clock() or 1965.0)
    # repetitions giving a few milliseconds per probe
    reps = {"lds128": 20000, "chunk_f32_ffma2": 80000, "ffma": 20000, "ffma2": 20000, "chunk_f16_ffma": 80000,
            "chunk_f16_ffma2": 80000, "chunk_bf16_ffma2": 80000, "chunk_f16_mixed": 80000,
            "ldg128_l1": 20000, "gather4": 2000, "gather8": 2000, "gather8_ffma": 2000, "alu": 20000,
            "ldg256_l1": 20000, "atoms_f32": 20000}
    res = {}
    for name in dcn._binding.PROBES:
        n = max(1, int(reps[name] * reps_scale))
        dcn._binding.probe_rate(name, max(1, n // 10))  # warm-up
        best, unit = 0.0, ""
        for _ in range(3):
            r, unit = dcn._binding.probe_rate(name, n)
            best = max(best, r)
        res[name] = {"per_sm_per_clk": round(best, 4), "unit": unit}
    samples = si.DCNV4_P4.samples
    for name in ("gather4", "gather8", "gather8_ffma"):
        r = res[name]["per_sm_per_clk"]
        res[name]["p4_floor_us"] = round(samples / (sms * r * clk_mhz * 1e6) * 1e6, 2)
    # smem-data floor of any design that reads every corner row from shared memory or L1 once per tap
    lds = res["lds128"]["per_sm_per_clk"]
    tap_bytes = samples * 4 * si.DCNV4_P4.C * 2
    res["p4_corner_bytes_floor_us"] = round(tap_bytes / (sms * lds * clk_mhz * 1e6) * 1e6, 2)
    # Sparse4D forward: every (unit, scale) tap reads four fp32 rows of G*C channels through L1
    a = si.SPARSE4D
    agg_bytes = a.samples // a.G * 4 * a.G * a.C * 4
    for name in ("ldg128_l1", "ldg256_l1"):
        r = res[name]["per_sm_per_clk"]
        res[f"sparse4d_corner_bytes_floor_us_{name}"] = round(agg_bytes / (sms * r * clk_mhz * 1e6) * 1e6, 2)
    for name, v in res.items():
        if isinstance(v, dict):
            extra = f"   P4 floor {v['p4_floor_us']} us" if "p4_floor_us" in v else ""
            print(f"{name:18s} {v['per_sm_per_clk']:10.3f} {v['unit']}/SM/clk{extra}")
    print(json.dumps({"ceilings": res, "sms": sms, "sm_max_mhz": clk_mhz}))


def _nvml_max_sm_clock():
    try:
        import pynvml

        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByIndex(torch.cuda.current_device())
        return pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
    except Exception:
        return None


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=14000)
    ap.add_argument("--warmup", type=int, default=140)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--e2e-steps", type=int, default=100)
    ap.add_argument("--no-rows", dest="rows", action="store_false")
    ap.add_argument("--no-cpu", dest="cpu", action="store_false")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--case", choices=CASES, default=None,
                    help="only call this workload's entry point --steps times, untimed (for profilers)")
    ap.add_argument("--ceilings", action="store_true",
                    help="only measure the on-chip rate probes (shared loads, conversions, FMAs, gather loops)")
    ap.add_argument("--ceilings-scale", type=float, default=1.0, help="scale of the probes' repetition counts")
    args = ap.parse_args()
    if args.ceilings:
        run_ceilings(args.ceilings_scale)
        return
    if args.case is not None:
        run_case(args.case, args.steps)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if world != args.gpus and world != 1:
        print(f"warning: WORLD_SIZE={world} but --gpus {args.gpus}", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
