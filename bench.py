"""Decode-step benchmark of the block-quantised weight GEMV on B200.

One step = one decode token through the whole weight stream of the workload:
every layer's projections in model order (q|k|v, o, gate|up with the SwiGLU
epilogue, down), each a GEMV with dequantisation in the inner loop, launched as
one CUDA graph of dependent launches.  Default workload: 64-layer dense decoder,
hidden 5120, FFN 25600, Q4, batch 1 (16.4 GB of packed weights per step, far
above the L2, so no flush is needed).  Other workloads (--workload): the
16-layer hidden-2048 and 36-layer hidden-4096 decoders in every format and
batch, matrix-shape sweeps, routed experts, the batched-verification step on
the tensor cores, and decode attention over a Q8 KV cache.  Weights and
activations are synthetic (seeded N(0, 0.02) weights, N(0, 1) fp16
activations), generated and quantised on the device.

Prints ONE JSON line (rank 0).  `value` = algorithmic bytes (packed codes +
scales + x + y) of all ranks per second of the slowest rank; tokens/s-equiv =
B / step time.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl bq|reference]
                  [--workload NAME] [--engine graph|step]

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
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

from quantised_weight_gemv_b200 import synth  # noqa: E402

METRIC = "weight-stream HBM GB/s (decode step, algorithmic bytes)"
L2_FLUSH_BYTES = 256 << 20   # twice the B200's 126 MB L2
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "source": "fallback"}


def kernel_source_hash(unit: str = "stream_gemv.cu") -> str:
    """sha256 over the sources one kernel is built from: its translation unit
    under csrc/ plus every shared header (csrc/*.cuh, csrc/*.h, include/bq.h).
    A profile's traffic figure is only used while these are byte-identical to
    the profiled ones."""
    import glob
    import hashlib
    csrc = os.path.join(ROOT, "quantised_weight_gemv_b200", "csrc")
    files = [os.path.join(csrc, unit)] + sorted(glob.glob(os.path.join(csrc, "*.cuh")) +
                                                glob.glob(os.path.join(csrc, "*.h")))
    files.append(os.path.join(ROOT, "include", "bq.h"))
    h = hashlib.sha256()
    for p in files:
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode())
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic(workload: str, engine: str, unit: str = "stream_gemv.cu"):
    """DRAM bytes per launch (read + write) from a committed ncu summary under
    profiles/: a line `<!-- bench-traffic: workload=... engine=...
    bytes_per_launch=... source_sha256=... -->`, the hash being
    kernel_source_hash(unit) of the profiled kernel.  None when no summary
    matches the current sources."""
    import glob
    import re
    cur = kernel_source_hash(unit)
    for p in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        with open(p) as f:
            for line in f:
                m = re.search(r"bench-traffic:(.*?)-->", line)
                if not m:
                    continue
                kv = dict(t.split("=", 1) for t in m.group(1).split() if "=" in t)
                if (kv.get("workload") == workload and kv.get("engine") == engine
                        and kv.get("source_sha256") == cur):
                    return int(float(kv["bytes_per_launch"]))
    return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d.get("bf16_tflops", 0)) or None,
                "source": "measured"}
    except Exception:
        return dict(PEAKS_FALLBACK)


WORKLOADS = {
    synth.DENSE_H2048.name: synth.DENSE_H2048,
    synth.dense_h2048(2).name: synth.dense_h2048(2),
    synth.dense_h2048(3).name: synth.dense_h2048(3),
    synth.dense_h2048(5).name: synth.dense_h2048(5),
    synth.dense_h2048(6).name: synth.dense_h2048(6),
    synth.dense_h2048(8).name: synth.dense_h2048(8),
    synth.SINGLE_Q8.name: synth.SINGLE_Q8,
    synth.DENSE_H5120.name: synth.DENSE_H5120,
}
for _b in (1, 8):
    _w = synth.moe_h2048(_b)
    WORKLOADS[_w.name] = _w
for _w in (synth.attn_h5120(1, 4096), synth.attn_h5120(8, 4096), synth.attn_h5120(1, 32768),
           synth.attn_h5120(1, 32768, layers=4), synth.attn_h2048(8, 8192)):
    WORKLOADS[_w.name] = _w
for _f in (4, 8):
    for _b in (16, 32):
        for _w in (synth.verify_h4096(_f, _b),
                   synth.verify_sweep_workload(_f, 24576, 4096, _b),
                   synth.verify_sweep_workload(_f, 4096, 12288, _b)):
            WORKLOADS[_w.name] = _w
for _f in (2, 3, 4, 5, 6, 8):
    for _b in (1, 2, 4, 8):
        _w = synth.dense_h4096(_f, _b)
        WORKLOADS[_w.name] = _w
    for _n, _k in synth.SWEEP_SHAPES:
        for _b in (1, 8):
            for _w in (synth.sweep_workload(_f, _n, _k, _b), synth.single_workload(_f, _n, _k, _b)):
                WORKLOADS[_w.name] = _w


def fused_stages(wl: synth.DenseWorkload):
    """Per layer: list of (stage, [Mat...]) -- matrices sharing a stage share x
    and are stored as one row-concatenated matrix."""
    st = {}
    for m in wl.mats:
        st.setdefault(m.stage, []).append(m)
    return [(s, st[s]) for s in sorted(st)]


# ------------------------------------------------------------- clocks ----
class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled DURING a region.

    A thread polls NVML every 10 ms (read-only queries: nothing on the GPU is
    set), so even a timed region of a tenth of a second yields samples; where
    NVML cannot be loaded it falls back to `nvidia-smi -lms 200`."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, phys_index: int, pci_bus_id: str | None = None, period_s: float = 0.01):
        self.idx = phys_index
        self.pci = pci_bus_id
        self.period = period_s
        self.proc = None
        self.thread = None
        self.rows = []          # (time, sm MHz, max sm MHz, [4 reason flags])
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        if self.pci:
            try:
                return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(self.pci)
            except Exception:
                pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.idx)

    def start(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            bits = [nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
                    nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap]
            self.stop_flag = threading.Event()

            def poll():
                while not self.stop_flag.is_set():
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                        rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.rows.append((time.time(), float(sm), float(mx),
                                          ["Active" if rs & b else "Not Active" for b in bits]))
                    except Exception:
                        pass
                    self.stop_flag.wait(self.period)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            self.source = "nvml, 10 ms"
            return
        except Exception:
            self.thread = None
        try:
            fd, self.path = tempfile.mkstemp(prefix="bq_clocks_", suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-i", str(self.idx), "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi, 200 ms"
        except Exception:
            self.proc = None

    def _smi_rows(self):
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [s.strip() for s in line.split(",")]
                if len(p) < 10:
                    continue
                try:
                    ts = time.mktime(time.strptime(p[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                    ts += float("0." + p[0].split(".")[1]) if "." in p[0] else 0.0
                    rows.append((ts, float(p[2]), float(p[3]), p[6:10]))
                except Exception:
                    continue
        os.unlink(self.path)
        return rows

    def stop(self, t_begin, t_end):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            rows = list(self.rows)
        elif self.proc is not None:
            rows = self._smi_rows()
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"], "samples": 0}
        inside = [r for r in rows if t_begin <= r[0] <= t_end]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0,
                    "source": self.source}
        reasons = sorted({self.NAMES[i] for r in inside for i, v in enumerate(r[3]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                "samples": len(inside), "source": self.source}


def phys_gpu_index(local_rank: int) -> int:
    cvd = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [s for s in cvd.split(",") if s.strip()]
    if ids and all(s.strip().isdigit() for s in ids) and local_rank < len(ids):
        return int(ids[local_rank])
    return local_rank


# ------------------------------------------------------ device workload ----
class DenseStep:
    """All matrices of one decode step resident in HBM, plus x / y buffers.

    Each layer's feed-forward block is fused: its gate and up projections form
    one matrix in SwiGLU pair order whose epilogue writes h = silu(gate) * up
    (fp16), and the down projection reads that h -- so the down stage really
    depends on the stage before it.  Every other stage reads its own seeded
    activations."""

    def __init__(self, wl: synth.DenseWorkload, device, seed: int = 0, ffn: bool = True):
        import torch
        from quantised_weight_gemv_b200 import bq
        ffn = ffn and not wl.verify      # a verification step: every matrix has its own x
        self.wl, self.device, self.bq = wl, device, bq
        self.B = wl.B
        self.fmt = wl.fmt
        self.launches = []      # (qmat, x, y, label, stage, epilogue)
        self.bytes_alg = 0
        self.bytes_by_label = {}
        self._keep = []
        st = torch.zeros(1, dtype=torch.int32, device=device)
        ws_max = 0
        stages = fused_stages(wl)
        Kc = lambda K: {2: K // 4, 3: 3 * K // 8, 4: K // 2, 5: 5 * K // 8, 6: 3 * K // 4,
                        8: K}[wl.fmt]   # code bytes per row
        pending = []            # (layer, stage, mats, K, Ntot, codes, scales, x-or-None, out spec)
        for layer in range(wl.layers):
            h_shape = None
            for s, mats in stages:
                K = mats[0].K
                Ntot = sum(m.N for m in mats)
                ldS = bq.scales_ld(K)
                names = [m.name for m in mats]
                swiglu = ffn and names in (["gate", "up"], ["gateup"])
                codes = torch.empty((Ntot, Kc(K)), dtype=torch.uint8, device=device)
                scales = torch.empty((Ntot, ldS), dtype=torch.int16, device=device)
                if swiglu:
                    # gate rows and up rows, each quantised on its own, then
                    # interleaved 8 at a time (SwiGLU pair order)
                    F = Ntot // 2
                    parts = []
                    if names == ["gate", "up"]:
                        for m in mats:
                            parts.append(synth.weights_f32_torch(
                                synth.key(seed, wl.wid, layer, wl.mats.index(m), synth.KIND_W),
                                m.N, K, device))
                    else:
                        w = synth.weights_f32_torch(
                            synth.key(seed, wl.wid, layer, wl.mats.index(mats[0]), synth.KIND_W),
                            Ntot, K, device)
                        parts = [w[:F], w[F:]]
                    cv = codes.view(F // 8, 2, 8, Kc(K))
                    sv = scales.view(F // 8, 2, 8, ldS)
                    for half, w in enumerate(parts):
                        ct = torch.empty((F, Kc(K)), dtype=torch.uint8, device=device)
                        stt = torch.empty((F, ldS), dtype=torch.int16, device=device)
                        bq.quantize_dev(wl.fmt, w.contiguous(), ct, stt, st)
                        cv[:, half].copy_(ct.view(F // 8, 8, Kc(K)))
                        sv[:, half].copy_(stt.view(F // 8, 8, ldS))
                    del parts
                else:
                    r0 = 0
                    for m in mats:
                        w = synth.weights_f32_torch(synth.key(seed, wl.wid, layer, wl.mats.index(m),
                                                              synth.KIND_W), m.N, K, device)
                        bq.quantize_dev(wl.fmt, w, codes[r0:r0 + m.N], scales[r0:r0 + m.N], st)
                        r0 += m.N
                        del w
                reads_h = ffn and names == ["down"] and h_shape is not None
                x = None if reads_h else synth.activations_f16_torch(
                    synth.key(seed, wl.wid, layer, s, synth.KIND_X), (self.B, K), device)
                out = ("h", (self.B, Ntot // 2)) if swiglu else ("y", (self.B, Ntot))
                pending.append((layer, s, "+".join(names), K, Ntot, codes, scales, x, out, reads_h))
                if swiglu:
                    h_shape = (self.B, Ntot // 2)
                self._keep += [codes, scales]
                nb = (synth.packed_bytes(wl.fmt, Ntot, K) + self.B * K * 2 +
                      (self.B * (Ntot // 2) * 2 if swiglu else self.B * Ntot * 4))
                self.bytes_alg += nb
                label = "+".join(names)
                self.bytes_by_label[label] = self.bytes_by_label.get(label, 0) + nb
                ws_max = max(ws_max, bq.lib().bq_verify_workspace_bytes(Ntot, K, self.B)
                             if wl.verify else bq.lib().bq_gemv_workspace_bytes(Ntot, K))

        # Every seeded x in one device buffer and every fp32 y in another
        # (64-byte aligned slices), so a step's inputs and results each move in
        # one copy; the SwiGLU outputs h live in a third buffer on the device.
        def pack(shapes, dtype):
            esz = torch.empty((), dtype=dtype).element_size()
            offs, n = [], 0
            for shp in shapes:
                offs.append(n)
                cnt = shp[0] * shp[1]
                n += -(-cnt * esz // 64) * 64 // esz
            buf = torch.zeros(max(n, 1), dtype=dtype, device=device)
            views = [buf[o:o + a * b].view(a, b) for o, (a, b) in zip(offs, shapes)]
            return buf, views
        self.x_all, xv = pack([p[7].shape for p in pending if p[7] is not None], torch.float16)
        self.y_all, yv = pack([p[8][1] for p in pending if p[8][0] == "y"], torch.float32)
        self.h_all, hv = pack([p[8][1] for p in pending if p[8][0] == "h"], torch.float16)
        xi = yi = hi = 0
        last_h = None
        for layer, s, label, K, Ntot, codes, scales, x, (kind, shp), reads_h in pending:
            if reads_h:
                xd = last_h
            else:
                xd = xv[xi]
                xd.copy_(x)
                xi += 1
            if kind == "h":
                yd, epi = hv[hi], bq.BQ_EPI_SWIGLU
                hi += 1
                last_h = yd
            else:
                yd, epi = yv[yi], bq.BQ_EPI_NONE
                yi += 1
            q = bq.qmat(codes, scales, Ntot, K)
            self.launches.append((q, xd, yd, label, wl.stage_of(layer, s), epi))
        torch.cuda.synchronize()
        if int(st.item()) != 0:
            raise RuntimeError(f"device quantiser status {int(st.item()):#x}")
        self.ws = bq.workspace(ws_max, device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.plan = None

    def build_plan(self):
        """The whole step as one plan (stages in model order), built once.
        (A plan holds at most 256 matrices; larger sets use --engine graph.)"""
        self.plan = self.bq.StepPlan(self.fmt, [(q, x, y, st, epi)
                                                for q, x, y, _, st, epi in self.launches],
                                     self.device)

    def run_step(self, stream):
        """One decode step through the plan: a single launch."""
        self.plan.run(self.status, stream)
        return 1

    def launch_one(self, entry, stream):
        import ctypes
        q, x, y, label, _, epi = entry
        if self.wl.verify:
            rc = self.bq.lib().bq_verify_gemm(self.fmt, ctypes.byref(q), x.data_ptr(), self.B,
                                              y.data_ptr(), self.ws.data_ptr(), self.ws.numel(),
                                              self.status.data_ptr(), stream.cuda_stream)
            if rc != 0:
                raise RuntimeError(f"bq_verify_gemm: {self.bq.bq_status_string(rc)}")
            return
        # the step's weights are resident and never written: each launch may
        # start loading them while the previous one drains
        rc = self.bq.lib().bq_gemv_ex(self.fmt, ctypes.byref(q), x.data_ptr(), self.B, y.data_ptr(),
                                      epi, self.bq.BQ_GEMV_STATIC_WEIGHTS, self.ws.data_ptr(),
                                      self.ws.numel(), self.status.data_ptr(), stream.cuda_stream)
        if rc != 0:
            raise RuntimeError(f"bq_gemv_ex: {self.bq.bq_status_string(rc)}")

    def launch(self, stream, only=None):
        """The step as per-matrix calls (the graph engine), in model order."""
        n = 0
        for e in self.launches:
            if only is not None and e[3] != only:
                continue
            self.launch_one(e, stream)
            n += 1
        return n

    def io_tensors(self):
        """The step's inputs (every x) and results (every y), each one buffer."""
        return self.x_all, self.y_all


class MoEStep:
    """A routed-expert decode step resident in HBM: per layer, the expert stack of
    gate|up (2*ffn x hidden, SwiGLU pair order) and of down (hidden x ffn), Q4,
    all E experts of all layers (~16.3 GB for 48 layers of 128 experts).  One
    step = per layer the gate|up call, whose SwiGLU epilogue writes each routed
    slot's h (fp16), and the down call reading h per slot, combined with the
    routing weights -- the expert feed-forward block with its activation fused.
    Algorithmic bytes count the distinct routed experts only."""

    def __init__(self, wl: synth.MoEWorkload, device, seed: int = 0):
        import torch
        from quantised_weight_gemv_b200 import bq
        self.wl, self.device, self.bq = wl, device, bq
        self.B, self.fmt = wl.B, 4
        E, topk, B = wl.E, wl.topk, wl.B
        (Ng, Kg), (Nd, Kd) = wl.gateup(), wl.down()
        F = Ng // 2
        st = torch.zeros(1, dtype=torch.int32, device=device)
        self.layers = []
        self.bytes_alg = 0
        self.distinct = []
        self._keep = []
        ins = []
        for layer in range(wl.layers):
            idx, r = synth.routing(synth.key(seed, wl.wid, layer, 0, synth.KIND_IDX),
                                   synth.key(seed, wl.wid, layer, 0, synth.KIND_LOGIT), B, E, topk)
            stacks = []
            for mid, (N, K) in ((0, (Ng, Kg)), (1, (Nd, Kd))):
                ldS = bq.scales_ld(K)
                codes = torch.empty((E, N, K // 2), dtype=torch.uint8, device=device)
                scales = torch.empty((E, N, ldS), dtype=torch.int16, device=device)
                w = synth.weights_f32_torch(synth.key(seed, wl.wid, layer, mid, synth.KIND_W),
                                            E * N, K, device)
                if mid == 0:
                    # expert e: rows [0, F) gate, [F, 2F) up; quantised row by
                    # row, then interleaved 8 rows at a time (SwiGLU pair order)
                    ct = torch.empty((E * N, K // 2), dtype=torch.uint8, device=device)
                    stt = torch.empty((E * N, ldS), dtype=torch.int16, device=device)
                    bq.quantize_dev(4, w, ct, stt, st)
                    codes.copy_(ct.view(E, 2, F // 8, 8, K // 2).transpose(1, 2).reshape(E, N, K // 2))
                    scales.copy_(stt.view(E, 2, F // 8, 8, ldS).transpose(1, 2).reshape(E, N, ldS))
                    del ct, stt
                else:
                    bq.quantize_dev(4, w, codes.view(E * N, K // 2), scales.view(E * N, ldS), st)
                del w
                stacks.append((bq.qmat(codes, scales, N, K), N * K // 2, N * ldS))
                self._keep += [codes, scales]
            x = synth.activations_f16_torch(synth.key(seed, wl.wid, layer, 0, synth.KIND_X),
                                            (B, Kg), device)
            ins.append(x)
            nd = len(set(idx.ravel().tolist()))
            self.distinct.append(nd)
            self.bytes_alg += (nd * (synth.packed_bytes(4, Ng, Kg) + synth.packed_bytes(4, Nd, Kd))
                               + x.numel() * 2 + 2 * (B * topk * F * 2) + B * Nd * 4)
            self.layers.append([stacks, torch.as_tensor(idx, device=device),
                                torch.as_tensor(r, device=device)])
        # Every input of the step (x, expert ids, routing weights) in one byte
        # buffer and every output in another, 64-byte aligned slices: one copy
        # each way end to end.  The per-slot h stay on the device.
        def pack(tensors):
            offs, n = [], 0
            for t in tensors:
                offs.append(n)
                n += -(-t.numel() * t.element_size() // 64) * 64
            buf = torch.zeros(n, dtype=torch.uint8, device=device)
            views = []
            for o, t in zip(offs, tensors):
                v = buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
                v.copy_(t)
                views.append(v)
            return buf, views
        in_t = []
        for li, L in enumerate(self.layers):
            in_t += [ins[li], L[1], L[2]]
        self.x_all, iv = pack(in_t)
        self.y_all, ov = pack([torch.zeros((B, Nd), dtype=torch.float32, device=device)
                               for _ in self.layers])
        self.h_all = torch.zeros((wl.layers, B, topk, F), dtype=torch.float16, device=device)
        for li, L in enumerate(self.layers):
            x, idx, r = iv[3 * li:3 * li + 3]
            L[1], L[2] = idx, r
            L += [x, self.h_all[li], ov[li]]
        ws = max(bq.lib().bq_moe_workspace_bytes(Ng, Kg, B, topk, E),
                 bq.lib().bq_moe_workspace_bytes(Nd, Kd, B, topk, E))
        self.ws = bq.workspace(ws, device)
        torch.cuda.synchronize()
        if int(st.item()) != 0:
            raise RuntimeError(f"device quantiser status {int(st.item()):#x}")
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.launches_per_step = 3 * wl.layers   # gate|up, down, combine

    def launch(self, stream, only=None):
        E = self.wl.E
        for stacks, idx, r, x, h, y in self.layers:
            (qg, cg, sg), (qd, cd, sd) = stacks
            self.bq.moe_gemv_q4(qg, E, cg, sg, x, False, idx, None, h, self.ws, self.status, stream,
                                epilogue=self.bq.BQ_EPI_SWIGLU)
            self.bq.moe_gemv_q4(qd, E, cd, sd, h, True, idx, r, y, self.ws, self.status, stream)
        return self.launches_per_step

    def io_tensors(self):
        return self.x_all, self.y_all


class AttnStep:
    """Decode attention of every layer over a Q8 KV cache resident in HBM:
    per layer the keys (position-major) and values (transposed) of every
    (sequence, KV head), Tmax positions each, quantised on the device from
    seeded N(0, 1) values, plus the layer's queries.  One step = one
    bq_attn_decode_q8 call per layer.  Algorithmic bytes: the cache bytes of
    the valid positions (codes + scales of keys and values) + q + o."""

    def __init__(self, wl: synth.AttnWorkload, device, seed: int = 0):
        import torch
        from quantised_weight_gemv_b200 import bq
        self.wl, self.device, self.bq = wl, device, bq
        self.B, self.fmt = wl.B, 8
        B, Hkv, G, T, D = wl.B, wl.Hkv, wl.G, wl.Tmax, wl.D
        rows = B * Hkv * T
        st = torch.zeros(1, dtype=torch.int32, device=device)
        lens = wl.lens(seed)
        self.lens_host = lens
        self.layers, self._keep = [], []
        qs = []
        for layer in range(wl.layers):
            planes = []
            for kind in (synth.KIND_KEY, synth.KIND_VAL):
                g = torch.Generator(device=device)
                g.manual_seed(synth.torch_seed(synth.key(seed, wl.wid, layer, 0, kind)))
                f = torch.randn((rows, D), generator=g, dtype=torch.float32, device=device)
                codes = torch.empty((rows, D), dtype=torch.uint8, device=device)
                sc = torch.empty((rows, bq.scales_ld(D)), dtype=torch.int16, device=device)
                bq.quantize_dev(8, f, codes, sc, st)
                del f
                sc4 = sc[:, :D // 32].contiguous().view(B, Hkv, T, D // 32)
                c4 = codes.view(B, Hkv, T, D)
                if kind == synth.KIND_VAL:
                    c4 = c4.transpose(2, 3).contiguous()          # [B, Hkv, D, T]
                planes += [c4, sc4]
            kv = bq.kv_cache(*planes)
            self._keep += planes
            q = synth.activations_f16_torch(synth.key(seed, wl.wid, layer, 0, synth.KIND_X),
                                            (B, Hkv * G, D), device)
            qs.append(q)
            self.layers.append(kv)
        torch.cuda.synchronize()
        if int(st.item()) != 0:
            raise RuntimeError(f"device quantiser status {int(st.item()):#x}")
        # every query of the step in one buffer, every output in another
        qn = B * Hkv * G * D
        self.x_all = torch.empty((wl.layers, qn), dtype=torch.float16, device=device)
        for li, q in enumerate(qs):
            self.x_all[li].copy_(q.view(-1))
        self.y_all = torch.zeros((wl.layers, B, Hkv * G, D), dtype=torch.float32, device=device)
        self.lens = torch.as_tensor(lens, device=device)
        self.ws = bq.workspace(bq.lib().bq_attn_workspace_bytes(B, Hkv), device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        L = int(sum(min(max(int(v), 0), T) for v in lens))       # valid positions of a layer
        self.bytes_alg = wl.layers * (L * Hkv * 2 * (D + 2 * (D // 32)) + qn * 2 + qn * 4)
        self.launches_per_step = wl.layers
        self.scale = 1.0 / math.sqrt(D)

    def launch(self, stream, only=None):
        wl = self.wl
        for li, kv in enumerate(self.layers):
            q = self.x_all[li].view(wl.B, wl.Hkv * wl.G, wl.D)
            self.bq.attn_decode_q8(kv, q, self.lens, wl.G, self.scale, self.y_all[li], self.ws,
                                   self.status, stream)
        return self.launches_per_step

    def io_tensors(self):
        return self.x_all, self.y_all


# ---------------------------------------------------------- CPU oracle ----
_SAMPLES = {}


def oracle_sample(wl: synth.DenseWorkload, seed: int = 0):
    """Packed planes (oracle quantiser) + x for one layer of the workload
    (built once per workload and seed)."""
    if (wl.name, seed) not in _SAMPLES:
        _SAMPLES[(wl.name, seed)] = _oracle_sample(wl, seed)
    return _SAMPLES[(wl.name, seed)]


def _oracle_sample(wl: synth.DenseWorkload, seed: int = 0):
    import numpy as np
    import oracle
    mats = []
    for s, group in fused_stages(wl):
        K = group[0].K
        parts = [synth.weights_f32(synth.key(seed, wl.wid, 0, wl.mats.index(m), synth.KIND_W), m.N, K)
                 for m in group]
        w = np.concatenate(parts, axis=0)
        codes, scales = {2: oracle.quantize_q2, 3: oracle.quantize_q3, 4: oracle.quantize_q4,
                         5: oracle.quantize_q5, 6: oracle.quantize_q6,
                         8: oracle.quantize_q8}[wl.fmt](w)
        x = synth.activations_f16_bits(synth.key(seed, wl.wid, 0, s, synth.KIND_X), wl.B, K)
        nbytes = synth.packed_bytes(wl.fmt, w.shape[0], K) + wl.B * K * 2 + wl.B * w.shape[0] * 4
        mats.append((codes, scales, x, nbytes))
    return mats


def moe_oracle_sample(wl: synth.MoEWorkload, seed: int = 0):
    """Layer 0 of a routed-expert workload for the oracle: the same routing as
    the GPU step, packed stacks (oracle quantiser) holding the routed experts,
    x and the per-slot h.  Returns (jobs, algorithmic bytes)."""
    import numpy as np
    import oracle
    E, topk, B = wl.E, wl.topk, wl.B
    idx, r = synth.routing(synth.key(seed, wl.wid, 0, 0, synth.KIND_IDX),
                           synth.key(seed, wl.wid, 0, 0, synth.KIND_LOGIT), B, E, topk)
    used = sorted(set(idx.ravel().tolist()))
    jobs, nbytes = [], 0
    for mid, (N, K) in ((0, wl.gateup()), (1, wl.down())):
        ldS = (K // 32 + 7) // 8 * 8
        codes = np.zeros((E, N, K // 2), dtype=np.uint8)
        scales = np.zeros((E, N, ldS), dtype=np.uint16)
        for e in used:
            w = synth.weights_f32(synth.key(seed, wl.wid, 0, mid * 1000 + e, synth.KIND_W), N, K)
            codes[e], scales[e] = oracle.quantize_q4(w)
        if mid == 0:
            x = synth.activations_f16_bits(synth.key(seed, wl.wid, 0, 0, synth.KIND_X), B, K)
            jobs.append((codes, scales, x, False, idx, None))
            nbytes += x.size * 2 + B * topk * (N // 2) * 2
        else:
            jobs.append((codes, scales, None, True, idx, r))   # x = h of the gate|up job
            nbytes += B * topk * K * 2 + B * N * 4
        nbytes += len(used) * synth.packed_bytes(4, N, K)
    return jobs, nbytes


def attn_oracle_job(wl, seed: int = 0):
    """Layer 0 of an attention workload for the oracle: the same seeded keys,
    values (quantised by the oracle's Q8 quantiser), queries and lengths.
    (The oracle's attention is single-threaded.)"""
    import numpy as np
    import oracle
    if ("attn", wl.name, seed) not in _SAMPLES:
        B, Hkv, G, T, D = wl.B, wl.Hkv, wl.G, wl.Tmax, wl.D
        rows = B * Hkv * T
        planes = []
        for kind in (synth.KIND_KEY, synth.KIND_VAL):
            f = synth.kv_values_f32(synth.key(seed, wl.wid, 0, 0, kind), rows, D)
            c, sc = oracle.quantize_q8(f)
            c = c.reshape(B, Hkv, T, D)
            if kind == synth.KIND_VAL:
                c = np.ascontiguousarray(c.transpose(0, 1, 3, 2))
            planes += [c, np.ascontiguousarray(sc[:, :D // 32]).reshape(B, Hkv, T, D // 32)]
        q = synth.activations_f16_bits(synth.key(seed, wl.wid, 0, 0, synth.KIND_X), B, Hkv * G, D)
        _SAMPLES[("attn", wl.name, seed)] = (planes, q, wl.lens(seed))
    planes, q, lens = _SAMPLES[("attn", wl.name, seed)]
    L = int(sum(min(max(int(v), 0), wl.Tmax) for v in lens))
    qn = wl.B * wl.Hkv * wl.G * wl.D
    nbytes = L * wl.Hkv * 2 * (wl.D + 2 * (wl.D // 32)) + qn * 2 + qn * 4

    def run():
        oracle.attn_decode_q8(*planes, q, lens, 1.0 / math.sqrt(wl.D))
    return run, nbytes


def oracle_job(wl, frac: float = 1.0, threads: int | None = None):
    """(run-once callable, algorithmic bytes) for the CPU oracle: layer 0 of the
    workload, or (dense workloads, frac < 1) a frac share of every matrix's rows
    per call, taken from a few row ranges spread over the matrix that successive
    calls cycle through."""
    import oracle
    threads = threads or os.cpu_count() or 1
    if isinstance(wl, synth.AttnWorkload):
        return attn_oracle_job(wl)
    if isinstance(wl, synth.MoEWorkload):
        jobs, nbytes = moe_oracle_sample(wl)

        def run():
            # gate|up per slot, SwiGLU (gate rows first, up rows second), down
            # per slot on h, combined with the routing weights
            (cg, sg, x, _, idx, _), (cd, sd, _, _, _, r) = jobs
            y, _, _ = oracle.moe_gemv_q4(cg, sg, x, False, idx, None, nthreads=threads)
            F = y.shape[2] // 2
            h = oracle.swiglu_f16(y[..., :F], y[..., F:])
            oracle.moe_gemv_q4(cd, sd, h, True, idx, r, nthreads=threads)
        return run, nbytes
    mats = oracle_sample(wl)
    gemv = {2: oracle.gemv_q2, 3: oracle.gemv_q3, 4: oracle.gemv_q4, 5: oracle.gemv_q5,
            6: oracle.gemv_q6, 8: oracle.gemv_q8}[wl.fmt]
    if frac >= 1.0:
        nbytes = sum(m[3] for m in mats)

        def run():
            for codes, scales, x, _ in mats:
                gemv(codes, scales, x, nthreads=threads)
        return run, nbytes
    n_slices = min(8, int(math.ceil(1.0 / frac)))
    sliced, nbytes = [], 0
    for codes, scales, x, _ in mats:
        N, K = codes.shape[0], x.shape[1]
        n = min(N, max(16, int(round(N * frac))))
        starts = [i * (N - n) // max(1, n_slices - 1) for i in range(n_slices)]
        sliced.append([(codes[r:r + n].copy(), scales[r:r + n].copy(), x) for r in starts])
        nbytes += synth.packed_bytes(wl.fmt, n, K) + wl.B * K * 2 + wl.B * n * 4
    turn = [0]

    def run():
        i = turn[0] % n_slices
        turn[0] += 1
        for sl in sliced:
            codes, scales, x = sl[i]
            gemv(codes, scales, x, nthreads=threads)
    return run, nbytes


def time_once(run):
    t0 = time.perf_counter()
    run()
    return time.perf_counter() - t0


def cpu_baseline(wl, budget_s=10.0):
    """The oracle timed on the host cores: all of them, and one thread (the
    same work), each for about budget_s seconds.  A pass is layer 0 of the
    workload, or a share of every matrix's rows of it when one pass of the
    whole layer would take longer than the budget."""
    legs = []
    for threads in (os.cpu_count() or 1, 1):
        frac = 1.0
        run, nbytes = oracle_job(wl, threads=threads)
        t1 = time_once(run)
        if t1 > budget_s and not isinstance(wl, (synth.MoEWorkload, synth.AttnWorkload)):
            frac = max(budget_s / (2 * t1), 1.0 / 256)
            run, nbytes = oracle_job(wl, frac, threads=threads)
        reps, total = 0, 0.0
        while total < budget_s or reps == 0:
            total += time_once(run)
            reps += 1
        what = (f"layer 0 of {wl.layers}" if frac >= 1.0 else
                f"{frac:.4f} of the rows of every matrix of layer 0 of {wl.layers}")
        legs.append({"value": round(nbytes * reps / total / 1e9, 4), "unit": "GB/s",
                     "cores": threads, "kind": "oracle",
                     "sample": f"{what} ({nbytes/1e6:.1f} MB algorithmic), {reps} pass(es), "
                               f"fp64 oracle, {threads} thread(s)"})
    out = dict(legs[0])
    out["single_thread"] = legs[1]
    return out


def run_reference(args, wl, rank):
    """The oracle on the host cores, on this workload's config and metric.  A
    step is layer 0; when steps + warm-up of whole layers would overrun the
    time budget, a step is the same share of every matrix's rows instead,
    sized so the run fits (at least 1/256 of the rows and 16 rows a matrix)."""
    if rank != 0:
        return
    threads = os.cpu_count() or 1
    run, nbytes = oracle_job(wl)
    t_layer = time_once(run)                       # a calibration pass (untimed)
    frac, sample = 1.0, f"layer 0 of {wl.layers} per step ({nbytes/1e6:.1f} MB)"
    budget = (args.steps + args.warmup) * t_layer
    if budget > args.ref_budget_s and not isinstance(wl, (synth.MoEWorkload, synth.AttnWorkload)):
        frac = max(args.ref_budget_s / budget, 1.0 / 256)
        run, nbytes = oracle_job(wl, frac)
        sample = (f"{frac:.4f} of the rows of every matrix of layer 0 of {wl.layers} per step "
                  f"({nbytes/1e6:.2f} MB), cycling over row ranges")
    for _ in range(args.warmup):
        time_once(run)
    t = 0.0
    for _ in range(args.steps):
        t += time_once(run)
    val = nbytes * args.steps / t / 1e9
    # ms_per_step is a whole layer's time: the time of the share timed, over
    # the share (the rate is the same either way)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t / args.steps / frac * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.B, "layers": wl.layers,
                   "sample": "one layer per step" if frac >= 1.0 else "a share of one layer per step",
                   "rows_share": round(frac, 6),
                   "ms_per_step_is": "one layer of the workload (scaled from the share timed)"},
        "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ replicas ----
def max_over_ranks(t: float, device, world: int) -> float:
    """The slowest rank's time (every rank takes part; the result is on all)."""
    if world == 1:
        return t
    import torch
    import torch.distributed as dist
    tt = torch.tensor([t], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def job_gbs(world: int, bytes_per_step: int, steps: int, t: float) -> float:
    """Whole-job GB/s: every replica streams bytes_per_step per step, timed by the
    slowest rank."""
    return world * bytes_per_step * steps / t / 1e9


# ---------------------------------------------------------------- main ----
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="bq", choices=["bq", "reference"])
    ap.add_argument("--workload", default=synth.DENSE_H5120.name, choices=sorted(WORKLOADS),
                    help="default: the 64-layer hidden-5120 dense decoder, Q4, batch 1 (16.4 GB "
                         "of packed weights per step), the largest workload that fits one GPU")
    ap.add_argument("--engine", default=None, choices=["step", "graph"],
                    help="graph (default): a CUDA graph of per-matrix bq_gemv_ex launches "
                         "with static weights; step: one cooperative launch per token "
                         "(bq_step_run)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-budget-s", type=float, default=90.0,
                    help="--impl reference: seconds of oracle work the steps and warm-up may take")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    wl = WORKLOADS[args.workload]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, wl, rank)
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=device)

    def barrier():
        if world > 1:
            dist.barrier()

    is_moe = isinstance(wl, synth.MoEWorkload)
    is_attn = isinstance(wl, synth.AttnWorkload)
    if is_attn:
        args.engine = "graph"   # one graph of the per-layer attention calls
        step = AttnStep(wl, device)
    elif is_moe:
        args.engine = "graph"   # one graph of the per-layer expert calls
        step = MoEStep(wl, device)
    else:
        if args.engine is None or wl.verify:
            # the chain of per-matrix launches with static weights: each launch
            # starts loading its weights while the previous one drains, which
            # measured faster than the one-launch plan's grid barriers (a
            # verification step has no plan form)
            args.engine = "graph"
        step = DenseStep(wl, device)
    stream = torch.cuda.Stream(device)
    peaks = load_peaks()

    # warm the kernels (attributes, module load) before capture
    if args.engine == "step":
        step.build_plan()
        with torch.cuda.stream(stream):
            n_launch = step.run_step(stream)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step.run_step(torch.cuda.current_stream())
        torch.cuda.synchronize()
    else:
        with torch.cuda.stream(stream):
            n_launch = step.launch(stream)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step.launch(torch.cuda.current_stream())
        torch.cuda.synchronize()

    props = torch.cuda.get_device_properties(device)
    pci = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
    sampler = ClockSampler(phys_gpu_index(local_rank), pci)
    sampler.start()
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g.replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    # A step smaller than twice the L2 would be served from L2 when replayed:
    # then every step is timed alone, after an untimed write of a buffer
    # larger than the L2.
    flush = None
    if step.bytes_alg < L2_FLUSH_BYTES:
        flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_begin = time.time()
    pairs = []
    with torch.cuda.stream(stream):
        if flush is None:
            e0.record(stream)
            for _ in range(args.steps):
                g.replay()
            e1.record(stream)
        else:
            for _ in range(args.steps):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                g.replay()
                b.record(stream)
                pairs.append((a, b))
    torch.cuda.synchronize()
    t_end = time.time()
    barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop(t_begin, t_end)
    t_local = (e0.elapsed_time(e1) if flush is None else sum(a.elapsed_time(b) for a, b in pairs)) / 1e3
    t_dev = max_over_ranks(t_local, device, world)
    if int(step.status.item()) != 0:
        raise RuntimeError(f"device status {int(step.status.item()):#x}")

    isolated = None
    if is_attn:
        # every launch is the attention kernel: its average launch
        dom = f"average of the {n_launch} per-layer launches of a step"
        dom_s = t_dev / args.steps / n_launch
        dom_bytes = step.bytes_alg / n_launch
    elif args.engine == "step" or is_moe:
        # the step kernel is the only kernel (one launch per step), or (routed
        # experts) the expert kernel is every launch but the small combine
        # kernels: timed over the timed region itself
        dom = "decode step (all stages)" if not is_moe else "routed-expert step (all launches)"
        dom_s = t_dev / args.steps
        dom_bytes = step.bytes_alg
    else:
        # every launch of the step is the same kernel: its average launch over
        # the timed region (bytes per launch = step bytes / launches)
        dom = f"average of the {n_launch} launches of a step"
        dom_s = t_dev / args.steps / n_launch
        dom_bytes = step.bytes_alg / n_launch
        # for reference: the largest projection's launch timed alone (no
        # neighbour to overlap its start with)
        big = max(step.bytes_by_label, key=step.bytes_by_label.get)
        durs = []
        with torch.cuda.stream(stream):
            for _ in range(3):
                for e in step.launches:
                    if e[3] != big:
                        continue
                    if flush is not None:
                        flush.zero_()   # a set smaller than the L2: time each call cold
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record(stream)
                    step.launch_one(e, stream)
                    b.record(stream)
                    durs.append((a, b))
        torch.cuda.synchronize()
        n_big = sum(1 for l in step.launches if l[3] == big)
        big_s = statistics.mean(a.elapsed_time(b) for a, b in durs) / 1e3
        isolated = {"launch": big, "us": round(big_s * 1e6, 3),
                    "GB/s": round(step.bytes_by_label[big] / n_big / big_s / 1e9, 1)}
    achieved = dom_bytes / dom_s / 1e9
    # the verification GEMM's tensor-core rate beside its HBM rate (2 B N K
    # flop a matrix; the dense f16 peak equals the measured bf16 one)
    verify = not is_moe and not is_attn and wl.verify
    tensor = None
    if verify:
        flops = 2.0 * wl.B * wl.layers * wl.layer_weights()
        tf = flops / (t_dev / args.steps) / 1e12
        tensor = {"achieved_tflops": round(tf, 1), "peak_tflops": peaks.get("bf16_tflops"),
                  "peak_source": "measured bf16 dense (f16 runs at the same rate)",
                  "frac": round(tf / peaks["bf16_tflops"], 4) if peaks.get("bf16_tflops") else None}

    # end to end: pinned host x -> device, step, y -> pinned host, every step
    # (one copy each way: every x of the step lives in one buffer, every y in
    # another)
    xs, ys = step.io_tensors()
    hx = xs.cpu().pin_memory()
    hy = torch.empty(ys.shape, dtype=ys.dtype).pin_memory()
    e2e_steps = max(1, min(args.steps, 500))
    with torch.cuda.stream(stream):
        for _ in range(3):
            xs.copy_(hx, non_blocking=True)
            g.replay()
            hy.copy_(ys, non_blocking=True)
    torch.cuda.synchronize()
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pairs = []
    with torch.cuda.stream(stream):
        if flush is None:
            f0.record(stream)
        for _ in range(e2e_steps):
            if flush is not None:
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
            xs.copy_(hx, non_blocking=True)
            g.replay()
            hy.copy_(ys, non_blocking=True)
            if flush is not None:
                b.record(stream)
                pairs.append((a, b))
        if flush is None:
            f1.record(stream)
    torch.cuda.synchronize()
    t_local = (f0.elapsed_time(f1) if flush is None else sum(a.elapsed_time(b) for a, b in pairs)) / 1e3
    t_e2e = max_over_ranks(t_local, device, world)
    h2d = xs.numel() * xs.element_size()
    d2h = ys.numel() * ys.element_size()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)

    if rank == 0:
        value = job_gbs(world, step.bytes_alg, args.steps, t_dev)
        ms = t_dev / args.steps * 1e3
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16",
            "arith": ("q8 KV codes as exact f16 subnormal mma operands, f16 q, f32 scores and "
                      "online softmax, p*dV*2^s rounded once to f16" if is_attn else
                      f"q{step.fmt} weights as f16 d(q-z)2^s (one rounding) in tcgen05 mma, f16 x, "
                      "f32 accumulation in tensor memory" if verify else
                      f"q{step.fmt} codes as exact f16 subnormal mma operands, f16 x, "
                      "f32 accumulation and scaling"),
            "data": "synthetic (seeded N(0,0.02) weights, N(0,1) fp16 activations)",
            "config": {"workload": wl.name, "batch": wl.B, "layers": wl.layers,
                       "launches_per_step": n_launch, "bytes_per_step": step.bytes_alg,
                       "engine": ("cuda-graph of per-layer bq_attn_decode_q8 calls" if is_attn else
                                  "cuda-graph of per-layer bq_moe_gemv_ex calls" if is_moe else
                                  "one cooperative launch per step (bq_step_run), graph-captured"
                                  if args.engine == "step" else
                                  "cuda-graph of per-matrix bq_verify_gemm launches" if verify else
                                  "cuda-graph of per-matrix bq_gemv_ex launches, static weights"),
                       "l2": ("inputs larger than L2 (no flush)" if flush is None else
                              f"L2 flushed before every step ({L2_FLUSH_BYTES >> 20} MB write, untimed); "
                              "steps timed one by one"),
                       "parallelism": f"replicas x{world}"},
            "tokens_per_s_equiv": round(world * wl.B / (t_dev / args.steps), 1),
            **({"distinct_experts_per_layer": round(statistics.mean(step.distinct), 2)}
               if is_moe else {}),
            "frac_of_measured_hbm": round(value / world / peaks["hbm_gbs"], 4),
            "frac_of_8TBps": round(value / world / 8000.0, 4),
            "roofline": {"bound": "hbm",
                         "kernel": (f"attn_decode q8 KV ({dom})" if is_attn else
                                    f"verify_gemm q{step.fmt} ({dom})" if verify else
                                    f"stream_gemv q{step.fmt} ({dom})"),
                         "timed": "CUDA events over the timed region",
                         "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                         "peak_source": peaks["source"], "unit": "GB/s",
                         "frac": round(achieved / peaks["hbm_gbs"], 4),
                         "traffic": profiled_traffic(wl.name, args.engine,
                                                     "attention.cu" if is_attn else
                                                     "verify_gemm.cu" if verify else "stream_gemv.cu"),
                         "bytes_per_launch": int(dom_bytes),
                         "launch_us": round(dom_s * 1e6, 3),
                         **({"isolated_launch": isolated} if isolated else {}),
                         **({"tensor": tensor} if tensor else {})},
            "cpu_baseline": cpu,
            "e2e": {"value": round(job_gbs(world, step.bytes_alg, e2e_steps, t_e2e), 2),
                    "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps},
            "gpu_launches": n_launch * args.steps,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    del g
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
