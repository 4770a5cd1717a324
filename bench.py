#!/usr/bin/env python3
"""Benchmark: weight GB/s and % of the B200 HBM roofline for one 27B weight pass.

Step = one pass of the whole hot path over resident synthetic weights:
  64 layers x {gate+up 5120->34816, down 17408->5120, qkv 5120->10240} NVFP4 GEMMs
  followed by the fused lm_head verify (5120->248,320 rows, argmax + accept length).
The headline is M = 17 (16 drafted tokens + 1). M = 1 (plain decode) and M = 68
(4 sequences x 17 sharing one read) are reported in ``per_m``. Each pass is one
weight pass of the library (activation prep, the persistent pass kernel over all
193 GEMMs with the lm_head as its verify problem, verify stage 2), captured in a
CUDA graph and replayed; CUDA events on the launching stream bracket every step.
Beside it, ``chained_ms_per_pass`` times the same work as 193 per-GEMM launches in
layer order. The weight stack (11.5 GB) is far larger than L2, so no flush is
needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With --gpus N > 1 (under torchrun) every rank runs its own replica of the pass
on its own GPU. There is no data-path collective, ``scaling`` is weak, and value
is the sum over ranks, taken over the max-over-ranks time.
"""

from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic as S  # noqa: E402

BYTES_PER_WEIGHT = 0.5 + 1.0 / 16.0          # E2M1 nibble + E4M3 scale per 16
METRIC = "weight GB/s and % of B200 HBM roofline per 27B weight pass at M=1/17/68"
WORKLOAD = ("27B weight pass: 64 x {gate_up 5120->34816, down 17408->5120, qkv 5120->10240} NVFP4 GEMMs "
            "+ lm_head verify 5120->248320 (argmax + accept)")


def weight_bytes(N: int, K: int) -> int:
    return N * K // 2 + N * K // 16


def stack_weight_bytes(layers: int = S.N_LAYERS) -> int:
    return layers * sum(weight_bytes(N, K) for (K, N) in (S.LAYER_SHAPES[n] for n in S.LAYER_ORDER))


def lmhead_weight_bytes() -> int:
    return weight_bytes(S.VOCAB, S.LMHEAD_K)


def pass_alg_bytes(M: int, layers: int = S.N_LAYERS) -> int:
    """Algorithmic bytes of one pass: every weight and scale read once, every
    activation row read once (bf16), every GEMM output written once (fp32), and the
    lm_head's weights and activations (its logits never leave the chip)."""
    total = 0
    for name in S.LAYER_ORDER:
        K, N = S.LAYER_SHAPES[name]
        total += weight_bytes(N, K) + M * K * 2 + M * N * 4
    return layers * total + lmhead_weight_bytes() + M * S.LMHEAD_K * 2


# Sources whose change invalidates a stored DRAM-traffic capture of the pass kernel.
PASS_KERNEL_SOURCES = ["nvfp4_weight_streaming_gemm_b200/csrc/mxf4.cu", "nvfp4_weight_streaming_gemm_b200/csrc/sync.cuh",
                       "nvfp4_weight_streaming_gemm_b200/csrc/common.cuh"]
TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "pass_kernel_dram_traffic.json")


def pass_kernel_source_hash() -> str:
    """Hash of the pass kernel's sources with comments and whitespace removed: a change
    of the code invalidates a stored capture, a change of its comments does not."""
    import hashlib
    import re
    h = hashlib.sha256()
    for rel in PASS_KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()


def measured_traffic(M: int, layers: int):
    """DRAM bytes (read + write) of one full-size pass_kernel launch at this M, from the stored
    ncu capture, or None when there is none for this M or the kernel sources changed since it
    was taken. The capture is of a reduced stack (its "layers"); its bytes are scaled to the
    64-layer pass by the ratio of the algorithmic bytes, which assumes the excess over them
    is the same fraction at both sizes."""
    if not os.path.exists(TRAFFIC_PROFILE) or layers != S.N_LAYERS:
        return None
    with open(TRAFFIC_PROFILE) as f:
        prof = json.load(f)
    if prof.get("source_sha256") != pass_kernel_source_hash():
        return None
    v = prof.get("per_m", {}).get(str(M))
    if v is None:
        return None
    cap_layers = int(prof.get("layers", S.N_LAYERS))
    return float(v["dram_read_bytes"] + v["dram_write_bytes"]) * pass_alg_bytes(M, layers) / pass_alg_bytes(M, cap_layers)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
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
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- our arm

def build_pass(nv, torch, dev, M_list, rank: int, layers: int):
    """Pack the layer stack and the lm_head on the GPU; make inputs for every M."""
    stack = []
    for layer in range(layers):
        for j, name in enumerate(S.LAYER_ORDER):
            K, N = S.LAYER_SHAPES[name]
            g = torch.Generator(device=dev)
            g.manual_seed(1000 * layer + j + 1_000_003 * rank)
            W = torch.randn(N, K, generator=g, device=dev, dtype=torch.float32).mul_(S.W_STD)
            q, sf, ts = nv.pack(W)
            del W
            stack.append((name, K, N, q, sf, ts))
    g = torch.Generator(device=dev)
    g.manual_seed(S.LMHEAD_W_SEED + 1_000_003 * rank)
    W = torch.randn(S.VOCAB, S.LMHEAD_K, generator=g, device=dev, dtype=torch.float32).mul_(S.W_STD)
    lm = nv.pack(W)
    del W
    torch.cuda.synchronize()
    return stack, lm


class Pass:
    """One M: per-layer X and Y, drafts, the weight pass (one persistent launch over the
    192 GEMMs with the lm_head verify as its last problem), and, for comparison, the
    chained per-GEMM launch sequence, each captured in a CUDA graph."""

    def __init__(self, nv, torch, dev, stack, lm, M: int, rank: int, chain: bool, tree: bool = False,
                 binv: bool = False, four_terms: bool = False):
        self.M = M
        self.tree = tree
        self.torch = torch
        self.B = max(1, M // (S.DRAFT_LEN + 1)) if M >= S.DRAFT_LEN + 1 else 1
        self.D = M // self.B - 1
        assert self.B * (self.D + 1) == M
        g = torch.Generator(device=dev)
        g.manual_seed(7 + M + 1_000_003 * rank)
        # one device buffer holds every per-layer X (plus the lm_head X) so one copy refreshes them all
        sizes = [M * K for (_, K, _, _, _, _) in stack] + [M * S.LMHEAD_K]
        self.x_all = torch.randn(sum(sizes), generator=g, device=dev).to(torch.bfloat16)
        self.xs, off = [], 0
        for n in sizes:
            self.xs.append(self.x_all[off: off + n])
            off += n
        self.ys = [torch.empty((M, N), dtype=torch.float32, device=dev) for (_, _, N, _, _, _) in stack]
        self.argmax = torch.empty(M, dtype=torch.int32, device=dev)
        self.accept = torch.empty(self.B, dtype=torch.int32, device=dev)
        self.vmax = torch.empty(M, dtype=torch.float32, device=dev)
        self.drafts = torch.zeros((self.B, self.D), dtype=torch.int32, device=dev)
        self.stack, self.lm, self.nv, self.chain = stack, lm, nv, chain
        problems = [(self.xs[i].view(M, K), q, sf, ts, self.ys[i]) for i, (_, K, _, q, sf, ts) in enumerate(stack)]
        ql, sfl, tsl = lm
        problems.append((self.xs[-1].view(M, S.LMHEAD_K), ql, sfl, tsl, None))
        verify = (self.drafts, self.argmax, self.accept, self.vmax)
        if tree:   # draft trees of D nodes per sequence instead of chains
            self.parents = torch.from_numpy(S.random_tree(self.B, self.D, seed=S.LMHEAD_L_SEED + M)).to(dev)
            self.node = torch.empty(self.B, dtype=torch.int32, device=dev)
            verify = verify + (self.parents, self.node)
        self.binv = binv
        self.four_terms = four_terms
        self.wp = nv.WeightPass(problems, M, verify=verify, batch_invariant=binv, four_terms=four_terms)
        self.problems, self.verify_bufs = problems, verify
        if chain:
            wsb = max(nv.gemm_workspace_bytes(M, N, K) for (_, K, N, _, _, _) in stack)
            self.gws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device=dev)
            self.vws = torch.zeros(max(nv.verify_workspace_bytes(M, S.VOCAB, S.LMHEAD_K), 16), dtype=torch.uint8,
                                   device=dev)
        # drafts: the target's own greedy tokens for a prefix L* ~ U{0..D}, then random ids
        self.wp.run()
        torch.cuda.synchronize()
        t = self.argmax.cpu().numpy()
        Lstar = np.random.default_rng(S.LMHEAD_L_SEED + M).integers(0, self.D + 1, size=self.B)
        if tree:
            d = S.tree_drafts(t, self.parents.cpu().numpy(), self.D, S.VOCAB, agree=0.8, seed=S.LMHEAD_L_SEED + M)
        else:
            d = S.drafts_with_prefix(t, Lstar, self.D, S.VOCAB)
        self.drafts.copy_(torch.from_numpy(d))
        self.Lstar = Lstar

    def chain_gemm_calls(self):
        nv, M = self.nv, self.M
        for i, (name, K, N, q, sf, ts) in enumerate(self.stack):
            X = self.xs[i].view(M, K)
            nv.gemm(X, q, sf, ts, out=self.ys[i], workspace=self.gws)

    def chain_verify_call(self):
        q, sf, ts = self.lm
        X = self.xs[-1].view(self.M, S.LMHEAD_K)
        if self.tree:
            self.nv.verify_tree(X, q, sf, ts, self.drafts, self.parents, workspace=self.vws,
                                out=(self.argmax, self.accept, self.node, self.vmax))
        else:
            self.nv.verify(X, q, sf, ts, self.drafts, workspace=self.vws, out=(self.argmax, self.accept, self.vmax))

    def capture(self):
        torch = self.torch
        lib = self.nv.lib()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):           # warm every path outside capture
            self.wp.run()
            if self.chain:
                self.chain_gemm_calls()
                self.chain_verify_call()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        n0 = lib.nvfp4ws_kernel_launches()
        self.g_pass = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_pass):
            self.wp.run()
        self.launches_pass = lib.nvfp4ws_kernel_launches() - n0
        if self.chain:
            self.g_chain = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.g_chain):
                self.chain_gemm_calls()
                self.chain_verify_call()
        torch.cuda.synchronize()

    def run_timed(self, steps: int, graph=None):
        torch = self.torch
        graph = graph or self.g_pass
        st = torch.cuda.current_stream()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        ev[0].record(st)
        for k in range(steps):
            graph.replay()
            ev[k + 1].record(st)
        torch.cuda.synchronize()
        per = np.array([ev[k].elapsed_time(ev[k + 1]) for k in range(steps)])
        return ev[0].elapsed_time(ev[-1]), per

    def add_second_input_buffer(self):
        """A second device copy of every X with its own weight pass and graph (same weights, Y
        and verify outputs), so that the end-to-end leg can copy step k+1's inputs in while
        step k's pass runs."""
        torch, M = self.torch, self.M
        self.x_all2 = torch.empty_like(self.x_all)
        xs2, off = [], 0
        for x in self.xs:
            xs2.append(self.x_all2[off: off + x.numel()])
            off += x.numel()
        probs2 = [(xs2[i].view(M, X.shape[1]), q, sf, ts, Y) for i, (X, q, sf, ts, Y) in enumerate(self.problems)]
        self.wp2 = self.nv.WeightPass(probs2, M, verify=self.verify_bufs, batch_invariant=self.binv,
                                      four_terms=self.four_terms)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.wp2.run()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.g_pass2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_pass2):
            self.wp2.run()
        torch.cuda.synchronize()

    def run_e2e(self, steps: int, x_host, out_host):
        """Through the public API with host buffers, every step: the step's inputs copied in
        from pinned host memory, the pass, and the verify result (argmax and accept lengths)
        copied out. Two device input buffers alternate: step k+1's copy runs on its own
        stream while step k's pass runs, and a buffer is refilled only after the pass that
        read it has finished. Returns the device time of the whole sequence (ms)."""
        torch = self.torch
        st = torch.cuda.current_stream()
        cp = torch.cuda.Stream()
        bufs, graphs = (self.x_all, self.x_all2), (self.g_pass, self.g_pass2)
        ev = lambda: torch.cuda.Event()                                        # noqa: E731
        copied, used = [ev() for _ in range(steps)], [ev() for _ in range(steps)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        cp.wait_stream(st)
        for k in range(min(2, steps)):                                         # fill both buffers
            with torch.cuda.stream(cp):
                bufs[k % 2].copy_(x_host[k % len(x_host)], non_blocking=True)
                copied[k].record(cp)
        for k in range(steps):
            st.wait_event(copied[k])
            graphs[k % 2].replay()
            used[k].record(st)
            out_host[0][k % len(out_host[0])][: self.M].copy_(self.argmax, non_blocking=True)
            out_host[1][k % len(out_host[1])][: self.B].copy_(self.accept, non_blocking=True)
            if k + 2 < steps:                                                  # refill this buffer
                cp.wait_event(used[k])
                with torch.cuda.stream(cp):
                    bufs[k % 2].copy_(x_host[(k + 2) % len(x_host)], non_blocking=True)
                    copied[k + 2].record(cp)
        e1.record(st)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)


def time_calls(torch, calls, reps: int) -> float:
    """Mean device time (us) of one call in a stream of ``calls`` repeated ``reps`` times:
    the calls are captured once into a CUDA graph, which is replayed after two warm-up
    replays, with CUDA events on the launching stream around the timed replays."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):                       # first calls outside capture (one-time set-up)
        for c in calls:
            c()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for c in calls:
            c()
    for _ in range(2):
        g.replay()
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(st)
    for _ in range(reps):
        g.replay()
    e1.record(st)
    torch.cuda.synchronize()
    del g
    return 1e3 * e0.elapsed_time(e1) / (reps * len(calls))


def _entry(us: float, wbytes: int, alg_bytes: int, peak: float, **kw) -> dict:
    d = {"us": round(us, 3), "weight_gbs": round(wbytes / us / 1e3, 1),
         "pct_of_8tbs": round(100.0 * wbytes / (us * 1e-6) / 8e12, 2),
         "alg_gbs": round(alg_bytes / us / 1e3, 1), "hbm_frac": round(alg_bytes / us / 1e3 / peak, 4)}
    d.update(kw)
    return d


def run_extras(nv, torch, dev, stack, lm, peak: float, reps: int) -> dict:
    """The measurement configurations beside the full pass, each a stream of single library
    calls timed as a CUDA graph, rotating through distinct weight copies so every call
    reads its weights from HBM:
      single_m1   one GEMM at M=1 (nvfp4_gemm_skinny, default path: the block-scaled tensor
                  cores) at each 27B layer shape, over the stack's 64 copies of that shape;
      single_m1_gemv  the same on the CUDA-core GEMV (register-prefetch variant);
      verify      the standalone fused verify (lmhead_verify_argmax_accept) at N=248,320
                  and at the 65,536-row slice (four disjoint slices in turn), M=17 and 68;
      m_sweep     one GEMM (nvfp4_gemm_skinny, default path) on gate+up 5120->34816 at
                  M in {1, 2, 4, 8, 17, 34, 68, 128}, over the 64 copies.
    Per entry: us per call, weight GB/s, % of 8 TB/s and the algorithmic bytes (weights,
    activations, outputs) over the measured HBM peak."""
    out = {}
    g = torch.Generator(device=dev)
    g.manual_seed(4242)
    by_shape = {n: [(q, sf, ts) for (nm, _, _, q, sf, ts) in stack if nm == n] for n in S.LAYER_ORDER}

    for key, path in (("single_m1", "auto"), ("single_m1_gemv", "gemv_regs")):
        single = {}
        for name in S.LAYER_ORDER:
            K, N = S.LAYER_SHAPES[name]
            X = torch.randn(1, K, generator=g, device=dev).to(torch.bfloat16)
            Y = torch.empty(1, N, device=dev)
            ws = torch.zeros(max(16, nv.gemm_workspace_bytes(1, N, K)), dtype=torch.uint8, device=dev)
            calls = [lambda q=q, sf=sf, ts=ts: nv.gemm(X, q, sf, ts, out=Y, workspace=ws, path=path)
                     for (q, sf, ts) in by_shape[name]]
            wb = weight_bytes(N, K)
            single[name] = _entry(time_calls(torch, calls, reps), wb, wb + K * 2 + N * 4, peak, N=N, K=K,
                                  copies=len(calls), path=path)
        out[key] = single

    ql, sfl, tsl = lm
    verify = {}
    for N in (S.VOCAB, S.VOCAB_SLICE):
        heads = [(ql[i:i + N], sfl[i:i + N]) for i in range(0, S.VOCAB - N + 1, N)][:4]
        for M in (17, 68):
            B = M // (S.DRAFT_LEN + 1)
            X = torch.randn(M, S.LMHEAD_K, generator=g, device=dev).to(torch.bfloat16)
            drafts = torch.randint(0, N, (B, S.DRAFT_LEN), generator=g, device=dev, dtype=torch.int32)
            o = (torch.empty(M, dtype=torch.int32, device=dev), torch.empty(B, dtype=torch.int32, device=dev),
                 torch.empty(M, dtype=torch.float32, device=dev))
            ws = torch.zeros(nv.verify_workspace_bytes(M, N, S.LMHEAD_K), dtype=torch.uint8, device=dev)
            calls = [lambda q=q, sf=sf: nv.verify(X, q, sf, tsl, drafts, workspace=ws, out=o) for (q, sf) in heads]
            wb = weight_bytes(N, S.LMHEAD_K)
            verify[f"N{N}_M{M}"] = _entry(time_calls(torch, calls, reps * 4), wb, wb + M * S.LMHEAD_K * 2, peak,
                                          N=N, M=M, B=B, copies=len(heads))
    out["verify"] = verify

    K, N = S.LAYER_SHAPES["gate_up"]
    sweep = {}
    for M in S.SWEEP_M:
        X = torch.randn(M, K, generator=g, device=dev).to(torch.bfloat16)
        Y = torch.empty(M, N, device=dev)
        ws = torch.zeros(max(16, nv.gemm_workspace_bytes(M, N, K)), dtype=torch.uint8, device=dev)
        calls = [lambda q=q, sf=sf, ts=ts: nv.gemm(X, q, sf, ts, out=Y, workspace=ws) for (q, sf, ts) in by_shape["gate_up"]]
        wb = weight_bytes(N, K)
        sweep[str(M)] = _entry(time_calls(torch, calls, reps), wb, wb + M * K * 2 + M * N * 4, peak,
                               copies=len(calls))
    out["m_sweep_gate_up"] = sweep
    return out


def run_fp8_extras(nv, torch, dev, peak: float, layers: int, reps: int) -> dict:
    """FP8 weights (E4M3, one fp32 scale per 128 x 128 block) in the pages' precision map: the
    64 qkv projections (5120->10240) and the 248,320-row output head, packed on the GPU from
    seeded N(0, 0.02) weights (4.63 GB, 37 times L2).
      pass_M{17,68}*    one FP8 weight pass over the 64 qkv GEMMs with the head as its verify
                        tail (fp8_pass_run), timed as a CUDA graph, on the f16 kernel and
                        (suffix _terms) on the E4M3-term kernel;
      head_verify_M*    the head's fused verify alone (fp8_lmhead_verify_path), on the f16
                        kernel and (suffix _terms) on the E4M3-term kernel;
      head_gemm_M1*     the head as a plain M=1 GEMM (fp8_gemm_skinny_path), both kernels.
    Per entry: us per call, weight GB/s, % of 8 TB/s and algorithmic bytes over the measured
    HBM peak."""
    K, N = S.LAYER_SHAPES["qkv"]
    qkv = []
    for layer in range(layers):
        g = torch.Generator(device=dev)
        g.manual_seed(7000 + layer)
        W = torch.randn(N, K, generator=g, device=dev).mul_(S.W_STD)
        qkv.append(nv.fp8_pack(W))
        del W
    g = torch.Generator(device=dev)
    g.manual_seed(S.LMHEAD_W_SEED)
    W = torch.randn(S.VOCAB, S.LMHEAD_K, generator=g, device=dev).mul_(S.W_STD)
    qh, sh = nv.fp8_pack(W)
    del W
    torch.cuda.synchronize()
    head_bytes = S.VOCAB * S.LMHEAD_K + sh.numel() * 4
    qkv_bytes = sum(N * K + sc.numel() * 4 for (_, sc) in qkv)
    out = {}
    gx = torch.Generator(device=dev)
    gx.manual_seed(77)
    for M in (17, 68):
        B = M // (S.DRAFT_LEN + 1)
        drafts = torch.zeros((B, S.DRAFT_LEN), dtype=torch.int32, device=dev)
        t = torch.empty(M, dtype=torch.int32, device=dev)
        L = torch.empty(B, dtype=torch.int32, device=dev)
        Xh = torch.randn(M, S.LMHEAD_K, generator=gx, device=dev).to(torch.bfloat16)
        probs = [(torch.randn(M, K, generator=gx, device=dev).to(torch.bfloat16), q, sc,
                  torch.empty((M, N), dtype=torch.bfloat16, device=dev)) for (q, sc) in qkv]
        probs.append((Xh, qh, sh, None))
        wb = qkv_bytes + head_bytes
        alg = wb + M * (K * 2 * layers + S.LMHEAD_K * 2) + M * N * 2 * layers
        for path, tag in (("f16", ""), ("terms", "_terms")):
            p8 = nv.Fp8Pass(probs, M, verify=(drafts, t, L, None), path=path)
            out[f"pass_M{M}{tag}"] = _entry(time_calls(torch, [p8.run], max(3, reps // 2)), wb, alg, peak, M=M,
                                            problems=len(probs), kernel=path)
            del p8
        del probs
        ws = torch.zeros(int(nv.lib().fp8_lmhead_verify_workspace_bytes(M, S.VOCAB, S.LMHEAD_K)), dtype=torch.uint8,
                         device=dev)
        for path, tag in (("f16", ""), ("terms", "_terms")):
            out[f"head_verify_M{M}{tag}"] = _entry(
                time_calls(torch, [lambda path=path: nv.fp8_verify(Xh, qh, sh, drafts, workspace=ws, path=path)],
                           reps * 4), head_bytes, head_bytes + M * S.LMHEAD_K * 2, peak, M=M, kernel=path)
    X1 = torch.randn(1, S.LMHEAD_K, generator=gx, device=dev).to(torch.bfloat16)
    Y1 = torch.empty(1, S.VOCAB, device=dev)
    ws = torch.zeros(int(nv.lib().fp8_gemm_workspace_bytes(1, S.VOCAB, S.LMHEAD_K)), dtype=torch.uint8, device=dev)
    for path, tag in (("f16", ""), ("terms", "_terms")):
        out[f"head_gemm_M1{tag}"] = _entry(
            time_calls(torch, [lambda path=path: nv.fp8_gemm(X1, qh, sh, out=Y1, workspace=ws, path=path)], reps * 4),
            head_bytes, head_bytes + S.LMHEAD_K * 2 + S.VOCAB * 4, peak, M=1, kernel=path)
    del qkv, qh, sh
    torch.cuda.synchronize()
    return {"fp8": out}


def cpu_baseline(seconds: float = 12.0):
    """The oracle, as it stands, on a bounded sample: dequant + float64 GEMM of the
    qkv matrix (5120->10240) at M=17, repeated until ``seconds`` have passed."""
    from oracle import gemm as G
    from oracle import nvfp4 as F
    W, x = S.layer("qkv", M=17)
    q, sf, ts = F.quantize_nvfp4(W)
    reps, t0 = 0, time.perf_counter()
    while True:
        G.gemm_ref(x, q, sf, ts)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    K, N = S.LAYER_SHAPES["qkv"]
    gbs = reps * weight_bytes(N, K) / el / 1e9
    try:
        from threadpoolctl import threadpool_info
        blas = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        blas = None
    cores = len(os.sched_getaffinity(0))
    return {"value": gbs, "unit": "GB/s", "cores": blas or cores, "kind": "oracle",
            "sample": f"{reps} x (dequantise + float64 GEMM) of qkv 5120->10240 at M=17, {el:.1f} s; "
                      f"host has {cores} cores, BLAS threads {blas}"}


def cpu_baseline_fp8(seconds: float = 12.0, rows: int = 4096):
    """The FP8 oracle, as it stands, on a bounded sample of the FP8 head: dequantise + float64
    GEMM of its first ``rows`` rows (K = 5120) at M=17, repeated until ``seconds`` have passed."""
    from oracle import fp8 as P8
    W, x = S.random_case(S.LMHEAD_W_SEED, S.DRAFT_LEN + 1, rows, S.LMHEAD_K)
    codes, scales = P8.quantize_fp8_blocks(W)
    reps, t0 = 0, time.perf_counter()
    while True:
        P8.gemm_fp8_ref(x, codes, scales)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    gbs = reps * (rows * S.LMHEAD_K + scales.size * 4) / el / 1e9
    cores = len(os.sched_getaffinity(0))
    return {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{reps} x (dequantise + float64 GEMM) of a {rows} x {S.LMHEAD_K} FP8 head slice at M=17, "
                      f"{el:.1f} s"}


def max_over_ranks(dist, torch, value: float, dev) -> float:
    """The largest of each rank's device-timed value: the slowest replica sets the step
    time of the whole job. ``dist`` is None on one GPU."""
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(world: int, nbytes: int, ms: float) -> float:
    """Whole-job throughput of ``world`` replicas that each stream ``nbytes`` per step."""
    return world * nbytes / (ms * 1e-3) / 1e9


def run_ours(args, rank, world, local_rank):
    import torch
    import nvfp4_weight_streaming_gemm_b200 as nv
    from nvfp4_weight_streaming_gemm_b200 import build as nvbuild
    nvbuild.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    M_list = [int(m) for m in args.ms.split(",")]
    stack, lm = build_pass(nv, torch, dev, M_list, rank, args.layers)
    head = 17 if 17 in M_list else M_list[0]
    passes = {M: Pass(nv, torch, dev, stack, lm, M, rank, chain=not args.no_chain, tree=args.tree, binv=args.binv,
                      four_terms=args.four_terms)
              for M in M_list}
    for p in passes.values():
        p.capture()
        for _ in range(args.warmup):
            p.g_pass.replay()
            if p.chain:
                p.g_chain.replay()
    torch.cuda.synchronize()

    wbytes = stack_weight_bytes(args.layers) + lmhead_weight_bytes()
    peak, peak_kind = measured_peaks()
    results, clocks = {}, None
    for M, p in passes.items():
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        sampler = ClockSampler(local_rank) if (M == head and rank == 0) else None
        if sampler:
            sampler.start()
        total_ms, per = p.run_timed(args.steps)
        if sampler:
            clocks = sampler.stop()
        total_ms = max_over_ranks(dist, torch, total_ms, dev)
        ms = total_ms / args.steps
        res = {
            "ms_per_pass": ms,
            "weight_gbs": job_gbs(world, wbytes, ms),
            "pct_of_8tbs": 100.0 * wbytes / (ms * 1e-3) / 8e12,
            "passes_per_s": world * 1e3 / ms,
            "alg_gbs": pass_alg_bytes(M, args.layers) / (ms * 1e-3) / 1e9,
            "ms_min": float(per.min()),
            "ms_max": float(per.max()),
            "launches_per_pass": p.launches_pass,
            "B": p.B, "D": p.D, "verify": "tree" if p.tree else "chain", "batch_invariant": p.binv,
            "gemm_activation_terms": 4 if p.four_terms else 5,
        }
        if p.chain:
            # the same work as 193 chained launches: each GEMM's activations are read only
            # after the previous GEMM has finished, as a decode step's layer order requires
            if dist:
                dist.barrier()
            chain_total, _ = p.run_timed(max(3, args.steps // 4), p.g_chain)
            chain_ms = max_over_ranks(dist, torch, chain_total / max(3, args.steps // 4), dev)
            res["chained_ms_per_pass"] = chain_ms
            res["chained_weight_gbs"] = job_gbs(world, wbytes, chain_ms)
        results[M] = res

    # single calls and the standalone verify (the other measurement configurations)
    extras, clocks_extras = None, None
    if not args.no_extras:
        if dist:
            dist.barrier()
        sampler = ClockSampler(local_rank) if rank == 0 else None
        if sampler:
            sampler.start()
        extras = run_extras(nv, torch, dev, stack, lm, peak, reps=max(3, args.steps // 4))
        extras.update(run_fp8_extras(nv, torch, dev, peak, args.layers, reps=max(3, args.steps // 4)))
        if sampler:
            clocks_extras = sampler.stop()

    # end to end through the public API with host buffers (headline M): two host input sets
    # (distinct values each step), two device input buffers, the result read back each step
    p = passes[head]
    p.add_second_input_buffer()
    x_host = [torch.empty(p.x_all.numel(), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    x_host[0].copy_(p.x_all.cpu())
    x_host[1].copy_(x_host[0].flip(0))
    out_host = ([torch.empty(p.M, dtype=torch.int32, pin_memory=True) for _ in range(2)],
                [torch.empty(p.B, dtype=torch.int32, pin_memory=True) for _ in range(2)])
    p.run_e2e(max(2, args.warmup), x_host, out_host)
    if dist:
        dist.barrier()
    e2e_ms = max_over_ranks(dist, torch, p.run_e2e(args.steps, x_host, out_host), dev) / args.steps
    h2d = p.x_all.numel() * 2
    d2h = p.M * 4 + p.B * 4

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    r = results[head]
    line = {
        "metric": METRIC,
        "value": r["weight_gbs"],
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": r["ms_per_pass"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("e2m1*e4m3 weights x bf16 activations (as %s residual e2m1*e4m3 terms) -> f32 accumulate"
                  % ("4 (GEMMs) and 5 (verify)" if args.four_terms else "5")),
        "data": "synthetic (seeded N(0,0.02) weights packed on the GPU, N(0,1) bf16 activations)",
        "config": {"workload": WORKLOAD if args.layers == S.N_LAYERS else
                   WORKLOAD.replace("64 x", f"{args.layers} x") + " (reduced stack: not the benchmark workload)",
                   "M": head, "B": r["B"], "D": r["D"], "layers": args.layers,
                   "weight_bytes_per_pass": wbytes, "l2": "inputs larger than L2 (11.5 GB weight stack, no flush)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "pct_of_8tbs": r["pct_of_8tbs"],
        "passes_per_s": r["passes_per_s"],
        "decode_steps_per_s": r["passes_per_s"],
        "per_m": {str(M): {k: (round(v, 4) if isinstance(v, float) else v) for k, v in res.items()}
                  for M, res in results.items()},
        "roofline": {"bound": "hbm", "kernel": "pass_kernel (one launch per pass; the prep and verify-stage-2 "
                                                 "launches are inside the timed step too)",
                     "achieved": r["alg_gbs"], "peak": peak, "unit": "GB/s",
                     "frac": r["alg_gbs"] / peak, "peak_kind": peak_kind,
                     "traffic": args.traffic if args.traffic is not None else measured_traffic(head, args.layers),
                     "algorithmic_bytes_per_launch": pass_alg_bytes(head, args.layers)},
        "e2e": {"value": job_gbs(world, wbytes, e2e_ms), "unit": "GB/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "what": "every X of the pass copied in from pinned host memory each step (double-buffered: the "
                        "next step's copy runs under the current pass); the verify result read back each step: "
                        "argmax [M] and accept_len [B] int32 (the GEMM outputs stay on the device for the next "
                        "layer)"},
        "gpu_launches": r["launches_per_pass"] * args.steps,
        "clocks": clocks,
    }
    if extras is not None:
        line.update(extras)
        line["clocks_extras"] = clocks_extras
    if not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- per-shape sweep

def run_sweep(args):
    """One matrix shape at several M (and paths), rotating through ``--copies``
    distinct packed copies of the weight so that every launch reads from HBM
    (copies x weight bytes > L2). Prints one JSON line per (M, path). This is the
    M sweep on the gate+up shape, and the small case ncu captures are taken on."""
    import torch
    import nvfp4_weight_streaming_gemm_b200 as nv
    from nvfp4_weight_streaming_gemm_b200 import build as nvbuild
    nvbuild.build()
    dev = torch.device("cuda", 0)
    K, N = S.LAYER_SHAPES[args.shape] if args.shape in S.LAYER_SHAPES else (S.LMHEAD_K, S.VOCAB)
    copies = []
    for i in range(args.copies):
        g = torch.Generator(device=dev)
        g.manual_seed(500 + i)
        W = torch.randn(N, K, generator=g, device=dev).mul_(S.W_STD)
        copies.append(nv.pack(W))
        del W
    peak, peak_kind = measured_peaks()
    for M in [int(m) for m in args.ms.split(",")]:
        X = torch.randn(M, K, device=dev).to(torch.bfloat16)
        Y = torch.empty(M, N, device=dev)
        ws = torch.zeros(max(16, nv.gemm_workspace_bytes(M, N, K)), dtype=torch.uint8, device=dev)
        for path in args.paths.split(","):
            try:
                for i in range(args.warmup):
                    q, sf, ts = copies[i % len(copies)]
                    nv.gemm(X, q, sf, ts, out=Y, workspace=ws, path=path)
            except Exception as e:  # a forced path that does not support this shape
                print(json.dumps({"shape": args.shape, "M": M, "path": path, "skipped": str(e)}), flush=True)
                continue
            torch.cuda.synchronize()
            # capture the launches in a CUDA graph: the replay times the GPU work and the
            # launch gaps a graph-captured pass has, without host-side launch overhead
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(args.steps):
                    q, sf, ts = copies[i % len(copies)]
                    nv.gemm(X, q, sf, ts, out=Y, workspace=ws, path=path)
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            del g
            us = 1e3 * e0.elapsed_time(e1) / args.steps
            alg = weight_bytes(N, K) + M * K * 2 + M * N * 4
            print(json.dumps({"shape": args.shape, "N": N, "K": K, "M": M, "path": path, "us_per_launch": us,
                              "weight_gbs": weight_bytes(N, K) / us / 1e3, "alg_gbs": alg / us / 1e3,
                              "frac_of_peak": alg / us / 1e3 / peak, "peak_kind": peak_kind,
                              "copies": args.copies}), flush=True)


# ----------------------------------------------------------------------------- reference arm

def run_w4a4(args):
    """The W4A4 weight pass at prefill-sized M: the 192 GEMMs of
    the 27B stack with their activations quantised to NVFP4, one persistent launch, timed
    as a CUDA graph. One JSON line per M with the weight GB/s against the HBM roofline and
    the tensor TFLOP/s against the fp4 peak (measured bf16 x 4, the nominal fp4/bf16
    ratio)."""
    import torch
    import nvfp4_weight_streaming_gemm_b200 as nv
    from nvfp4_weight_streaming_gemm_b200 import build as nvbuild
    nvbuild.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    M_list = [int(m) for m in args.ms.split(",")]
    stack, _ = build_pass(nv, torch, dev, M_list, 0, args.layers)
    wbytes = stack_weight_bytes(args.layers)
    flop_per_m = 2.0 * sum(N * K for (_, K, N, _, _, _) in stack)
    hbm, hbm_kind = measured_peaks()
    bf16, pk = 1590.0, os.path.join(ROOT, "MEASURED_PEAKS.json")     # the recipe's fallback when absent
    if os.path.exists(pk):
        with open(pk) as f:
            bf16 = float(json.load(f).get("bf16_tflops", bf16))
    fp4_peak = 4.0 * bf16
    for M in M_list:
        g = torch.Generator(device=dev)
        g.manual_seed(11 + M)
        probs = [(torch.randn(M, K, generator=g, device=dev).to(torch.bfloat16), q, sf, ts,
                  torch.empty((M, N), dtype=torch.bfloat16, device=dev)) for (_, K, N, q, sf, ts) in stack]
        wp = nv.WeightPass(probs, M, w4a4=True)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            wp.run(s)
        torch.cuda.current_stream().wait_stream(s)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            wp.run()
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()
        st = torch.cuda.current_stream()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        ev[0].record(st)
        for k in range(args.steps):
            graph.replay()
            ev[k + 1].record(st)
        torch.cuda.synchronize()
        per = np.array([ev[k].elapsed_time(ev[k + 1]) for k in range(args.steps)])
        ms = ev[0].elapsed_time(ev[-1]) / args.steps
        tflops = flop_per_m * M / (ms * 1e-3) / 1e12
        print(json.dumps({
            "metric": "W4A4 27B weight pass (NVFP4 activations, prefill-sized M)", "M": M, "layers": args.layers,
            "ms_per_pass": ms, "ms_min": float(per.min()), "weight_gbs": wbytes / (ms * 1e-3) / 1e9,
            "hbm_frac": wbytes / (ms * 1e-3) / 1e9 / hbm, "hbm_peak_kind": hbm_kind,
            "tflops": tflops, "fp4_peak_tflops": fp4_peak, "tensor_frac": tflops / fp4_peak,
            "y_dtype": "bf16", "steps": args.steps, "warmup": args.warmup}), flush=True)
        del graph, wp, probs
        torch.cuda.synchronize()


def run_fp8(args):
    """The FP8 output head: E4M3 codes with one fp32 scale per 128 x 128 block over the
    full 248,320 x 5120 vocabulary (1.27 GB, ten times L2), packed on the GPU from a seeded
    N(0, 0.02) weight. Per M, the fused verify (M a multiple of 17: B sequences of 16 drafts
    + 1) and the plain GEMM, each timed by CUDA events over `steps` calls after `warmup`.
    One JSON line per (call, M) with the weight GB/s against the HBM roofline."""
    import torch
    import nvfp4_weight_streaming_gemm_b200 as nv
    from nvfp4_weight_streaming_gemm_b200 import build as nvbuild
    nvbuild.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    N, K = args.fp8_rows, S.LMHEAD_K
    g = torch.Generator(device=dev)
    g.manual_seed(S.LMHEAD_W_SEED)
    W = torch.randn(N, K, generator=g, device=dev) * S.W_STD
    q, sc = nv.fp8_pack(W)
    del W
    wbytes = N * K + sc.numel() * 4
    hbm, hbm_kind = measured_peaks()
    st = torch.cuda.current_stream()
    cpu = None if args.no_cpu_baseline else cpu_baseline_fp8(args.cpu_seconds)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        ev[0].record(st)
        for k in range(args.steps):
            fn()
            ev[k + 1].record(st)
        torch.cuda.synchronize()
        nv.check()
        per = np.array([ev[k].elapsed_time(ev[k + 1]) for k in range(args.steps)])
        return ev[0].elapsed_time(ev[-1]) / args.steps, float(per.min())

    for M in [int(m) for m in args.ms.split(",")]:
        X = torch.randn(M, K, generator=g, device=dev).to(torch.bfloat16)
        calls = []
        if M % (S.DRAFT_LEN + 1) == 0:
            B = M // (S.DRAFT_LEN + 1)
            drafts = torch.zeros((B, S.DRAFT_LEN), dtype=torch.int32, device=dev)
            wsv = torch.zeros(int(nv.lib().fp8_lmhead_verify_workspace_bytes(M, N, K)), dtype=torch.uint8, device=dev)
            calls.append(("verify", lambda: nv.fp8_verify(X, q, sc, drafts, workspace=wsv, path=args.fp8_path)))
        Y = torch.empty((M, N), dtype=torch.float32, device=dev)
        wsg = torch.zeros(int(nv.lib().fp8_gemm_workspace_bytes(M, N, K)), dtype=torch.uint8, device=dev)
        calls.append(("gemm", lambda: nv.fp8_gemm(X, q, sc, out=Y, workspace=wsg, path=args.fp8_path)))
        for name, fn in calls:
            ms, ms_min = timed(fn)
            gbs = wbytes / (ms * 1e-3) / 1e9
            print(json.dumps({
                "metric": f"FP8 lm_head {name} (E4M3, 128x128 fp32 block scales)", "M": M, "N": N, "K": K,
                "fp8_path": args.fp8_path,
                "ms": ms, "ms_min": ms_min, "weight_gbs": gbs, "hbm_frac": gbs / hbm, "hbm_peak_kind": hbm_kind,
                "steps": args.steps, "warmup": args.warmup, "cpu_baseline": cpu}), flush=True)


def run_mixed(args):
    """The pages' precision map for the 27B step: per layer the gate+up and down projections
    in NVFP4 and the qkv projection in FP8 (E4M3, 128x128 fp32 block scales), then an FP8
    lm_head with the fused verify. One NVFP4 pass (128 GEMMs) and one FP8 pass (64 GEMMs and
    the head), captured together in one CUDA graph and timed by CUDA events. One JSON line per
    M with the weight GB/s against the HBM roofline."""
    import torch
    import nvfp4_weight_streaming_gemm_b200 as nv
    from nvfp4_weight_streaming_gemm_b200 import build as nvbuild
    nvbuild.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    nv4, f8 = [], []
    for layer in range(args.layers):
        for j, name in enumerate(S.LAYER_ORDER):
            K, N = S.LAYER_SHAPES[name]
            g = torch.Generator(device=dev)
            g.manual_seed(1000 * layer + j)
            W = torch.randn(N, K, generator=g, device=dev, dtype=torch.float32).mul_(S.W_STD)
            if name == "qkv":
                f8.append((K, N) + nv.fp8_pack(W))
            else:
                nv4.append((K, N) + nv.pack(W))
            del W
    g = torch.Generator(device=dev)
    g.manual_seed(S.LMHEAD_W_SEED)
    W = torch.randn(S.VOCAB, S.LMHEAD_K, generator=g, device=dev, dtype=torch.float32).mul_(S.W_STD)
    qh, sh = nv.fp8_pack(W)
    del W
    torch.cuda.synchronize()
    wbytes = (sum(weight_bytes(N, K) for (K, N, _, _, _) in nv4) +
              sum(N * K + sc.numel() * 4 for (K, N, _, sc) in f8) + S.VOCAB * S.LMHEAD_K + sh.numel() * 4)
    hbm, hbm_kind = measured_peaks()
    st = torch.cuda.current_stream()
    for M in [int(m) for m in args.ms.split(",")]:
        B = max(1, M // (S.DRAFT_LEN + 1))
        D = M // B - 1
        if B * (D + 1) != M:
            raise SystemExit(f"--mixed: M={M} is not B*(D+1)")
        gx = torch.Generator(device=dev)
        gx.manual_seed(11 + M)
        p4 = nv.WeightPass([(torch.randn(M, K, generator=gx, device=dev).to(torch.bfloat16), q, sf, ts,
                             torch.empty((M, N), dtype=torch.bfloat16, device=dev)) for (K, N, q, sf, ts) in nv4], M)
        drafts = torch.zeros((B, D), dtype=torch.int32, device=dev)
        t = torch.empty(M, dtype=torch.int32, device=dev)
        L = torch.empty(B, dtype=torch.int32, device=dev)
        probs8 = [(torch.randn(M, K, generator=gx, device=dev).to(torch.bfloat16), q, sc,
                   torch.empty((M, N), dtype=torch.bfloat16, device=dev)) for (K, N, q, sc) in f8]
        probs8.append((torch.randn(M, S.LMHEAD_K, generator=gx, device=dev).to(torch.bfloat16), qh, sh, None))
        p8 = nv.Fp8Pass(probs8, M, verify=(drafts, t, L, None), path=args.fp8_path)
        s = torch.cuda.Stream()
        s.wait_stream(st)
        with torch.cuda.stream(s):
            p4.run(s)
            p8.run(s)
        st.wait_stream(s)
        torch.cuda.synchronize()
        nv.check()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            p4.run()
            p8.run()
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        ev[0].record(st)
        for k in range(args.steps):
            graph.replay()
            ev[k + 1].record(st)
        torch.cuda.synchronize()
        nv.check()
        per = np.array([ev[k].elapsed_time(ev[k + 1]) for k in range(args.steps)])
        ms = ev[0].elapsed_time(ev[-1]) / args.steps
        gbs = wbytes / (ms * 1e-3) / 1e9
        print(json.dumps({
            "metric": "27B step with the pages' precision map (NVFP4 MLP, FP8 qkv and lm_head verify)", "M": M,
            "layers": args.layers, "fp8_kernel": args.fp8_path, "ms_per_step": ms, "ms_min": float(per.min()),
            "weight_bytes": wbytes,
            "weight_gbs": gbs, "hbm_frac": gbs / hbm, "hbm_peak_kind": hbm_kind, "y_dtype": "bf16",
            "steps": args.steps, "warmup": args.warmup}), flush=True)
        del graph, p4, p8, probs8
        torch.cuda.synchronize()


def run_reference(args, rank, world):
    """The CPU oracle timed as it stands: each step dequantises and multiplies one qkv
    matrix (5120->10240) in float64 at M=17. That is a bounded sample of the pass, in
    the same unit (weight GB/s)."""
    if rank != 0:
        return
    from oracle import gemm as G
    from oracle import nvfp4 as F
    W, x = S.layer("qkv", M=17)
    q, sf, ts = F.quantize_nvfp4(W)
    for _ in range(args.warmup):
        G.gemm_ref(x, q, sf, ts)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        G.gemm_ref(x, q, sf, ts)
    el = time.perf_counter() - t0
    K, N = S.LAYER_SHAPES["qkv"]
    gbs = args.steps * weight_bytes(N, K) / el / 1e9
    cores = len(os.sched_getaffinity(0))
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD + " -- sampled: one qkv matrix per step", "M": 17},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": "one qkv 5120->10240 dequant + float64 GEMM at M=17 per step"},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--ms", default="17,1,68", help="comma list of M; the first 17 (else the first) is the headline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-chain", action="store_true", help="skip the chained per-GEMM comparison")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the single-call, standalone-verify and M-sweep entries of the default line")
    ap.add_argument("--layers", type=int, default=S.N_LAYERS,
                    help="layers in the stack (the default is the 27B model's; fewer only for small profiling cases)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per pass_kernel launch (default: the stored ncu capture in profiles/, "
                         "when the kernel sources still match it)")
    ap.add_argument("--tree", action="store_true",
                    help="verify draft trees of D nodes per sequence (seeded random parents) instead of chains")
    ap.add_argument("--binv", action="store_true", help="batch-invariant passes (same row bits for every M)")
    ap.add_argument("--four-terms", action="store_true",
                    help="GEMMs on four residual activation terms (NVFP4WS_PASS_FOUR_TERMS; the verify keeps five)")
    ap.add_argument("--w4a4", action="store_true",
                    help="time W4A4 passes (NVFP4 activations) over the stack at the --ms values, e.g. 128,256")
    ap.add_argument("--mixed", action="store_true",
                    help="the 27B step with NVFP4 MLP weights and an FP8 qkv projection and lm_head")
    ap.add_argument("--fp8", action="store_true",
                    help="the FP8 (E4M3, 128x128 block-scaled) output head: verify and GEMM per M")
    ap.add_argument("--fp8-rows", type=int, default=S.VOCAB,
                    help="rows of the FP8 head for --fp8 (fewer only for small profiling cases)")
    ap.add_argument("--fp8-path", choices=["f16", "terms"], default="f16",
                    help="FP8 kernel: codes dequantised to f16, or straight into the FP8 tensor cores")
    ap.add_argument("--sweep", action="store_true", help="time one matrix shape per M and path (no pass)")
    ap.add_argument("--shape", default="gate_up", help="sweep shape: gate_up, down, qkv or lm_head")
    ap.add_argument("--paths", default="auto,gemv,mma")
    ap.add_argument("--copies", type=int, default=4)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.sweep:
        run_sweep(args)
    elif args.w4a4:
        run_w4a4(args)
    elif args.fp8:
        run_fp8(args)
    elif args.mixed:
        run_mixed(args)
    elif args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
