"""Benchmark: compressed-KV decode attention on B200 (one JSON line on rank 0).

Workload (default ``llama8b``): Llama-3.1-8B-shaped decode, batch 1, 32 query /
8 KV heads, head_dim 128, 32768 cached tokens per layer in 16-token pages, keys
3-bit + QJL (m = 128), values 2-bit, 32 layers. One step = one generated token:
for each of the 32 layers, one tq_decode_step call quantizes and appends the new
token's K/V (8 heads) and runs decode attention for the 32 query heads over the
whole cache (one kernel launch per layer: the CTA that owns the sequence's last page
quantizes the new token while the other CTAs already stream their pages). The 32 layer
caches (about 0.86 GB) exceed the 126 MB L2, so every step streams from HBM.

``value``   decode tokens/s with inputs resident in HBM (CUDA-graph replay of
            K steps, CUDA events on the launching stream, max over ranks).
``e2e``     the same steps through the C ABI with host buffers: per step the
            new K/V and queries are copied from pinned host memory and the
            attention outputs copied back, inside the timed region. The copies
            run on a second stream and overlap the layers' work (layer 0's
            inputs first; each layer's outputs as soon as it ends), checked
            against the same steps with every copy in line.
``roofline`` the kernel the timed step launches (decode_kernel via
            tq_decode_step: append, query transform, split-K decode and merge,
            once per layer) against the measured HBM copy bandwidth: algorithmic
            bytes = compressed bytes of every cached token-head read (102 B each)
            over its mean launch time in the timed replays. ``roofline_attention``
            is the same for tq_decode_attention (no append) at the final context.
``parity``  a sampled oracle check of the bench's own cache after the timed
            steps (appended tokens' codes, signs and norms; decode outputs of a few
            (sequence, KV head) pairs over the full context).
``cpu_baseline`` the float64 oracle on the host, on a bounded sample.

Multi-GPU: one process per GPU (torchrun); each rank serves its own sequence
(weak scaling, no collective on the data path); value = all ranks' tokens /
slowest rank's time.
"""

import argparse
import re
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "compressed-KV decode attention tokens/s & HBM GB/s vs roofline; quantize GB/s"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_hash():
    """Hash of the library's code with comments and whitespace removed, so that a
    recorded ncu measurement stays tied to the code it was taken on, not its comments."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "decode_attention_seeded_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if not f.endswith((".cu", ".cuh", ".cpp", ".h")):
            continue
        src = open(os.path.join(csrc, f)).read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update("".join(src.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kind):
    """Per-launch DRAM bytes from the committed ncu summary, if it matches these sources."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("source_hash") != kernel_source_hash():
        return None
    return d.get(kind)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Polls SM clock and throttle reasons through NVML while the GPU works."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _handle(self, device_index):
        import torch
        nv = self.nv
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            return nv.nvmlDeviceGetHandleByUUID(uuid.encode())
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(device_index)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------- GPU workload
class DecodeBench:
    L2_BYTES = 126e6

    def __init__(self, wl, steps, warmup, device, rank, sparse_v=0.0, peaked=False):
        import torch
        from decode_attention_seeded_b200 import binding, synth
        self.torch, self.binding, self.synth = torch, binding, synth
        self.wl, self.dev = wl, device
        self.steps, self.warmup = steps, warmup
        gen0 = synth.Generator(wl, layer=0)
        self.seeds = gen0.method_seeds()
        self.ctx = binding.Context(wl.key_bits, wl.value_bits, self.seeds, device=device.index)
        self.ctx.set_sparse_v(sparse_v)
        n_kv, nq, B = wl.n_kv_heads, wl.n_q_heads, wl.batch
        self.lens0 = gen0.seq_lens().astype(np.int64)            # cached tokens per sequence before step 0
        self.T0 = int(self.lens0[0])
        self.total_steps = warmup + steps
        self.max_len = int(self.lens0.max()) + self.total_steps
        pages = (self.lens0 + self.total_steps + 15) // 16
        bpt = self.ctx.block_bytes // 16
        per_layer = int(np.sum(self.lens0)) * n_kv * bpt
        # rotate through enough layer caches that they exceed the L2 several times over
        self.n_layers = bench_layers(wl, self.ctx.block_bytes, self.L2_BYTES)
        assert per_layer > 0
        self.page_bytes = self.ctx.page_bytes(n_kv)
        self.caches, self.btabs = [], []
        g = torch.Generator(device=device)
        self.newk = torch.empty((self.n_layers, self.total_steps, B, n_kv, 128), dtype=torch.bfloat16,
                                device=device)
        self.newv = torch.empty_like(self.newk)
        self.q = (torch.randn((self.total_steps, self.n_layers, B, nq, 128), generator=g, device=device)
                  .to(torch.bfloat16))
        for layer in range(self.n_layers):
            gen = synth.Generator(wl, layer=layer)
            bt, n_pages = gen.page_pool(pages)
            cache = torch.empty(n_pages * self.page_bytes, dtype=torch.uint8, device=device)
            btt = torch.from_numpy(bt).to(device)
            g.manual_seed(wl.seed * 1000 + layer + 7919 * rank)
            sk = torch.from_numpy(gen.scales["k"]).float().to(device)
            sv = torch.from_numpy(gen.scales["v"]).float().to(device)
            for b in range(B):
                L = int(self.lens0[b])
                k = (torch.randn((L + self.total_steps, n_kv, 128), generator=g, device=device) * sk).to(torch.bfloat16)
                v = (torch.randn((L + self.total_steps, n_kv, 128), generator=g, device=device) * sv).to(torch.bfloat16)
                self.ctx.quantize_prefill(k[:L], v[:L], btt[b], 0, cache, n_pages)
                self.newk[layer, :, b] = k[L:]
                self.newv[layer, :, b] = v[L:]
                if peaked:
                    # concentrated attention: each query is 5 x the sum of the unit
                    # directions of 3 cached keys of its KV head
                    idx = torch.randint(0, L, (self.total_steps, nq, 3), generator=g, device=device)
                    hk = (torch.arange(nq, device=device) // (nq // n_kv)).view(1, nq, 1).expand_as(idx)
                    kk = k[idx, hk].float()
                    kk = kk / kk.norm(dim=-1, keepdim=True)
                    self.q[:, layer, b] = (5.0 * kk.sum(dim=2)).to(torch.bfloat16)
                del k, v
            self.caches.append((cache, n_pages))
            self.btabs.append(btt)
        torch.cuda.synchronize(device)
        steps_ar = torch.arange(1, self.total_steps + 1, dtype=torch.int64).reshape(-1, 1)
        self.lens = (torch.from_numpy(self.lens0).reshape(1, -1) + steps_ar).to(torch.int32).to(device)
        self.out = torch.zeros((self.n_layers, B, nq, 128), dtype=torch.float32, device=device)
        self.ws_bytes = self.ctx.decode_workspace_bytes(B, nq, n_kv, self.max_len)
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=device)
        # host-side buffers for the end-to-end arm: per step and layer the new K, the
        # new V and the queries back to back, so that one copy moves any run of layers
        self.n_k, self.n_qe = B * n_kv * 128, B * nq * 128
        row = 2 * self.n_k + self.n_qe
        self.h_in = torch.empty((self.total_steps, self.n_layers, row), dtype=torch.bfloat16, pin_memory=True)
        nk = self.n_k
        self.h_in[:, :, :nk].copy_(self.newk.transpose(0, 1).reshape(self.total_steps, self.n_layers, nk).cpu())
        self.h_in[:, :, nk:2 * nk].copy_(self.newv.transpose(0, 1).reshape(self.total_steps, self.n_layers, nk).cpu())
        self.h_in[:, :, 2 * nk:].copy_(self.q.reshape(self.total_steps, self.n_layers, self.n_qe).cpu())
        self.h_out = torch.empty((self.total_steps, self.n_layers, B, nq, 128), dtype=torch.float32,
                                 pin_memory=True)
        self.d_in = torch.empty((self.n_layers, row), dtype=torch.bfloat16, device=device)
        self.copy_stream = torch.cuda.Stream(device=device)
        self.ev_in, self.ev_out = torch.cuda.Event(), (torch.cuda.Event(), torch.cuda.Event())

    @property
    def cache_tokens(self):
        """Cached tokens read by one decode call at the final step (all sequences)."""
        return int(np.sum(self.lens0)) + self.wl.batch * self.total_steps

    # one decode step (all layers) with inputs already on the device
    def step(self, s):
        wl = self.wl
        for layer in range(self.n_layers):
            cache, n_pages = self.caches[layer]
            self.ctx.decode_step(self.newk[layer, s], self.newv[layer, s], self.q[s, layer], cache,
                                 n_pages, self.btabs[layer], self.lens[s], wl.n_kv_heads, self.max_len,
                                 self.out[layer], self.ws)

    # the same step through host buffers, copies overlapped with the layers' work.
    # Layer 0's inputs are copied on the launching stream; the other layers'
    # inputs follow on a copy stream (layer 1 waits for them) while layer 0 runs.
    # The outputs of all but the last two layers go back on the copy stream while
    # those two run; the last two layers' outputs end the step.
    def step_e2e(self, s):
        torch = self.torch
        main, cs = torch.cuda.current_stream(self.dev), self.copy_stream
        n = self.n_layers
        split = max(n - 2, 0)
        self.d_in[0].copy_(self.h_in[s, 0], non_blocking=True)
        cs.wait_stream(main)                  # after layer 0's copy and the previous step
        with torch.cuda.stream(cs):
            if n > 1:
                self.d_in[1:].copy_(self.h_in[s, 1:], non_blocking=True)
            self.ev_in.record(cs)
        for layer in range(n):
            if layer == 1:
                main.wait_event(self.ev_in)
            self.decode_layer_e2e(layer, s)
            for a, b, ev in ((0, split, self.ev_out[0]), (split, n, self.ev_out[1])):
                if layer == b - 1:
                    ev.record(main)
                    with torch.cuda.stream(cs):
                        cs.wait_event(ev)
                        self.h_out[s, a:b].copy_(self.out[a:b], non_blocking=True)
        main.wait_stream(cs)

    # the same step through host buffers, every copy in line with the layers (the
    # order check of the overlapped step compares against it)
    def step_e2e_serial(self, s):
        self.d_in.copy_(self.h_in[s], non_blocking=True)
        for layer in range(self.n_layers):
            self.decode_layer_e2e(layer, s)
        self.h_out[s].copy_(self.out, non_blocking=True)

    def decode_layer_e2e(self, layer, s):
        wl, nk = self.wl, self.n_k
        cache, n_pages = self.caches[layer]
        k = self.d_in[layer, :nk].view(wl.batch, wl.n_kv_heads, 128)
        v = self.d_in[layer, nk:2 * nk].view(wl.batch, wl.n_kv_heads, 128)
        q = self.d_in[layer, 2 * nk:].view(wl.batch, wl.n_q_heads, 128)
        self.ctx.decode_step(k, v, q, cache, n_pages, self.btabs[layer], self.lens[s], wl.n_kv_heads,
                             self.max_len, self.out[layer], self.ws)

    def e2e_bytes(self):
        """Bytes the end-to-end step copies in (h_in[s]) and out (h_out[s])."""
        return (self.h_in[0].numel() * self.h_in.element_size(),
                self.h_out[0].numel() * self.h_out.element_size())

    def capture(self, fn, steps):
        torch = self.torch
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(device=self.dev)
        s.wait_stream(torch.cuda.current_stream(self.dev))
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for i in steps:
                    fn(i)
        torch.cuda.current_stream(self.dev).wait_stream(s)
        return g

    def graph_seconds(self, calls, reps=1):
        """Device seconds per call of `calls` (zero-argument callables that launch
        work on the current stream), each run once eagerly (library set-up, first-use
        allocations), then `reps` times over captured in one CUDA graph, replayed once
        untimed and timed on one more replay with CUDA events: the host's launch
        overhead stays out of the figure, as it does for the decode steps."""
        torch = self.torch
        for c in calls:
            c()
        torch.cuda.synchronize(self.dev)
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(device=self.dev)
        s.wait_stream(torch.cuda.current_stream(self.dev))
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for _ in range(reps):
                    for c in calls:
                        c()
        torch.cuda.current_stream(self.dev).wait_stream(s)
        g.replay()
        torch.cuda.synchronize(self.dev)
        t = timed(torch, self.dev, g.replay)
        del g
        return t / (reps * len(calls))

    def quantize_timing(self, reps=6):
        """Quantize-prefill of one layer's full context (K and V of every KV head).

        Algorithmic bytes = the K/V inputs read + the compressed blocks written.
        Layers rotate so that the inputs (0.13 GB per layer) are not L2-resident."""
        torch, wl = self.torch, self.wl
        n_kv = wl.n_kv_heads
        g = torch.Generator(device=self.dev)
        g.manual_seed(wl.seed * 7 + 11)
        bufs = []
        for i in range(2):
            gen = self.synth.Generator(wl, layer=i)
            sc = torch.from_numpy(gen.scales["k"]).float().to(self.dev)
            k = (torch.randn((self.T0, n_kv, 128), generator=g, device=self.dev) * sc).to(torch.bfloat16)
            v = (torch.randn((self.T0, n_kv, 128), generator=g, device=self.dev) * sc).to(torch.bfloat16)
            bufs.append((k, v))
        cache, n_pages = self.caches[0]
        bt = self.btabs[0][0]
        calls = [lambda k=k, v=v: self.ctx.quantize_prefill(k, v, bt, 0, cache, n_pages) for k, v in bufs]
        secs = self.graph_seconds(calls, reps=reps // 2)
        bytes_in = 2 * self.T0 * n_kv * 128 * 2
        bytes_out = self.T0 * n_kv * (self.ctx.block_bytes // 16)
        return {"gbs": (bytes_in + bytes_out) / secs / 1e9, "us_per_call": secs * 1e6,
                "tokens": self.T0, "kv_heads": n_kv, "bytes_in": bytes_in, "bytes_out": bytes_out,
                "timing": f"CUDA graph of {reps} calls on two alternating input buffers",
                "kernel": "quantize_prefill_tc_kernel via tq_quantize_prefill (bf16 K/V, one layer)"}

    def logits_timing(self, reps=10):
        """Logits only (tq_decode_logits) against logits from full-precision fp32 keys.

        The pages compare attention-logit speed on compressed keys with 32-bit keys.
        Ours reads the key codes, sign bits and norms of every cached token-head and
        writes fp32 logits; the comparison is one cuBLAS batched product of the
        queries with an fp32 key cache of the same shape. Both rotate over the layer
        caches, so both stream from HBM."""
        torch, wl = self.torch, self.wl
        n_kv, nq, B, T = wl.n_kv_heads, wl.n_q_heads, wl.batch, self.max_len
        g = nq // n_kv
        last = self.total_steps - 1
        out = torch.empty((B, nq, T), dtype=torch.float32, device=self.dev)

        def run_ours(layer):
            cache, n_pages = self.caches[layer]
            self.ctx.decode_logits(self.q[last, layer], cache, n_pages, self.btabs[layer], self.lens[last], n_kv,
                                   T, out)

        def time_it(fn, layers):
            return self.graph_seconds([lambda layer=layer: fn(layer) for layer in range(layers)], reps=reps)

        ours = time_it(run_ours, self.n_layers)
        key_bytes = self.cache_tokens * n_kv * key_bytes_per_token(wl.key_bits)
        res = {"kernel": "decode_kernel (logits mode) via tq_decode_logits", "us_per_layer": ours * 1e6,
               "timing": f"CUDA graph of {reps} passes over the layer caches (both arms)",
               "key_bytes_per_layer": key_bytes, "gbs": key_bytes / ours / 1e9,
               "logit_bytes_written": nq * int(self.lens[last].sum().item()) * 4}
        try:
            gen = torch.Generator(device=self.dev)
            gen.manual_seed(5)
            k32 = [torch.randn((B, n_kv, T, 128), generator=gen, device=self.dev) for _ in range(self.n_layers)]
            q32 = self.q[last].float().view(self.n_layers, B, n_kv, g, 128)
            o32 = torch.empty((B, n_kv, g, T), dtype=torch.float32, device=self.dev)
            fp32 = time_it(lambda layer: torch.matmul(q32[layer], k32[layer].transpose(-1, -2), out=o32),
                           self.n_layers)
            b32 = B * n_kv * T * 128 * 4
            res.update({"fp32_keys": f"torch {torch.__version__} matmul (cuBLAS), fp32 keys",
                        "fp32_keys_us_per_layer": fp32 * 1e6, "fp32_key_bytes_per_layer": b32,
                        "fp32_keys_gbs": b32 / fp32 / 1e9, "speedup_vs_fp32_keys": fp32 / ours,
                        "key_bytes_ratio": b32 / key_bytes})
            del k32
            torch.cuda.empty_cache()
        except Exception as e:                       # comparison unavailable
            res["fp32_keys_error"] = repr(e)[:200]
        return res

    def bf16_baseline(self, reps=3):
        """Decode attention over an uncompressed bf16 KV cache of the same shape (context only).

        The faster of flash-attention's KV-cache decode and PyTorch SDPA (GQA), timed
        over the same number of layer caches as the compressed path, so that the
        caches stream from HBM. Library kernels: a comparison point, not this path."""
        torch, wl = self.torch, self.wl
        n_kv, nq, T, B = wl.n_kv_heads, wl.n_q_heads, self.max_len, wl.batch
        g = torch.Generator(device=self.dev)
        g.manual_seed(99)
        layers = self.n_layers
        kc = [torch.randn((B, T, n_kv, 128), generator=g, device=self.dev).to(torch.bfloat16) for _ in range(layers)]
        vc = [torch.randn((B, T, n_kv, 128), generator=g, device=self.dev).to(torch.bfloat16) for _ in range(layers)]
        q = torch.randn((B, 1, nq, 128), generator=g, device=self.dev).to(torch.bfloat16)
        lens = self.lens[-1]                          # final step's lengths (int32, per sequence)
        ragged = bool((lens != lens[0]).any())
        st = torch.cuda.current_stream(self.dev)
        results, errors, timing = {}, {}, {}

        def time_it(fn, name):
            # a CUDA graph like the compressed path; eager launches if the library
            # call cannot be captured
            try:
                t = self.graph_seconds([lambda layer=layer: fn(layer) for layer in range(layers)], reps=reps)
                timing[name] = "cuda graph"
                return t
            except Exception as e:
                errors[name + " (graph capture)"] = repr(e)[:200]
                torch.cuda.synchronize(self.dev)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(st)
            for _ in range(reps):
                for layer in range(layers):
                    fn(layer)
            b.record(st)
            b.synchronize()
            timing[name] = "eager"
            return a.elapsed_time(b) / 1e3 / (reps * layers)

        try:
            from flash_attn import __version__ as fav
            from flash_attn import flash_attn_with_kvcache
            name = f"flash_attn {fav} flash_attn_with_kvcache"
            results[name] = time_it(lambda l: flash_attn_with_kvcache(q, kc[l], vc[l], cache_seqlens=lens), name)
        except Exception as e:                       # library kernel unavailable on this build
            errors["flash_attn"] = repr(e)[:200]
        try:
            if ragged:
                raise ValueError("ragged lengths: SDPA would attend the padding")
            import torch.nn.functional as F
            qs = q.transpose(1, 2)                   # [B, nq, 1, 128]
            kt = [k.transpose(1, 2) for k in kc]
            vt = [v.transpose(1, 2) for v in vc]
            name = f"torch {torch.__version__} scaled_dot_product_attention (enable_gqa)"
            results[name] = time_it(lambda l: F.scaled_dot_product_attention(qs, kt[l], vt[l], enable_gqa=True), name)
        except Exception as e:
            errors["sdpa"] = repr(e)[:200]
        del kc, vc
        torch.cuda.empty_cache()
        if not results:
            return {"unavailable": errors}
        name, secs = min(results.items(), key=lambda kv: kv[1])
        nbytes = 2 * int(lens.sum().item()) * n_kv * 128 * 2
        return {"kernel": name, "us_per_layer": secs * 1e6, "bytes_per_layer": nbytes,
                "gbs": nbytes / secs / 1e9, "all_us": {k: v * 1e6 for k, v in results.items()},
                "timing": timing, "errors": errors or None}

    def decode_only_graph(self, reps):
        """reps x (32 layers of tq_decode_attention) at the final context length."""
        wl = self.wl
        last = self.total_steps - 1

        def body(_):
            for layer in range(self.n_layers):
                cache, n_pages = self.caches[layer]
                self.ctx.decode_attention(self.q[last, layer], cache, n_pages, self.btabs[layer], self.lens[last],
                                          wl.n_kv_heads, self.max_len, self.out[layer], self.ws)
        return self.capture(body, range(reps))


def key_bytes_per_token(key_bits):
    """Key bytes one token-head contributes to its logits: q8_0 = 128 int8 values + 4 fp16
    block scales; TurboQuant = b-bit codes + 128 sign bits + fp16 norm and residual norm."""
    return 136 if key_bits == 8 else 16 * key_bits + 16 + 4


def key_format(key_bits):
    return "q8_0 keys" if key_bits == 8 else f"{key_bits}-bit keys + QJL"


def max_over_ranks(x, world, device):
    """The largest of the ranks' values (every rank gets it); x itself when world == 1."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, seconds):
    """Whole-job rate: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / seconds


def timed(torch, dev, fn):
    st = torch.cuda.current_stream(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    a.record(st)
    fn()
    b.record(st)
    b.synchronize()
    return a.elapsed_time(b) / 1e3


def bench_layers(wl, block_bytes, l2_bytes=126e6):
    """Layer caches the bench rotates through: the workload's layers, or more, so that
    they exceed the L2 four times over (at most 64)."""
    per_layer = int(np.sum(seq_lens_of(wl))) * wl.n_kv_heads * (block_bytes // 16)
    return max(wl.n_layers, min(64, int(np.ceil(4 * l2_bytes / per_layer))))


def seq_lens_of(wl):
    from decode_attention_seeded_b200 import synth
    return synth.Generator(wl, layer=0).seq_lens().astype(np.int64)


def block_bytes_of(wl):
    """Bytes of one (page, KV head) block (include/tq.h): 16 tokens x per-token bytes."""
    if wl.key_bits == 8:
        return 16 * (128 + 8 + 16 * wl.value_bits + 2)
    return 16 * (16 * wl.key_bits + 16 + 4 + 16 * wl.value_bits + 2)


def workload_config(wl, world, steps, warmup, sparse_v=0.0, peaked=False):
    """The `config` object of the JSON line; both arms print the same one."""
    bb = block_bytes_of(wl)
    lens0 = seq_lens_of(wl)
    layers = bench_layers(wl, bb)
    pages = (lens0 + steps + warmup + 15) // 16
    step_bytes = layers * int(np.sum(pages) + 3) * wl.n_kv_heads * bb
    return {"workload": wl.name, "batch": wl.batch, "q_heads": wl.n_q_heads, "kv_heads": wl.n_kv_heads,
            "head_dim": 128, "context": wl.context, "context_lens": [int(x) for x in lens0[:16]],
            "layers": layers, "key_bits": wl.key_bits, "value_bits": wl.value_bits,
            "qjl_rows": 0 if wl.key_bits == 8 else 128, "page_tokens": 16,
            "l2": f"inputs larger than L2: {layers} layer caches, about {step_bytes / 1e9:.2f} GB per step",
            "parallelism": f"replica x{world} (each GPU serves its own batch)",
            "sparse_v": sparse_v, "queries": "peaked (5 x 3 cached key directions)" if peaked else "N(0,1)"}


# -------------------------------------------------------------- CPU baseline
def oracle_sample(wl, budget_s=12.0, gpu_cache=None):
    """Time the float64 oracle on a bounded sample of one decode step.

    Sample: for one layer, quantize one new token for every KV head and decode
    the query heads of one KV head over the full context, from packed cache
    bytes; repeated for successive KV heads until the budget is used. The per
    step time is extrapolated to all KV heads and layers.
    """
    import threadpoolctl
    from oracle import decode as odec, layout as lay, quantize as oq, codebook as ocb, rng as orng, q8 as oq8
    from decode_attention_seeded_b200 import synth
    gen = synth.Generator(wl, layer=0)
    seeds = gen.method_seeds()
    q8k = wl.key_bits == 8
    kb, vb = ocb.codebook(2 if q8k else wl.key_bits), ocb.codebook(wl.value_bits)
    tab = dict(signs_k=orng.sign_vector(seeds[0], 128), signs_v=orng.sign_vector(seeds[1], 128),
               sketch=orng.gaussian_sketch(seeds[2], 128, 128), centroids_k=kb.centroids,
               centroids_v=vb.centroids, bk=wl.key_bits, bv=wl.value_bits)
    T = wl.context
    g = wl.group
    rng = np.random.default_rng(0)
    if gpu_cache is None:
        # packed bytes of a synthetic cache (random bits: the oracle's cost does not depend on them)
        npg = (T + 15) // 16
        blocks = rng.integers(0, 256, size=(npg, lay.block_bytes(wl.key_bits, wl.value_bits)), dtype=np.uint8)
        off = lay.section_offsets(wl.key_bits, wl.value_bits)
        no, nn = off["norm"], blocks.shape[1] - off["norm"]
        blocks[:, no:] = np.frombuffer(np.abs(rng.standard_normal((npg, nn // 2))).astype(np.float16).tobytes(),
                                       dtype=np.uint8).reshape(npg, nn)
        if q8k:                                    # finite fp16 block scales
            so = off["sign"]                       # the scale section
            blocks[:, so:so + 128] = np.frombuffer(np.abs(rng.standard_normal((npg, 64))).astype(np.float16)
                                                   .tobytes(), dtype=np.uint8).reshape(npg, 128)
    else:
        blocks = gpu_cache
    bt = np.arange(blocks.shape[0])
    heads_done = 0
    t0 = time.perf_counter()
    with threadpoolctl.threadpool_limits(1):
        while True:
            x = rng.standard_normal((1, 128))
            if q8k:
                oq8.quantize_q8(x)
            else:
                oq.quantize(x, tab["signs_k"], kb.centroids, kb.thresholds, tab["sketch"])
            oq.quantize(x, tab["signs_v"], vb.centroids, vb.thresholds)
            if q8k:
                k8, sc, vc, nv = odec.gather_sequence_q8(blocks[:, None, :], bt, T, 0, wl.value_bits)
            else:
                kc, sb, vc, nk, gm, nv = odec.gather_sequence(blocks[:, None, :], bt, T, 0, wl.key_bits,
                                                              wl.value_bits)
            for hh in range(g):
                if q8k:
                    lg = oq8.logits_q8(rng.standard_normal(128), k8, sc, 1 / np.sqrt(128))
                else:
                    qt, p = odec.transform_query(rng.standard_normal(128), tab["signs_k"], tab["sketch"])
                    lg = odec.logits(qt, p, kc, nk, gm, sb, kb.centroids, 1 / np.sqrt(128), 128)
                odec.attend(lg, vc, nv, vb.centroids, tab["signs_v"])
            heads_done += 1
            el = time.perf_counter() - t0
            if el >= budget_s or heads_done >= wl.n_kv_heads * wl.n_layers:
                break
    per_head = el / heads_done
    per_step = per_head * wl.n_kv_heads * wl.n_layers
    return {"value": wl.batch / per_step, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{heads_done} (layer, KV head) decode groups of {g} query heads over {T} tokens "
                      f"plus one token quantize each, float64 NumPy, 1 thread; extrapolated x"
                      f"{wl.n_kv_heads * wl.n_layers} to a full step", "seconds": round(el, 2)}


# ------------------------------------------------------------------- parity
def bench_parity(bench, layer, pairs=4, near=1e-5, rtol=1e-3):
    """Sampled oracle check of the bench's own cache (one layer, after the timed steps).

    Quantize: every token the timed decode steps appended to this layer (all KV
    heads), unpacked from the GPU cache and compared with the oracle's
    quantization of the same bf16 rows: codes and sign bits bit-exact except
    within `near` of a decision boundary (counted as excused), fp16 norms within
    one unit in the last place. Decode: `pairs` (sequence, KV head) pairs decoded
    by the oracle over the full context from the bytes the GPU wrote, against
    the outputs of the last decode call on this layer."""
    from oracle import codebook as ocb, decode as odec, layout as lay, quantize as oq, rng as orng
    torch, wl = bench.torch, bench.wl
    if wl.key_bits == 8:
        return {"skipped": "q8_0 keys: checked by the q8 tests"}
    bk, bv, n_kv = wl.key_bits, wl.value_bits, wl.n_kv_heads
    kb, vb = ocb.codebook(bk), ocb.codebook(bv)
    seeds = bench.seeds
    tab = dict(signs_k=orng.sign_vector(seeds[0], 128), signs_v=orng.sign_vector(seeds[1], 128),
               sketch=orng.gaussian_sketch(seeds[2], 128, 128), centroids_k=kb.centroids,
               centroids_v=vb.centroids, bk=bk, bv=bv)
    cache, n_pages = bench.caches[layer]
    host = cache.view(n_pages, n_kv, -1).cpu().numpy()
    bt = bench.btabs[layer].cpu().numpy()
    res = {"layer": layer}
    # quantize: the appended tokens
    xk = bench.newk[layer].float().cpu().numpy().astype(np.float64)     # [steps, B, n_kv, 128]
    xv = bench.newv[layer].float().cpu().numpy().astype(np.float64)
    fk, fv, fs, nk, gm, nv, rk, rv = [], [], [], [], [], [], [], []
    for s in range(bench.total_steps):
        for b in range(wl.batch):
            pos = int(bench.lens0[b]) + s
            for h in range(n_kv):
                f = lay.read_page(host[bt[b, pos // 16], h], bk, bv)
                tau = pos % 16
                fk.append(f[0][tau]); fs.append(f[1][tau]); fv.append(f[2][tau])
                nk.append(f[3][tau]); gm.append(f[4][tau]); nv.append(f[5][tau])
                rk.append(xk[s, b, h]); rv.append(xv[s, b, h])
    qk = oq.quantize(np.array(rk), tab["signs_k"], kb.centroids, kb.thresholds, tab["sketch"])
    qv = oq.quantize(np.array(rv), tab["signs_v"], vb.centroids, vb.thresholds)
    near_k = np.min(np.abs(qk.y[..., None] - kb.thresholds), axis=-1) < near
    near_v = np.min(np.abs(qv.y[..., None] - vb.thresholds), axis=-1) < near
    dk, dv = np.array(fk) != qk.codes, np.array(fv) != qv.codes
    same = ~np.any(dk, axis=1)
    near_s = np.abs(qk.projection) < near * np.linalg.norm(qk.residual, axis=1)[:, None]
    ds = (np.array(fs) != qk.sign_bits) & same[:, None]

    def ulps(a, b):
        ia = np.asarray(a, dtype=np.float16).view(np.int16).astype(np.int64)
        ib = np.asarray(b, dtype=np.float16).view(np.int16).astype(np.int64)
        ia = np.where(ia < 0, -(ia & 0x7FFF), ia)
        ib = np.where(ib < 0, -(ib & 0x7FFF), ib)
        return np.abs(ia - ib)

    res.update({"quantize_rows": len(rk), "bad_k_codes": int(np.sum(dk & ~near_k)),
                "excused_k_codes": int(np.sum(dk & near_k)), "bad_v_codes": int(np.sum(dv & ~near_v)),
                "excused_v_codes": int(np.sum(dv & near_v)), "bad_signs": int(np.sum(ds & ~near_s)),
                "excused_signs": int(np.sum(ds & near_s)),
                "bad_norms": int(np.sum(ulps(nk, qk.norm16) > 1) + np.sum(ulps(nv, qv.norm16) > 1)
                                 + np.sum(ulps(np.array(gm)[same], qk.gamma16[same]) > 1))})
    # decode: sampled (sequence, KV head) pairs of the last call on this layer
    last = bench.total_steps - 1
    L = bench.lens[last].cpu().numpy()
    q = bench.q[last, layer].float().cpu().numpy().astype(np.float64)
    out = bench.out[layer].cpu().numpy().astype(np.float64)
    g = wl.n_q_heads // n_kv
    rng = np.random.default_rng(0)
    allp = [(b, h) for b in range(wl.batch) for h in range(n_kv)]
    pick = [allp[int(i)] for i in rng.permutation(len(allp))[:pairs]]
    worst, worst_e, nonfinite = 0.0, 0.0, 0
    for b, h in pick:
        want = odec.decode_paged(host[:, h:h + 1], bt[b:b + 1], [int(L[b])], q[b:b + 1, h * g:(h + 1) * g], tab)[0]
        w, we, nf = decode_row_errors(out[b, h * g:(h + 1) * g], want)
        worst, worst_e, nonfinite = max(worst, w), max(worst_e, we), nonfinite + nf
    res.update({"decode_pairs": [list(x) for x in pick], "decode_tokens": [int(L[b]) for b, _ in pick],
                "worst_rel_err": worst, "worst_elem_err": worst_e, "nonfinite_outputs": nonfinite,
                "tolerance": rtol,
                "ok": bool(nonfinite == 0 and worst <= rtol and worst_e <= rtol and all(
                    res[k] == 0 for k in res if isinstance(k, str) and k.startswith("bad")))})
    return res


def decode_row_errors(got, want):
    """(worst per-head relative error, worst element error, count of non-finite
    outputs) of decode outputs got [heads, 128] against the oracle's want. The
    element error is relative to the element, floored at the head's rms element
    size. Non-finite outputs are counted, not folded into the maxima (a NaN would
    otherwise compare as no error)."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    nonfinite = int(np.sum(~np.isfinite(got)))
    if nonfinite:
        return 0.0, 0.0, nonfinite
    ref = np.linalg.norm(want, axis=-1)
    worst = float(np.max(np.linalg.norm(got - want, axis=-1) / ref))
    floor = ref[:, None] / np.sqrt(want.shape[-1])
    worst_e = float(np.max(np.abs(got - want) / np.maximum(np.abs(want), floor)))
    return worst, worst_e, 0


def reference_arm(wl, args, world):
    """The float64 oracle on the host's cores, timed over K sample steps after W warm-up ones.

    One sample step: quantize one new token (K and V) of one KV head, and decode
    that KV head's query heads over a slice of the context of `sample_pages`
    pages, from packed bytes. Its time scales to a full step (every page of every
    sequence, KV head and layer, and every appended token): the line's value is
    that extrapolation, and ms_per_step is the time of one sample step."""
    import threadpoolctl
    from oracle import codebook as ocb, decode as odec, layout as lay, quantize as oq, rng as orng, q8 as oq8
    from decode_attention_seeded_b200 import synth
    gen = synth.Generator(wl, layer=0)
    seeds = gen.method_seeds()
    q8k = wl.key_bits == 8
    kb, vb = ocb.codebook(2 if q8k else wl.key_bits), ocb.codebook(wl.value_bits)
    tab = dict(signs_k=orng.sign_vector(seeds[0], 128), signs_v=orng.sign_vector(seeds[1], 128),
               sketch=orng.gaussian_sketch(seeds[2], 128, 128))
    rng = np.random.default_rng(0)
    lens0 = seq_lens_of(wl)
    total_pages = int(np.sum((lens0 + 15) // 16))
    budget = min(args.oracle_budget * 5, 120.0)                  # seconds for the whole run
    # packed bytes of a synthetic slice (random bits: the oracle's cost does not depend on them)
    npg = min(total_pages, 2048)
    blocks = rng.integers(0, 256, size=(npg, lay.block_bytes(wl.key_bits, wl.value_bits)), dtype=np.uint8)
    off = lay.section_offsets(wl.key_bits, wl.value_bits)
    no = off["norm"]
    blocks[:, no:] = np.frombuffer(np.abs(rng.standard_normal((npg, (blocks.shape[1] - no) // 2)))
                                   .astype(np.float16).tobytes(), dtype=np.uint8).reshape(npg, -1)
    if q8k:
        so = off["sign"]
        blocks[:, so:so + 128] = np.frombuffer(np.abs(rng.standard_normal((npg, 64))).astype(np.float16)
                                               .tobytes(), dtype=np.uint8).reshape(npg, 128)
    bt = np.arange(npg)

    def sample_step(pages):
        x = rng.standard_normal((1, 128))
        if q8k:
            oq8.quantize_q8(x)
        else:
            oq.quantize(x, tab["signs_k"], kb.centroids, kb.thresholds, tab["sketch"])
        oq.quantize(x, tab["signs_v"], vb.centroids, vb.thresholds)
        T = pages * 16
        if q8k:
            k8, sc, vc, nv = odec.gather_sequence_q8(blocks[:, None, :], bt, T, 0, wl.value_bits)
        else:
            kc, sb, vc, nk, gm, nv = odec.gather_sequence(blocks[:, None, :], bt, T, 0, wl.key_bits, wl.value_bits)
        for _ in range(wl.group):
            if q8k:
                lg = oq8.logits_q8(rng.standard_normal(128), k8, sc, 1 / np.sqrt(128))
            else:
                qt, p = odec.transform_query(rng.standard_normal(128), tab["signs_k"], tab["sketch"])
                lg = odec.logits(qt, p, kc, nk, gm, sb, kb.centroids, 1 / np.sqrt(128), 128)
            odec.attend(lg, vc, nv, vb.centroids, tab["signs_v"])

    with threadpoolctl.threadpool_limits(1):
        t0 = time.perf_counter()
        sample_step(1)
        t_one = time.perf_counter() - t0
        t0 = time.perf_counter()
        sample_step(min(npg, 64))
        per_page = max((time.perf_counter() - t0 - t_one) / max(min(npg, 64) - 1, 1), 1e-7)
        fixed = max(t_one - per_page, 0.0)
        per_step = budget / (args.steps + args.warmup)
        pages = int(min(npg, max(1, (per_step - fixed) / per_page)))
        for _ in range(args.warmup):
            sample_step(pages)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            sample_step(pages)
        el = time.perf_counter() - t0
    t_sample = el / args.steps
    # a full step: every page of every (sequence, KV head) of every layer, plus the
    # fixed per-(sequence, KV head) cost (quantize of the new token, query transform)
    page_cost = max(t_sample - fixed, 0.0) / pages
    layers = bench_layers(wl, block_bytes_of(wl))
    full_step = layers * wl.n_kv_heads * (total_pages * page_cost + wl.batch * fixed)
    value = wl.batch / full_step
    cpu = {"kind": "oracle", "cores": 1, "value": value, "unit": "tokens/s",
           "sample": f"{args.steps} sample steps after {args.warmup} warm-up ones, each: quantize one token-head "
                     f"(K and V) and decode {wl.group} query heads of one KV head over {pages} pages "
                     f"({pages * 16} tokens), float64 NumPy, 1 thread; scaled to a full step of "
                     f"{layers} layers x {wl.n_kv_heads} KV heads x {total_pages} pages"}
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_sample * 1e3,
            "ms_per_full_step_extrapolated": full_step * 1e3, "extrapolated": True,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, world, args.steps, args.warmup, args.sparse_v, args.peaked),
            "cpu_baseline": cpu,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# --------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=128)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama8b")
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-parity", action="store_true", help="skip the sampled oracle check (profiling runs)")
    ap.add_argument("--oracle-budget", type=float, default=12.0)
    ap.add_argument("--sparse-v", type=float, default=0.0,
                    help="Sparse V threshold (relative attention weight; 0 = dense)")
    ap.add_argument("--peaked", action="store_true",
                    help="queries built from a few cached keys each (concentrated attention)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    from decode_attention_seeded_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    if args.layers:
        import dataclasses
        wl = dataclasses.replace(wl, n_layers=args.layers)

    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(reference_arm(wl, args, world)), flush=True)
        return

    import torch
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    bench = DecodeBench(wl, args.steps, args.warmup, dev, rank, sparse_v=args.sparse_v, peaked=args.peaked)
    W, K = args.warmup, args.steps
    g_warm = bench.capture(bench.step, range(W))
    g_main = bench.capture(bench.step, range(W, W + K))
    g_warm.replay()
    # one untimed replay of the timed graph: its first launch uploads the graph to
    # the device; the K steps rewrite the same slots with the same data when timed
    g_main.replay()
    torch.cuda.synchronize(dev)
    assert bench.ctx.device_error() == 0

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)

    barrier()
    with ClockSampler(local) as clk:
        t_main = timed(torch, dev, g_main.replay)
    barrier()
    t_main = max_over_ranks(t_main, world, dev)
    clocks = clk.summary()

    # end-to-end arm: same K steps from host buffers (state rewinds: same slots rewritten)
    g_e2e = bench.capture(bench.step_e2e, range(W, W + K))
    g_e2e_w = bench.capture(bench.step_e2e, range(W))
    # order check of the overlapped copies: the same steps with every copy in line
    # with the layers give the host the same outputs (up to the summation order of
    # the split-K merge, which depends on which warp took which page)
    g_ser = bench.capture(bench.step_e2e_serial, range(W, W + K))
    g_e2e_w.replay()
    g_ser.replay()
    torch.cuda.synchronize(dev)
    ref_out = bench.h_out[W:W + K].clone()
    del g_ser
    g_e2e_w.replay()
    g_e2e.replay()                                        # graph upload, untimed (as above)
    torch.cuda.synchronize(dev)
    e2e_dev = float((bench.h_out[W:W + K] - ref_out).abs().max() / ref_out.abs().max().clamp_min(1e-30))
    assert e2e_dev < 1e-4, f"overlapped end-to-end copies disagree with the in-line ones: {e2e_dev}"
    del ref_out
    barrier()
    t_e2e = max_over_ranks(timed(torch, dev, g_e2e.replay), world, dev)
    barrier()

    # decode attention alone (no append), back-to-back over the layer caches
    reps = 4
    g_dec = bench.decode_only_graph(reps)
    g_dec.replay()
    barrier()
    t_dec = max_over_ranks(timed(torch, dev, g_dec.replay), world, dev)
    n_dec = reps * bench.n_layers
    dec_s = t_dec / n_dec
    assert bench.ctx.device_error() == 0
    parity = bench_parity(bench, bench.n_layers - 1) if rank == 0 and not args.no_parity else None

    base16 = bench.bf16_baseline()
    logits_cmp = bench.logits_timing()
    quant = bench.quantize_timing()
    quant["frac"] = quant["gbs"] / load_peaks()[0]
    peak, peak_kind = load_peaks()
    bpt = bench.ctx.block_bytes // 16                     # bytes per token-head (102 for 3/2 bits)
    alg_bytes = bpt * bench.cache_tokens * wl.n_kv_heads
    # the timed step launches one decode kernel per layer and nothing else
    step_launch_s = t_main / (K * bench.n_layers)
    # cached tokens per call, averaged over the timed steps (the context grows by one each step)
    step_tokens = int(np.sum(bench.lens0)) + wl.batch * (W + (K + 1) / 2)
    step_bytes = bpt * step_tokens * wl.n_kv_heads
    achieved = step_bytes / step_launch_s / 1e9
    traffic = recorded_traffic("bytes_per_launch")

    tokens = K * wl.batch * world
    value = job_throughput(K * wl.batch, world, t_main)
    h2d, d2h = bench.e2e_bytes()
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": t_main / K * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": f"int8/fp16 tensor-core, fp32 accumulate ({key_format(wl.key_bits)}, {wl.value_bits}-bit values)",
        "data": "synthetic",
        "config": workload_config(wl, world, K, W, args.sparse_v, args.peaked),
        "e2e": {"value": job_throughput(K * wl.batch, world, t_e2e), "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "copies": "layer 0's inputs in line, the others' on a copy stream; outputs in two copies, the first overlapping the last two layers",
                "order_check_max_rel_diff": e2e_dev},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "peak_kind": peak_kind,
                     "kernel": "decode_kernel via tq_decode_step (append, query transform, split-K decode, "
                               "merge): the one kernel the timed step launches, once per layer",
                     "us_per_launch": step_launch_s * 1e6, "alg_bytes_per_launch": step_bytes,
                     "timing": "CUDA events around the timed graph replays / launches"},
        "roofline_attention": {"bound": "hbm", "achieved": alg_bytes / dec_s / 1e9, "peak": peak, "unit": "GB/s",
                               "frac": alg_bytes / dec_s / 1e9 / peak, "peak_kind": peak_kind,
                               "kernel": "decode_kernel via tq_decode_attention (no append), final context",
                               "us_per_launch": dec_s * 1e6, "alg_bytes_per_launch": alg_bytes},
        "parity": parity,
        "quantize": quant,
        "logits": logits_cmp,
        "bf16_baseline": dict(base16, **({"compressed_us_per_layer": dec_s * 1e6,
                                          "speedup_vs_bf16": base16["us_per_layer"] / (dec_s * 1e6),
                                          "cache_bytes_ratio": base16["bytes_per_layer"] / alg_bytes}
                                         if "us_per_layer" in base16 else {})),
        "gpu_launches": K * bench.n_layers,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_sample(wl, budget_s=args.oracle_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
