"""Device state and the decode step, issued through the C ABI.

``MLARunner`` owns the device buffers of one workload (weights, RoPE tables, the paged
latent cache, per-step inputs and outputs, workspaces; all allocated with torch) and runs
a decode step as four library calls on one stream:

    mla_append_cache     the step's new tokens -> cache            (step 1)
    mla_absorb_query     q_lat = W_UK^T q_nope, q_rope rotated     (step 2)
    mla_decode_attention split-KV attention + log-sum-exp combine  (steps 3, 4)
    mla_output_up        out = W_UV o_lat                          (step 5)

Sequence b holds L_b tokens after the step: L_b - S_q cached before it, and the S_q new
tokens at positions L_b - S_q .. L_b - 1, whose queries attend causally when S_q > 1.
"""
from __future__ import annotations

import numpy as np
import torch

from . import _binding as B
from . import workloads as wl

_ACT = {"f32": B.MLA_F32, "bf16": B.MLA_BF16}
_CACHE = {"f32": B.MLA_F32, "bf16": B.MLA_BF16, "fp8": B.MLA_FP8_E4M3}
_TORCH = {"f32": torch.float32, "bf16": torch.bfloat16}


def make_dims(w: wl.Workload) -> B.mla_dims:
    return B.mla_dims(w.d_model, w.d_c, w.d_rope, w.d_nope, w.d_v, w.n_heads, wl.PAGE_SIZE,
                      _ACT[w.act_dtype], _CACHE[w.cache_dtype], w.scale)


def nvml_handle(device):
    """(pynvml module, NVML handle) of a torch CUDA device, matched by UUID so that a remapped
    CUDA_VISIBLE_DEVICES does not pick another GPU."""
    import pynvml
    pynvml.nvmlInit()
    uuid = str(torch.cuda.get_device_properties(device).uuid)
    if not uuid.startswith("GPU-"):
        uuid = "GPU-" + uuid
    return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid)


def bind_host_to_device(device):
    """Restrict the calling thread (and threads it starts later) to the CPUs NVML reports as
    local to ``device``, so that pinned host buffers allocated afterwards sit on the GPU's NUMA
    node and host<->device copies run at the link's full rate.  Returns the CPU list, or None
    when NVML gives no affinity (the affinity is then left unchanged)."""
    import os
    try:
        nv, h = nvml_handle(device)
        words = (os.cpu_count() + 63) // 64
        masks = nv.nvmlDeviceGetCpuAffinity(h, words)
    except Exception:
        return None
    cpus = {64 * i + b for i, m in enumerate(masks) for b in range(64) if (int(m) >> b) & 1}
    cpus &= os.sched_getaffinity(0)
    if not cpus:
        return None
    os.sched_setaffinity(0, cpus)
    return sorted(cpus)


class PagedCache:
    """Device tensors of a paged latent cache plus its ``mla_cache`` descriptor."""

    def __init__(self, w: wl.Workload, num_pages: int, block_table: np.ndarray, device):
        self.w = w
        page = wl.PAGE_SIZE
        if w.cache_dtype == "fp8":
            self.rows = torch.zeros((num_pages, page, w.d_c), dtype=torch.uint8, device=device)
            self.scales = torch.ones((num_pages, page, w.d_c // 128), dtype=torch.float32, device=device)
            self.rope = torch.zeros((num_pages, page, w.d_rope), dtype=torch.bfloat16, device=device)
        else:
            self.rows = torch.zeros((num_pages, page, w.row_width), dtype=_TORCH[w.cache_dtype],
                                    device=device)
            self.scales = None
            self.rope = None
        self.block_table = torch.as_tensor(block_table, dtype=torch.int32, device=device).contiguous()
        self.num_pages = num_pages
        self.desc = B.mla_cache(
            self.rows.data_ptr(), None if self.scales is None else self.scales.data_ptr(),
            None if self.rope is None else self.rope.data_ptr(), self.block_table.data_ptr(),
            self.block_table.shape[1], num_pages, self.block_table.shape[0])


class MLARunner:
    def __init__(self, w: wl.Workload, lengths=None, device=None, n_split=None, stream=None):
        self.w = w
        self.device = torch.device(device or "cuda")
        self.lengths = np.asarray(wl.draw_lengths(w) if lengths is None else lengths, dtype=np.int32)
        assert (self.lengths >= w.s_q).all(), "every sequence holds at least the step's new tokens"
        self.batch = len(self.lengths)
        self.dims = make_dims(w)
        self.n_split = w.n_split if n_split is None else n_split
        self.stream = stream
        dt = _TORCH[w.act_dtype]
        dev = self.device
        table, num_pages = wl.make_block_table(self.lengths, 0, w.shuffle_pages, wl.rng_for(w, 6))
        self.cache = PagedCache(w, num_pages, table, dev)
        self.block_table_np = table
        # weights
        w_dkv, w_kr, w_uk, w_uv = wl.draw_weights(w)
        self.w_dkv = torch.from_numpy(w_dkv).to(dev, dt).contiguous()
        self.w_kr = torch.from_numpy(w_kr).to(dev, dt).contiguous()
        self.w_uk = torch.from_numpy(w_uk).to(dev, dt).contiguous()
        self.w_uv = torch.from_numpy(w_uv).to(dev, dt).contiguous()
        # RoPE tables
        self.rope_rows = int(table.shape[1] * wl.PAGE_SIZE)
        half = w.d_rope // 2
        self.rope_cos = torch.empty((self.rope_rows, half), dtype=torch.float32, device=dev)
        self.rope_sin = torch.empty((self.rope_rows, half), dtype=torch.float32, device=dev)
        B.mla_rope_table(w.d_rope, self.rope_rows, w.theta, self.rope_cos, self.rope_sin, self.stream)
        # step geometry: S_q new tokens per sequence at positions L_b - S_q .. L_b - 1
        T = self.batch * w.s_q
        self.n_tok = T
        seq_idx = np.repeat(np.arange(self.batch, dtype=np.int32), w.s_q)
        pos = (np.repeat(self.lengths, w.s_q) - w.s_q + np.tile(np.arange(w.s_q), self.batch)).astype(np.int32)
        self.seq_idx = torch.as_tensor(seq_idx, device=dev)
        self.pos = torch.as_tensor(pos, device=dev)
        self.seq_lens = torch.as_tensor(self.lengths, device=dev)
        # step buffers
        self.h_new = torch.zeros((T, w.d_model), dtype=dt, device=dev)
        self.q_nope = torch.zeros((T, w.n_heads, w.d_nope), dtype=dt, device=dev)
        self.q_rope = torch.zeros((T, w.n_heads, w.d_rope), dtype=dt, device=dev)
        self.q_packed = torch.empty((T, w.n_heads, w.row_width), dtype=dt, device=dev)
        self.o_lat = torch.empty((T, w.n_heads, w.d_c), dtype=dt, device=dev)
        self.lse = torch.empty((T, w.n_heads), dtype=torch.float32, device=dev)
        self.out = torch.empty((T, w.n_heads, w.d_v), dtype=dt, device=dev)
        self.append_ws_bytes = B.mla_append_workspace_size(self.dims, T)
        self.append_ws = torch.empty(max(1, self.append_ws_bytes), dtype=torch.uint8, device=dev)
        self.decode_ws_bytes = B.mla_decode_workspace_size(self.dims, self.batch, w.s_q, self.n_split,
                                                           int(table.shape[1]))
        self.decode_ws = torch.empty(max(1, self.decode_ws_bytes), dtype=torch.uint8, device=dev)

    # ------------------------------------------------------------------ cache contents
    def fill_cache_projected(self, chunk: int = 16384, seed: int = 0):
        """Write the L_b - S_q tokens that precede the step by running mla_append_cache over
        hidden states h ~ N(0, 1) drawn on the device from a seeded generator."""
        w = self.w
        gen = torch.Generator(device=self.device)
        gen.manual_seed(1000 + 17 * w.seed + seed)
        pre = self.lengths - w.s_q
        seq = np.repeat(np.arange(self.batch, dtype=np.int32), pre)
        pos = np.concatenate([np.arange(n, dtype=np.int32) for n in pre]) if pre.sum() else np.zeros(0, np.int32)
        total = len(seq)
        dt = _TORCH[w.act_dtype]
        ws_bytes = B.mla_append_workspace_size(self.dims, min(chunk, max(total, 1)))
        ws = torch.empty(max(1, ws_bytes), dtype=torch.uint8, device=self.device)
        for lo in range(0, total, chunk):
            hi = min(total, lo + chunk)
            h = torch.randn((hi - lo, w.d_model), generator=gen, device=self.device, dtype=torch.float32).to(dt)
            s_t = torch.as_tensor(seq[lo:hi], device=self.device)
            p_t = torch.as_tensor(pos[lo:hi], device=self.device)
            B.mla_append_cache(self.dims, h, hi - lo, s_t, p_t, self.w_dkv, self.w_kr, self.rope_cos,
                               self.rope_sin, self.rope_rows, self.cache.desc, ws, ws_bytes, self.stream)

    def fill_cache_direct(self, seed: int = 0):
        """Draw every cache row directly from the distribution the projection produces
        (entries ~ N(0, 1)); bf16 / f32 caches only."""
        assert self.w.cache_dtype != "fp8"
        gen = torch.Generator(device=self.device)
        gen.manual_seed(2000 + 17 * self.w.seed + seed)
        rows = self.cache.rows
        rows.copy_(torch.randn(rows.shape, generator=gen, device=self.device, dtype=torch.float32))

    def draw_step_inputs(self, seed: int = 0):
        w = self.w
        gen = torch.Generator(device=self.device)
        gen.manual_seed(3000 + 17 * w.seed + seed)
        for t in (self.h_new, self.q_nope, self.q_rope):
            t.copy_(torch.randn(t.shape, generator=gen, device=self.device, dtype=torch.float32))

    # ------------------------------------------------------------------ the step
    def append(self, stream=None):
        B.mla_append_cache(self.dims, self.h_new, self.n_tok, self.seq_idx, self.pos, self.w_dkv,
                           self.w_kr, self.rope_cos, self.rope_sin, self.rope_rows, self.cache.desc,
                           self.append_ws, self.append_ws_bytes, stream or self.stream)

    def absorb(self, stream=None):
        B.mla_absorb_query(self.dims, self.q_nope, self.q_rope, self.pos, self.n_tok, self.w_uk,
                           self.rope_cos, self.rope_sin, self.rope_rows, self.q_packed,
                           stream or self.stream)

    def decode(self, stream=None):
        B.mla_decode_attention(self.dims, self.q_packed, self.cache.desc, self.seq_lens, self.batch,
                               self.w.s_q, int(self.w.causal or self.w.s_q > 1), self.n_split,
                               self.decode_ws, self.decode_ws_bytes, self.o_lat, self.lse,
                               stream or self.stream)

    def output(self, stream=None):
        B.mla_output_up(self.dims, self.o_lat, self.n_tok, self.w_uv, self.out, stream or self.stream)

    def step(self, stream=None):
        self.append(stream)
        self.absorb(stream)
        self.decode(stream)
        self.output(stream)
        return self.out

    # ------------------------------------------------------------------ steps fed from host memory
    def run_host_steps(self, h_host, q_nope_host, q_rope_host, out_host, copy_streams=None):
        """Run ``len(h_host)`` decode steps whose inputs sit in host memory and whose outputs go
        back to host memory, overlapping the transfers with the kernels.

        ``h_host[i]``, ``q_nope_host[i]``, ``q_rope_host[i]`` are step i's inputs and
        ``out_host[i]`` receives its output (CPU tensors shaped like ``h_new``, ``q_nope``,
        ``q_rope`` and ``out``; pinned - allocated after bind_host_to_device, so that they sit
        on the GPU's NUMA node - or the copies serialise with the host).  Entries may
        repeat the same tensor.  Two device copies of the per-step inputs and of ``out`` are
        used in turn: the host-to-device copy of step i + 1 and the device-to-host copy of
        step i - 1 run on their own streams while step i's kernels run on the compute stream,
        each ordered by events against the step that last used the same device copy.

        Every event operation on the compute stream sits between step i's absorb and its decode
        (a boundary the library does not overlap): one between two programmatically launched
        kernels (output -> next append, append -> absorb, combine -> output) would end their
        overlap.  So step i waits there for step i + 1's inputs, and marks step i - 1's output
        as ready there, one absorb later than it could.

        Every copy and every kernel is enqueued before the call returns; synchronise the compute
        stream to wait for all of it (its last operation waits for the final output copy)."""
        n = len(h_host)
        assert len(q_nope_host) == n and len(q_rope_host) == n and len(out_host) == n
        if n == 0:
            return
        compute = self.stream if self.stream is not None else torch.cuda.current_stream(self.device)
        if copy_streams is None:
            if not hasattr(self, "_copy_streams"):
                self._copy_streams = (torch.cuda.Stream(self.device), torch.cuda.Stream(self.device))
            copy_streams = self._copy_streams
        s_in, s_out = copy_streams
        if not hasattr(self, "_host_sets"):
            self._host_sets = [(self.h_new, self.q_nope, self.q_rope, self.out),
                               (torch.empty_like(self.h_new), torch.empty_like(self.q_nope),
                                torch.empty_like(self.q_rope), torch.empty_like(self.out))]
        sets = self._host_sets
        ev = lambda: torch.cuda.Event()
        loaded, consumed, produced, drained = ([ev(), ev()] for _ in range(4))
        used = [False, False]
        start = ev()
        start.record(compute)
        s_in.wait_event(start)
        s_out.wait_event(start)

        def load(i):
            k = i % 2
            h, qn, qr, _ = sets[k]
            with torch.cuda.stream(s_in):
                if used[k]:
                    s_in.wait_event(consumed[k])
                h.copy_(h_host[i], non_blocking=True)
                qn.copy_(q_nope_host[i], non_blocking=True)
                qr.copy_(q_rope_host[i], non_blocking=True)
                loaded[k].record(s_in)

        def drain(i):
            k = i % 2
            produced[k].record(compute)
            with torch.cuda.stream(s_out):
                s_out.wait_event(produced[k])
                out_host[i].copy_(sets[k][3], non_blocking=True)
                drained[k].record(s_out)

        load(0)
        compute.wait_event(loaded[0])
        for i in range(n):
            k = i % 2
            if i + 1 < n:
                load(i + 1)
            h, qn, qr, out = sets[k]
            B.mla_append_cache(self.dims, h, self.n_tok, self.seq_idx, self.pos, self.w_dkv, self.w_kr,
                               self.rope_cos, self.rope_sin, self.rope_rows, self.cache.desc,
                               self.append_ws, self.append_ws_bytes, compute)
            B.mla_absorb_query(self.dims, qn, qr, self.pos, self.n_tok, self.w_uk, self.rope_cos,
                               self.rope_sin, self.rope_rows, self.q_packed, compute)
            # -- the one boundary with event operations --
            consumed[k].record(compute)
            used[k] = True
            if i + 1 < n:
                compute.wait_event(loaded[(i + 1) % 2])
            if i >= 1:
                drain(i - 1)
            if i >= 2:
                compute.wait_event(drained[k])  # step i - 2's output copy left this buffer
            B.mla_decode_attention(self.dims, self.q_packed, self.cache.desc, self.seq_lens, self.batch,
                                   self.w.s_q, int(self.w.causal or self.w.s_q > 1), self.n_split,
                                   self.decode_ws, self.decode_ws_bytes, self.o_lat, self.lse, compute)
            B.mla_output_up(self.dims, self.o_lat, self.n_tok, self.w_uv, out, compute)
        drain(n - 1)
        compute.wait_event(drained[(n - 1) % 2])
