"""Sets a multi-layer SegPaged prefill workload up on one GPU through the C ABI and runs it.

Per layer: the storage accounting (segpaged_pages_bytes) gives every (sequence, KV head) its stored
page count, the caller-side page assignment hands out physical ids in one shared pool, segpaged_build
scatters the layer's dense K/V into the pool (with the RoPE re-alignment when the workload asks for
it), segpaged_prefill_plan produces the work units, and segpaged_attn_prefill runs the attention.
Device memory comes from PyTorch; every computation runs in libsegpaged.so.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

from . import segpaged as sp
from . import synth
from .counts import visible_counts, visible_flops  # noqa: F401  (re-exported)


@dataclass
class LayerState:
    cls: np.ndarray            # [B, Hkv, 3]
    pages_per_head: np.ndarray
    table: np.ndarray          # int32, physical ids
    offs: np.ndarray           # int32 [B*Hkv+1]
    units: np.ndarray | None = None       # plan records (work units, then combine records)
    info: dict | None = None
    table_dev: torch.Tensor | None = None
    offs_dev: torch.Tensor | None = None
    cls_dev: torch.Tensor | None = None
    units_dev: torch.Tensor | None = None
    units_host: torch.Tensor | None = None   # pinned staging copy of the plan
    upload_done: torch.cuda.Event | None = None
    q: torch.Tensor | None = None
    o: torch.Tensor | None = None
    lse: torch.Tensor | None = None
    stored_bytes: int = 0
    dense_bytes: int = 0
    k_new: torch.Tensor | None = None         # append: the query rows' keys / values [total_q, Hkv, D]
    v_new: torch.Tensor | None = None
    mass_items: np.ndarray | None = None     # token-mass plan (sparse-FFN score)
    mass_items_dev: torch.Tensor | None = None
    mass: torch.Tensor | None = None


class Runner:
    """One workload's pools, page tables, plans, queries and outputs on one device.

    shared_dense: all layers scatter the same dense K/V (drawn for layer 0) through their own tables,
    class maps and queries -- for many-layer workloads whose dense K/V would not fit in memory at once.
    keep_dense: keep each layer's dense K/V on the device after set-up (tests compare against them).
    mass: also plan and hold the per-token attention mass (the sparse-FFN score) of every layer.
    frags: gather-time RoPE fragments (frag_offs [B+1], frag_start [F], frag_cos_sin [F, D/2, 2] numpy arrays):
    the pools keep the keys as drawn and prefill and token mass re-align them per fragment as they load them.
    append: fused append-and-attend -- the build writes only the rows before each query range (the query
    rows' pool slots get unrelated values) and each prefill writes the query rows' keys/values into the pool
    while attending over them.
    graphs: run each layer's plain prefill call as a CUDA graph, captured once per plan shape, so that the
    call's launches (counter clear, prefill, combine) reach the GPU as one submission and its short launches
    do not wait on the host between them. The graph reads the same buffers as the call it was captured from,
    so every replay sees the plan, queries and pages the step has just written.
    """

    def __init__(self, w: synth.Workload, device="cuda", layers=None, keep_dense=False, page_seed_offset=0,
                 shared_dense=False, split_ctas=None, mass=False, frags=None, append=False, graphs=False):
        self.w = w
        self.device = torch.device(device)
        # long units are split across CTAs when one alone exceeds a CTA's share (short query ranges)
        self.split_ctas = (torch.cuda.get_device_properties(self.device).multi_processor_count
                           if split_ctas is None else int(split_ctas))
        self.layers = list(range(w.layers)) if layers is None else list(layers)
        self.keep_dense = keep_dense or shared_dense
        self.shared_dense = shared_dense
        self.dense = {}
        B, H = w.num_seqs, w.num_kv_heads
        self.dims = sp.Dims(B, w.num_q_heads, H, w.head_dim, w.page_size, 0)
        self.ctx = np.asarray(w.ctx_lens, np.int32)
        self.ql = np.asarray(w.q_lens, np.int32)
        self.state = {}
        base = 0
        for li in self.layers:
            cls = np.ascontiguousarray(w.classes[li], dtype=np.int32)
            stored, dense, per = sp.segpaged_pages_bytes(self.dims, self.ctx, self.ql, cls)
            table, offs, n = synth.assign_pages(per.reshape(B, H), w.page_order, seed=w.seed + 7919 * li + page_seed_offset)
            self.state[li] = LayerState(cls=cls, pages_per_head=per, table=table + base, offs=offs,
                                        stored_bytes=stored, dense_bytes=dense)
            base += n
        self.num_pages = max(base, 1)
        if w.page_order == "shuffled" and len(self.layers) > 1:   # one permutation over the whole pool
            perm = np.random.default_rng(w.seed + 104729 + page_seed_offset).permutation(self.num_pages).astype(np.int32)
            for st in self.state.values():
                st.table = perm[st.table]
        self.dims.num_pages = self.num_pages
        D, P = w.head_dim, w.page_size
        self.k_pool = torch.empty(self.num_pages, P, D, dtype=torch.bfloat16, device=self.device)
        self.v_pool = torch.empty(self.num_pages, P, D, dtype=torch.bfloat16, device=self.device)
        self.cu_k_dev = torch.from_numpy(w.cu_k()).to(self.device)
        self.ql_dev = torch.from_numpy(self.ql).to(self.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.workspace = None
        self.mass_workspace = None
        self.with_mass = mass
        self.cu_q_dev = torch.from_numpy(w.cu_q().astype(np.int32)).to(self.device)
        if append and (w.rope_theta is not None or frags is not None):
            raise ValueError("append mode takes the new keys as given; it does not combine with RoPE re-alignment")
        self.append = append
        self.frags = None
        if frags is not None:
            fo, fs, fc = frags
            self.frags = (torch.from_numpy(np.ascontiguousarray(fo, dtype=np.int32)).to(self.device),
                          torch.from_numpy(np.ascontiguousarray(fs, dtype=np.int32)).to(self.device),
                          torch.from_numpy(np.ascontiguousarray(fc, dtype=np.float32)).to(self.device))
        self.rope = None
        if w.rope_theta is not None:
            self.rope = torch.from_numpy(sp.segpaged_rope_cos_sin(w.rope_theta, w.rope_deltas, D)).to(self.device)
        if self.frags is not None:
            self.rope = None          # the pools keep the keys as drawn; prefill re-aligns them per fragment
        self.scale = 1.0 / math.sqrt(D)
        # per layer: the build and plain-prefill calls with their arguments marshalled once (PreparedCall), so a
        # step's host overhead per call is one ctypes call; rebuilt when the plan's shape or the workspace changes
        self._prep_build, self._prep_prefill = {}, {}
        self.graphs = graphs
        for li in self.layers:
            self._setup_layer(li)

    # ------------------------------------------------------------------------------------ set-up
    def _setup_layer(self, li):
        w, st = self.w, self.state[li]
        st.table_dev = torch.from_numpy(st.table).to(self.device)
        st.offs_dev = torch.from_numpy(st.offs).to(self.device)
        st.cls_dev = torch.from_numpy(st.cls.reshape(-1)).to(self.device)
        if self.shared_dense:
            if not self.dense:
                _, k, v = synth.layer_inputs(w, 0, device=self.device)
                self.dense[0] = (k, v)
            q = synth.layer_inputs(w, li, device=self.device, parts="q")[0]
        else:
            q, k, v = synth.layer_inputs(w, li, device=self.device)
            if self.keep_dense:
                self.dense[li] = (k, v)
            else:
                self._tmp_dense = (k, v)
        st.q = q
        if self.append:
            k, v = self.dense_of(li)
            cq, ck = w.cu_q(), w.cu_k()
            rows = torch.cat([torch.arange(int(ck[b + 1]) - w.q_lens[b], int(ck[b + 1]), device=self.device)
                              for b in range(w.num_seqs)]) if w.total_q else torch.zeros(0, dtype=torch.long,
                                                                                          device=self.device)
            st.k_new = k[rows].contiguous()
            st.v_new = v[rows].contiguous()
        st.o = torch.empty_like(q)
        st.lse = torch.empty(w.num_q_heads, w.total_q, dtype=torch.float32, device=self.device)
        self.build_layer(li)
        self._tmp_dense = None
        self.plan_layer(li)
        st.units_dev = torch.from_numpy(np.ascontiguousarray(st.units)).to(self.device)
        st.units_host = torch.from_numpy(np.ascontiguousarray(st.units)).pin_memory()
        need = sp.segpaged_prefill_workspace_bytes(self.dims, st.info)
        if self.workspace is None or self.workspace.numel() * 4 < need:
            self.workspace = torch.zeros((need + 3) // 4, dtype=torch.int32, device=self.device)
        if self.with_mass:
            self.plan_mass(li)
            st.mass_items_dev = torch.from_numpy(np.ascontiguousarray(st.mass_items)).to(self.device)
            st.mass = torch.zeros(w.total_q, dtype=torch.float32, device=self.device)
            need = sp.segpaged_mass_workspace_bytes(self.dims, w.total_q)
            if self.mass_workspace is None or self.mass_workspace.numel() * 4 < need:
                self.mass_workspace = torch.zeros((need + 3) // 4, dtype=torch.int32, device=self.device)

    def dense_of(self, li):
        if self._tmp_dense is not None:
            return self._tmp_dense
        return self.dense[0 if self.shared_dense else li]

    _tmp_dense = None

    # -------------------------------------------------------------------------------- hot path
    def account_layer(self, li):
        """Storage accounting of one layer (host): stored and dense K+V bytes."""
        st = self.state[li]
        stored, dense, _ = sp.segpaged_pages_bytes(self.dims, self.ctx, self.ql, st.cls)
        return stored, dense

    def plan_layer(self, li):
        """Host planning of one layer's work units (SELECTVISIBLESTATE)."""
        st = self.state[li]
        plan = sp.segpaged_prefill_plan_append if self.append else sp.segpaged_prefill_plan
        st.units, st.info = plan(self.dims, self.ctx, self.ql, st.cls, st.offs, self.split_ctas)
        return st.units

    def upload_plan(self, li, stream=None):
        st = self.state[li]
        if st.upload_done is not None:
            st.upload_done.synchronize()     # the previous copy out of the staging buffer has finished
        st.units_host.numpy()[:] = st.units
        s = torch.cuda.current_stream(self.device) if stream is None else stream
        with torch.cuda.stream(s):
            st.units_dev.copy_(st.units_host, non_blocking=True)
        st.upload_done = torch.cuda.Event()
        st.upload_done.record(s)

    def build_layer(self, li, stream=None):
        k, v = self.dense_of(li)
        st = self.state[li]
        if self.append and st.k_new is not None:
            # the pool gets unrelated (finite) values in the query rows: the fused prefill must overwrite them
            w = self.w
            ck = w.cu_k()
            k, v = k.clone(), v.clone()
            for b in range(w.num_seqs):
                lo, hi = int(ck[b + 1]) - w.q_lens[b], int(ck[b + 1])
                k[lo:hi] = -3.0 * k[lo:hi] + 1.0
                v[lo:hi] = 0.5 * v[lo:hi] - 2.0
        if self.append or self._tmp_dense is not None:       # per-call inputs: marshal them each time
            sp.segpaged_build(self.dims, k, v, self.cu_k_dev, self.ql_dev, st.cls_dev, st.table_dev, st.offs_dev,
                              self.rope, self.k_pool, self.v_pool, self.status, stream)
            return
        call = self._prep_build.get(li)
        if call is None:
            call = self._prep_build[li] = sp.prepare_build(self.dims, k, v, self.cu_k_dev, self.ql_dev, st.cls_dev,
                                                            st.table_dev, st.offs_dev, self.rope, self.k_pool,
                                                            self.v_pool, self.status)
        call(stream)

    def prefill(self, li, stream=None):
        st = self.state[li]
        if self.append:
            sp.segpaged_attn_prefill_append(self.dims, st.q, st.k_new, st.v_new, self.k_pool, self.v_pool, st.table_dev,
                                            st.units_dev, st.info, self.scale, st.o, st.lse, self.workspace,
                                            self.status, stream)
            return
        if self.frags is not None:
            sp.segpaged_attn_prefill_rope(self.dims, st.q, self.k_pool, self.v_pool, st.table_dev, st.units_dev, st.info,
                                          self.scale, *self.frags, st.o, st.lse, self.workspace, self.status, stream)
            return
        key = (id(self.workspace), tuple(st.info.values()))
        cached = self._prep_prefill.get(li)
        if cached is None or cached[0] != key:
            call = sp.prepare_attn_prefill(self.dims, st.q, self.k_pool, self.v_pool, st.table_dev, st.units_dev,
                                           st.info, self.scale, st.o, st.lse, self.workspace, self.status)
            if not self.graphs:
                cached = self._prep_prefill[li] = (key, call, None)
            else:
                call(stream)     # this call's prefill, issued directly; the graph serves the calls after it
                self._prep_prefill[li] = (key, call, capture_graph(call, self.device))
                return
        _, call, graph = cached
        if graph is None:
            call(stream)
        elif stream is None:
            graph.replay()
        else:
            with torch.cuda.stream(stream):
                graph.replay()

    def rope_realign_preferred(self) -> bool:
        """Which gather-time RoPE path the caller should take (see prefill_rope_auto): the re-alignment pass when
        some (sequence, KV head) has more than one work unit, i.e. its query range spans more than 2 x 128 / G
        positions, so that every K tile would be rotated once per unit that loads it."""
        return rope_realign_preferred(self.w.q_lens, self.w.group)

    def prefill_rope_auto(self, li, k_scratch, stream=None):
        """Prefill with the fragments' RoPE re-alignment (self.frags) by the cheaper of the two exact paths:
        segpaged_rope_realign of the layer's K pages into k_scratch (a second pool of the same shape) followed by
        the plain prefill on it, when rope_realign_preferred(); else the gather-time kernel, which rotates each K
        tile in shared memory as it lands. Both give bit-identical O and LSE."""
        st = self.state[li]
        if not self.rope_realign_preferred():
            self.prefill(li, stream)
            return "gather"
        sp.segpaged_rope_realign(self.dims, self.cu_k_dev, self.ql_dev, st.cls_dev, st.table_dev, st.offs_dev,
                                 *self.frags, self.k_pool, k_scratch, self.status, stream)
        sp.segpaged_attn_prefill(self.dims, st.q, k_scratch, self.v_pool, st.table_dev, st.units_dev, st.info,
                                 self.scale, st.o, st.lse, self.workspace, self.status, stream)
        return "realign"

    def plan_mass(self, li):
        """Host planning of one layer's token-mass items."""
        st = self.state[li]
        st.mass_items = sp.segpaged_mass_plan(self.dims, self.ctx, self.ql, st.cls, st.offs)
        return st.mass_items

    def token_mass(self, li, stream=None):
        """Attention mass each query row's token receives (needs this layer's prefill LSE)."""
        st = self.state[li]
        sp.segpaged_token_mass(self.dims, st.q, self.k_pool, st.table_dev, st.mass_items_dev, st.lse, self.scale, st.mass,
                               self.mass_workspace, self.status, stream, frags=self.frags)

    def select_topk(self, li, k_per_seq: torch.Tensor, selected: torch.Tensor, stream=None):
        """Top-k rows per sequence by this layer's mass into `selected`."""
        sp.segpaged_select_topk(self.state[li].mass, self.cu_q_dev, k_per_seq, selected, stream)

    def step(self, stream=None):
        """Prefill of every layer (pools and plans already in place)."""
        for li in self.layers:
            self.prefill(li, stream)

    def full_step(self, stream=None, on_prefill=None):
        """One pass of the whole hot path for every layer: storage accounting and planning on the host,
        the build scatter and the prefill on the device. on_prefill(li, start) brackets each prefill
        launch (start=True before, False after) for per-kernel timing."""
        for li in self.layers:
            self.account_layer(li)
            self.plan_layer(li)
            self.upload_plan(li, stream)
            self.build_layer(li, stream)
            if on_prefill:
                on_prefill(li, True)
            self.prefill(li, stream)
            if on_prefill:
                on_prefill(li, False)

    def check_status(self):
        s = int(self.status.item())
        if s:
            raise RuntimeError(f"device status word {s:#x}")


def capture_graph(call, device) -> torch.cuda.CUDAGraph:
    """A CUDA graph of one prepared C-ABI call that has already run once on `device` (the library configures
    a kernel on its first launch on a device, which must not happen inside a capture). Capturing launches
    nothing; replaying the graph repeats the call's launches with the same arguments."""
    with torch.cuda.device(device):
        g = torch.cuda.CUDAGraph()
        # thread_local: CUDA calls other threads make meanwhile (a process group's watchdog, for one) are not
        # checked against this capture
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            call(None)
    return g


def rope_realign_preferred(q_lens, group: int) -> bool:
    """True when some sequence's query range spans more than one work unit (2 x 128 / G positions) per KV head:
    each K tile is then loaded, and rotated at gather time, by several units, and one re-alignment pass over the
    stored pages costs less."""
    return max(q_lens, default=0) > 2 * (128 // group)


def main(argv=None):
    """Sets one or more layers of a workload up and runs their prefill launches back to back (for a profiler:
    `python -m head_sparse_paged_b200.runner dsv4-flash --layers 3 --launches 2`). Layers draw their own dense
    K/V, which is freed after the build, so only the pool, the queries and the outputs stay on the device."""
    import argparse
    ap = argparse.ArgumentParser(description=main.__doc__)
    ap.add_argument("workload")
    ap.add_argument("--layers", default="0", help="comma-separated layer indices")
    ap.add_argument("--launches", type=int, default=2, help="prefill launches per layer")
    args = ap.parse_args(argv)
    w = synth.get(args.workload)
    layers = [int(x) for x in args.layers.split(",")]
    r = Runner(w, layers=layers)
    torch.cuda.synchronize()
    for _ in range(args.launches):
        for li in layers:
            r.prefill(li)
    torch.cuda.synchronize()
    r.check_status()
    print(f"{w.name}: layers {layers}, {args.launches} prefill launches each, pool {r.num_pages} pages, "
          f"{torch.cuda.max_memory_allocated() / 1e9:.2f} GB peak device memory")
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
