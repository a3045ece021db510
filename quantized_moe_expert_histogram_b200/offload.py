"""Offload mode: stacked MoE layers whose experts live in pinned host memory.

Each layer keeps all of its packed experts in pinned host memory and a GPU
slot pool of a few experts; ``moe_slot_stage`` brings the experts a layer
step routes to into the pool on a copy stream (hits first, then misses by
token count, in waves of half the slots) and ``moe_slot_ffn`` runs the
grouped FFN wave by wave as the copies land.  Pages: ExactMoE (compressed
experts in host memory, GPU-resident slot cache, every routed expert
executed), EdgeMoE (expert buffer filled on activation), D2MoE (loading the
next expert while computing the current one), Read-ME (a pre-gating router
decoupled from the backbone decides every layer's experts before the layers
compute, which allows lookahead scheduling of expert loads).

``OffloadStack.step`` runs one decode step through all layers in one of
two schedules:

* per-layer routing (``lookahead=False``): route layer l (the expert ids may
  be forced from a trace), one device-to-host copy of the routed ids and a
  host wait per layer, stage, permute, slot FFN, combine with the residual.
  With ``prefetch`` (EdgeMoE's expert preloading), once layer l's ids are
  known a host predictor (moe_predictor_*) names layer l+1's likely experts
  and ``moe_slot_prefetch`` copies the confident ones (expected to receive
  at least ``prefetch_min_score`` assignments, one by default; at most
  ``prefetch_max`` copies, a quarter of a cache by default) into layer
  l+1's slots behind layer l's own copies.
* lookahead (``lookahead=True``, Read-ME's pre-gating): every layer's
  expert ids for the step are known before the first layer computes -- the
  forced trace, or, without one, each layer's router applied to the step's
  input -- and reach the host in one copy per step.  The host then plans
  and enqueues every layer's staging and FFN back to back with no further
  wait, so layer l+1's copies are queued while layer l computes; layers
  alternate between two copy streams so that one layer's later waves (which
  wait for its own compute to free slots) do not hold back the next layer's
  first copies.  Gates still come from each layer's router logits at the
  given ids (the layer's own input), so the results equal the resident path
  fed the same ids.
Nested-plane layers (layout "planes"): every layer gets a bit-width gate
(D2MoE's dual routing) whose widths reach the host with the ids, and the
caches are plane-mode caches by default (``plane_staging``): an expert
moves only the planes up to the widest width its assignments use, and a
resident expert later needed wider receives only the missing planes (D2MoE's
bit-width-aware I/O).  ``set_plane_staging(False)`` swaps in whole-blob
caches over the same host blobs, for comparison.  In lookahead mode the
widths are pre-gated like the ids: each layer's bit gate applied to the
step's input at the pre-gated ids.
This module only orchestrates calls of the C ABI; torch supplies device
memory, pinned host memory and streams.
"""
from __future__ import annotations

import torch

from . import inputs as I
from . import moeq
from .layer import QuantMoELayer


class OffloadStack:
    def __init__(self, shape, layers: int, slots: int, batch: int, seed: int = 0, device="cuda",
                 prefetch: bool = False, lookahead: bool = False, plane_staging: bool = True,
                 prefetch_min_score: float = 1.0, prefetch_max: int | None = None):
        self.shape, self.n_layers, self.slots, self.batch = shape, layers, slots, batch
        self.prefetch, self.lookahead = prefetch, lookahead
        # prefetch policy: experts whose expected assignment count at the next
        # layer reaches min_score, at most prefetch_max (default: a quarter of a cache)
        self.prefetch_min_score = prefetch_min_score
        self.prefetch_max = slots // 4 if prefetch_max is None else prefetch_max
        self.nested = shape.layout == "planes"
        self.predictor = moeq.RoutePredictor(layers, shape.E) if prefetch else None
        self.prefetched = 0
        self.layers, self.host, self.pools, self.caches = [], [], [], []
        for l in range(layers):
            w = I.make_expert_weights(shape, seed=seed + 101 * l, device=device)
            r = I.make_router(shape, seed=seed + 101 * l + 1, device=device)
            layer = QuantMoELayer.from_weights(shape, r["w_router"], r["bias"], w["w_gate"], w["w_up"],
                                               w["w_down"], max_tokens=batch)
            del w
            if self.nested:
                gb = I.make_bit_gate(shape, seed=seed + 101 * l + 2, device=device, bias=True)
                layer.w_bit, layer.bias_bit = gb["w_bit"], gb["bias_bit"]
            host = layer.blobs.cpu().pin_memory()
            pool = torch.empty(slots, layer.blobs.shape[1], dtype=torch.uint8, device=device)
            layer.blobs = None  # the experts now live in host memory only
            self.layers.append(layer)
            self.host.append(host)
            self.pools.append(pool)
        self.blob_bytes = self.host[0].shape[1]
        self.plane_staging = False
        self.set_plane_staging(plane_staging)
        self.copy = torch.cuda.Stream()
        self.copy2 = torch.cuda.Stream()  # lookahead: odd layers' copies
        self.side = torch.cuda.Stream()   # lookahead: the per-step id copy
        self.compute = torch.cuda.current_stream()
        self.ids_host = [torch.empty(batch, shape.k, dtype=torch.int32).pin_memory() for _ in range(layers)]
        self.ids_all_host = torch.empty(layers, batch, shape.k, dtype=torch.int32).pin_memory()
        self.ids_pregated = torch.empty(layers, batch, shape.k, dtype=torch.int32, device=device)
        # nested layers: the widths, on the device and on the host
        self.bits_host = [torch.empty(batch, shape.k, dtype=torch.uint8).pin_memory() for _ in range(layers)]
        self.bits_all_host = torch.empty(layers, batch, shape.k, dtype=torch.uint8).pin_memory()
        self.bits_pregated = torch.empty(layers, batch, shape.k, dtype=torch.uint8, device=device)
        self._marks = None  # busy-time events of the compute stream's own segments

    def set_plane_staging(self, enable: bool):
        """(Re)create every layer's slot cache, empty: plane-mode caches when
        ``enable`` and the layers are nested-plane layers, whole-blob caches
        otherwise."""
        for c in self.caches:
            c.close()
        planes = (self.shape.d, self.shape.F, self.shape.group) if enable and self.nested else None
        self.caches = [moeq.SlotCache(self.shape.E, self.slots, self.blob_bytes, h, p, planes=planes)
                       for h, p in zip(self.host, self.pools)]
        self.plane_staging = planes is not None

    def timing(self, enable: bool):
        """Record busy time from now on: each cache's copies and FFN waves
        (moe_slot_timing) and, on the compute stream, the route + permute and
        combine segments (wait-free, so event pairs measure their work)."""
        for c in self.caches:
            c.timing(enable)
        self._marks = [] if enable else None

    def timing_read(self):
        """(copy_ms, compute_ms) since timing(True) or the last read."""
        copy_ms = ffn_ms = 0.0
        for c in self.caches:
            cm, fm = c.timing_read()
            copy_ms, ffn_ms = copy_ms + cm, ffn_ms + fm
        seg = 0.0
        if self._marks:
            self._marks[-1][1].synchronize()
            seg = sum(a.elapsed_time(b) for a, b in self._marks)
            self._marks = []
        return copy_ms, ffn_ms + seg

    def _mark(self):
        if self._marks is None:
            return None
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(self.compute)
        return ev

    def _segment(self, start):
        if start is not None:
            self._marks.append((start, self._mark()))

    def step(self, x, forced_ids=None):
        """One decode step of the batch x (bf16 [batch][d]) through all layers.
        forced_ids: int32 [layers][batch][k] on the device, or None (the
        routers decide).  Returns (y, per-layer [hits, misses, bytes, waves])."""
        if self.lookahead:
            return self._step_lookahead(x, forced_ids)
        sh, stats = self.shape, []
        for l, layer in enumerate(self.layers):
            v = layer.views(self.batch)
            t0 = self._mark()
            moeq.moe_route_topk(x, layer.w_router, layer.bias, sh.k,
                                forced_idx=None if forced_ids is None else forced_ids[l].contiguous(),
                                topk_idx=v["topk_idx"], topk_w=v["topk_w"], workspace=v["route_ws"])
            bits = None
            if self.nested:
                bits = moeq.moe_bit_gate(x, layer.w_bit, layer.bias_bit, v["topk_idx"], bits=v["bits"],
                                         status=v["status"])
            moeq.moe_permute(v["topk_idx"], sh.E, bits=bits, x=x, out=v, status=v["status"])
            self._segment(t0)
            # the one device -> host crossing per layer: the routed ids (and widths)
            self.ids_host[l].copy_(v["topk_idx"], non_blocking=True)
            if bits is not None:
                self.bits_host[l].copy_(bits, non_blocking=True)
            self.compute.synchronize()
            n_waves, st = self.caches[l].stage(self.ids_host[l].reshape(-1), self.copy, self.compute,
                                               bits_host=self._bits_for(self.bits_host[l]))
            self.caches[l].ffn(v["x_perm"], v["offsets"], self.batch, sh.d, sh.F, sh.group, layer.layout,
                               v["workspace"], v["y_perm"], v["status"], self.copy, self.compute)
            if self.prefetch and self.predictor is not None:
                if l > 0:
                    self.predictor.observe(l, self.ids_host[l - 1], self.ids_host[l],
                                           prev2_ids=self.ids_host[l - 2] if l >= 2 else None)
                if l + 1 < self.n_layers:
                    # confident predictions only: the link is the bottleneck, and a
                    # wrong copy costs a slot and bandwidth; keyed by the experts of
                    # this layer and the one before it (EdgeMoE's profile key)
                    pred = self.predictor.predict(l + 1, self.ids_host[l], self.prefetch_max,
                                                  min_score=self.prefetch_min_score,
                                                  prev2_ids=self.ids_host[l - 1] if l >= 1 else None)
                    if pred.numel():
                        self.prefetched += self.caches[l + 1].prefetch(pred, self.prefetch_max, self.copy)
            y = torch.empty_like(x)
            t0 = self._mark()
            moeq.moe_unpermute_combine(v["y_perm"], v["inv_perm"], v["topk_w"], residual=x, y=y)
            self._segment(t0)
            stats.append(st + [n_waves])
            x = y
        return x, stats

    def _bits_for(self, bits_host):
        """Widths for moe_slot_stage: only a plane-mode cache uses them."""
        return bits_host.reshape(-1) if self.plane_staging else None

    def pregate(self, x, forced_ids=None):
        """Every layer's expert ids for the step from the step's input (each
        layer's router applied to x; or the forced ids) as int32
        [layers][batch][k] on the device; for nested layers also the widths,
        each layer's bit gate applied to x at those ids (uint8, same shape;
        else None)."""
        for l, layer in enumerate(self.layers):
            v = layer.views(self.batch)
            if forced_ids is None:
                moeq.moe_route_topk(x, layer.w_router, layer.bias, self.shape.k, topk_idx=self.ids_pregated[l],
                                    topk_w=v["topk_w"], workspace=v["route_ws"])
            if self.nested:
                moeq.moe_bit_gate(x, layer.w_bit, layer.bias_bit,
                                  self.ids_pregated[l] if forced_ids is None else forced_ids[l].contiguous(),
                                  bits=self.bits_pregated[l], status=v["status"])
        ids = self.ids_pregated if forced_ids is None else forced_ids
        return ids, (self.bits_pregated if self.nested else None)

    def _step_lookahead(self, x, forced_ids):
        sh, stats = self.shape, []
        ids, bits_all = self.pregate(x, forced_ids)
        # the one device -> host crossing per step: all layers' ids (and widths)
        ev = torch.cuda.Event()
        ev.record(self.compute)
        self.side.wait_event(ev)
        with torch.cuda.stream(self.side):
            self.ids_all_host.copy_(ids, non_blocking=True)
            if bits_all is not None:
                self.bits_all_host.copy_(bits_all, non_blocking=True)
        self.side.synchronize()
        for l, layer in enumerate(self.layers):
            copy = self.copy if l % 2 == 0 else self.copy2
            v = layer.views(self.batch)
            t0 = self._mark()
            moeq.moe_route_topk(x, layer.w_router, layer.bias, sh.k, forced_idx=ids[l].contiguous(),
                                topk_idx=v["topk_idx"], topk_w=v["topk_w"], workspace=v["route_ws"])
            moeq.moe_permute(v["topk_idx"], sh.E, bits=None if bits_all is None else bits_all[l], x=x, out=v,
                             status=v["status"])
            self._segment(t0)
            n_waves, st = self.caches[l].stage(self.ids_all_host[l].reshape(-1), copy, self.compute,
                                               bits_host=self._bits_for(self.bits_all_host[l]))
            self.caches[l].ffn(v["x_perm"], v["offsets"], self.batch, sh.d, sh.F, sh.group, layer.layout,
                               v["workspace"], v["y_perm"], v["status"], copy, self.compute)
            y = torch.empty_like(x)
            t0 = self._mark()
            moeq.moe_unpermute_combine(v["y_perm"], v["inv_perm"], v["topk_w"], residual=x, y=y)
            self._segment(t0)
            stats.append(st + [n_waves])
            x = y
        return x, stats

    def close(self):
        for c in self.caches:
            c.close()
        self.caches = []
        if self.predictor is not None:
            self.predictor.close()
            self.predictor = None
