"""A whole 5-s clip through the attention layers, optionally captured as one CUDA graph.

UnStep paper (arXiv 2609.32518), Table 3: a clip is seven causal chunks of three latent frames;
every chunk runs its denoising steps plus one clean-cache pass (23 DiT forwards with UnStep,
35 with the original four-step schedule), and every forward runs every layer.  Each layer's part
of the hot path is ``rope_kv_append`` + ``window_attn`` on that layer's own ring cache; after each
forward the chunk's latent is renoised to the next noise level (``schedule``), the last time to
the near-clean level of the clean-cache pass.  The DiT's own projections and prediction are not
part of this library: q, k, v of every (forward, layer) and the clean-latent prediction are
seeded synthetic tensors, generated on the device before the clip runs.
"""
from __future__ import annotations

from typing import Callable, List, Optional

import torch

from . import binding
from . import schedule as S
from . import workloads as W

LATENT_CHANNELS = 16


class ClipDriver:
    def __init__(self, workload: W.Workload, layers: Optional[int] = None, kind: str = "unstep",
                 seed: int = 0, device: Optional[torch.device] = None):
        self.wl = workload
        self.shape = s = workload.shape
        self.layers = workload.layers if layers is None else layers
        self.sched = S.clip_schedule(kind, workload.chunks)
        self.device = dev = torch.device(device) if device is not None else torch.device(
            "cuda", torch.cuda.current_device())
        first = binding.LayerCache(s.B, s.H, s.D, s.Hg, s.Wg, s.d_t, s.d_h, s.d_w,
                                   cap_frames=workload.cap,
                                   max_pos_t=workload.frame_idx(workload.chunks), device=dev)
        # one attention scratch for every layer: their calls are ordered on one stream
        self.caches = [first] + [
            binding.LayerCache(s.B, s.H, s.D, s.Hg, s.Wg, s.d_t, s.d_h, s.d_w,
                               cap_frames=workload.cap,
                               max_pos_t=workload.frame_idx(workload.chunks), device=dev,
                               scratch=first.scratch)
            for _ in range(self.layers - 1)]
        self.inputs = []   # [forward][layer] -> (q, k, v)
        for n, f in enumerate(self.sched):
            row = []
            for layer in range(self.layers):
                row.append(W.gen_qkv(W.qkv_seed(seed, layer=layer, chunk=f.chunk,
                                                forward=n), s, device=str(dev)))
            self.inputs.append(row)
        self.outs = [torch.empty((s.B, s.L, s.H, s.D), dtype=torch.bfloat16, device=dev)
                     for _ in range(self.layers)]
        lat = (s.B, s.chunk_frames, LATENT_CHANNELS, 2 * s.Hg, 2 * s.Wg)
        g = torch.Generator(device=dev)
        g.manual_seed(seed + 99)
        self.x_hat = torch.randn(lat, generator=g, device=dev).to(torch.bfloat16)
        self.eps = [torch.randn(lat, generator=g, device=dev).to(torch.bfloat16)
                    for _ in self.sched]
        self.latent = torch.empty(lat, dtype=torch.bfloat16, device=dev)
        self.graph: Optional[torch.cuda.CUDAGraph] = None

    @property
    def calls(self) -> int:
        return len(self.sched) * self.layers

    def attn_flops(self) -> int:
        return sum(self.wl.attn_flops(f.chunk) for f in self.sched) * self.layers

    def reset(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        for c in self.caches:
            c.reset(stream=stream)

    def _issue(self, stream: Optional[torch.cuda.Stream] = None,
               on_forward: Optional[Callable[[int], None]] = None) -> None:
        F = self.shape.chunk_frames
        for n, f in enumerate(self.sched):
            f0 = self.wl.frame_idx(f.chunk)
            for layer, cache in enumerate(self.caches):
                q, k, v = self.inputs[n][layer]
                cache.rope_kv_append(q, k, v, f0, F, stream=stream)
                cache.window_attn(q, self.wl.window, out=self.outs[layer], stream=stream)
            binding.renoise(self.x_hat, self.eps[n], f.next_sigma, out=self.latent, stream=stream)
            if on_forward is not None:
                on_forward(n)

    def run(self, on_forward: Optional[Callable[[int], None]] = None) -> None:
        """One clip, eagerly (each call launched from the host as it comes).  ``on_forward(n)``
        runs on the host after forward n's calls are enqueued (e.g. to copy its outputs)."""
        self._issue(on_forward=on_forward)

    def capture(self) -> torch.cuda.CUDAGraph:
        """Capture one clip as a CUDA graph (call reset() before replaying it)."""
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self._issue(stream=torch.cuda.current_stream())
        return self.graph

    def replay(self) -> None:
        assert self.graph is not None
        self.graph.replay()
