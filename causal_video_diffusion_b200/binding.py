"""ctypes binding of ``libunstep.so`` (include/unstep.h).

Argument marshalling only: torch tensors are turned into device pointers and the current CUDA
stream, shapes are checked against the cache, and every step of the layer runs inside the
library's kernels.  There is no fallback: if the library cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libunstep.so")

UNSTEP_OK = 0
UNSTEP_ERR_ARG = -1
UNSTEP_ERR_SHAPE = -2
UNSTEP_ERR_ALIGN = -3
UNSTEP_ERR_FRAME_ORDER = -4
UNSTEP_ERR_WINDOW = -5
UNSTEP_ERR_UNSUPPORTED = -6
UNSTEP_ERR_CUDA = -7
UNSTEP_ERR_DEVICE_TIMEOUT = -8
UNSTEP_ERR_SCRATCH_LIMIT = -9
UNSTEP_ERR_DEVICE_BOUNDS = -10

UNSTEP_APPEND_DEFER_Q_ROPE = 1   # unstep_rope_kv_append_ex: leave q alone
UNSTEP_ATTN_ROPE_Q = 1           # unstep_window_attn_ex: q is un-rotated, rotate it in-kernel


class unstep_cache_t(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("D", ctypes.c_int),
        ("Hg", ctypes.c_int), ("Wg", ctypes.c_int),
        ("d_t", ctypes.c_int), ("d_h", ctypes.c_int), ("d_w", ctypes.c_int),
        ("theta", ctypes.c_double),
        ("cap_frames", ctypes.c_int), ("max_pos_t", ctypes.c_int),
        ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
        ("slot_frame", ctypes.c_void_p), ("cos_sin", ctypes.c_void_p),
        ("dev_error", ctypes.c_void_p),
        ("attn_scratch", ctypes.c_void_p), ("attn_scratch_bytes", ctypes.c_size_t),
        ("frames_written", ctypes.c_int), ("first_frame", ctypes.c_int),
        ("last_chunk_start", ctypes.c_int), ("last_chunk_frames", ctypes.c_int),
        ("initialized", ctypes.c_int),
        ("act_B", ctypes.c_int), ("act_H", ctypes.c_int),
        ("b0", ctypes.c_int), ("h0", ctypes.c_int),
    ]


class unstep_grid_t(ctypes.Structure):
    _fields_ = [("frames", ctypes.c_int), ("Hg", ctypes.c_int), ("Wg", ctypes.c_int)]


class unstep_window_plan_t(ctypes.Structure):
    _fields_ = [("first_frame", ctypes.c_int), ("last_frame", ctypes.c_int),
                ("keys", ctypes.c_int), ("seg_row", ctypes.c_int * 2),
                ("seg_len", ctypes.c_int * 2)]


# every symbol include/unstep.h declares, with its ctypes signature
_SIGNATURES = {
    "unstep_version": ([], ctypes.c_int),
    "unstep_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "unstep_cache_table_bytes": ([ctypes.POINTER(unstep_cache_t)], ctypes.c_size_t),
    "unstep_cache_kv_bytes": ([ctypes.POINTER(unstep_cache_t)], ctypes.c_size_t),
    "unstep_attn_scratch_bytes": ([ctypes.POINTER(unstep_cache_t)], ctypes.c_size_t),
    "unstep_cache_init": ([ctypes.POINTER(unstep_cache_t), ctypes.c_void_p], ctypes.c_int),
    "unstep_append_plan": ([ctypes.POINTER(unstep_cache_t), ctypes.c_int, unstep_grid_t,
                            ctypes.POINTER(ctypes.c_int)], ctypes.c_int),
    "unstep_rope_kv_append": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                               ctypes.POINTER(unstep_cache_t), ctypes.c_int, unstep_grid_t,
                               ctypes.c_void_p], ctypes.c_int),
    "unstep_rope_kv_append_ex": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.POINTER(unstep_cache_t), ctypes.c_int, unstep_grid_t,
                                  ctypes.c_uint, ctypes.c_void_p], ctypes.c_int),
    "unstep_window_plan": ([ctypes.POINTER(unstep_cache_t), ctypes.c_int,
                            ctypes.POINTER(unstep_window_plan_t)], ctypes.c_int),
    "unstep_window_attn": ([ctypes.c_void_p, ctypes.POINTER(unstep_cache_t), ctypes.c_int,
                            ctypes.c_void_p, ctypes.c_void_p], ctypes.c_int),
    "unstep_window_attn_ex": ([ctypes.c_void_p, ctypes.POINTER(unstep_cache_t), ctypes.c_int,
                               ctypes.c_void_p, ctypes.c_uint, ctypes.c_void_p], ctypes.c_int),
    "unstep_window_attn_noalloc": ([ctypes.c_void_p, ctypes.POINTER(unstep_cache_t),
                                    ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p],
                                   ctypes.c_int),
    "unstep_gemm_bf16": ([ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int,
                          ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                          ctypes.c_void_p, ctypes.c_void_p], ctypes.c_int),
    "unstep_lowrank_linear": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                               ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                               ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p], ctypes.c_int),
    "unstep_renoise": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong,
                        ctypes.c_float, ctypes.c_void_p], ctypes.c_int),
    "unstep_conv3d_causal": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                              ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                              ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                              ctypes.c_void_p], ctypes.c_int),
    "unstep_conv3d_scratch_bytes": ([], ctypes.c_size_t),
    "unstep_cache_state_bytes": ([ctypes.POINTER(unstep_cache_t)], ctypes.c_size_t),
    "unstep_cache_save": ([ctypes.POINTER(unstep_cache_t), ctypes.c_void_p, ctypes.c_size_t,
                           ctypes.c_void_p], ctypes.c_int),
    "unstep_cache_restore": ([ctypes.POINTER(unstep_cache_t), ctypes.c_void_p, ctypes.c_size_t,
                              ctypes.c_void_p], ctypes.c_int),
    "unstep_get_device_error": ([ctypes.POINTER(unstep_cache_t), ctypes.c_void_p], ctypes.c_int),
    "unstep_selftest_wait_timeout": ([ctypes.c_void_p, ctypes.c_uint64, ctypes.c_void_p],
                                     ctypes.c_int),
    "unstep_selftest_exp2": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                              ctypes.c_void_p], ctypes.c_int),
}

_LIB: Optional[ctypes.CDLL] = None


class UnstepError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})" if what else
                         f"{status_string(status)} ({status})")


def lib() -> ctypes.CDLL:
    """Load libunstep.so; raises if it is missing (build it with causal_video_diffusion_b200.build)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: the CUDA library has not been built "
                               "(python -m causal_video_diffusion_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _LIB = L
    return _LIB


def status_string(rc: int) -> str:
    try:
        return lib().unstep_status_string(int(rc)).decode()
    except Exception:  # noqa: BLE001 - used while formatting an error
        return "status"


def _check(rc: int, what: str) -> int:
    if rc < 0:
        raise UnstepError(rc, what)
    return rc


def _stream_handle(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _dev_ptr(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return int(t.data_ptr())


class LayerCache:
    """One attention layer's ring-buffer KV cache and RoPE tables, in caller-owned torch memory.

    All device memory is allocated here by torch; the library only reads and writes it.

    ``shard=(b0, h0, act_B, act_H)`` makes this cache one shard of a larger layer: it holds
    streams ``b0 .. b0+B-1`` and heads ``h0 .. h0+H-1`` of activations shaped
    ``[act_B][L][act_H][D]``, and its calls read and write only those rows of q, k, v and out.
    """

    def __init__(self, B: int, H: int, D: int, Hg: int, Wg: int, d_t: int, d_h: int, d_w: int,
                 cap_frames: int, max_pos_t: int, theta: float = 10000.0,
                 device: Optional[torch.device] = None,
                 stream: Optional[torch.cuda.Stream] = None,
                 scratch: Optional[torch.Tensor] = None, use_scratch: bool = True,
                 shard: Optional[Tuple[int, int, int, int]] = None):
        L = lib()
        dev = torch.device(device) if device is not None else torch.device("cuda",
                                                                           torch.cuda.current_device())
        c = unstep_cache_t()
        c.B, c.H, c.D, c.Hg, c.Wg = B, H, D, Hg, Wg
        c.d_t, c.d_h, c.d_w, c.theta = d_t, d_h, d_w, float(theta)
        c.cap_frames, c.max_pos_t = cap_frames, max_pos_t
        # an unsharded cache leaves the shard fields at zero (the activations are [B][L][H][D])
        b0, h0, act_B, act_H = shard if shard is not None else (0, 0, B, H)
        if shard is not None:
            c.b0, c.h0, c.act_B, c.act_H = b0, h0, act_B, act_H
        self.act_B, self.act_H = act_B, act_H
        tab_bytes = L.unstep_cache_table_bytes(ctypes.byref(c))
        if tab_bytes == 0:
            raise UnstepError(UNSTEP_ERR_ARG, "cache shape rejected")
        self.Tf = Hg * Wg
        self.rows = cap_frames * self.Tf
        self.k_cache = torch.empty((B, H, self.rows, D), dtype=torch.bfloat16, device=dev)
        self.v_cache = torch.empty_like(self.k_cache)
        self.slot_frame = torch.empty((cap_frames,), dtype=torch.int32, device=dev)
        self.cos_sin = torch.empty((tab_bytes // 4,), dtype=torch.float32, device=dev)
        self.dev_error = torch.zeros((1,), dtype=torch.int32, device=dev)
        c.k_cache = self.k_cache.data_ptr()
        c.v_cache = self.v_cache.data_ptr()
        c.slot_frame = self.slot_frame.data_ptr()
        c.cos_sin = self.cos_sin.data_ptr()
        c.dev_error = self.dev_error.data_ptr()
        # attention scratch: given (shared between caches on one stream), or allocated here
        self.scratch = None
        if use_scratch:
            with torch.cuda.device(dev):
                need = L.unstep_attn_scratch_bytes(ctypes.byref(c))
            if need == 0:
                raise UnstepError(UNSTEP_ERR_ARG, "attention scratch size")
            if scratch is None:
                scratch = torch.empty((need,), dtype=torch.uint8, device=dev)
            if scratch.numel() * scratch.element_size() < need:
                raise ValueError(f"scratch has {scratch.numel() * scratch.element_size()} bytes, "
                                 f"needs {need}")
            self.scratch = scratch
            c.attn_scratch = scratch.data_ptr()
            c.attn_scratch_bytes = scratch.numel() * scratch.element_size()
        self.c = c
        self.device = dev
        with torch.cuda.device(dev):
            _check(L.unstep_cache_init(ctypes.byref(c), _stream_handle(stream)),
                   "unstep_cache_init")

    def reset(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        """Back to an empty cache (zeroed K/V, no frames), as after construction."""
        with torch.cuda.device(self.device):
            _check(lib().unstep_cache_init(ctypes.byref(self.c), _stream_handle(stream)),
                   "unstep_cache_init")

    # -- metadata ---------------------------------------------------------------------------
    @property
    def shape(self):
        c = self.c
        return c.B, c.H, c.D

    @property
    def frames_written(self) -> int:
        return self.c.frames_written

    @property
    def last_chunk(self):
        return self.c.last_chunk_start, self.c.last_chunk_frames

    def chunk_len(self, frames: int) -> int:
        return frames * self.Tf

    def _check_act(self, t: torch.Tensor, L: int, name: str):
        c = self.c
        if t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be bfloat16")
        want = (self.act_B, L, self.act_H, c.D)
        if tuple(t.shape) != want:
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {want}")
        if t.device != self.device:
            raise ValueError(f"{name} is on {t.device}, the cache on {self.device}")

    # -- the library calls ------------------------------------------------------------------
    def append_plan(self, frame_idx: int, frames: int):
        slots = (ctypes.c_int * max(1, frames))()
        g = unstep_grid_t(frames, self.c.Hg, self.c.Wg)
        rc = lib().unstep_append_plan(ctypes.byref(self.c), int(frame_idx), g, slots)
        _check(rc, "unstep_append_plan")
        return bool(rc), list(slots)[:frames]

    def window_plan(self, window: int) -> unstep_window_plan_t:
        plan = unstep_window_plan_t()
        _check(lib().unstep_window_plan(ctypes.byref(self.c), int(window), ctypes.byref(plan)),
               "unstep_window_plan")
        return plan

    def rope_kv_append(self, q: Optional[torch.Tensor], k: torch.Tensor, v: torch.Tensor,
                       frame_idx: int, frames: int,
                       stream: Optional[torch.cuda.Stream] = None,
                       defer_q: bool = False) -> Optional[torch.Tensor]:
        """Rotate q in place, append rotated k and v to the ring; returns q.

        ``defer_q``: q is left alone (it may be None) and only k, v are processed; the queries
        are then rotated inside :meth:`window_attn` with ``rope_q=True``.
        """
        L = self.chunk_len(frames)
        acts = ((k, "k"), (v, "v")) if defer_q and q is None else ((q, "q"), (k, "k"), (v, "v"))
        for t, n in acts:
            self._check_act(t, L, n)
        g = unstep_grid_t(frames, self.c.Hg, self.c.Wg)
        qp = None if q is None else _dev_ptr(q, "q")
        if defer_q:
            rc = lib().unstep_rope_kv_append_ex(qp, _dev_ptr(k, "k"), _dev_ptr(v, "v"),
                                                ctypes.byref(self.c), int(frame_idx), g,
                                                UNSTEP_APPEND_DEFER_Q_ROPE,
                                                _stream_handle(stream))
            _check(rc, "unstep_rope_kv_append_ex")
        else:
            rc = lib().unstep_rope_kv_append(qp, _dev_ptr(k, "k"), _dev_ptr(v, "v"),
                                             ctypes.byref(self.c), int(frame_idx), g,
                                             _stream_handle(stream))
            _check(rc, "unstep_rope_kv_append")
        return q

    def window_attn(self, q: torch.Tensor, window: int, out: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None,
                    rope_q: bool = False) -> torch.Tensor:
        """Attention of the latest chunk's queries over the last ``window`` frames.

        q is the rotated queries (as :meth:`rope_kv_append` leaves them), or with ``rope_q`` the
        un-rotated ones, which the kernel rotates after loading them.
        """
        L = self.chunk_len(self.c.last_chunk_frames)
        self._check_act(q, L, "q")
        if out is None:
            out = torch.empty_like(q)
        self._check_act(out, L, "out")
        if rope_q:
            rc = lib().unstep_window_attn_ex(_dev_ptr(q, "q"), ctypes.byref(self.c), int(window),
                                             _dev_ptr(out, "out"), UNSTEP_ATTN_ROPE_Q,
                                             _stream_handle(stream))
            _check(rc, "unstep_window_attn_ex")
        else:
            rc = lib().unstep_window_attn(_dev_ptr(q, "q"), ctypes.byref(self.c), int(window),
                                          _dev_ptr(out, "out"), _stream_handle(stream))
            _check(rc, "unstep_window_attn")
        return out

    # -- checkpoint / resume -----------------------------------------------------------------
    def state_bytes(self) -> int:
        return lib().unstep_cache_state_bytes(ctypes.byref(self.c))

    def save_state(self, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """The layer's state (ring K/V rows, slot_frame, metadata) in a pinned host buffer."""
        buf = torch.empty((self.state_bytes(),), dtype=torch.uint8).pin_memory()
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        with torch.cuda.device(self.device):
            _check(lib().unstep_cache_save(ctypes.byref(self.c), buf.data_ptr(), buf.numel(),
                                           _stream_handle(s)), "unstep_cache_save")
        s.synchronize()
        return buf

    def restore_state(self, buf: torch.Tensor, stream: Optional[torch.cuda.Stream] = None):
        """Continue the stream a :meth:`save_state` buffer describes (same shape required)."""
        if buf.device.type != "cpu" or buf.dtype != torch.uint8 or not buf.is_contiguous():
            raise ValueError("state must be a contiguous uint8 host tensor")
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        with torch.cuda.device(self.device):
            _check(lib().unstep_cache_restore(ctypes.byref(self.c), buf.data_ptr(), buf.numel(),
                                              _stream_handle(s)), "unstep_cache_restore")
        s.synchronize()     # the host buffer may be reused once the copies have run

    def device_error(self, stream: Optional[torch.cuda.Stream] = None) -> int:
        return lib().unstep_get_device_error(ctypes.byref(self.c), _stream_handle(stream))

    def step_from_host(self, q_h: torch.Tensor, k_h: torch.Tensor, v_h: torch.Tensor,
                       frame_idx: int, frames: int, window: int, out_h: torch.Tensor,
                       bufs: dict, stream: Optional[torch.cuda.Stream] = None,
                       rope_q_in_attn: bool = False) -> torch.Tensor:
        """One layer step from pinned host tensors: copy in, append, attend, copy out.

        ``bufs`` holds the device staging tensors ``q``, ``k``, ``v``, ``out`` (reused).
        The copies and both calls are enqueued on the stream; ``out_h`` is valid after a sync.
        ``rope_q_in_attn``: deferred-q append, queries rotated inside the attention.
        """
        s = stream if stream is not None else torch.cuda.current_stream()
        with torch.cuda.stream(s):
            bufs["q"].copy_(q_h, non_blocking=True)
            bufs["k"].copy_(k_h, non_blocking=True)
            bufs["v"].copy_(v_h, non_blocking=True)
            self.rope_kv_append(bufs["q"], bufs["k"], bufs["v"], frame_idx, frames, stream=s,
                                defer_q=rope_q_in_attn)
            self.window_attn(bufs["q"], window, out=bufs["out"], stream=s, rope_q=rope_q_in_attn)
            out_h.copy_(bufs["out"], non_blocking=True)
        return out_h


class HostStepPipeline:
    """Layer steps fed from pinned host memory, with copies overlapped with compute.

    Step i copies its q, k, v host->device on one copy stream, runs ``rope_kv_append`` and
    ``window_attn`` on the compute stream, and copies its output device->host on a second copy
    stream; two sets of device buffers alternate, so step i+1's input copy and step i-1's output
    copy run while step i computes.  Every step still moves all of its inputs and its output
    across the host link.
    """

    def __init__(self, cache: LayerCache, device=None, rope_q_in_attn: bool = False):
        c = cache.c
        dev = cache.device if device is None else torch.device(device)
        self.cache = cache
        self.rope_q_in_attn = rope_q_in_attn   # deferred-q append + in-kernel query RoPE
        self.h2d = torch.cuda.Stream(device=dev)
        self.d2h = torch.cuda.Stream(device=dev)
        self.compute = torch.cuda.Stream(device=dev)
        self.device = dev
        self.sets = []
        self.c = c

    def _bufs(self, L: int):
        c = self.c
        if not self.sets or self.sets[0]["q"].shape[1] != L:
            act = (self.cache.act_B, L, self.cache.act_H, c.D)
            self.sets = [{n: torch.empty(act, dtype=torch.bfloat16,
                                         device=self.device) for n in ("q", "k", "v", "out")}
                         for _ in range(2)]
        return self.sets

    def run(self, q_h: torch.Tensor, k_h: torch.Tensor, v_h: torch.Tensor, frame_idx: int,
            frames: int, window: int, out_h: torch.Tensor, steps: int) -> float:
        """Run ``steps`` steps (the same chunk re-forwarded; inputs copied every step) and return
        the device time in ms from the first input copy to the last output copy."""
        sets = self._bufs(q_h.shape[1])
        ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
        start, end = ev(), ev()
        in_ready = [None, None]
        computed = [None, None]
        out_done = [None, None]
        torch.cuda.synchronize(self.device)
        start.record(self.h2d)
        for i in range(steps):
            b = i & 1
            bufs = sets[b]
            with torch.cuda.stream(self.h2d):
                if computed[b] is not None:
                    self.h2d.wait_event(computed[b])   # the set's previous step is done with it
                bufs["q"].copy_(q_h, non_blocking=True)
                bufs["k"].copy_(k_h, non_blocking=True)
                bufs["v"].copy_(v_h, non_blocking=True)
                in_ready[b] = ev()
                in_ready[b].record(self.h2d)
            with torch.cuda.stream(self.compute):
                self.compute.wait_event(in_ready[b])
                if out_done[b] is not None:
                    self.compute.wait_event(out_done[b])  # its output has left the device
                fq = self.rope_q_in_attn
                self.cache.rope_kv_append(bufs["q"], bufs["k"], bufs["v"], frame_idx, frames,
                                          stream=self.compute, defer_q=fq)
                self.cache.window_attn(bufs["q"], window, out=bufs["out"], stream=self.compute,
                                       rope_q=fq)
                computed[b] = ev()
                computed[b].record(self.compute)
            with torch.cuda.stream(self.d2h):
                self.d2h.wait_event(computed[b])
                out_h.copy_(bufs["out"], non_blocking=True)
                out_done[b] = ev()
                out_done[b].record(self.d2h)
        self.h2d.wait_stream(self.d2h)
        self.h2d.wait_stream(self.compute)
        end.record(self.h2d)
        end.synchronize()
        return start.elapsed_time(end)


def _err_word(dev_error: Optional[torch.Tensor], like: torch.Tensor) -> torch.Tensor:
    if dev_error is None:
        dev_error = torch.zeros(1, dtype=torch.int32, device=like.device)
    return dev_error


def gemm_bf16(a: torch.Tensor, b: torch.Tensor, out: Optional[torch.Tensor] = None,
              dev_error: Optional[torch.Tensor] = None,
              stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """out[M][N] = a[M][K] @ b[N][K]^T on the tensor cores (bf16 in, fp32 accumulate, bf16 out)."""
    for t, n in ((a, "a"), (b, "b")):
        if t.dtype != torch.bfloat16 or t.dim() != 2:
            raise ValueError(f"{n} must be a 2-D bfloat16 tensor")
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K:
        raise ValueError("a and b disagree on K")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    err = _err_word(dev_error, a)
    _check(lib().unstep_gemm_bf16(_dev_ptr(a, "a"), K, _dev_ptr(b, "b"), K, _dev_ptr(out, "out"),
                                  N, M, N, K, _dev_ptr(err, "dev_error"), _stream_handle(stream)),
           "unstep_gemm_bf16")
    return out


def conv3d_scratch(device: Optional[torch.device] = None) -> torch.Tensor:
    """A zero-filled scratch buffer for conv3d_causal's stream-K tail on `device` (its size
    depends on the device's SM count only).  Calls sharing one buffer must be ordered."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        need = int(lib().unstep_conv3d_scratch_bytes())
    if need <= 0:
        raise UnstepError(UNSTEP_ERR_CUDA, "unstep_conv3d_scratch_bytes")
    return torch.zeros((need,), dtype=torch.uint8, device=dev)


def conv3d_causal(x: torch.Tensor, w: torch.Tensor, bias: Optional[torch.Tensor] = None,
                  out: Optional[torch.Tensor] = None, dev_error: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None,
                  scratch: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Causal 3x3x3 convolution, channels-last, on the tensor cores.

    x [B][T+2][H][W][C_in] bf16 (each stream's first two frames are its causal history),
    w [C_out][3][3][3][C_in] bf16, bias [C_out] fp32 or None -> y [B][T][H][W][C_out] bf16.
    scratch: a conv3d_scratch() buffer to split the last partial wave of tiles over all SMs
    (stream-K), or None to run every tile whole.
    """
    if x.dtype != torch.bfloat16 or x.dim() != 5 or w.dtype != torch.bfloat16 or w.dim() != 5:
        raise ValueError("x and w must be 5-D bfloat16 tensors")
    B, Tin, H, Wd, C_in = x.shape
    C_out = w.shape[0]
    if tuple(w.shape[1:]) != (3, 3, 3, C_in):
        raise ValueError(f"w has shape {tuple(w.shape)}, expected {(C_out, 3, 3, 3, C_in)}")
    if Tin < 3:
        raise ValueError("x needs the two history frames and at least one frame")
    if bias is not None and (bias.dtype != torch.float32 or tuple(bias.shape) != (C_out,)):
        raise ValueError("bias must be float32 [C_out]")
    if out is None:
        out = torch.empty((B, Tin - 2, H, Wd, C_out), dtype=torch.bfloat16, device=x.device)
    err = _err_word(dev_error, x)
    bp = None if bias is None else _dev_ptr(bias, "bias")
    sp, sb = None, 0
    if scratch is not None:
        sp, sb = _dev_ptr(scratch, "scratch"), scratch.numel() * scratch.element_size()
    _check(lib().unstep_conv3d_causal(_dev_ptr(x, "x"), _dev_ptr(w, "w"), bp, _dev_ptr(out, "out"),
                                      B, Tin - 2, H, Wd, C_in, C_out, sp, sb,
                                      _dev_ptr(err, "dev_error"), _stream_handle(stream)),
           "unstep_conv3d_causal")
    return out


def lowrank_linear(x: torch.Tensor, w1: torch.Tensor, w2: torch.Tensor,
                   t: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                   dev_error: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """y = (x @ w1^T) @ w2^T: a linear layer through its truncated-SVD factors."""
    M, d_in = x.shape
    rank = w1.shape[0]
    d_out = w2.shape[0]
    if w1.shape[1] != d_in or w2.shape[1] != rank:
        raise ValueError("factor shapes do not chain")
    for tt, n in ((x, "x"), (w1, "w1"), (w2, "w2")):
        if tt.dtype != torch.bfloat16:
            raise ValueError(f"{n} must be bfloat16")
    if t is None:
        t = torch.empty((M, rank), dtype=torch.bfloat16, device=x.device)
    if y is None:
        y = torch.empty((M, d_out), dtype=torch.bfloat16, device=x.device)
    err = _err_word(dev_error, x)
    _check(lib().unstep_lowrank_linear(_dev_ptr(x, "x"), _dev_ptr(w1, "w1"), _dev_ptr(w2, "w2"),
                                       _dev_ptr(t, "t"), _dev_ptr(y, "y"), M, d_in, rank, d_out,
                                       _dev_ptr(err, "dev_error"), _stream_handle(stream)),
           "unstep_lowrank_linear")
    return y


def renoise(x0: torch.Tensor, eps: torch.Tensor, sigma: float,
            out: Optional[torch.Tensor] = None,
            stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """out = (1 - sigma) * x0 + sigma * eps (bf16 latents of any shape)."""
    if x0.dtype != torch.bfloat16 or eps.dtype != torch.bfloat16 or x0.shape != eps.shape:
        raise ValueError("x0 and eps must be bf16 tensors of one shape")
    if out is None:
        out = torch.empty_like(x0)
    _check(lib().unstep_renoise(_dev_ptr(x0, "x0"), _dev_ptr(eps, "eps"), _dev_ptr(out, "out"),
                                x0.numel(), float(sigma), _stream_handle(stream)),
           "unstep_renoise")
    return out


def selftest_wait_timeout(dev_error: torch.Tensor, limit_ns: int,
                          stream: Optional[torch.cuda.Stream] = None) -> None:
    _check(lib().unstep_selftest_wait_timeout(_dev_ptr(dev_error, "dev_error"), int(limit_ns),
                                              _stream_handle(stream)),
           "unstep_selftest_wait_timeout")


def selftest_exp2(x: torch.Tensor, stream: Optional[torch.cuda.Stream] = None):
    """(polynomial, hardware) base-2 exponentials of the fp32 device tensor x."""
    if x.dtype != torch.float32:
        raise ValueError("x must be float32")
    yp = torch.empty_like(x)
    ym = torch.empty_like(x)
    _check(lib().unstep_selftest_exp2(_dev_ptr(x, "x"), _dev_ptr(yp, "y_poly"),
                                      _dev_ptr(ym, "y_mufu"), x.numel(), _stream_handle(stream)),
           "unstep_selftest_exp2")
    return yp, ym


def declared_symbols(header: Optional[str] = None):
    """Function names declared in include/unstep.h (parsed from the header text)."""
    import re
    header = header or os.path.join(os.path.dirname(_HERE), "include", "unstep.h")
    text = open(header).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\**\s*(unstep_[a-z_0-9]+)\s*\(",
                                 text, flags=re.M)))
