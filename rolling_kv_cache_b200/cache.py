"""User-facing Python API over the C ABI.

``RollingKVCache`` owns one rc handle and its device memory block (a torch
uint8 tensor; torch is used only for memory and streams). ``step`` runs one
chunk through one layer in the library's kernels; it accepts device tensors,
or host tensors (pinned for speed), in which case it copies them to the
device, runs the step and copies the output back.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import binding as B


def make_config(*, layers: int, heads: int, head_dim: int, grid_h: int, grid_w: int,
                sink_frames: int, window_frames: int, chunk_frames: int = 3,
                policy: int = B.RC_SLIDING, mask_block_frames: int = 1, theta: float = 10000.0,
                t_max: int = 4096, rope_pairs=(0, 0, 0), rs_bank_blocks: int = 0,
                rs_sink_blocks: int = 0, rs_static_semantics: int = 0, ir_f_limit: int = 0,
                ir_sink_blocks: int = 0, ir_cache_blocks: int = 0,
                df_budget_tokens: int = 0, rf_history_frames: int = 0,
                rf_weight: float = 0.5, mr_alpha_long: float = 0.0,
                mr_alpha_short: float = 0.0) -> B.rc_config:
    cfg = B.rc_config_init(layers, heads, head_dim, grid_h * grid_w, sink_frames, window_frames)
    cfg.grid_h, cfg.grid_w = grid_h, grid_w
    cfg.chunk_frames = chunk_frames
    cfg.policy = policy
    cfg.mask_block_frames = mask_block_frames
    cfg.theta = theta
    cfg.t_max = t_max
    cfg.rope_t_pairs, cfg.rope_h_pairs, cfg.rope_w_pairs = rope_pairs
    cfg.rs_bank_blocks, cfg.rs_sink_blocks = rs_bank_blocks, rs_sink_blocks
    cfg.rs_static_semantics = rs_static_semantics
    cfg.ir_f_limit, cfg.ir_sink_blocks, cfg.ir_cache_blocks = ir_f_limit, ir_sink_blocks, ir_cache_blocks
    cfg.df_budget_tokens = df_budget_tokens
    cfg.rf_history_frames, cfg.rf_weight = rf_history_frames, rf_weight
    cfg.mr_alpha_long, cfg.mr_alpha_short = mr_alpha_long, mr_alpha_short
    return cfg


class RollingKVCache:
    """Bounded KV cache of every layer of one video stream.

    device=None creates a host-only handle (integer state only, no GPU).
    """

    def __init__(self, cfg: B.rc_config, device: Optional[torch.device] = torch.device("cuda"),
                 mem: Optional[torch.Tensor] = None):
        """``mem``: optional caller-owned uint8 device tensor of at least
        rc_cache_bytes(cfg) + 256 bytes to hold the cache (default: allocated
        here); the cache uses its first 256-byte-aligned rc_cache_bytes(cfg)
        bytes."""
        self.cfg = cfg
        self.nbytes = B.rc_cache_bytes(cfg)
        self.device = device
        self.mem = None
        ptr = 0
        if device is not None:
            if not torch.cuda.is_available():
                raise RuntimeError("a device cache needs CUDA")
            if mem is None:
                mem = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device)
            elif (mem.dtype != torch.uint8 or not mem.is_contiguous() or mem.device.type != "cuda"
                  or mem.numel() < self.nbytes + 256):
                raise ValueError("mem must be a contiguous uint8 CUDA tensor of rc_cache_bytes + 256 bytes")
            self.mem = mem
            ptr = (self.mem.data_ptr() + 255) // 256 * 256
        self.handle = B.rc_cache_create(cfg, ptr, self.nbytes)
        self._staging = {}

    def close(self) -> None:
        if getattr(self, "handle", None):
            B.rc_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass

    @property
    def policy(self) -> int:
        return self.cfg.policy

    def _stream(self) -> int:
        return torch.cuda.current_stream(self.device).cuda_stream if self.device is not None else 0

    def step(self, layer: int, q, k, v, frame_start: int, out=None, lse=None, scores=None,
             topc=None, C: int = 0):
        """One chunk through one layer. q/k/v: [n_frames*F, H, d] bf16.

        Host-only handles take q=k=v=None and only advance the state.
        Returns ``out`` ([n_frames*F, H, d] bf16).
        """
        F = self.cfg.frame_seqlen
        if self.device is None:
            B.rc_step(self.handle, layer, 0, 0, 0, frame_start, self._n_frames(q, frame_start),
                      self.cfg.policy, 0)
            return None
        host = not q.is_cuda
        if host:
            q = q.to(self.device, non_blocking=True)
            k = k.to(self.device, non_blocking=True)
            v = v.to(self.device, non_blocking=True)
        for t in (q, k, v):
            if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 3:
                raise ValueError("q/k/v must be contiguous [n_tok, H, d] bf16")
        n_tok = q.shape[0]
        if n_tok % F:
            raise ValueError("token count must be whole frames")
        if out is None or host:
            out_dev = torch.empty_like(q)
        else:
            out_dev = out
        B.rc_step(self.handle, layer, q.data_ptr(), k.data_ptr(), v.data_ptr(), frame_start,
                  n_tok // F, self.cfg.policy, out_dev.data_ptr(),
                  lse.data_ptr() if lse is not None else 0,
                  scores.data_ptr() if scores is not None else 0,
                  topc.data_ptr() if topc is not None else 0, C, self._stream())
        if host:
            if out is None:
                out = torch.empty(out_dev.shape, dtype=out_dev.dtype, pin_memory=True)
            out.copy_(out_dev, non_blocking=True)
            return out
        return out_dev

    def comp_tokens(self, layer: int = 0):
        """Deep Forcing: (frames, tokens) of the layer's compressed region, in
        region order (synchronizes the cache's stream)."""
        n = self.state(layer).comp_tokens
        return B.rc_comp_tokens(self.handle, layer, n, self._stream())

    def pool_scores(self, layer: int = 0):
        """Relax Forcing: scores of the pool at the layer's last frame selection
        (empty if its last new chunk needed none)."""
        return B.rc_pool_scores(self.handle, layer, self._stream())

    def select_topc(self, layer: int, scores, C: int, topc=None):
        """Top-C over ``scores`` ([n_candidates] fp32 on this device, e.g. the
        sum of the head shards' score vectors) in ``layer``'s candidate order
        of its last step. Returns ``topc`` ([C] int32)."""
        if self.device is None:
            raise ValueError("select_topc needs a device cache")
        if scores.dtype != torch.float32 or not scores.is_cuda or not scores.is_contiguous():
            raise ValueError("scores must be a contiguous fp32 device tensor")
        if topc is None:
            topc = torch.empty(C, dtype=torch.int32, device=self.device)
        B.rc_select_topc(self.handle, layer, scores.data_ptr(), C, topc.data_ptr(), self._stream())
        return topc

    def host_pipeline(self, depth: int = 2) -> "HostPipeline":
        """Pipelined stepping from host buffers (see HostPipeline)."""
        return HostPipeline(self, depth)

    def _n_frames(self, q, frame_start):
        return self.cfg.chunk_frames if q is None else q.shape[0] // self.cfg.frame_seqlen

    def reindex(self, t_delta: int, flags: int) -> None:
        B.rc_reindex(self.handle, self.cfg.policy, t_delta, flags, 0)

    def state(self, layer: int = 0) -> B.rc_state:
        return B.rc_get_state(self.handle, layer)

    def kept(self, layer: int = 0):
        """[(content, tau, region, rank, slot, stored_time)] in logical order."""
        st = self.state(layer)
        return [(e.content, e.tau, e.region, e.rank, e.slot, e.stored_time)
                for e in st.kept[:st.n_kept]]

    def device_status(self) -> None:
        B.rc_device_status(self.handle, self._stream())

    def _region(self, offset: int, nbytes: int) -> torch.Tensor:
        base = (self.mem.data_ptr() + 255) // 256 * 256 - self.mem.data_ptr()
        return self.mem[base + offset: base + offset + nbytes]

    def cache_views(self, layer: int):
        """(K, V) [H, capacity, d] bf16 of one layer's ring buffers.

        The buffers keep each head in 64-dim planes ([H][d/64][capacity][64]);
        for d > 64 the returned tensors are copies in token-major order (index
        [h, t, j] is dim j of token row t), for d = 64 views."""
        if self.mem is None:
            raise RuntimeError("host-only handle")
        lay = B.rc_cache_layout(self.handle)
        H, d = self.cfg.heads, self.cfg.head_dim
        P, cap = d // 64, lay.capacity
        n = H * cap * d * 2
        o = layer * lay.kv_layer_stride

        def logical(off):
            planes = self._region(off, n).view(torch.bfloat16).view(H, P, cap, 64)
            return planes.permute(0, 2, 1, 3).flatten(2) if P > 1 else planes.view(H, cap, 64)

        return logical(lay.k_offset + o), logical(lay.v_offset + o)

    def raw_views(self, layer: int):
        """(raw K, raw V or None) views [H, raw_frames*F, d] of the pristine source."""
        lay = B.rc_cache_layout(self.handle)
        H, d, F = self.cfg.heads, self.cfg.head_dim, self.cfg.frame_seqlen
        n = H * lay.raw_frames * F * d * 2
        o = layer * lay.raw_layer_stride
        rk = self._region(lay.raw_k_offset + o, n).view(torch.bfloat16).view(H, -1, d) if lay.raw_k_offset else None
        rv = self._region(lay.raw_v_offset + o, n).view(torch.bfloat16).view(H, -1, d) if lay.raw_v_offset else None
        return rk, rv

    def q_rot_view(self, n_tok: int):
        """Rotated queries [H, n_tok, d] of the last step (scratch; valid until the next step)."""
        lay = B.rc_cache_layout(self.handle)
        H, d = self.cfg.heads, self.cfg.head_dim
        stride = self.cfg.chunk_frames * self.cfg.frame_seqlen
        full = self._region(lay.q_offset, H * stride * d * 2).view(torch.bfloat16).view(H, stride, d)
        return full[:, :n_tok]

    def watchdog_selftest(self, limit_us: int = 20000) -> None:
        B.rc_watchdog_selftest(self.handle, limit_us, self._stream())


class HostPipeline:
    """Steps a cache from host (pinned) q/k/v into host output buffers with
    the transfers overlapped with the kernels.

    ``depth`` device staging sets are used round robin. Call i's upload runs
    on a copy-in stream while call i-1 computes on the cache's stream, and
    call i-1's output download runs on a copy-out stream while call i
    computes; events order each staging set's reuse. ``submit`` returns at
    once; ``synchronize`` waits for every download. Host buffers must stay
    untouched until their call's download is done (after ``synchronize``).
    """

    def __init__(self, cache: RollingKVCache, depth: int = 2):
        if cache.device is None:
            raise RuntimeError("host pipelines need a device cache")
        self.cache = cache
        self.depth = max(1, depth)
        dev = cache.device
        self.compute = torch.cuda.current_stream(dev)
        self.copy_in = torch.cuda.Stream(dev)
        self.copy_out = torch.cuda.Stream(dev)
        self.sets = []
        self.i = 0

    def _set(self, q):
        n = self.i % self.depth
        if len(self.sets) <= n:
            dev = self.cache.device
            self.sets.append(dict(
                q=torch.empty(q.shape, dtype=torch.bfloat16, device=dev),
                k=torch.empty(q.shape, dtype=torch.bfloat16, device=dev),
                v=torch.empty(q.shape, dtype=torch.bfloat16, device=dev),
                out=torch.empty(q.shape, dtype=torch.bfloat16, device=dev),
                read=None, downloaded=None))
        s = self.sets[n]
        if s["q"].shape != q.shape:
            raise ValueError("every call of a pipeline must have the same shape")
        return s

    def submit(self, layer: int, q, k, v, frame_start: int, out_host, lse=None, scores=None,
               topc=None, C: int = 0) -> None:
        s = self._set(q)
        # upload: staging inputs are free once the previous compute using them read them
        if s["read"] is not None:
            self.copy_in.wait_event(s["read"])
        with torch.cuda.stream(self.copy_in):
            s["q"].copy_(q, non_blocking=True)
            s["k"].copy_(k, non_blocking=True)
            s["v"].copy_(v, non_blocking=True)
            uploaded = torch.cuda.Event()
            uploaded.record(self.copy_in)
        # compute: needs the upload, and the staging output downloaded
        self.compute.wait_event(uploaded)
        if s["downloaded"] is not None:
            self.compute.wait_event(s["downloaded"])
        self.cache.step(layer, s["q"], s["k"], s["v"], frame_start, out=s["out"], lse=lse,
                        scores=scores, topc=topc, C=C)
        done = torch.cuda.Event()
        done.record(self.compute)
        s["read"] = done
        # download on its own stream
        self.copy_out.wait_event(done)
        with torch.cuda.stream(self.copy_out):
            out_host.copy_(s["out"], non_blocking=True)
            dl = torch.cuda.Event()
            dl.record(self.copy_out)
        s["downloaded"] = dl
        self.i += 1

    def record_done(self) -> torch.cuda.Event:
        """An event on the cache's stream after every submitted download."""
        for s in self.sets:
            if s["downloaded"] is not None:
                self.compute.wait_event(s["downloaded"])
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(self.compute)
        return ev

    def synchronize(self) -> None:
        self.record_done().synchronize()
