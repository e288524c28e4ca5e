"""Helpers for the GPU tests: device tensors from seeded inputs, a CPU fp32
restatement of the RoPE kernels' arithmetic (for bit-exact checks), and a
stream driver that runs a workload through the library and the oracle side
by side."""
from __future__ import annotations

import numpy as np
import torch

import rc_synth
from oracle import KeptToken, OracleStream
from rolling_kv_cache_b200 import binding as B
from rolling_kv_cache_b200.cache import RollingKVCache

from rcutil import config_for, lib_kept, near_tie_violations, oracle_df_frames, oracle_kept

TOL_MAX, TOL_MEAN, TOL_LSE = 2e-2, 2e-3, 1e-2

GUARD_BYTES = 4096
GUARD_BYTE = 0xA5


class Guarded:
    """A device buffer between two guard regions the library must never write.

    ``view(dtype, shape)`` is the usable part; ``intact()`` checks that every
    byte outside it, the guards and any alignment slack, still holds the
    pattern. Bounds checks in place of a memory checker."""

    def __init__(self, nbytes: int, device="cuda"):
        self.nbytes = int(nbytes)
        self.full = torch.full((GUARD_BYTES + self.nbytes + GUARD_BYTES,), GUARD_BYTE, dtype=torch.uint8,
                               device=device)
        self.inner = self.full[GUARD_BYTES:GUARD_BYTES + self.nbytes]

    def view(self, dtype, shape):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        if n > self.nbytes:
            raise ValueError("view larger than the buffer")
        return self.inner[:n].view(dtype).view(shape)

    def intact(self, used: int = None) -> bool:
        used = self.nbytes if used is None else used
        lo = self.full[:GUARD_BYTES]
        hi = self.full[GUARD_BYTES + used:]
        return bool((lo == GUARD_BYTE).all()) and bool((hi == GUARD_BYTE).all())


def guarded_like(shape, dtype, fill=None, device="cuda"):
    """(buffer, tensor): a guarded tensor of ``shape`` (filled with ``fill``)."""
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    g = Guarded(n, device)
    t = g.view(dtype, shape)
    if fill is not None:
        t.fill_(fill)
    return g, t


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f32(bits):
    return rc_synth.bf16_bits_to_f32(bits)


def rope_fp32(x_bits, t_pos, h_pos, w_pos, tables, pairs):
    """The kernels' rotation restated in numpy fp32: x [n, H, d] bf16 bits."""
    return rope_fp32_values(f32(x_bits).astype(np.float32), t_pos, h_pos, w_pos, tables, pairs)


def rope_fp32_values(x, t_pos, h_pos, w_pos, tables, pairs):
    """Same rotation of fp32 values x [n, H, d]; returns bf16 bits."""
    pt, ph, pw = pairs
    x = np.asarray(x, dtype=np.float32)
    n, H, d = x.shape
    c = np.empty((n, d // 2), np.float32)
    s = np.empty((n, d // 2), np.float32)
    tt, th, tw = (tb.reshape(-1, P, 2) for tb, P in zip(tables, pairs))
    c[:, :pt], s[:, :pt] = tt[t_pos, :, 0], tt[t_pos, :, 1]
    c[:, pt:pt + ph], s[:, pt:pt + ph] = th[h_pos, :, 0], th[h_pos, :, 1]
    c[:, pt + ph:], s[:, pt + ph:] = tw[w_pos, :, 0], tw[w_pos, :, 1]
    c, s = c[:, None, :], s[:, None, :]
    xe, xo = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = (xe * c).astype(np.float32) - (xo * s).astype(np.float32)
    out[..., 1::2] = (xe * s).astype(np.float32) + (xo * c).astype(np.float32)
    return rc_synth.f32_to_bf16_bits(out.astype(np.float32))


def rope_fp32_delta(x_bits, delta, tables, pairs):
    """In-place time re-rotation by delta on the t pairs only (fp32 restatement)."""
    pt = pairs[0]
    x = f32(x_bits).astype(np.float32)
    tt = tables[0].reshape(-1, pt, 2)
    c = tt[abs(delta), :, 0].astype(np.float32)
    s = (np.float32(-1.0 if delta < 0 else 1.0) * tt[abs(delta), :, 1]).astype(np.float32)
    xe, xo = x[..., 0:2 * pt:2].copy(), x[..., 1:2 * pt:2].copy()
    x[..., 0:2 * pt:2] = (xe * c).astype(np.float32) - (xo * s).astype(np.float32)
    x[..., 1:2 * pt:2] = (xe * s).astype(np.float32) + (xo * c).astype(np.float32)
    return rc_synth.f32_to_bf16_bits(x.astype(np.float32))


def compare(o_gpu, lse_gpu, ref, rows, heads):
    """Float parity bar: O max-abs / mean-abs and LSE max-abs against fp64."""
    og = f32(o_gpu)[rows][:, heads].astype(np.float64)
    err = np.abs(og - ref["o"])
    lg = lse_gpu[heads][:, rows]
    lerr = np.abs(lg - ref["lse"])
    return err.max(), err.mean(), lerr.max()


class Runner:
    """Runs one layer of a workload through the library and the oracle."""

    def __init__(self, w: rc_synth.Workload, layer: int = 0, seed: int = 0, layers=None):
        self.w = w
        self.layer = layer
        self.seed = seed
        cfg = config_for(w, layers=layers if layers is not None else w.layers)
        # the cache block sits between guard regions, checked after every step
        self.block = Guarded(B.rc_cache_bytes(cfg) + 256)
        self.cache = RollingKVCache(cfg, mem=self.block.inner)
        assert self.block.inner.data_ptr() % 256 == 0
        self.oracle = OracleStream(w, layer=layer, seed=seed)
        self.pairs = (cfg.rope_t_pairs, cfg.rope_h_pairs, cfg.rope_w_pairs)
        if self.pairs == (0, 0, 0):
            from oracle import rope_pair_split
            self.pairs = rope_pair_split(w.head_dim)
        self.tables = [B.rc_rope_table(self.cache.handle, a) for a in range(3)]
        self.last = None
        self.df = w.policy == rc_synth.POLICY_DEEP_FORCING
        self.rf = w.policy == rc_synth.POLICY_RELAX_FORCING
        self.mr = w.policy == rc_synth.POLICY_MEMROPE
        self.mem_state = None     # MemRoPE: fp32 restatement of the device EMA [2 kv][2 mem][F, H, d]
        self.mem_folded = 0
        self.prev_scores = None   # Deep Forcing: the last step's candidate scores (next pool)
        self.ref_scores = None    # fp64 candidate scores of the current step, when check_float computed them
        self.df_fp64_checked = 0  # Deep Forcing compactions checked against the fp64 selection

    def step(self, chunk: int, pass_: int, cut: bool = False, scores: bool = False, check: bool = True):
        """One rc_step of (chunk, pass_) and the oracle's step beside it.

        The integer state is compared on every call. With ``check`` (the
        default) every buffer the call touches sits between guard regions
        that are checked afterwards, and the inputs are checked unchanged;
        ``check=False`` drives the stream quickly to a later event."""
        w = self.w
        prev_ref, self.ref_scores = self.ref_scores, None
        if cut:
            self.cache.reindex(w.cut_delta, B.RC_REINDEX_FLUSH | B.RC_REINDEX_CUT)
            self.oracle.reindex(1 | 2, w.cut_delta)
        q, k, v = rc_synth.chunk_qkv(w, self.layer, chunk, pass_, self.seed)
        Nq = q.shape[0]
        # every buffer the call touches sits between guard regions
        guards = []

        def guarded_input(bits):
            if not check:
                return dev_bf16(bits)
            g, t = guarded_like(bits.shape, torch.bfloat16)
            t.copy_(dev_bf16(bits))
            guards.append(g)
            return t

        def guarded_out(shape, dtype, fill=None):
            if not check:
                t = torch.empty(shape, dtype=dtype, device="cuda")
                return t if fill is None else t.fill_(fill)
            g, t = guarded_like(shape, dtype, fill=fill)
            guards.append(g)
            return t
        qd, kd, vd = guarded_input(q), guarded_input(k), guarded_input(v)
        lse = guarded_out((w.heads, Nq), torch.float32)
        out_d = guarded_out(qd.shape, torch.bfloat16)
        sc = tc = None
        if scores or self.df:
            sc = guarded_out((w.footprint_tokens,), torch.float32, fill=-1.0)
        if scores and w.topc:
            tc = guarded_out((w.topc,), torch.int32, fill=-7)
        out = self.cache.step(self.layer, qd, kd, vd, chunk * w.chunk_frames, out=out_d,
                              lse=lse, scores=sc, topc=tc, C=w.topc if tc is not None else 0)
        assert out.data_ptr() == out_d.data_ptr()
        if self.df:
            # the region is chosen from the library's own scores of the last step (DF2)
            kept = self.oracle.step(chunk, pass_, pool_scores=self.prev_scores)
        else:
            kept = self.oracle.step(chunk, pass_)
        torch.cuda.synchronize()
        self.cache.device_status()
        # nothing written outside the cache block or the output tensors, and
        # the inputs are left as they were
        assert self.block.intact(self.cache.nbytes), "write outside the cache block"
        assert all(g.intact() for g in guards), "write outside an input or output tensor"
        if check:
            for dev, bits in ((qd, q), (kd, k), (vd, v)):
                assert np.array_equal(bits_of(dev), bits.view(np.uint16).reshape(dev.shape)), "input modified"
        st = self.cache.state(self.layer)
        if self.rf:
            kept = self._check_rf_selection(st)
        elif self.mr:
            assert lib_kept(st) == oracle_df_frames(kept)
            self._fold_memory()
        elif self.df:
            assert lib_kept(st) == oracle_df_frames(kept)
            comp = self.oracle.df.comp
            assert st.comp_tokens == len(comp)
            if comp:
                frames, toks = self.cache.comp_tokens(self.layer)
                assert list(zip(frames, toks)) == comp          # the selection, bit-exact
                assert st.comp_tau0 == self.oracle.df.frame_taus()[1]
            if self.oracle.df.last_selection is not None and prev_ref is not None:
                self._check_df_selection_fp64(prev_ref)
            self.prev_scores = sc.cpu().numpy()[:st.n_candidates]
        else:
            assert lib_kept(st) == oracle_kept(kept)
        self.last = dict(q=q, k=k, v=v, out=bits_of(out), lse=lse.cpu().numpy(), state=st,
                         scores=None if sc is None else sc.cpu().numpy()[:st.n_candidates],
                         topc=None if tc is None else tc.cpu().numpy())
        return self.last

    def check_append_bitexact(self):
        """Current chunk's K/V slots == fp32 restatement of RoPE(k) / raw v."""
        w, st, last = self.w, self.last["state"], self.last
        F = w.frame_seqlen
        kc, vc = self.cache.cache_views(self.layer)
        n = np.arange(F)
        hh, ww = n // w.grid_w, n % w.grid_w
        for e in st.kept[:st.n_kept]:
            if e.region != 2:
                continue
            r = e.rank
            sl = slice(r * F, (r + 1) * F)
            want_k = rope_fp32(last["k"][sl], np.full(F, e.stored_time), hh, ww, self.tables, self.pairs)
            got_k = bits_of(kc[:, e.slot * F:(e.slot + 1) * F]).transpose(1, 0, 2)
            assert np.array_equal(got_k, want_k), ("K slot", e.slot)
            got_v = bits_of(vc[:, e.slot * F:(e.slot + 1) * F]).transpose(1, 0, 2)
            assert np.array_equal(got_v, last["v"][sl]), ("V slot", e.slot)
        qr = bits_of(self.cache.q_rot_view(w.query_tokens)).transpose(1, 0, 2)
        cur = {e.rank: e.stored_time for e in st.kept[:st.n_kept] if e.region == 2}
        tq = np.repeat([cur[r] for r in range(w.chunk_frames)], F)
        want_q = rope_fp32(last["q"], tq, np.tile(hh, w.chunk_frames), np.tile(ww, w.chunk_frames),
                           self.tables, self.pairs)
        assert np.array_equal(qr, want_q)

    def _check_df_selection_fp64(self, ref_scores):
        """Deep Forcing: the region the device chose at this compaction (equal,
        bit for bit, to the top-C of the device's own scores of the last pass,
        which the oracle was fed) against the region the fp64 scores of that
        pass choose. They may differ only among near-ties: every pool token in
        the symmetric difference has an fp64 score within SCORE_TOL of the
        C-th highest fp64 pool score (the same allowance as the top-C of the
        token scores, reading S1 (ii))."""
        df = self.oracle.df
        pool = df.last_pool
        s64 = np.asarray(ref_scores[:len(pool)], dtype=np.float64)
        assert len(s64) == len(pool), "fp64 scores do not cover the pool"
        assert len(df.last_selection) == df.C
        bad = near_tie_violations(s64, df.last_selection, df.C)
        assert not bad, ("selection differs from fp64 beyond near-ties", bad[:8])
        self.df_fp64_checked += 1

    def _check_rf_selection(self, st):
        """Relax Forcing: the device's pool scores match fp64 within 1e-4, its
        selection is the top-K of its own scores bit for bit, and differs from
        the fp64 selection only among near-ties (then the oracle follows the
        device's choice so both keep the same frames)."""
        from oracle.relax_forcing import select_frames
        rf, F = self.oracle.rf, self.w.frame_seqlen
        gpu = np.array(self.cache.pool_scores(self.layer), dtype=np.float64)
        if rf.last_scores is None:
            assert len(gpu) == 0
        else:
            assert len(gpu) == len(rf.last_scores)
            assert np.max(np.abs(gpu - rf.last_scores)) <= 1e-4, np.max(np.abs(gpu - rf.last_scores))
            sel = select_frames(gpu.astype(np.float32), rf.K)
            if sel != rf.last_selection:
                kth = np.sort(rf.last_scores)[::-1][rf.K - 1]
                for i in set(sel) ^ set(rf.last_selection):
                    assert abs(rf.last_scores[i] - kth) <= 1e-4
                rf.hist = [rf.last_pool[i] for i in sel]
                rf.last_selection = sel
        kept = rf.kept()
        self.oracle.kept = kept
        self.oracle.kept_tokens = [KeptToken(k.content, t, k.tau, k.region, k.rank) for k in kept for t in range(F)]
        hist = set(rf.hist)
        assert lib_kept(st) == [(k.content, k.tau, k.region, k.rank) for k in kept
                                if not (k.region == "hist" and k.content in hist)]
        assert st.comp_tokens == len(rf.hist) * F
        if rf.hist:
            frames, toks = self.cache.comp_tokens(self.layer)
            assert frames == [g for g in rf.hist for _ in range(F)]
            assert toks == list(range(F)) * len(rf.hist)
        return kept

    def _fold_memory(self):
        """MemRoPE: fold newly evicted frames into the fp32 restatement of the
        device state, in the device's operation order."""
        w, mr = self.w, self.oracle.mr
        F, Bf = w.frame_seqlen, w.chunk_frames
        a = [np.float32(w.mr_alpha_long), np.float32(w.mr_alpha_short)]
        b = [np.float32(1.0 - w.mr_alpha_long), np.float32(1.0 - w.mr_alpha_short)]
        for g in mr.folded[self.mem_folded:]:
            c, o = divmod(g, Bf)
            x = [f32(rc_synth.chunk_tensor(w, self.layer, c, self.oracle.last_pass[c], tid, self.seed)
                     [o * F:(o + 1) * F]).astype(np.float32) for tid in (rc_synth.TENSOR_K, rc_synth.TENSOR_V)]
            if self.mem_state is None:
                self.mem_state = [[x[kv].copy(), x[kv].copy()] for kv in range(2)]
            else:
                for kv in range(2):
                    for m in range(2):
                        self.mem_state[kv][m] = ((a[m] * self.mem_state[kv][m]).astype(np.float32) +
                                                 (b[m] * x[kv]).astype(np.float32)).astype(np.float32)
        self.mem_folded = len(mr.folded)

    def check_mem_bitexact(self):
        """MemRoPE: both memory frames' K / V rows == the fp32 restatement,
        keys rotated to the memories' times at each token's (h, w)."""
        if self.mem_state is None:
            return
        w, st = self.w, self.last["state"]
        F = w.frame_seqlen
        kc, vc = self.cache.cache_views(self.layer)
        t = np.arange(F)
        mem = {e.content: e for e in st.kept[:st.n_kept] if e.content < 0}
        for m, content in enumerate((-1, -2)):
            e = mem[content]
            rows = slice(e.slot * F, (e.slot + 1) * F)
            want_k = rope_fp32_values(self.mem_state[0][m], np.full(F, e.tau), t // w.grid_w, t % w.grid_w,
                                      self.tables, self.pairs)
            assert np.array_equal(bits_of(kc[:, rows]).transpose(1, 0, 2), want_k), content
            want_v = rc_synth.f32_to_bf16_bits(self.mem_state[1][m])
            assert np.array_equal(bits_of(vc[:, rows]).transpose(1, 0, 2), want_v), content

    def check_df_region_bitexact(self):
        """Deep Forcing: every region key == fp32 restatement of RoPE(raw key of
        its source token) at the region's time for its position; V == raw v."""
        w, st = self.w, self.last["state"]
        if st.comp_tokens == 0:
            return
        F, Bf = w.frame_seqlen, w.chunk_frames
        frames, toks = self.cache.comp_tokens(self.layer)
        kc, vc = self.cache.cache_views(self.layer)
        rows = slice(st.comp_row0, st.comp_row0 + st.comp_tokens)
        got_k = bits_of(kc[:, rows]).transpose(1, 0, 2)
        got_v = bits_of(vc[:, rows]).transpose(1, 0, 2)
        raw_k = np.empty_like(got_k)
        raw_v = np.empty_like(got_v)
        frames, t = np.array(frames), np.array(toks)
        for c in np.unique(frames // Bf):          # regenerate each source chunk once
            kk, vv = (rc_synth.chunk_tensor(w, self.layer, int(c), self.oracle.last_pass[int(c)], tid, self.seed)
                      for tid in (rc_synth.TENSOR_K, rc_synth.TENSOR_V))
            sel = np.nonzero(frames // Bf == c)[0]
            src = (frames[sel] % Bf) * F + t[sel]
            raw_k[sel], raw_v[sel] = kk[src], vv[src]
        # Deep Forcing: the region's packed times; Relax Forcing: each frame its own index
        tau = frames if self.rf else st.comp_tau0 + np.arange(st.comp_tokens) // F
        want_k = rope_fp32(raw_k, tau, t // w.grid_w, t % w.grid_w, self.tables, self.pairs)
        assert np.array_equal(got_k, want_k)
        assert np.array_equal(got_v, raw_v)

    def check_float(self, rows=None, heads=None, scores=False):
        """O / LSE of the last step against fp64 (sampled rows and heads, or
        all). With ``scores`` (every row and head) the fp64 candidate scores
        are kept for the next step: a Deep Forcing compaction there is
        checked against the selection they make."""
        ref = self.oracle.outputs(heads=heads, rows=rows, want_scores=scores)
        rows = ref["rows"]
        mx, mean, lmx = compare(self.last["out"], self.last["lse"], ref, rows, ref["heads"])
        assert mx <= TOL_MAX and mean <= TOL_MEAN and lmx <= TOL_LSE, (mx, mean, lmx)
        if scores:
            self.ref_scores = ref["scores"]
        return ref, (mx, mean, lmx)

    def close(self):
        self.cache.close()
