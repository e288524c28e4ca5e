"""Test helpers: library config from a workload, state comparisons."""
import rc_synth
from rolling_kv_cache_b200 import binding as B
from rolling_kv_cache_b200.cache import make_config

REGION = {0: "sink", 1: "hist", 2: "cur"}

# Token scores against the fp64 oracle, as a fraction of max(1, the largest
# score). The cache stores rotated keys, and the attention reads rotated
# queries, in bf16 (unit roundoff u = 2^-9), so every logit the scores sum
# over carries that rounding, and keys re-rotated in place after a RoPE cut
# carry one more. The bar is u; test_score_tolerance_covers_bf16_storage
# measures the part the storage rounding alone causes on the parity streams
# and checks the bar leaves room above it.
SCORE_TOL = 2.0 ** -9


def near_tie_violations(scores64, got, C: int, tol: float = SCORE_TOL):
    """Indices where a selection of C candidates differs from the fp64 top-C
    by more than a near-tie.

    ``scores64`` are the fp64 scores of the candidates (index = position),
    ``got`` the selected positions. The fp64 selection is the C highest,
    ties to the lower index (reading S1); a position in the symmetric
    difference of the two selections is allowed only if its fp64 score lies
    within ``tol * max(1, kth)`` of the C-th highest fp64 score ``kth``.
    Returns the offending positions (empty: the selection passes)."""
    import numpy as np
    from oracle import top_c
    s = np.asarray(scores64, dtype=np.float64)
    got = np.asarray(got, dtype=np.int64)
    if len(s) <= C:
        return sorted(set(range(len(s))) ^ set(got.tolist()))
    want = top_c(s, np.arange(len(s)), C)
    kth = np.sort(s)[::-1][C - 1]
    bad = [int(i) for i in set(want.tolist()) ^ set(got.tolist())
           if not (0 <= i < len(s)) or abs(s[i] - kth) > tol * max(1.0, kth)]
    if len(set(got.tolist())) != C:
        bad.append(-1)
    return sorted(bad)


def config_for(w: rc_synth.Workload, **over):
    kw = dict(layers=w.layers, heads=w.heads, head_dim=w.head_dim, grid_h=w.grid_h,
              grid_w=w.grid_w, sink_frames=w.sink_frames, window_frames=w.window_frames,
              chunk_frames=w.chunk_frames, policy=w.policy, mask_block_frames=w.mask_block_frames,
              theta=w.theta, t_max=w.t_max, rs_bank_blocks=w.rs_bank_blocks,
              rs_sink_blocks=w.rs_sink_blocks, rs_static_semantics=w.rs_static_semantics,
              ir_f_limit=w.ir_f_limit, ir_sink_blocks=w.ir_sink_blocks,
              ir_cache_blocks=w.ir_cache_blocks, df_budget_tokens=w.df_budget_tokens,
              rf_history_frames=w.rf_history_frames, rf_weight=w.rf_weight,
              mr_alpha_long=w.mr_alpha_long, mr_alpha_short=w.mr_alpha_short)
    kw.update(over)
    return make_config(**kw)


def lib_kept(state):
    return [(e.content, e.tau, REGION[e.region], e.rank) for e in state.kept[:state.n_kept]]


def oracle_kept(kept):
    return [(k.content, k.tau, k.region, k.rank) for k in kept]


def oracle_df_frames(kept_tokens):
    """Deep Forcing oracle tokens -> the frame entries the library reports
    (sink, history, current; the compressed region is reported as a count)."""
    out = []
    for k in kept_tokens:
        if k.region == "comp":
            continue
        e = (k.content, k.tau, k.region, k.rank)
        if not out or out[-1] != e:
            out.append(e)
    return out
