"""fp64 CPU oracle for the chunked attention step over a bounded KV cache.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, calls or links
this package; only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline leg (and its ``--impl reference`` arm) use it. It shares no code
with the CUDA path: the only module both sides import is ``rc_synth`` (seeded
input generators and workload sizes, no arithmetic of the method).

The oracle is plain and slow on purpose. It keeps the whole history of the
stream, recomputes from it which frames each cache policy keeps and at which
RoPE time index, rotates raw keys and queries in fp64 and runs a masked
softmax attention with a dense matmul. Each function cites the page passage it
follows; the pages are

* rCM page  -- "rCM length extrapolation" guide (dpshk.com, news/6097349):
  strategies 1-5 (Sliding Window, Rolling Sink, Infinity-RoPE, Deep Forcing,
  Relax Forcing), the MemRoPE tip and the practical tips. Deep Forcing,
  Relax Forcing and MemRoPE have their own modules (deep_forcing.py,
  relax_forcing.py, memrope.py), each listing the readings it takes.
* Causal-Forcing page -- "Causal-Forcing inference walkthrough" (lqnn.cn,
  news/227985): section 3 (KV cache) and section 4 (block-wise denoising).
* LingBot page -- "LingBot-World 2.0 rolling KV cache" explainer
  (icman.com.cn, news/50396): sections on chunked inference, the
  local_attn_size sliding window, the sink_size attention sink and the two
  easily-missed details.
* Rolling Sink digest -- digest of "Rolling Sink: Bridging Limited-Horizon
  Training and Open-Ended Testing in Autoregressive Video Diffusion"
  (paper.rainbus.top, paper/2602.07775): method-step details, RoPE background.

Parity status: every function here is pinned by a ``-m "not gpu"`` test
against something other than itself (hand enumerations, closed forms,
invariants, torch's SDPA, brute force). See tests/test_oracle_*.py.
"""
from .policy import PolicyOracle, KeptFrame, roll_index
from .rope import rope_pair_split, rope_angles, rope_apply, token_grid_positions
from .attention import masked_sdpa, visibility, column_scores, top_c
from .deep_forcing import DeepForcingOracle, KeptToken
from .relax_forcing import RelaxForcingOracle
from .memrope import MemRopeOracle
from .stream import OracleStream

__all__ = [
    "PolicyOracle", "KeptFrame", "roll_index", "rope_pair_split", "rope_angles",
    "rope_apply", "token_grid_positions", "masked_sdpa", "visibility",
    "column_scores", "top_c", "OracleStream", "DeepForcingOracle", "KeptToken",
    "RelaxForcingOracle", "MemRopeOracle",
]
