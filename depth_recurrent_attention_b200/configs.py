"""The five synthetic workloads of the Dreamer depth-recurrent core forward.

Each workload is one shared Dreamer layer unrolled over L depths (papernotes.org notes on
"Depth-Recurrent Attention Mixtures", section "Overall framework", flowchart).  Sizes:

  tiny     fp32   b=1  s=16   h=64   4x16   L=4   E=16   k=2  m=16  dense
  small    bf16   b=4  s=512  h=512  8x64   L=8   E=256  k=4  m=64  dense
  medium   bf16   b=8  s=2048 h=1024 16x64  L=16  E=1024 k=8  m=32  linear-MoE P=8
  decode   bf16   64 sequences x 4096 cached tokens, 1 new token, h=1024 16x64, L=32,
                  E=4096 k=16 m=16, dense
  large    bf16   b=2  s=8192 h=2048 16x128 L=64  E=2048 k=8  m=64  linear-MoE P=16

The router key dimension d_r equals the head dimension d where the workload does not state
it.  This module holds sizes only; it computes nothing of the method.
"""
from dataclasses import dataclass, asdict, replace


@dataclass(frozen=True)
class DreamerConfig:
    name: str
    batch: int          # b (prefill) or number of decode sequences
    seq: int            # s (prefill); 1 for decode
    hidden: int         # h = n_heads * head_dim
    n_heads: int        # H
    head_dim: int       # d
    depth: int          # L
    n_experts: int      # E
    top_k: int          # k
    expert_hidden: int  # m
    router_dim: int     # d_r
    n_proj_experts: int  # P, 0 = dense QKV/O projections
    dtype: str          # "fp32" or "bf16"
    seed: int
    bias_range: float   # b ~ U(-bias_range, bias_range)
    cache_len: int = 0  # decode: past tokens per sequence
    rope_base: float = 10000.0
    rms_eps: float = 1e-6
    variant: int = 0    # block layout: 0 DA||SA then EA (default), 1 serial, 2 fully parallel,
                        # 3 without depth attention (the DR-without-DA comparison arm)
    da_window: int = 0  # 0: DA over all earlier depths; W > 0: over the last W depths

    @property
    def tokens(self) -> int:
        """T: rows processed per depth (b*s for prefill, b for decode)."""
        return self.batch * self.seq

    @property
    def units(self) -> int:
        """token-depth-steps per call."""
        return self.tokens * self.depth

    @property
    def is_decode(self) -> bool:
        return self.cache_len > 0

    def with_(self, **kw) -> "DreamerConfig":
        return replace(self, **kw)

    def as_dict(self) -> dict:
        return asdict(self)


TINY = DreamerConfig("tiny", batch=1, seq=16, hidden=64, n_heads=4, head_dim=16, depth=4,
                     n_experts=16, top_k=2, expert_hidden=16, router_dim=16,
                     n_proj_experts=0, dtype="fp32", seed=0, bias_range=0.1)

SMALL = DreamerConfig("small", batch=4, seq=512, hidden=512, n_heads=8, head_dim=64, depth=8,
                      n_experts=256, top_k=4, expert_hidden=64, router_dim=64,
                      n_proj_experts=0, dtype="bf16", seed=1, bias_range=0.1)

MEDIUM = DreamerConfig("medium", batch=8, seq=2048, hidden=1024, n_heads=16, head_dim=64,
                       depth=16, n_experts=1024, top_k=8, expert_hidden=32, router_dim=64,
                       n_proj_experts=8, dtype="bf16", seed=2, bias_range=0.1)

DECODE = DreamerConfig("decode", batch=64, seq=1, hidden=1024, n_heads=16, head_dim=64,
                       depth=32, n_experts=4096, top_k=16, expert_hidden=16, router_dim=64,
                       n_proj_experts=0, dtype="bf16", seed=3, bias_range=0.05,
                       cache_len=4096)

LARGE = DreamerConfig("large", batch=2, seq=8192, hidden=2048, n_heads=16, head_dim=128,
                      depth=64, n_experts=2048, top_k=8, expert_hidden=64, router_dim=128,
                      n_proj_experts=16, dtype="bf16", seed=4, bias_range=0.1)

# the comparison arms and the sparse-DA outlook on the large shapes: DR without depth
# attention (variant 3) and depth attention over the last 8 depths; the pages' other block
# layouts: serial DA -> SA -> EA (variant 1) and fully parallel DA + SA + EA (variant 2)
LARGE_NODA = LARGE.with_(name="large-noda", variant=3)
LARGE_W8 = LARGE.with_(name="large-w8", da_window=8)
LARGE_SERIAL = LARGE.with_(name="large-serial", variant=1)
LARGE_PARALLEL = LARGE.with_(name="large-parallel", variant=2)
CONFIGS = {c.name: c for c in (TINY, SMALL, MEDIUM, DECODE, LARGE, LARGE_NODA, LARGE_W8,
                               LARGE_SERIAL, LARGE_PARALLEL)}
