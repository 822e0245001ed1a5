"""The MoE-layer workloads this library is measured and tested on.

Shapes follow the Qwen3.8-Flash-Next MoE block described in "个人开发者用 AI
十天写出 Strata 引擎，让 12GB 显存跑起 1250 亿参数的 Qwen 3.8 Flash Next"
(section "1250 亿参数，每个词只用得上 2%": 48 layers, 512 experts per layer,
10 routed experts plus one shared expert per token), with the MTP verify batch of
one token plus three drafts (section "命中率七成，代价是答案会变") and prefill chunks of
at most 8192 tokens (section "等最久的，是它读完你的代码"). The expert width f=768 and
hidden size d=2048 give 4.72 M weights per expert, about 1.47 MB at 2.5 bits per
weight, consistent with that page's figure of roughly 700 experts per GB of
VRAM (section "命中率七成，代价是答案会变").
"""
from __future__ import annotations

from dataclasses import dataclass, replace

# Strength of the per-expert Zipf bias (router bias = -ZIPF_ALPHA * 1.1 * ln(rank)).
# Chosen so that over an 8192-token chunk the most popular expert receives about
# 2000 tokens; oracle/calibrate_zipf.py re-derives it.
ZIPF_ALPHA = 0.2575
ZIPF_S = 1.1


@dataclass(frozen=True)
class Workload:
    name: str
    T: int          # tokens per layer call
    d: int          # hidden size
    E: int          # routed experts per layer
    k: int          # experts per token
    f: int          # expert intermediate size
    fmt: int        # 2 = Q2, 3 = Q3
    layers: int = 1
    zipf: bool = True
    resident: int = -1   # resident experts per layer (-1 = all)
    seed: int = 0
    q3_top: int = 0      # mixed pool: the q3_top most popular experts of a layer are stored Q3, the rest fmt
    chunk: int = 0       # prefill chunk loop: T tokens processed in chunks of this many (0 = one call)

    @property
    def resident_count(self) -> int:
        return self.E if self.resident < 0 else self.resident

    def expert_fmt(self, rank: int) -> int:
        """Storage format of an expert of popularity rank `rank` (1 = most popular)."""
        return 3 if self.q3_top > 0 and rank <= self.q3_top else self.fmt

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_T16_d512_E64_k4_f256_q2": Workload("tiny_T16_d512_E64_k4_f256_q2", 16, 512, 64, 4, 256, 2, zipf=False),
    "decode_T1_d2048_E512_k10_f768_q2": Workload("decode_T1_d2048_E512_k10_f768_q2", 1, 2048, 512, 10, 768, 2),
    "verify_T4_d2048_E512_k10_f768_q3": Workload("verify_T4_d2048_E512_k10_f768_q3", 4, 2048, 512, 10, 768, 3),
    # wider MTP verify batches (1 token + 1 or 7 drafts), same layer
    "verify_T2_d2048_E512_k10_f768_q3": Workload("verify_T2_d2048_E512_k10_f768_q3", 2, 2048, 512, 10, 768, 3),
    "verify_T8_d2048_E512_k10_f768_q3": Workload("verify_T8_d2048_E512_k10_f768_q3", 8, 2048, 512, 10, 768, 3),
    "prefill_T8192_d2048_E512_k10_f768_q2": Workload("prefill_T8192_d2048_E512_k10_f768_q2", 8192, 2048, 512, 10, 768, 2),
    "stack48_T1_d2048_E512_k10_f768_q2_res25": Workload(
        "stack48_T1_d2048_E512_k10_f768_q2_res25", 1, 2048, 512, 10, 768, 2, layers=48, resident=128),
    # the prefill layer with uniform routing (no popularity bias): ~160 tokens per expert
    "prefill_T8192_d2048_E512_k10_f768_q2_uniform": Workload(
        "prefill_T8192_d2048_E512_k10_f768_q2_uniform", 8192, 2048, 512, 10, 768, 2, zipf=False),
    # a 32K-token prompt through one layer in four 8192-token chunks
    "prefill_chunks4_T32768_d2048_E512_k10_f768_q2": Workload(
        "prefill_chunks4_T32768_d2048_E512_k10_f768_q2", 32768, 2048, 512, 10, 768, 2, chunk=8192),
    # the 3-bit tier at prefill size
    "prefill_T8192_d2048_E512_k10_f768_q3": Workload("prefill_T8192_d2048_E512_k10_f768_q3", 8192, 2048, 512, 10,
                                                      768, 3),
    # a pool with both tiers: the 128 most popular experts of the layer in Q3, the rest in Q2
    "prefill_T8192_d2048_E512_k10_f768_mixed_q3top128": Workload(
        "prefill_T8192_d2048_E512_k10_f768_mixed_q3top128", 8192, 2048, 512, 10, 768, 2, q3_top=128),
}

TINY = WORKLOADS["tiny_T16_d512_E64_k4_f256_q2"]
DECODE = WORKLOADS["decode_T1_d2048_E512_k10_f768_q2"]
VERIFY = WORKLOADS["verify_T4_d2048_E512_k10_f768_q3"]
PREFILL = WORKLOADS["prefill_T8192_d2048_E512_k10_f768_q2"]
STACK48 = WORKLOADS["stack48_T1_d2048_E512_k10_f768_q2_res25"]


def expert_bytes(fmt: int, d: int, f: int) -> int:
    """Stored bytes of one expert (codes + fp16 scales [+ fp16 mins]) for 3*d*f weights."""
    weights = 3 * d * f
    per_block = 20 if fmt == 2 else 26   # 16 B codes + 2 B scale + 2 B min | 24 B codes + 2 B scale
    return weights // 64 * per_block
