"""The synthetic workloads (shapes, selection settings, generator knobs).

Each workload stands in for a latent grid of the video DiT's refinement stage
("LongCat-Video Technical Report", sections "Block Sparse Attention (BSA)" and
"Efficiency Results": 480p / 720p generation, 93.75% sparsity, i.e. r = N_k/16
key chunks per query chunk). No dataset is involved; the inputs are the seeded
smooth fields of ``synth.c``.
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    heads: int
    T: int
    H: int
    W: int
    d: int
    mode: str = "topk"          # "topk" | "cdf" | "topk_cdf" (chunks kept by both rules)
    topk: int = 0
    cdf_p: float = 0.9
    cdf_cap_frac: float = 0.25
    t_cond: int = 0             # latent frames of condition tokens (block-causal mask)
    q_begin: int = 0            # first latent frame whose queries are computed (KV-cached step)
    kchunk: tuple = (4, 4, 8)   # key chunk shape (multiples of the (4,4,8) query chunk)
    qchunk: tuple = (4, 4, 8)   # query chunk shape: (4,4,8), or (4,4,4) for 64-token chunks
    scale: float = 0.0          # softmax scale; 0 = 1/sqrt(d)
    tfreq_mult: float = 1.0     # temporal frequency multiplier of the smooth field
    seed: int = 0
    cond_seed: int = 1

    @property
    def softmax_scale(self) -> float:
        """The scale the library applies: the given one rounded to float, else
        1/sqrt(d) (the library takes the scale as a float)."""
        import numpy as np
        if self.scale:
            return float(np.float32(self.scale))
        return 1.0 / self.d ** 0.5

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def NH(self) -> int:
        return -(-self.H // 4)

    @property
    def NW(self) -> int:
        """(4,4,8) boxes along w."""
        return -(-self.W // 8)

    @property
    def NWq(self) -> int:
        """Query chunks along w."""
        return -(-self.W // self.qchunk[2])

    @property
    def Nc(self) -> int:
        """Query chunks per (batch, head): ceil(T/4) * ceil(H/4) * ceil(W/qw); edge
        chunks of a grid that is not a multiple of the chunk shape are partial."""
        return -(-self.T // 4) * self.NH * self.NWq

    @property
    def n_cond(self) -> int:
        """Condition chunks: chunks whose 4 frames all lie below t_cond."""
        return (self.t_cond // 4) * self.NH * self.NWq

    @property
    def Nk(self) -> int:
        """Key chunks per (batch, head)."""
        kt, kh, kw = self.kchunk
        return -(-self.T // kt) * -(-self.H // kh) * -(-self.W // kw)

    @property
    def n_cond_k(self) -> int:
        """Condition key chunks."""
        kt, kh, kw = self.kchunk
        return (self.t_cond // kt) * -(-self.H // kh) * -(-self.W // kw)

    @property
    def q_skip(self) -> int:
        """Query chunks before q_begin (not computed)."""
        return (self.q_begin // 4) * self.NH * self.NWq

    @property
    def Nq(self) -> int:
        """Query chunks computed per (batch, head)."""
        return self.Nc - self.q_skip

    @property
    def rows(self) -> int:
        return self.B * self.heads * self.Nq

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # 512 tokens, 4 chunks, keep 2
    "tiny": Workload("tiny", B=1, heads=2, T=4, H=8, W=16, d=64, topk=2),
    # 480p-like: 28,672 tokens, 224 chunks, keep 14
    "480p": Workload("480p", B=1, heads=32, T=16, H=32, W=56, d=128, topk=14),
    # 720p-like refinement grid: 92,160 tokens, 720 chunks, keep 45
    "720p": Workload("720p", B=1, heads=32, T=24, H=48, W=80, d=128, topk=45),
    # long video: 215,040 tokens, 1,680 chunks, keep 105, faster motion
    "long": Workload("long", B=1, heads=32, T=56, H=48, W=80, d=128, topk=105,
                     tfreq_mult=2.0),
    # block-causal video continuation with CDF selection (p = 0.9, cap 25%)
    "causal_cdf": Workload("causal_cdf", B=2, heads=32, T=24, H=48, W=80, d=128,
                           mode="cdf", cdf_p=0.9, cdf_cap_frac=0.25, t_cond=8),
    # the actual 720p token grid of the pages (1280x720 frames at 16x16 compression: 80x45
    # tokens per latent frame, 93 frames -> 24 latent frames): H = 45 leaves a last chunk
    # row of one token, so 80 of the 720 chunks are partial (32 of 128 tokens)
    "720p_real": Workload("720p_real", B=1, heads=32, T=24, H=45, W=80, d=128, topk=45),
    # 480p the same way (832x480 -> 52x30 tokens): partial chunks along H and W
    "480p_real": Workload("480p_real", B=1, heads=32, T=24, H=30, W=52, d=128, topk=21),
    # key chunks of 512 tokens (8,8,8) over the 720p-like grid: 180 key chunks, keep 11 (93.9 %)
    "720p_k512": Workload("720p_k512", B=1, heads=32, T=24, H=48, W=80, d=128, topk=11,
                          kchunk=(8, 8, 8)),
    # 87.5 % sparsity (r = N_k / 8): 90 of 720 chunks
    "720p_r8": Workload("720p_r8", B=1, heads=32, T=24, H=48, W=80, d=128, topk=90),
    # combination of both rules: CDF p = 0.1 (29-66 chunks on these inputs, median 41)
    # bounded by k = 45, so each rule decides part of the rows
    "720p_topk_cdf": Workload("720p_topk_cdf", B=1, heads=32, T=24, H=48, W=80, d=128,
                              mode="topk_cdf", topk=45, cdf_p=0.1, cdf_cap_frac=0.25),
    # 64-token query and key chunks (4,4,4) over the 720p-like grid ([P1] block-size
    # robustness): 1,440 chunks per head, keep 90 (93.75 %)
    "720p_q64": Workload("720p_q64", B=1, heads=32, T=24, H=48, W=80, d=128, topk=90,
                         qchunk=(4, 4, 4), kchunk=(4, 4, 4)),
    # the same video-continuation input at a later denoising step: the condition
    # frames' K/V are cached, only the noisy queries (frames >= 8) are computed
    "causal_cdf_kv": Workload("causal_cdf_kv", B=2, heads=32, T=24, H=48, W=80, d=128,
                              mode="cdf", cdf_p=0.9, cdf_cap_frac=0.25, t_cond=8, q_begin=8),
}
