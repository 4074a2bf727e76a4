"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random inputs.  It holds none of the decision path's
arithmetic (no gate, no counting, no planning, no split, no assignment), so
both the CUDA path and the CPU oracle can be fed the same bytes from it.

Recipe (one reading of the workload descriptions; real routing traces,
datasets and weights are not available, so these stand in for them):
  * h_0 ~ N(0,1) in fp32, rounded to bf16 (round to nearest even).
  * h_{l+1} = bf16(f32(h_l) + d * N(0,1)), drift d per workload.
  * gate W_l ~ N(0, 1/H), stored [E,H] bf16 (row e = expert e's weights).
  * bias b_l[e] = 2.0 * rank_l(e)^(-s): a Zipf(s) profile whose hottest
    expert gets +2.0.  rank_l is the 1-based position of e when a latent
    z_l is sorted in descending order; z_l = rho z_{l-1} + sqrt(1-rho^2) xi
    (rho = layer-to-layer or step-to-step correlation, 0 when unstated).
  * decode steps: ids are drawn directly as the k largest of
    bias_step[e] + N(0,1) per (token, expert), which has the law of
    h.W + b for W ~ N(0,1/H) up to the cross-expert correlation of a token.
Seeds: base seed per workload, stream id per tensor kind, index per layer or
step, combined as base * 10**6 + stream * 10**4 + index.
"""
from dataclasses import dataclass, field
import math

import torch

S_HIDDEN, S_WEIGHT, S_LATENT, S_DECODE = 1, 2, 3, 4


@dataclass(frozen=True)
class Workload:
    name: str
    T: int          # tokens per problem (all ranks together)
    H: int          # hidden size
    E: int          # routed experts
    k: int          # experts per token
    G: int          # expert-parallel ranks
    N: int          # extra replica slots per rank
    alpha: float    # share of the N slots filled by locality (phase 1)
    layers: int     # layers (or decode steps)
    drift: float    # hidden-state drift per layer
    zipf_s: float   # Zipf exponent of the expert bias
    rho: float      # correlation of the bias latent between layers/steps
    seed: int       # base seed
    decode_T: tuple = field(default=())   # per-step token counts (decode sweep)

    @property
    def L(self) -> int:
        """Phase-1 replica count per rank: floor(N * alpha)."""
        return int(math.floor(self.N * self.alpha))

    def with_(self, **kw):
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    "tiny": Workload("tiny", T=256, H=128, E=16, k=2, G=4, N=1, alpha=0.5, layers=1,
                     drift=0.1, zipf_s=1.2, rho=0.0, seed=1),
    "tiny-p1": Workload("tiny-p1", T=256, H=128, E=16, k=2, G=4, N=2, alpha=0.5, layers=1,
                        drift=0.1, zipf_s=1.2, rho=0.0, seed=11),
    "olmoe": Workload("olmoe", T=4096, H=2048, E=64, k=8, G=8, N=2, alpha=0.5, layers=16,
                      drift=0.1, zipf_s=1.1, rho=0.0, seed=2),
    "qwen3-30b": Workload("qwen3-30b", T=16384, H=2048, E=128, k=8, G=16, N=2, alpha=0.5,
                          layers=48, drift=0.15, zipf_s=1.2, rho=0.8, seed=3),
    "qwen3-235b": Workload("qwen3-235b", T=32768, H=4096, E=128, k=8, G=8, N=4, alpha=0.5,
                           layers=94, drift=0.1, zipf_s=1.3, rho=0.0, seed=4),
    "decode": Workload("decode", T=8192, H=7168, E=256, k=8, G=64, N=2, alpha=0.5,
                       layers=1000, drift=0.0, zipf_s=1.2, rho=0.5, seed=5,
                       decode_T=(64, 256, 1024, 4096, 8192)),
}


def seed_of(w: Workload, stream: int, index: int) -> int:
    return w.seed * 10**6 + stream * 10**4 + index


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def bias_latents(w: Workload, count: int) -> torch.Tensor:
    """[count, E] fp32 latents z_0..z_{count-1} (CPU)."""
    out = torch.empty(count, w.E, dtype=torch.float32)
    z = None
    c = math.sqrt(max(0.0, 1.0 - w.rho * w.rho))
    for i in range(count):
        xi = torch.randn(w.E, generator=_gen("cpu", seed_of(w, S_LATENT, i)), dtype=torch.float32)
        z = xi if z is None else w.rho * z + c * xi
        out[i] = z
    return out


def biases(w: Workload, count: int) -> torch.Tensor:
    """[count, E] fp32: b[e] = 2.0 * rank(e)^(-s), rank from the latent (CPU)."""
    z = bias_latents(w, count)
    order = torch.argsort(-z, dim=1, stable=True)
    rank = torch.empty_like(order)
    pos = torch.arange(1, w.E + 1).expand(count, w.E)
    rank.scatter_(1, order, pos)
    return (2.0 * rank.to(torch.float64).pow(-w.zipf_s)).to(torch.float32)


def hidden_chain(w: Workload, count: int, device="cpu", T=None, out=None) -> torch.Tensor:
    """[count, T, H] bf16: h_0 .. h_{count-1}.  `out` may be a preallocated
    bf16 tensor of that shape (e.g. a slice of a larger buffer)."""
    T = w.T if T is None else T
    if out is None:
        out = torch.empty(count, T, w.H, dtype=torch.bfloat16, device=device)
    h = None
    for i in range(count):
        g = _gen(out.device, seed_of(w, S_HIDDEN, i))
        noise = torch.randn(T, w.H, generator=g, device=out.device, dtype=torch.float32)
        h = noise if h is None else h.float() + w.drift * noise
        h = h.to(torch.bfloat16)
        out[i].copy_(h)
    return out


def gate_weights(w: Workload, count: int, device="cpu") -> torch.Tensor:
    """[count, E, H] bf16, W_l ~ N(0, 1/H)."""
    out = torch.empty(count, w.E, w.H, dtype=torch.bfloat16, device=device)
    std = 1.0 / math.sqrt(w.H)
    for i in range(count):
        g = _gen(out.device, seed_of(w, S_WEIGHT, i))
        out[i].copy_((torch.randn(w.E, w.H, generator=g, device=out.device) * std).to(torch.bfloat16))
    return out


def decode_ids(w: Workload, T: int, steps, device="cpu") -> torch.Tensor:
    """[len(steps), T, k] int32 expert ids for decode steps, drawn as the k
    largest of bias_step[e] + N(0,1).  Continuous noise makes ties
    impossible in practice, so the ids of a row are distinct."""
    steps = list(steps)
    b = biases(w, max(steps) + 1)
    out = torch.empty(len(steps), T, w.k, dtype=torch.int32, device=device)
    for n, s in enumerate(steps):
        g = _gen(device, seed_of(w, S_DECODE, s) + 7919 * T)
        x = torch.randn(T, w.E, generator=g, device=device) + b[s].to(device)
        out[n].copy_(torch.topk(x, w.k, dim=1).indices.to(torch.int32))
    return out


def bf16_bits(t: torch.Tensor):
    """uint16 numpy view of a bf16 tensor's bit patterns (host copy)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
