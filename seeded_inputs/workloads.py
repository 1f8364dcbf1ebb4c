"""The synthetic optimizer-step workloads: parameter lists, simulated rank counts,
ZeRO stage, bucket size, input distributions and AdamW hyper-parameters.

Each full-size workload has a reduced twin of the same structure (same stage, same
rank count, ragged sizes, several buckets and shards, a padded tail) that the CPU
oracle finishes in seconds; those are the element-by-element parity cases.
"""
import math
from dataclasses import dataclass, replace

import numpy as np

from . import DEFAULT_SEED, STREAM_SIZES, extra_words


@dataclass(frozen=True)
class Workload:
    name: str
    description: str
    tensors: tuple            # element count of each parameter tensor, in list order
    units: tuple              # first tensor index of each stage-3 gather unit; () = one unit
    n_ranks: int              # simulated data-parallel ranks N
    stage: int                # 0 = DDP, 1/2/3 = ZeRO stage
    bucket_elems: int         # bucket size in elements; <= 0 means one bucket
    steps: int
    loss_scale: float
    grad_sigma: float = 1e-3
    master_sigma: float = 0.02
    m_sigma: float = 0.0      # warm first moment ~ N(0, m_sigma^2); 0 = zeros
    v_sigma: float = 0.0      # warm second moment ~ |N(0, v_sigma^2)|; 0 = zeros
    heavy_frac: float = 0.0   # fraction of gradient entries multiplied by heavy_mult
    heavy_mult: float = 1.0
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.01
    pad_align: int = 128
    seed: int = DEFAULT_SEED

    @property
    def psi(self):
        return int(sum(self.tensors))

    def with_(self, **kw):
        return replace(self, **kw)


# ------------------------------------------------------------ parameter lists

def gpt2_tensors(vocab=50257, ctx=1024, d=768, layers=12):
    """GPT-2 parameter list: wte, wpe, per block [ln_1 w,b; c_attn w,b; attn c_proj w,b;
    ln_2 w,b; c_fc w,b; mlp c_proj w,b], final ln w,b.  Gather units: embeddings, each
    block, final norm."""
    t = [vocab * d, ctx * d]
    units = [0]
    for _ in range(layers):
        units.append(len(t))
        t += [d, d, d * 3 * d, 3 * d, d * d, d, d, d, d * 4 * d, 4 * d, 4 * d * d, d]
    units.append(len(t))
    t += [d, d]
    return tuple(t), tuple(units)


def llama_tensors(vocab=32000, d=3072, ffn=8192, layers=26):
    """Llama-style list with tied embeddings: embedding, per layer [attn RMSNorm, wq, wk,
    wv, wo, ffn RMSNorm, w_gate, w_up, w_down], final RMSNorm.  Gather units: embedding,
    each layer, final norm."""
    t = [vocab * d]
    units = [0]
    for _ in range(layers):
        units.append(len(t))
        t += [d, d * d, d * d, d * d, d * d, d, ffn * d, ffn * d, d * ffn]
    units.append(len(t))
    t += [d]
    return tuple(t), tuple(units)


def ragged_sizes(count=2000, max_size=4_000_000, seed=DEFAULT_SEED):
    """Log-uniform sizes in [1, max_size]: floor(exp(u * ln(max_size))), u uniform on
    [0, 1) from the top 24 bits of the SIZES stream's per-index word."""
    words = extra_words(count, seed, STREAM_SIZES)
    u = (words >> np.uint32(8)).astype(np.float64) / float(1 << 24)
    lnmax = math.log(max_size)
    return tuple(max(1, int(math.floor(math.exp(float(x) * lnmax)))) for x in u)


# ------------------------------------------------------------ full-size workloads

def _gpt2_small():
    t, u = gpt2_tensors()
    return Workload(
        name="gpt2_small_n8_zero2",
        description="GPT-2-small parameter list (148 tensors, psi=124,439,808), N=8, "
                    "25M-element buckets, ZeRO-2, fp16 grads N(0,1e-3)*1024, 5 AdamW steps",
        tensors=t, units=u, n_ranks=8, stage=2, bucket_elems=25_000_000, steps=5,
        loss_scale=1024.0)


def _llama_3b():
    t, u = llama_tensors()
    return Workload(
        name="llama3b_n8_zero3",
        description="Llama-shaped list (26 layers, hidden 3072, FFN 8192, vocab 32000, tied "
                    "embedding, psi=3,042,868,224), N=8, 50M-element buckets, ZeRO-3 with the "
                    "per-layer fp16 all-gather, 5 AdamW steps",
        tensors=t, units=u, n_ranks=8, stage=3, bucket_elems=50_000_000, steps=5,
        loss_scale=1024.0)


def _ragged():
    return Workload(
        name="ragged2000_n16_zero2",
        description="2000 tensors, sizes log-uniform in [1, 4M], N=16 (padded shards), "
                    "1M-element buckets, ZeRO-2, fp16 grads N(0,1e-3)*1024 with 1% of "
                    "entries x100, 20 AdamW steps",
        tensors=ragged_sizes(), units=(), n_ranks=16, stage=2, bucket_elems=1_000_000,
        steps=20, loss_scale=1024.0, heavy_frac=0.01, heavy_mult=100.0)


def full_workloads():
    """The five workloads, smallest first.  Building the ragged list calls the host
    generator, so this is a function rather than a module constant."""
    return {
        "ring3_psi1m_zero1": Workload(
            name="ring3_psi1m_zero1",
            description="psi=2^20 flat, N=3 simulated ranks (the 3-GPU ring example), one "
                        "bucket, ZeRO-1, fp16 grads fp16(1024*N(0,1e-3)), 3 AdamW steps",
            tensors=(1 << 20,), units=(), n_ranks=3, stage=1, bucket_elems=0, steps=3,
            loss_scale=1024.0),
        "gpt2_small_n8_zero2": _gpt2_small(),
        "flat1p3b_n4_zero1": Workload(
            name="flat1p3b_n4_zero1",
            description="psi=1.3e9 flat, N=4, 50M-element buckets, ZeRO-1, warm state "
                        "m~N(0,1e-4) v=|N(0,1e-6)|, fp16 grads N(0,1e-3)*4096, 10 AdamW steps",
            tensors=(1_300_000_000,), units=(), n_ranks=4, stage=1, bucket_elems=50_000_000,
            steps=10, loss_scale=4096.0, m_sigma=1e-4, v_sigma=1e-6),
        "llama3b_n8_zero3": _llama_3b(),
        "ragged2000_n16_zero2": _ragged(),
    }


def reduced_workloads():
    """Same structure at sizes the oracle finishes in seconds (full element-wise parity)."""
    full = full_workloads()
    t_gpt, u_gpt = gpt2_tensors(vocab=503, ctx=64, d=64, layers=2)
    t_ll, u_ll = llama_tensors(vocab=1000, d=96, ffn=256, layers=3)
    return {
        "ring3_psi1m_zero1": full["ring3_psi1m_zero1"],
        "gpt2_small_n8_zero2": full["gpt2_small_n8_zero2"].with_(
            name="gpt2_tiny_n8_zero2", tensors=t_gpt, units=u_gpt, bucket_elems=25_013,
            description="GPT-2 list at d=64, 2 blocks, vocab 503"),
        "flat1p3b_n4_zero1": full["flat1p3b_n4_zero1"].with_(
            name="flat3m_n4_zero1", tensors=(3_000_017,), bucket_elems=500_003, steps=4,
            description="flat psi=3,000,017, N=4, 500,003-element buckets, warm state"),
        "llama3b_n8_zero3": full["llama3b_n8_zero3"].with_(
            name="llama_tiny_n8_zero3", tensors=t_ll, units=u_ll, bucket_elems=50_000, steps=3,
            description="Llama list at d=96, FFN 256, 3 layers, vocab 1000"),
        "ragged2000_n16_zero2": full["ragged2000_n16_zero2"].with_(
            name="ragged200_n16_zero2", tensors=ragged_sizes(200, 40_000), bucket_elems=10_007,
            steps=4, description="200 tensors log-uniform in [1, 40000], N=16, heavy tails"),
    }
