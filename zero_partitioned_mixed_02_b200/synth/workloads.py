"""The synthetic workloads: shapes, value distributions, hyper-parameters.

Input recipes only (no optimizer arithmetic). Each gradient element of virtual
rank r at step s is drawn from key(seed, STREAM_GRAD, s, r) at its flat index;
initial master weights from key(seed, STREAM_MASTER, 0, 0) at the flat index.
So every rank view (full, or one partition) sees the same virtual job.
"""
from __future__ import annotations

from dataclasses import dataclass, field

from . import Dist, normal, normal_tiny, signed_mag, uniform


def gpt2_tensors(n_layer=48, d=1600, vocab=50257, ctx=1024):
    """GPT-2 1.5B parameter list, tied head: wte, wpe, 48 blocks, ln_f.
    Layer units for a stage-3 gather: embeddings = 0, block i = i + 1, ln_f = last."""
    t = [(vocab * d, 0), (ctx * d, 0)]
    for i in range(n_layer):
        u = i + 1
        t += [(d, u), (d, u),                    # ln_1 weight, bias
              (d * 3 * d, u), (3 * d, u),        # c_attn weight, bias
              (d * d, u), (d, u),                # attn c_proj weight, bias
              (d, u), (d, u),                    # ln_2 weight, bias
              (d * 4 * d, u), (4 * d, u),        # c_fc weight, bias
              (4 * d * d, u), (d, u)]            # mlp c_proj weight, bias
    t += [(d, n_layer + 1), (d, n_layer + 1)]    # ln_f weight, bias
    return t


def llama_tensors(n_layer=32, d=2560, ffn=6912, vocab=32000):
    """Llama-shaped ~2.7B list, untied embeddings, RMSNorm, SwiGLU.
    Units: embedding = 0, block i = i + 1, final norm + lm_head = last."""
    t = [(vocab * d, 0)]
    for i in range(n_layer):
        u = i + 1
        t += [(d, u),                                        # attention_norm
              (d * d, u), (d * d, u), (d * d, u), (d * d, u),  # wq, wk, wv, wo
              (d, u),                                        # ffn_norm
              (ffn * d, u), (ffn * d, u), (d * ffn, u)]      # w1 (gate), w3 (up), w2 (down)
    t += [(d, n_layer + 1), (vocab * d, n_layer + 1)]        # norm, lm_head
    return t


@dataclass
class Workload:
    name: str
    psi: int
    nd: int
    stage: int
    steps: int
    loss_scale: float
    grad: Dist
    master: Dist
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.0
    rank_view: int = -1
    tensors: list | None = None
    # (step index, rank, flat index, fp16 bits) written over the generated gradient
    inject: list = field(default_factory=list)
    seed: int = 0

    @property
    def hyper(self):
        return dict(lr=self.lr, beta1=self.beta1, beta2=self.beta2, eps=self.eps,
                    weight_decay=self.weight_decay)


def flat_1m() -> Workload:
    return Workload("flat-1M-nd4-stage2", psi=1_048_576, nd=4, stage=2, steps=3,
                    loss_scale=1024.0, grad=normal(1e-3, 1024.0), master=uniform(-0.1, 0.1))


def stress_16m() -> Workload:
    # |master| ~ U(1, 10) with random sign, so an Adam step of ~lr = 1e-3 is at
    # most |w|/2048 for |w| >= 2.048 (swamped in fp16); 10% of the unscaled
    # per-rank gradients have magnitude in [2^-26, 2^-24) (below fp16's 2^-24);
    # loss scale 65536; the second step carries one +inf on rank 3.
    return Workload("stress-16M-nd8-stage1", psi=16_777_216, nd=8, stage=1, steps=3,
                    loss_scale=65536.0,
                    grad=normal_tiny(1e-4, 0.10, 2.0**-26, 2.0**-24, 65536.0),
                    master=signed_mag(1.0, 10.0), inject=[(1, 3, 0, 0x7C00)])


def gpt2_1p5b() -> Workload:
    t = gpt2_tensors()
    return Workload("gpt2-1.5B-nd8-stage2", psi=sum(n for n, _ in t), nd=8, stage=2, steps=5,
                    loss_scale=4096.0, grad=normal(1e-3, 4096.0), master=uniform(-0.1, 0.1),
                    weight_decay=0.01, tensors=t)


def running_example_7p5b() -> Workload:
    return Workload("7.5B-nd64-rank0-view-stage1", psi=7_500_000_000, nd=64, stage=1, steps=5,
                    loss_scale=1024.0, grad=normal(1e-3, 1024.0), master=uniform(-0.1, 0.1),
                    rank_view=0)


def llama_2p7b() -> Workload:
    t = llama_tensors()
    return Workload("llama-2.7B-nd8-stage3", psi=sum(n for n, _ in t), nd=8, stage=3, steps=3,
                    loss_scale=1024.0, grad=normal(1e-3, 1024.0), master=uniform(-0.1, 0.1),
                    tensors=t)


ALL = {1: flat_1m, 2: stress_16m, 3: gpt2_1p5b, 4: running_example_7p5b, 5: llama_2p7b}


# Small cases of the large workloads' kernels for profiler captures: inputs
# well above the 126 MB L2, a few GB on the device in all.
def flat_64m() -> Workload:
    """The GPT-2 workload's stage-2 step at psi = 2^26 (one tensor, same value
    distributions and Nd): about 3.6 GB on the device, 3.8 GB moved per step,
    so the lines still dirty in L2 when a kernel ends are ~1-2 % of its bytes."""
    return Workload("flat-64M-nd8-stage2", psi=1 << 26, nd=8, stage=2, steps=5,
                    loss_scale=4096.0, grad=normal(1e-3, 4096.0), master=uniform(-0.1, 0.1),
                    weight_decay=0.01)


def llama_block() -> Workload:
    """One block of the Llama-shaped 2.7B list (d = 2560, ffn 6912: 79.3M
    parameters, 158.6 MB of fp16) between a 1024-row embedding (unit 0) and the
    final norm + a 1024-row head (unit 2), Nd = 8, stage 3: the block's layer
    gather has the full model's tensor and chunk shapes; about 3.7 GB on the
    device."""
    d, ffn = 2560, 6912
    t = [(1024 * d, 0)]
    t += [(d, 1), (d * d, 1), (d * d, 1), (d * d, 1), (d * d, 1), (d, 1), (ffn * d, 1), (ffn * d, 1), (d * ffn, 1)]
    t += [(d, 2), (1024 * d, 2)]
    return Workload("llama-block-nd8-stage3", psi=sum(n for n, _ in t), nd=8, stage=3, steps=3,
                    loss_scale=1024.0, grad=normal(1e-3, 1024.0), master=uniform(-0.1, 0.1),
                    tensors=t)


def view_1g() -> Workload:
    """The 7.5B running example's single-rank view at psi = 2^30, Nd = 64:
    partition 0 of 16,777,216 parameters (64 gradient slices of it, 2.1 GB;
    the fp16 buffer of psi, 2.1 GB; 0.4 GB of state), 2.6 GB moved per step."""
    return Workload("view-1G-nd64-rank0-view-stage1", psi=1 << 30, nd=64, stage=1, steps=5,
                    loss_scale=1024.0, grad=normal(1e-3, 1024.0), master=uniform(-0.1, 0.1),
                    rank_view=0)


PROFILE = {"flat-64m": flat_64m, "llama-block": llama_block, "view-1g": view_1g}
