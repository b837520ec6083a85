"""Seeded synthetic inputs shaped like DeepSeek-V3 layers.

This module is the only code shared by the oracle side (tests, CPU
baseline) and the CUDA side (tests, bench).  It draws random tensors and
routings and holds none of the method's arithmetic: no amax, no scale, no
E4M3 rounding, no GEMM.

Recipe (every tensor has its own seed, ``seed_for(config, tensor)``):
  * entries are ``torch.randn`` draws from a ``torch.Generator`` seeded with
    that seed on the target device, times the stated standard deviation;
    bf16 tensors are the fp32 draw rounded to bf16 (round to nearest even);
  * "p outliers x f": an independent Bernoulli(p) mask (own seed) and the
    masked entries multiplied by f;
  * "p set to +-v": a Bernoulli(p) mask and a fair sign (own seeds), the
    masked entries replaced by +v or -v;
  * MoE routing: every token picks ``topk`` distinct experts uniformly at
    random (the first ``topk`` of a seeded random permutation per token);
    routed rows are sorted by expert, ties in token order.

The six workloads follow the DeepSeek-V3 shapes the FP8 scheme is used on
(hidden 7168, FFN 18432, 256 experts with top-8 routing, expert dims
2048 / 4096).
"""
from dataclasses import dataclass, field

import torch

BASE_SEED = 0xF8F80000


def seed_for(config_id: int, tensor_id: int) -> int:
    return BASE_SEED + 16 * config_id + tensor_id


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shape, std, seed, device="cpu", dtype=torch.bfloat16):
    """N(0, std^2) entries, drawn in fp32 and rounded to ``dtype``."""
    x = torch.randn(tuple(shape), generator=_gen(device, seed), device=device,
                    dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def scale_outliers(x, p, factor, seed):
    """Multiply a Bernoulli(p) subset of entries by ``factor`` (in place)."""
    u = torch.rand(x.shape, generator=_gen(x.device, seed), device=x.device)
    mask = u < p
    x[mask] = (x[mask].float() * factor).to(x.dtype)
    return x


def set_outliers(x, p, value, seed_mask, seed_sign):
    """Replace a Bernoulli(p) subset of entries by +-value, fair sign (in place)."""
    u = torch.rand(x.shape, generator=_gen(x.device, seed_mask), device=x.device)
    sgn = torch.rand(x.shape, generator=_gen(x.device, seed_sign), device=x.device)
    mask = u < p
    vals = torch.where(sgn < 0.5, -value, value).to(x.dtype)
    x[mask] = vals[mask]
    return x


def moe_routing(tokens, experts, topk, seed, device="cpu"):
    """Uniform top-k routing.

    Returns (token_of_row int64 [tokens*topk], offsets int32 [experts+1]):
    row r of the expert-sorted activation matrix is token ``token_of_row[r]``;
    expert g owns rows [offsets[g], offsets[g+1]).
    """
    g = _gen(device, seed)
    keys = torch.rand((tokens, experts), generator=g, device=device)
    choice = keys.argsort(dim=1)[:, :topk]                    # distinct experts
    expert_of = choice.reshape(-1)
    token_of = torch.arange(tokens, device=device).repeat_interleave(topk)
    order = torch.argsort(expert_of * tokens + token_of)      # by expert, then token
    counts = torch.bincount(expert_of, minlength=experts)
    offsets = torch.zeros(experts + 1, dtype=torch.int64, device=device)
    offsets[1:] = torch.cumsum(counts, 0)
    return token_of[order].contiguous(), offsets.to(torch.int32)


def moe_dispatch_dest(token_of_row, tokens, topk):
    """The routing of ``moe_routing`` in token order: dest int32 [tokens,
    topk] with dest[t, j] the j-th expert-sorted row (in row order) that
    holds token t, the inverse of ``token_of_row``.  Index bookkeeping only."""
    R = token_of_row.numel()
    rows = torch.arange(R, device=token_of_row.device)
    perm = torch.argsort(token_of_row.long() * R + rows)      # by token, then row
    return perm.to(torch.int32).view(tokens, topk).contiguous()


@dataclass
class Workload:
    name: str
    config_id: int
    desc: str
    shapes: dict = field(default_factory=dict)


# The six workloads (names are used by tests and by bench.py).
TINY = Workload("tiny_e2e_128x256x256", 0,
                "A fp32 [128x256], B fp32 [256x256], N(0,1) with 1% set to +-50; "
                "1x128 act quant, 128x128 weight quant, block-scaled GEMM -> fp32 C",
                dict(M=128, K=256, N=256))
QUANT = Workload("quant_bw_act8192x7168_w7168x18432", 1,
                 "act bf16 [8192x7168] and weight bf16 [7168x18432], N(0,0.02), "
                 "0.1% outliers x100", dict(M=8192, K=7168, N=18432))
FFN = Workload("ffn_up_fwd_4096x18432x7168", 2,
               "X bf16 [4096x7168] N(0,1) 0.1% outliers x100, W bf16 [7168x18432] "
               "N(0,0.02); online quant of both, block-scaled GEMM -> bf16 [4096x18432]",
               dict(M=4096, K=7168, N=18432))
MOE = Workload("moe_grouped_8192tok_top8_256exp", 3,
               "8192 tokens x top-8 of 256 experts, gate+up W [7168x4096] and down W "
               "[2048x7168] per expert, bf16 N(0,0.02); grouped GEMM over ragged M",
               dict(tokens=8192, experts=256, topk=8, hidden=7168, inter=2048))
DGRAD = Workload("dgrad_16384x7168x18432", 4,
                 "dY bf16 [16384x18432] N(0,1e-3) 0.1% outliers x100, W [7168x18432] "
                 "N(0,0.02); dX = dY W^T -> bf16 [16384x7168]",
                 dict(M=16384, K=18432, N=7168))

WGRAD = Workload("wgrad_7168x18432_over_16384tok", 5,
                 "X bf16 [16384x7168] N(0,1) 0.1% outliers x100, dY bf16 [16384x18432] "
                 "N(0,1e-3) 0.1% outliers x100; dW = X^T dY -> fp32 [7168x18432], both "
                 "operands 1x128 along the 16384 tokens",
                 dict(M=16384, K=7168, N=18432))

WORKLOADS = {w.name: w for w in (TINY, QUANT, FFN, MOE, DGRAD, WGRAD)}


def tiny_inputs(device="cpu"):
    """A fp32 [128,256], B fp32 [256,256]: N(0,1), 1% set to +-50."""
    c = TINY.config_id
    a = normal((128, 256), 1.0, seed_for(c, 0), device, torch.float32)
    set_outliers(a, 0.01, 50.0, seed_for(c, 1), seed_for(c, 2))
    b = normal((256, 256), 1.0, seed_for(c, 3), device, torch.float32)
    set_outliers(b, 0.01, 50.0, seed_for(c, 4), seed_for(c, 5))
    return a, b


def act_input(M, K, std, outlier_p, outlier_factor, config_id, device="cpu",
              dtype=torch.bfloat16, tensor_id=0):
    x = normal((M, K), std, seed_for(config_id, tensor_id), device, dtype)
    if outlier_p > 0:
        scale_outliers(x, outlier_p, outlier_factor, seed_for(config_id, tensor_id + 1))
    return x


def weight_input(K, N, std, config_id, device="cpu", dtype=torch.bfloat16, tensor_id=8):
    return normal((K, N), std, seed_for(config_id, tensor_id), device, dtype)


def quant_inputs(device="cpu"):
    c = QUANT.config_id
    x = act_input(8192, 7168, 0.02, 1e-3, 100.0, c, device)
    w = normal((7168, 18432), 0.02, seed_for(c, 8), device)
    scale_outliers(w, 1e-3, 100.0, seed_for(c, 9))
    return x, w


def ffn_inputs(device="cpu", M=4096, K=7168, N=18432):
    c = FFN.config_id
    x = act_input(M, K, 1.0, 1e-3, 100.0, c, device)
    w = weight_input(K, N, 0.02, c, device)
    return x, w


def dgrad_inputs(device="cpu", M=16384, K=18432, N=7168):
    """dY [M, K] (K = forward N, the contraction here) and W [N, K] (forward [K_fwd, N_fwd])."""
    c = DGRAD.config_id
    dy = act_input(M, K, 1e-3, 1e-3, 100.0, c, device)
    w = weight_input(N, K, 0.02, c, device)
    return dy, w


def wgrad_inputs(device="cpu", M=16384, K=7168, N=18432):
    """X [M, K] (the layer input) and dY [M, N] (its output gradient); the
    weight gradient contracts over the M tokens."""
    c = WGRAD.config_id
    x = act_input(M, K, 1.0, 1e-3, 100.0, c, device)
    dy = act_input(M, N, 1e-3, 1e-3, 100.0, c, device, tensor_id=2)
    return x, dy


def moe_inputs(device="cpu", tokens=8192, experts=256, topk=8, hidden=7168, inter=2048,
               with_weights=True):
    """Routed activations and expert weights for the MoE grouped GEMMs.

    Returns dict with: x bf16 [tokens, hidden] (the tokens), x_routed bf16
    [tokens*topk, hidden] (x[token_of]: rows sorted by expert), token_of int64
    [tokens*topk], offsets int32 [experts+1], h_down bf16 [tokens*topk, inter]
    (input of the down projection, N(0,1)), and when ``with_weights``:
    w_gate_up bf16 [experts, hidden, 2*inter], w_down bf16 [experts, inter, hidden]
    (built expert by expert with ``moe_expert_weight``).
    """
    c = MOE.config_id
    x = act_input(tokens, hidden, 1.0, 1e-3, 100.0, c, device)
    token_of, offsets = moe_routing(tokens, experts, topk, seed_for(c, 2), device)
    out = dict(x=x, x_routed=x[token_of].contiguous(), offsets=offsets, token_of=token_of)
    out["h_down"] = normal((tokens * topk, inter), 1.0, seed_for(c, 3), device)
    if with_weights:
        out["w_gate_up"] = torch.stack([moe_expert_weight(e, "gate_up", device, hidden, inter)
                                        for e in range(experts)])
        out["w_down"] = torch.stack([moe_expert_weight(e, "down", device, hidden, inter)
                                     for e in range(experts)])
    return out


def moe_expert_weight(e, which, device="cpu", hidden=7168, inter=2048):
    """Expert e's weight, bf16 N(0, 0.02): "gate_up" [hidden, 2*inter] (gate
    and up projections side by side along N) or "down" [inter, hidden]."""
    c = MOE.config_id
    if which == "gate_up":
        shape, tid = (hidden, 2 * inter), 8
    elif which == "down":
        shape, tid = (inter, hidden), 9
    else:
        raise ValueError(which)
    return normal(shape, 0.02, seed_for(c, tid) + (e + 1) * 1_000_003, device)
