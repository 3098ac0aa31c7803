"""Seeded synthetic inputs for the block-wise FP8 linear layer.

This module only draws random numbers with the shapes, value distributions and
structure of the workloads; it contains none of the quantization or GEMM
arithmetic.  It is the one module that both the CPU oracle's tests and the
CUDA path's tests and benchmark import.

Shapes are those of the Llama-3.1-8B and Qwen3-30B-A3B linear layers named by
the article "NVIDIA NeMo RL Achieves 48% Speedup With End-to-End FP8 Precision
Training" (sections "Technical breakthrough" and "Real-world performance
gains"); no weights of those models are used, only their shapes.

Recipe (every tensor has its own seed derived from a base seed):
  activations  X ~ N(0, 1) in bf16, with a seeded set of K-channels (columns)
               multiplied by 20 (4 channels for the single-linear case, 1% of
               K for the Llama-shaped cases: 41 of 4096, 143 of 14336);
  weights      W ~ N(0, 0.02) in bf16;
  weight step  W <- bf16(W + 1e-3 * n * |W|), n ~ N(0, 1) (stands in for one
               optimizer update before a recalibration);
  MoE routing  expert popularity p_i ~ i^-1.1 over 128 experts (Zipf), each
               token picks 8 distinct experts by Gumbel-top-8 on log p; rows are
               sorted by expert and offsets[e] marks the first row of expert e.
"""
import torch

# Llama-3.1-8B projection shapes (N, K): out features, in features.
LLAMA8B_SHAPES = {
    "qkv": (6144, 4096),
    "o": (4096, 4096),
    "gate_up": (28672, 4096),
    "down": (4096, 14336),
}
LLAMA8B_LAYERS = 32
PREFILL_TOKENS = 8192          # 4 sequences x 2048 tokens
DECODE_TOKENS = (1, 16, 64, 256)

# Qwen3-30B-A3B expert shapes.
MOE_TOKENS = 4096
MOE_HIDDEN = 2048
MOE_INTER = 768
MOE_EXPERTS = 128
MOE_TOPK = 8
MOE_ZIPF_S = 1.1


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def outlier_channels(K, n, seed):
    """Seeded choice of n distinct columns (independent of the device)."""
    g = _gen(seed, "cpu")
    return torch.randperm(K, generator=g)[:n]


def n_outliers(K):
    """1% of the channels, rounded down (41 for K=4096, 143 for K=14336)."""
    return max(1, K // 100)


def activations(M, K, seed, n_out=None, device="cpu"):
    """X bf16 [M, K] ~ N(0,1) with n_out seeded columns scaled by 20."""
    n_out = n_outliers(K) if n_out is None else n_out
    g = _gen(seed, device)
    x = torch.randn((M, K), generator=g, device=device, dtype=torch.float32)
    if n_out > 0:
        cols = outlier_channels(K, n_out, seed + 7919).to(device)
        x[:, cols] *= 20.0
    return x.to(torch.bfloat16)


def weights(N, K, seed, device="cpu", std=0.02):
    """W bf16 [N, K] ~ N(0, std)."""
    g = _gen(seed, device)
    w = torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * std
    return w.to(torch.bfloat16)


def weight_step(w, seed, rel=1e-3):
    """W <- bf16(W + rel * n * |W|), n ~ N(0,1): a synthetic optimizer update."""
    g = _gen(seed, w.device)
    wf = w.float()
    n = torch.randn(wf.shape, generator=g, device=w.device, dtype=torch.float32)
    return (wf + rel * n * wf.abs()).to(torch.bfloat16)


def single_linear(seed=0, device="cpu"):
    """The single block-scaled linear: X [256, 512] (4 outlier channels), W [512, 512]."""
    x = activations(256, 512, seed, n_out=4, device=device)
    w = weights(512, 512, seed + 1, device=device)
    return x, w


def llama_layer(seed=0, M=PREFILL_TOKENS, device="cpu"):
    """Inputs of one Llama-8B-shaped layer's four linears at M tokens: {name: (X, W)}."""
    out = {}
    for i, (name, (N, K)) in enumerate(LLAMA8B_SHAPES.items()):
        out[name] = (activations(M, K, seed + 100 * i, device=device),
                     weights(N, K, seed + 100 * i + 1, device=device))
    return out


def layer_weight_seed(layer, name, seed=0):
    i = list(LLAMA8B_SHAPES).index(name)
    return seed + 1000 * (layer + 1) + 10 * i


def model_weights_after_step(layers=LLAMA8B_LAYERS, device="cpu"):
    """The recalibration workload: every layer's four Llama-8B-shaped weights,
    each after one synthetic update step.  Yields (layer, name, W bf16 [N, K])."""
    for layer in range(layers):
        for name, (N, K) in LLAMA8B_SHAPES.items():
            seed = layer_weight_seed(layer, name)
            yield layer, name, weight_step(weights(N, K, seed, device=device), seed + 1)


def zipf_probs(E=MOE_EXPERTS, s=MOE_ZIPF_S):
    r = torch.arange(1, E + 1, dtype=torch.float64)
    p = r.pow(-s)
    return p / p.sum()


def moe_routing(T=MOE_TOKENS, E=MOE_EXPERTS, topk=MOE_TOPK, s=MOE_ZIPF_S, seed=0):
    """Seeded top-k routing with Zipf expert popularity.

    Returns (token_of_row int64 [T*topk], expert_of_row int64 [T*topk],
    offsets int64 [E+1]) with rows sorted by expert (stable in token order).
    """
    g = _gen(seed, "cpu")
    logp = zipf_probs(E, s).log()
    u = torch.rand((T, E), generator=g, dtype=torch.float64).clamp_(1e-300, 1.0)
    gumbel = -torch.log(-torch.log(u))
    experts = torch.topk(logp[None, :] + gumbel, topk, dim=1).indices      # [T, topk]
    tok = torch.arange(T).repeat_interleave(topk)
    exp = experts.reshape(-1)
    order = torch.sort(exp * T + tok).indices                               # stable by (expert, token)
    exp_sorted = exp[order]
    tok_sorted = tok[order]
    counts = torch.bincount(exp_sorted, minlength=E)
    offsets = torch.zeros(E + 1, dtype=torch.int64)
    offsets[1:] = torch.cumsum(counts, 0)
    return tok_sorted, exp_sorted, offsets


def moe_layer(seed=0, T=MOE_TOKENS, H=MOE_HIDDEN, I=MOE_INTER, E=MOE_EXPERTS,
              topk=MOE_TOPK, device="cpu"):
    """Inputs of the MoE expert GEMMs: routed activations and per-expert weights.

    Returns dict with offsets [E+1], x_up bf16 [T*topk, H] (each token's row
    repeated for its experts), w_up bf16 [E, 2I, H], x_down bf16 [T*topk, I],
    w_down bf16 [E, H, I].
    """
    tok, _, offsets = moe_routing(T, E, topk, seed=seed)
    x = activations(T, H, seed + 11, n_out=0, device=device)
    x_up = x[tok.to(device)]
    x_down = activations(T * topk, I, seed + 12, n_out=0, device=device)
    w_up = weights(E * 2 * I, H, seed + 13, device=device).reshape(E, 2 * I, H)
    w_down = weights(E * H, I, seed + 14, device=device).reshape(E, H, I)
    return {"offsets": offsets, "x_up": x_up, "w_up": w_up, "x_down": x_down, "w_down": w_down}


def gemm_flops(M, N, K):
    return 2.0 * M * N * K


def ceil_div(a, b):
    return -(-a // b)

