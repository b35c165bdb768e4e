"""Named workload shapes and their algorithmic FLOP counts.

Shapes are those of the pages' fine-tuning runs: batch 4 x seq 2048 tokens
and Llama-7B d=4096 / h=11008 ([Mistral blog] benchmark configuration and
"10、11. 手动 Autograd"), Mistral-7B h=14336 with GQA k/v projections to 1024
and Gemma-7B d=3072 / h=24576 at batch 2 x seq 8192 ([Gemma blog], VRAM
section and table).  LoRA rank 16, alpha 16 throughout ([Mistral blog]
benchmark configuration).
"""

LINEAR_WORKLOADS = {
    "tiny_linear": dict(M=256, K=512, N=1024, r=16, alpha=16.0, seed=0),
    "llama7b_q_proj": dict(M=8192, K=4096, N=4096, r=16, alpha=16.0, seed=0),
    "mistral7b_k_proj": dict(M=8192, K=4096, N=1024, r=16, alpha=16.0, seed=1),
    "mistral7b_v_proj": dict(M=8192, K=4096, N=1024, r=16, alpha=16.0, seed=2),
    "gemma7b_q_proj": dict(M=16384, K=3072, N=4096, r=16, alpha=16.0, seed=1),
}

# nq / nkv: the same models' attention projection widths (q, and each of k and v;
# Mistral's grouped-query k/v are 1024 wide), for the fused Q/K/V projection.
MLP_WORKLOADS = {
    "llama7b_swiglu_mlp": dict(M=8192, d=4096, h=11008, r=16, alpha=16.0, act="swiglu", seed=0, nq=4096, nkv=4096),
    "mistral7b_swiglu_mlp": dict(M=8192, d=4096, h=14336, r=16, alpha=16.0, act="swiglu", seed=0, nq=4096,
                                 nkv=1024),
    "gemma7b_geglu_mlp": dict(M=16384, d=3072, h=24576, r=16, alpha=16.0, act="geglu_tanh", seed=0, nq=4096,
                              nkv=4096),
}


def linear_flops(M, K, N, r):
    """Algorithmic FLOP of one QLoRA linear forward + backward (no dW).

    Dense: forward 2MKN + dX 2MKN.  LoRA: forward 2Mr(K+N), backward
    4Mr(K+N) (G = dY B^T, dB, dA and the G A^T term; X A is reused).
    Dequantisation counts as no FLOP.
    """
    return 4 * M * K * N + 6 * M * r * (K + N)


def mlp_flops(M, d, h, r):
    """Algorithmic FLOP of the gated MLP forward + backward (three linears)."""
    return 2 * linear_flops(M, d, h, r) + linear_flops(M, h, d, r)
